"""The multi-rank path of bench.py on the CPU: two gloo ranks (independent replicas) combine their
timings (max over ranks) and their work (sum over ranks) the way the GPU run does over NCCL."""

from __future__ import annotations

import importlib.util
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    spec = importlib.util.spec_from_file_location("_bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    bench = _load_bench()
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        # rank r: step 1.0 + r ms, e2e 2.0 + 3r ms; it moved (r + 1) GB of KV for 64 (r + 1) sequences
        times, totals = bench.reduce_over_ranks([1.0 + rank, 2.0 + 3 * rank], [(rank + 1) * 1e9, 64 * (rank + 1)],
                                                world, torch.device("cpu"))
        q.put((rank, times, totals))
    finally:
        dist.destroy_process_group()


def test_reduce_over_ranks_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0, f"rank process exited with {p.exitcode}"
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, times, totals in got:
        assert times == [2.0, 5.0]            # the slowest rank's times, on every rank
        assert totals == [3e9, 192.0]         # every rank's work
    # the aggregate the bench reports: all ranks' bytes over the slowest rank's time
    times, totals = got[0][1], got[0][2]
    assert totals[0] / (times[0] * 1e-3) / 1e9 == pytest.approx(1500.0)


def test_reduce_over_ranks_single_process_is_identity():
    bench = _load_bench()
    times, totals = bench.reduce_over_ranks([1.5, 2.5], [10, 20], 1, torch.device("cpu"))
    assert times == [1.5, 2.5] and totals == [10.0, 20.0]


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    """Under torchrun the reference arm (the oracle) is timed by rank 0 alone; other ranks exit 0."""
    bench = _load_bench()
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")

    class Args:
        workload = "tiny"
        ref_seqs = 4
        ref_budget = 0.1
        steps = 1
        warmup = 0
        gpus = 2

    assert bench.run_reference(Args()) == 0
    assert capsys.readouterr().out == ""


@pytest.mark.parametrize("workload,metric_attr,unit", [("tiny", "METRIC", "GB/s"), ("prefill", "PREFILL_METRIC", "TFLOP/s"),
                                                        ("rope_write", "ROPE_METRIC", "GB/s")])
def test_reference_arm_times_the_matching_oracle(monkeypatch, capsys, workload, metric_attr, unit):
    """`--impl reference` times the oracle of the same workload, on the metric and unit of our arm's line."""
    import json
    bench = _load_bench()
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)

    class Args:
        ref_seqs = 4
        ref_budget = 0.2
        steps = 1
        warmup = 0
        gpus = 1

    Args.workload = workload
    assert bench.run_reference(Args()) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == getattr(bench, metric_attr) and line["unit"] == unit
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["unit"] == unit
    assert line["e2e"] == {"value": line["value"], "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_staged_inputs_pack_and_views(monkeypatch):
    """The end-to-end loop's staging buffer: every input at a 256-byte offset of one buffer, one copy of
    `nbytes` moves all of them, and the typed device views read back each input unchanged (CPU stand-in for
    pinned and device memory)."""
    bench = _load_bench()
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    g = torch.Generator().manual_seed(11)
    host = dict(q=torch.randn(3, 4, 128, generator=g).to(torch.bfloat16), sm=torch.arange(5, dtype=torch.int64),
                bt=torch.randint(0, 9, (3, 7), dtype=torch.int32, generator=g), empty=torch.zeros(0, dtype=torch.int32),
                lens=torch.tensor([1, 2, 3], dtype=torch.int32))
    st = bench.StagedInputs(host, "cpu")
    ends = []
    for name, t in host.items():
        v = st.views[1][name]
        assert v.dtype == t.dtype and v.shape == t.shape
        if t.numel():
            off = v.data_ptr() - st.d[1].data_ptr()
            assert off % 256 == 0
            ends.append(off + t.numel() * t.element_size())
    assert st.nbytes == max(ends)
    st.d[1][:st.nbytes].copy_(st.h[:st.nbytes])
    for name, t in host.items():
        assert torch.equal(st.views[1][name], t), name
