#!/usr/bin/env python
"""Benchmark: paged decode KV GB/s (and decode tokens/s) at batch 128, Qwen3-0.6B-shaped heads.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step = the whole decode hot path over one batch: pa_write_kv of each
sequence's new token into its slot, then pa_decode (one kernel: block-table
gather, attention, split-K merge) over every sequence's paged context.  Each
call is captured once in a CUDA graph and replayed, so the timed loop measures
the GPU rather than Python launch overhead.  Inputs are resident in
HBM; the KV working set (~295 MB) is larger than the 126 MB L2, so no flush is
needed between steps.  Timed with CUDA events on the launching stream,
bracketed by barrier + synchronize, max over ranks.  N > 1 runs independent
data-parallel replicas (each rank its own batch of sequences and its own
pool; no collective on the data path), so the scaling is weak.

`--impl reference` times the CPU oracle (oracle/) on the host cores on
bounded samples of the same workload; it is the deliberately slow baseline.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode KV GB/s (% of HBM peak) and decode tokens/s at batch 128"
UNIT = "GB/s"
PREFILL_METRIC = "chunked prefill TFLOP/s (bf16, causal, paged context)"
ROPE_METRIC = "rotary embedding + KV cache write GB/s (% of HBM peak)"
FALLBACK_HBM_GBS = 6650.0

WORKLOAD_TEXT = {
    "qwen_decode": "Qwen3-0.6B-shaped decode: batch 128, 16 q / 8 kv heads (GQA 2), head_dim 128, bf16, block_size 16, "
                   "context_lens uniform[100,1024], blocks shuffled over a pool of total context + 10% free",
    "llama70b_long": "Llama-2-70B-shaped long decode: batch 64, 64 q / 8 kv heads (GQA 8), head_dim 128, bf16, "
                     "block_size 16, context_lens uniform[4096,8192]",
    "prefix_sweep": "prefix-shared decode: batch 256 = 8 groups x 32 sharing a 2048-token prefix, suffix uniform[0,512], "
                    "16 q / 8 kv heads, head_dim 128, bf16",
    "tiny": "tiny decode: 4 seqs, 4/4 heads, head_dim 64, fp16, block_size 16",
    "prefill": "chunked prefill: 8 seqs, each a 512-token causal chunk appended to an 8192-token paged context, "
               "32 q / 8 kv heads, head_dim 128, bf16, block_size 16",
    "pool_host": "host block pool of the Qwen3-0.6B-shaped decode batch (128 sequences, block_size 16): per step, one "
                 "batched append of a token to every sequence and the block-table export (CPU only)",
    "rope_write": "rotary embedding + KV cache write of the chunked-prefill step's 4096 new tokens (8 seqs x 512 at "
                  "positions 8192..8703), 32 q / 8 kv heads, head_dim 128, bf16, block_size 16, fp32 cos/sin "
                  "tables of 16384 positions; before every timed launch L2 is flushed by a 512 MB write followed by a 512 MB "
                  "read of another buffer (the launch starts on a cold L2 that holds no dirty lines)",
}

# DRAM bytes (read + write) per launch of the workload's dominant kernel from one ncu capture,
# valid only for the kernel source it was taken on (sha256 prefix of the listed csrc files).
DECODE_SRC = ("decode.cu", "common.cuh")
PREFILL_SRC = ("prefill.cu", "common.cuh")
ROPE_SRC = ("rope_write_kv.cu", "common.cuh")
CASCADE_SRC = ("decode.cu", "prefill.cu", "common.cuh")  # suffix decode + prefill kernel in shared-prefix mode
NCU_TRAFFIC = {
    "qwen_decode": {"bytes": 313_004_032, "src": "95dca1d0ca960523", "files": DECODE_SRC},
    "qwen_decode_int8": {"bytes": 164_869_376, "src": "95dca1d0ca960523", "files": DECODE_SRC},
    "llama70b_long_int8": {"bytes": 844_040_448, "src": "95dca1d0ca960523", "files": DECODE_SRC},
    # both kernels of one cascade call at block size 16 (suffix decode + shared-prefix pass)
    "prefix_sweep_cascade": {"bytes": 351_881_984, "src": "f86ad8eda4abdac4", "files": CASCADE_SRC},
    "llama70b_long": {"bytes": 1_584_821_760, "src": "95dca1d0ca960523", "files": DECODE_SRC},
    "prefill": {"bytes": 347_949_824, "src": "168c732c524f5c1a", "files": PREFILL_SRC},
    "rope_write": {"bytes": 55_998_208, "src": "e527154b96c52f4d", "files": ROPE_SRC},
}


def kernel_source_hash(files=DECODE_SRC) -> str:
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "paged_kv_cache_330_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_bf16_peak():
    """(burst, sustained) dense bf16 TFLOP/s measured on this machine, or the fallback figure."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            d = json.load(fh)
        return float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return 1590.0, 1400.0, "fallback"


def prefill_flops(wl) -> float:
    """4*D flops per visible (query, key) pair: query i of a C-token chunk on L tokens sees L-C+i+1 keys."""
    c = wl.cfg
    tot = 0
    for b in range(wl.batch):
        C = int(wl.query_start_loc[b + 1] - wl.query_start_loc[b])
        L = int(wl.context_lens[b])
        tot += C * (L - C) + C * (C + 1) // 2
    return float(tot) * c["num_q_heads"] * 4 * c["head_dim"]


def measured_hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------------------------------------ clocks
class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML (read-only) while a region runs."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.mem_samples, self.power_w = [], []
        self.period = period_s
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def sample(self):
        """One reading (SM and memory clock, power, active reasons); a no-op without NVML."""
        nv = self._nv
        if nv is None:
            return
        try:
            self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
            self.mem_samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_MEM))
            self.power_w.append(nv.nvmlDeviceGetPowerUsage(self._h) / 1000.0)
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            for bit, name in self.REASONS.items():
                if r & bit and name != "gpu_idle":
                    self.reasons.add(name)
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self.sample()
            time.sleep(self.period)

    def __enter__(self):
        if self._nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        med = lambda v: statistics.median(v) if v else None
        return {"sm_mhz": med(self.samples), "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples), "mem_mhz": med(self.mem_samples),
                "power_w_median": med(self.power_w), "power_w_max": max(self.power_w) if self.power_w else None}


# ------------------------------------------------------------------------------------------------ helpers
def kv_bytes(wl) -> int:
    """Algorithmic bytes of one decode: every context token's K and V row of every KV head, read once."""
    c = wl.cfg
    return int(wl.context_lens.astype(np.int64).sum()) * c["num_kv_heads"] * c["head_dim"] * 2 * 2


def unique_kv_bytes(wl) -> int:
    """For shared prefixes, bytes of distinct cache rows read (each shared block counted once)."""
    c = wl.cfg
    if c["kind"] != "prefix":
        return kv_bytes(wl)
    toks = c["groups"] * c["prefix_len"] + int((wl.context_lens - c["prefix_len"]).sum())
    return toks * c["num_kv_heads"] * c["head_dim"] * 2 * 2


def io_bytes(wl) -> int:
    """q read + out written + block tables + context lengths, per decode call."""
    c = wl.cfg
    qo = wl.batch * c["num_q_heads"] * c["head_dim"] * 2 * 2
    bt = int(sum(-(-int(L) // c["block_size"]) for L in wl.context_lens)) * 4
    return qo + bt + wl.batch * 4


def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# ------------------------------------------------------------------------------------------------ reference arm
def oracle_step_cpu(wl, n_seqs=None):
    """One oracle pass (pool replay, byte write, fp64 decode) over the first n_seqs sequences."""
    import oracle
    from oracle import attention as oatt
    import torch
    pool, rows, lens, slots, _ = oracle.replay(wl.ops, wl.num_blocks, wl.cfg["block_size"], wl.free_order, wl.batch)
    kc = wl.k_cache0.view(torch.int16).numpy().view(np.uint16).copy()
    vc = wl.v_cache0.view(torch.int16).numpy().view(np.uint16).copy()
    oracle.write_kv(wl.k_new.view(torch.int16).numpy().view(np.uint16), wl.v_new.view(torch.int16).numpy().view(np.uint16),
                    slots, kc, vc)
    n = wl.batch if n_seqs is None else n_seqs
    dt = wl.k_cache0.dtype
    kt = torch.from_numpy(kc.view(np.int16)).view(dt)
    vt = torch.from_numpy(vc.view(np.int16)).view(dt)
    return oatt.decode_attention(wl.q[:n], kt, vt, rows[:n], lens[:n], wl.scale)


def time_oracle(wl, budget_s: float, n_seqs: int):
    """Repeat the oracle step on the first n_seqs sequences until budget_s of CPU time; returns (GB/s, desc, threads)."""
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        threads = 1
    c = wl.cfg
    bytes_per = int(wl.context_lens[:n_seqs].astype(np.int64).sum()) * c["num_kv_heads"] * c["head_dim"] * 4
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle_step_cpu(wl, n_seqs)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    gbs = bytes_per * reps / el / 1e9
    desc = (f"oracle (numpy fp64, pool replay + byte write + decode) on the first {n_seqs} of {wl.batch} sequences "
            f"of {wl.name}, {reps} repetitions in {el:.1f} s; GB/s counts those sequences' KV bytes")
    return gbs, desc, threads, el / reps


def _oracle_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return 1


def time_oracle_prefill(wl, budget_s: float):
    """Oracle chunked prefill (pool replay, byte write of the chunk, fp64 causal attention) over
    (sequence, head) pairs in order until budget_s; returns (TFLOP/s, desc, threads, seconds of the sample)."""
    import oracle
    from oracle import attention as oatt
    import torch
    t0 = time.perf_counter()
    _, rows, lens, slots, _ = oracle.replay(wl.ops, wl.num_blocks, wl.cfg["block_size"], wl.free_order, wl.batch)
    kc = wl.k_cache0.view(torch.int16).numpy().view(np.uint16).copy()
    vc = wl.v_cache0.view(torch.int16).numpy().view(np.uint16).copy()
    oracle.write_kv(wl.k_new.view(torch.int16).numpy().view(np.uint16),
                    wl.v_new.view(torch.int16).numpy().view(np.uint16), slots, kc, vc)
    dt = wl.k_cache0.dtype
    kt, vt = torch.from_numpy(kc.view(np.int16)).view(dt), torch.from_numpy(vc.view(np.int16)).view(dt)
    D, Hq = wl.cfg["head_dim"], wl.cfg["num_q_heads"]
    flops, pairs = 0.0, 0
    for b in range(wl.batch):
        C = int(wl.query_start_loc[b + 1] - wl.query_start_loc[b])
        L = int(wl.context_lens[b])
        for h in range(Hq):
            oatt.prefill_attention(wl.q, wl.query_start_loc, kt, vt, rows, lens, wl.scale, seqs=[b], heads=[h])
            flops += (C * (L - C) + C * (C + 1) // 2) * 4.0 * D
            pairs += 1
            if time.perf_counter() - t0 >= budget_s:
                break
        if time.perf_counter() - t0 >= budget_s:
            break
    el = time.perf_counter() - t0
    desc = (f"oracle (numpy fp64: pool replay, byte write of the chunk, causal attention) on the first {pairs} of "
            f"{wl.batch * Hq} (sequence, head) pairs of {wl.name} in {el:.1f} s; TFLOP/s counts those pairs' flops")
    return flops / el / 1e12, desc, _oracle_threads(), el


def time_oracle_rope(wl, budget_s: float):
    """Oracle rotary + cache write of the prefill step's new tokens, repeated until budget_s; returns
    (GB/s of the same algorithmic bytes as the GPU line, desc, threads, seconds per step)."""
    import oracle
    from oracle import rope as orope
    from workloads import new_token_positions, rope_tables
    import torch
    c = wl.cfg
    pos = new_token_positions(wl)
    cos, sin = rope_tables(16384, c["head_dim"])
    _, _, _, slots, _ = oracle.replay(wl.ops, wl.num_blocks, c["block_size"], wl.free_order, wl.batch)
    vcb = wl.v_cache0.view(torch.int16).numpy().view(np.uint16).copy()
    vb = wl.v_new.view(torch.int16).numpy().view(np.uint16)
    qd, kd = wl.q.double().numpy(), wl.k_new.double().numpy()
    nbytes = rope_bytes(int(pos.shape[0]), c["num_q_heads"], c["num_kv_heads"], c["head_dim"], len(np.unique(pos)))
    reps, t0 = 0, time.perf_counter()
    while True:
        orope.rope_write_kv(qd, kd, vb, pos, cos.numpy(), sin.numpy(), slots, vcb)
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    el = time.perf_counter() - t0
    desc = (f"oracle (numpy fp64 rotation + byte write of V) on the whole {pos.shape[0]}-token step, {reps} "
            f"repetitions in {el:.1f} s; GB/s counts the same algorithmic bytes")
    return nbytes * reps / el / 1e9, desc, _oracle_threads(), el / reps


def run_reference(args):
    ws, rank, _ = dist_setup()
    if rank != 0:
        return 0
    from workloads import make_workload
    wname = "prefill" if args.workload == "rope_write" else args.workload
    wl = make_workload(wname, block_size=getattr(args, "block_size", None))
    metric, unit, sample = METRIC, UNIT, {}
    if args.workload == "prefill":
        metric, unit = PREFILL_METRIC, "TFLOP/s"
        sample_fn = lambda: time_oracle_prefill(wl, args.ref_budget)
    elif args.workload == "rope_write":
        metric = ROPE_METRIC
        sample_fn = lambda: time_oracle_rope(wl, args.ref_budget)
    else:
        n = min(wl.batch, args.ref_seqs)
        sample = {"sample_seqs": n}
        sample_fn = lambda: time_oracle(wl, args.ref_budget, n)
    step_times = []
    vals = []
    desc = threads = None
    for i in range(args.warmup + args.steps):
        v, desc, threads, per = sample_fn()
        if i >= args.warmup:
            step_times.append(per)
            vals.append(v)
    value = float(np.mean(vals))
    line = {
        "impl": "reference", "metric": metric, "value": value, "unit": unit, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * float(np.mean(step_times)), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT.get(args.workload, args.workload), **sample},
        "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


class StagedInputs:
    """One step's host inputs packed into ONE pinned buffer (each tensor at a 256-byte boundary) and two
    device copies of it with typed views, so that a step's inputs cross PCIe as a single copy and step k+1's
    copy can run while step k computes."""

    def __init__(self, host: dict, dev):
        import torch
        layout, off = {}, 0
        for name, t in host.items():
            t = t.contiguous()
            n = t.numel() * t.element_size()
            layout[name] = (off, n, t.dtype, tuple(t.shape), t)
            off = (off + n + 255) // 256 * 256
        self.nbytes = max(o + n for o, n, *_ in layout.values())  # bytes copied per step
        self.h = torch.empty(max(off, 256), dtype=torch.uint8).pin_memory()
        for o, n, _, _, t in layout.values():
            if n:
                self.h[o:o + n].copy_(t.reshape(-1).view(torch.uint8))
        self.d = [torch.empty(max(off, 256), dtype=torch.uint8, device=dev) for _ in range(2)]
        self.views = [{name: d[o:o + n].view(dt).view(shape) for name, (o, n, dt, shape, _) in layout.items()}
                      for d in self.d]


def pipelined_e2e(stage: StagedInputs, out_like, step, K: int, repeats: int, warmup: int, dev, barrier):
    """End-to-end steps as a serving loop issues them: per step one H2D copy of the packed inputs on a
    copy stream, the step's library calls on the compute stream, the D2H of its output on a second copy
    stream; inputs and outputs are double-buffered, so copies of neighbouring steps overlap the compute.
    Returns the median over `repeats` of the ms per step (device events, first copy to last copy back), the
    repeats, the bytes copied in and out per step, and the median host time per step spent issuing them.
    Copies go through the library's pa_copy_async on the copy streams (no torch stream switch per copy)."""
    import torch
    import paged_kv_cache_330_b200 as pa
    main = torch.cuda.current_stream(dev)
    cin, cout = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    outs = [torch.empty_like(out_like) for _ in range(2)]
    h_outs = [torch.empty(out_like.shape, dtype=out_like.dtype).pin_memory() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]    # compute of the slot's last step finished
    freed = [torch.cuda.Event() for _ in range(2)]   # the slot's output is back on the host
    landed = [torch.cuda.Event() for _ in range(2)]  # the slot's inputs are on the device
    nb = stage.nbytes
    h_in, d_in = stage.h[:nb], [d[:nb] for d in stage.d]

    def run(n):
        for k in range(n):
            i = k & 1
            cin.wait_event(done[i])                  # step k-2 no longer reads this input slot
            pa.copy_async(d_in[i], h_in, stream=cin)
            landed[i].record(cin)
            main.wait_event(landed[i])
            main.wait_event(freed[i])                # step k-2's output has left this output slot
            step(main, stage.views[i], outs[i])
            done[i].record(main)
            cout.wait_event(done[i])
            pa.copy_async(h_outs[i], outs[i], stream=cout)
            freed[i].record(cout)

    run(warmup)
    torch.cuda.synchronize(dev)
    ms, host = [], []
    for _ in range(repeats):
        barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(main)
        cin.wait_stream(main)
        cout.wait_stream(main)
        h0 = time.perf_counter()
        run(K)
        host.append((time.perf_counter() - h0) * 1e3 / K)
        main.wait_stream(cin)
        main.wait_stream(cout)
        e1.record(main)
        torch.cuda.synchronize(dev)
        ms.append(e0.elapsed_time(e1) / K)
    barrier()
    d2h = outs[0].numel() * outs[0].element_size()
    return float(statistics.median(ms)), ms, nb, d2h, float(statistics.median(host))


def reduce_over_ranks(times_ms, totals, world_size, device):
    """Max over ranks of each timed duration, sum over ranks of each count (bytes, sequences).

    The ranks are independent replicas, so the job takes its slowest rank's time and does every
    rank's work; every rank makes the same two collective calls in the same order."""
    import torch
    import torch.distributed as dist
    vals = torch.tensor([float(t) for t in times_ms], dtype=torch.float64, device=device)
    tot = torch.tensor([float(t) for t in totals], dtype=torch.float64, device=device)
    if world_size > 1:
        dist.all_reduce(vals, op=dist.ReduceOp.MAX)
        dist.all_reduce(tot, op=dist.ReduceOp.SUM)
    return vals.tolist(), tot.tolist()


# ------------------------------------------------------------------------------------------------ our arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    import paged_kv_cache_330_b200 as pa
    from workloads import make_workload

    ws, rank, local = dist_setup()
    if ws > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl = make_workload(args.workload, seed=None if rank == 0 else 1000 * rank + 1, block_size=args.block_size)
    c = wl.cfg
    int8 = args.kv == "int8"
    _, bt, lens, sm, _ = pa.replay_ops(wl.ops, wl.num_blocks, c["block_size"], wl.free_order, wl.batch)
    maxL = int(lens.max())
    B, Hq, Hkv, D = wl.batch, c["num_q_heads"], c["num_kv_heads"], c["head_dim"]
    plan = pa.decode_int8_plan if int8 else pa.decode_plan
    grid, maxp, wsb = plan(B, Hq, Hkv, D, maxL, args.num_partitions)

    # device-resident inputs
    NB, bs = wl.k_cache0.shape[0], c["block_size"]
    host = dict(q=wl.q, kn=wl.k_new, vn=wl.v_new, sm=torch.from_numpy(sm), bt=torch.from_numpy(bt),
                lens=torch.from_numpy(lens))  # one step's inputs, as the scheduler hands them over
    if args.cascade:
        if c["kind"] != "prefix":
            raise SystemExit("--cascade needs the prefix-shared workload")
        per = B // c["groups"]   # groups of consecutive sequences share a prefix
        host["gs"] = torch.arange(0, B + 1, per, dtype=torch.int32)
        host["sp"] = torch.full((B,), c["prefix_len"], dtype=torch.int32)
    base = {k: v.to(dev) for k, v in host.items()}
    q, kn, vn, smd, btd, lensd = (base[k] for k in ("q", "kn", "vn", "sm", "bt", "lens"))
    out = torch.empty_like(q)
    work = torch.zeros(max(wsb, 256), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    if int8:  # the pool's prior contents, quantised into a fresh INT8 cache by the library's own write
        kq = torch.zeros((NB, bs, Hkv, D), dtype=torch.int8, device=dev)
        vq = torch.zeros_like(kq)
        ksc = torch.zeros((NB, Hkv, bs), dtype=torch.float32, device=dev)
        vsc = torch.zeros_like(ksc)
        pa.write_kv_int8(wl.k_cache0.to(dev).view(NB * bs, Hkv, D), wl.v_cache0.to(dev).view(NB * bs, Hkv, D),
                         torch.arange(NB * bs, dtype=torch.int64, device=dev), kq, vq, ksc, vsc)

        def wr(st, x=base):
            pa.write_kv_int8(x["kn"], x["vn"], x["sm"], kq, vq, ksc, vsc, stream=st)

        def dec(st, x=base, o=out):
            pa.decode_int8(x["q"], kq, vq, ksc, vsc, x["bt"], x["lens"], maxL, wl.scale, out=o, workspace=work,
                           num_partitions=args.num_partitions, stream=st)
    elif args.cascade:  # shared prefixes read once for all sharers (groups of consecutive sequences)
        kc = wl.k_cache0.to(dev)
        vc = wl.v_cache0.to(dev)
        work = torch.zeros(pa.decode_cascade_workspace_size(B, Hq, Hkv, D, maxL, c["groups"], per, c["prefix_len"],
                                                            args.num_partitions), dtype=torch.uint8, device=dev)

        def wr(st, x=base):
            pa.write_kv(x["kn"], x["vn"], x["sm"], kc, vc, stream=st)

        def dec(st, x=base, o=out):
            pa.decode_cascade(x["q"], kc, vc, x["bt"], x["lens"], maxL, wl.scale, x["gs"], x["sp"], per, c["prefix_len"],
                              out=o, workspace=work, num_partitions=args.num_partitions, stream=st)
    else:
        kc = wl.k_cache0.to(dev)
        vc = wl.v_cache0.to(dev)

        def wr(st, x=base):
            pa.write_kv(x["kn"], x["vn"], x["sm"], kc, vc, stream=st)

        def dec(st, x=base, o=out):
            pa.decode(x["q"], kc, vc, x["bt"], x["lens"], maxL, wl.scale, out=o, workspace=work,
                      num_partitions=args.num_partitions, stream=st)

    def barrier():
        if ws > 1:
            dist.barrier()

    # eager warm-up (first calls set kernel attributes), then CUDA graphs of several whole steps so
    # the timed loop measures the GPU, not Python launch overhead
    for _ in range(args.warmup):
        wr(stream)
        dec(stream)
    torch.cuda.synchronize(dev)
    assert pa.device_error() == 0

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap_stream):
            fn()
        return g

    cap_stream = torch.cuda.Stream(dev)
    S = args.steps_per_graph
    K = args.steps
    if K % S:
        S = 1
    # one graph = S whole steps (write + decode each); a second graph = S decodes alone, for the
    # decode kernel's own average duration (the roofline denominator's time)
    g_steps = capture(lambda: [(wr(cap_stream), dec(cap_stream)) for _ in range(S)])
    g_decs = capture(lambda: [dec(cap_stream) for _ in range(S)])
    for _ in range(max(1, args.warmup // S)):
        g_steps.replay()
    torch.cuda.synchronize(dev)

    # The K-step loop is timed `repeats` times (each bracketed by barrier + synchronize); the median of the
    # repeats is reported.  Each repeat is followed by the decode kernel alone, same launch count.
    step_ms, dec_ms = [], []
    with ClockSampler(local) as clk:
        for _ in range(args.repeats):
            t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            d_start, d_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            barrier()
            torch.cuda.synchronize(dev)
            t_start.record(stream)
            for _ in range(K // S):
                g_steps.replay()
            t_end.record(stream)
            torch.cuda.synchronize(dev)
            barrier()
            d_start.record(stream)
            for _ in range(K // S):
                g_decs.replay()
            d_end.record(stream)
            torch.cuda.synchronize(dev)
            step_ms.append(t_start.elapsed_time(t_end) / K)
            dec_ms.append(d_start.elapsed_time(d_end) / K)
    ms_step = float(statistics.median(step_ms))
    assert pa.device_error() == 0

    # ---- end to end through the public API: pinned host inputs -> device, step, result -> host.
    # (a) pipelined, as a serving loop runs: one packed H2D copy per step on a copy stream, the binding
    #     calls (argument checks, ctypes, tensor-map encode, launches) on the compute stream, the D2H of
    #     the output on a second copy stream, inputs and outputs double-buffered.
    stage = StagedInputs(host, dev)
    e2e_ms, e2e_rep, h2d, d2h, e2e_host = pipelined_e2e(stage, out, lambda st, x, o: (wr(st, x), dec(st, x, o)), K,
                                              args.repeats, args.warmup, dev, barrier)
    # (b) sequential: every step copies its inputs in, runs, copies the output out, all on one stream
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    x0 = stage.views[0]

    def e2e_step(st):
        x0_bytes = stage.d[0][:stage.nbytes]
        x0_bytes.copy_(stage.h[:stage.nbytes], non_blocking=True)
        wr(st, x0)
        dec(st, x0)
        h_out.copy_(out, non_blocking=True)

    for _ in range(args.warmup):
        e2e_step(stream)
    torch.cuda.synchronize(dev)
    seq = []
    for _ in range(args.repeats):
        barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K):
            e2e_step(stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        seq.append(e0.elapsed_time(e1) / K)
    barrier()
    e2e_seq_ms = float(statistics.median(seq))
    # (c) the sequential steps captured once in a CUDA graph and replayed (host work paid once, at capture)
    g_e2e = capture(lambda: [e2e_step(cap_stream) for _ in range(S)])
    g_e2e.replay()
    torch.cuda.synchronize(dev)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K // S):
        g_e2e.replay()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_graph_ms = e0.elapsed_time(e1) / K
    assert pa.device_error() == 0
    del g_steps, g_decs, g_e2e

    # ---- max over ranks, totals.  With shared prefixes the metric counts distinct cache rows (each shared
    # block once); the logical bytes (every sequence's rows, shared ones again) are reported beside it.
    kvb = unique_kv_bytes(wl)
    kvb_logical = kv_bytes(wl)
    if int8:  # one byte per element plus one fp32 scale per (token, KV head) row, for K and for V
        kvb = kvb // (2 * D) * (D + 4)
        kvb_logical = kvb_logical // (2 * D) * (D + 4)
    (ms_step, e2e_ms, e2e_seq_ms, e2e_graph_ms, dec_avg), (kv_all, kvl_all, seqs_all) = reduce_over_ranks(
        [ms_step, e2e_ms, e2e_seq_ms, e2e_graph_ms, float(statistics.median(dec_ms))], [kvb, kvb_logical, B],
        ws, dev)
    value = kv_all / (ms_step * 1e-3) / 1e9
    e2e_value = kv_all / (e2e_ms * 1e-3) / 1e9

    peak, peak_kind = measured_hbm_peak()
    alg = kvb + io_bytes(wl)
    achieved = alg / (dec_avg * 1e-3) / 1e9
    tr = NCU_TRAFFIC.get(args.workload + ("_int8" if int8 else "") + ("_cascade" if args.cascade else ""))
    if tr and args.cascade and c["block_size"] != 16:
        tr = None  # captured at block size 16
    traffic = tr["bytes"] if tr and tr.get("src") == kernel_source_hash(tr["files"]) else None
    launches_per_step = 3 if args.cascade else 2  # write_kv, decode (split-K merge inside)[, shared-prefix pass]
    if rank == 0:
        cpu = None
        if ws == 1 and not args.no_cpu_baseline:
            gbs, desc, threads, _ = time_oracle(wl, args.ref_budget, min(wl.batch, args.ref_seqs))
            cpu = {"value": gbs, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc,
                   "host_cpus": os.cpu_count()}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": K, "warmup": args.warmup,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": str(c["dtype"]) + ("+int8 cache" if int8 else ""), "data": "synthetic",
            "config": {"workload": WORKLOAD_TEXT.get(args.workload, args.workload), "global_batch": int(seqs_all),
                       "kv_cache": "int8 codes + fp32 row scales" if int8 else str(c["dtype"]),
                       "decode": "cascade over shared prefixes" if args.cascade else "per-sequence",
                       "block_size": int(c["block_size"]),
                       "parallelism": f"dp{ws} (independent replicas)", "l2": "inputs larger than L2 (no flush)",
                       "decode_grid": grid, "repeats": args.repeats,
                       "ms_per_step_repeats": step_ms},
            "tokens_per_s": seqs_all / (ms_step * 1e-3),
            "pct_hbm_peak": {"of_measured": value / ws / peak if peak_kind == "measured" else None,
                             "of_nominal_8000": value / ws / 8000.0},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms, "ms_per_step_repeats": e2e_rep,
                    "host_issue_ms_per_step": e2e_host,
                    "how": "pipelined eager steps: per step one pinned H2D copy of the packed inputs (q, new "
                           "K/V, slots, block tables, lengths" + (", group starts, prefix lengths" if args.cascade
                                                                   else "") +
                           ") on a copy stream, the binding's write and decode calls (argument checks, ctypes, "
                           "tensor-map encode, launches) on the compute stream, D2H of out on a second copy "
                           "stream; inputs and outputs double-buffered; median of repeats",
                    "sequential": {"value": kv_all / (e2e_seq_ms * 1e-3) / 1e9, "ms_per_step": e2e_seq_ms,
                                   "how": "copy in, calls, copy out on one stream, step after step"},
                    "graph_replay": {"value": kv_all / (e2e_graph_ms * 1e-3) / 1e9, "ms_per_step": e2e_graph_ms,
                                     "how": "the sequential steps captured in a CUDA graph"}},
            "roofline": {"bound": "hbm", "kernel": ("pa_decode_int8" if int8 else
                                                    "pa_decode_cascade (suffix decode + shared-prefix pass)"
                                                    if args.cascade else "pa_decode") +
                         ("" if args.cascade else " (one kernel: gather, attention, split-K merge)"),
                         "achieved": achieved, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic, "algorithmic_bytes": alg,
                         "avg_launch_ms": dec_avg, "avg_launch_ms_repeats": dec_ms,
                         "timing": "decode-only graph replays, same launch count, right after each timed loop; "
                                   "median of repeats"},
            "gpu_launches": launches_per_step * K,
            "clocks": clk.summary(),
            "cpu_baseline": cpu,
        }
        if kvl_all != kv_all:
            line["logical_gbs"] = kvl_all / (ms_step * 1e-3) / 1e9
            line["config"]["kv_bytes"] = {"unique": int(kv_all), "logical": int(kvl_all)}
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.destroy_process_group()
    return 0


def run_prefill(args):
    """Chunked-prefill step: pa_write_kv of every chunk token, then pa_prefill_chunk (tcgen05)."""
    import torch
    import paged_kv_cache_330_b200 as pa
    from workloads import make_workload

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    wl = make_workload("prefill")
    c = wl.cfg
    _, bt, lens, sm, _ = pa.replay_ops(wl.ops, wl.num_blocks, c["block_size"], wl.free_order, wl.batch)
    kc, vc = wl.k_cache0.to(dev), wl.v_cache0.to(dev)
    host = dict(q=wl.q, kn=wl.k_new, vn=wl.v_new, sm=torch.from_numpy(sm), bt=torch.from_numpy(bt),
                lens=torch.from_numpy(lens), qsl=torch.from_numpy(wl.query_start_loc))
    base = {k: v.to(dev) for k, v in host.items()}
    Cmax = int(np.diff(wl.query_start_loc).max())
    out = torch.empty_like(base["q"])
    cs = torch.cuda.Stream(dev)
    stream = torch.cuda.current_stream(dev)
    wr = lambda st, x=base: pa.write_kv(x["kn"], x["vn"], x["sm"], kc, vc, stream=st)
    pf = lambda st, x=base, o=out: pa.prefill_chunk(x["q"], x["qsl"], kc, vc, x["bt"], x["lens"], Cmax, wl.scale,
                                                    out=o, stream=st)
    for _ in range(args.warmup):
        wr(stream)
        pf(stream)
    torch.cuda.synchronize(dev)
    assert pa.device_error() == 0

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cs):
            fn()
        return g

    g_step = capture(lambda: (wr(cs), pf(cs)))
    g_pf = capture(lambda: pf(cs))
    K = args.steps
    for _ in range(3):
        g_step.replay()
    torch.cuda.synchronize(dev)
    step_ms, pf_ms = [], []
    with ClockSampler(0) as clk:
        for _ in range(args.repeats):
            e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            torch.cuda.synchronize(dev)
            e[0].record(stream)
            for _ in range(K):
                g_step.replay()
            e[1].record(stream)
            e[2].record(stream)
            for _ in range(K):
                g_pf.replay()
            e[3].record(stream)
            torch.cuda.synchronize(dev)
            step_ms.append(e[0].elapsed_time(e[1]) / K)
            pf_ms.append(e[2].elapsed_time(e[3]) / K)
    assert pa.device_error() == 0
    ms_step = float(statistics.median(step_ms))
    ms_pf = float(statistics.median(pf_ms))
    # The same launches timed the way the burst bf16 peak is measured (single GEMMs with the GPU idle
    # between them): bursts of 10 launches (~7 ms), each after 0.2 s idle, so the clocks are those of a GPU
    # below its power limit; the clocks are read from the host while each burst runs.  The K-launch loops
    # above run for seconds at the power limit and stay the line's `frac`.
    burst_ms = []
    bclk = ClockSampler(0)
    for _ in range(9):
        time.sleep(0.2)
        e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        e[0].record(stream)
        for _ in range(10):
            g_pf.replay()
        e[1].record(stream)
        for _ in range(3):
            time.sleep(0.001)
            bclk.sample()
        torch.cuda.synchronize(dev)
        burst_ms.append(e[0].elapsed_time(e[1]) / 10)
    assert pa.device_error() == 0
    ms_burst = float(statistics.median(burst_ms))

    # ---- end to end through the public API: pinned host inputs -> device, step, result -> host
    # (a) pipelined: one packed H2D copy per step on a copy stream, the calls on the compute stream, the
    #     D2H of out on a second copy stream, double-buffered; (b) sequential on one stream; (c) (b) in a graph
    stage = StagedInputs(host, dev)
    e2e_ms, e2e_rep, h2d, d2h, e2e_host = pipelined_e2e(stage, out, lambda st, x, o: (wr(st, x), pf(st, x, o)), K,
                                              args.repeats, args.warmup, dev, lambda: None)
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    x0 = stage.views[0]

    def e2e_step(st):
        stage.d[0][:stage.nbytes].copy_(stage.h[:stage.nbytes], non_blocking=True)
        wr(st, x0)
        pf(st, x0)
        h_out.copy_(out, non_blocking=True)

    for _ in range(args.warmup):
        e2e_step(stream)
    torch.cuda.synchronize(dev)
    e4, e5 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e4.record(stream)
    for _ in range(K):
        e2e_step(stream)
    e5.record(stream)
    torch.cuda.synchronize(dev)
    e2e_seq_ms = e4.elapsed_time(e5) / K
    g_e2e = capture(lambda: e2e_step(cs))
    g_e2e.replay()
    torch.cuda.synchronize(dev)
    e4, e5 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e4.record(stream)
    for _ in range(K):
        g_e2e.replay()
    e5.record(stream)
    torch.cuda.synchronize(dev)
    e2e_graph_ms = e4.elapsed_time(e5) / K
    assert pa.device_error() == 0
    del g_step, g_pf, g_e2e
    fl = prefill_flops(wl)
    cpu = None
    if not args.no_cpu_baseline:
        v, desc, threads, _ = time_oracle_prefill(wl, 10.0)
        cpu = {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc}
    tr = NCU_TRAFFIC["prefill"]
    pf_traffic = tr["bytes"] if tr["src"] == kernel_source_hash(tr["files"]) else None
    burst, sustained, kind = measured_bf16_peak()
    line = {
        "metric": PREFILL_METRIC, "value": fl / (ms_step * 1e-3) / 1e12,
        "unit": "TFLOP/s", "n_gpus": 1, "steps": K, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": str(c["dtype"]),
        "data": "synthetic", "config": {"workload": WORKLOAD_TEXT["prefill"], "flops_per_step": fl,
                                        "repeats": args.repeats, "ms_per_step_repeats": step_ms},
        "roofline": {"bound": "tensor", "kernel": "pa_prefill_chunk (tcgen05/TMEM, TMA)",
                     "achieved": fl / (ms_pf * 1e-3) / 1e12, "peak": burst, "peak_kind": kind + " burst",
                     "unit": "TFLOP/s", "frac": fl / (ms_pf * 1e-3) / 1e12 / burst,
                     "frac_of_sustained": fl / (ms_pf * 1e-3) / 1e12 / sustained, "traffic": pf_traffic,
                     "avg_launch_ms": ms_pf, "avg_launch_ms_repeats": pf_ms,
                     "burst": {"achieved": fl / (ms_burst * 1e-3) / 1e12, "frac": fl / (ms_burst * 1e-3) / 1e12 / burst,
                               "avg_launch_ms": ms_burst, "avg_launch_ms_bursts": burst_ms,
                               "clocks": bclk.summary(),
                               "how": "9 bursts of 10 launches (CUDA events per burst), each after 0.2 s idle; "
                                      "median; against the burst peak, measured the same way"}},
        "e2e": {"value": fl / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "ms_per_step_repeats": e2e_rep,
                    "host_issue_ms_per_step": e2e_host,
                "how": "pipelined eager steps: one packed pinned H2D copy of q, new K/V, slots, block tables, "
                       "lengths and chunk starts on a copy stream, binding.write_kv + binding.prefill_chunk on "
                       "the compute stream, D2H of out on a second copy stream, double-buffered",
                "sequential": {"value": fl / (e2e_seq_ms * 1e-3) / 1e12, "ms_per_step": e2e_seq_ms},
                "graph_replay": {"value": fl / (e2e_graph_ms * 1e-3) / 1e12, "ms_per_step": e2e_graph_ms}},
        "cpu_baseline": cpu,
        "gpu_launches": 2 * K,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def rope_bytes(T, Hq, Hkv, D, distinct_positions) -> int:
    """Algorithmic bytes of one rotary + cache-write launch: q read and q_out written, k and v read and their
    cache rows written (16-bit), the int64 position and slot of every token, and one fp32 cos and sin row
    (D/2 entries each) per distinct position."""
    return T * (Hq * D * 2 * 2 + Hkv * D * 2 * 4 + 16) + distinct_positions * D * 4


def run_rope(args):
    """Rotary + KV write step (pa_rope_write_kv) on the chunked-prefill step's new tokens, L2 flushed between
    timed launches (its ~100 MB working set fits in L2).  The flush is a write of one buffer and a read of
    another: a write alone would leave L2 full of dirty lines whose write-back the timed launch would pay."""
    import torch
    import paged_kv_cache_330_b200 as pa
    from workloads import make_workload, new_token_positions, rope_tables

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    wl = make_workload("prefill")
    c = wl.cfg
    T, Hq, Hkv, D = int(wl.k_new.shape[0]), c["num_q_heads"], c["num_kv_heads"], c["head_dim"]
    _, bt, lens, sm, _ = pa.replay_ops(wl.ops, wl.num_blocks, c["block_size"], wl.free_order, wl.batch)
    pos_h = new_token_positions(wl)
    cos_h, sin_h = rope_tables(16384, D)
    kc, vc = wl.k_cache0.to(dev), wl.v_cache0.to(dev)
    host = dict(q=wl.q, kn=wl.k_new, vn=wl.v_new, sm=torch.from_numpy(sm), pos=torch.from_numpy(pos_h))
    base = {k: v.to(dev) for k, v in host.items()}
    cos, sin = cos_h.to(dev), sin_h.to(dev)
    q_out = torch.empty_like(base["q"])
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    scrub = torch.zeros(128 << 20, dtype=torch.float32, device=dev)
    cs = torch.cuda.Stream(dev)
    stream = torch.cuda.current_stream(dev)
    step = lambda st, x=base, o=q_out: pa.rope_write_kv(x["q"], x["kn"], x["vn"], x["pos"], cos, sin, x["sm"], kc, vc,
                                                        q_out=o, stream=st)
    for _ in range(max(3, args.warmup)):
        step(stream)
    torch.cuda.synchronize(dev)
    assert pa.device_error() == 0

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cs):
            fn()
        return g

    g_step = capture(lambda: step(cs))
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    with ClockSampler(0) as clk:
        for i in range(K):
            flush.fill_(i & 0xFF)          # evict q/k/v and the cache rows from L2 (not timed) ...
            scrub.sum()                    # ... and write the flush's dirty lines back before the launch
            ev[i][0].record(stream)
            step(stream)                   # eager: queued while the flush runs, so no launch gap is timed
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
    assert pa.device_error() == 0
    times = sorted(a.elapsed_time(b) for a, b in ev)
    ms = float(np.mean(times))
    nbytes = rope_bytes(T, Hq, Hkv, D, len(np.unique(pos_h)))
    gbs = nbytes / (ms * 1e-3) / 1e9

    # ---- end to end through the public API: pinned host q/k/v/positions/slots -> device, step, q_out -> host
    # (a) pipelined (one packed H2D copy per step on a copy stream, the call on the compute stream, D2H on a
    #     second copy stream, double-buffered); (b) the sequential step captured in a CUDA graph
    stage = StagedInputs(host, dev)
    e2e_ms, e2e_rep, h2d, d2h, e2e_host = pipelined_e2e(stage, q_out, lambda st, x, o: step(st, x, o), K, args.repeats,
                                              max(3, args.warmup), dev, lambda: None)
    h_out = torch.empty(q_out.shape, dtype=q_out.dtype).pin_memory()
    x0 = stage.views[0]

    def e2e_step(st):
        stage.d[0][:stage.nbytes].copy_(stage.h[:stage.nbytes], non_blocking=True)
        step(st, x0)
        h_out.copy_(q_out, non_blocking=True)

    for _ in range(3):
        e2e_step(stream)
    torch.cuda.synchronize(dev)
    g_e2e = capture(lambda: e2e_step(cs))
    g_e2e.replay()
    torch.cuda.synchronize(dev)
    e4, e5 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e4.record(stream)
    for _ in range(K):
        g_e2e.replay()
    e5.record(stream)
    torch.cuda.synchronize(dev)
    e2e_graph_ms = e4.elapsed_time(e5) / K
    assert pa.device_error() == 0
    del g_step, g_e2e

    cpu = None
    if not args.no_cpu_baseline:
        v, desc, threads, _ = time_oracle_rope(wl, 10.0)
        cpu = {"value": v, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": desc}
    tr = NCU_TRAFFIC.get("rope_write")
    traffic = tr["bytes"] if tr and tr["src"] == kernel_source_hash(tr["files"]) else None
    peak, kind = measured_hbm_peak()
    line = {
        "metric": ROPE_METRIC, "value": gbs, "unit": "GB/s",
        "n_gpus": 1, "steps": K, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": str(c["dtype"]), "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT["rope_write"], "bytes_per_step": nbytes, "l2": "flushed"},
        "roofline": {"bound": "hbm", "kernel": "pa_rope_write_kv", "achieved": gbs, "peak": peak,
                     "peak_kind": kind, "unit": "GB/s", "frac": gbs / peak, "traffic": traffic,
                     "avg_launch_ms": ms, "median_launch_ms": times[len(times) // 2],
                     "timing": "CUDA events around each eager launch, queued behind a 512 MB L2 flush"},
        "e2e": {"value": nbytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "ms_per_step_repeats": e2e_rep,
                    "host_issue_ms_per_step": e2e_host,
                "how": "pipelined eager binding.rope_write_kv calls, one packed pinned H2D copy and one D2H "
                       "per step on copy streams, double-buffered",
                "graph_replay": {"value": nbytes / (e2e_graph_ms * 1e-3) / 1e9, "ms_per_step": e2e_graph_ms,
                                 "how": "sequential copy in, call, copy out captured in a CUDA graph"}},
        "cpu_baseline": cpu,
        "gpu_launches": K,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def run_pool_host(args):
    """Host block pool cost per decode step (the block-allocation row, on the CPU): append one token to each of
    the batch's sequences with one native call, then export the block table; against one call per sequence
    and against the oracle's pool doing the same step."""
    import paged_kv_cache_330_b200 as pa
    from oracle.block_pool import replay as oreplay
    from workloads import make_workload

    wl = make_workload("qwen_decode")
    B, bs = wl.batch, wl.cfg["block_size"]
    steps, warm = max(1, args.steps), max(3, args.warmup)
    grow = -(-(steps + warm) // bs) + 1
    NB = wl.num_blocks + B * 2 * grow
    order = np.arange(NB, dtype=np.int32)
    ids = np.arange(B, dtype=np.int64)

    def timed(step_fn, n):
        t0 = time.perf_counter()
        for _ in range(n):
            step_fn()
        return (time.perf_counter() - t0) / n * 1e6

    pool, bt, _, _, _ = pa.replay_ops(wl.ops, NB, bs, order, B)
    mb = bt.shape[1] + 2 * grow

    def batched():
        pool.append_batch(ids, 1)
        pool.block_table(ids, mb)

    for _ in range(warm):
        batched()
    us_batched = timed(batched, steps)
    pool2, _, _, _, _ = pa.replay_ops(wl.ops, NB, bs, order, B)

    def per_seq():
        for b in range(B):
            pool2.append(b, 1)
        pool2.block_table(ids, mb)

    n_seq = min(steps, 200)
    us_per_seq = timed(per_seq, n_seq)
    opool, _, _, _, _ = oreplay(wl.ops, NB, bs, order, B)

    def oracle_step():
        for b in range(B):
            opool.append(b, 1)
        opool.block_table(list(range(B)), mb)

    n_or = min(steps, 200)
    us_oracle = timed(oracle_step, n_or)
    line = {
        "metric": "host block-pool us per decode step (batch 128)", "value": us_batched, "unit": "us",
        "n_gpus": 0, "steps": steps, "warmup": warm, "ms_per_step": us_batched / 1e3, "higher_is_better": False,
        "scaling": "none", "vs_baseline": None, "dtype": "int64", "data": "synthetic",
        "config": {"workload": WORKLOAD_TEXT["pool_host"], "one_call_per_sequence_us": us_per_seq},
        "cpu_baseline": {"value": us_oracle, "unit": "us", "cores": 1, "kind": "oracle",
                         "sample": f"the oracle's Python pool doing the same step {n_or} times"},
        "host": os.cpu_count(),
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="qwen_decode", choices=sorted(WORKLOAD_TEXT))
    ap.add_argument("--num-partitions", type=int, default=0, help="decode CTAs (0 = fill the GPU)")
    ap.add_argument("--steps-per-graph", type=int, default=10, help="whole steps captured per CUDA graph")
    ap.add_argument("--repeats", type=int, default=5, help="timed K-step loops; the median is reported")
    ap.add_argument("--block-size", type=int, default=None, help="override the workload's block size")
    ap.add_argument("--cascade", action="store_true",
                    help="prefix-shared workload: read each shared prefix once for all sharers (pa_decode_cascade)")
    ap.add_argument("--kv", choices=["bf16", "int8"], default="bf16",
                    help="decode workloads: the cache format (int8 = codes + fp32 row scales)")
    ap.add_argument("--ref-budget", type=float, default=12.0, help="seconds of oracle time per reference sample")
    ap.add_argument("--ref-seqs", type=int, default=128)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.impl == "reference":
        if args.steps * args.ref_budget > 120:
            args.ref_budget = max(1.0, 120.0 / max(1, args.steps + args.warmup))
        return run_reference(args)
    if args.workload == "prefill":
        return run_prefill(args)
    if args.workload == "rope_write":
        return run_rope(args)
    if args.workload == "pool_host":
        return run_pool_host(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
