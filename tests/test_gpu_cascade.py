"""GPU parity of the cascade decode over shared prefixes (pa_decode_cascade) through the C ABI, against the
oracle's float64 attention over the whole context: the prefix-shared workload at every block size, ragged
groups (sizes past one 64-row tile, prefix lengths from 0 up, empty suffixes) at every group size, head_dim
and dtype, shared against copied prefix blocks (bit-identical), and workspace reuse."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from tests.gpu_common import assert_close, gpu_step, oracle_step
from workloads import make_prefix_groups, make_workload

pytestmark = pytest.mark.gpu

pa = pytest.importorskip("paged_kv_cache_330_b200")


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    assert pa.device_error() == 0, "a kernel recorded a device-side error"


def _groups(sizes, plens, B):
    gs = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    assert gs[-1] == B
    spl = np.repeat(np.asarray(plens, dtype=np.int32), sizes)
    return gs, spl


def _cascade(wl, sizes, plens, bt=None, kc=None, vc=None, num_partitions=0, workspace=None):
    out_plain, kc0, vc0, bt0, lens, bt_h, lens_h = gpu_step(wl)
    kc = kc0 if kc is None else kc
    vc = vc0 if vc is None else vc
    bt = bt0 if bt is None else bt
    gs, spl = _groups(sizes, plens, wl.batch)
    out = pa.decode_cascade(wl.q.cuda(), kc, vc, bt, lens, int(lens_h.max()), wl.scale, torch.from_numpy(gs).cuda(),
                            torch.from_numpy(spl).cuda(), max(sizes), max(plens), num_partitions=num_partitions,
                            workspace=workspace)
    torch.cuda.synchronize()
    return out, out_plain, (kc0, vc0, bt0, lens, bt_h, lens_h)


def _sample_rows(wl, n, seed):
    rng = np.random.default_rng(seed)
    B, Hq = wl.batch, wl.cfg["num_q_heads"]
    rows = {(0, 0), (B - 1, Hq - 1), (int(np.argmax(wl.context_lens)), Hq // 2)}
    while len(rows) < n:
        rows.add((int(rng.integers(B)), int(rng.integers(Hq))))
    return sorted(rows)


def test_cascade_prefix_sweep_bs16_all_rows():
    wl = make_workload("prefix_sweep")
    out, plain, _ = _cascade(wl, [32] * 8, [2048] * 8)
    okc, ovc, rows, lens, _ = oracle_step(wl)
    ref = oatt.decode_attention(wl.q, okc, ovc, rows, lens, wl.scale)
    assert_close(out.float().cpu().numpy(), ref, "cascade prefix_sweep bs16")
    assert_close(plain.float().cpu().numpy(), ref, "plain prefix_sweep bs16")


@pytest.mark.parametrize("bs", [32, 64, 128, 256])
def test_cascade_prefix_sweep_sampled(bs):
    wl = make_workload("prefix_sweep", block_size=bs)
    out, _, _ = _cascade(wl, [32] * 8, [2048] * 8)
    rows = _sample_rows(wl, 48, bs)
    okc, ovc, orows, lens, _ = oracle_step(wl)
    ref = oatt.decode_rows(wl.q, okc, ovc, orows, lens, wl.scale, rows)
    got = np.stack([out[b, h].float().cpu().numpy() for b, h in rows])
    assert_close(got, ref, f"cascade prefix_sweep bs{bs}")


CASES = [  # group sizes, prefix lengths
    ([1, 3, 40, 2, 70], [16, 0, 512, 2048, 160]),
    ([5, 1, 1, 9], [1024, 0, 48, 256]),
]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 4), (8, 2), (16, 2), (16, 1)])
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_cascade_ragged_groups(D, Hq, Hkv, dtype):
    for ci, (sizes, plens) in enumerate(CASES):
        bs = (16, 64)[ci % 2]
        wl = make_prefix_groups(seed=7 * Hq + D + ci, group_sizes=sizes, prefix_lens=plens, suffix_lo=0,
                                suffix_hi=300, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D, block_size=bs,
                                dtype=dtype)
        okc, ovc, rows, lens, _ = oracle_step(wl)
        ref = oatt.decode_attention(wl.q, okc, ovc, rows, lens, wl.scale)
        for ns in (0, 7):
            out, _, _ = _cascade(wl, sizes, plens, num_partitions=ns)
            assert_close(out.float().cpu().numpy(), ref, f"cascade D{D} G{Hq // Hkv} {dtype} case{ci} part{ns}")


def test_cascade_shared_and_copied_prefix_blocks_bit_identical():
    """Members whose prefix entries point at private copies of the shared blocks (same bytes) get exactly the
    same output: the prefix is read through the group's first member."""
    sizes, plens = [6, 4], [512, 256]
    wl = make_prefix_groups(seed=3, group_sizes=sizes, prefix_lens=plens, suffix_lo=1, suffix_hi=90, num_q_heads=8,
                            num_kv_heads=2, head_dim=128, block_size=16)
    out, _, (kc, vc, bt, lens, bt_h, lens_h) = _cascade(wl, sizes, plens)
    NB = kc.shape[0]
    extra = sum((n - 1) * (P // 16) for n, P in zip(sizes, plens))
    kc2 = torch.cat([kc, torch.zeros((extra,) + tuple(kc.shape[1:]), dtype=kc.dtype, device=kc.device)])
    vc2 = torch.cat([vc, torch.zeros_like(kc2[NB:])])
    bt2 = bt_h.copy()
    nxt, first = NB, 0
    for n, P in zip(sizes, plens):
        for m in range(first + 1, first + n):
            for j in range(P // 16):
                kc2[nxt] = kc[bt_h[first, j]]
                vc2[nxt] = vc[bt_h[first, j]]
                bt2[m, j] = nxt
                nxt += 1
        first += n
    out2, _, _ = _cascade(wl, sizes, plens, bt=torch.from_numpy(bt2).cuda(), kc=kc2, vc=vc2)
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


def test_cascade_workspace_reuse_and_split_counters():
    """Counters return to zero: one workspace serves repeated calls with identical results."""
    wl = make_workload("prefix_sweep", block_size=64)
    B, Hq, Hkv, D = wl.batch, 16, 8, 128
    need = pa.decode_cascade_workspace_size(B, Hq, Hkv, D, int(wl.context_lens.max()), 8, 32, 2048)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    outs = [_cascade(wl, [32] * 8, [2048] * 8, workspace=ws)[0] for _ in range(3)]
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
