"""GPU parity: pa_prefill_chunk (causal chunked prefill over the paged cache, tcgen05/TMEM) against the oracle."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from tests.gpu_common import assert_close, gpu_step, oracle_step
from workloads import make_custom, make_workload

pytestmark = pytest.mark.gpu

pa = pytest.importorskip("paged_kv_cache_330_b200")


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    assert pa.device_error() == 0, "a kernel recorded a device-side error"


def gpu_prefill(wl, device="cuda"):
    """pa_write_kv of the chunk (C++ pool slots), then pa_prefill_chunk."""
    _, kc, vc, bt_d, lens_d, bt, lens = gpu_step(wl)
    qsl = torch.from_numpy(wl.query_start_loc).to(device)
    C = np.diff(wl.query_start_loc)
    out = pa.prefill_chunk(wl.q.to(device), qsl, kc, vc, bt_d, lens_d, int(C.max()), wl.scale)
    return out, kc, vc, bt_d, lens_d, bt, lens


def oracle_prefill(wl, seqs=None, heads=None):
    okc, ovc, rows, lens, _ = oracle_step(wl)
    return oatt.prefill_attention(wl.q, wl.query_start_loc, okc, ovc, rows, lens, wl.scale, seqs=seqs, heads=heads)


def _compare(out, ref, wl, what):
    qsl = wl.query_start_loc
    for (b, h), r in ref.items():
        got = out[qsl[b]:qsl[b + 1], h].float().cpu().numpy()
        assert_close(got, r, f"{what} seq{b} head{h}")


def test_prefill_small_no_prefix():
    """The chunk is the whole sequence (query i sees keys 0..i), one 128-row tile plus a ragged one."""
    wl = make_custom(seed=11, lens=[200], chunk_lens=[200], kind="prefill", num_q_heads=4, num_kv_heads=2,
                     head_dim=128, block_size=16)
    out, *_ = gpu_prefill(wl)
    _compare(out, oracle_prefill(wl), wl, "no prefix")


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 4), (8, 2), (8, 1), (16, 1)])
@pytest.mark.parametrize("bs", [16, 64, 256])
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_prefill_ragged(Hq, Hkv, bs, dtype):
    """Several sequences with ragged prefixes and chunks (tiles that straddle the causal diagonal,
    partial key tiles, chunks that are not multiples of 128)."""
    lens = [1, 17, 130, 300, 700]
    chunks = [1, 5, 129, 128, 250]
    wl = make_custom(seed=Hq * 31 + Hkv * 7 + bs, lens=lens, chunk_lens=chunks, kind="prefill", num_q_heads=Hq,
                     num_kv_heads=Hkv, head_dim=128, block_size=bs, dtype=dtype)
    out, *_ = gpu_prefill(wl)
    _compare(out, oracle_prefill(wl), wl, f"ragged G{Hq // Hkv} bs{bs} {dtype}")


def test_prefill_large_logits():
    wl = make_custom(seed=5, lens=[400, 260], chunk_lens=[150, 260], kind="prefill", num_q_heads=8, num_kv_heads=2,
                     head_dim=128, block_size=16, q_scale=10.0)
    out, *_ = gpu_prefill(wl)
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    _compare(out, oracle_prefill(wl), wl, "q x10")


def test_prefill_full_workload_sampled():
    """8 sequences x 512-token chunk on an 8192-token context, 32/8 heads: sampled (sequence, head) pairs,
    every query row of each."""
    wl = make_workload("prefill")
    out, *_ = gpu_prefill(wl)
    pairs = [(0, 0), (3, 13), (7, 31), (5, 6)]
    for b, h in pairs:
        ref = oracle_prefill(wl, seqs=[b], heads=[h])
        _compare(out, ref, wl, "prefill workload")


def test_prefill_row_equals_decode():
    """Prefill row i equals a decode of the first prefix+i+1 tokens (same cache, same kernels' inputs)."""
    P, Cn = 333, 140
    wl = make_custom(seed=9, lens=[P + Cn], chunk_lens=[Cn], kind="prefill", num_q_heads=8, num_kv_heads=2,
                     head_dim=128, block_size=16)
    out, kc, vc, bt_d, lens_d, bt, lens = gpu_prefill(wl)
    rows = [0, 1, 63, 127, 128, 139]
    q = wl.q[rows].cuda()
    ctx = torch.tensor([P + i + 1 for i in rows], dtype=torch.int32, device="cuda")
    btr = bt_d.expand(len(rows), -1).contiguous()
    dec = pa.decode(q, kc, vc, btr, ctx, int(ctx.max()), wl.scale)
    diff = (dec.float() - out[rows].float()).abs().max().item()
    assert diff < 2e-2, diff


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (16, 8)])
@pytest.mark.parametrize("bs", [32, 128])
def test_prefill_pair_edges(Hq, Hkv, bs):
    """CTA-pair edges: with one head per KV group a pair covers two consecutive 128-row tiles, so a
    300-token chunk has three tiles and the second pair holds one tile past the chunk's end; chunks of
    1, 127, 128 and 129 rows sit on tile boundaries; block sizes 32 and 128."""
    lens = [300, 900, 129, 128, 60, 1]
    chunks = [300, 299, 129, 127, 60, 1]
    wl = make_custom(seed=bs + Hq, lens=lens, chunk_lens=chunks, kind="prefill", num_q_heads=Hq, num_kv_heads=Hkv,
                     head_dim=128, block_size=bs)
    out, *_ = gpu_prefill(wl)
    _compare(out, oracle_prefill(wl), wl, f"pair edges G{Hq // Hkv} bs{bs}")


def test_prefill_mixed_prefix_lengths():
    """Sequences with and without earlier context in one batch: a chunk that is the whole sequence next to
    chunks appended after long contexts (key tiles fully visible, diagonal tiles, fully masked tiles)."""
    wl = make_custom(seed=23, lens=[128, 2048, 700, 4097], chunk_lens=[128, 64, 700, 257], kind="prefill",
                     num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16, dtype="f16")
    out, *_ = gpu_prefill(wl)
    _compare(out, oracle_prefill(wl), wl, "mixed prefixes f16")
