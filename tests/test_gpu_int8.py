"""GPU parity of the INT8 KV cache through the C ABI: the quantising write (pa_write_kv_int8) and the block
copy (pa_copy_blocks_int8) bit for bit against the oracle's codes and scales, and decode over the INT8
cache (pa_decode_int8) within the attention tolerance of the oracle's float64 attention over the
dequantised cache."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from oracle import kv_quant as oq
from tests.gpu_common import assert_close, gpu_step_int8, oracle_step_int8
from workloads import make_custom, make_workload

pytestmark = pytest.mark.gpu

pa = pytest.importorskip("paged_kv_cache_330_b200")


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    assert pa.device_error() == 0, "a kernel recorded a device-side error"


def _sample_rows(wl, n, seed):
    rng = np.random.default_rng(seed)
    B, Hq = wl.batch, wl.cfg["num_q_heads"]
    rows = {(0, 0), (B - 1, Hq - 1), (int(np.argmax(wl.context_lens)), Hq // 2),
            (int(np.argmin(wl.context_lens)), 1 % Hq)}
    while len(rows) < n:
        rows.add((int(rng.integers(B)), int(rng.integers(Hq))))
    return sorted(rows)


def _check_codes(gpu, ref):
    _, kq, vq, ks, vs, *_ = gpu
    okq, ovq, oks, ovs = ref[:4]
    np.testing.assert_array_equal(kq.cpu().numpy(), okq)
    np.testing.assert_array_equal(vq.cpu().numpy(), ovq)
    np.testing.assert_array_equal(ks.cpu().numpy().view(np.uint32), oks.view(np.uint32))
    np.testing.assert_array_equal(vs.cpu().numpy().view(np.uint32), ovs.view(np.uint32))


# ------------------------------------------------------------------------------------------ write
@pytest.mark.parametrize("name", ["tiny", "qwen_decode", "prefill"])
def test_write_int8_bit_exact_workloads(name):
    """Every row of the pool (quantised as the cache's prior contents) and every new token's row."""
    wl = make_workload(name)
    _check_codes(gpu_step_int8(wl, decode=False), oracle_step_int8(wl))


@pytest.mark.parametrize("Hkv,D,dt,bs", [(1, 64, torch.float16, 16), (8, 128, torch.bfloat16, 32),
                                         (3, 64, torch.bfloat16, 256), (2, 128, torch.float16, 64)])
def test_write_int8_sentinels_skips_and_special_rows(Hkv, D, dt, bs):
    """Untouched rows keep their sentinel bytes, slot -1 writes nothing, and the special rows land exactly:
    zeros (zero codes, scale 0), one non-zero element (+-127), a row of equal magnitudes, the dtype's largest
    finite value, subnormal-sized values and rows on a power-of-two grid."""
    g = torch.Generator().manual_seed(Hkv * 1000 + D + bs)
    NB, T = 9, 5 * bs
    k = (torch.randn(T, Hkv, D, generator=g) * torch.exp(torch.randn(T, Hkv, 1, generator=g) * 3)).clamp(-6e4, 6e4)
    k = k.to(dt)
    v = torch.randn(T, Hkv, D, generator=g).to(dt)
    big = 65504.0 if dt == torch.float16 else 3.0e38
    k[0] = 0
    k[1] = 0
    k[1, :, D // 3] = -2.5
    k[2] = 0.75
    k[2, :, ::2] = -0.75
    k[3, :, 0] = big
    k[4] = (torch.randint(-8, 9, (Hkv, D), generator=g).float() / 8).to(dt)
    v[5] = torch.full((Hkv, D), 1e-5 if dt == torch.float16 else 1e-30).to(dt)
    slots = torch.randperm(NB * bs, generator=g)[:T].to(torch.int64)
    slots[7::5] = -1
    kq0 = torch.full((NB, bs, Hkv, D), 0x5A, dtype=torch.int8)
    ks0 = torch.full((NB, Hkv, bs), -7.25, dtype=torch.float32)
    okq, ovq, oks, ovs = kq0.numpy().copy(), kq0.numpy().copy(), ks0.numpy().copy(), ks0.numpy().copy()
    oq.write_kv_int8(k.float().numpy(), v.float().numpy(), slots.numpy(), okq, ovq, oks, ovs)
    kq, vq, ks, vs = kq0.cuda(), kq0.clone().cuda(), ks0.cuda(), ks0.clone().cuda()
    pa.write_kv_int8(k.cuda(), v.cuda(), slots.cuda(), kq, vq, ks, vs)
    np.testing.assert_array_equal(kq.cpu().numpy(), okq)
    np.testing.assert_array_equal(vq.cpu().numpy(), ovq)
    np.testing.assert_array_equal(ks.cpu().numpy().view(np.uint32), oks.view(np.uint32))
    np.testing.assert_array_equal(vs.cpu().numpy().view(np.uint32), ovs.view(np.uint32))


def test_copy_blocks_int8_bit_exact():
    g = torch.Generator().manual_seed(11)
    NB, bs, Hkv, D = 20, 32, 4, 128
    kq = torch.randint(-127, 128, (NB, bs, Hkv, D), generator=g, dtype=torch.int8)
    vq = torch.randint(-127, 128, (NB, bs, Hkv, D), generator=g, dtype=torch.int8)
    ks = torch.rand(NB, Hkv, bs, generator=g)
    vs = torch.rand(NB, Hkv, bs, generator=g)
    pairs = torch.tensor([[3, 7], [0, 19], [12, 1]], dtype=torch.int32)
    d = [t.cuda() for t in (kq, vq, ks, vs)]
    pa.copy_blocks_int8(pairs.cuda(), *d)
    for s_, t_ in pairs.tolist():
        for x in (kq, vq, ks, vs):
            x[t_] = x[s_]
    for got, ref in zip(d, (kq, vq, ks, vs)):
        assert torch.equal(got.cpu(), ref)


# ------------------------------------------------------------------------------------------ decode
def _oracle_decode_int8(wl, rows=None):
    ref = oracle_step_int8(wl)
    kd, vd, bt, lens = ref[4], ref[5], ref[6], ref[7]
    if rows is None:
        return oatt.decode_attention(wl.q, kd, vd, bt, lens, wl.scale), ref
    return oatt.decode_rows(wl.q, kd, vd, bt, lens, wl.scale, rows), ref


@pytest.mark.parametrize("name", ["tiny", "qwen_decode"])
def test_decode_int8_full_workload(name):
    wl = make_workload(name)
    gpu = gpu_step_int8(wl)
    ref, oref = _oracle_decode_int8(wl)
    _check_codes(gpu, oref)
    assert_close(gpu[0].float().cpu().numpy(), ref, f"int8 {name}")


def test_decode_int8_llama70b_long_sampled():
    wl = make_workload("llama70b_long")
    out = gpu_step_int8(wl)[0]
    rows = _sample_rows(wl, 40, 0)
    ref, _ = _oracle_decode_int8(wl, rows)
    got = np.stack([out[b, h].float().cpu().numpy() for b, h in rows])
    assert_close(got, ref, "int8 llama70b_long")


@pytest.mark.parametrize("bs", [16, 64, 256])
def test_decode_int8_prefix_shared_sampled(bs):
    wl = make_workload("prefix_sweep", block_size=bs)
    out = gpu_step_int8(wl)[0]
    rows = _sample_rows(wl, 40, bs)
    ref, _ = _oracle_decode_int8(wl, rows)
    got = np.stack([out[b, h].float().cpu().numpy() for b, h in rows])
    assert_close(got, ref, f"int8 prefix bs={bs}")


RAGGED = [0, 1, 2, 15, 16, 17, 31, 32, 33, 63, 64, 65, 127, 128, 129, 255, 256, 257, 511, 777, 1000, 1500]


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 4), (8, 2), (16, 2), (16, 1)])
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_decode_int8_ragged_shapes(D, Hq, Hkv, dtype):
    for bs, seed in ((16, 1), (64, 2), (256, 3)):
        wl = make_custom(seed=seed * 89 + Hq * 5 + D, lens=RAGGED, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                         block_size=bs, dtype=dtype)
        ref, _ = _oracle_decode_int8(wl)
        for ns in (0, 1, 7, 64):
            out = gpu_step_int8(wl, num_partitions=ns)[0]
            got = out.float().cpu().numpy()
            assert_close(got, ref, f"int8 D{D} G{Hq // Hkv} bs{bs} {dtype} partitions{ns}")
            assert (got[0] == 0).all()          # empty sequence -> zeros


def test_decode_int8_partition_count_invariance():
    wl = make_workload("qwen_decode")
    ref, _ = _oracle_decode_int8(wl)
    for ns in (0, 1, 2, 5, 16, 1000, 40000):
        out = gpu_step_int8(wl, num_partitions=ns)[0]
        assert_close(out.float().cpu().numpy(), ref, f"int8 partitions={ns}")


def test_decode_int8_large_logits():
    """q x10: softmax far from uniform; fp32 state and the q prescale keep parity."""
    wl = make_workload("qwen_decode", q_scale=10.0)
    out = gpu_step_int8(wl)[0]
    ref, _ = _oracle_decode_int8(wl)
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    assert_close(got, ref, "int8 q x10")


def test_decode_int8_row_scales_spanning_decades():
    """Per-token magnitudes that differ by up to ~2^40 across a sequence (each row scaled by exp(N(0, 6))):
    the V scales' running maximum grows many times inside one piece, the K scales move logits by large
    amounts, and both must still match the oracle."""
    wl = make_custom(seed=21, lens=[3000, 1, 700, 2048, 65], num_q_heads=16, num_kv_heads=4, head_dim=128,
                     block_size=16)
    g = torch.Generator().manual_seed(5)
    for name in ("k_cache0", "v_cache0", "k_new", "v_new"):
        t = getattr(wl, name)
        f = torch.exp(torch.randn(*t.shape[:-1], 1, generator=g) * 6.0)
        setattr(wl, name, (t.float() * f).to(t.dtype))
    wl.q = (wl.q.float() * 0.02).to(wl.q.dtype)
    out = gpu_step_int8(wl)[0]
    ref, _ = _oracle_decode_int8(wl)
    assert_close(out.float().cpu().numpy(), ref, "int8 spanning scales")


def test_decode_int8_zero_value_rows():
    """All-zero V rows (scale 0) and all-zero K rows: the output is exactly the oracle's (zeros where every
    V row is zero)."""
    wl = make_custom(seed=23, lens=[40, 300, 17], num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16)
    wl.v_cache0 = torch.zeros_like(wl.v_cache0)
    wl.v_new = torch.zeros_like(wl.v_new)
    wl.k_cache0[::2] = 0
    out = gpu_step_int8(wl)[0]
    ref, _ = _oracle_decode_int8(wl)
    assert (out.float().cpu() == 0).all()
    assert_close(out.float().cpu().numpy(), ref, "int8 zero rows")


@pytest.mark.parametrize("D", [64, 128])
def test_decode_int8_offset_cancellation(D):
    """The codes enter the fp16 products as 1152 + code and the offset is taken out in fp32: 1152 * sum(q)
    per score, 1152 * sum(P') per output.  Stress both subtractions: q with a common component 50x its spread
    (sum(q) large against sum(q * code)), small K rows so the attention spreads evenly over thousands of
    tokens (the V offset accumulates over every tile of a piece), zero-mean V, ragged lengths."""
    wl = make_custom(seed=31, lens=[8192, 5000, 1, 33, 2048], num_q_heads=16, num_kv_heads=2, head_dim=D,
                     block_size=16)
    g = torch.Generator().manual_seed(7)
    wl.q = (4.0 + 0.08 * torch.randn(tuple(wl.q.shape), generator=g)).to(wl.q.dtype)
    for name in ("k_cache0", "k_new"):
        t = getattr(wl, name)
        setattr(wl, name, (t.float() * 0.05).to(t.dtype))
    ref, _ = _oracle_decode_int8(wl)
    for ns in (0, 64):
        out = gpu_step_int8(wl, num_partitions=ns)[0]
        assert_close(out.float().cpu().numpy(), ref, f"int8 offset cancellation D{D} partitions{ns}")


@pytest.mark.parametrize("B", [257, 600])
def test_decode_int8_batches_over_256(B):
    """Above 256 sequences the producer's lookups scan the lengths in memory (see the 16-bit case)."""
    rng = np.random.default_rng(B)
    lens = rng.integers(0, 300, B)
    lens[::89] = 0
    wl = make_custom(seed=B * 11, lens=lens.tolist(), num_q_heads=16, num_kv_heads=2, head_dim=128, block_size=16,
                     dtype="bf16")
    ref, _ = _oracle_decode_int8(wl)
    for ns in (0, 7):
        out = gpu_step_int8(wl, num_partitions=ns)[0]
        got = out.float().cpu().numpy()
        assert_close(got, ref, f"int8 B{B} partitions{ns}")
        assert (got[lens == 0] == 0).all()
