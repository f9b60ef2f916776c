"""GPU parity: pa_rope_write_kv (rotary embedding of q and k fused with the cache write) against the oracle,
alone and chained into pa_decode / pa_prefill_chunk.

Tolerance of a rotated element, derived from the arithmetic: the kernel forms x1*c - x2*s (and x2*c + x1*s)
in fp32 from exact 16-bit inputs and fp32 table entries (two roundings of at most 2^-24 relative each), then
rounds to the 16-bit type (at most half an ulp: 2^-8 |y| for bf16, 2^-11 |y| for fp16, plus 2^-25 absolute
in fp16's subnormal range).  So |gpu - y| <= u |y| (1 + 2^-6) + 2^-22 (|x1| + |x2|) + 2^-24 with y the exact
fp64 result.  V rows and every untouched cache row are compared bit for bit.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from oracle import rope as orope
from oracle import write_kv as owrite
from oracle import replay as oreplay
from tests.gpu_common import assert_close, bits, from_bits
from workloads import make_custom, make_rope_case, make_workload, new_token_positions, rope_tables

pytestmark = pytest.mark.gpu

pa = pytest.importorskip("paged_kv_cache_330_b200")

UNIT = {torch.bfloat16: 2.0 ** -8, torch.float16: 2.0 ** -11}


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    assert pa.device_error() == 0, "a kernel recorded a device-side error"


def _pair_mag(x: np.ndarray) -> np.ndarray:
    """|x1| + |x2| of each element's rotation pair, laid out like x [..., D]."""
    half = x.shape[-1] // 2
    m = np.abs(x[..., :half]) + np.abs(x[..., half:])
    return np.concatenate([m, m], axis=-1)


def assert_rotated(got: torch.Tensor, ref: np.ndarray, x: np.ndarray, dtype, what: str):
    g = got.float().cpu().numpy().astype(np.float64)
    tol = UNIT[dtype] * np.abs(ref) * (1 + 2.0 ** -6) + 2.0 ** -22 * _pair_mag(x) + 2.0 ** -24
    err = np.abs(g - ref)
    bad = ~(err <= tol)
    if bad.any():
        idx = np.argwhere(bad)[:5].tolist()
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} out of tolerance; first {idx} "
                             f"got {[float(g[tuple(i)]) for i in idx]} ref {[float(ref[tuple(i)]) for i in idx]}")


def _run_case(c, dtype, in_place=False):
    dev = "cuda"
    q = c.q.to(dev)
    kc, vc = c.k_cache0.to(dev), c.v_cache0.to(dev)
    q_out = q if in_place else None
    out = pa.rope_write_kv(q, c.k.to(dev), c.v.to(dev), c.positions.to(dev), c.cos.to(dev), c.sin.to(dev),
                           c.slots.to(dev), kc, vc, q_out=q_out)
    torch.cuda.synchronize()
    # oracle
    vcb = bits(c.v_cache0).copy()
    q_rot, k_rot = orope.rope_write_kv(c.q.double().numpy(), c.k.double().numpy(), bits(c.v), c.positions.numpy(),
                                       c.cos.numpy(), c.sin.numpy(), c.slots.numpy(), vcb)
    assert_rotated(out, q_rot, c.q.double().numpy(), dtype, "q_out")
    NB, bs, Hkv, D = c.k_cache0.shape
    krows = kc.cpu().view(NB * bs, Hkv, D)
    k0 = c.k_cache0.view(NB * bs, Hkv, D)
    slots = c.slots.numpy()
    written = np.zeros(NB * bs, dtype=bool)
    for t, s in enumerate(slots):
        if s >= 0:
            written[s] = True
            assert_rotated(krows[s], k_rot[t], c.k[t].double().numpy(), dtype, f"k cache slot {s}")
    # untouched K rows keep their bytes; V equals the oracle's byte write everywhere
    assert np.array_equal(bits(krows[~torch.from_numpy(written)]), bits(k0[~torch.from_numpy(written)]))
    assert np.array_equal(bits(vc.cpu()), vcb)
    return out, q


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("Hq,Hkv,D", [(32, 8, 128), (4, 4, 64), (16, 2, 128), (8, 1, 64)])
@pytest.mark.parametrize("bs", [16, 64, 256])
def test_rope_write_random(dtype, Hq, Hkv, D, bs):
    """Ragged token counts, positions over the whole table (first and last rows included), 10% of slots -1."""
    for T in (1, 37, 515):
        c = make_rope_case(seed=T * 7 + Hq + bs, num_tokens=T, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
                           block_size=bs, num_blocks=-(-T // bs) + 3, dtype=dtype, max_position=4096)
        _run_case(c, c.q.dtype)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_rope_write_random_angles(dtype):
    """Table angles uniform over the whole circle (large rotations of every pair, both signs of cos/sin)."""
    c = make_rope_case(seed=3, num_tokens=300, num_q_heads=16, num_kv_heads=8, head_dim=128, block_size=16,
                       num_blocks=30, dtype=dtype, max_position=64, random_angles=True)
    _run_case(c, c.q.dtype)


def test_rope_write_in_place():
    c = make_rope_case(seed=9, num_tokens=129, num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=32,
                       num_blocks=8, max_position=1024)
    out, q_dev = _run_case(c, torch.bfloat16, in_place=True)
    assert out.data_ptr() == q_dev.data_ptr()     # rotated the device copy in place and returned it


def test_rope_write_empty_is_noop():
    kc = torch.zeros(4, 16, 2, 64, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    e3 = torch.empty(0, 2, 64, dtype=torch.bfloat16, device="cuda")
    cos, sin = (t.cuda() for t in rope_tables(16, 64))
    out = pa.rope_write_kv(torch.empty(0, 4, 64, dtype=torch.bfloat16, device="cuda"), e3, e3,
                           torch.empty(0, dtype=torch.int64, device="cuda"), cos, sin,
                           torch.empty(0, dtype=torch.int64, device="cuda"), kc, vc)
    assert out.shape[0] == 0 and int(kc.abs().sum()) == 0


def test_rope_write_out_of_range_indices_are_recorded():
    """A position past the tables and a slot past the pool: the kernel's own bounds checks skip those rows
    and set the index bit of the device error word; every other token is written normally."""
    c = make_rope_case(seed=4, num_tokens=40, num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16,
                       num_blocks=4, max_position=128, skip_frac=0.0)
    bad_pos, bad_slot = 5, 11
    pos = c.positions.clone()
    pos[bad_pos] = 128
    slots = c.slots.clone()
    slots[bad_slot] = 4 * 16
    dev = "cuda"
    kc, vc = c.k_cache0.to(dev), c.v_cache0.to(dev)
    q_out = torch.zeros_like(c.q, device=dev)
    pa.rope_write_kv(c.q.to(dev), c.k.to(dev), c.v.to(dev), pos.to(dev), c.cos.to(dev), c.sin.to(dev),
                     slots.to(dev), kc, vc, q_out=q_out)
    assert pa.device_error() == 2
    assert int(q_out[bad_pos].abs().sum()) == 0          # nothing written for the bad position
    ok = [t for t in range(40) if t not in (bad_pos, bad_slot)]
    q_rot, k_rot = orope.rope_tokens(c.q.double().numpy(), c.positions.numpy(), c.cos.numpy(), c.sin.numpy()), \
        orope.rope_tokens(c.k.double().numpy(), c.positions.numpy(), c.cos.numpy(), c.sin.numpy())
    assert_rotated(q_out[ok], q_rot[ok], c.q[ok].double().numpy(), torch.bfloat16, "q_out")
    assert_rotated(q_out[bad_slot], q_rot[bad_slot], c.q[bad_slot].double().numpy(), torch.bfloat16, "q (bad slot)")
    krows = kc.cpu().view(64, 2, 64)
    for t in ok:
        assert_rotated(krows[int(slots[t])], k_rot[t], c.k[t].double().numpy(), torch.bfloat16, f"k {t}")
    # the bad position's slot keeps its old bytes
    s = int(slots[bad_pos])
    assert np.array_equal(bits(krows[s]), bits(c.k_cache0.view(64, 2, 64)[s]))


def _oracle_cache_after_rope(wl, positions, cos, sin):
    """Oracle chain: its pool replay, fp64 rotation, rounding of q and k to the cache type (the bytes the
    attention step reads), byte write of k and v; returns (q_rot rounded, caches, rows, lens)."""
    dt = wl.k_cache0.dtype
    _, rows, lens, slots, _ = oreplay(wl.ops, wl.num_blocks, wl.cfg["block_size"], wl.free_order, wl.batch)
    q_rot = orope.rope_tokens(wl.q.double().numpy(), positions, cos.numpy(), sin.numpy())
    k_rot = orope.rope_tokens(wl.k_new.double().numpy(), positions, cos.numpy(), sin.numpy())
    qr = torch.from_numpy(q_rot).to(dt)
    kr = torch.from_numpy(k_rot).to(dt)
    kc, vc = bits(wl.k_cache0).copy(), bits(wl.v_cache0).copy()
    owrite(bits(kr), bits(wl.v_new), slots, kc, vc)
    return qr, from_bits(kc, dt), from_bits(vc, dt), rows, lens


def test_rope_then_decode():
    """Rotary + cache write of each sequence's new token, then decode on the rotated q: against the oracle's
    chain (rotation in fp64, rounded to bf16 where the cache and q hold it)."""
    wl = make_custom(seed=31, lens=[1, 17, 300, 1024, 2049], num_q_heads=16, num_kv_heads=8, head_dim=128,
                     block_size=16)
    positions = new_token_positions(wl)          # decode: each new token's position = its context index
    cos, sin = rope_tables(4096, 128)
    _, bt, lens, sm, _ = pa.replay_ops(wl.ops, wl.num_blocks, 16, wl.free_order, wl.batch)
    kc, vc = wl.k_cache0.cuda(), wl.v_cache0.cuda()
    q = pa.rope_write_kv(wl.q.cuda(), wl.k_new.cuda(), wl.v_new.cuda(), torch.from_numpy(positions).cuda(),
                         cos.cuda(), sin.cuda(), torch.from_numpy(sm).cuda(), kc, vc)
    out = pa.decode(q, kc, vc, torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda(), int(lens.max()), wl.scale)
    qr, okc, ovc, rows, olens = _oracle_cache_after_rope(wl, positions, cos, sin)
    ref = oatt.decode_attention(qr, okc, ovc, rows, olens, wl.scale)
    assert_close(out.float().cpu().numpy(), ref, "rope -> decode")


def test_rope_then_prefill():
    """Rotary + cache write of each sequence's chunk, then chunked prefill on the rotated queries."""
    wl = make_custom(seed=32, lens=[300, 900, 129], chunk_lens=[300, 200, 129], kind="prefill", num_q_heads=8,
                     num_kv_heads=2, head_dim=128, block_size=16)
    positions = new_token_positions(wl)
    cos, sin = rope_tables(1024, 128)
    _, bt, lens, sm, _ = pa.replay_ops(wl.ops, wl.num_blocks, 16, wl.free_order, wl.batch)
    kc, vc = wl.k_cache0.cuda(), wl.v_cache0.cuda()
    q = pa.rope_write_kv(wl.q.cuda(), wl.k_new.cuda(), wl.v_new.cuda(), torch.from_numpy(positions).cuda(),
                         cos.cuda(), sin.cuda(), torch.from_numpy(sm).cuda(), kc, vc)
    qsl = torch.from_numpy(wl.query_start_loc).cuda()
    out = pa.prefill_chunk(q, qsl, kc, vc, torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda(),
                           int(np.diff(wl.query_start_loc).max()), wl.scale)
    qr, okc, ovc, rows, olens = _oracle_cache_after_rope(wl, positions, cos, sin)
    ref = oatt.prefill_attention(qr, wl.query_start_loc, okc, ovc, rows, olens, wl.scale)
    qsl_h = wl.query_start_loc
    for (b, h), r in ref.items():
        assert_close(out[qsl_h[b]:qsl_h[b + 1], h].float().cpu().numpy(), r, f"rope -> prefill seq{b} head{h}")


def test_rope_write_full_prefill_workload():
    """The benchmarked shape: 8 x 512 chunk tokens at positions 8192..8703, 32 q / 8 kv heads, every element."""
    wl = make_workload("prefill")
    positions = new_token_positions(wl)
    cos, sin = rope_tables(16384, 128)
    _, bt, lens, sm, _ = pa.replay_ops(wl.ops, wl.num_blocks, 16, wl.free_order, wl.batch)
    kc, vc = wl.k_cache0.cuda(), wl.v_cache0.cuda()
    q = pa.rope_write_kv(wl.q.cuda(), wl.k_new.cuda(), wl.v_new.cuda(), torch.from_numpy(positions).cuda(),
                         cos.cuda(), sin.cuda(), torch.from_numpy(sm).cuda(), kc, vc)
    q_rot = orope.rope_tokens(wl.q.double().numpy(), positions, cos.numpy(), sin.numpy())
    k_rot = orope.rope_tokens(wl.k_new.double().numpy(), positions, cos.numpy(), sin.numpy())
    assert_rotated(q, q_rot, wl.q.double().numpy(), torch.bfloat16, "q_out")
    NB, bs, Hkv, D = wl.k_cache0.shape
    _, _, _, oslots, _ = oreplay(wl.ops, wl.num_blocks, bs, wl.free_order, wl.batch)   # the oracle's own slots
    idx = torch.from_numpy(np.asarray(oslots, dtype=np.int64))
    krows = kc.cpu().view(NB * bs, Hkv, D)[idx]
    assert_rotated(krows, k_rot, wl.k_new.double().numpy(), torch.bfloat16, "k cache rows")
    vrows = vc.cpu().view(NB * bs, Hkv, D)[idx]
    assert np.array_equal(bits(vrows), bits(wl.v_new))
