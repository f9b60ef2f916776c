"""Shared helpers for the GPU parity tests: run one workload step through the C ABI and through the
oracle, independently, from the same seeded inputs."""

from __future__ import annotations

import numpy as np
import torch

import oracle
from oracle import attention as oatt

ATOL, RTOL = 2e-3, 1e-2   # |gpu - oracle| <= ATOL + RTOL * |oracle|, bf16/fp16 I/O with fp32 accumulation


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw 16-bit words of an fp16/bf16 CPU tensor."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits(a: np.ndarray, dtype) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(dtype)


def assert_close(got: np.ndarray, ref: np.ndarray, what: str = ""):
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = ~(err <= bound)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} elements out of tolerance; max err "
                             f"{float(np.nanmax(err)):.3e}; first {idx.tolist()} got "
                             f"{[float(got[tuple(i)]) for i in idx]} ref {[float(ref[tuple(i)]) for i in idx]}")


def oracle_step(wl):
    """Oracle side: its own pool replay, byte write, then return (caches after the write as torch CPU
    tensors, block table rows, context lengths, slot mapping)."""
    pool, rows, lens, slots, _ = oracle.replay(wl.ops, wl.num_blocks, wl.cfg["block_size"], wl.free_order, wl.batch)
    kc = bits(wl.k_cache0).copy()
    vc = bits(wl.v_cache0).copy()
    oracle.write_kv(bits(wl.k_new), bits(wl.v_new), slots, kc, vc)
    dt = wl.k_cache0.dtype
    return from_bits(kc, dt), from_bits(vc, dt), rows, lens, slots


def gpu_step(wl, num_partitions: int = 0, device="cuda"):
    """Product side: C++ pool replay, then pa_write_kv and pa_decode (or nothing else for prefill)."""
    import paged_kv_cache_330_b200 as pa
    _, bt, lens, sm, _ = pa.replay_ops(wl.ops, wl.num_blocks, wl.cfg["block_size"], wl.free_order, wl.batch)
    kc = wl.k_cache0.to(device)
    vc = wl.v_cache0.to(device)
    bt_d = torch.from_numpy(bt).to(device)
    lens_d = torch.from_numpy(lens).to(device)
    pa.write_kv(wl.k_new.to(device), wl.v_new.to(device), torch.from_numpy(sm).to(device), kc, vc)
    out = None
    if wl.cfg["kind"] != "prefill":
        out = pa.decode(wl.q.to(device), kc, vc, bt_d, lens_d, int(lens.max()), wl.scale, num_partitions=num_partitions)
    return out, kc, vc, bt_d, lens_d, bt, lens


# ---------------------------------------------------------------------------------------------- INT8 cache
def oracle_step_int8(wl):
    """Oracle side of a step over the INT8 cache: the pool's 16-bit contents quantised row by row (the
    cache before this step), the new tokens quantised into their slots, then the dequantised float64
    caches.  Returns (k_codes, v_codes, k_scales [NB, Hkv, bs], v_scales, k_deq, v_deq, rows, lens, slots)."""
    from oracle import kv_quant as oq
    _, rows, lens, slots, _ = oracle.replay(wl.ops, wl.num_blocks, wl.cfg["block_size"], wl.free_order, wl.batch)
    kq, ks = oq.quantize_rows(wl.k_cache0.float().numpy())
    vq, vs = oq.quantize_rows(wl.v_cache0.float().numpy())
    ks, vs = np.ascontiguousarray(ks.transpose(0, 2, 1)), np.ascontiguousarray(vs.transpose(0, 2, 1))
    oq.write_kv_int8(wl.k_new.float().numpy(), wl.v_new.float().numpy(), slots, kq, vq, ks, vs)
    return kq, vq, ks, vs, oq.dequantized_cache(kq, ks), oq.dequantized_cache(vq, vs), rows, lens, slots


def gpu_step_int8(wl, num_partitions: int = 0, device="cuda", decode: bool = True):
    """Product side: the pool's 16-bit contents quantised into a fresh INT8 cache by pa_write_kv_int8 (every
    slot), the C++ pool replayed, the new tokens written by pa_write_kv_int8, then pa_decode_int8.
    Returns (out or None, k_codes, v_codes, k_scales, v_scales, bt_d, lens_d, bt, lens)."""
    import paged_kv_cache_330_b200 as pa
    NB, bs, Hkv, D = wl.k_cache0.shape
    kq = torch.zeros((NB, bs, Hkv, D), dtype=torch.int8, device=device)
    vq = torch.zeros_like(kq)
    ks = torch.zeros((NB, Hkv, bs), dtype=torch.float32, device=device)
    vs = torch.zeros_like(ks)
    all_slots = torch.arange(NB * bs, dtype=torch.int64, device=device)
    pa.write_kv_int8(wl.k_cache0.to(device).view(NB * bs, Hkv, D), wl.v_cache0.to(device).view(NB * bs, Hkv, D),
                     all_slots, kq, vq, ks, vs)
    _, bt, lens, sm, _ = pa.replay_ops(wl.ops, wl.num_blocks, bs, wl.free_order, wl.batch)
    bt_d, lens_d = torch.from_numpy(bt).to(device), torch.from_numpy(lens).to(device)
    pa.write_kv_int8(wl.k_new.to(device), wl.v_new.to(device), torch.from_numpy(sm).to(device), kq, vq, ks, vs)
    out = None
    if decode:
        out = pa.decode_int8(wl.q.to(device), kq, vq, ks, vs, bt_d, lens_d, int(lens.max()), wl.scale,
                             num_partitions=num_partitions)
    return out, kq, vq, ks, vs, bt_d, lens_d, bt, lens
