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
