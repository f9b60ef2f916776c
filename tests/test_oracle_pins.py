"""Pins of the CPU oracle against the pages and the mathematics (no GPU)."""

from __future__ import annotations

import numpy as np
import pytest

import oracle
from oracle import attention as att
from oracle import block_pool
from oracle.block_pool import replay
from tests import oracle_checks, pool_checks
from workloads import make_workload


# --------------------------------------------------------------------------- block pool (pages + invariants)
@pytest.mark.parametrize("check", pool_checks.ALL_CHECKS, ids=lambda c: c.__name__)
def test_pool_pin(check):
    check(block_pool)


def test_kv_write_bytes_sentinel_and_skip():
    rng = np.random.default_rng(5)
    kc = np.full((8, 16, 2, 8), 0xA5A5, dtype=np.uint16)
    vc = kc.copy()
    k = rng.integers(0, 1 << 16, size=(5, 2, 8), dtype=np.uint16)
    v = rng.integers(0, 1 << 16, size=(5, 2, 8), dtype=np.uint16)
    slots = [3, -1, 127, 16, 40]
    oracle.write_kv(k, v, slots, kc, vc)
    want_k = np.full_like(kc, 0xA5A5)
    for t, s in enumerate(slots):                           # scalar twin of the scatter
        if s >= 0:
            for h in range(2):
                for d in range(8):
                    want_k[s // 16, s % 16, h, d] = k[t, h, d]
    np.testing.assert_array_equal(kc, want_k)
    assert (vc[0, 3] == v[0]).all() and (vc[7, 15] == v[2]).all()
    assert not (kc == k[1][None, None]).all(axis=(2, 3)).any()   # the skipped row is nowhere


# --------------------------------------------------------------------------- attention pins
@pytest.mark.parametrize("check", oracle_checks.ALL_CHECKS, ids=lambda c: c.__name__)
def test_attention_pin(check):
    check(att)


def test_decode_rows_matches_full():
    wl = make_workload("tiny")
    pool, rows, lens, slots, _ = replay(wl.ops, wl.num_blocks, wl.cfg["block_size"], wl.free_order, wl.batch)
    full = att.decode_attention(wl.q, wl.k_cache0, wl.v_cache0, rows, lens, wl.scale)
    pairs = [(b, h) for b in range(wl.batch) for h in range(wl.cfg["num_q_heads"])]
    sub = att.decode_rows(wl.q, wl.k_cache0, wl.v_cache0, rows, lens, wl.scale, pairs)
    np.testing.assert_allclose(sub, np.stack([full[b, h] for b, h in pairs]), rtol=1e-13, atol=1e-14)
