"""Pins of the CPU oracle against the pages and the mathematics (no GPU)."""

from __future__ import annotations

import json
import os
import random

import numpy as np
import pytest

import oracle
from oracle import attention as att
from oracle.block_pool import OraclePool, OutOfBlocks, blocks_for, replay
from tests import oracle_checks
from workloads import make_workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------- block arithmetic (pages)
def test_worked_block_example():
    g = json.load(open(os.path.join(GOLDEN, "block_arithmetic.json")))
    bs, n = g["block_size"], g["tokens"]
    pool = OraclePool(100, bs)
    pool.alloc(7, n)
    st = pool.stats()
    assert st["used_blocks"] == g["blocks"] == blocks_for(n, bs)
    assert st["used_blocks"] * bs == g["slots"]
    waste = (g["slots"] - n) / g["slots"]
    assert abs(waste - g["waste_fraction_printed"]) <= g["waste_fraction_printed_precision"]
    assert abs((1 - st["utilisation"]) - waste) < 1e-15
    s = g["static_prealloc"]
    assert abs((s["capacity_tokens"] - s["used_tokens"]) / s["capacity_tokens"] - s["waste_fraction_printed"]) <= s["precision"]
    assert st["utilisation"] > g["paged_utilisation_floor_printed"]


def test_utilisation_on_qwen_lengths():
    """Lengths uniform in 100..1024 (the Qwen3-0.6B batching workload) at block size 16: above the printed 93%."""
    g = json.load(open(os.path.join(GOLDEN, "block_arithmetic.json")))
    wl = make_workload("qwen_decode")
    pool, rows, lens, slots, cow = replay(wl.ops, wl.num_blocks, wl.cfg["block_size"], wl.free_order, wl.batch)
    st = pool.stats()
    assert st["utilisation"] > g["paged_utilisation_floor_printed"]
    assert lens == list(wl.context_lens)
    assert cow == []


# --------------------------------------------------------------------------- pool invariants
def _invariants(pool: OraclePool):
    st = pool.stats()
    assert st["ref_sum"] == st["table_refs"]            # every table entry is one reference
    assert st["free_blocks"] + st["used_blocks"] == pool.num_blocks
    assert len(set(pool.free)) == len(pool.free)
    for b in pool.free:
        assert pool.ref[b] == 0
    for s in pool.seqs.values():
        assert len(s["blocks"]) == blocks_for(s["len"], pool.block_size)


def test_pool_random_ops_no_leak():
    rnd = random.Random(11)
    for bs in (16, 32, 64):
        pool = OraclePool(200, bs, list(np.random.default_rng(bs).permutation(200)))
        live = []
        nid = 0
        for _ in range(600):
            r = rnd.random()
            try:
                if r < 0.3 or not live:
                    pool.alloc(nid, rnd.randint(0, 300)); live.append(nid); nid += 1
                elif r < 0.45:
                    p = rnd.choice(live)
                    pool.fork(p, nid, rnd.randint(0, pool.seqs[p]["len"])); live.append(nid); nid += 1
                elif r < 0.8:
                    pool.append(rnd.choice(live), rnd.randint(0, 40))
                else:
                    s = rnd.choice(live); pool.free_seq(s); live.remove(s)
            except OutOfBlocks:
                pass
            _invariants(pool)
        for s in list(live):
            pool.free_seq(s)
        _invariants(pool)
        assert sorted(pool.free) == list(range(200))       # every block came back


def test_fork_refcount_and_copy_on_write():
    pool = OraclePool(10, 16, list(range(10)))
    pool.alloc(0, 40)                                      # blocks 0,1,2 (last one partly filled)
    for c in range(1, 32):
        if c < 4:
            pool.fork(0, c, 40)
    assert [pool.ref[b] for b in (0, 1, 2)] == [4, 4, 4]
    slots, pairs = pool.append(1, 3)                       # appending into shared partial block 2 copies it
    assert pairs == [(2, 3)]
    assert pool.seqs[1]["blocks"] == [0, 1, 3]
    assert slots == [3 * 16 + 8, 3 * 16 + 9, 3 * 16 + 10]
    assert pool.ref[2] == 3 and pool.ref[3] == 1
    # aligned prefix: no copy, a fresh block
    pool2 = OraclePool(10, 16, list(range(10)))
    pool2.alloc(0, 32)
    pool2.fork(0, 1, 32)
    slots, pairs = pool2.append(1, 1)
    assert pairs == [] and slots == [2 * 16]
    _invariants(pool); _invariants(pool2)


def test_out_of_blocks_is_atomic():
    pool = OraclePool(4, 16)
    pool.alloc(0, 60)
    with pytest.raises(OutOfBlocks):
        pool.append(0, 10)
    assert pool.seqs[0]["len"] == 60 and len(pool.free) == 0
    with pytest.raises(OutOfBlocks):
        pool.alloc(1, 1)
    assert 1 not in pool.seqs


def test_write_then_gather_roundtrip():
    """Tokens written through their slots come back in order through the block table (the slot rule and the
    gather rule agree)."""
    rng = np.random.default_rng(3)
    for bs in (16, 32, 128):
        pool = OraclePool(40, bs, list(rng.permutation(40)))
        pool.alloc(0, 0)
        kc = rng.integers(0, 1 << 16, size=(40, bs, 2, 8), dtype=np.uint16)
        vc = kc.copy()
        toks = rng.integers(0, 1 << 16, size=(300, 2, 8), dtype=np.uint16)
        pos = 0
        for n in (1, 15, 16, 17, 100, 151):
            slots, _ = pool.append(0, n)
            oracle.write_kv(toks[pos:pos + n], toks[pos:pos + n], slots, kc, vc)
            pos += n
        rows, lens = pool.block_table([0], 40)
        np.testing.assert_array_equal(att.gather_kv(kc, rows[0], lens[0]), toks[:pos])


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
