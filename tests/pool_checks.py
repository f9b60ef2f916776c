"""Checks that pin the block-pool oracle (oracle/block_pool.py) to the pages and to invariants.

Each ``check_*`` takes the pool module under test (normally ``oracle.block_pool``) and raises
AssertionError on a mismatch; the mutation test feeds broken copies of the module through the same
checks.
"""

from __future__ import annotations

import json
import os
import random

import numpy as np
import pytest

import oracle
from oracle import attention as att
from workloads import make_workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------- block arithmetic (pages)
def check_worked_block_example(m):
    g = json.load(open(os.path.join(GOLDEN, "block_arithmetic.json")))
    bs, n = g["block_size"], g["tokens"]
    pool = m.OraclePool(100, bs)
    pool.alloc(7, n)
    st = pool.stats()
    assert st["used_blocks"] == g["blocks"] == m.blocks_for(n, bs)
    assert st["used_blocks"] * bs == g["slots"]
    waste = (g["slots"] - n) / g["slots"]
    assert abs(waste - g["waste_fraction_printed"]) <= g["waste_fraction_printed_precision"]
    assert abs((1 - st["utilisation"]) - waste) < 1e-15
    s = g["static_prealloc"]
    assert abs((s["capacity_tokens"] - s["used_tokens"]) / s["capacity_tokens"] - s["waste_fraction_printed"]) <= s["precision"]
    assert st["utilisation"] > g["paged_utilisation_floor_printed"]


def check_utilisation_on_qwen_lengths(m):
    """Lengths uniform in 100..1024 (the Qwen3-0.6B batching workload) at block size 16: above the printed 93%."""
    g = json.load(open(os.path.join(GOLDEN, "block_arithmetic.json")))
    wl = make_workload("qwen_decode")
    pool, rows, lens, slots, cow = m.replay(wl.ops, wl.num_blocks, wl.cfg["block_size"], wl.free_order, wl.batch)
    st = pool.stats()
    assert st["utilisation"] > g["paged_utilisation_floor_printed"]
    assert lens == list(wl.context_lens)
    assert cow == []


# --------------------------------------------------------------------------- pool invariants
def _invariants(m, pool):
    st = pool.stats()
    assert st["ref_sum"] == st["table_refs"]            # every table entry is one reference
    assert st["free_blocks"] + st["used_blocks"] == pool.num_blocks
    assert len(set(pool.free)) == len(pool.free)
    for b in pool.free:
        assert pool.ref[b] == 0
    for s in pool.seqs.values():
        assert len(s["blocks"]) == m.blocks_for(s["len"], pool.block_size)


def check_random_ops_no_leak(m):
    rnd = random.Random(11)
    for bs in (16, 32, 64):
        pool = m.OraclePool(200, bs, list(np.random.default_rng(bs).permutation(200)))
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
            except m.OutOfBlocks:
                pass
            _invariants(m, pool)
        for s in list(live):
            pool.free_seq(s)
        _invariants(m, pool)
        assert sorted(pool.free) == list(range(200))       # every block came back


def check_fork_refcount_and_copy_on_write(m):
    pool = m.OraclePool(10, 16, list(range(10)))
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
    pool2 = m.OraclePool(10, 16, list(range(10)))
    pool2.alloc(0, 32)
    pool2.fork(0, 1, 32)
    slots, pairs = pool2.append(1, 1)
    assert pairs == [] and slots == [2 * 16]
    _invariants(m, pool); _invariants(m, pool2)


def check_out_of_blocks_is_atomic(m):
    pool = m.OraclePool(4, 16)
    pool.alloc(0, 60)
    with pytest.raises(m.OutOfBlocks):
        pool.append(0, 10)
    assert pool.seqs[0]["len"] == 60 and len(pool.free) == 0
    with pytest.raises(m.OutOfBlocks):
        pool.alloc(1, 1)
    assert 1 not in pool.seqs


def check_write_then_gather_roundtrip(m):
    """Tokens written through their slots come back in order through the block table (the slot rule and the
    gather rule agree)."""
    rng = np.random.default_rng(3)
    for bs in (16, 32, 128):
        pool = m.OraclePool(40, bs, list(rng.permutation(40)))
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


ALL_CHECKS = [check_worked_block_example, check_utilisation_on_qwen_lengths, check_random_ops_no_leak,
              check_fork_refcount_and_copy_on_write, check_out_of_blocks_is_atomic,
              check_write_then_gather_roundtrip]
