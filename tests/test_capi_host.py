"""Host-side tests of the C ABI (no GPU): exported symbols, argument validation, decode planning,
and the C++ block pool against the oracle's pool (bit-exact block tables, slots, counts)."""

from __future__ import annotations

import ctypes
import os
import random
import re

import numpy as np
import pytest

import paged_kv_cache_330_b200 as pa
from oracle.block_pool import OraclePool, OutOfBlocks, replay
from workloads import CONFIGS, make_workload

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "paged_attn.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 18
    for n in names:
        assert hasattr(pa.lib, n), f"{n} declared in include/paged_attn.h but not exported"


def test_status_strings():
    for code in range(-8, 1):
        assert pa.lib.pa_strerror(code).decode().startswith("PA_")
    assert pa.version().count(".") == 2


# --------------------------------------------------------------------------- validation before any launch
FAKE = ctypes.c_void_p(0x10000)      # aligned, never dereferenced: every call below fails validation first
MISALIGNED = ctypes.c_void_p(0x10008)
NULL = ctypes.c_void_p(0)


def test_copy_async_host_checks():
    """pa_copy_async: zero bytes is a no-op and NULL addresses are rejected, both before any CUDA call."""
    assert pa.lib.pa_copy_async(None, None, 0, None) == pa.PA_OK
    assert pa.lib.pa_copy_async(None, ctypes.c_void_p(16), 64, None) == -1
    assert pa.lib.pa_copy_async(ctypes.c_void_p(16), None, 64, None) == -1


def test_write_kv_validation():
    L = pa.lib
    # unsupported dtype / block size / negative sizes
    assert L.pa_write_kv(FAKE, FAKE, FAKE, 4, FAKE, FAKE, 8, 16, 2, 64, 7, NULL) == -2
    assert L.pa_write_kv(FAKE, FAKE, FAKE, 4, FAKE, FAKE, 8, 24, 2, 64, 1, NULL) == -2
    assert L.pa_write_kv(FAKE, FAKE, FAKE, -1, FAKE, FAKE, 8, 16, 2, 64, 1, NULL) == -1
    assert L.pa_write_kv(FAKE, FAKE, NULL, 4, FAKE, FAKE, 8, 16, 2, 64, 1, NULL) == -1
    assert L.pa_write_kv(FAKE, FAKE, FAKE, 4, NULL, FAKE, 8, 16, 2, 64, 1, NULL) == -1
    assert L.pa_write_kv(MISALIGNED, FAKE, FAKE, 4, FAKE, FAKE, 8, 16, 2, 64, 1, NULL) == -3
    assert L.pa_write_kv(FAKE, FAKE, FAKE, 4, MISALIGNED, FAKE, 8, 16, 2, 64, 1, NULL) == -3
    assert L.pa_write_kv(FAKE, FAKE, FAKE, 0, FAKE, FAKE, 8, 16, 2, 64, 1, NULL) == 0   # no-op, nothing launched


def _rope(**kw):
    a = dict(q=FAKE, qo=FAKE, k=FAKE, v=FAKE, pos=FAKE, cos=FAKE, sin=FAKE, maxpos=64, slots=FAKE, T=4, Hq=8,
             kc=FAKE, vc=FAKE, NB=8, bs=16, Hkv=2, D=128, dt=1)
    a.update(kw)
    return pa.lib.pa_rope_write_kv(a["q"], a["qo"], a["k"], a["v"], a["pos"], a["cos"], a["sin"], a["maxpos"],
                                   a["slots"], a["T"], a["Hq"], a["kc"], a["vc"], a["NB"], a["bs"], a["Hkv"],
                                   a["D"], a["dt"], NULL)


def test_rope_write_kv_validation():
    assert _rope(dt=7) == -2 and _rope(D=96) == -2 and _rope(bs=24) == -2
    assert _rope(T=-1) == -1 and _rope(maxpos=0) == -1 and _rope(Hq=0) == -1 and _rope(NB=-1) == -1
    for name in ("q", "qo", "k", "v", "pos", "cos", "sin", "slots", "kc", "vc"):
        assert _rope(**{name: NULL}) == -1, name
    for name in ("q", "qo", "k", "v", "cos", "sin", "kc", "vc"):
        assert _rope(**{name: MISALIGNED}) == -3, name
    assert _rope(pos=ctypes.c_void_p(0x10004)) == -3 and _rope(slots=ctypes.c_void_p(0x10004)) == -3
    assert _rope(T=0, q=NULL, k=NULL, v=NULL, pos=NULL, slots=NULL) == 0      # no-op: only the caches are checked
    assert _rope(T=0, kc=MISALIGNED) == -3
    assert _rope(T=1 << 26) == -2                                               # item count past 2^31


def _dec(**kw):
    a = dict(q=FAKE, kc=FAKE, vc=FAKE, bt=FAKE, mb=8, cl=FAKE, B=2, Hq=8, Hkv=2, D=128, bs=16, NB=16, maxL=100,
             scale=0.1, dt=1, ws=FAKE, wsb=1 << 30, ns=0, out=FAKE)
    a.update(kw)
    return pa.lib.pa_decode(a["q"], a["kc"], a["vc"], a["bt"], a["mb"], a["cl"], a["B"], a["Hq"], a["Hkv"], a["D"],
                            a["bs"], a["NB"], a["maxL"], a["scale"], a["dt"], a["ws"], a["wsb"], a["ns"], a["out"],
                            NULL)


def test_decode_validation():
    assert _dec(D=96) == -2
    assert _dec(bs=8) == -2
    assert _dec(dt=3) == -2
    assert _dec(Hq=6, Hkv=4) == -1          # not a multiple
    assert _dec(Hq=64, Hkv=2) == -2         # group 32 unsupported
    assert _dec(q=NULL) == -1
    assert _dec(out=MISALIGNED) == -3
    assert _dec(mb=4) == -1                 # block-table rows too short for max_context_len
    assert _dec(maxL=5000, mb=400, ws=NULL) == -4
    assert _dec(maxL=5000, mb=400, wsb=16) == -4
    assert _dec(B=0) == 0


def test_prefill_validation():
    L = pa.lib
    args = [FAKE, FAKE, 64, 64, FAKE, FAKE, FAKE, 8, FAKE, 1, 8, 2, 128, 16, 16, 0.1, 1, FAKE, NULL]
    bad = list(args); bad[0] = NULL
    assert L.pa_prefill_chunk(*bad) == -1
    bad = list(args); bad[12] = 80
    assert L.pa_prefill_chunk(*bad) == -2
    bad = list(args); bad[17] = MISALIGNED
    assert L.pa_prefill_chunk(*bad) == -3


def test_decode_plan():
    for name in ("tiny", "qwen_decode", "llama70b_long", "prefix_sweep"):
        c = CONFIGS[name]
        B, Hq, Hkv, D = c["batch"], c["num_q_heads"], c["num_kv_heads"], c["head_dim"]
        grid, maxp, ws = pa.decode_plan(B, Hq, Hkv, D, 1000)
        assert grid >= 1 and maxp == B * Hkv + grid
        G = Hq // Hkv
        assert ws >= B * Hkv * 4 + maxp * G * (D + 2) * 4
        assert pa.lib.pa_decode_workspace_size(B, Hq, Hkv, D, 1000, 0) == ws
    grid, maxp, ws = pa.decode_plan(4, 8, 2, 128, 1000, num_partitions=7)
    assert grid == 7 and maxp == 4 * 2 + 7
    assert pa.lib.pa_decode_workspace_size(4, 8, 2, 96, 1000, 0) == 0      # unsupported head_dim
    assert pa.lib.pa_decode_workspace_size(4, 6, 4, 128, 1000, 0) == 0     # heads not a multiple


# --------------------------------------------------------------------------- C++ pool vs oracle pool
def _compare_pools(cpp: pa.BlockPool, orc: OraclePool, live):
    st, so = cpp.stats(), orc.stats()
    for k in ("num_blocks", "free_blocks", "used_blocks", "shared_blocks", "num_seqs", "tokens", "table_refs", "ref_sum"):
        assert st[k] == so[k], k
    assert abs(st["utilisation"] - so["utilisation"]) < 1e-12
    if live:
        mb = max(len(orc.seqs[s]["blocks"]) for s in live) + 1
        bt, lens = cpp.block_table(live, mb)
        rows, olens = orc.block_table(live, mb)
        np.testing.assert_array_equal(bt, np.array(rows, dtype=np.int32))
        np.testing.assert_array_equal(lens, np.array(olens, dtype=np.int32))
    for b in range(orc.num_blocks):
        assert cpp.ref_count(b) == orc.ref[b]


def test_pool_parity_random_ops():
    rnd = random.Random(5)
    for bs in (16, 32, 64, 256):
        NB = 150
        order = list(np.random.default_rng(bs).permutation(NB))
        cpp, orc = pa.BlockPool(NB, bs, order), OraclePool(NB, bs, order)
        live, nid = [], 0
        for step in range(800):
            r = rnd.random()
            if r < 0.3 or not live:
                op = ("alloc", nid, rnd.randint(0, 400)); nid += 1
            elif r < 0.45:
                p = rnd.choice(live)
                op = ("fork", p, nid, rnd.randint(0, orc.seqs[p]["len"])); nid += 1
            elif r < 0.8:
                op = ("append", rnd.choice(live), rnd.randint(0, 50))
            else:
                op = ("free", rnd.choice(live))
            o_err = c_err = None
            try:
                if op[0] == "alloc": orc.alloc(op[1], op[2])
                elif op[0] == "fork": orc.fork(op[1], op[2], op[3])
                elif op[0] == "append": o_res = orc.append(op[1], op[2])
                else: orc.free_seq(op[1])
            except OutOfBlocks:
                o_err = "oom"
            try:
                if op[0] == "alloc": cpp.alloc(op[1], op[2])
                elif op[0] == "fork": cpp.fork(op[1], op[2], op[3])
                elif op[0] == "append": c_res = cpp.append(op[1], op[2])
                else: cpp.free(op[1])
            except pa.PoolOutOfBlocks:
                c_err = "oom"
            assert o_err == c_err, (step, op)
            if o_err is None:
                if op[0] in ("alloc", "fork"):
                    live.append(op[-2] if op[0] == "fork" else op[1])
                elif op[0] == "free":
                    live.remove(op[1])
                elif op[0] == "append":
                    np.testing.assert_array_equal(c_res[0], np.array(o_res[0], dtype=np.int64))
                    assert c_res[1] == o_res[1]
            if step % 50 == 0:
                _compare_pools(cpp, orc, live)
        _compare_pools(cpp, orc, live)
        for s in list(live):
            cpp.free(s); orc.free_seq(s)
        _compare_pools(cpp, orc, [])
        assert cpp.stats()["free_blocks"] == NB


def test_pool_errors_leave_state_unchanged():
    p = pa.BlockPool(4, 16)
    p.alloc(0, 60)
    with pytest.raises(pa.PoolOutOfBlocks):
        p.append(0, 10)
    assert p.info(0) == (60, 4)
    with pytest.raises(pa.PagedAttnError):
        p.alloc(0, 1)                        # duplicate id
    with pytest.raises(pa.PagedAttnError):
        p.fork(0, 1, 61)                     # longer than parent
    with pytest.raises(pa.PagedAttnError):
        p.free(9)
    with pytest.raises(ValueError):
        pa.BlockPool(4, 16, [0, 1, 1, 2])    # not a permutation
    assert p.stats()["used_blocks"] == 4


def _oracle_batch(orc: OraclePool, ids, counts):
    """The oracle's reading of a batched append: one append per sequence, in batch order."""
    slots, pairs = [], []
    for sid, n in zip(ids, counts):
        s, p = orc.append(sid, n)
        slots += s
        pairs += p
    return slots, pairs


def _snapshot(pool: pa.BlockPool, ids, nb):
    mb = max(pool.info(i)[1] for i in ids) + 1
    return pool.stats(), pool.block_table(ids, mb), [pool.ref_count(b) for b in range(nb)]


def test_append_batch_matches_sequential_appends():
    """Random batches over forked sequences (shared full and partial blocks): the native batched append gives
    the oracle's sequential result — slots, copy-on-write pairs, block tables, reference counts."""
    rnd = random.Random(23)
    for bs in (16, 32, 128):
        NB = 12000                                                    # never exhausted by 120 batches
        order = list(np.random.default_rng(bs + 1).permutation(NB))
        cpp, orc = pa.BlockPool(NB, bs, order), OraclePool(NB, bs, order)
        live = []
        for sid in range(6):
            n = rnd.randint(1, 5 * bs)
            cpp.alloc(sid, n); orc.alloc(sid, n); live.append(sid)
        nid = 6
        for step in range(120):
            if rnd.random() < 0.35:                                   # fork at any point (partial blocks too)
                p = rnd.choice(live)
                k = rnd.randint(0, orc.seqs[p]["len"])
                cpp.fork(p, nid, k); orc.fork(p, nid, k); live.append(nid); nid += 1
            if len(live) > 24:
                s = live.pop(rnd.randrange(len(live)))
                cpp.free(s); orc.free_seq(s)
            batch = rnd.sample(live, rnd.randint(1, len(live)))
            counts = [rnd.choice([0, 1, 1, 1, 2, bs - 1, bs, bs + 3]) for _ in batch]
            o_res = _oracle_batch(orc, batch, counts)
            c_slots, c_pairs = cpp.append_batch(batch, counts)
            np.testing.assert_array_equal(c_slots, np.array(o_res[0], dtype=np.int64))
            assert c_pairs == o_res[1], (step, batch, counts)
            if step % 10 == 0:
                _compare_pools(cpp, orc, live)
        _compare_pools(cpp, orc, live)


def test_append_batch_two_sharers_of_one_partial_block():
    """Two sequences share a partly filled last block: the first append copies it, after which the second
    holds it alone and appends in place (no second copy) — and a pool with exactly the blocks that needs
    accepts the batch."""
    for make in (lambda: pa.BlockPool(4, 16), lambda: OraclePool(4, 16)):
        pool = make()
        pool.alloc(0, 20)                       # blocks 0, 1 (the second partly filled)
        pool.fork(0, 1, 20)                     # both hold blocks 0 and 1
        assert len(pool.free) == 2 if isinstance(pool, OraclePool) else pool.stats()["free_blocks"] == 2
    cpp, orc = pa.BlockPool(3, 16), OraclePool(3, 16)
    for p in (cpp, orc):
        p.alloc(0, 20); p.fork(0, 1, 20)
    slots, pairs = cpp.append_batch([0, 1], [1, 1])    # one free block: enough, since only one copy is made
    o_slots, o_pairs = _oracle_batch(orc, [0, 1], [1, 1])
    assert pairs == o_pairs == [(1, 2)]
    np.testing.assert_array_equal(slots, np.array(o_slots, dtype=np.int64))
    assert slots.tolist() == [2 * 16 + 4, 1 * 16 + 4]
    _compare_pools(cpp, orc, [0, 1])


def test_append_batch_is_all_or_nothing():
    cpp = pa.BlockPool(10, 16)
    cpp.alloc(0, 30); cpp.alloc(1, 5); cpp.fork(1, 2, 5)
    before = _snapshot(cpp, [0, 1, 2], 10)
    with pytest.raises(pa.PoolOutOfBlocks):
        cpp.append_batch([0, 1, 2], [16, 16, 200])          # the last one cannot fit: nothing is applied
    with pytest.raises(pa.PagedAttnError):
        cpp.append_batch([0, 1, 0], [1, 1, 1])              # repeated id
    with pytest.raises(pa.PagedAttnError):
        cpp.append_batch([0, 7], [1, 1])                    # unknown id
    with pytest.raises(pa.PagedAttnError):
        cpp.append_batch([0, 1], [1, -1])                   # negative count
    after = _snapshot(cpp, [0, 1, 2], 10)
    assert before[0] == after[0] and before[2] == after[2]
    for x, y in zip(before[1], after[1]):
        np.testing.assert_array_equal(x, y)
    slots, pairs = cpp.append_batch([], [])
    assert slots.shape == (0,) and pairs == []


def test_alloc_and_free_batches_match_sequential_calls():
    """Admission and retirement in batches: the same block tables, counts and free list as one call per
    sequence in order (compared with the oracle pool), interleaved with batched appends and forks."""
    rnd = random.Random(31)
    for bs in (16, 64):
        NB = 3000
        order = list(np.random.default_rng(bs + 7).permutation(NB))
        cpp, orc = pa.BlockPool(NB, bs, order), OraclePool(NB, bs, order)
        live, nid = [], 0
        for step in range(60):
            k = rnd.randint(0, 6)
            ids = list(range(nid, nid + k))
            lens = [rnd.randint(0, 3 * bs) for _ in ids]
            nid += k
            cpp.alloc_batch(ids, lens)
            for i, n in zip(ids, lens):
                orc.alloc(i, n)
            live += ids
            if live and rnd.random() < 0.4:
                p = rnd.choice(live)
                f = rnd.randint(0, orc.seqs[p]["len"])
                cpp.fork(p, nid, f); orc.fork(p, nid, f); live.append(nid); nid += 1
            if live:
                batch = rnd.sample(live, rnd.randint(1, len(live)))
                cpp.append_batch(batch, 1)
                _oracle_batch(orc, batch, [1] * len(batch))
            if len(live) > 8:
                gone = rnd.sample(live, rnd.randint(1, len(live) // 2))
                cpp.free_batch(gone)
                for g in gone:
                    orc.free_seq(g)
                    live.remove(g)
            _compare_pools(cpp, orc, live)
        cpp.free_batch(live)
        for g in live:
            orc.free_seq(g)
        _compare_pools(cpp, orc, [])
        assert cpp.stats()["free_blocks"] == NB


def test_alloc_and_free_batches_are_all_or_nothing():
    cpp = pa.BlockPool(6, 16)
    cpp.alloc_batch([0, 1], [20, 16])                        # 3 blocks
    before = _snapshot(cpp, [0, 1], 6)
    with pytest.raises(pa.PoolOutOfBlocks):
        cpp.alloc_batch([2, 3], [16, 40])                    # needs 4 of the 3 free blocks
    with pytest.raises(pa.PagedAttnError):
        cpp.alloc_batch([2, 2], [1, 1])                      # repeated id
    with pytest.raises(pa.PagedAttnError):
        cpp.alloc_batch([2, 1], [1, 1])                      # a live id
    with pytest.raises(pa.PagedAttnError):
        cpp.alloc_batch([2, 3], [1, -1])                     # negative count
    with pytest.raises(pa.PagedAttnError):
        cpp.free_batch([0, 5])                               # unknown id: sequence 0 stays
    with pytest.raises(pa.PagedAttnError):
        cpp.free_batch([1, 1])                               # repeated id
    after = _snapshot(cpp, [0, 1], 6)
    assert before[0] == after[0] and before[2] == after[2]
    for x, y in zip(before[1], after[1]):
        np.testing.assert_array_equal(x, y)
    cpp.alloc_batch([2, 3, 4], [0, 16, 1])                   # 0 + 1 + 1 blocks of the 3 free
    assert cpp.stats()["free_blocks"] == 1
    cpp.free_batch([0, 1, 2, 3, 4])
    assert cpp.stats()["free_blocks"] == 6 and cpp.stats()["num_seqs"] == 0
    cpp.alloc_batch([], [])
    cpp.free_batch([])


@pytest.mark.parametrize("name,bs", [("tiny", None), ("qwen_decode", None), ("llama70b_long", None),
                                     ("prefix_sweep", 16), ("prefix_sweep", 256), ("prefill", None)])
def test_workload_replay_parity(name, bs):
    """The C++ pool and the oracle pool hand out identical block tables and slots for every workload."""
    wl = make_workload(name, block_size=bs) if bs else make_workload(name)
    bsz = wl.cfg["block_size"]
    _, bt, lens, sm, cow = pa.replay_ops(wl.ops, wl.num_blocks, bsz, wl.free_order, wl.batch)
    pool, rows, olens, osm, ocow = replay(wl.ops, wl.num_blocks, bsz, wl.free_order, wl.batch)
    np.testing.assert_array_equal(bt, np.array(rows, dtype=np.int32))
    np.testing.assert_array_equal(lens, wl.context_lens)
    np.testing.assert_array_equal(sm, np.array(osm, dtype=np.int64))
    assert cow == ocow == []
    if name == "prefix_sweep":
        st = pool.stats()
        per_prefix = -(-wl.cfg["prefix_len"] // bsz)
        assert st["shared_blocks"] == wl.cfg["groups"] * per_prefix
        assert max(pool.ref) == wl.batch // wl.cfg["groups"]        # ref_count 32 on prefix blocks
