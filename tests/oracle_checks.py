"""Checks that pin the attention oracle to facts outside itself.

Each ``check_*`` takes the attention module under test (normally
``oracle.attention``) and raises AssertionError on a mismatch.  The mutation
test feeds deliberately broken copies of the module through the same checks
to show that each plausible slip (a wrong head mapping, a dropped scale, a
wrong gather index, an off-by-one causal limit, a swapped operand) fails at
least one of them.
"""

from __future__ import annotations

import math

import numpy as np
import torch
import torch.nn.functional as F

from oracle import brute


def _rng(seed):
    return np.random.default_rng(seed)


def scatter_dense(K: np.ndarray, table, bs: int, NB: int, fill_rng) -> np.ndarray:
    """Place a dense [L, Hkv, D] sequence into a fresh paged cache block by block (test helper;
    a block-wise copy, not the oracle's per-token gather)."""
    L, Hkv, D = K.shape
    cache = fill_rng.standard_normal((NB, bs, Hkv, D))
    for j in range(-(-L // bs)):
        rows = K[j * bs:(j + 1) * bs]
        cache[table[j], : rows.shape[0]] = rows
    return cache


def _paged_case(seed, B, Hq, Hkv, D, bs, lens, extra_blocks=5):
    rng = _rng(seed)
    nblk = [-(-L // bs) for L in lens]
    NB = sum(nblk) + extra_blocks
    perm = rng.permutation(NB)
    tables, off = [], 0
    for n in nblk:
        tables.append(list(perm[off:off + n]) + [-1] * (max(nblk + [1]) - n))
        off += n
    Ks = [rng.standard_normal((L, Hkv, D)) for L in lens]
    Vs = [rng.standard_normal((L, Hkv, D)) for L in lens]
    kc = rng.standard_normal((NB, bs, Hkv, D))
    vc = rng.standard_normal((NB, bs, Hkv, D))
    for b in range(B):
        for j in range(nblk[b]):
            r = Ks[b][j * bs:(j + 1) * bs]
            kc[tables[b][j], : r.shape[0]] = r
            vc[tables[b][j], : r.shape[0]] = Vs[b][j * bs:(j + 1) * bs]
    q = rng.standard_normal((B, Hq, D))
    return q, kc, vc, tables, list(lens), Ks, Vs


def check_sdpa_decode(att, seed=0):
    """Paged decode == torch float64 scaled_dot_product_attention on the dense sequence
    (consecutive GQA grouping through enable_gqa)."""
    for (Hq, Hkv, D, bs) in [(4, 4, 64, 16), (8, 2, 32, 16), (16, 8, 64, 32), (8, 1, 16, 64)]:
        lens = [1, 17, 50, 33]
        q, kc, vc, tables, lens, Ks, Vs = _paged_case(seed, 4, Hq, Hkv, D, bs, lens)
        scale = 1.0 / math.sqrt(D)
        got = att.decode_attention(q, kc, vc, tables, lens, scale)
        for b in range(4):
            qt = torch.from_numpy(q[b]).view(1, Hq, 1, D)
            kt = torch.from_numpy(Ks[b]).permute(1, 0, 2).unsqueeze(0)
            vt = torch.from_numpy(Vs[b]).permute(1, 0, 2).unsqueeze(0)
            ref = F.scaled_dot_product_attention(qt, kt, vt, scale=scale, enable_gqa=(Hq != Hkv))
            np.testing.assert_allclose(got[b], ref[0, :, 0].numpy(), rtol=1e-10, atol=1e-12)


def check_sdpa_prefill_no_prefix(att, seed=1):
    """A chunk that is the whole sequence (no earlier context) == causal SDPA."""
    for (Hq, Hkv, D, bs, C) in [(4, 2, 32, 16, 37), (2, 2, 64, 32, 64)]:
        rng = _rng(seed)
        K = rng.standard_normal((C, Hkv, D))
        V = rng.standard_normal((C, Hkv, D))
        NB = -(-C // bs) + 3
        table = list(rng.permutation(NB)[: -(-C // bs)])
        kc = scatter_dense(K, table, bs, NB, rng)
        vc = scatter_dense(V, table, bs, NB, rng)
        q = rng.standard_normal((C, Hq, D))
        scale = 1.0 / math.sqrt(D)
        got = att.prefill_attention(q, [0, C], kc, vc, [table], [C], scale)
        ref = F.scaled_dot_product_attention(
            torch.from_numpy(q).permute(1, 0, 2).unsqueeze(0),
            torch.from_numpy(K).permute(1, 0, 2).unsqueeze(0),
            torch.from_numpy(V).permute(1, 0, 2).unsqueeze(0),
            is_causal=True, scale=scale, enable_gqa=(Hq != Hkv))[0]
        for h in range(Hq):
            np.testing.assert_allclose(got[(0, h)], ref[h].numpy(), rtol=1e-10, atol=1e-12)


def check_prefill_equals_decode(att, seed=2):
    """Prefill row i of a chunk appended after P tokens == decode over the first P+i+1 tokens."""
    Hq, Hkv, D, bs = 4, 2, 32, 16
    P, C = 45, 20
    L = P + C
    q, kc, vc, tables, lens, Ks, Vs = _paged_case(seed, 1, Hq, Hkv, D, bs, [L])
    rng = _rng(seed + 100)
    qc = rng.standard_normal((C, Hq, D))
    scale = 0.17
    got = att.prefill_attention(qc, [0, C], kc, vc, tables, [L], scale)
    for i in range(C):
        dec = att.decode_attention(qc[i][None], kc, vc, tables, [P + i + 1], scale)[0]
        for h in range(Hq):
            np.testing.assert_allclose(got[(0, h)][i], dec[h], rtol=1e-11, atol=1e-13)


def check_closed_forms(att, seed=3):
    """Closed forms: one key -> V_0 exactly; q = 0 -> mean of V; constant V -> that constant;
    identical keys -> mean of V."""
    Hq, Hkv, D, bs = 4, 2, 16, 16
    q, kc, vc, tables, lens, Ks, Vs = _paged_case(seed, 3, Hq, Hkv, D, bs, [1, 40, 23])
    scale = 0.25
    out = att.decode_attention(q, kc, vc, tables, lens, scale)
    G = Hq // Hkv
    for h in range(Hq):
        np.testing.assert_array_equal(out[0, h], Vs[0][0, h // G])
    q0 = np.zeros_like(q)
    out0 = att.decode_attention(q0, kc, vc, tables, lens, scale)
    for b in range(3):
        for h in range(Hq):
            np.testing.assert_allclose(out0[b, h], Vs[b][:, h // G].mean(axis=0), rtol=1e-12, atol=1e-12)
    # constant V and identical K rows, written through the block table
    rng = _rng(seed + 7)
    L = 37
    c = rng.standard_normal(D)
    krow = rng.standard_normal(D)
    NB = 6
    table = [4, 1, 5]
    kc2 = scatter_dense(np.tile(krow, (L, Hkv, 1)), table, bs, NB, rng)
    vc2 = scatter_dense(np.tile(c, (L, Hkv, 1)), table, bs, NB, rng)
    Vrand = rng.standard_normal((L, Hkv, D))
    vc3 = scatter_dense(Vrand, table, bs, NB, rng)
    qq = rng.standard_normal((1, Hq, D))
    o2 = att.decode_attention(qq, kc2, vc2, [table], [L], scale)
    o3 = att.decode_attention(qq, kc2, vc3, [table], [L], scale)
    for h in range(Hq):
        np.testing.assert_allclose(o2[0, h], c, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(o3[0, h], Vrand[:, h // G].mean(axis=0), rtol=1e-12, atol=1e-12)


def check_brute_twin(att, seed=4):
    """numpy oracle == scalar pure-Python twin on tiny random cases (decode and prefill, all block sizes)."""
    rng = _rng(seed)
    for bs in (16, 32, 64, 128, 256):
        for (Hq, Hkv) in ((2, 2), (4, 2), (4, 1)):
            D = 8
            lens = [int(x) for x in rng.integers(1, 70, size=3)]
            q, kc, vc, tables, lens, _, _ = _paged_case(int(rng.integers(1 << 30)), 3, Hq, Hkv, D, bs, lens)
            scale = 1.0 / math.sqrt(D)
            got = att.decode_attention(q, kc, vc, tables, lens, scale)
            ref = brute.decode(q.tolist(), kc.tolist(), vc.tolist(), [list(map(int, t)) for t in tables], lens, scale)
            np.testing.assert_allclose(got, np.array(ref), rtol=1e-10, atol=1e-12)
            # prefill: last C tokens of each sequence are the chunk
            Cs = [max(1, L // 3) for L in lens]
            qsl = [0]
            for C in Cs:
                qsl.append(qsl[-1] + C)
            qp = rng.standard_normal((qsl[-1], Hq, D))
            gotp = att.prefill_attention(qp, qsl, kc, vc, tables, lens, scale)
            refp = brute.prefill(qp.tolist(), qsl, kc.tolist(), vc.tolist(), [list(map(int, t)) for t in tables], lens, scale)
            for b in range(3):
                for h in range(Hq):
                    np.testing.assert_allclose(gotp[(b, h)], np.array([refp[qsl[b] + i][h] for i in range(Cs[b])]),
                                               rtol=1e-10, atol=1e-12)


def check_permutation_and_sharing(att, seed=5):
    """Invariant under any permutation of physical blocks, and under shared vs copied prefix blocks."""
    Hq, Hkv, D, bs = 4, 2, 16, 16
    rng = _rng(seed)
    P, S1, S2 = 48, 13, 30             # prefix of 3 full blocks, two private suffixes
    pre_k = rng.standard_normal((P, Hkv, D))
    pre_v = rng.standard_normal((P, Hkv, D))
    suf = [(rng.standard_normal((S, Hkv, D)), rng.standard_normal((S, Hkv, D))) for S in (S1, S2)]
    q = rng.standard_normal((2, Hq, D))
    scale = 0.3
    outs = []
    for shared in (True, False):
        for trial in range(3):
            NB = 16
            perm = list(rng.permutation(NB))
            kc = rng.standard_normal((NB, bs, Hkv, D))
            vc = rng.standard_normal((NB, bs, Hkv, D))
            pre_blocks = perm[:3]
            tables = []
            nxt = 3
            for b in range(2):
                if shared:
                    blocks = list(pre_blocks)
                else:
                    blocks = perm[nxt:nxt + 3]
                    nxt += 3
                for j in range(3):
                    kc[blocks[j]] = pre_k[j * bs:(j + 1) * bs]
                    vc[blocks[j]] = pre_v[j * bs:(j + 1) * bs]
                sk, sv = suf[b]
                for j in range(-(-sk.shape[0] // bs)):
                    blk = perm[nxt]
                    nxt += 1
                    kc[blk, : sk[j * bs:(j + 1) * bs].shape[0]] = sk[j * bs:(j + 1) * bs]
                    vc[blk, : sv[j * bs:(j + 1) * bs].shape[0]] = sv[j * bs:(j + 1) * bs]
                    blocks.append(blk)
                tables.append(blocks + [-1] * (6 - len(blocks)))
            outs.append(att.decode_attention(q, kc, vc, tables, [P + S1, P + S2], scale))
    for o in outs[1:]:
        np.testing.assert_allclose(o, outs[0], rtol=1e-12, atol=1e-13)
    # and it equals dense attention over the concatenated sequence
    for b in range(2):
        K = np.concatenate([pre_k, suf[b][0]])
        V = np.concatenate([pre_v, suf[b][1]])
        ref = F.scaled_dot_product_attention(torch.from_numpy(q[b]).view(1, Hq, 1, D),
                                             torch.from_numpy(K).permute(1, 0, 2).unsqueeze(0),
                                             torch.from_numpy(V).permute(1, 0, 2).unsqueeze(0),
                                             scale=scale, enable_gqa=True)
        np.testing.assert_allclose(outs[0][b], ref[0, :, 0].numpy(), rtol=1e-10, atol=1e-12)


def check_split_merge(att, seed=6):
    """Merging per-split (m, l, o) with the log-sum-exp rule reproduces the full softmax."""
    rng = _rng(seed)
    L, D = 300, 32
    K = rng.standard_normal((L, D)) * 3
    V = rng.standard_normal((L, D))
    q = rng.standard_normal(D) * 2
    for S in (1, 7, 64, 128, 299, 300, 512):
        m, l, o = att.split_partials(q, K, V, 0.2, S)
        M = m.max()
        w = np.exp(m - M)
        merged = (w[:, None] * o).sum(0) / (w * l).sum()
        x = 0.2 * K @ q
        p = np.exp(x - x.max())
        np.testing.assert_allclose(merged, (p / p.sum()) @ V, rtol=1e-11, atol=1e-13)


def check_large_logits(att, seed=7):
    """q scaled x10 (large logits, the overflow case that moved softmax out of fp16) stays finite and
    matches the scalar twin."""
    Hq, Hkv, D, bs = 2, 1, 64, 16
    q, kc, vc, tables, lens, _, _ = _paged_case(seed, 2, Hq, Hkv, D, bs, [40, 64])
    q = q * 10
    got = att.decode_attention(q, kc, vc, tables, lens, 1 / 8)
    assert np.isfinite(got).all()
    ref = brute.decode(q.tolist(), kc.tolist(), vc.tolist(), [list(map(int, t)) for t in tables], lens, 1 / 8)
    np.testing.assert_allclose(got, np.array(ref), rtol=1e-9, atol=1e-11)


ALL_CHECKS = [check_sdpa_decode, check_sdpa_prefill_no_prefix, check_prefill_equals_decode, check_closed_forms,
              check_brute_twin, check_permutation_and_sharing, check_split_merge, check_large_logits]
