"""Scalar pure-Python twin of the attention oracle, for tiny cases (test infrastructure only).

It walks the block table token by token and uses only ``math.exp`` and plain
loops, so it shares no code path with the numpy version in ``attention.py``.
Same definition: page "Nano-vLLM-Ascend: lightweight LLM inference framework
for Ascend NPU", sections 2.1 (block table) and 2.2.1 (softmax(q k^T / sqrt(d)) v).
"""

from __future__ import annotations

import math


def _row(cache, block_table_row, bs, t, g):
    blk = block_table_row[t // bs]
    return cache[blk][t % bs][g]


def attend_one(q, cache_k, cache_v, block_table_row, bs, n_keys, g, scale):
    """softmax over keys 0..n_keys-1 of KV head g for one query vector (lists of floats)."""
    if n_keys == 0:
        return [0.0] * len(q)
    scores = []
    for t in range(n_keys):
        k = _row(cache_k, block_table_row, bs, t, g)
        scores.append(scale * sum(qi * ki for qi, ki in zip(q, k)))
    m = max(scores)
    w = [math.exp(s - m) for s in scores]
    z = sum(w)
    out = [0.0] * len(q)
    for t in range(n_keys):
        v = _row(cache_v, block_table_row, bs, t, g)
        for d in range(len(q)):
            out[d] += w[t] / z * v[d]
    return out


def decode(q, cache_k, cache_v, block_tables, context_lens, scale):
    """q: nested lists [B][Hq][D]; caches nested [NB][bs][Hkv][D]; returns [B][Hq][D]."""
    bs = len(cache_k[0])
    Hkv = len(cache_k[0][0])
    out = []
    for b, qb in enumerate(q):
        G = len(qb) // Hkv
        out.append([attend_one(qb[h], cache_k, cache_v, block_tables[b], bs, context_lens[b], h // G, scale)
                    for h in range(len(qb))])
    return out


def prefill(q, query_start_loc, cache_k, cache_v, block_tables, context_lens, scale):
    """q nested [sum C][Hq][D]; returns nested [sum C][Hq][D]."""
    bs = len(cache_k[0])
    Hkv = len(cache_k[0][0])
    out = [None] * len(q)
    for b in range(len(query_start_loc) - 1):
        C = query_start_loc[b + 1] - query_start_loc[b]
        L = context_lens[b]
        for i in range(C):
            row = query_start_loc[b] + i
            G = len(q[row]) // Hkv
            out[row] = [attend_one(q[row][h], cache_k, cache_v, block_tables[b], bs, L - C + i + 1, h // G, scale)
                        for h in range(len(q[row]))]
    return out
