"""Decode with each sequence's context split across devices (oracle; test infrastructure only).

Page "In-depth analysis of vllm-ascend: LLM inference architecture on Ascend
hardware", sections 1.1 and 3.1: in the DCP mode the KV cache of a long
sequence is spread over several devices, each device computes attention over
the part it holds, the intermediate results are gathered from every device
(a global AllGather) and combined.  The pages give neither the split rule nor
the combination; the readings taken here:

* Split (reading): block-interleaved.  Logical block j of every sequence (its
  tokens j*bs .. j*bs + bs - 1) lives on rank j mod W.  Every rank's share
  then differs by at most one block, and a token appended at position p goes
  to rank (p // bs) mod W, so shares stay balanced as sequences grow.
* Intermediate result of rank r for (sequence, query head): its attention
  output over the tokens it holds, normalised over those tokens only, and the
  log-sum-exp of their scores, lse_r = ln sum_{t on r} exp(s_t)  (lse = -inf
  and output 0 when the rank holds no token of the sequence).
* Combination: out = sum_r exp(lse_r - M) o_r / sum_r exp(lse_r - M) with
  M = max_r lse_r; this is the softmax over all tokens (exp(lse_r) o_r is rank
  r's unnormalised sum).  All ranks' parts empty gives out = 0.
"""

from __future__ import annotations

import numpy as np

from .attention import gather_kv, to_f64


def shard_positions(context_len: int, block_size: int, world: int, rank: int) -> np.ndarray:
    """Logical token positions of one sequence that rank `rank` holds, in increasing order."""
    t = np.arange(int(context_len))
    return t[(t // block_size) % world == rank]


def local_len(context_len: int, block_size: int, world: int, rank: int) -> int:
    return int(shard_positions(context_len, block_size, world, rank).shape[0])


def attend_lse(q_heads: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float):
    """One query token over the rows K/V [n, Hkv, D]: (out [Hq, D] normalised over these rows, lse [Hq])."""
    Hq, D = q_heads.shape
    n, Hkv, _ = K.shape
    G = Hq // Hkv
    out = np.zeros((Hq, D))
    lse = np.full(Hq, -np.inf)
    if n == 0:
        return out, lse
    for h in range(Hq):
        g = h // G
        s = scale * (K[:, g, :] @ q_heads[h])
        mx = s.max()
        e = np.exp(s - mx)
        out[h] = (e / e.sum()) @ V[:, g, :]
        lse[h] = mx + np.log(e.sum())
    return out, lse


def shard_partials(q, k_cache, v_cache, block_tables, context_lens, scale: float, world: int, rank: int):
    """Rank `rank`'s intermediate results for a batch whose caches are given whole (global block tables):
    (outs [B, Hq, D], lses [B, Hq]) over the tokens the split rule gives that rank."""
    q = to_f64(q)
    kc, vc = to_f64(k_cache), to_f64(v_cache)
    bs = kc.shape[1]
    B = q.shape[0]
    outs = np.zeros(q.shape)
    lses = np.full(q.shape[:2], -np.inf)
    for b in range(B):
        L = int(context_lens[b])
        pos = shard_positions(L, bs, world, rank)
        K = gather_kv(kc, block_tables[b], L)[pos]
        V = gather_kv(vc, block_tables[b], L)[pos]
        outs[b], lses[b] = attend_lse(q[b], K, V, float(scale))
    return outs, lses


def merge_states(outs, lses) -> np.ndarray:
    """outs [P, ..., D], lses [P, ...] -> the combined output [..., D] (zeros where every part is empty)."""
    outs = np.asarray(outs, dtype=np.float64)
    lses = np.asarray(lses, dtype=np.float64)
    M = lses.max(axis=0)
    finite = np.isfinite(M)
    Ms = np.where(finite, M, 0.0)
    w = np.where(np.isfinite(lses), np.exp(lses - Ms[None]), 0.0)
    den = w.sum(axis=0)
    num = (w[..., None] * outs).sum(axis=0)
    res = np.zeros(num.shape)
    res[finite] = num[finite] / den[finite][..., None]
    return res
