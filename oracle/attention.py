"""Paged attention in float64 (oracle; test infrastructure only).

Definition (page "Nano-vLLM-Ascend: lightweight LLM inference framework for
Ascend NPU", section 2.2.1, the unfused form ``softmax(q @ k.T / sqrt(d)) @ v``,
and section 4.2, which names the 1/sqrt(d) scaling factor):

1. Gather: logical token t of sequence b lives in physical block
   ``block_table[b][t // block_size]`` at row ``t % block_size`` (section 2.1,
   BlockTable's logical-to-physical map over the Block layout).
2. Query head h reads KV head ``h // G`` with ``G = Hq / Hkv`` (the pages do not
   state a grouping; consecutive grouping is the reading taken here).
3. ``s_t = scale * <q_h, K_t>``; ``p = exp(s - max s) / sum exp(s - max s)``;
   ``out_h = sum_t p_t V_t``.  All in float64 (page "Ascend NPU LLM inference
   optimisation: the vLLM-Ascend approach", section 3.1, takes softmax out of
   fp16 to stop rare wrong outputs; fp64 is at least that).
4. Chunked prefill (page "In-depth analysis of vllm-ascend", section 1.1, PCP:
   prefill cut into chunks on one device): query i of a chunk of C tokens
   appended to a sequence that now holds L tokens sits at position L - C + i
   and attends to keys 0 .. L - C + i.

Inputs are the exact fp16/bf16 values the GPU sees, upcast to float64.
"""

from __future__ import annotations

import numpy as np


def to_f64(x) -> np.ndarray:
    """torch tensor (any float dtype) or numpy array -> float64 numpy array."""
    if hasattr(x, "detach"):
        return x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def gather_kv(cache: np.ndarray, block_table_row, context_len: int) -> np.ndarray:
    """Dense [L, Hkv, D] rows of one sequence, in logical token order."""
    bs = cache.shape[1]
    t = np.arange(context_len)
    phys = np.asarray(block_table_row, dtype=np.int64)[t // bs]
    return cache[phys, t % bs]


def attend(q_heads: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """One query token: q_heads [Hq, D], K/V [L, Hkv, D] -> out [Hq, D] (zeros when L == 0)."""
    Hq, D = q_heads.shape
    L, Hkv, _ = K.shape
    G = Hq // Hkv
    out = np.zeros((Hq, D))
    if L == 0:
        return out
    for h in range(Hq):
        g = h // G
        s = scale * (K[:, g, :] @ q_heads[h])
        p = np.exp(s - s.max())
        out[h] = (p / p.sum()) @ V[:, g, :]
    return out


def decode_attention(q, k_cache, v_cache, block_tables, context_lens, scale: float) -> np.ndarray:
    """Single-token decode for a batch: q [B, Hq, D] -> out [B, Hq, D] (float64)."""
    q = to_f64(q)
    kc = to_f64(k_cache)
    vc = to_f64(v_cache)
    scale = float(scale)
    out = np.zeros(q.shape)
    for b in range(q.shape[0]):
        L = int(context_lens[b])
        K = gather_kv(kc, block_tables[b], L)
        V = gather_kv(vc, block_tables[b], L)
        out[b] = attend(q[b], K, V, scale)
    return out


def decode_rows(q, k_cache, v_cache, block_tables, context_lens, scale: float, rows) -> np.ndarray:
    """Decode output for selected (b, h) pairs only, without materialising the whole cache in fp64."""
    res = []
    bs = k_cache.shape[1]
    Hq = q.shape[1]
    Hkv = k_cache.shape[2]
    G = Hq // Hkv
    for b, h in rows:
        L = int(context_lens[b])
        g = h // G
        t = np.arange(L)
        phys = np.asarray(block_tables[b], dtype=np.int64)[t // bs]
        K = k_cache[phys, t % bs, g].double().numpy() if hasattr(k_cache, "double") else np.asarray(k_cache[phys, t % bs, g], np.float64)
        V = v_cache[phys, t % bs, g].double().numpy() if hasattr(v_cache, "double") else np.asarray(v_cache[phys, t % bs, g], np.float64)
        qh = to_f64(q[b, h])
        if L == 0:
            res.append(np.zeros(qh.shape))
            continue
        s = float(scale) * (K @ qh)
        p = np.exp(s - s.max())
        res.append((p / p.sum()) @ V)
    return np.stack(res)


def prefill_attention(q, query_start_loc, k_cache, v_cache, block_tables, context_lens, scale: float,
                      seqs=None, heads=None) -> dict:
    """Causal chunked prefill over the paged context.

    q [sum C, Hq, D]; sequence b owns q rows query_start_loc[b] .. query_start_loc[b+1]-1.
    Returns {(b, h): out [C_b, D]} for the requested sequences and heads (all by default).
    """
    qsl = [int(x) for x in query_start_loc]
    Hq = q.shape[1]
    Hkv = k_cache.shape[2]
    G = Hq // Hkv
    bs = k_cache.shape[1]
    seqs = range(len(qsl) - 1) if seqs is None else seqs
    heads = range(Hq) if heads is None else heads
    res = {}
    for b in seqs:
        C = qsl[b + 1] - qsl[b]
        L = int(context_lens[b])
        t = np.arange(L)
        phys = np.asarray(block_tables[b], dtype=np.int64)[t // bs]
        for h in heads:
            g = h // G
            K = to_f64(k_cache[phys, t % bs, g])
            V = to_f64(v_cache[phys, t % bs, g])
            Q = to_f64(q[qsl[b]:qsl[b + 1], h])
            out = np.zeros((C, Q.shape[1]))
            for i in range(C):
                last = L - C + i          # position of query i; keys 0..last are visible
                s = float(scale) * (K[: last + 1] @ Q[i])
                p = np.exp(s - s.max())
                out[i] = (p / p.sum()) @ V[: last + 1]
            res[(b, h)] = out
    return res


def split_partials(q_head: np.ndarray, K_g: np.ndarray, V_g: np.ndarray, scale: float, split_len: int):
    """Per-split softmax statistics of one query head over contiguous token ranges of ``split_len``.

    For split s covering tokens [s*S, min(L, (s+1)*S)): m_s = max_t x_t, l_s = sum_t e^(x_t - m_s),
    o_s = sum_t e^(x_t - m_s) V_t, with x_t = scale * <q, K_t>.  Merging them,
    out = sum_s e^(m_s - M) o_s / sum_s e^(m_s - M) l_s with M = max_s m_s, is the full softmax
    (single-device reading of the context split on the vllm-ascend page, section 3.1).
    """
    L = K_g.shape[0]
    ms, ls, os_ = [], [], []
    for s0 in range(0, L, split_len):
        x = scale * (K_g[s0:s0 + split_len] @ q_head)
        m = x.max()
        e = np.exp(x - m)
        ms.append(m)
        ls.append(e.sum())
        os_.append(e @ V_g[s0:s0 + split_len])
    return np.array(ms), np.array(ls), np.array(os_)
