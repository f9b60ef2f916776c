"""Seeded workload generator (inputs only; no attention or slot arithmetic).

Every workload is a list of block-pool operations plus dense random tensors:

* ``ops``: the order in which sequences are created, forked and extended.
  Both the oracle's pool and the C++ pool replay the same list and must hand
  out the same physical blocks, because both are given the same
  ``free_order`` (the order of the free list at pool creation).  A random
  ``free_order`` is what scatters each sequence's blocks across the pool.
* ``append_new`` entries mark the tokens whose K/V are written this step
  (one per sequence for decode, a whole chunk for chunked prefill); the rows
  of ``k_new``/``v_new`` follow the order of those entries.
* ``k_cache0``/``v_cache0``: the pool's contents before the write, drawn
  N(0,1) everywhere (used and free blocks alike), so a gather that strays into
  a wrong block changes the result.

Workload shapes follow the pages' own workloads: Qwen3-0.6B-shaped heads with
random lengths 100..1024 (page "Nano-vLLM-Ascend: lightweight LLM inference
framework for Ascend NPU", section 3.2.1 batching), Llama-2-70B-shaped heads
with 8k-token contexts and shared prefixes (page "Ascend NPU LLM inference
optimisation: the vLLM-Ascend approach", section 4 deployment results), and
chunked prefill (page "In-depth analysis of vllm-ascend", section 1.1 PCP).
"""

from __future__ import annotations

import dataclasses
import math
from typing import Any

import numpy as np
import torch

# name -> parameters.  Lengths are inclusive ranges; context_lens counts the
# token written in this step (it is attended to by the decode that follows).
CONFIGS: dict[str, dict[str, Any]] = {
    "tiny": dict(kind="decode", batch=4, num_q_heads=4, num_kv_heads=4, head_dim=64,
                 block_size=16, dtype="f16", len_lo=1, len_hi=64, num_blocks=64, seed=0),
    "qwen_decode": dict(kind="decode", batch=128, num_q_heads=16, num_kv_heads=8, head_dim=128,
                        block_size=16, dtype="bf16", len_lo=100, len_hi=1024, free_frac=0.10, seed=1),
    "llama70b_long": dict(kind="decode", batch=64, num_q_heads=64, num_kv_heads=8, head_dim=128,
                          block_size=16, dtype="bf16", len_lo=4096, len_hi=8192, free_frac=0.10, seed=2),
    "prefix_sweep": dict(kind="prefix", batch=256, groups=8, prefix_len=2048, suffix_lo=0, suffix_hi=512,
                         num_q_heads=16, num_kv_heads=8, head_dim=128, block_size=16, dtype="bf16",
                         free_frac=0.10, seed=3),
    "prefill": dict(kind="prefill", batch=8, chunk_len=512, ctx_len=8192, num_q_heads=32, num_kv_heads=8,
                    head_dim=128, block_size=16, dtype="bf16", free_frac=0.10, seed=4),
}

TORCH_DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16}


@dataclasses.dataclass
class Workload:
    name: str
    cfg: dict
    ops: list                    # pool operations, replayed by both sides
    free_order: np.ndarray       # int32 [num_blocks], initial free-list order
    num_blocks: int
    context_lens: np.ndarray     # int32 [batch], tokens per sequence after this step's write
    q: torch.Tensor              # [batch, Hq, D] (decode) or [sum C, Hq, D] (prefill)
    k_new: torch.Tensor          # [T, Hkv, D] rows written this step
    v_new: torch.Tensor
    k_cache0: torch.Tensor       # [num_blocks, block_size, Hkv, D] pool contents before the write
    v_cache0: torch.Tensor
    query_start_loc: np.ndarray | None  # int32 [batch+1] (prefill only)
    scale: float                 # softmax scale, fp32 value of 1/sqrt(head_dim)

    @property
    def batch(self) -> int:
        return int(self.cfg["batch"])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if len(self.context_lens) else 0


def _randn(g: torch.Generator, shape, dtype, chunk_elems: int = 1 << 26) -> torch.Tensor:
    """N(0,1) draws in fp32, rounded to ``dtype`` (round-to-nearest-even), drawn in chunks."""
    n = int(np.prod(shape))
    out = torch.empty(n, dtype=dtype)
    for s in range(0, n, chunk_elems):
        e = min(n, s + chunk_elems)
        out[s:e] = torch.randn(e - s, generator=g, dtype=torch.float32).to(dtype)
    return out.view(*shape)


def ops_for(cfg: dict, lens_before: np.ndarray, new_tokens: np.ndarray, suffix: np.ndarray | None = None):
    """Pool-operation script for a config: which sequence is created, forked or extended, in order."""
    ops = []
    kind = cfg["kind"]
    B = cfg["batch"]
    if kind in ("decode", "prefill"):
        for b in range(B):
            ops.append(("alloc", b, int(lens_before[b])))
        for b in range(B):
            ops.append(("append_new", b, int(new_tokens[b])))
    elif kind == "prefix":
        per = B // cfg["groups"]
        P = cfg["prefix_len"]
        for grp in range(cfg["groups"]):
            first = grp * per
            ops.append(("alloc", first, P))
            for m in range(first + 1, first + per):
                ops.append(("fork", first, m, P))
        for b in range(B):
            if suffix[b] > 0:
                ops.append(("append", b, int(suffix[b])))
        for b in range(B):
            ops.append(("append_new", b, 1))
    else:
        raise ValueError(kind)
    return ops


def make_workload(name: str, *, seed: int | None = None, block_size: int | None = None,
                  q_scale: float = 1.0, **overrides) -> Workload:
    """Build a workload by name.  ``block_size`` overrides the config (prefix sweep);
    ``q_scale`` multiplies q (large-logit stress case); ``overrides`` replace config keys."""
    cfg = dict(CONFIGS[name])
    cfg.update(overrides)
    if block_size is not None:
        cfg["block_size"] = block_size
    if seed is None:
        seed = cfg["seed"]
    g = torch.Generator().manual_seed(int(seed))
    B, Hq, Hkv, D, bs = cfg["batch"], cfg["num_q_heads"], cfg["num_kv_heads"], cfg["head_dim"], cfg["block_size"]
    dt = TORCH_DTYPES[cfg["dtype"]]
    kind = cfg["kind"]
    suffix = None
    qsl = None
    if kind == "decode":
        L = torch.randint(cfg["len_lo"], cfg["len_hi"] + 1, (B,), generator=g).numpy().astype(np.int32)
        new = np.ones(B, dtype=np.int32)
        unique_tokens = int(L.sum())
    elif kind == "prefix":
        suffix = torch.randint(cfg["suffix_lo"], cfg["suffix_hi"] + 1, (B,), generator=g).numpy().astype(np.int32)
        L = (cfg["prefix_len"] + suffix + 1).astype(np.int32)
        new = np.ones(B, dtype=np.int32)
        unique_tokens = int(cfg["groups"] * cfg["prefix_len"] + (suffix + 1).sum())
    elif kind == "prefill":
        C = cfg["chunk_len"]
        L = np.full(B, cfg["ctx_len"] + C, dtype=np.int32)
        new = np.full(B, C, dtype=np.int32)
        unique_tokens = int(L.sum())
        qsl = np.zeros(B + 1, dtype=np.int32)
        qsl[1:] = np.cumsum(new)
    else:
        raise ValueError(kind)
    lens_before = (L - new).astype(np.int32)
    if "num_blocks" in cfg:
        NB = int(cfg["num_blocks"])
    else:
        # room for every token, one partial block per sequence, plus the free share
        NB = int(math.ceil((unique_tokens / bs + B) * (1.0 + cfg["free_frac"])))
    free_order = torch.randperm(NB, generator=g).numpy().astype(np.int32)
    T = int(new.sum())
    nq = B if kind != "prefill" else T
    q = _randn(g, (nq, Hq, D), dt)
    if q_scale != 1.0:
        q = (q.float() * q_scale).to(dt)
    k_new = _randn(g, (T, Hkv, D), dt)
    v_new = _randn(g, (T, Hkv, D), dt)
    k_cache0 = _randn(g, (NB, bs, Hkv, D), dt)
    v_cache0 = _randn(g, (NB, bs, Hkv, D), dt)
    ops = ops_for(cfg, lens_before, new, suffix)
    scale = float(np.float32(1.0) / np.sqrt(np.float32(D)))
    return Workload(name=name, cfg=cfg, ops=ops, free_order=free_order, num_blocks=NB, context_lens=L,
                    q=q, k_new=k_new, v_new=v_new, k_cache0=k_cache0, v_cache0=v_cache0,
                    query_start_loc=qsl, scale=scale)


def fill_cache_blocks(shape, dtype: str, seed: int) -> torch.Tensor:
    """A standalone N(0,1) cache tensor (used by tests that need a fresh pool)."""
    g = torch.Generator().manual_seed(int(seed))
    return _randn(g, shape, TORCH_DTYPES[dtype])


def make_custom(*, seed: int, lens, num_q_heads: int, num_kv_heads: int, head_dim: int, block_size: int,
                dtype: str = "bf16", kind: str = "decode", chunk_lens=None, free_frac: float = 0.25,
                q_scale: float = 1.0) -> Workload:
    """A small workload with explicit per-sequence lengths (ragged edge cases).

    kind="decode": ``lens`` are context lengths after the write (0 allowed: that sequence writes nothing).
    kind="prefill": ``lens`` are the final lengths and ``chunk_lens`` the chunk appended to each.
    """
    g = torch.Generator().manual_seed(int(seed))
    L = np.asarray(lens, dtype=np.int32)
    B = len(L)
    if kind == "decode":
        new = (L > 0).astype(np.int32)
    else:
        new = np.asarray(chunk_lens, dtype=np.int32)
    before = (L - new).astype(np.int32)
    NB = int(math.ceil((int(L.sum()) / block_size + B + 1) * (1.0 + free_frac)))
    free_order = torch.randperm(NB, generator=g).numpy().astype(np.int32)
    T = int(new.sum())
    dt = TORCH_DTYPES[dtype]
    nq = B if kind == "decode" else T
    q = _randn(g, (nq, num_q_heads, head_dim), dt)
    if q_scale != 1.0:
        q = (q.float() * q_scale).to(dt)
    k_new = _randn(g, (T, num_kv_heads, head_dim), dt)
    v_new = _randn(g, (T, num_kv_heads, head_dim), dt)
    k_cache0 = _randn(g, (NB, block_size, num_kv_heads, head_dim), dt)
    v_cache0 = _randn(g, (NB, block_size, num_kv_heads, head_dim), dt)
    ops = [("alloc", b, int(before[b])) for b in range(B)]
    ops += [("append_new", b, int(new[b])) for b in range(B) if new[b] > 0]
    qsl = None
    if kind == "prefill":
        qsl = np.zeros(B + 1, dtype=np.int32)
        qsl[1:] = np.cumsum(new)
    cfg = dict(kind=kind, batch=B, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads, head_dim=head_dim,
               block_size=block_size, dtype=dtype, seed=seed)
    scale = float(np.float32(1.0) / np.sqrt(np.float32(head_dim)))
    return Workload(name="custom", cfg=cfg, ops=ops, free_order=free_order, num_blocks=NB, context_lens=L, q=q,
                    k_new=k_new, v_new=v_new, k_cache0=k_cache0, v_cache0=v_cache0, query_start_loc=qsl,
                    scale=scale)


def make_prefix_groups(*, seed: int, group_sizes, prefix_lens, suffix_lo: int, suffix_hi: int, num_q_heads: int,
                       num_kv_heads: int, head_dim: int, block_size: int, dtype: str = "bf16",
                       free_frac: float = 0.2) -> Workload:
    """Groups of sequences forked from one parent each (the parent is the group's first sequence): group i has
    group_sizes[i] members sharing its first prefix_lens[i] tokens, then every member appends a private
    suffix of uniform[suffix_lo, suffix_hi] tokens and one new token.  Members of a group are consecutive
    in the batch.  ``cfg`` carries "group_sizes" and "prefix_lens" for the caller."""
    g = torch.Generator().manual_seed(int(seed))
    sizes = [int(x) for x in group_sizes]
    plens = [int(x) for x in prefix_lens]
    B = sum(sizes)
    suffix = torch.randint(suffix_lo, suffix_hi + 1, (B,), generator=g).numpy().astype(np.int32)
    ops, first = [], 0
    prefix_of = np.zeros(B, dtype=np.int32)
    for n, P in zip(sizes, plens):
        ops.append(("alloc", first, P))
        for m in range(first + 1, first + n):
            ops.append(("fork", first, m, P))
        prefix_of[first:first + n] = P
        first += n
    for b in range(B):
        if suffix[b] > 0:
            ops.append(("append", b, int(suffix[b])))
    for b in range(B):
        ops.append(("append_new", b, 1))
    L = (prefix_of + suffix + 1).astype(np.int32)
    unique = sum(plens) + int((suffix + 1).sum())
    NB = int(math.ceil((unique / block_size + 2 * B) * (1.0 + free_frac)))
    free_order = torch.randperm(NB, generator=g).numpy().astype(np.int32)
    dt = TORCH_DTYPES[dtype]
    q = _randn(g, (B, num_q_heads, head_dim), dt)
    k_new = _randn(g, (B, num_kv_heads, head_dim), dt)
    v_new = _randn(g, (B, num_kv_heads, head_dim), dt)
    k_cache0 = _randn(g, (NB, block_size, num_kv_heads, head_dim), dt)
    v_cache0 = _randn(g, (NB, block_size, num_kv_heads, head_dim), dt)
    cfg = dict(kind="prefix_groups", batch=B, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads, head_dim=head_dim,
               block_size=block_size, dtype=dtype, seed=seed, group_sizes=sizes, prefix_lens=plens)
    scale = float(np.float32(1.0) / np.sqrt(np.float32(head_dim)))
    return Workload(name="prefix_groups", cfg=cfg, ops=ops, free_order=free_order, num_blocks=NB, context_lens=L,
                    q=q, k_new=k_new, v_new=v_new, k_cache0=k_cache0, v_cache0=v_cache0, query_start_loc=None,
                    scale=scale)


def new_token_positions(wl: Workload) -> np.ndarray:
    """int64 [T]: the index within its sequence of every token written this step, in the order of the
    ``append_new`` entries (the row order of k_new/v_new).  Pool-script bookkeeping only."""
    length: dict[int, int] = {}
    out = []
    for op in wl.ops:
        if op[0] == "alloc":
            length[op[1]] = op[2]
        elif op[0] == "fork":
            length[op[2]] = op[3]
        elif op[0] == "append":
            length[op[1]] += op[2]
        elif op[0] == "append_new":
            b, n = op[1], op[2]
            out.extend(range(length[b], length[b] + n))
            length[b] += n
    return np.asarray(out, dtype=np.int64)


def rope_tables(max_position: int, head_dim: int, base: float = 10000.0):
    """fp32 cos/sin tables [max_position, head_dim/2] of the usual rotary frequency schedule,
    angle(p, i) = p * base^(-2i/head_dim), evaluated in float64 and rounded to fp32.  The tables are data
    handed to the rotary operator (it receives cos and sin, not a schedule)."""
    inv = base ** (-np.arange(0, head_dim, 2, dtype=np.float64) / head_dim)
    ang = np.outer(np.arange(max_position, dtype=np.float64), inv)
    return torch.from_numpy(np.cos(ang).astype(np.float32)), torch.from_numpy(np.sin(ang).astype(np.float32))


@dataclasses.dataclass
class RopeCase:
    q: torch.Tensor              # [T, Hq, D]
    k: torch.Tensor              # [T, Hkv, D]
    v: torch.Tensor
    positions: torch.Tensor      # int64 [T]
    cos: torch.Tensor            # fp32 [max_position, D/2]
    sin: torch.Tensor
    slots: torch.Tensor          # int64 [T], distinct, -1 = no cache write
    k_cache0: torch.Tensor       # [NB, bs, Hkv, D]
    v_cache0: torch.Tensor


def make_rope_case(*, seed: int, num_tokens: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                   block_size: int, num_blocks: int, dtype: str = "bf16", max_position: int = 4096,
                   skip_frac: float = 0.1, random_angles: bool = False) -> RopeCase:
    """A standalone rotary + cache-write case: N(0,1) q/k/v and caches, positions uniform in
    [0, max_position) with the first and last table rows always used (when T >= 2), distinct random slots
    of the pool with a ``skip_frac`` share set to -1.  ``random_angles`` draws every table angle uniformly
    in [-pi, pi) instead of the frequency schedule."""
    g = torch.Generator().manual_seed(int(seed))
    dt = TORCH_DTYPES[dtype]
    T = int(num_tokens)
    q = _randn(g, (T, num_q_heads, head_dim), dt)
    k = _randn(g, (T, num_kv_heads, head_dim), dt)
    v = _randn(g, (T, num_kv_heads, head_dim), dt)
    pos = torch.randint(0, max_position, (T,), generator=g, dtype=torch.int64)
    if T >= 2:
        pos[0], pos[-1] = 0, max_position - 1
    nslots = num_blocks * block_size
    assert T <= nslots
    slots = torch.randperm(nslots, generator=g)[:T].to(torch.int64)
    skip = torch.rand(T, generator=g) < skip_frac
    slots[skip] = -1
    if random_angles:
        ang = (torch.rand((max_position, head_dim // 2), generator=g, dtype=torch.float64) * 2 - 1) * math.pi
        cos, sin = torch.cos(ang).to(torch.float32), torch.sin(ang).to(torch.float32)
    else:
        cos, sin = rope_tables(max_position, head_dim)
    kc = _randn(g, (num_blocks, block_size, num_kv_heads, head_dim), dt)
    vc = _randn(g, (num_blocks, block_size, num_kv_heads, head_dim), dt)
    return RopeCase(q=q, k=k, v=v, positions=pos, cos=cos.contiguous(), sin=sin.contiguous(), slots=slots,
                    k_cache0=kc, v_cache0=vc)
