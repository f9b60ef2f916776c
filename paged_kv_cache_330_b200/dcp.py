"""Decode with each sequence's context split across devices (one process per GPU).

Page "In-depth analysis of vllm-ascend: LLM inference architecture on Ascend hardware", sections 1.1 and
3.1 (DCP): every device attends over the part of the KV cache it holds, the intermediate results of all
devices are gathered (a global AllGather) and combined.  Split rule (C ABI, ``pa_dcp_*``): logical block j
of every sequence lives on rank j mod W, where it is local block j // W, so each rank keeps an ordinary
block pool and paged cache of its own tokens.  One decode step on every rank:

1. ``binding.decode_lse`` over the rank's local cache: its output normalised over its own tokens and the
   log-sum-exp of its scores (one kernel);
2. all-gather of both over the process group (NCCL on GPUs, gloo in the CPU tests);
3. ``binding.merge_attn_states``: the softmax-weighted combination by log-sum-exp (one kernel).

Every rank takes the same collective steps in the same order.  Steps 1 and 3 are the library's kernels;
``partial`` and ``merge`` exist so the host-side protocol can be exercised where no GPU is present.
"""

from __future__ import annotations

import ctypes

import numpy as np

from . import _check, _i32p, decode_lse, lib, merge_attn_states


def owner(position: int, block_size: int, world: int) -> int:
    """Rank that holds token `position` of a sequence."""
    r = lib.pa_dcp_owner(int(position), int(block_size), int(world))
    _check(min(r, 0), "pa_dcp_owner")
    return r


def local_position(position: int, block_size: int, world: int) -> int:
    """Index of token `position` in its rank's local sequence."""
    r = lib.pa_dcp_local_position(int(position), int(block_size), int(world))
    _check(int(min(r, 0)), "pa_dcp_local_position")
    return int(r)


def local_lens(context_lens, block_size: int, world: int, rank: int) -> np.ndarray:
    """int32 [B]: tokens of every sequence that `rank` holds (host arrays)."""
    lens = np.ascontiguousarray(np.asarray(context_lens, dtype=np.int32))
    out = np.empty_like(lens)
    _check(lib.pa_dcp_local_lens(lens.ctypes.data_as(_i32p), len(lens), int(block_size), int(world), int(rank),
                                 out.ctypes.data_as(_i32p)), "pa_dcp_local_lens")
    return out


def _all_gather(x, group):
    import torch
    import torch.distributed as dist
    W = dist.get_world_size(group)
    if dist.get_backend(group) == "nccl":
        buf = torch.empty((W,) + tuple(x.shape), dtype=x.dtype, device=x.device)
        dist.all_gather_into_tensor(buf, x.contiguous(), group=group)
        return buf
    bufs = [torch.empty_like(x) for _ in range(W)]
    dist.all_gather(bufs, x.contiguous(), group=group)
    return torch.stack(bufs)


def dcp_decode(q, k_cache, v_cache, block_tables, context_lens, max_context_len: int, scale: float, group=None,
               partial=None, merge=None, stream=None):
    """One decode step with the context split over the ranks of `group`.

    q [B, Hq, D] is the same on every rank; k_cache/v_cache, block_tables and context_lens describe this
    rank's local share (its own pool; context_lens are the local lengths).  Returns out [B, Hq, D] on every
    rank.  `partial(q, ...) -> (out, lse)` and `merge(parts, lses) -> out` default to the library's kernels."""
    if partial is None:
        partial = lambda *a: decode_lse(*a, stream=stream)
    if merge is None:
        merge = lambda parts, lses: merge_attn_states(parts, lses, stream=stream)
    o, lse = partial(q, k_cache, v_cache, block_tables, context_lens, int(max_context_len), float(scale))
    parts = _all_gather(o, group)
    lses = _all_gather(lse, group)
    return merge(parts, lses)
