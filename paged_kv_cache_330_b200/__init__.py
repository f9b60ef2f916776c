"""Python binding of libpaged_attn.so: paged KV-cache attention for B200 (sm_100a).

Argument marshalling only.  Every step of the compute path runs in the CUDA
kernels behind the C ABI declared in ``include/paged_attn.h``; PyTorch is used
for device memory and streams.  There is no CPU or PyTorch fallback: if the
shared library is missing, importing this package raises ImportError.

Calls (see the header for exact semantics):

* ``write_kv``       - scatter new tokens' K/V into their cache slots
* ``copy_blocks``    - copy whole blocks (copy-on-write of shared blocks)
* ``rope_write_kv``  - rotary embedding of new tokens' q and k, fused with the K/V cache write
* ``decode``         - one-token paged attention, split-K with the merge in the same kernel
* ``prefill_chunk``  - causal chunked-prefill attention over the paged cache
* ``write_kv_int8``, ``decode_int8``, ``copy_blocks_int8`` - the same over an INT8 cache (codes + fp32 scales)
* ``BlockPool``      - host block pool: blocks, block tables, reference counts
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

__all__ = ["PagedAttnError", "PoolOutOfBlocks", "BlockPool", "write_kv", "copy_blocks", "rope_write_kv", "decode",
           "decode_plan",
           "decode_static_scratch",
           "prefill_chunk", "device_error", "lib", "LIB_PATH", "replay_ops", "version",
           "write_kv_int8", "copy_blocks_int8", "decode_int8", "decode_int8_plan", "decode_lse", "merge_attn_states",
           "decode_cascade", "decode_cascade_workspace_size", "copy_async"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpaged_attn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python paged_kv_cache_330_b200/build.py` "
                      "(there is no fallback path)")

lib = ctypes.CDLL(LIB_PATH)

_vp, _i, _i64, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_ip = ctypes.POINTER(ctypes.c_int)


class _PoolStats(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int64), ("free_blocks", ctypes.c_int64), ("used_blocks", ctypes.c_int64),
                ("shared_blocks", ctypes.c_int64), ("num_seqs", ctypes.c_int64), ("tokens", ctypes.c_int64),
                ("table_refs", ctypes.c_int64), ("ref_sum", ctypes.c_int64), ("utilisation", ctypes.c_double)]


_SIGS = {
    "pa_strerror": (ctypes.c_char_p, [_i]),
    "pa_version": (ctypes.c_char_p, []),
    "pa_copy_async": (_i, [_vp, _vp, _sz, _vp]),
    "pa_write_kv": (_i, [_vp, _vp, _vp, _i, _vp, _vp, _i, _i, _i, _i, _i, _vp]),
    "pa_copy_blocks": (_i, [_vp, _i, _vp, _vp, _i, _i, _i, _i, _i, _vp]),
    "pa_rope_write_kv": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _i, _vp, _vp, _i, _i, _i, _i, _i, _vp]),
    "pa_decode_plan": (_i, [_i, _i, _i, _i, _i, _i, _ip, _ip, ctypes.POINTER(_sz)]),
    "pa_decode_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "pa_decode": (_i, [_vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _i, _vp, _sz, _i, _vp, _vp]),
    "pa_decode_static_scratch": (_i, [_vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _i, _i, _vp, _vp]),
    "pa_prefill_chunk": (_i, [_vp, _vp, _i, _i, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp, _vp]),
    "pa_device_error": (_i, [_ip]),
    "pa_decode_lse": (_i, [_vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _i, _vp, _sz, _i, _vp, _vp,
                           _vp]),
    "pa_decode_cascade_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i, _i, _i]),
    "pa_decode_cascade": (_i, [_vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _i, _i, _vp, _vp, _i, _i,
                               _vp, _sz, _i, _vp, _vp]),
    "pa_merge_attn_states": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _vp, _vp]),
    "pa_dcp_owner": (_i, [_i64, _i, _i]),
    "pa_dcp_local_position": (_i64, [_i64, _i, _i]),
    "pa_dcp_local_lens": (_i, [_i32p, _i, _i, _i, _i, _i32p]),
    "pa_write_kv_int8": (_i, [_vp, _vp, _vp, _i, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]),
    "pa_copy_blocks_int8": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp]),
    "pa_decode_int8_plan": (_i, [_i, _i, _i, _i, _i, _i, _ip, _ip, ctypes.POINTER(_sz)]),
    "pa_decode_int8_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "pa_decode_int8": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _i, _vp, _sz, _i,
                            _vp, _vp]),
    "pa_pool_create": (_vp, [_i, _i, _i32p]),
    "pa_pool_destroy": (None, [_vp]),
    "pa_seq_alloc": (_i, [_vp, _i64, _i]),
    "pa_seq_fork": (_i, [_vp, _i64, _i64, _i]),
    "pa_seq_append": (_i, [_vp, _i64, _i, _i64p, _i32p, _ip]),
    "pa_pool_append_batch": (_i, [_vp, _i64p, _i32p, _i, _i64p, _i32p, _ip]),
    "pa_pool_alloc_batch": (_i, [_vp, _i64p, _i32p, _i]),
    "pa_pool_free_batch": (_i, [_vp, _i64p, _i]),
    "pa_seq_free": (_i, [_vp, _i64]),
    "pa_seq_info": (_i, [_vp, _i64, _ip, _ip]),
    "pa_pool_block_table": (_i, [_vp, _i64p, _i, _i32p, _i, _i32p]),
    "pa_pool_ref_count": (_i, [_vp, _i]),
    "pa_pool_stats": (_i, [_vp, ctypes.POINTER(_PoolStats)]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

PA_OK, PA_ERR_OOM, PA_ERR_NOT_FOUND = 0, -6, -7


class PagedAttnError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = lib.pa_strerror(status).decode()
        super().__init__(f"{what}: {msg}" if what else msg)


class PoolOutOfBlocks(PagedAttnError):
    pass


def _check(status: int, what: str = "") -> None:
    if status != PA_OK:
        raise PagedAttnError(status, what)


def version() -> str:
    return lib.pa_version().decode()


def copy_async(dst, src, stream=None) -> None:
    """Copy the bytes of contiguous tensor src into dst (same byte size; host, pinned host or device memory on
    either side) on `stream`, without waiting for it: one pa_copy_async call, no stream switch on the torch
    side.  Pinned host memory is what makes a host-side copy asynchronous."""
    n = src.numel() * src.element_size()
    if dst.numel() * dst.element_size() != n:
        raise ValueError(f"copy_async: {n} bytes into {dst.numel() * dst.element_size()}")
    if not (src.is_contiguous() and dst.is_contiguous()):
        raise ValueError("copy_async takes contiguous tensors")
    _check(lib.pa_copy_async(ctypes.c_void_p(dst.data_ptr()), ctypes.c_void_p(src.data_ptr()), n,
                             _stream_handle(stream)), "pa_copy_async")


# ---------------------------------------------------------------------------------------------- device calls
_TORCH = None


def _torch():
    global _TORCH
    if _TORCH is None:
        import torch
        _TORCH = torch
    return _TORCH


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return 1
    if t.dtype == torch.float16:
        return 0
    raise ValueError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def _stream_handle(stream):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _want(name, t, dtype=None, shape=None, ndim=None):
    """Host-side check of one tensor argument's dtype / shape (None: not checked)."""
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got shape {tuple(t.shape)}")
    if shape is not None and t.shape != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _caches(k_cache, v_cache):
    """Both caches [num_blocks, block_size, Hkv, D], same shape and 16-bit dtype; returns the shape."""
    ks = k_cache.shape
    if len(ks) != 4 or v_cache.dtype != k_cache.dtype or v_cache.shape != ks:
        _want("k_cache", k_cache, ndim=4)
        _want("v_cache", v_cache, dtype=k_cache.dtype, shape=ks)
    _dtype_code(k_cache)
    return tuple(ks)


def _device_slow(stream, tensors):
    """The precise error for a failed _device check."""
    torch = _torch()
    dev = None
    for t in tensors:
        if t is None:
            continue
        if t.device.type != "cuda":
            raise ValueError(f"device calls take CUDA tensors; got a tensor on {t.device}")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"tensor arguments on {dev} and {t.device}")
    if dev is not None:
        if dev.index != torch.cuda.current_device():
            raise ValueError(f"tensors are on {dev} but the current device is cuda:{torch.cuda.current_device()}")
        if stream is not None and stream.device != dev:
            raise ValueError(f"stream belongs to {stream.device}, tensors to {dev}")
    raise AssertionError("device check failed without a reason")


def _device(stream, *tensors):
    """Every tensor argument must live on the current CUDA device (a host pointer, or another device's memory,
    must never reach a kernel), and a given stream must belong to that device.  Checked after the dtype and
    shape checks, before anything is launched.  (Device indices as ints; the torch.device objects only to
    word an error.)"""
    idx = None
    for t in tensors:
        if t is None:
            continue
        d = t.get_device()  # -1 for host memory
        if idx is None:
            idx = d
        elif d != idx:
            _device_slow(stream, tensors)
    if idx is None:
        return
    if idx < 0 or idx != _torch().cuda.current_device() or (stream is not None and stream.device_index != idx):
        _device_slow(stream, tensors)


def write_kv(k, v, slot_mapping, k_cache, v_cache, stream=None) -> None:
    """k, v [T, Hkv, D]; slot_mapping int64 [T] (-1 = skip); caches [NB, bs, Hkv, D]."""
    torch = _torch()
    _contig(k, v, slot_mapping, k_cache, v_cache)
    NB, bs, Hkv, D = _caches(k_cache, v_cache)
    T = int(k.shape[0]) if k.dim() > 0 else -1
    _want("k", k, dtype=k_cache.dtype, shape=(T, Hkv, D))
    _want("v", v, dtype=k_cache.dtype, shape=(T, Hkv, D))
    _want("slot_mapping", slot_mapping, dtype=torch.int64, shape=(T,))
    _device(stream, k, v, slot_mapping, k_cache, v_cache)
    _check(lib.pa_write_kv(_ptr(k), _ptr(v), _ptr(slot_mapping), int(k.shape[0]), _ptr(k_cache), _ptr(v_cache),
                           NB, bs, Hkv, D, _dtype_code(k_cache), _stream_handle(stream)), "pa_write_kv")


def copy_blocks(pairs, k_cache, v_cache, stream=None) -> None:
    """pairs int32 [n, 2] (src, dst) on the device."""
    torch = _torch()
    _contig(pairs, k_cache, v_cache)
    NB, bs, Hkv, D = _caches(k_cache, v_cache)
    _want("pairs", pairs, dtype=torch.int32, ndim=2)
    _want("pairs", pairs, shape=(pairs.shape[0], 2))
    _device(stream, pairs, k_cache, v_cache)
    _check(lib.pa_copy_blocks(_ptr(pairs), int(pairs.shape[0]), _ptr(k_cache), _ptr(v_cache), NB, bs, Hkv, D,
                              _dtype_code(k_cache), _stream_handle(stream)), "pa_copy_blocks")


def rope_write_kv(q, k, v, positions, cos_table, sin_table, slot_mapping, k_cache, v_cache, q_out=None,
                  stream=None):
    """Rotate q [T, Hq, D] and k [T, Hkv, D] by the rows positions (int64 [T]) of the fp32 tables
    cos_table/sin_table [max_position, D/2]; write the rotated k and the unrotated v into the cache slots
    (slot_mapping int64 [T], -1 = no cache write).  Returns q_out (a new tensor unless given; q_out=q
    rotates in place)."""
    torch = _torch()
    if q_out is None:
        q_out = torch.empty_like(q)
    _contig(q, q_out, k, v, positions, cos_table, sin_table, slot_mapping, k_cache, v_cache)
    if cos_table.dtype != torch.float32 or sin_table.dtype != torch.float32:
        raise ValueError("cos/sin tables must be float32")
    if q_out.shape != q.shape or q_out.dtype != q.dtype:
        raise ValueError("q_out must match q")
    NB, bs, Hkv, D = _caches(k_cache, v_cache)
    _want("q", q, dtype=k_cache.dtype, ndim=3)
    T, Hq = int(q.shape[0]), int(q.shape[1])
    if tuple(k.shape) != (T, Hkv, D) or tuple(v.shape) != (T, Hkv, D) or q.shape[2] != D:
        raise ValueError("q/k/v shapes do not match the cache")
    _want("k", k, dtype=k_cache.dtype)
    _want("v", v, dtype=k_cache.dtype)
    _want("positions", positions, dtype=torch.int64, shape=(T,))
    _want("slot_mapping", slot_mapping, dtype=torch.int64, shape=(T,))
    if cos_table.dim() != 2 or tuple(cos_table.shape) != tuple(sin_table.shape) or cos_table.shape[1] != D // 2:
        raise ValueError("cos/sin tables must be [max_position, head_dim/2]")
    _device(stream, q, q_out, k, v, positions, cos_table, sin_table, slot_mapping, k_cache, v_cache)
    _check(lib.pa_rope_write_kv(_ptr(q), _ptr(q_out), _ptr(k), _ptr(v), _ptr(positions), _ptr(cos_table),
                                _ptr(sin_table), int(cos_table.shape[0]), _ptr(slot_mapping), T, Hq,
                                _ptr(k_cache), _ptr(v_cache), NB, bs, Hkv, D, _dtype_code(k_cache),
                                _stream_handle(stream)), "pa_rope_write_kv")
    return q_out


def decode_plan(batch, num_q_heads, num_kv_heads, head_dim, max_context_len, num_partitions=0):
    """(grid, max_pieces, workspace_bytes) the decode call will use on the current device."""
    gr, mp, ws = ctypes.c_int(), ctypes.c_int(), ctypes.c_size_t()
    _check(lib.pa_decode_plan(batch, num_q_heads, num_kv_heads, head_dim, max_context_len, num_partitions,
                              ctypes.byref(gr), ctypes.byref(mp), ctypes.byref(ws)), "pa_decode_plan")
    return gr.value, mp.value, ws.value


def _decode_args(q, k_cache, v_cache, block_tables, context_lens, out):
    """Shapes and dtypes of a decode call: q [B, Hq, D] in the caches' dtype, block_tables int32 [B, n],
    context_lens int32 [B], out (if given) like q.  Returns (B, Hq, D)."""
    torch = _torch()
    ks, qs, dt = k_cache.shape, q.shape, k_cache.dtype
    if (len(ks) == 4 and v_cache.shape == ks and v_cache.dtype == dt and len(qs) == 3 and q.dtype == dt
            and qs[2] == ks[3] and block_tables.dtype == torch.int32 and block_tables.dim() == 2
            and block_tables.shape[0] == qs[0] and context_lens.dtype == torch.int32
            and context_lens.shape == (qs[0],) and (out is None or (out.dtype == dt and out.shape == qs))):
        _dtype_code(k_cache)
        return qs[0], qs[1], qs[2]
    _, _, _, D = _caches(k_cache, v_cache)
    _want("q", q, dtype=k_cache.dtype, ndim=3)
    B, Hq = int(q.shape[0]), int(q.shape[1])
    _want("q", q, shape=(B, Hq, D))
    _want("block_tables", block_tables, dtype=torch.int32, ndim=2)
    _want("block_tables", block_tables, shape=(B, block_tables.shape[1]))
    _want("context_lens", context_lens, dtype=torch.int32, shape=(B,))
    if out is not None:
        _want("out", out, dtype=q.dtype, shape=q.shape)
    return B, Hq, D


def decode(q, k_cache, v_cache, block_tables, context_lens, max_context_len: int, scale: float, out=None,
           workspace=None, num_partitions: int = 0, stream=None):
    """q [B, Hq, D]; block_tables int32 [B, max_blocks]; context_lens int32 [B]. Returns out [B, Hq, D]."""
    torch = _torch()
    _contig(q, k_cache, v_cache, block_tables, context_lens, out, workspace)
    B, Hq, D = _decode_args(q, k_cache, v_cache, block_tables, context_lens, out)
    NB, bs, Hkv, _ = k_cache.shape
    _device(stream, q, k_cache, v_cache, block_tables, context_lens, out, workspace)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:  # zero-filled once; every call leaves it zeroed again (a given one is checked by the library)
        _, _, need = decode_plan(B, Hq, Hkv, D, max_context_len, num_partitions)
        workspace = torch.zeros(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.pa_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), int(block_tables.shape[1]),
                         _ptr(context_lens), B, Hq, Hkv, D, bs, NB, int(max_context_len), float(scale),
                         _dtype_code(q), _ptr(workspace), ws_bytes, int(num_partitions), _ptr(out),
                         _stream_handle(stream)), "pa_decode")
    return out


def decode_static_scratch(q, k_cache, v_cache, block_tables, context_lens, max_context_len: int, scale: float,
                          out=None, num_partitions: int = 0, stream=None):
    """pa_decode without a workspace argument: the library's static device scratch is used instead (for callers
    that must not allocate where they run decode).  Calls overlapping on the GPU race on that scratch."""
    torch = _torch()
    _contig(q, k_cache, v_cache, block_tables, context_lens, out)
    B, Hq, D = _decode_args(q, k_cache, v_cache, block_tables, context_lens, out)
    NB, bs, Hkv, _ = k_cache.shape
    _device(stream, q, k_cache, v_cache, block_tables, context_lens, out)
    if out is None:
        out = torch.empty_like(q)
    _check(lib.pa_decode_static_scratch(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                                        int(block_tables.shape[1]), _ptr(context_lens), B, Hq, Hkv, D, bs, NB,
                                        int(max_context_len), float(scale), _dtype_code(q), int(num_partitions),
                                        _ptr(out), _stream_handle(stream)), "pa_decode_static_scratch")
    return out


def prefill_chunk(q, query_start_loc, k_cache, v_cache, block_tables, context_lens, max_chunk_len: int,
                  scale: float, out=None, stream=None):
    """q [sum C, Hq, D]; query_start_loc int32 [B+1]; returns out [sum C, Hq, D]."""
    torch = _torch()
    _contig(q, query_start_loc, k_cache, v_cache, block_tables, context_lens, out)
    NB, bs, Hkv, D = _caches(k_cache, v_cache)
    _want("q", q, dtype=k_cache.dtype, ndim=3)
    T, Hq = int(q.shape[0]), int(q.shape[1])
    _want("q", q, shape=(T, Hq, D))
    _want("context_lens", context_lens, dtype=torch.int32, ndim=1)
    B = int(context_lens.shape[0])
    _want("query_start_loc", query_start_loc, dtype=torch.int32, shape=(B + 1,))
    _want("block_tables", block_tables, dtype=torch.int32, ndim=2)
    _want("block_tables", block_tables, shape=(B, block_tables.shape[1]))
    if out is not None:
        _want("out", out, dtype=q.dtype, shape=q.shape)
    _device(stream, q, query_start_loc, k_cache, v_cache, block_tables, context_lens, out)
    if out is None:
        out = torch.empty_like(q)
    _check(lib.pa_prefill_chunk(_ptr(q), _ptr(query_start_loc), T, int(max_chunk_len), _ptr(k_cache), _ptr(v_cache),
                                _ptr(block_tables), int(block_tables.shape[1]), _ptr(context_lens), B, Hq, Hkv, D,
                                bs, NB, float(scale), _dtype_code(q), _ptr(out), _stream_handle(stream)),
           "pa_prefill_chunk")
    return out


def decode_lse(q, k_cache, v_cache, block_tables, context_lens, max_context_len: int, scale: float, out=None,
               lse=None, workspace=None, num_partitions: int = 0, stream=None):
    """pa_decode that also returns the log-sum-exp of each (sequence, head)'s scores: (out [B, Hq, D],
    lse float32 [B, Hq]); lse is -inf (and out 0) for a sequence with no tokens."""
    torch = _torch()
    _contig(q, k_cache, v_cache, block_tables, context_lens, out, lse, workspace)
    B, Hq, D = _decode_args(q, k_cache, v_cache, block_tables, context_lens, out)
    NB, bs, Hkv, _ = k_cache.shape
    if lse is not None:
        _want("lse", lse, dtype=torch.float32, shape=(B, Hq))
    _device(stream, q, k_cache, v_cache, block_tables, context_lens, out, lse, workspace)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    if workspace is None:
        _, _, need = decode_plan(B, Hq, Hkv, D, max_context_len, num_partitions)
        workspace = torch.zeros(need, dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.pa_decode_lse(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), int(block_tables.shape[1]),
                             _ptr(context_lens), B, Hq, Hkv, D, bs, NB, int(max_context_len), float(scale),
                             _dtype_code(q), _ptr(workspace), ws_bytes, int(num_partitions), _ptr(out), _ptr(lse),
                             _stream_handle(stream)), "pa_decode_lse")
    return out, lse


def decode_cascade_workspace_size(batch, num_q_heads, num_kv_heads, head_dim, max_context_len, num_groups,
                                  max_group_size, max_prefix_len, num_partitions=0) -> int:
    n = lib.pa_decode_cascade_workspace_size(batch, num_q_heads, num_kv_heads, head_dim, max_context_len,
                                             num_partitions, num_groups, max_group_size, max_prefix_len)
    if n == 0:
        raise PagedAttnError(-1, "pa_decode_cascade_workspace_size")
    return n


def decode_cascade(q, k_cache, v_cache, block_tables, context_lens, max_context_len: int, scale: float, group_start,
                   seq_prefix_len, max_group_size: int, max_prefix_len: int, out=None, workspace=None,
                   num_partitions: int = 0, stream=None):
    """Decode with every shared prefix read once for all its sharers.  group_start int32 [G+1] (device):
    group g = sequences group_start[g] .. group_start[g+1]-1; seq_prefix_len int32 [B] (device): each
    sequence's shared prefix length (a multiple of 16; 0 = none).  Returns out [B, Hq, D]."""
    torch = _torch()
    _contig(q, k_cache, v_cache, block_tables, context_lens, group_start, seq_prefix_len, out, workspace)
    B, Hq, D = _decode_args(q, k_cache, v_cache, block_tables, context_lens, out)
    NB, bs, Hkv, _ = k_cache.shape
    _want("group_start", group_start, dtype=torch.int32, ndim=1)
    _want("seq_prefix_len", seq_prefix_len, dtype=torch.int32, shape=(B,))
    ngroups = max(int(group_start.shape[0]) - 1, 0)
    _device(stream, q, k_cache, v_cache, block_tables, context_lens, group_start, seq_prefix_len, out, workspace)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:  # zero-filled once; every call leaves its counters zeroed again
        need = decode_cascade_workspace_size(B, Hq, Hkv, D, max_context_len, ngroups, max_group_size,
                                             max_prefix_len, num_partitions)
        workspace = torch.zeros(need, dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.pa_decode_cascade(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                                 int(block_tables.shape[1]), _ptr(context_lens), B, Hq, Hkv, D, bs, NB,
                                 int(max_context_len), float(scale), _dtype_code(q), ngroups, _ptr(group_start),
                                 _ptr(seq_prefix_len), int(max_group_size), int(max_prefix_len), _ptr(workspace),
                                 ws_bytes, int(num_partitions), _ptr(out), _stream_handle(stream)),
           "pa_decode_cascade")
    return out


def merge_attn_states(parts, lses, out=None, stream=None):
    """parts [P, B, H, D] (bf16/fp16), lses float32 [P, B, H] -> out [B, H, D]: the softmax-weighted
    combination of the parts by their log-sum-exps."""
    torch = _torch()
    _contig(parts, lses, out)
    _want("parts", parts, ndim=4)
    P, B, H, D = (int(x) for x in parts.shape)
    _want("lses", lses, dtype=torch.float32, shape=(P, B, H))
    if out is not None:
        _want("out", out, dtype=parts.dtype, shape=(B, H, D))
    _device(stream, parts, lses, out)
    if out is None:
        out = torch.empty((B, H, D), dtype=parts.dtype, device=parts.device)
    _check(lib.pa_merge_attn_states(_ptr(parts), _ptr(lses), P, B, H, D, _dtype_code(parts), _ptr(out),
                                    _stream_handle(stream)), "pa_merge_attn_states")
    return out


# ---------------------------------------------------------------------------------------------- INT8 cache
def _int8_caches(k_codes, v_codes, k_scales, v_scales):
    """Codes int8 [NB, bs, Hkv, D] (both alike), scales float32 [NB, Hkv, bs] (both alike); returns the shape."""
    torch = _torch()
    _want("k_codes", k_codes, dtype=torch.int8, ndim=4)
    _want("v_codes", v_codes, dtype=torch.int8, shape=k_codes.shape)
    NB, bs, Hkv, D = (int(x) for x in k_codes.shape)
    _want("k_scales", k_scales, dtype=torch.float32, shape=(NB, Hkv, bs))
    _want("v_scales", v_scales, dtype=torch.float32, shape=(NB, Hkv, bs))
    return NB, bs, Hkv, D


def write_kv_int8(k, v, slot_mapping, k_codes, v_codes, k_scales, v_scales, stream=None) -> None:
    """Quantise k, v [T, Hkv, D] (bf16/fp16) into the INT8 cache rows of slot_mapping int64 [T] (-1 = skip)."""
    torch = _torch()
    _contig(k, v, slot_mapping, k_codes, v_codes, k_scales, v_scales)
    NB, bs, Hkv, D = _int8_caches(k_codes, v_codes, k_scales, v_scales)
    _want("k", k, ndim=3)
    T = int(k.shape[0])
    _dtype_code(k)
    _want("k", k, shape=(T, Hkv, D))
    _want("v", v, dtype=k.dtype, shape=(T, Hkv, D))
    _want("slot_mapping", slot_mapping, dtype=torch.int64, shape=(T,))
    _device(stream, k, v, slot_mapping, k_codes, v_codes, k_scales, v_scales)
    _check(lib.pa_write_kv_int8(_ptr(k), _ptr(v), _ptr(slot_mapping), T, _ptr(k_codes), _ptr(v_codes),
                                _ptr(k_scales), _ptr(v_scales), NB, bs, Hkv, D, _dtype_code(k),
                                _stream_handle(stream)), "pa_write_kv_int8")


def copy_blocks_int8(pairs, k_codes, v_codes, k_scales, v_scales, stream=None) -> None:
    """pairs int32 [n, 2] (src, dst) on the device: copy whole blocks of the INT8 codes and scales."""
    torch = _torch()
    _contig(pairs, k_codes, v_codes, k_scales, v_scales)
    NB, bs, Hkv, D = _int8_caches(k_codes, v_codes, k_scales, v_scales)
    _want("pairs", pairs, dtype=torch.int32, ndim=2)
    _want("pairs", pairs, shape=(pairs.shape[0], 2))
    _device(stream, pairs, k_codes, v_codes, k_scales, v_scales)
    _check(lib.pa_copy_blocks_int8(_ptr(pairs), int(pairs.shape[0]), _ptr(k_codes), _ptr(v_codes), _ptr(k_scales),
                                   _ptr(v_scales), NB, bs, Hkv, D, _stream_handle(stream)), "pa_copy_blocks_int8")


def decode_int8_plan(batch, num_q_heads, num_kv_heads, head_dim, max_context_len, num_partitions=0):
    """(grid, max_pieces, workspace_bytes) of decode over the INT8 cache on the current device."""
    gr, mp, ws = ctypes.c_int(), ctypes.c_int(), ctypes.c_size_t()
    _check(lib.pa_decode_int8_plan(batch, num_q_heads, num_kv_heads, head_dim, max_context_len, num_partitions,
                                   ctypes.byref(gr), ctypes.byref(mp), ctypes.byref(ws)), "pa_decode_int8_plan")
    return gr.value, mp.value, ws.value


def decode_int8(q, k_codes, v_codes, k_scales, v_scales, block_tables, context_lens, max_context_len: int,
                scale: float, out=None, workspace=None, num_partitions: int = 0, stream=None):
    """Decode over the INT8 cache: q [B, Hq, D] bf16/fp16; returns out [B, Hq, D] in q's dtype."""
    torch = _torch()
    _contig(q, k_codes, v_codes, k_scales, v_scales, block_tables, context_lens, out, workspace)
    NB, bs, Hkv, D = _int8_caches(k_codes, v_codes, k_scales, v_scales)
    _want("q", q, ndim=3)
    _dtype_code(q)
    B, Hq = int(q.shape[0]), int(q.shape[1])
    _want("q", q, shape=(B, Hq, D))
    _want("block_tables", block_tables, dtype=torch.int32, ndim=2)
    _want("block_tables", block_tables, shape=(B, block_tables.shape[1]))
    _want("context_lens", context_lens, dtype=torch.int32, shape=(B,))
    if out is not None:
        _want("out", out, dtype=q.dtype, shape=q.shape)
    _device(stream, q, k_codes, v_codes, k_scales, v_scales, block_tables, context_lens, out, workspace)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:  # zero-filled once; every call leaves it zeroed again (a given one is checked by the library)
        _, _, need = decode_int8_plan(B, Hq, Hkv, D, max_context_len, num_partitions)
        workspace = torch.zeros(need, dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.pa_decode_int8(_ptr(q), _ptr(k_codes), _ptr(v_codes), _ptr(k_scales), _ptr(v_scales),
                              _ptr(block_tables), int(block_tables.shape[1]), _ptr(context_lens), B, Hq, Hkv, D, bs,
                              NB, int(max_context_len), float(scale), _dtype_code(q), _ptr(workspace), ws_bytes,
                              int(num_partitions), _ptr(out), _stream_handle(stream)), "pa_decode_int8")
    return out


def device_error() -> int:
    """Synchronise the device, return and clear the kernels' error bits (0 = none)."""
    v = ctypes.c_int()
    _check(lib.pa_device_error(ctypes.byref(v)), "pa_device_error")
    return v.value


# ---------------------------------------------------------------------------------------------- host pool
class BlockPool:
    """Host block pool (C++): blocks, per-sequence block tables, reference counts, copy-on-write."""

    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        self.block_size = block_size
        self.num_blocks = num_blocks
        arr = None
        if free_order is not None:
            arr = np.ascontiguousarray(np.asarray(free_order, dtype=np.int32))
            if arr.shape != (num_blocks,):
                raise ValueError("free_order must have num_blocks entries")
        ptr = arr.ctypes.data_as(_i32p) if arr is not None else None
        self._h = lib.pa_pool_create(num_blocks, block_size, ptr)
        if not self._h:
            raise ValueError("pa_pool_create rejected its arguments")

    def close(self):
        if getattr(self, "_h", None):
            lib.pa_pool_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    @staticmethod
    def _pool_check(status, what):
        if status == PA_ERR_OOM:
            raise PoolOutOfBlocks(status, what)
        _check(status, what)

    def alloc(self, seq_id: int, num_tokens: int) -> None:
        self._pool_check(lib.pa_seq_alloc(self._h, seq_id, num_tokens), "alloc")

    def fork(self, parent: int, child: int, n_prefix: int) -> None:
        self._pool_check(lib.pa_seq_fork(self._h, parent, child, n_prefix), "fork")

    def append(self, seq_id: int, n: int):
        """Returns (slots int64[n], copy-on-write pairs [(src, dst)])."""
        slots = np.empty(max(n, 1), dtype=np.int64)
        pair = np.empty(2, dtype=np.int32)
        ncow = ctypes.c_int(0)
        self._pool_check(lib.pa_seq_append(self._h, seq_id, n, slots.ctypes.data_as(_i64p), pair.ctypes.data_as(_i32p),
                                           ctypes.byref(ncow)), "append")
        return slots[:n], ([(int(pair[0]), int(pair[1]))] if ncow.value else [])

    def append_batch(self, seq_ids, counts):
        """Extend every sequence of seq_ids by its count (an int applies to all) in one native call; the
        same result as append() per sequence in order, all or nothing.  Returns (slots int64[sum counts] in
        batch order, copy-on-write pairs [(src, dst)])."""
        ids = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int64))
        cnt = np.ascontiguousarray(np.broadcast_to(np.asarray(counts, dtype=np.int32), ids.shape))
        total = int(cnt.sum()) if len(cnt) else 0
        slots = np.empty(max(total, 1), dtype=np.int64)
        pairs = np.empty((max(len(ids), 1), 2), dtype=np.int32)
        ncow = ctypes.c_int(0)
        self._pool_check(lib.pa_pool_append_batch(self._h, ids.ctypes.data_as(_i64p), cnt.ctypes.data_as(_i32p),
                                                  len(ids), slots.ctypes.data_as(_i64p), pairs.ctypes.data_as(_i32p),
                                                  ctypes.byref(ncow)), "append_batch")
        return slots[:total], [(int(a), int(b)) for a, b in pairs[:ncow.value]]

    def alloc_batch(self, seq_ids, num_tokens) -> None:
        """New sequences (num_tokens per id, or one int for all) in one native call; all or nothing."""
        ids = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int64))
        cnt = np.ascontiguousarray(np.broadcast_to(np.asarray(num_tokens, dtype=np.int32), ids.shape))
        self._pool_check(lib.pa_pool_alloc_batch(self._h, ids.ctypes.data_as(_i64p), cnt.ctypes.data_as(_i32p),
                                                 len(ids)), "alloc_batch")

    def free_batch(self, seq_ids) -> None:
        """Drop every sequence of seq_ids in one native call; all or nothing."""
        ids = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int64))
        self._pool_check(lib.pa_pool_free_batch(self._h, ids.ctypes.data_as(_i64p), len(ids)), "free_batch")

    def free(self, seq_id: int) -> None:
        self._pool_check(lib.pa_seq_free(self._h, seq_id), "free")

    def info(self, seq_id: int):
        n, nb = ctypes.c_int(), ctypes.c_int()
        self._pool_check(lib.pa_seq_info(self._h, seq_id, ctypes.byref(n), ctypes.byref(nb)), "info")
        return n.value, nb.value

    def block_table(self, seq_ids, max_blocks: int):
        ids = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int64))
        out = np.empty((len(ids), max(max_blocks, 0)), dtype=np.int32)
        lens = np.empty(len(ids), dtype=np.int32)
        self._pool_check(lib.pa_pool_block_table(self._h, ids.ctypes.data_as(_i64p), len(ids),
                                                 out.ctypes.data_as(_i32p), max_blocks, lens.ctypes.data_as(_i32p)),
                         "block_table")
        return out, lens

    def ref_count(self, block_id: int) -> int:
        return lib.pa_pool_ref_count(self._h, block_id)

    def stats(self) -> dict:
        st = _PoolStats()
        _check(lib.pa_pool_stats(self._h, ctypes.byref(st)), "stats")
        return {f: getattr(st, f) for f, _ in _PoolStats._fields_}


def replay_ops(ops, num_blocks: int, block_size: int, free_order, batch: int):
    """Run a list of pool operations ('alloc', id, n) / ('fork', parent, child, n) / ('append', id, n) /
    ('append_new', id, n) on a new BlockPool.

    Returns (pool, block_tables int32 [batch, max_blocks], context_lens int32 [batch], slot_mapping int64
    of the 'append_new' tokens in order, copy-on-write pairs)."""
    pool = BlockPool(num_blocks, block_size, free_order)
    slots, pairs = [], []
    for op in ops:
        if op[0] == "alloc":
            pool.alloc(op[1], op[2])
        elif op[0] == "fork":
            pool.fork(op[1], op[2], op[3])
        elif op[0] in ("append", "append_new"):
            s, p = pool.append(op[1], op[2])
            pairs += p
            if op[0] == "append_new":
                slots.append(s)
        else:
            raise ValueError(op[0])
    max_blocks = max([pool.info(b)[1] for b in range(batch)] + [1])
    bt, lens = pool.block_table(list(range(batch)), max_blocks)
    sm = np.concatenate(slots) if slots else np.zeros(0, dtype=np.int64)
    return pool, bt, lens, sm, pairs
