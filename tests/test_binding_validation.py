"""Host-side argument checks of the Python binding (no GPU): valid calls, built the way the GPU tests and the
bench build them, get through every dtype and shape check and stop only at the device check (CPU tensors
never reach a kernel); each kind of bad argument is rejected with its own message, before any library call."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import paged_kv_cache_330_b200 as pa
from workloads import make_custom, make_rope_case, new_token_positions, rope_tables

DEVICE_MSG = "device calls take CUDA tensors"


@pytest.fixture(autouse=True)
def _no_library_calls(monkeypatch):
    """A device call that reaches the library here would be a bug: the checks must stop it first (the host
    pool calls stay open; the workloads are replayed through them)."""
    device_calls = ("pa_write_kv", "pa_copy_blocks", "pa_rope_write_kv", "pa_decode", "pa_decode_plan",
                    "pa_decode_static_scratch", "pa_prefill_chunk", "pa_device_error")
    real = pa.lib

    class Trap:
        def __getattr__(self, name):
            if name in device_calls:
                raise AssertionError(f"{name} reached the library from a CPU-tensor call")
            return getattr(real, name)
    monkeypatch.setattr(pa, "lib", Trap())


def _decode_case():
    wl = make_custom(seed=1, lens=[5, 40, 17], num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16)
    _, bt, lens, sm, _ = pa.replay_ops(wl.ops, wl.num_blocks, 16, wl.free_order, wl.batch)
    return wl, torch.from_numpy(bt), torch.from_numpy(lens), torch.from_numpy(sm)


def _prefill_case():
    wl = make_custom(seed=2, lens=[300, 129], chunk_lens=[200, 129], kind="prefill", num_q_heads=8, num_kv_heads=2,
                     head_dim=128, block_size=16)
    _, bt, lens, sm, _ = pa.replay_ops(wl.ops, wl.num_blocks, 16, wl.free_order, wl.batch)
    return wl, torch.from_numpy(bt), torch.from_numpy(lens), torch.from_numpy(sm)


def _raises(msg, fn, *a, **kw):
    with pytest.raises(ValueError, match=msg):
        fn(*a, **kw)


def test_write_kv_checks():
    wl, bt, lens, sm = _decode_case()
    kc, vc = wl.k_cache0, wl.v_cache0
    _raises(DEVICE_MSG, pa.write_kv, wl.k_new, wl.v_new, sm, kc, vc)
    _raises("slot_mapping must be torch.int64", pa.write_kv, wl.k_new, wl.v_new, sm.to(torch.int32), kc, vc)
    _raises("slot_mapping must have shape", pa.write_kv, wl.k_new, wl.v_new, sm[:-1], kc, vc)
    _raises("k must be", pa.write_kv, wl.k_new.half(), wl.v_new, sm, kc, vc)
    _raises("v must have shape", pa.write_kv, wl.k_new, wl.v_new[:, :1].contiguous(), sm, kc, vc)
    _raises("v_cache must be", pa.write_kv, wl.k_new, wl.v_new, sm, kc, vc.half())
    _raises("unsupported dtype", pa.write_kv, wl.k_new.float(), wl.v_new.float(), sm, kc.float(), vc.float())


def test_copy_blocks_checks():
    kc = torch.zeros(8, 16, 2, 64, dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    pairs = torch.tensor([[1, 2], [3, 4]], dtype=torch.int32)
    _raises(DEVICE_MSG, pa.copy_blocks, pairs, kc, vc)
    _raises("pairs must be torch.int32", pa.copy_blocks, pairs.long(), kc, vc)
    _raises("pairs must have shape", pa.copy_blocks, torch.zeros(2, 3, dtype=torch.int32), kc, vc)
    _raises("v_cache must have shape", pa.copy_blocks, pairs, kc, vc[:4].contiguous())


def test_decode_checks():
    wl, bt, lens, sm = _decode_case()
    kc, vc, q = wl.k_cache0, wl.v_cache0, wl.q
    maxL = int(lens.max())
    for fn in (pa.decode, pa.decode_static_scratch):
        _raises(DEVICE_MSG, fn, q, kc, vc, bt, lens, maxL, wl.scale)
        _raises(DEVICE_MSG, fn, q, kc, vc, bt, lens, maxL, wl.scale, out=torch.empty_like(q))
        _raises("block_tables must be torch.int32", fn, q, kc, vc, bt.long(), lens, maxL, wl.scale)
        _raises("block_tables must have shape", fn, q, kc, vc, bt[:2].contiguous(), lens, maxL, wl.scale)
        _raises("context_lens must be torch.int32", fn, q, kc, vc, bt, lens.long(), maxL, wl.scale)
        _raises("context_lens must have shape", fn, q, kc, vc, bt, lens[:2].contiguous(), maxL, wl.scale)
        _raises("q must be", fn, q.half(), kc, vc, bt, lens, maxL, wl.scale)
        _raises("q must have shape", fn, q[:, :, :64].contiguous(), kc, vc, bt, lens, maxL, wl.scale)
        _raises("out must be", fn, q, kc, vc, bt, lens, maxL, wl.scale, out=torch.empty_like(q).half())
        _raises("out must have shape", fn, q, kc, vc, bt, lens, maxL, wl.scale, out=torch.empty_like(q[:2]))
    ws = torch.zeros(1 << 20, dtype=torch.uint8)
    _raises(DEVICE_MSG, pa.decode, q, kc, vc, bt, lens, maxL, wl.scale, workspace=ws, num_partitions=3)
    # the rows-of-one-sequence form used by the prefill-row test
    btr = bt[:1].expand(4, -1).contiguous()
    ctx = torch.tensor([10, 11, 12, 13], dtype=torch.int32)
    _raises(DEVICE_MSG, pa.decode, q[:1].expand(4, -1, -1).contiguous(), kc, vc, btr, ctx, 13, wl.scale)


def test_prefill_checks():
    wl, bt, lens, sm = _prefill_case()
    kc, vc, q = wl.k_cache0, wl.v_cache0, wl.q
    qsl = torch.from_numpy(wl.query_start_loc)
    C = int(np.diff(wl.query_start_loc).max())
    _raises(DEVICE_MSG, pa.prefill_chunk, q, qsl, kc, vc, bt, lens, C, wl.scale)
    _raises(DEVICE_MSG, pa.prefill_chunk, q, qsl, kc, vc, bt, lens, C, wl.scale, out=torch.empty_like(q))
    _raises("query_start_loc must be torch.int32", pa.prefill_chunk, q, qsl.long(), kc, vc, bt, lens, C, wl.scale)
    _raises("query_start_loc must have shape", pa.prefill_chunk, q, qsl[:-1].contiguous(), kc, vc, bt, lens, C,
            wl.scale)
    _raises("block_tables must have shape", pa.prefill_chunk, q, qsl, kc, vc, bt[:1].contiguous(), lens, C, wl.scale)
    _raises("context_lens must be torch.int32", pa.prefill_chunk, q, qsl, kc, vc, bt, lens.long(), C, wl.scale)
    _raises("q must be", pa.prefill_chunk, q.half(), qsl, kc, vc, bt, lens, C, wl.scale)


def test_rope_write_kv_checks():
    c = make_rope_case(seed=3, num_tokens=9, num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16, num_blocks=2,
                       max_position=32)
    a = (c.q, c.k, c.v, c.positions, c.cos, c.sin, c.slots, c.k_cache0, c.v_cache0)
    _raises(DEVICE_MSG, pa.rope_write_kv, *a)
    _raises(DEVICE_MSG, pa.rope_write_kv, *a, q_out=c.q)
    bad = list(a)
    bad[3] = c.positions.to(torch.int32)
    _raises("positions must be torch.int64", pa.rope_write_kv, *bad)
    bad = list(a)
    bad[6] = c.slots[:-1].contiguous()
    _raises("slot_mapping must have shape", pa.rope_write_kv, *bad)
    bad = list(a)
    bad[4] = c.cos.double()
    _raises("cos/sin tables must be float32", pa.rope_write_kv, *bad)
    bad = list(a)
    bad[4], bad[5] = c.cos[:, :16].contiguous(), c.sin[:, :16].contiguous()
    _raises("cos/sin tables must be", pa.rope_write_kv, *bad)
    bad = list(a)
    bad[1] = c.k.half()
    _raises("k must be", pa.rope_write_kv, *bad)
    # the prefill-step form used by the bench and the chained tests
    wl, bt, lens, sm = _prefill_case()
    cos, sin = rope_tables(1024, 128)
    pos = torch.from_numpy(new_token_positions(wl))
    _raises(DEVICE_MSG, pa.rope_write_kv, wl.q, wl.k_new, wl.v_new, pos, cos, sin, sm, wl.k_cache0, wl.v_cache0)


def test_write_kv_from_a_shape_only_row():
    """A 0-d tensor for k is rejected by the shape check, not by an index error."""
    kc = torch.zeros(2, 16, 2, 64, dtype=torch.bfloat16)
    _raises("k must have shape", pa.write_kv, torch.tensor(1.0, dtype=torch.bfloat16), kc[0, 0], torch.zeros(1,
            dtype=torch.int64), kc, kc.clone())
