"""Pins of the INT8 KV-cache oracle (oracle/kv_quant.py) to facts outside itself, and planted mistakes that
each must fail at least one pin.

The pins: a row's largest magnitude encodes to +-127 with its sign; every element is within half a step
(scale / 2, plus the fp32 rounding of the two divisions and the product) of code * scale; a zero row gives
zero codes and a zero scale, and a single non-zero element gives +-127; rows that already lie on a
power-of-two grid come back exactly; torch's own int8 quantiser (round half to even) gives the same codes
from the same scale except, by one step, next to a .5 tie; and the cache write puts codes and scales at
cache row `slot` of the flat view.
"""

from __future__ import annotations

import os
import types

import numpy as np
import pytest
import torch

from oracle import kv_quant as oq

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "kv_quant.py")


def _rows(seed, n=257, D=128, dtype=torch.bfloat16, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(n, D, generator=g) * scale).to(dtype).float().numpy()


def check_amax_maps_to_127(m):
    for seed, dt, sc in ((1, torch.bfloat16, 1.0), (2, torch.float16, 30.0), (3, torch.bfloat16, 1e-3)):
        x = _rows(seed, dtype=dt, scale=sc)
        codes, scales = m.quantize_rows(x)
        j = np.argmax(np.abs(x), axis=1)
        top = codes[np.arange(x.shape[0]), j].astype(np.int32)
        assert np.array_equal(top, np.where(x[np.arange(x.shape[0]), j] > 0, 127, -127))
        assert np.abs(codes.astype(np.int32)).max() == 127


def check_half_step_bound(m):
    for seed, dt, sc in ((4, torch.bfloat16, 1.0), (5, torch.float16, 7.0), (6, torch.bfloat16, 300.0)):
        x = _rows(seed, dtype=dt, scale=sc)
        codes, scales = m.quantize_rows(x)
        err = np.abs(x.astype(np.float64) - m.dequantize_rows(codes, scales))
        assert (err <= scales.astype(np.float64)[:, None] * (0.5 + 1e-4)).all()


def check_zero_and_single_element_rows(m):
    x = np.zeros((3, 64), dtype=np.float32)
    x[1, 5] = -3.5
    x[2, 63] = 0.125
    codes, scales = m.quantize_rows(x)
    assert np.array_equal(codes[0], np.zeros(64, dtype=np.int8)) and scales[0] == 0
    assert codes[1, 5] == -127 and np.count_nonzero(codes[1]) == 1 and scales[1] == np.float32(3.5) / np.float32(127)
    assert codes[2, 63] == 127 and np.count_nonzero(codes[2]) == 1
    assert np.array_equal(m.dequantize_rows(codes[:1], scales[:1]), np.zeros((1, 64)))


def check_grid_rows_exact(m):
    rng = np.random.default_rng(7)
    for e in (-10, -3, 0, 2, 6):
        k = rng.integers(-127, 128, size=(20, 128))
        k[:, 0] = rng.choice([-127, 127], size=20)
        c = 2.0 ** e
        codes, scales = m.quantize_rows((k * c).astype(np.float32))
        assert np.array_equal(codes.astype(np.int64), k)
        assert (scales == np.float32(c)).all()


def check_torch_quantizer_agrees(m):
    """torch rounds x * (1/scale) half to even; the codes here round x * (127/amax).  The two products differ
    by ~1e-5, so the codes may differ only by one step and only where x/scale lies next to a .5 tie."""
    x = _rows(8, n=256)
    codes, scales = m.quantize_rows(x)
    for r in range(x.shape[0]):
        tq = torch.quantize_per_tensor(torch.from_numpy(x[r]), float(scales[r]), 0, torch.qint8).int_repr().numpy()
        d = np.abs(tq.astype(np.int32) - codes[r].astype(np.int32))
        assert d.max() <= 1
        ratio = x[r].astype(np.float64) / float(scales[r])
        near_tie = np.abs(np.abs(ratio - np.floor(ratio)) - 0.5) < 1e-4
        assert not (d.astype(bool) & ~near_tie).any()


def check_write_places_rows(m):
    rng = np.random.default_rng(9)
    T, Hkv, D, NB, bs = 6, 2, 64, 4, 4
    k = _rows(10, n=T * Hkv, D=D).reshape(T, Hkv, D)
    v = _rows(11, n=T * Hkv, D=D).reshape(T, Hkv, D)
    kc = rng.integers(-127, 128, size=(NB, bs, Hkv, D)).astype(np.int8)
    vc = rng.integers(-127, 128, size=(NB, bs, Hkv, D)).astype(np.int8)
    ks = rng.random((NB, Hkv, bs)).astype(np.float32)
    vs = rng.random((NB, Hkv, bs)).astype(np.float32)
    old = [a.copy() for a in (kc, vc, ks, vs)]
    slots = np.array([3, -1, 14, 0, 9, 15])
    m.write_kv_int8(k, v, slots, kc, vc, ks, vs)
    kq, kss = m.quantize_rows(k)
    vq, vss = m.quantize_rows(v)
    # every array viewed as [NB * bs rows, ...]: codes directly, scales after moving the token axis forward
    rows = lambda a: a.reshape(NB * bs, *a.shape[2:]) if a.ndim == 4 else a.transpose(0, 2, 1).reshape(NB * bs, Hkv)
    flat = [rows(a) for a in (kc, vc, ks, vs)]
    flat_old = [rows(a) for a in old]
    for t, s in enumerate(slots):
        if s >= 0:
            assert np.array_equal(flat[0][s], kq[t]) and np.array_equal(flat[1][s], vq[t])
            assert np.array_equal(flat[2][s], kss[t]) and np.array_equal(flat[3][s], vss[t])
    untouched = [r for r in range(NB * bs) if r not in set(int(s) for s in slots if s >= 0)]
    for a, b in zip(flat, flat_old):
        assert np.array_equal(a[untouched], b[untouched])


def check_dequantized_cache(m):
    """The cache attention reads: element [b, r, h, d] = code[b, r, h, d] * scale[b, h, r]."""
    rng = np.random.default_rng(12)
    codes = rng.integers(-127, 128, size=(3, 4, 2, 8)).astype(np.int8)
    scales = rng.random((3, 2, 4)).astype(np.float32)
    deq = m.dequantized_cache(codes, scales)
    for b, r, h, d in [(0, 0, 0, 0), (2, 3, 1, 7), (1, 2, 0, 5), (2, 1, 1, 0)]:
        assert deq[b, r, h, d] == float(codes[b, r, h, d]) * float(scales[b, h, r])


ALL_CHECKS = [check_amax_maps_to_127, check_half_step_bound, check_zero_and_single_element_rows,
              check_grid_rows_exact, check_torch_quantizer_agrees, check_write_places_rows,
              check_dequantized_cache]


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda f: f.__name__)
def test_kv_quant_oracle_pin(check):
    check(oq)


MUTATIONS = {
    "floor_not_round": ("np.clip(np.rint(prod)", "np.clip(np.floor(prod)"),
    "qmax_128": ("QMAX = 127", "QMAX = 128"),
    "scale_from_mean": ("amax = np.max(np.abs(xf), axis=-1)", "amax = np.mean(np.abs(xf), axis=-1)"),
    "scale_not_divided": ("scales[nz] = amax[nz] / np.float32(QMAX)", "scales[nz] = amax[nz]"),
    "row_uses_block_index": ("blk, row = slot // bs, slot % bs", "blk, row = slot // bs, (slot // bs) % bs"),
    "v_scale_from_k": ("v_scales[blk, :, row] = vs[t]", "v_scales[blk, :, row] = ks[t]"),
    "scales_not_transposed": ("np.transpose(scales, (0, 2, 1))", "scales.reshape(scales.shape[0], scales.shape[2], "
                              "scales.shape[1])"),
}


def _mutant(name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor missing: {name}"
    mod = types.ModuleType(f"oracle_kv_quant_mutant_{name}")
    mod.__package__ = "oracle"
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_kv_quant_planted_mistake_is_caught(name):
    mod = _mutant(name)
    failed = []
    for check in ALL_CHECKS:
        try:
            with np.errstate(over="ignore", invalid="ignore"):
                check(mod)
        except (AssertionError, IndexError, ValueError, OverflowError):
            failed.append(check.__name__)
    assert failed, f"mutation {name} passed every pin"
