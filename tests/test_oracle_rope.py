"""Pins of the rotary-embedding oracle (oracle/rope.py) to facts outside itself, and planted mistakes
that each must fail at least one pin.

The pins: a zero angle is the identity; a quarter turn maps (x1, x2) to (-x2, x1) and a half turn to -x
(closed forms of a rotation, which also fix the rotate-half pairing); the page's backward rule (the same
operator with sin negated) undoes the forward one; turns compose by adding angles; each pair keeps its
length; dot products of rotated queries and keys depend only on the position difference; and every
pair equals complex multiplication by e^{i theta} done by torch's complex arithmetic.
"""

from __future__ import annotations

import importlib.util
import os
import types

import numpy as np
import pytest
import torch

from oracle import rope as orope

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "rope.py")


def _angles(rng, n, half):
    return rng.uniform(-np.pi, np.pi, size=(n, half))


def _tables(theta):
    return np.cos(theta), np.sin(theta)


def _schedule(max_pos, D, base=10000.0):
    """Angle table pos * base^(-2i/D), the usual rotary frequency schedule (test input)."""
    inv = base ** (-np.arange(0, D, 2, dtype=np.float64) / D)
    return np.outer(np.arange(max_pos, dtype=np.float64), inv)


# ----------------------------------------------------------------------------------------------- checks
def check_zero_angle_is_identity(m):
    rng = np.random.default_rng(1)
    x = rng.standard_normal((3, 5, 64))
    c, s = np.ones((3, 1, 32)), np.zeros((3, 1, 32))
    assert np.array_equal(m.rotary(x, c, s), x)
    # through the position lookup: table row 0 holds angle 0, other rows do not
    theta = _schedule(16, 64)
    ct, st = _tables(theta)
    assert np.array_equal(m.rope_tokens(x, np.zeros(3, dtype=np.int64), ct, st), x)


def check_quarter_and_half_turn(m):
    rng = np.random.default_rng(2)
    x = rng.standard_normal((4, 2, 128))
    x1, x2 = x[..., :64], x[..., 64:]
    q = m.rotary(x, np.zeros((4, 1, 64)), np.ones((4, 1, 64)))
    assert np.array_equal(q, np.concatenate([-x2, x1], axis=-1))
    h = m.rotary(x, -np.ones((4, 1, 64)), np.zeros((4, 1, 64)))
    assert np.array_equal(h, -x)


def check_backward_rule_inverts(m):
    """The page's gradient is the same operator with sin negated: applied after the forward, x comes back."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((6, 4, 128))
    c, s = _tables(_angles(rng, 6, 64)[:, None, :])
    back = m.rotary(m.rotary(x, c, s), c, -s)
    assert np.allclose(back, x, rtol=0, atol=1e-13)


def check_angles_add(m):
    rng = np.random.default_rng(4)
    x = rng.standard_normal((5, 3, 64))
    a, b = _angles(rng, 5, 32)[:, None, :], _angles(rng, 5, 32)[:, None, :]
    two = m.rotary(m.rotary(x, *_tables(a)), *_tables(b))
    one = m.rotary(x, *_tables(a + b))
    assert np.allclose(two, one, rtol=0, atol=1e-13)


def check_pairs_keep_length(m):
    rng = np.random.default_rng(5)
    x = rng.standard_normal((7, 2, 128))
    y = m.rotary(x, *_tables(_angles(rng, 7, 64)[:, None, :]))
    n0 = x[..., :64] ** 2 + x[..., 64:] ** 2
    n1 = y[..., :64] ** 2 + y[..., 64:] ** 2
    assert np.allclose(n0, n1, rtol=1e-13, atol=1e-13)


def check_relative_position(m):
    """<R(m) q, R(n) k> depends on m - n only (the defining property of rotary embeddings)."""
    rng = np.random.default_rng(6)
    D = 128
    ct, st = _tables(_schedule(4096, D))
    q = rng.standard_normal((1, 1, D))
    k = rng.standard_normal((1, 1, D))
    for mpos, npos, shift in ((100, 37, 900), (5, 4000, 17), (0, 0, 333)):
        a = float(np.sum(m.rope_tokens(q, [mpos], ct, st) * m.rope_tokens(k, [npos], ct, st)))
        b = float(np.sum(m.rope_tokens(q, [mpos + shift], ct, st) * m.rope_tokens(k, [npos + shift], ct, st)))
        assert abs(a - b) <= 1e-9 * (1 + abs(a))


def check_complex_multiplication(m):
    """Pair i is the complex number x1[i] + i x2[i]; the rotation multiplies it by e^{i theta_i}."""
    rng = np.random.default_rng(7)
    x = rng.standard_normal((9, 4, 64))
    theta = _angles(rng, 9, 32)
    z = torch.complex(torch.from_numpy(x[..., :32]), torch.from_numpy(x[..., 32:]))
    w = z * torch.polar(torch.ones(9, 1, 32, dtype=torch.float64), torch.from_numpy(theta[:, None, :]))
    y = m.rotary(x, np.cos(theta)[:, None, :], np.sin(theta)[:, None, :])
    assert np.allclose(y[..., :32], w.real.numpy(), rtol=0, atol=1e-13)
    assert np.allclose(y[..., 32:], w.imag.numpy(), rtol=0, atol=1e-13)


def check_tokens_use_their_own_row(m):
    """Token t turns by table row positions[t], for every head (per-token loop over the rows)."""
    rng = np.random.default_rng(8)
    T, H, D = 11, 3, 64
    x = rng.standard_normal((T, H, D))
    ct, st = _tables(_angles(rng, 50, D // 2))
    pos = rng.integers(0, 50, size=T)
    got = m.rope_tokens(x, pos, ct, st)
    for t in range(T):
        for h in range(H):
            ref = m.rotary(x[t, h][None, None], ct[pos[t]][None, None], st[pos[t]][None, None])[0, 0]
            assert np.array_equal(got[t, h], ref)


def check_fused_step(m):
    """rope_write_kv: rotated q and k per token; V rows land bitwise at cache row `slot` (the pool viewed as
    [num_blocks * block_size] rows), other rows untouched; slot -1 writes nothing."""
    rng = np.random.default_rng(9)
    T, Hq, Hkv, D, NB, bs = 6, 4, 2, 64, 5, 4
    q = rng.standard_normal((T, Hq, D))
    k = rng.standard_normal((T, Hkv, D))
    v = rng.integers(0, 2 ** 16, size=(T, Hkv, D), dtype=np.uint16)
    vc = rng.integers(0, 2 ** 16, size=(NB, bs, Hkv, D), dtype=np.uint16)
    vc0 = vc.copy()
    slots = np.array([7, -1, 0, 19, 12, 3], dtype=np.int64)
    ct, st = _tables(_angles(rng, 30, D // 2))
    pos = np.array([0, 29, 5, 5, 17, 1], dtype=np.int64)
    q_rot, k_rot = m.rope_write_kv(q, k, v, pos, ct, st, slots, vc)
    assert np.array_equal(q_rot, m.rope_tokens(q, pos, ct, st))
    assert np.array_equal(k_rot, m.rope_tokens(k, pos, ct, st))
    rows, rows0 = vc.reshape(NB * bs, Hkv, D), vc0.reshape(NB * bs, Hkv, D)
    written = set()
    for t, s in enumerate(slots):
        if s >= 0:
            assert np.array_equal(rows[s], v[t])
            written.add(int(s))
    for r in range(NB * bs):
        if r not in written:
            assert np.array_equal(rows[r], rows0[r])


ALL_CHECKS = [check_zero_angle_is_identity, check_quarter_and_half_turn, check_backward_rule_inverts,
              check_angles_add, check_pairs_keep_length, check_relative_position, check_complex_multiplication,
              check_tokens_use_their_own_row, check_fused_step]


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda f: f.__name__)
def test_rope_oracle_pin(check):
    check(orope)


# ------------------------------------------------------------------------------------------ planted mistakes
MUTATIONS = {
    "sign_flipped": ("x1 * c - x2 * s", "x1 * c + x2 * s"),
    "turns_backwards": ("[x1 * c - x2 * s, x2 * c + x1 * s]", "[x1 * c + x2 * s, x2 * c - x1 * s]"),
    "interleaved_pairs": ("x1, x2 = x[..., :half], x[..., half:]", "x1, x2 = x[..., 0::2], x[..., 1::2]"),
    "cos_sin_swapped": ("c = np.asarray(cos, dtype=np.float64)\n    s = np.asarray(sin, dtype=np.float64)",
                        "s = np.asarray(cos, dtype=np.float64)\n    c = np.asarray(sin, dtype=np.float64)"),
    "row_off_by_one": ("np.float64)[pos][:, None, :]   #", "np.float64)[pos + 1][:, None, :]   #"),
    "one_table_row_for_all": ("[pos][:, None, :]   #", "[pos[:1]][:, None, :]   #"),
    "v_not_written": ("    write_kv(v_bits, v_bits, slot_mapping, dummy, v_cache_bits)\n", ""),
}


def _mutant(name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor missing: {name}"
    mod = types.ModuleType(f"oracle_rope_mutant_{name}")
    mod.__package__ = "oracle"
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_rope_planted_mistake_is_caught(name):
    mod = _mutant(name)
    failed = []
    for check in ALL_CHECKS:
        try:
            check(mod)
        except (AssertionError, IndexError, ValueError):
            failed.append(check.__name__)
    assert failed, f"mutation {name} passed every pin"
