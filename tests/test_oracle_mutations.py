"""Planted mistakes in a copy of the oracle (on the CPU) must each fail at least one pin.

This shows the pins are strong enough: a wrong GQA head mapping, a dropped
scale, a wrong gather index, an off-by-one causal limit or a swapped operand
would not slip through.
"""

from __future__ import annotations

import importlib.util
import os
import types

import pytest

from tests import oracle_checks

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "attention.py")

MUTATIONS = {
    "gqa_mod_instead_of_div": ("        g = h // G\n        s = scale", "        g = h % G\n        s = scale"),
    "scale_dropped": ("        s = scale * (K[:, g, :] @ q_heads[h])", "        s = (K[:, g, :] @ q_heads[h])"),
    "gather_row_uses_block_index": ("    return cache[phys, t % bs]", "    return cache[phys, (t // bs) % bs]"),
    "causal_off_by_one": ("last = L - C + i ", "last = L - C + i - 1 "),
    "pv_uses_keys": ("        out[h] = (p / p.sum()) @ V[:, g, :]", "        out[h] = (p / p.sum()) @ K[:, g, :]"),
    "softmax_not_normalised": ("        out[h] = (p / p.sum()) @ V[:, g, :]", "        out[h] = p @ V[:, g, :]"),
    "block_lookup_off_by_one": ("[t // bs]\n    return", "[(t // bs + 1) % len(block_table_row)]\n    return"),
}


def _mutant(name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor missing: {name}"
    src = src.replace(old, new)
    mod = types.ModuleType(f"oracle_attention_mutant_{name}")
    exec(compile(src, f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name):
    mod = _mutant(name)
    failed = []
    for check in oracle_checks.ALL_CHECKS:
        try:
            check(mod)
        except AssertionError:
            failed.append(check.__name__)
        except (IndexError, ValueError, FloatingPointError):
            failed.append(check.__name__)
    assert failed, f"mutation {name} passed every pin"
