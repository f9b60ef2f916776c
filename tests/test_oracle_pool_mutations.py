"""Planted mistakes in a copy of the block-pool oracle (on the CPU) must each fail at least one pool pin
(tests/pool_checks.py): a round-down block count, a fork that does not count its references, no
copy-on-write, a copy that leaves the old block's count, a slot that forgets the block size, a free that
never returns a block, an exhaustion check that lets a pool run dry."""

from __future__ import annotations

import os
import types

import pytest

from tests import pool_checks

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "block_pool.py")

MUTATIONS = {
    "blocks_round_down": ("return -(-n_tokens // block_size)", "return n_tokens // block_size"),
    "fork_without_refcount": ("        for b in shared:\n            self.ref[b] += 1\n", ""),
    "no_copy_on_write": ("cow = n_tokens > 0 and n0 % bs != 0 and self.ref[s[\"blocks\"][-1]] > 1",
                         "cow = False"),
    "copy_keeps_old_count": ("            self.ref[old] -= 1\n", ""),
    "slot_without_block_size": ("slots.append(s[\"blocks\"][p // bs] * bs + p % bs)",
                                "slots.append(s[\"blocks\"][p // bs] + p % bs)"),
    "free_never_returns": ("            if self.ref[b] == 0:\n                self.free.append(b)\n", ""),
    "exhaustion_off_by_one": ("        if need > len(self.free):\n            raise OutOfBlocks(\"alloc\")",
                              "        if need > len(self.free) + 1:\n            raise OutOfBlocks(\"alloc\")"),
}


def _mutant(name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor missing or ambiguous: {name}"
    mod = types.ModuleType(f"oracle_block_pool_mutant_{name}")
    mod.__package__ = "oracle"
    exec(compile(src.replace(old, new), f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pool_planted_mistake_is_caught(name):
    mod = _mutant(name)
    failed = []
    for check in pool_checks.ALL_CHECKS:
        try:
            check(mod)
        except (AssertionError, IndexError, KeyError, ValueError):
            failed.append(check.__name__)
    assert failed, f"mutation {name} passed every pin"
