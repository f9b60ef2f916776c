"""The seeded input generators (workloads/): structure only — lengths in their ranges, a free list that is a
permutation of the pool, one row of new K/V per written token, each new token's position equal to its index
in the sequence, distinct slots and in-range positions for the rotary cases, and the same draws for the
same seed."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from workloads import CONFIGS, make_custom, make_rope_case, make_workload, new_token_positions, rope_tables


@pytest.mark.parametrize("name", ["tiny", "qwen_decode"])
def test_decode_workload_structure(name):
    wl = make_workload(name)
    c = CONFIGS[name]
    assert wl.batch == c["batch"] and len(wl.context_lens) == wl.batch
    assert (wl.context_lens >= c["len_lo"]).all() and (wl.context_lens <= c["len_hi"]).all()
    assert sorted(wl.free_order.tolist()) == list(range(wl.num_blocks))
    assert wl.k_new.shape == (wl.batch, c["num_kv_heads"], c["head_dim"]) == wl.v_new.shape
    assert wl.q.shape == (wl.batch, c["num_q_heads"], c["head_dim"])
    # decode: the written token is the last of its sequence
    assert np.array_equal(new_token_positions(wl), wl.context_lens.astype(np.int64) - 1)


def test_prefill_workload_positions():
    wl = make_workload("prefill")
    C, L = CONFIGS["prefill"]["chunk_len"], CONFIGS["prefill"]["ctx_len"] + CONFIGS["prefill"]["chunk_len"]
    pos = new_token_positions(wl)
    assert pos.shape == (wl.batch * C,) == (wl.k_new.shape[0],)
    for b in range(wl.batch):
        assert np.array_equal(pos[b * C:(b + 1) * C], np.arange(L - C, L))
    assert np.array_equal(np.diff(wl.query_start_loc), np.full(wl.batch, C))


def test_prefix_workload_positions():
    wl = make_workload("prefix_sweep")
    assert np.array_equal(new_token_positions(wl), wl.context_lens.astype(np.int64) - 1)


def test_custom_ragged_prefill_positions():
    wl = make_custom(seed=3, lens=[300, 1, 129], chunk_lens=[200, 1, 129], kind="prefill", num_q_heads=4,
                     num_kv_heads=2, head_dim=64, block_size=16)
    assert np.array_equal(new_token_positions(wl), np.r_[np.arange(100, 300), [0], np.arange(0, 129)])


def test_rope_case_structure():
    c = make_rope_case(seed=1, num_tokens=500, num_q_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                       num_blocks=40, max_position=1000, skip_frac=0.2)
    pos, slots = c.positions.numpy(), c.slots.numpy()
    assert pos.dtype == np.int64 and slots.dtype == np.int64
    assert pos[0] == 0 and pos[-1] == 999 and ((pos >= 0) & (pos < 1000)).all()
    live = slots[slots >= 0]
    assert len(np.unique(live)) == len(live) and (live < 40 * 16).all()
    assert 0.1 < (slots < 0).mean() < 0.3
    assert c.cos.shape == c.sin.shape == (1000, 64) and c.cos.dtype == torch.float32


def test_rope_tables_are_unit_rotations():
    cos, sin = rope_tables(64, 128)
    r = cos.double() ** 2 + sin.double() ** 2
    assert torch.allclose(r, torch.ones_like(r), atol=1e-6)
    assert torch.equal(cos[0], torch.ones(64)) and torch.equal(sin[0], torch.zeros(64))


def test_same_seed_same_draws():
    a, b = make_workload("tiny"), make_workload("tiny")
    assert torch.equal(a.q, b.q) and torch.equal(a.k_cache0, b.k_cache0) and np.array_equal(a.free_order, b.free_order)
    c = make_workload("tiny", seed=99)
    assert not torch.equal(a.q, c.q)
