"""Pins of the context-split oracle (oracle/context_split.py) to facts outside itself, and planted mistakes
that each must fail at least one pin.

The pins: the shards of all ranks partition every sequence's tokens; the page's 1000-token sequence in
16-token blocks over dcp = 3 ranks splits 336 / 336 / 328 (63 blocks: 21, 21 and 21 of which the last holds
8 tokens); each rank's log-sum-exp equals torch.logsumexp of the same scores and its normalised output
equals torch's float64 scaled_dot_product_attention over its rows; merging every rank's parts gives the
full-context attention (torch SDPA and the oracle's own decode) for any world size; and the merge ignores
empty parts, keeps a single part, and stays finite for logits far outside exp's range.
"""

from __future__ import annotations

import os
import types

import numpy as np
import pytest
import torch

from oracle import attention as att
from oracle import context_split as cs

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "context_split.py")


def _case(seed, B=3, Hq=8, Hkv=2, D=64, bs=16, lo=1, hi=200, q_scale=1.0):
    g = torch.Generator().manual_seed(seed)
    lens = torch.randint(lo, hi + 1, (B,), generator=g).numpy()
    nblk = [-(-int(L) // bs) for L in lens]
    NB = sum(nblk) + 3
    perm = torch.randperm(NB, generator=g).numpy()
    bt = np.full((B, max(nblk)), -1, dtype=np.int64)
    i = 0
    for b, n in enumerate(nblk):
        bt[b, :n] = perm[i:i + n]
        i += n
    kc = torch.randn(NB, bs, Hkv, D, generator=g, dtype=torch.float64)
    vc = torch.randn(NB, bs, Hkv, D, generator=g, dtype=torch.float64)
    q = torch.randn(B, Hq, D, generator=g, dtype=torch.float64) * q_scale
    return q, kc, vc, bt, lens


def check_shards_partition(m):
    for L in (0, 1, 15, 16, 17, 100, 257, 1000):
        for bs in (16, 64):
            for W in (1, 2, 3, 4, 8):
                parts = [m.shard_positions(L, bs, W, r) for r in range(W)]
                allp = np.sort(np.concatenate(parts)) if parts else np.zeros(0)
                assert np.array_equal(allp, np.arange(L))
                assert sum(len(p) for p in parts) == L
                sizes = [m.local_len(L, bs, W, r) for r in range(W)]
                assert max(sizes) - min(sizes) <= bs
                for r, p in enumerate(parts):   # every position of a block sits with the block's rank
                    assert all(((t // bs) % W) == r for t in p)


def check_page_example_split(m):
    """1000 tokens, 16-token blocks ("Nano-vLLM-Ascend..." section 2.1) over dcp = 3 ("In-depth analysis of
    vllm-ascend" section 3.1): blocks 0, 3, ..., 60 and 1, 4, ..., 61 are full (21 x 16 = 336 each); rank 2
    holds blocks 2, 5, ..., 62, of which block 62 holds tokens 992..999 (20 x 16 + 8 = 328)."""
    assert [m.local_len(1000, 16, 3, r) for r in range(3)] == [336, 336, 328]
    assert m.shard_positions(1000, 16, 3, 2)[-1] == 999 and m.shard_positions(1000, 16, 3, 0)[16] == 48


def check_lse_matches_torch_logsumexp(m):
    q, kc, vc, bt, lens = _case(1)
    for W in (1, 3):
        for r in range(W):
            outs, lses = m.shard_partials(q, kc, vc, bt, lens, 0.125, W, r)
            for b in range(q.shape[0]):
                pos = m.shard_positions(int(lens[b]), 16, W, r)
                K = att.gather_kv(kc.numpy(), bt[b], int(lens[b]))[pos]
                V = att.gather_kv(vc.numpy(), bt[b], int(lens[b]))[pos]
                for h in range(q.shape[1]):
                    g = h // 4
                    s = 0.125 * (torch.from_numpy(K[:, g]) @ q[b, h])
                    if len(pos) == 0:
                        assert lses[b, h] == -np.inf and (outs[b, h] == 0).all()
                        continue
                    assert lses[b, h] == pytest.approx(float(torch.logsumexp(s, 0)), rel=1e-12, abs=1e-12)
                    ref = torch.nn.functional.scaled_dot_product_attention(
                        q[b, h][None, None, None], torch.from_numpy(K[:, g])[None, None],
                        torch.from_numpy(V[:, g])[None, None], scale=0.125)[0, 0, 0].numpy()
                    np.testing.assert_allclose(outs[b, h], ref, rtol=1e-10, atol=1e-12)


def check_merge_equals_full_attention(m):
    for seed, W in ((2, 1), (3, 2), (4, 3), (5, 4), (6, 8)):
        q, kc, vc, bt, lens = _case(seed, hi=300)
        parts = [m.shard_partials(q, kc, vc, bt, lens, 0.2, W, r) for r in range(W)]
        got = m.merge_states([p[0] for p in parts], [p[1] for p in parts])
        ref = att.decode_attention(q, kc, vc, bt, lens, 0.2)
        np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-12)
        for b in range(q.shape[0]):   # and torch's SDPA over the contiguous sequence
            L = int(lens[b])
            K = torch.from_numpy(att.gather_kv(kc.numpy(), bt[b], L)).permute(1, 0, 2)[None]
            V = torch.from_numpy(att.gather_kv(vc.numpy(), bt[b], L)).permute(1, 0, 2)[None]
            sd = torch.nn.functional.scaled_dot_product_attention(q[b][None, :, None], K, V, scale=0.2,
                                                                  enable_gqa=True)[0, :, 0].numpy()
            np.testing.assert_allclose(got[b], sd, rtol=1e-10, atol=1e-12)


def check_merge_special_cases(m):
    rng = np.random.default_rng(7)
    o = rng.standard_normal((1, 5, 4, 32))
    l = rng.standard_normal((1, 5, 4))
    np.testing.assert_allclose(m.merge_states(o, l), o[0], rtol=1e-14)          # a single part
    o2 = np.concatenate([o, rng.standard_normal((1, 5, 4, 32)) * 1e6])
    l2 = np.concatenate([l, np.full((1, 5, 4), -np.inf)])
    np.testing.assert_allclose(m.merge_states(o2, l2), o[0], rtol=1e-14)        # an empty part adds nothing
    assert (m.merge_states(o2[:1] * 0 + 3, np.full((1, 5, 4), -np.inf)) == 0).all()  # all parts empty -> 0
    # two parts: the weights are softmax(lse) (torch.softmax over the parts' log-sum-exps)
    o3 = rng.standard_normal((2, 3, 16))
    l3 = rng.standard_normal((2, 3)) * 5
    w = torch.softmax(torch.from_numpy(l3), dim=0).numpy()
    np.testing.assert_allclose(m.merge_states(o3, l3), (w[..., None] * o3).sum(0), rtol=1e-12)


def check_large_logits_stay_finite(m):
    q, kc, vc, bt, lens = _case(8, q_scale=300.0, hi=120)
    parts = [m.shard_partials(q, kc, vc, bt, lens, 1.0, 2, r) for r in range(2)]
    assert np.isfinite(np.concatenate([p[1][np.isfinite(p[1])] for p in parts])).all()
    got = m.merge_states([p[0] for p in parts], [p[1] for p in parts])
    assert np.isfinite(got).all()
    np.testing.assert_allclose(got, att.decode_attention(q, kc, vc, bt, lens, 1.0), rtol=1e-9, atol=1e-9)


ALL_CHECKS = [check_shards_partition, check_page_example_split, check_lse_matches_torch_logsumexp,
              check_merge_equals_full_attention, check_merge_special_cases, check_large_logits_stay_finite]


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda c: c.__name__)
def test_context_split_oracle_pin(check):
    check(cs)


MUTATIONS = {
    "owner_from_row_not_block": ("t[(t // block_size) % world == rank]", "t[(t % block_size) % world == rank]"),
    "owner_shifted": ("t[(t // block_size) % world == rank]", "t[(t // block_size + 1) % world == rank]"),
    "lse_without_max": ("lse[h] = mx + np.log(e.sum())", "lse[h] = np.log(e.sum())"),
    "merge_without_max": ("w = np.where(np.isfinite(lses), np.exp(lses - Ms[None]), 0.0)",
                          "w = np.where(np.isfinite(lses), np.exp(lses), 0.0)"),
    "merge_not_normalised": ("res[finite] = num[finite] / den[finite][..., None]", "res[finite] = num[finite]"),
    "partial_not_normalised": ("out[h] = (e / e.sum()) @ V[:, g, :]", "out[h] = e @ V[:, g, :]"),
}


def _mutant(name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor missing: {name}"
    src = src.replace(old, new).replace("from .attention import", "from oracle.attention import")
    mod = types.ModuleType(f"oracle_context_split_mutant_{name}")
    exec(compile(src, f"<mutant {name}>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name):
    mod = _mutant(name)
    failed = []
    for check in ALL_CHECKS:
        try:
            with np.errstate(all="ignore"):
                check(mod)
        except (AssertionError, IndexError, ValueError, FloatingPointError):
            failed.append(check.__name__)
    assert failed, f"mutation {name} passed every pin"
