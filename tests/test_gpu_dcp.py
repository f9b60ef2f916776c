"""GPU parity of the context split's kernels through the C ABI: pa_decode_lse (output and log-sum-exp of a
rank's share) and pa_merge_attn_states, against the oracle.  The ranks of a split are emulated one after
another on the one GPU (each rank's share is an ordinary paged cache, so no rank waits on another); the
stacked per-rank results stand for the all-gather."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from oracle import context_split as ocs
from tests.dcp_shards import local_share
from tests.gpu_common import assert_close, gpu_step, oracle_step
from workloads import make_custom, make_workload

pytestmark = pytest.mark.gpu

pa = pytest.importorskip("paged_kv_cache_330_b200")

# |lse_gpu - lse_oracle| <= LSE_ATOL + LSE_RTOL |lse|: fp32 scores over head_dim products (relative ~D 2^-24
# of sum |q_d k_d| scale) and the MUFU exp2/log2 (~2^-22) give errors of order 1e-5 at these logit sizes.
LSE_ATOL, LSE_RTOL = 1e-3, 1e-4


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    assert pa.device_error() == 0, "a kernel recorded a device-side error"


def _check_lse(got, ref, what):
    got = np.asarray(got, dtype=np.float64)
    inf = ~np.isfinite(ref)
    assert (got[inf] == -np.inf).all(), f"{what}: empty rows must give -inf"
    err = np.abs(got[~inf] - ref[~inf])
    assert (err <= LSE_ATOL + LSE_RTOL * np.abs(ref[~inf])).all(), f"{what}: lse max err {err.max():.3e}"


@pytest.mark.parametrize("name", ["tiny", "qwen_decode"])
def test_decode_lse_whole_context(name):
    """One rank holding everything: out equals pa_decode's result and the oracle; lse equals the oracle's."""
    wl = make_workload(name)
    out_ref, kc, vc, bt, lens, bt_h, lens_h = gpu_step(wl)
    out, lse = pa.decode_lse(wl.q.cuda(), kc, vc, bt, lens, int(lens_h.max()), wl.scale)
    okc, ovc, rows, olens, _ = oracle_step(wl)
    ro, rl = ocs.shard_partials(wl.q, okc, ovc, rows, olens, wl.scale, 1, 0)
    assert torch.equal(out.view(torch.int16), out_ref.view(torch.int16))
    assert_close(out.float().cpu().numpy(), ro, f"{name} decode_lse out")
    _check_lse(lse.cpu().numpy(), rl, name)


def _split_case(wl, world, rows=None):
    """Emulated split: every rank's share decoded with pa_decode_lse, then pa_merge_attn_states."""
    _, kc, vc, bt, lens, bt_h, lens_h = gpu_step(wl)
    okc, ovc, orows, olens, _ = oracle_step(wl)
    q = wl.q.cuda()
    parts, lses = [], []
    for r in range(world):
        kl, vl, btl, lensl = local_share(kc, vc, bt_h, lens_h, world, r, free_order_seed=world)
        o, l = pa.decode_lse(q, kl, vl, torch.from_numpy(btl).cuda(), torch.from_numpy(lensl).cuda(),
                             int(lensl.max()), wl.scale, num_partitions=0 if r % 2 == 0 else 37)
        ro, rl = ocs.shard_partials(wl.q, okc, ovc, orows, olens, wl.scale, world, r) if rows is None else (None, None)
        if ro is not None:
            assert_close(o.float().cpu().numpy(), ro, f"rank {r} of {world} out")
            _check_lse(l.cpu().numpy(), rl, f"rank {r} of {world}")
        parts.append(o)
        lses.append(l)
    merged = pa.merge_attn_states(torch.stack(parts), torch.stack(lses))
    torch.cuda.synchronize()
    if rows is None:
        ref = oatt.decode_attention(wl.q, okc, ovc, orows, olens, wl.scale)
        assert_close(merged.float().cpu().numpy(), ref, f"merged over {world} ranks")
    else:
        ref = oatt.decode_rows(wl.q, okc, ovc, orows, olens, wl.scale, rows)
        got = np.stack([merged[b, h].float().cpu().numpy() for b, h in rows])
        assert_close(got, ref, f"merged over {world} ranks (sampled)")


@pytest.mark.parametrize("world", [2, 3, 4])
def test_split_ragged_all_rows(world):
    wl = make_custom(seed=40 + world, lens=[0, 1, 15, 16, 17, 47, 48, 49, 300, 1000, 2049, 64], num_q_heads=16,
                     num_kv_heads=4, head_dim=128, block_size=16)
    _split_case(wl, world)


@pytest.mark.parametrize("world", [2, 8])
def test_split_llama70b_long_sampled(world):
    wl = make_workload("llama70b_long")
    rng = np.random.default_rng(world)
    rows = sorted({(int(rng.integers(wl.batch)), int(rng.integers(64))) for _ in range(32)} | {(0, 0), (63, 63)})
    _split_case(wl, world, rows)


@pytest.mark.parametrize("D,dt", [(128, torch.bfloat16), (64, torch.float16)])
def test_merge_kernel_against_oracle(D, dt):
    """Random parts with log-sum-exps spread over +-40, some parts empty (lse -inf, NaN bytes that must not be
    read), and rows where every part is empty."""
    g = torch.Generator().manual_seed(D)
    P, B, H = 5, 33, 6
    parts = torch.randn(P, B, H, D, generator=g).to(dt)
    lses = (torch.rand(P, B, H, generator=g) * 80 - 40).float()
    empty = torch.rand(P, B, H, generator=g) < 0.3
    lses[empty] = -float("inf")
    parts[empty] = float("nan")
    lses[:, 7] = -float("inf")
    out = pa.merge_attn_states(parts.cuda(), lses.cuda())
    pf = parts.double().numpy()
    pf[empty.numpy()] = 0.0          # the oracle's merge multiplies; an empty part's bytes are not data
    ref = ocs.merge_states(pf, lses.double().numpy())
    got = out.float().cpu().numpy()
    assert (got[7] == 0).all()
    assert_close(got, ref, f"merge D{D}")
