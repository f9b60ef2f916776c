"""Decode through the allocation-free entry point (pa_decode_static_scratch).

Callers that cannot allocate device memory where they run decode (inside CUDA
graph capture, under a fixed memory pool, on a serving path that must not
block) use the library's static device scratch instead of a workspace.  This
file runs last so that a failure here comes after every other test has run;
it also passes on its own in a fresh process, where the first call sets up
the scratch address.
"""

from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from tests.gpu_common import assert_close, gpu_step, oracle_step
from workloads import make_workload

pa = pytest.importorskip("paged_kv_cache_330_b200")

STATIC_SCRATCH_BYTES = 8 << 20  # PA_DECODE_STATIC_SCRATCH_BYTES in include/paged_attn.h


def test_oversized_plan_exceeds_static_scratch():
    """The batch used below to test the refusal really needs more than the static scratch (no GPU needed)."""
    need = pa.lib.pa_decode_workspace_size(1 << 16, 16, 8, 128, 100, 0)
    assert need > STATIC_SCRATCH_BYTES


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["qwen_decode", "llama70b_long"])
def test_static_scratch_decode_matches_workspace_decode(name):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    wl = make_workload(name)
    ref, kc, vc, bt, lens, bt_h, lens_h = gpu_step(wl)           # pa_write_kv + pa_decode (caller workspace)
    ref = ref.float().cpu().numpy().astype(np.float64)
    maxL = int(lens_h.max())
    q = wl.q.cuda()
    for _ in range(2):                                            # two calls in a row share the static scratch
        out = torch.full_like(q, float("nan"))
        pa.decode_static_scratch(q, kc, vc, bt, lens, maxL, wl.scale, out=out)
        torch.cuda.synchronize()
        assert_close(out.float().cpu().numpy(), ref, f"{name} static scratch")
    assert pa.device_error() == 0


@pytest.mark.gpu
def test_static_scratch_decode_matches_oracle():
    """The whole Qwen3-0.6B-shaped batch (every row) against the fp64 oracle, twice in a row."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    wl = make_workload("qwen_decode")
    _, kc, vc, bt, lens, _, lens_h = gpu_step(wl)
    okc, ovc, rows, olens, _ = oracle_step(wl)
    ref = oatt.decode_attention(wl.q, okc, ovc, rows, olens, wl.scale)
    q = wl.q.cuda()
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        pa.decode_static_scratch(q, kc, vc, bt, lens, int(lens_h.max()), wl.scale, out=out)
        torch.cuda.synchronize()
        assert_close(out.float().cpu().numpy(), ref, "qwen_decode static scratch vs oracle")
    assert pa.device_error() == 0


@pytest.mark.gpu
def test_static_scratch_rejects_oversized_batch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    null = ctypes.c_void_p(0)                                      # no tensor: a regressed check cannot launch
    big_batch = 1 << 16                                            # needs far more than the static scratch
    st = pa.lib.pa_decode_static_scratch(null, null, null, null, 8, null, big_batch, 16, 8, 128, 16, 16, 100, 0.1,
                                         1, 0, null, null)
    assert st == -4                                                # PA_ERR_WORKSPACE, nothing launched


@pytest.mark.gpu
def test_static_scratch_rejected_call_enqueues_nothing():
    """A call refused by the argument checks (a null q) returns PA_ERR_INVALID before anything is enqueued,
    and the next accepted call is still correct."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    wl = make_workload("tiny")
    ref, kc, vc, bt, lens, _, lens_h = gpu_step(wl)
    torch.cuda.synchronize()
    out = torch.full_like(ref, float("nan"))
    NB, bs, Hkv, D = kc.shape
    st = pa.lib.pa_decode_static_scratch(ctypes.c_void_p(0), ctypes.c_void_p(kc.data_ptr()),
                                         ctypes.c_void_p(vc.data_ptr()), ctypes.c_void_p(bt.data_ptr()),
                                         int(bt.shape[1]), ctypes.c_void_p(lens.data_ptr()), wl.batch,
                                         wl.cfg["num_q_heads"], Hkv, D, bs, NB, int(lens_h.max()), wl.scale, 0, 0,
                                         ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(0))
    assert st == -1                                                # PA_ERR_INVALID
    torch.cuda.synchronize()
    assert torch.isnan(out.float()).all()                          # nothing ran
    pa.decode_static_scratch(wl.q.cuda(), kc, vc, bt, lens, int(lens_h.max()), wl.scale, out=out)
    torch.cuda.synchronize()
    assert_close(out.float().cpu().numpy(), ref.float().cpu().numpy().astype(np.float64), "tiny static scratch")
    assert pa.device_error() == 0
