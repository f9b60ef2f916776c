"""Decode through the allocation-free entry point (pa_decode_static_scratch) matches pa_decode.

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

from tests.gpu_common import assert_close, gpu_step
from workloads import make_workload

pytestmark = pytest.mark.gpu

pa = pytest.importorskip("paged_kv_cache_330_b200")


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


def test_static_scratch_rejects_oversized_batch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    fake = ctypes.c_void_p(0x10000)
    big_batch = 1 << 16                                            # needs far more than the static scratch
    st = pa.lib.pa_decode_static_scratch(fake, fake, fake, fake, 8, fake, big_batch, 16, 8, 128, 16, 16, 100, 0.1,
                                         1, 0, fake, ctypes.c_void_p(0))
    assert st == -4                                                # PA_ERR_WORKSPACE, nothing launched
