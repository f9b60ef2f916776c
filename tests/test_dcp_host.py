"""The context split's host side on the CPU: the library's split helpers (pa_dcp_owner,
pa_dcp_local_position, pa_dcp_local_lens) against the oracle's split rule, and one decode step of
binding.dcp.dcp_decode over two gloo ranks (the all-gather protocol, each rank's local share built with the
library's block pool) against the oracle's full-context attention.  On the CPU each rank's partial result
and the merge come from the oracle; on a GPU they are the library's kernels (tests/test_gpu_dcp.py)."""

from __future__ import annotations

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import context_split as ocs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pa = pytest.importorskip("paged_kv_cache_330_b200")
from paged_kv_cache_330_b200 import dcp  # noqa: E402


@pytest.mark.parametrize("bs", [16, 32, 256])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_split_helpers_match_oracle(bs, world):
    lens = np.array([0, 1, bs - 1, bs, bs + 1, 3 * bs, 1000, 4097, 8192, 777], dtype=np.int32)
    for r in range(world):
        got = dcp.local_lens(lens, bs, world, r)
        ref = [ocs.local_len(int(L), bs, world, r) for L in lens]
        assert got.tolist() == ref
    for L in (1, 5 * bs + 3, 1000):
        for p in range(L):
            r = dcp.owner(p, bs, world)
            pos = ocs.shard_positions(L, bs, world, r)
            assert dcp.local_position(p, bs, world) == int(np.searchsorted(pos, p)) and pos[np.searchsorted(pos, p)] == p


def test_split_helpers_reject_bad_arguments():
    assert lib_status(pa.lib.pa_dcp_owner(-1, 16, 2)) < 0
    assert lib_status(pa.lib.pa_dcp_owner(5, 0, 2)) < 0
    assert pa.lib.pa_dcp_local_position(5, 16, 0) < 0
    with pytest.raises(pa.PagedAttnError):
        dcp.local_lens([10], 16, 2, 2)         # rank outside the world
    with pytest.raises(pa.PagedAttnError):
        dcp.local_lens([-3], 16, 2, 0)         # negative length


def lib_status(x):
    return int(x)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_partial(q, k, v, bt, lens, max_len, scale):
    out, lse = ocs.shard_partials(q, k, v, bt, lens, scale, 1, 0)   # attention over all the rows given
    return torch.from_numpy(out), torch.from_numpy(lse)


def _oracle_merge(parts, lses):
    return torch.from_numpy(ocs.merge_states(parts.numpy(), lses.numpy()))


def _rank_main(rank, world, port, q_out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    from tests.dcp_shards import local_share
    from tests.gpu_common import oracle_step
    from workloads import make_custom
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        wl = make_custom(seed=31, lens=[1, 15, 16, 17, 300, 1000, 0, 64], num_q_heads=8, num_kv_heads=2, head_dim=64,
                         block_size=16)
        kc, vc, bt, lens, _ = oracle_step(wl)                 # the global caches after this step's write
        kl, vl, btl, lensl = local_share(kc.double(), vc.double(), bt, lens, world, rank)
        out = dcp.dcp_decode(wl.q.double(), kl, vl, btl, lensl, int(lensl.max()), wl.scale,
                             partial=_oracle_partial, merge=_oracle_merge)
        q_out.put((rank, out.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_dcp_decode_gloo_ranks(world):
    from oracle import attention as oatt
    from tests.gpu_common import oracle_step
    from workloads import make_custom
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(world):        # read the results before joining: a child holding queued data cannot exit
            r, out = q.get(timeout=180)
            got[r] = out
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    for p in procs:
        assert p.exitcode == 0, f"rank exited with {p.exitcode}"
    wl = make_custom(seed=31, lens=[1, 15, 16, 17, 300, 1000, 0, 64], num_q_heads=8, num_kv_heads=2, head_dim=64,
                     block_size=16)
    kc, vc, bt, lens, _ = oracle_step(wl)
    ref = oatt.decode_attention(wl.q, kc, vc, bt, lens, wl.scale)
    for r in range(world):                                 # every rank ends with the whole result
        np.testing.assert_allclose(got[r], ref, rtol=1e-10, atol=1e-12)
