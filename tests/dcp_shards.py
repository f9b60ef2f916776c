"""Test harness for the context split: build one rank's local share of a workload's global step (its own
block pool from the library, its local block tables and lengths, and its local caches filled with the
global rows it holds).  Index bookkeeping only; no attention arithmetic."""

from __future__ import annotations

import numpy as np
import torch


def local_share(global_k, global_v, global_bt, global_lens, world: int, rank: int, free_order_seed: int = 0):
    """global_k/global_v [NB, bs, Hkv, D] (any device), global_bt int [B, n], global_lens int [B] (host).

    Returns (k_local, v_local, bt_local int32 [B, m], lens_local int32 [B]) on global_k's device.  The local
    pool is the library's BlockPool with a shuffled free list, so local physical blocks are scattered too."""
    import paged_kv_cache_330_b200 as pa
    from paged_kv_cache_330_b200 import dcp
    NB, bs, Hkv, D = global_k.shape
    lens = np.asarray(global_lens, dtype=np.int32)
    B = len(lens)
    loc = dcp.local_lens(lens, bs, world, rank)
    nb_local = int(sum(-(-int(x) // bs) for x in loc)) + 2
    order = np.random.default_rng(free_order_seed + 17 * rank).permutation(nb_local).astype(np.int32)
    pool = pa.BlockPool(nb_local, bs, order)
    for b in range(B):
        pool.alloc(b, int(loc[b]))
    m = max([-(-int(x) // bs) for x in loc] + [1])
    bt_l, lens_l = pool.block_table(list(range(B)), m)
    pool.close()
    src_rows, dst_rows = [], []
    gbt = np.asarray(global_bt, dtype=np.int64)
    for b in range(B):
        i = np.arange(int(loc[b]))
        p = ((i // bs) * world + rank) * bs + i % bs          # global position of local token i
        src_rows.append(gbt[b][p // bs] * bs + p % bs)
        dst_rows.append(bt_l[b][i // bs].astype(np.int64) * bs + i % bs)
    src = torch.from_numpy(np.concatenate(src_rows) if src_rows else np.zeros(0, np.int64)).to(global_k.device)
    dst = torch.from_numpy(np.concatenate(dst_rows) if dst_rows else np.zeros(0, np.int64)).to(global_k.device)
    kl = torch.zeros((nb_local, bs, Hkv, D), dtype=global_k.dtype, device=global_k.device)
    vl = torch.zeros_like(kl)
    kl.view(-1, Hkv, D)[dst] = global_k.reshape(-1, Hkv, D)[src]
    vl.view(-1, Hkv, D)[dst] = global_v.reshape(-1, Hkv, D)[src]
    return kl, vl, bt_l.astype(np.int32), lens_l.astype(np.int32)
