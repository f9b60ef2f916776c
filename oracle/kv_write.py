"""Writing new tokens' K/V into their cache slots, as bytes (oracle; test infrastructure only).

The cache is stacked from the per-block layout of the Block structure on the
page "Nano-vLLM-Ascend: lightweight LLM inference framework for Ascend NPU",
section 2.1: each block holds ``[block_size, num_heads, head_dim]`` for K and
the same for V, so the pool is ``[num_blocks, block_size, num_kv_heads,
head_dim]``.  Slot s is block s // block_size, row s % block_size.  A slot of
-1 means "no write" (padding).  The copy is bitwise: fp16/bf16 values are
moved as 16-bit words, never converted.
"""

from __future__ import annotations

import numpy as np


def write_kv(k_new: np.ndarray, v_new: np.ndarray, slot_mapping, k_cache: np.ndarray, v_cache: np.ndarray) -> None:
    """In place: cache[slot // bs, slot % bs] = new row, for every slot >= 0.

    Arrays are raw 16-bit words (``np.uint16``); k_new/v_new are [T, Hkv, D],
    caches [num_blocks, block_size, Hkv, D].
    """
    assert k_new.dtype == np.uint16 and k_cache.dtype == np.uint16
    bs = k_cache.shape[1]
    for t, slot in enumerate(slot_mapping):
        slot = int(slot)
        if slot < 0:
            continue
        k_cache[slot // bs, slot % bs] = k_new[t]
        v_cache[slot // bs, slot % bs] = v_new[t]
