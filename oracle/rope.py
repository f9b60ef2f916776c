"""Rotary position embedding fused with the KV write (oracle; test infrastructure only).

The page "Nano-vLLM-Ascend: lightweight LLM inference framework for Ascend
NPU" has every model supply its own rotary embedding (section 3.1, model
adaptation) and builds it as a custom device operator in section 5.1: a
rotary multiply of x by per-position cos and sin tables, whose gradient is the
same operator with sin negated, i.e. the inverse rotation.

The pages do not say which elements of a head form a rotating pair.  Reading
taken here (the rotate-half form of a rotary multiply over head_dim-wide x):
the first head_dim/2 elements x1 and the second head_dim/2 elements x2 pair
element by element, and pair i turns by the angle whose cosine and sine are
cos[pos][i], sin[pos][i]:

    out[i]         = x1[i] * cos[i] - x2[i] * sin[i]
    out[i + D/2]   = x2[i] * cos[i] + x1[i] * sin[i]

The tables are inputs (one fp32 row of D/2 entries per position), as on the
page, where the operator receives cos and sin rather than an angle schedule.

The fused step applies this to every query head and every key head of each
new token, then stores the rotated keys and the unrotated values into the
token's cache slot (block slot // block_size, row slot % block_size), exactly
as ``kv_write.write_kv`` does for plain K/V.  Everything is float64; the V copy
stays bitwise.
"""

from __future__ import annotations

import numpy as np

from .kv_write import write_kv


def rotary(x: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Rotate-half rotary multiply of x [..., D] by cos/sin [..., D/2] (broadcast over the leading axes)."""
    x = np.asarray(x, dtype=np.float64)
    half = x.shape[-1] // 2
    x1, x2 = x[..., :half], x[..., half:]
    c = np.asarray(cos, dtype=np.float64)
    s = np.asarray(sin, dtype=np.float64)
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def rope_tokens(x: np.ndarray, positions, cos_table: np.ndarray, sin_table: np.ndarray) -> np.ndarray:
    """x [T, H, D]: token t's heads turn by table row positions[t] (every position must index the tables)."""
    pos = np.asarray(positions, dtype=np.int64)
    assert pos.ndim == 1 and pos.shape[0] == x.shape[0]
    assert (pos >= 0).all() and (pos < cos_table.shape[0]).all(), "position outside the cos/sin tables"
    c = np.asarray(cos_table, dtype=np.float64)[pos][:, None, :]   # [T, 1, D/2], shared by all heads
    s = np.asarray(sin_table, dtype=np.float64)[pos][:, None, :]
    return rotary(x, c, s)


def rope_write_kv(q: np.ndarray, k: np.ndarray, v_bits: np.ndarray, positions, cos_table: np.ndarray,
                  sin_table: np.ndarray, slot_mapping, v_cache_bits: np.ndarray):
    """The fused step.

    q [T, Hq, D] and k [T, Hkv, D] as float64 (the 16-bit inputs upcast exactly); v_bits [T, Hkv, D] and
    v_cache_bits [NB, bs, Hkv, D] as raw 16-bit words (``np.uint16``).  Returns (q_rot, k_rot), both
    float64: q_rot is every token's rotated query; k_rot[t] is what slot_mapping[t] receives in the K
    cache (a slot of -1 receives nothing).  V rows are written into v_cache_bits in place, bitwise.
    """
    q_rot = rope_tokens(q, positions, cos_table, sin_table)
    k_rot = rope_tokens(k, positions, cos_table, sin_table)
    dummy = np.zeros_like(v_cache_bits)
    write_kv(v_bits, v_bits, slot_mapping, dummy, v_cache_bits)
    return q_rot, k_rot
