"""INT8 KV cache: per-row symmetric quantisation on write, dequantisation on read (oracle; test
infrastructure only).

The pages list KV-cache compression and INT8 quantisation among the advanced
optimisations ("Nano-vLLM-Ascend: lightweight LLM inference framework for
Ascend NPU", section 4.3, tuning checklist) and name INT8 as the way to raise
throughput beyond the FP16-only operator, once the accuracy of the attention
scores after quantisation is handled ("Ascend NPU LLM inference optimisation:
the vLLM-Ascend approach", section 5).  They give no format.  Reading taken
here, the plainest one that needs no re-quantisation when a token is appended
to a partly filled block: every (token, KV head) row of D values gets its own
fp32 scale, symmetric, absmax; the scores are formed in fp32 or better from
the dequantised values, so only the stored K/V carry the quantisation error:

    amax    = max_d |x_d|                       (x: the 16-bit value, exact in fp32)
    inv     = 127 / amax   in fp32              (0 when amax == 0)
    code_d  = round_half_even(fp32(x_d * inv)), clamped to [-127, 127], int8
    scale   = amax / 127   in fp32              (0 when amax == 0)
    x_d    ~= code_d * scale

The codes are integers decided by floating point, so they are computed here
with the same fp32 operations in the same order that a device kernel uses
(an IEEE fp32 division, an fp32 multiply, round to nearest even): numpy's
float32 arithmetic is IEEE, so both sides reach the same codes bit for bit.
Attention over the quantised cache is the plain definition of
``attention.py`` applied to the dequantised rows, in float64.
"""

from __future__ import annotations

import numpy as np

QMAX = 127


def quantize_rows(x) -> tuple[np.ndarray, np.ndarray]:
    """x [..., D] (fp16/bf16 values as float32, or anything exactly representable in fp32).

    Returns (codes int8 [..., D], scales float32 [...]): one scale per row of the last axis."""
    xf = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(xf), axis=-1)
    nz = amax > 0
    inv = np.zeros_like(amax)
    inv[nz] = np.float32(QMAX) / amax[nz]                      # fp32 IEEE division
    prod = (xf * inv[..., None]).astype(np.float32)            # fp32 multiply
    codes = np.clip(np.rint(prod), -QMAX, QMAX).astype(np.int8)  # np.rint rounds half to even
    scales = np.zeros_like(amax)
    scales[nz] = amax[nz] / np.float32(QMAX)                   # fp32 IEEE division
    return codes, scales.astype(np.float32)


def dequantize_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """code * scale per element, float64 (exact: an int8 times an fp32 fits a double)."""
    return np.asarray(codes, dtype=np.float64) * np.asarray(scales, dtype=np.float64)[..., None]


def write_kv_int8(k_new, v_new, slot_mapping, k_codes: np.ndarray, v_codes: np.ndarray,
                  k_scales: np.ndarray, v_scales: np.ndarray) -> None:
    """In place: quantise each new token's K and V rows (per KV head) into the INT8 caches.

    k_new/v_new [T, Hkv, D] (16-bit values as float32); code caches int8 [NB, bs, Hkv, D], laid out like
    the 16-bit caches; scale caches float32 [NB, Hkv, bs], so that the scales of consecutive tokens of one
    head are contiguous (a 16-token chunk's scales are one 64-byte run).  Slot s is block s // bs, row
    s % bs; a slot of -1 writes nothing."""
    bs = k_codes.shape[1]
    kq, ks = quantize_rows(k_new)
    vq, vs = quantize_rows(v_new)
    for t, slot in enumerate(slot_mapping):
        slot = int(slot)
        if slot < 0:
            continue
        blk, row = slot // bs, slot % bs
        k_codes[blk, row] = kq[t]
        v_codes[blk, row] = vq[t]
        k_scales[blk, :, row] = ks[t]
        v_scales[blk, :, row] = vs[t]


def dequantized_cache(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """The float64 cache [NB, bs, Hkv, D] that attention over the INT8 cache reads (scales [NB, Hkv, bs])."""
    return dequantize_rows(codes, np.transpose(scales, (0, 2, 1)))
