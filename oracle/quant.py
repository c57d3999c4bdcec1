"""Oracle: symmetric per-group INT4 quantiser, nibble packing, dequant, BF16 rounding.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Passages followed:
  * "Benchmark Comparison" (measured benchmarks), section 7 "Quantization floor":
    symmetric per-group min-max quantisation with no calibration.
  * Same page, section 5 "Asymmetric-correction overhead": the symmetric
    convention W = (q - 8) * scale, i.e. the stored unsigned nibble is offset by 8.
  * "CLI Reference", Environment Variables, TINYLOOP_KV_H_MODE + TINYLOOP_KV_INT4:
    signed 4-bit values in [-7, 7], the even-indexed element in the low nibble
    and the odd-indexed element in the high nibble of each byte.
  * Workload model definitions: group size 32 or 128, one FP16 scale per group.

Readings where the pages are silent: the scale is max|w| / 7 rounded to FP16
(round to nearest even); the code is round-half-even of w / scale, with the
division done in float64 at the FP16 scale's exact value, clamped to [-7, 7];
an all-zero group has scale 0 and codes 0.  Stored nibble u = q + 8 lies in
[1, 15]; a nibble of 0 decodes to -8.
"""
from __future__ import annotations

import numpy as np


def quantize_int4(w: np.ndarray, group: int) -> tuple[np.ndarray, np.ndarray]:
    """w float64 [N, K] -> (packed uint8 [N, K/2], scales float16 [N, K/group])."""
    w = np.asarray(w, dtype=np.float64)
    N, K = w.shape
    if K % group or group % 2:
        raise ValueError("K must be a multiple of an even group size")
    wg = w.reshape(N, K // group, group)
    amax = np.abs(wg).max(axis=2)
    scale = (amax / 7.0).astype(np.float16)          # fp64 -> fp16, round to nearest even
    s = scale.astype(np.float64)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(s > 0, np.clip(np.rint(wg / s), -7, 7), 0.0)
    u = (q.reshape(N, K) + 8).astype(np.uint8)
    packed = (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)
    return packed, scale


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    """uint8 [N, K/2] -> stored nibbles uint8 [N, K] (even element from the low nibble)."""
    packed = np.asarray(packed, dtype=np.uint8)
    N, half = packed.shape
    u = np.empty((N, 2 * half), dtype=np.uint8)
    u[:, 0::2] = packed & 0x0F
    u[:, 1::2] = packed >> 4
    return u


def dequantize_int4(packed: np.ndarray, scale: np.ndarray, group: int) -> np.ndarray:
    """(packed, fp16 scales) -> float64 [N, K] with w' = (u - 8) * s (exact)."""
    u = unpack_nibbles(packed).astype(np.float64)
    N, K = u.shape
    s = np.asarray(scale).astype(np.float64)
    return ((u - 8.0).reshape(N, K // group, group) * s[..., None]).reshape(N, K)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """float64 -> nearest bfloat16 value (ties to even), returned as float64.

    Rounds the 8-bit significand directly from the float64 value (no detour
    through float32, which could round twice)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                 # x = m * 2^e, 0.5 <= |m| < 1
    ec = np.maximum(e, -125)           # below 2^-126 the spacing stays 2^-133 (subnormals)
    r = np.ldexp(np.rint(np.ldexp(m, 8 + e - ec)), ec - 8)
    return np.where(x == 0, x, r)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float64 -> uint16 bit patterns of the nearest bfloat16 values."""
    r = round_bf16(x).astype(np.float32)  # exact: every bf16 value is a float32 value
    return (r.view(np.uint32) >> 16).astype(np.uint16)


def bf16_from_bits(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)
