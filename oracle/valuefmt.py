"""Coefficient value formats other than NVFP4 (TEST INFRASTRUCTURE).

The paper's Table 4 (reproduced in the technical review, "From retained values
to measured decoding") keeps the dictionary in NVFP4 and stores the coefficient
values of C_l in FP16, FP8 or INT8. The table's gains pin the byte accounting:
with a fraction r of the factorised model's values in D, 16 / (4.5 r + 16 (1-r))
= 1.61 and 16 / (4.5 r + 8 (1-r)) = 2.60 hold for one r (about 0.53), so FP8 and
INT8 values cost 8 bits each, with no per-block scale. The pages name only the
formats; these are plain readings, each with one fp32 per-tensor scale s:

  fp16   IEEE binary16 of x, round to nearest even; s = 1 (no scale).
  fp8    OFP8 E4M3FN: s = amax|C| / 448 (s = 1 if amax = 0); code = sign bit |
         the E4M3 magnitude code nearest to |x| / s (ties to the even code,
         saturating at 448); -0 written as 0. Value = s * E4M3(code).
  int8   s = amax|C| / 127 (s = 1 if amax = 0); code = the integer nearest to
         x / s (ties to even), clamped to [-127, 127], two's complement.
         Value = s * code.

All divisions are IEEE fp32 (numpy float32), as in the NVFP4 quantiser.
"""
from __future__ import annotations

import numpy as np

from .nvfp4 import E4M3_MAX, E4M3_TABLE, e4m3_encode

FORMATS = ("nvfp4", "fp16", "fp8", "int8")
BITS_PER_VALUE = {"nvfp4": 4.5, "fp16": 16.0, "fp8": 8.0, "int8": 8.0}
INT8_MAX = 127


def fp8_scale(x: np.ndarray) -> np.float32:
    x = np.asarray(x, dtype=np.float32)
    amax = np.float32(np.max(np.abs(x))) if x.size else np.float32(0.0)
    return np.float32(1.0) if amax == 0 else np.float32(amax / np.float32(E4M3_MAX))


def int8_scale(x: np.ndarray) -> np.float32:
    x = np.asarray(x, dtype=np.float32)
    amax = np.float32(np.max(np.abs(x))) if x.size else np.float32(0.0)
    return np.float32(1.0) if amax == 0 else np.float32(amax / np.float32(INT8_MAX))


def fp8_encode(x: np.ndarray, s: np.float32) -> np.ndarray:
    """Signed E4M3 codes of x / s (magnitude to nearest, ties to even, saturating)."""
    q = (np.asarray(x, dtype=np.float32) / np.float32(s)).astype(np.float32)
    mag = e4m3_encode(np.abs(q))
    neg = (q < 0) & (mag != 0)
    return (mag | (neg.astype(np.uint8) << 7)).astype(np.uint8)


def fp8_decode(codes: np.ndarray, s: float) -> np.ndarray:
    return float(s) * E4M3_TABLE[np.asarray(codes, dtype=np.int64)]


def round_half_even(v: np.ndarray) -> np.ndarray:
    """Nearest integer, ties to the even one, written out from the definition."""
    v = np.asarray(v, dtype=np.float64)
    f = np.floor(v)
    d = v - f
    up = (d > 0.5) | ((d == 0.5) & (np.mod(f, 2) == 1))
    return f + up


def int8_encode(x: np.ndarray, s: np.float32) -> np.ndarray:
    q = (np.asarray(x, dtype=np.float32) / np.float32(s)).astype(np.float32)
    c = np.clip(round_half_even(q), -INT8_MAX, INT8_MAX)
    return c.astype(np.int8)


def int8_decode(codes: np.ndarray, s: float) -> np.ndarray:
    return float(s) * np.asarray(codes, dtype=np.int8).astype(np.float64)


def fp16_encode(x: np.ndarray) -> np.ndarray:
    """binary16 bit patterns of x (round to nearest even); |x| must be finite in fp16."""
    with np.errstate(over="ignore"):
        h = np.asarray(x, dtype=np.float32).astype(np.float16)
    if not np.all(np.isfinite(h)):
        raise ValueError("value outside the fp16 range")
    return h.view(np.uint16)


def fp16_decode(bits: np.ndarray) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def table4_gain(fmt_c: str, r: float) -> float:
    """Compression gain against the factorised FP16 model when a fraction r of
    its values are dictionary values (NVFP4) and the rest coefficient values in
    format fmt_c (Table 4's accounting: value bits only)."""
    return 16.0 / (BITS_PER_VALUE["nvfp4"] * r + BITS_PER_VALUE[fmt_c] * (1.0 - r))


def table4_dictionary_fraction(gain_fp16_c: float) -> float:
    """r solved from the NVFP4 / FP16 row of Table 4."""
    b = BITS_PER_VALUE["nvfp4"]
    return (16.0 - 16.0 / gain_fp16_c) / (16.0 - b)


__all__ = ["FORMATS", "BITS_PER_VALUE", "fp8_scale", "int8_scale", "fp8_encode", "fp8_decode", "round_half_even",
           "int8_encode", "int8_decode", "fp16_encode", "fp16_decode", "table4_gain", "table4_dictionary_fraction"]
