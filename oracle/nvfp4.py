"""NVFP4 codec, written from the public format definitions (TEST INFRASTRUCTURE).

The technical review ("From retained values to measured decoding") fixes the
block structure: 4-bit values with one shared 8-bit scale per block of sixteen
values, 4.5 bits per value.  The element and scale encodings are the OCP
Microscaling / OFP8 ones:

  E2M1   bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa;
         exponent 0 is subnormal (value = m * 0.5).  Magnitudes of codes 0..7
         are 0, 0.5, 1, 1.5, 2, 3, 4, 6.
  E4M3   (E4M3FN) bit 7 sign, bits 6..3 exponent (bias 7), bits 2..0 mantissa;
         exponent 0 is subnormal (value = m/8 * 2^-6); 0x7F / 0xFF are NaN;
         no infinities; largest finite 448.

Quantiser (a plain round-to-nearest reading; the paper's Hessian-aware
quantiser needs calibration data and is out of scope).  For a tensor T split
into blocks of 16 values, all arithmetic in IEEE fp32 as numpy float32:

  s_T  = amax|T| / 2688           (2688 = 6 * 448; s_T = 1 if amax == 0)
  r_b  = amax_b / (6 * s_T)        per block
  sc_b = E4M3 nearest to r_b, ties to even code, saturating at 448
  q_i  = x_i / (E4M3(sc_b) * s_T)
  c_i  = E2M1 nearest to q_i, ties to even mantissa, saturating at 6;
         -0 is written as code 0.  A block whose scale decodes to 0 has all
         codes 0.

Decoded value = s_T * E4M3(sc_b) * E2M1(c_i).
"""
from __future__ import annotations

import numpy as np

E2M1_BLOCK = 16
E4M3_MAX = 448.0
E2M1_MAX = 6.0


def e2m1_value(code: int) -> float:
    """Value of a 4-bit E2M1 code from its sign / exponent / mantissa fields."""
    s = (code >> 3) & 1
    e = (code >> 1) & 3
    m = code & 1
    mag = m * 0.5 if e == 0 else (2.0 ** (e - 1)) * (1.0 + m / 2.0)
    return -mag if s else mag


def e4m3_value(code: int) -> float:
    """Value of an 8-bit E4M3FN code (NaN for 0x7F / 0xFF)."""
    s = (code >> 7) & 1
    e = (code >> 3) & 15
    m = code & 7
    if e == 15 and m == 7:
        return float("nan")
    mag = (m / 8.0) * 2.0 ** -6 if e == 0 else (2.0 ** (e - 7)) * (1.0 + m / 8.0)
    return -mag if s else mag


E2M1_TABLE = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)
E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)

# non-negative finite E4M3 values: codes 0x00..0x7E, ascending with the code
_E4M3_POS = E4M3_TABLE[:0x7F].copy()
# non-negative E2M1 magnitudes: codes 0..7, ascending with the code
_E2M1_POS = E2M1_TABLE[:8].copy()


def _nearest_even(table: np.ndarray, v: np.ndarray) -> np.ndarray:
    """Index of the entry of the ascending `table` nearest to each v >= 0.

    Ties go to the even index (which is the even mantissa bit for both E2M1 and
    E4M3, whose non-negative codes are ascending).  Values above the last
    entry saturate to it.  Distances are taken in fp64, exactly."""
    v = np.asarray(v, dtype=np.float64)
    hi = np.searchsorted(table, v, side="left")  # first entry >= v
    hi = np.clip(hi, 0, len(table) - 1)
    lo = np.clip(hi - 1, 0, len(table) - 1)
    d_lo = np.abs(v - table[lo])
    d_hi = np.abs(table[hi] - v)
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(v >= table[-1], len(table) - 1, idx)
    return idx.astype(np.int64)


def e4m3_encode(r: np.ndarray) -> np.ndarray:
    """E4M3 code nearest to each non-negative fp32 r (ties to even, saturating)."""
    r = np.asarray(r, dtype=np.float32)
    if np.any(r < 0) or not np.all(np.isfinite(r)):
        raise ValueError("block scale ratio must be finite and non-negative")
    return _nearest_even(_E4M3_POS, r).astype(np.uint8)


def e2m1_encode(q: np.ndarray) -> np.ndarray:
    """E2M1 code nearest to each fp32 q (ties to even mantissa, saturating at 6)."""
    q = np.asarray(q, dtype=np.float32)
    mag = _nearest_even(_E2M1_POS, np.abs(q).astype(np.float64))
    neg = (q < 0) & (mag != 0)
    return (mag | (neg.astype(np.int64) << 3)).astype(np.uint8)


def tensor_scale(x: np.ndarray) -> np.float32:
    """Per-tensor fp32 scale s_T = amax / (6 * 448); 1 for an all-zero tensor."""
    x = np.asarray(x, dtype=np.float32)
    if x.size == 0:
        return np.float32(1.0)
    amax = np.float32(np.max(np.abs(x)))
    if amax == 0:
        return np.float32(1.0)
    return np.float32(amax / np.float32(E2M1_MAX * E4M3_MAX))


def quantize_blocks(blocks: np.ndarray, s_t: np.float32):
    """Quantise rows of 16 fp32 values with tensor scale s_t.

    Returns (codes uint8 [n, 16], scale codes uint8 [n])."""
    b = np.asarray(blocks, dtype=np.float32)
    if b.ndim != 2 or b.shape[1] != E2M1_BLOCK:
        raise ValueError("blocks must be [n, 16]")
    if not np.all(np.isfinite(b)):
        raise ValueError("non-finite value")
    s_t = np.float32(s_t)
    amax_b = np.max(np.abs(b), axis=1).astype(np.float32) if b.shape[0] else np.zeros(0, np.float32)
    den = np.float32(np.float32(E2M1_MAX) * s_t)
    r = (amax_b / den).astype(np.float32)
    sc = e4m3_encode(r)
    scale_f = (E4M3_TABLE[sc].astype(np.float32) * s_t).astype(np.float32)
    codes = np.zeros(b.shape, dtype=np.uint8)
    live = scale_f != 0
    if np.any(live):
        q = (b[live] / scale_f[live, None]).astype(np.float32)
        codes[live] = e2m1_encode(q)
    return codes, sc


def dequantize(codes: np.ndarray, scale_codes: np.ndarray, s_t: float) -> np.ndarray:
    """fp64 values s_T * E4M3(sc) * E2M1(code) for codes [n, 16], scales [n]."""
    return float(s_t) * E4M3_TABLE[scale_codes][:, None] * E2M1_TABLE[codes]
