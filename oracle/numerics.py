"""Bit-level number formats used by the oracle: bf16 and OCP FP8 E4M3.

bf16 <-> fp32 is done on the integer bit patterns (no torch in the arithmetic):
widening is ``u16 << 16``; narrowing is round-to-nearest-even on the low 16 bits.
E4M3 is the OCP 8-bit floating point format E4M3FN (bias 7, no infinities, max
448, NaN = S.1111.111), encoded with round-to-nearest-even and saturation to
+-448 ("satfinite").
"""
from __future__ import annotations

import numpy as np


def bf16_bits_to_f32(u16: np.ndarray) -> np.ndarray:
    """Widen raw bf16 bit patterns (uint16) to float32 exactly."""
    u = np.asarray(u16, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 with round-to-nearest-even; returns uint16 bits.

    NaN handling is not needed by the method (finite inputs only).
    """
    u = np.ascontiguousarray(np.asarray(x, dtype=np.float32)).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return (r & np.uint64(0xFFFF)).astype(np.uint16)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """float32 -> nearest-even bf16 value, returned as float32."""
    return bf16_bits_to_f32(f32_to_bf16_bits(x))


E4M3_MAX = 448.0


def e4m3_decode(code: np.ndarray) -> np.ndarray:
    """Decode E4M3FN bytes to float64 (NaN for the two NaN codes)."""
    c = np.asarray(code, dtype=np.uint8).astype(np.int64)
    s = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    sub = m.astype(np.float64) / 8.0 * 2.0 ** -6
    nrm = (1.0 + m.astype(np.float64) / 8.0) * np.exp2((e - 7).astype(np.float64))
    v = np.where(e == 0, sub, nrm)
    v = np.where((e == 0xF) & (m == 0x7), np.nan, v)
    return s * v


def e4m3_encode_satfinite(v: np.ndarray) -> np.ndarray:
    """Encode float32 values to E4M3FN with round-to-nearest-even, saturating.

    Magnitudes at or above 448 map to 448. The arithmetic is exact in float64:
    the quantum of the target binade is a power of two, and v is an fp32 value.
    """
    v = np.asarray(v, dtype=np.float32).astype(np.float64)
    sign = np.signbit(v)
    a = np.abs(v)
    # binade exponent, clamped to the subnormal range (minimum normal exponent -6)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    # guard against log2 rounding at exact powers of two
    e = np.where(np.exp2(e) > a, e - 1, e)
    e = np.where(np.exp2(e + 1) <= a, e + 1, e)
    e = np.maximum(e, -6.0)
    quantum = np.exp2(e - 3.0)
    m = a / quantum  # exact (division by a power of two)
    fl = np.floor(m)
    frac = m - fl
    up = (frac > 0.5) | ((frac == 0.5) & (np.mod(fl, 2.0) == 1.0))
    mq = fl + up.astype(np.float64)
    r = mq * quantum
    r = np.minimum(r, E4M3_MAX)
    # re-derive fields from the rounded magnitude r
    out = np.zeros(a.shape, dtype=np.int64)
    is_sub = r < 2.0 ** -6
    sub_m = np.round(r / 2.0 ** -9).astype(np.int64)  # exact multiples
    with np.errstate(divide="ignore"):
        er = np.floor(np.log2(np.where(r > 0, r, 1.0)))
    er = np.where(np.exp2(er) > r, er - 1, er)
    er = np.where(np.exp2(er + 1) <= r, er + 1, er)
    nm = np.round((r / np.exp2(er) - 1.0) * 8.0).astype(np.int64)
    nrm_code = ((er + 7).astype(np.int64) << 3) | nm
    out = np.where(is_sub, sub_m, nrm_code)
    out = np.where(sign, out | 0x80, out)
    return out.astype(np.uint8)
