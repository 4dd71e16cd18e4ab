"""Number formats the layer uses, written from their published definitions.

e4m3fn (OCP 8-bit floating point specification, E4M3 variant "fn"):
  1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0 encodes
  subnormals (2^-6 * m/8); no infinities; S.1111.111 is NaN; largest finite 448.
Encoding here is round-to-nearest, ties-to-even, saturating to +-448 (the "satfinite"
behaviour), with NaN -> 0x7F.

bf16: the top 16 bits of an IEEE binary32 (8 exponent bits, 7 stored mantissa bits);
rounding from a wider value is round-to-nearest, ties-to-even.

Block-FP8 is the expert precision on the FFN side (FastAFD, "Methodology / System
Design", item 1: "block-FP8 expert precision").
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def _decode_code(c: int) -> float:
    s = -1.0 if (c >> 7) & 1 else 1.0
    e = (c >> 3) & 0xF
    m = c & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** (-6)
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_TABLE = np.array([_decode_code(c) for c in range(256)], dtype=np.float64)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """uint8 codes -> float64 values (exact)."""
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def _rne(x: np.ndarray) -> np.ndarray:
    """Round to nearest integer, ties to even (x float64, |x| < 2^52)."""
    return np.rint(x)  # numpy rint rounds half to even


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """float values -> uint8 codes, RNE with saturation to +-448; NaN -> 0x7F.

    For |v| in binade [2^E, 2^(E+1)) with E >= -6 the spacing of e4m3 values is
    2^(E-3); below 2^-6 (subnormals) it is 2^-9. Rounding |v| to a multiple of that
    spacing (ties to even multiple) gives the nearest representable magnitude, which
    may be the first value of the next binade.
    """
    v = np.asarray(v, dtype=np.float64)
    out = np.zeros(v.shape, dtype=np.uint8)
    nan = np.isnan(v)
    a = np.abs(np.where(nan, 0.0, v))
    a = np.minimum(a, E4M3_MAX)
    with np.errstate(divide="ignore"):
        E = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    E = np.maximum(E, -6.0)
    q = np.exp2(E - 3.0)
    mag = _rne(a / q) * q
    mag = np.minimum(mag, E4M3_MAX)
    # magnitude -> code by exact lookup in the non-negative half of the table
    pos_vals = E4M3_TABLE[:127]          # codes 0x00..0x7E, ascending, all finite
    idx = np.searchsorted(pos_vals, mag)
    assert np.all(pos_vals[np.minimum(idx, 126)] == mag), "value not representable"
    code = idx.astype(np.uint8)
    neg = np.signbit(v) & ~nan
    code = np.where(neg, code | 0x80, code).astype(np.uint8)
    code = np.where(nan, np.uint8(0x7F), code).astype(np.uint8)
    return code


def bf16_round(v: np.ndarray) -> np.ndarray:
    """float64 values -> the nearest bf16 values (RNE), returned as float64.

    Normal bf16 numbers in binade [2^E, 2^(E+1)) are spaced 2^(E-7); subnormals
    (below 2^-126) are spaced 2^-133. Overflow beyond the largest finite bf16 goes to inf.
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    with np.errstate(divide="ignore"):
        E = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    E = np.maximum(E, -126.0)
    q = np.exp2(E - 7.0)
    mag = _rne(a / q) * q
    bf16_max = (2.0 - 2.0 ** -7) * 2.0 ** 127
    mag = np.where(mag > bf16_max, np.inf, mag)
    out = np.copysign(mag, v)
    return np.where(np.isnan(v), np.nan, out)


def bf16_bits(v: np.ndarray) -> np.ndarray:
    """float64 values that are exactly bf16 -> uint16 bit patterns."""
    f32 = np.asarray(v, dtype=np.float32)
    return (f32.view(np.uint32) >> 16).astype(np.uint16)


def bf16_from_bits(b: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns -> float64 values."""
    u = np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)
