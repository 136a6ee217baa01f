"""Quantised cache codecs, restated from their definitions.

Test infrastructure (see ``oracle/__init__.py``).
"""
from __future__ import annotations

import numpy as np


def absmax_quantize(values, bits: int, float_type=np.float64):
    """Symmetric absmax quantiser over one group of values.

    "KV Cache Engineering for LLM Serving", section 8 (Quantization), worked
    example: the largest code is 2**(bits-1) - 1, the scale is the largest
    magnitude divided by that code, codes are the values divided by the scale,
    rounded to the nearest integer (ties to even, as numpy's rint) and clipped
    to +-largest; restored values are codes times the scale.

    ``float_type`` fixes the precision of the scale and of the division: the
    page's example runs in float64; the int8 cache writer uses IEEE float32.
    Reading for an all-zero group (the page divides by the scale): scale 0 and
    codes 0.

    Returns (codes as int64, scale as ``float_type``, restored as float64).
    """
    x = np.asarray(values).astype(float_type)
    largest = float_type(2 ** (bits - 1) - 1)
    amax = float_type(np.max(np.abs(x))) if x.size else float_type(0)
    scale = float_type(amax / largest)
    if scale == 0:
        codes = np.zeros(x.shape, dtype=np.int64)
    else:
        q = (x / scale).astype(float_type)
        codes = np.clip(np.rint(q), -largest, largest).astype(np.int64)
    restored = codes.astype(np.float64) * np.float64(scale)
    return codes, scale, restored


# --------------------------------------------------------------- FP8 E4M3
def _e4m3_value(byte: int) -> float:
    """Value of one E4M3 byte from the OCP 8-bit floating point definition.

    Layout S.EEEE.MMM, exponent bias 7, no infinities, S.1111.111 is NaN;
    exponent field 0 encodes subnormals 2**-6 * M/8.
    """
    s = -1.0 if byte & 0x80 else 1.0
    e = (byte >> 3) & 0xF
    m = byte & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (2.0 ** -6) * (m / 8.0)
    return s * (2.0 ** (e - 7)) * (1.0 + m / 8.0)


def e4m3_value_table() -> np.ndarray:
    """float64 [256]: value of every E4M3 byte."""
    return np.array([_e4m3_value(b) for b in range(256)], dtype=np.float64)


_TABLE = e4m3_value_table()
_POS = _TABLE[:0x7F]  # magnitudes of codes 0x00..0x7E, increasing; 0x7F is NaN
E4M3_MAX = float(_POS[-1])  # 448


def e4m3_decode(codes) -> np.ndarray:
    return _TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(y) -> np.ndarray:
    """Round float values to E4M3: nearest representable, ties to the even code.

    Magnitudes above the largest finite value (448) saturate to it (the
    "satfinite" behaviour a scaled cache needs); the sign bit follows the input,
    so -0.0 encodes as 0x80.  NaN encodes as 0x7F.
    """
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    idx = np.searchsorted(_POS, np.minimum(a, E4M3_MAX))
    idx = np.clip(idx, 0, len(_POS) - 1)
    lo = np.clip(idx - 1, 0, len(_POS) - 1)
    d_lo = np.abs(a - _POS[lo])
    d_hi = np.abs(_POS[idx] - a)
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (idx % 2 == 0))
    mag = np.where(pick_hi, idx, lo)
    mag = np.where(a >= E4M3_MAX, 0x7E, mag)
    code = mag.astype(np.uint8) | np.where(np.signbit(y), 0x80, 0).astype(np.uint8)
    return np.where(np.isnan(y), np.uint8(0x7F), code).astype(np.uint8)


# --------------------------------------------------------------- FP8 E5M2
def _e5m2_value(byte: int) -> float:
    """Value of one E5M2 byte from the OCP 8-bit floating point definition.

    Layout S.EEEEE.MM, exponent bias 15, IEEE-like: exponent field 31 with
    mantissa 0 is infinity, with mantissa != 0 NaN; exponent field 0 encodes
    subnormals 2**-14 * M/4.
    """
    s = -1.0 if byte & 0x80 else 1.0
    e = (byte >> 2) & 0x1F
    m = byte & 0x3
    if e == 0x1F:
        return s * float("inf") if m == 0 else float("nan")
    if e == 0:
        return s * (2.0 ** -14) * (m / 4.0)
    return s * (2.0 ** (e - 15)) * (1.0 + m / 4.0)


def e5m2_value_table() -> np.ndarray:
    """float64 [256]: value of every E5M2 byte."""
    return np.array([_e5m2_value(b) for b in range(256)], dtype=np.float64)


_TABLE52 = e5m2_value_table()
_POS52 = _TABLE52[:0x7C]  # magnitudes of the finite codes 0x00..0x7B, increasing
E5M2_MAX = float(_POS52[-1])  # 57344


def e5m2_decode(codes) -> np.ndarray:
    return _TABLE52[np.asarray(codes, dtype=np.uint8)]


def e5m2_encode(y) -> np.ndarray:
    """Round float values to E5M2: nearest finite value, ties to the even code.

    As for E4M3, a scaled cache saturates: magnitudes above 57344 (infinities
    included) become +-57344; the sign bit follows the input; NaN encodes as
    0x7F.
    """
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    idx = np.searchsorted(_POS52, np.minimum(a, E5M2_MAX))
    idx = np.clip(idx, 0, len(_POS52) - 1)
    lo = np.clip(idx - 1, 0, len(_POS52) - 1)
    d_lo = np.abs(a - _POS52[lo])
    d_hi = np.abs(_POS52[idx] - a)
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (idx % 2 == 0))
    mag = np.where(pick_hi, idx, lo)
    mag = np.where(a >= E5M2_MAX, 0x7B, mag)
    code = mag.astype(np.uint8) | np.where(np.signbit(y), 0x80, 0).astype(np.uint8)
    return np.where(np.isnan(y), np.uint8(0x7F), code).astype(np.uint8)


# --------------------------------------------------------------- INT4
def pack_int4(codes) -> np.ndarray:
    """Signed 4-bit codes [..., d] (d even, values in [-8, 7]) -> bytes [..., d/2].

    Storage reading for the 4-bit cache ("KV Cache Engineering", section 8:
    a 4-bit format cuts the payload to a quarter of BF16): two's-complement
    nibbles, the code of element 2j in the low nibble of byte j and that of
    element 2j+1 in the high nibble.
    """
    c = np.asarray(codes, dtype=np.int64)
    nib = (c & 0xF).astype(np.uint8)
    return (nib[..., 0::2] | (nib[..., 1::2] << 4)).astype(np.uint8)


def unpack_int4(packed) -> np.ndarray:
    """Bytes [..., d/2] -> signed codes [..., d] (inverse of pack_int4)."""
    b = np.asarray(packed, dtype=np.uint8).astype(np.int64)
    lo, hi = b & 0xF, b >> 4
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.int64)
    out[..., 0::2] = np.where(lo >= 8, lo - 16, lo)
    out[..., 1::2] = np.where(hi >= 8, hi - 16, hi)
    return out


def pack_int2(codes) -> np.ndarray:
    """Signed 2-bit codes [..., d] (d a multiple of 4, values in [-2, 1]) -> bytes [..., d/4].

    Storage reading for the 2-bit KIVI cache ("KV Cache Engineering", section 8;
    "Chapter 18 - KV-Cache Optimization Strategies", KV-Cache Quantization
    table): two's-complement bit pairs, the code of element 4j + m in bits
    [2m, 2m + 1] of byte j.
    """
    c = np.asarray(codes, dtype=np.int64)
    pairs = (c & 0x3).astype(np.uint8)
    return (pairs[..., 0::4] | (pairs[..., 1::4] << 2) | (pairs[..., 2::4] << 4) | (pairs[..., 3::4] << 6)).astype(
        np.uint8)


def unpack_int2(packed) -> np.ndarray:
    """Bytes [..., d/4] -> signed codes [..., d] (inverse of pack_int2)."""
    b = np.asarray(packed, dtype=np.uint8).astype(np.int64)
    out = np.empty(b.shape[:-1] + (4 * b.shape[-1],), dtype=np.int64)
    for m in range(4):
        v = (b >> (2 * m)) & 0x3
        out[..., m::4] = np.where(v >= 2, v - 4, v)
    return out
