"""Plain codecs for the number formats of the SVDQuant W4A4 NVFP4 layer.

Test infrastructure only (see the package docstring).  Every routine works
on whole NumPy arrays of raw codes or float64 values and is written for
obviousness, not speed.

Formats
-------
* E2M1 (FP4): 1 sign bit, 2 exponent bits, 1 mantissa bit, as the Z-Image
  NVFP4 blog states in "NVFP4 技术背景 / 什么是 NVFP4？".  With exponent bias 1
  the eight magnitudes are {0, 0.5, 1, 1.5, 2, 3, 4, 6}; code 0x8 is -0.
* float8_e4m3fn: the scale dtype of the model card's "What's stored on
  disk" table (wscales).  1 sign, 4 exponent bits (bias 7), 3 mantissa
  bits, subnormals m * 2^-9, no infinities, 0x7F / 0xFF are NaN, largest
  finite magnitude 448 (the "约 ±448" row of the SD.Next SDNQ guide's type
  table).
* bfloat16: the dtype of x, smooth_factor, wcscales, wtscale, proj_down and
  proj_up in the same table; handled as raw uint16 bit patterns.

Rounding: round-to-nearest, ties to the even code, with saturation to the
largest finite value (the plainest reading of "quant(...)" in the model
card's runtime formula; the pages name no other rounding).
"""

from __future__ import annotations

import numpy as np

# Magnitudes of the 8 non-negative E2M1 codes, in code order.  Derived from
# the 1-2-1 bit layout: code = e1 e0 m; e == 0 is subnormal (m * 0.5),
# otherwise (1 + m/2) * 2^(e-1).
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)


def _e4m3_magnitude(code: int) -> float:
    """Value of a non-negative e4m3fn code 0..0x7E (0x7F is NaN)."""
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0:
        return m * 2.0 ** -9
    return (1.0 + m / 8.0) * 2.0 ** (e - 7)


# Value of every finite non-negative e4m3 code, indexed by code 0..0x7E.
# Strictly increasing in the code, which the encoder below relies on.
_E4M3_POS = np.array([_e4m3_magnitude(c) for c in range(0x7F)], dtype=np.float64)


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Decode raw bfloat16 bit patterns (uint16) to float64, exactly."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


# bfloat16: 8 significant bits, exponent range of float32.  Smallest normal
# 2^-126; subnormals are multiples of 2^-133; the largest finite value is
# (2 - 2^-7) 2^127 and anything at or above (2 - 2^-8) 2^127 rounds to inf.
_BF16_MIN_NORMAL = 2.0 ** -126
_BF16_SUBNORMAL_QUANTUM = 2.0 ** -133
_BF16_OVERFLOW = (2.0 - 2.0 ** -8) * 2.0 ** 127


def f64_to_bf16_bits_rne(values) -> np.ndarray:
    """Round float64 values to bfloat16 (nearest, ties to even), raw bits.

    Rounds straight from float64 (no float32 step, so no double rounding),
    as IEEE 754 rounds to a binary format with 8 significant bits and
    float32's exponent range: normal results keep 8 significant bits,
    results below 2^-126 are rounded to a multiple of the subnormal
    quantum 2^-133 (gradual underflow), and magnitudes from the overflow
    threshold (2 - 2^-8) 2^127 up give infinity.  The sign is kept, also
    for results that round to zero.
    """
    v = np.asarray(values, dtype=np.float64)
    m, e = np.frexp(v)                      # v = m * 2^e, 0.5 <= |m| < 1
    normal = np.ldexp(np.rint(m * 256.0), e - 8)  # 8 significant bits, half-even
    sub = np.rint(v / _BF16_SUBNORMAL_QUANTUM) * _BF16_SUBNORMAL_QUANTUM
    r = np.where(np.abs(v) < _BF16_MIN_NORMAL, sub, normal)
    r = np.where(np.abs(v) >= _BF16_OVERFLOW, np.copysign(np.inf, v), r)
    r = np.copysign(r, v)                   # a result that rounds to 0 keeps its sign
    out = r.astype(np.float32).view(np.uint32) >> np.uint32(16)
    return out.astype(np.uint16)


def decode_e2m1(codes) -> np.ndarray:
    """E2M1 codes (low 4 bits used) -> float64.  Code 0x8 gives -0.0."""
    c = np.asarray(codes, dtype=np.uint8) & np.uint8(0xF)
    mag = E2M1_MAGNITUDES[c & np.uint8(0x7)]
    return np.where(c & np.uint8(0x8), -mag, mag)


def decode_e4m3(codes) -> np.ndarray:
    """float8_e4m3fn codes -> float64 (NaN for 0x7F and 0xFF)."""
    c = np.asarray(codes, dtype=np.uint8)
    mag_code = c & np.uint8(0x7F)
    mag = np.where(mag_code == 0x7F, np.nan,
                   _E4M3_POS[np.minimum(mag_code, 0x7E)])
    return np.where(c & np.uint8(0x80), -mag, mag)


def _round_to_table(mag: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Index of the nearest entry of the increasing ``table`` to each ``mag``.

    Ties go to the even index.  For E2M1 and e4m3 the index is the code and
    the code's lowest bit is the mantissa's lowest bit, so "even index" is
    "even mantissa".  Values above the last entry saturate to it.
    """
    mag = np.asarray(mag, dtype=np.float64)
    top = len(table) - 1
    lo = np.clip(np.searchsorted(table, mag, side="right") - 1, 0, top)
    hi = np.minimum(lo + 1, top)
    below = table[lo]
    above = table[hi]
    mid = (below + above) / 2.0          # exact: both are short dyadics
    pick_hi = (mag > mid) | ((mag == mid) & (lo % 2 == 1))
    idx = np.where(pick_hi & (hi != lo), hi, lo)
    return np.where(mag >= table[top], top, idx)


def encode_e4m3_rne_satfinite(values) -> np.ndarray:
    """float64 -> float8_e4m3fn code: nearest, ties to even, saturating.

    Magnitudes at or above 448 give 448 (0x7E); magnitudes below half the
    smallest subnormal (2^-10) give zero, and exactly 2^-10 is a tie that
    goes to the even code 0.  The sign bit is kept, so -0.0 gives 0x80.
    """
    v = np.asarray(values, dtype=np.float64)
    code = _round_to_table(np.abs(v), _E4M3_POS).astype(np.uint8)
    return np.where(np.signbit(v), code | np.uint8(0x80), code).astype(np.uint8)


def encode_e2m1_rne_sat(values) -> np.ndarray:
    """float64 -> E2M1 code (0..15): nearest, ties to even, saturating at 6.

    The sign is kept even when the magnitude rounds to zero, so a negative
    input below 0.25 in magnitude (or -0.0) gives code 0x8.
    """
    v = np.asarray(values, dtype=np.float64)
    code = _round_to_table(np.abs(v), E2M1_MAGNITUDES).astype(np.uint8)
    return np.where(np.signbit(v), code | np.uint8(0x8), code).astype(np.uint8)


def pack_nibbles(codes) -> np.ndarray:
    """[..., K] E2M1 codes -> [..., K/2] bytes, low nibble = even k.

    The nibble order is the one the model card's "What's stored on disk"
    table gives for qweight ("FP4 nibble pack, low nibble = even-k").
    """
    c = np.asarray(codes, dtype=np.uint8) & np.uint8(0xF)
    assert c.shape[-1] % 2 == 0
    return (c[..., 0::2] | (c[..., 1::2] << np.uint8(4))).astype(np.uint8)


def unpack_nibbles(packed) -> np.ndarray:
    """[..., K/2] bytes -> [..., K] E2M1 codes; inverse of ``pack_nibbles``."""
    p = np.asarray(packed).view(np.uint8) if np.asarray(packed).dtype == np.int8 \
        else np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & np.uint8(0xF)
    out[..., 1::2] = p >> np.uint8(4)
    return out
