"""Reference (fp64, CPU) SVDQuant W4A4 NVFP4 linear layer.

Test infrastructure only (see the package docstring).

The layer, as the "nunchaku-z-image-turbo-svdq" model card writes it in
"What's stored on disk":

    y = scaled_mma(quant(x * smooth), qweight, ascales, wscales)
        * wtscale * wcscales + (x @ proj_down) @ proj_up^T + bias

with the operand table of the same section:

    qweight   [N, K/2]  int8      FP4 nibble pack, low nibble = even k
    wscales   [K/16, N] e4m3fn    one scale per 16 k per output channel
    wcscales  [N]       bf16      per-output-channel scale
    wtscale   [1]       bf16      global alpha
    smooth    [K]       bf16      per-input-channel smoothing factor
    proj_down [K, R]    bf16      SVD residual, down factor (R = 128)
    proj_up   [N, R]    bf16      SVD residual, up factor

Readings taken where the card is silent:

* ``quant`` is dynamic NVFP4 quantization of each 16-element group along
  K: scale = e4m3(amax / 6), element = E2M1(v / scale), both rounded to
  nearest with ties to even and saturating; 6 is the largest E2M1
  magnitude.  A group whose scale rounds to zero gets zero codes (sign
  kept).
* ``x * smooth`` is a multiply by the stored factor, computed exactly.
* The low-rank branch takes the raw x, as the formula is written.
* ``bias`` is an optional bf16 [N]; the card's table has no bias row.

All arrays are NumPy; bf16 tensors are raw uint16 bit patterns and FP8 /
FP4 tensors raw uint8 codes.
"""

from __future__ import annotations

import numpy as np

from .nvfp4 import (
    bf16_bits_to_f64,
    f64_to_bf16_bits_rne,
    decode_e2m1,
    decode_e4m3,
    encode_e2m1_rne_sat,
    encode_e4m3_rne_satfinite,
    pack_nibbles,
    unpack_nibbles,
)

GROUP = 16          # elements per scale along K (model card, first paragraph)
E2M1_MAX = 6.0      # largest E2M1 magnitude


def quantize_act(x_bits, smooth_bits):
    """quant(x * smooth) -> (qact [M, K/2] uint8, ascales [M, K/16] uint8).

    Model card "What's stored on disk": the runtime formula's
    ``quant(x * smooth)``, producing the same packed layout as qweight
    (low nibble = even k) and one e4m3 scale per 16 k, as for wscales.

    Steps, per row m and group g = k // 16:
      1. v = x[m, k] * smooth[k] (exact in float64: both are bf16).
      2. a = max_k |v| over the group.
      3. s = e4m3_rne_satfinite(a / 6); d = decoded value of s.
      4. code = E2M1_rne_sat(v / d), or a signed zero code if d == 0.
      5. pack codes two per byte, low nibble = even k.
    """
    x = bf16_bits_to_f64(x_bits)
    smooth = bf16_bits_to_f64(smooth_bits)
    M, K = x.shape
    assert K % GROUP == 0 and smooth.shape == (K,)
    v = x * smooth[None, :]
    vg = v.reshape(M, K // GROUP, GROUP)
    amax = np.abs(vg).max(axis=2)
    ascales = encode_e4m3_rne_satfinite(amax / E2M1_MAX)
    d = decode_e4m3(ascales)[:, :, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(d == 0.0, 0.0 * vg, vg / np.where(d == 0.0, 1.0, d))
    codes = encode_e2m1_rne_sat(q).reshape(M, K)
    return pack_nibbles(codes), ascales


def dequant_act(qact, ascales):
    """Decoded activation operand [M, K] float64: e2m1(code) * e4m3(scale)."""
    a = decode_e2m1(unpack_nibbles(qact))
    s = decode_e4m3(ascales)
    return a * np.repeat(s, GROUP, axis=1)


def dequant_weight(qweight, wscales):
    """Decoded weight [N, K] float64 from qweight [N, K/2], wscales [K/16, N]."""
    w = decode_e2m1(unpack_nibbles(qweight))
    s = decode_e4m3(wscales).T                     # -> [N, K/16]
    return w * np.repeat(s, GROUP, axis=1)


def lowrank_down(x_bits, proj_down_bits):
    """L = x @ proj_down, float64 [M, R] (model card runtime formula)."""
    return bf16_bits_to_f64(x_bits) @ bf16_bits_to_f64(proj_down_bits)


def w4a4_linear(qact, ascales, qweight, wscales, wcscales_bits, wtscale_bits,
                proj_up_bits, bias_bits, L):
    """y = scaled_mma(...) * wtscale * wcscales + L @ proj_up^T + bias.

    ``scaled_mma`` is the block-scaled product
    acc[m, n] = sum_k e2m1(qa[m,k]) sa[m,k/16] e2m1(qw[n,k]) sw[k/16,n],
    done as one float64 matmul of the decoded operands.  ``L`` is the
    low-rank down product (float64 [M, R]); ``bias_bits`` may be None.
    Returns float64 [M, N].
    """
    acc = dequant_act(qact, ascales) @ dequant_weight(qweight, wscales).T
    alpha = bf16_bits_to_f64(np.asarray(wtscale_bits).reshape(-1))[0]
    c = bf16_bits_to_f64(wcscales_bits)
    y = acc * alpha * c[None, :] + L @ bf16_bits_to_f64(proj_up_bits).T
    if bias_bits is not None:
        y = y + bf16_bits_to_f64(bias_bits)[None, :]
    return y


def svdq_linear_from_x(x_bits, smooth_bits, proj_down_bits, qweight, wscales,
                       wcscales_bits, wtscale_bits, proj_up_bits, bias_bits):
    """The whole layer from raw x: quantize, low-rank down, then the linear.

    Returns (y float64 [M, N], qact, ascales, L float64 [M, R]).
    """
    qact, ascales = quantize_act(x_bits, smooth_bits)
    L = lowrank_down(x_bits, proj_down_bits)
    y = w4a4_linear(qact, ascales, qweight, wscales, wcscales_bits,
                    wtscale_bits, proj_up_bits, bias_bits, L)
    return y, qact, ascales, L


def _bf16_rounding_slack(v):
    """Distance of each float64 value from the nearest bf16 rounding
    boundary (a midpoint between neighbouring bf16 values), relative to |v|."""
    v = np.abs(np.asarray(v, dtype=np.float64))
    m, e = np.frexp(v)
    quantum = np.where(v < 2.0 ** -126, 2.0 ** -133, np.ldexp(1.0, e - 8))
    frac = v / quantum - np.floor(v / quantum)      # exact: v / quantum is a power-of-2 scaling
    with np.errstate(divide="ignore", invalid="ignore"):
        return np.abs(frac - 0.5) * quantum / v


def _round_fraction_to_bf16_bits(f, sign_negative):
    """Exact rational magnitude |f| > 0 -> bf16 bits, nearest, ties to even."""
    from fractions import Fraction
    f = abs(f)
    e = f.numerator.bit_length() - f.denominator.bit_length()
    if Fraction(2) ** e > f:
        e -= 1                                      # now 2^e <= f < 2^(e+1)
    q = Fraction(2) ** (max(e, -126) - 7)           # bf16 spacing there
    n, rem = divmod(f, q)
    n = int(n)
    if rem * 2 > q or (rem * 2 == q and n % 2 == 1):
        n += 1
    val = n * q
    bits = 0x7F80 if val >= 2 ** 128 else int(
        np.array(float(val), dtype=np.float32).view(np.uint32) >> 16)
    return bits | (0x8000 if sign_negative else 0)


def _silu_mul_exact_bits(a: float, b: float) -> int:
    """bf16 bits of silu(a) * b from 400-digit decimal arithmetic, rounded
    exactly.  400 digits hold every product of two bf16 values exactly (a
    bf16 value is an integer below 2^8 times a power of two no smaller than
    2^-133, whose decimal expansion has fewer than 140 digits).  The exact
    product is not a bf16 midpoint for a, b != 0 (it is transcendental);
    where the 400-digit value still lands on one (a > 0 with exp(-a) below
    the working precision), the exact value lies just inside it in
    magnitude, because silu(a) = a sigma(a) with sigma(a) < 1, so it rounds
    toward zero there."""
    import decimal
    from fractions import Fraction
    ctx = decimal.Context(prec=400, Emin=-10 ** 9, Emax=10 ** 9)
    da, db = decimal.Decimal(a), decimal.Decimal(b)
    d = ctx.multiply(ctx.divide(da, ctx.add(1, ctx.exp(ctx.minus(da)))), db)
    f = Fraction(d)
    if f == 0:
        return 0x8000 if (np.signbit(a) != np.signbit(b)) else 0
    bits = _round_fraction_to_bf16_bits(f, f < 0)
    if a > 0:
        # a tie at this precision: take the magnitude just below it
        mag = abs(f)
        lo = _round_fraction_to_bf16_bits(mag - mag * Fraction(1, 10 ** 500), f < 0)
        hi = _round_fraction_to_bf16_bits(mag + mag * Fraction(1, 10 ** 500), f < 0)
        if lo != hi:
            bits = lo
    return bits


def silu_mul(a_bits, b_bits):
    """h = bf16(silu(a) * b), silu(a) = a / (1 + exp(-a)): the input of the
    w2 linear of a DiT feed-forward block.

    The Z-Image NVFP4 blog, section "Z-Image NVFP4 模型变体", names the
    feed-forward linears w1, w2 and w3; the reading taken for how they
    combine is the gated form w2(silu(w1 x) * (w3 x)) those names denote,
    with a = w1's bf16 output and b = w3's.  h is the exact product rounded
    once to bf16 (nearest, ties to even, with gradual underflow and
    overflow to inf).

    Steps: evaluate silu(a) * b in float64 (relative error a few 2^-53)
    and round it; where that value lies within 2^-44 (relative) of a bf16
    rounding boundary, float64 cannot decide the rounding, and the product
    is evaluated again with 400-digit decimal arithmetic and rounded
    exactly (``_silu_mul_exact_bits``).  For a below about -709 exp(-a)
    overflows float64 and a / inf is a signed zero, which is also what the
    exact value (below 2^-1000 in magnitude) rounds to.  Inputs must be
    finite.  Returns raw bf16 bits, same shape.
    """
    a = bf16_bits_to_f64(a_bits)
    b = bf16_bits_to_f64(b_bits)
    assert a.shape == b.shape
    assert np.all(np.isfinite(a)) and np.all(np.isfinite(b))
    with np.errstate(over="ignore"):
        v = a / (1.0 + np.exp(-a)) * b
    out = f64_to_bf16_bits_rne(v)
    near = (v != 0) & (_bf16_rounding_slack(v) <= 2.0 ** -44)
    for i in np.flatnonzero(near.reshape(-1)):
        out.reshape(-1)[i] = _silu_mul_exact_bits(float(a.reshape(-1)[i]),
                                                   float(b.reshape(-1)[i]))
    return out


BF16_ONE = 0x3F80


def plain_linear_from_x(x_bits, qweight, wscales, wcscales_bits, wtscale_bits, bias_bits,
                        smooth_bits=None):
    """The layer without the low-rank branch (R = 0): the plain NVFP4 linear
    of the Z-Image NVFP4 blog's comfy-kitchen deployment (weights quantized
    once, activations quantized dynamically at inference).

        y = scaled_mma(quant(x * smooth), qweight, ascales, wscales)
            * wtscale * wcscales + bias

    with smooth = 1 (no smoothing) when ``smooth_bits`` is None.  Returns
    (y float64 [M, N], qact, ascales).
    """
    M, K = x_bits.shape
    N = qweight.shape[0]
    if smooth_bits is None:
        smooth_bits = np.full(K, BF16_ONE, dtype=np.uint16)
    qact, ascales = quantize_act(x_bits, smooth_bits)
    y = w4a4_linear(qact, ascales, qweight, wscales, wcscales_bits, wtscale_bits,
                    np.zeros((N, 0), dtype=np.uint16), bias_bits, np.zeros((M, 0)))
    return y, qact, ascales
