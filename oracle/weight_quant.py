"""Reference for the offline weight side of the SVDQuant W4A4 NVFP4 layer.

Test infrastructure only (see the package docstring).

The "nunchaku-z-image-turbo-svdq" model card's first paragraph describes the
stored model as a 4-bit-weight, 4-bit-activation quantization "via
SVDQuant" in NVFP4 "with rank-128 SVD residual", and its "What's stored on
disk" table gives the operands (qweight, wscales, wcscales, wtscale,
smooth_factor, proj_down, proj_up); the SD.Next guide's "Nunchaku Z-Image
Turbo" section names SVDQuant as the method.  Neither page says how the
operands are derived from a trained bf16 weight, so every step below is a
reading, chosen as the plainest one that reproduces the card's runtime
formula

    y = scaled_mma(quant(x * smooth), qweight, ascales, wscales)
        * wtscale * wcscales + (x @ proj_down) @ proj_up^T + bias

as closely as the formats allow for y = x @ W^T + bias:

1. Smoothed weight W_s[n, k] = W[n, k] / smooth[k] (so that
   (x * smooth) @ W_s^T = x @ W^T).
2. Low-rank part: the rank-R truncation of W_s by its singular value
   decomposition W_s = U S V^T (the Eckart-Young optimum in the Frobenius
   norm), split as proj_up = U_R S_R^(1/2) and, because the low-rank branch
   of the formula takes the raw x, proj_down = diag(smooth) V_R S_R^(1/2);
   both rounded to bf16 (the table's dtype).
3. Residual, in the smoothed space and against the rounded factors:
   res[n, k] = (W[n, k] - (proj_up @ proj_down^T)[n, k]) / smooth[k].
4. NVFP4 encoding of the residual with the table's three scale levels:
   wtscale = bf16(A / (6 * 448)) with A = max |res| (1 if A == 0): the
   per-tensor level, so that the largest block scale is near 448, the
   largest e4m3 value; wcscales[n] = bf16(a_n / A) with a_n = max_k
   |res[n, k]|: the per-output-channel level; then per 16 k the block
   scale wscales[k/16, n] = e4m3(a_g / (6 d_n)) with d_n = wtscale *
   wcscales[n] and a_g the group's amax, and the element codes
   E2M1(res / (e4m3_value * d_n)).  A block whose scale (or d_n) is zero
   gets signed zero codes.

Steps 3-4 decide integers (codes, scales) from real numbers; both this
reference and the CUDA kernel take those decisions on float32 values with
correctly rounded float32 operations in the order written here (float32 is
the precision of the kernel's arithmetic; the pages fix none), and encode
the float32 results with nearest-even rounding.  Step 2 is a float64 SVD;
the CUDA path's float32 SVD is compared with it by the quality of the
truncation, not bit for bit.
"""

from __future__ import annotations

import numpy as np

from .nvfp4 import (
    bf16_bits_to_f64,
    decode_e4m3,
    encode_e2m1_rne_sat,
    encode_e4m3_rne_satfinite,
    f64_to_bf16_bits_rne,
    pack_nibbles,
)

GROUP = 16
E2M1_MAX = 6.0
E4M3_MAX = 448.0
BF16_ONE = 0x3F80


def smoothed_weight(W_bits, smooth_bits):
    """W_s = W / smooth in float64 (exact inputs, one rounding), [N, K]."""
    return bf16_bits_to_f64(W_bits) / bf16_bits_to_f64(smooth_bits)[None, :]


def lowrank_factors(W_bits, smooth_bits, R):
    """Step 2: (proj_down [K, R], proj_up [N, R]) as bf16 bits from the
    float64 SVD of the smoothed weight, and the float64 singular values."""
    Ws = smoothed_weight(W_bits, smooth_bits)
    U, S, Vt = np.linalg.svd(Ws, full_matrices=False)
    sq = np.sqrt(S[:R])
    proj_up = f64_to_bf16_bits_rne(U[:, :R] * sq[None, :])
    s = bf16_bits_to_f64(smooth_bits)
    proj_down = f64_to_bf16_bits_rne(Vt[:R].T * sq[None, :] * s[:, None])
    return proj_down, proj_up, S


def lowrank_product_f32(proj_up_bits, proj_down_bits):
    """proj_up @ proj_down^T [N, K], float64 product rounded to float32."""
    return (bf16_bits_to_f64(proj_up_bits) @ bf16_bits_to_f64(proj_down_bits).T).astype(np.float32)


def residual_f32(W_bits, smooth_bits, lowrank_f32=None):
    """Step 3 on float32 values: res = (W - lowrank) / smooth, each operation
    correctly rounded to float32 (lowrank None: zero)."""
    W = bf16_bits_to_f64(W_bits).astype(np.float32)
    s = bf16_bits_to_f64(smooth_bits).astype(np.float32)
    diff = W if lowrank_f32 is None else (W - np.asarray(lowrank_f32, dtype=np.float32))
    return (diff / s[None, :]).astype(np.float32)


def quantize_residual(res_f32):
    """Step 4: res [N, K] float32 -> (qweight [N, K/2] uint8, wscales [K/16, N]
    uint8, wcscales [N] bf16 bits, wtscale [1] bf16 bits).

    Float32 arithmetic, in this order (every operation correctly rounded):
      A   = max |res|;  alpha = bf16(A / 2688) (bf16(1) if A == 0)
      a_n = max_k |res[n, k]|;  c_n = bf16(a_n / A) (0 if A == 0)
      d_n = alpha * c_n                       (exact: two 8-bit significands)
      per group g of row n: t = a_g / (6 d_n); s = e4m3(t)   (0 if d_n == 0)
      per element: S = e4m3value(s) * d_n (exact), q = res / S;
      code = E2M1(q), or a zero code with res's sign if s == 0.
    """
    r = np.asarray(res_f32, dtype=np.float32)
    N, K = r.shape
    assert K % GROUP == 0
    f32 = np.float32
    absr = np.abs(r)
    A = absr.max() if r.size else f32(0)
    if A == 0:
        alpha_bits = np.uint16(BF16_ONE)
        c_bits = np.zeros(N, dtype=np.uint16)
    else:
        alpha_bits = f64_to_bf16_bits_rne(np.float64(f32(A / f32(6.0 * E4M3_MAX))))
        a_n = absr.max(axis=1)
        c_bits = f64_to_bf16_bits_rne((a_n / A).astype(np.float32).astype(np.float64))
    alpha = bf16_bits_to_f64(alpha_bits).astype(np.float32)
    c = bf16_bits_to_f64(c_bits).astype(np.float32)
    d = (alpha * c).astype(np.float32)                                  # [N]
    rg = r.reshape(N, K // GROUP, GROUP)
    a_g = np.abs(rg).max(axis=2)                                        # [N, G]
    six_d = (f32(6.0) * d).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(six_d[:, None] > 0, a_g / six_d[:, None], f32(0)).astype(np.float32)
    s_codes = encode_e4m3_rne_satfinite(t.astype(np.float64))         # [N, G]
    S = (decode_e4m3(s_codes).astype(np.float32) * d[:, None]).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(S[:, :, None] > 0, rg / S[:, :, None], f32(0) * rg).astype(np.float32)
    codes = encode_e2m1_rne_sat(q.astype(np.float64)).reshape(N, K)
    qweight = pack_nibbles(codes)
    wscales = np.ascontiguousarray(s_codes.T).astype(np.uint8)         # [K/16, N]
    return qweight, wscales, c_bits.astype(np.uint16), np.array([alpha_bits], dtype=np.uint16)


def quantize_weights(W_bits, smooth_bits, R=128):
    """Steps 1-4 for a bf16 weight [N, K] and smoothing factor [K] ->
    dict(qweight, wscales, wcscales, wtscale, proj_down, proj_up, res, S)."""
    if R > 0:
        proj_down, proj_up, S = lowrank_factors(W_bits, smooth_bits, R)
        lr = lowrank_product_f32(proj_up, proj_down)
    else:
        N, K = np.asarray(W_bits).shape
        proj_down = np.zeros((K, 0), dtype=np.uint16)
        proj_up = np.zeros((N, 0), dtype=np.uint16)
        S = None
        lr = None
    res = residual_f32(W_bits, smooth_bits, lr)
    qweight, wscales, wcscales, wtscale = quantize_residual(res)
    return dict(qweight=qweight, wscales=wscales, wcscales=wcscales, wtscale=wtscale,
                proj_down=proj_down, proj_up=proj_up, res=res, S=S)


def effective_weight(q):
    """The weight the stored operands represent, in the raw input space
    (float64 [N, K]): (e2m1 * wscales * wtscale * wcscales) * smooth +
    proj_up @ proj_down^T -- what y = x @ W_eff^T computes through the
    runtime formula.  `q` also needs 'smooth' (bf16 bits)."""
    from .svdq_ref import dequant_weight
    Wq = dequant_weight(q["qweight"], q["wscales"])
    alpha = bf16_bits_to_f64(np.asarray(q["wtscale"]).reshape(-1))[0]
    c = bf16_bits_to_f64(q["wcscales"])
    s = bf16_bits_to_f64(q["smooth"])
    W_eff = Wq * alpha * c[:, None] * s[None, :]
    if q["proj_up"].shape[1]:
        W_eff = W_eff + bf16_bits_to_f64(q["proj_up"]) @ bf16_bits_to_f64(q["proj_down"]).T
    return W_eff
