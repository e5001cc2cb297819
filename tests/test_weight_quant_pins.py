"""Pins for the offline weight-side oracle (oracle/weight_quant.py), all on
the CPU:

* weights built on the NVFP4 grid (power-of-two wtscale and wcscales,
  random e4m3 block scales, every block holding a +-6 code) come back as
  exactly the codes and scales they were built from;
* an exhaustive search over all e4m3 scales and all 16 E2M1 codes, written
  apart from the oracle's table search, picks the same scale and codes on
  random float32 residuals (zeros, signed zeros and an all-zero channel
  included);
* the low-rank part is the Eckart-Young optimum of the smoothed weight: the
  truncation error equals the discarded singular values up to the bf16
  rounding of the factors, and its singular values are the top R;
* on a weight with a few large singular directions (the outliers SVDQuant
  moves to the low-rank branch) the stored operands reproduce the weight
  far better with R > 0 than the NVFP4 residual alone does.
"""

import numpy as np
import pytest
import torch

from oracle import nvfp4 as nv
from oracle import weight_quant as wq
from oracle.svdq_ref import dequant_weight

F32 = np.float32


def _bf16(x):
    t = torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _grid_weight(N, K, seed):
    """Codes and scales chosen first, the weight (smooth = powers of two)
    built from them exactly."""
    rng = np.random.default_rng(seed)
    G = K // 16
    alpha = 2.0 ** -rng.integers(3, 9)
    c = 2.0 ** -rng.integers(0, 5, N).astype(np.float64)
    c[rng.integers(N)] = 1.0
    s = 2.0 ** rng.integers(-2, 3, K).astype(np.float64)
    sw = rng.integers(0x08, 0x7F, (N, G)).astype(np.uint8)          # normal e4m3 codes
    for n in range(N):
        sw[n, rng.integers(G)] = 0x7E                                 # 448: the channel's amax block
    codes = rng.integers(0, 16, (N, K)).astype(np.uint8)
    for n in range(N):
        for g in range(G):
            j = 16 * g + rng.integers(16)
            codes[n, j] = 0x7 if rng.integers(2) else 0xF                  # +-6 in every block
    val = nv.decode_e2m1(codes) * np.repeat(nv.decode_e4m3(sw), 16, axis=1) * alpha * c[:, None]
    W = val * s[None, :]
    W_bits, s_bits = _bf16(W), _bf16(s)
    assert np.array_equal(nv.bf16_bits_to_f64(W_bits), W), "grid weight must be bf16"
    return W_bits, s_bits, codes, sw, _bf16(c), _bf16([alpha])


@pytest.mark.parametrize("N,K,seed", [(8, 64, 1), (33, 128, 2), (64, 512, 3)])
def test_weight_quantizer_round_trips_grid_weights(N, K, seed):
    W_bits, s_bits, codes, sw, c_bits, a_bits = _grid_weight(N, K, seed)
    q = wq.quantize_weights(W_bits, s_bits, R=0)
    assert np.array_equal(q["wtscale"], a_bits)
    assert np.array_equal(q["wcscales"], c_bits)
    assert np.array_equal(q["wscales"], sw.T)
    assert np.array_equal(q["qweight"], nv.pack_nibbles(codes))


def _e4m3_by_search(t):
    """Nearest e4m3 code to t >= 0 (ties to the even code, 448 above the
    top), by scanning every code."""
    vals = [nv.decode_e4m3(np.uint8(cd)) for cd in range(0x7F)]
    best, bd = 0, None
    for cd, v in enumerate(vals):
        d = abs(float(v) - float(t))
        if bd is None or d < bd or (d == bd and cd % 2 == 0 and best % 2 == 1):
            best, bd = cd, d
    return 0x7E if t >= 448 else best


def _e2m1_by_search(q):
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    m = abs(float(q))
    best, bd = 0, None
    for cd, v in enumerate(mags):
        d = abs(v - m)
        if bd is None or d < bd or (d == bd and cd % 2 == 0 and best % 2 == 1):
            best, bd = cd, d
    if m >= 6:
        best = 7
    return best | (8 if np.signbit(q) else 0)


def test_weight_quantizer_matches_exhaustive_search():
    rng = np.random.default_rng(7)
    N, K = 6, 64
    res = (rng.standard_normal((N, K)) * np.exp(rng.uniform(-6, 4, (N, 1)))).astype(F32)
    res[1, 5:21] = 0.0
    res[2, 0:16] = -0.0
    res[3, :] = 0.0                                   # an all-zero channel
    res[4, 16:32] = rng.choice([-1, 1], 16) * 1e-30   # tiny block
    qw, ws, cb, ab = wq.quantize_residual(res)
    codes = nv.unpack_nibbles(qw)
    A = np.abs(res).max()
    alpha = nv.bf16_bits_to_f64(_bf16([F32(A / F32(2688.0))]))[0]
    assert nv.bf16_bits_to_f64(ab)[0] == alpha
    for n in range(N):
        a_n = np.abs(res[n]).max()
        c = nv.bf16_bits_to_f64(_bf16([F32(a_n / A)]))[0]
        assert nv.bf16_bits_to_f64(cb[n]) == c
        d = F32(F32(alpha) * F32(c))
        for g in range(K // 16):
            grp = res[n, 16 * g:16 * g + 16]
            a_g = np.abs(grp).max()
            t = F32(a_g / F32(F32(6.0) * d)) if d > 0 else F32(0)
            s_code = _e4m3_by_search(t)
            assert ws[g, n] == s_code, (n, g)
            S = F32(F32(nv.decode_e4m3(np.uint8(s_code))) * d)
            for j in range(16):
                q = F32(grp[j] / S) if S > 0 else F32(0) * grp[j]
                assert codes[n, 16 * g + j] == _e2m1_by_search(q), (n, g, j)


def _spectral_weight(N, K, seed, top=(64.0, 32.0, 16.0), tail=1.0):
    """A weight with a few large singular directions over a dense tail."""
    rng = np.random.default_rng(seed)
    Q1, _ = np.linalg.qr(rng.standard_normal((N, N)))
    Q2, _ = np.linalg.qr(rng.standard_normal((K, K)))
    r = min(N, K)
    sig = tail * np.exp(-np.arange(r) / r)
    sig[:len(top)] = top
    W = (Q1[:, :r] * sig) @ Q2[:, :r].T
    s = rng.uniform(0.5, 2.0, K)
    return _bf16(W), _bf16(s)


def test_lowrank_part_is_the_truncated_svd():
    W_bits, s_bits = _spectral_weight(48, 96, 11)
    R = 8
    pd, pu, S = wq.lowrank_factors(W_bits, s_bits, R)
    Ws = wq.smoothed_weight(W_bits, s_bits)
    s = nv.bf16_bits_to_f64(s_bits)
    LRs = (nv.bf16_bits_to_f64(pu) @ nv.bf16_bits_to_f64(pd).T) / s[None, :]
    err = np.linalg.norm(Ws - LRs)
    opt = np.sqrt((S[R:] ** 2).sum())
    lr_norm = np.linalg.norm(LRs)
    # Eckart-Young: the truncation error is the discarded spectrum, up to
    # the bf16 rounding of the two factors (relative 2^-8 each)
    assert abs(err - opt) <= 2.0 ** -7 * lr_norm + 1e-12
    sv = np.linalg.svd(LRs, compute_uv=False)[:R]
    assert np.allclose(sv, S[:R], rtol=2.0 ** -6)


def test_lowrank_branch_absorbs_outlier_directions():
    # SVDQuant's premise: large singular directions quantize badly in 4
    # bits; moved to the 16-bit low-rank branch, the rest quantizes well.
    W_bits, s_bits = _spectral_weight(64, 128, 12, top=(400.0, 300.0, 200.0, 100.0), tail=1.0)
    W = nv.bf16_bits_to_f64(W_bits)
    errs = {}
    for R in (0, 4):
        q = wq.quantize_weights(W_bits, s_bits, R=R)
        q["smooth"] = s_bits
        errs[R] = np.linalg.norm(wq.effective_weight(q) - W) / np.linalg.norm(W)
    assert errs[4] < 0.25 * errs[0], errs
    assert errs[4] < 0.02, errs


def test_effective_weight_is_the_formula():
    # effective_weight spells out the runtime formula's weight: dequantized
    # residual * wtscale * wcscales * smooth + proj_up @ proj_down^T
    W_bits, s_bits = _spectral_weight(16, 32, 13)
    q = wq.quantize_weights(W_bits, s_bits, R=2)
    q["smooth"] = s_bits
    Wq = dequant_weight(q["qweight"], q["wscales"])
    a = nv.bf16_bits_to_f64(q["wtscale"])[0]
    c = nv.bf16_bits_to_f64(q["wcscales"])
    s = nv.bf16_bits_to_f64(s_bits)
    x = np.random.default_rng(0).standard_normal((5, 32))
    y_formula = ((x * s) @ Wq.T) * a * c[None, :] + (x @ nv.bf16_bits_to_f64(q["proj_down"])) \
        @ nv.bf16_bits_to_f64(q["proj_up"]).T
    assert np.allclose(x @ wq.effective_weight(q).T, y_formula, rtol=1e-12, atol=1e-12)
