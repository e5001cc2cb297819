"""Shared helpers for the GPU parity tests: run a layer through the C ABI,
run the oracle on the same seeded inputs, and compare.

Tolerances (from the method's arithmetic):
  * qact bytes and the logical activation scales: bit-exact;
  * y: relative Frobenius error <= 5e-3, and per element
    |error| <= 2e-2 * rms(y_ref) + 2^-8 * |y_ref|.
    The GPU accumulates in fp32, rounds L to bf16 before the up-projection
    (<= 2^-8 relative on the low-rank term) and stores y as bf16, whose
    rounding alone is up to half an ulp = 2^-8 |y| (unit roundoff of an
    8-significant-bit format).  For outputs above ~5 rms that rounding by
    itself exceeds 2e-2 * rms, so the per-element bound is the stated
    2e-2 * rms plus the output format's own rounding.  The observed
    Frobenius error (~1.7e-3) is the bf16 output rounding.
  * L = x @ proj_down: |L_gpu - L_ref| <= 2^-8 |L_ref| + 1e-3 rms(L_ref)
    (bf16 rounding of an fp32 sum of K products).
"""

from __future__ import annotations

import numpy as np
import torch

import oracle
from oracle import svdq_ref as ref
from nvfp4_w4a4_quantized_smooth_b200 import synth

Y_REL_FROB = 5e-3
Y_MAX_REL_RMS = 2e-2
Y_OUT_ROUNDING = 2.0 ** -8   # half an ulp of bf16, relative


def svdq():
    from nvfp4_w4a4_quantized_smooth_b200 import svdq as mod
    return mod


def to_dev(L: synth.LayerOperands, dev="cuda"):
    return {k: (None if v is None else v.to(dev)) for k, v in vars(L).items()}


def gpu_layer(L: synth.LayerOperands, x_override=None):
    """Run quantize + linear on the GPU; return CPU results: y with the
    low-rank product in its own accumulator (the formula's order) and
    y_fold with the folded up-projection (fold_proj_up), the form the
    CTA-pair GEMM (M > 128) takes it in; smaller M ignore the folded factor."""
    s = svdq()
    d = to_dev(L)
    if x_override is not None:
        d["x"] = x_override
    M, K = d["x"].shape
    wt = s.repack_weights(d["wscales"])
    qact, asc, lr = s.quantize_act(d["x"], d["smooth"], d["proj_down"])
    y = s.w4a4_linear(qact, asc, lr, d["qweight"], wt, d["wcscales"], d["wtscale"],
                      d["proj_up"], d["bias"])
    folded, bad = s.fold_proj_up(d["proj_up"], d["wcscales"], d["wtscale"])
    assert bad == 0, f"{bad} up-projection elements do not fold"
    y_fold = s.w4a4_linear(qact, asc, lr, d["qweight"], wt, d["wcscales"], d["wtscale"],
                           d["proj_up"], d["bias"], proj_up_folded=folded)
    s.check_device_error()
    asc_logical = s.unpack_scales(asc, M, K)
    torch.cuda.synchronize()
    return dict(qact=qact.cpu(), ascales=asc_logical.cpu(), lowrank=lr.cpu(), y=y.cpu(),
                y_fold=y_fold.cpu(), wtiled=wt)


def bits(t):
    return synth.bits(t)


def oracle_quant(x_cpu_bf16, smooth_cpu):
    return ref.quantize_act(bits(x_cpu_bf16), bits(smooth_cpu))


def oracle_y(L: synth.LayerOperands, rows=None, cols=None, x=None):
    """fp64 oracle output on the selected rows / columns (all by default)."""
    x = L.x if x is None else x
    xb = bits(x)
    if rows is not None:
        xb = xb[rows]
    qw = bits(L.qweight)
    ws = bits(L.wscales)
    wc = bits(L.wcscales)
    pu = bits(L.proj_up)
    bb = None if L.bias is None else bits(L.bias)
    if cols is not None:
        qw, ws, wc, pu = qw[cols], ws[:, cols], wc[cols], pu[cols]
        bb = None if bb is None else bb[cols]
    y, qact, asc, Lr = ref.svdq_linear_from_x(xb, bits(L.smooth), bits(L.proj_down), qw, ws,
                                              wc, bits(L.wtscale), pu, bb)
    return y, qact, asc, Lr


def gpu_plain_layer(L: synth.LayerOperands, with_smooth: bool):
    """The layer without the low-rank branch (R = 0) on the GPU."""
    s = svdq()
    d = to_dev(L)
    M, K = d["x"].shape
    wt = s.repack_weights(d["wscales"])
    qact, asc, lr = s.quantize_act(d["x"], d["smooth"] if with_smooth else None, None)
    assert lr is None
    y = s.w4a4_linear(qact, asc, None, d["qweight"], wt, d["wcscales"], d["wtscale"], None,
                      d["bias"])
    s.check_device_error()
    asc_logical = s.unpack_scales(asc, M, K)
    torch.cuda.synchronize()
    return dict(qact=qact.cpu(), ascales=asc_logical.cpu(), y=y.cpu())


def oracle_plain_y(L: synth.LayerOperands, with_smooth: bool, rows=None):
    xb = bits(L.x)
    if rows is not None:
        xb = xb[rows]
    bb = None if L.bias is None else bits(L.bias)
    return ref.plain_linear_from_x(xb, bits(L.qweight), bits(L.wscales), bits(L.wcscales),
                                   bits(L.wtscale), bb,
                                   smooth_bits=bits(L.smooth) if with_smooth else None)


def assert_y_close(y_gpu_bf16: torch.Tensor, y_ref: np.ndarray, what=""):
    yg = y_gpu_bf16.to(torch.float64).numpy()
    assert yg.shape == y_ref.shape
    assert np.all(np.isfinite(yg)), f"{what}: non-finite output"
    err = yg - y_ref
    rms = np.sqrt(np.mean(y_ref ** 2))
    rel = np.linalg.norm(err) / max(np.linalg.norm(y_ref), 1e-300)
    mx = np.abs(err).max() / max(rms, 1e-300)
    assert rel <= Y_REL_FROB, f"{what}: rel Frobenius error {rel:.3e} > {Y_REL_FROB}"
    bound = Y_MAX_REL_RMS * rms + Y_OUT_ROUNDING * np.abs(y_ref)
    bad = np.abs(err) > bound
    assert not bad.any(), (f"{what}: {bad.sum()} outputs beyond 2e-2 rms + 2^-8 |y|; "
                           f"worst excess {(np.abs(err) - bound).max():.3e}")
    return rel, mx


def assert_lowrank_close(lr_gpu_bf16: torch.Tensor, L_ref: np.ndarray, what=""):
    lg = lr_gpu_bf16.to(torch.float64).numpy()
    rms = np.sqrt(np.mean(L_ref ** 2))
    bound = 2.0 ** -8 * np.abs(L_ref) + 1e-3 * rms
    bad = np.abs(lg - L_ref) > bound
    assert not bad.any(), (f"{what}: {bad.sum()} low-rank values out of tolerance, "
                           f"worst {np.abs(lg - L_ref).max():.3e}")


def assert_quant_exact(qact_gpu: torch.Tensor, asc_gpu: torch.Tensor, qact_ref, asc_ref, what=""):
    qg = qact_gpu.numpy()
    ag = asc_gpu.numpy()
    if not np.array_equal(ag, asc_ref):
        idx = np.argwhere(ag != asc_ref)
        r, c = idx[0]
        raise AssertionError(f"{what}: {len(idx)} scale bytes differ; first at {tuple(idx[0])}: "
                             f"gpu {ag[r, c]:#04x} oracle {asc_ref[r, c]:#04x}")
    if not np.array_equal(qg, qact_ref):
        idx = np.argwhere(qg != qact_ref)
        r, c = idx[0]
        raise AssertionError(f"{what}: {len(idx)} code bytes differ; first at {tuple(idx[0])}: "
                             f"gpu {qg[r, c]:#04x} oracle {qact_ref[r, c]:#04x}")


def sample_rows(M, n, seed=0):
    """Sorted distinct rows: first, last, and a seeded spread."""
    if M <= n:
        return np.arange(M)
    rng = np.random.default_rng(seed)
    rows = set([0, M - 1, M // 2]) | set(rng.choice(M, n - 3, replace=False).tolist())
    return np.array(sorted(rows))[:n]
