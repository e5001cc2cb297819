"""The offline weight side on the GPU (svdq_quantize_weights and svdq.py's
quantize_weights) against oracle/weight_quant.py.

* The residual's NVFP4 encoding -- codes, block scales, per-channel and
  per-tensor scales -- is a function of float32 inputs; given the same W,
  smooth and float32 low-rank part as the oracle it must be identical bit
  for bit (zeros, signed zeros, an all-zero channel, tiny and huge
  channels, a 16-but-not-64 multiple K included), also at the qkv shape.
* Weights built on the NVFP4 grid come back exactly.
* The whole pipeline (float32 SVD on the device) against the float64
  oracle: the low-rank part meets the Eckart-Young bound up to the float32
  SVD and bf16 factor rounding, the stored operands reproduce the weight
  as well as the oracle's do, and the layer run through the CUDA GEMM with
  them matches x @ W^T to that accuracy.
"""

import numpy as np
import pytest
import torch

from oracle import nvfp4 as nv
from oracle import weight_quant as wq
import gpu_helpers as H
import test_weight_quant_pins as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from nvfp4_w4a4_quantized_smooth_b200 import build
    build.build()
    torch.cuda.init()
    yield


def _t16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def _assert_same_encoding(got, want, what):
    names = ("qweight", "wscales", "wcscales", "wtscale")
    for name, g, w in zip(names, got, want):
        g = g.cpu()
        g = H.bits(g) if g.dtype == torch.bfloat16 else g.numpy()
        if not np.array_equal(g, w):
            bad = np.argwhere(g != w)
            raise AssertionError(f"{what}: {name} differs at {len(bad)} places, first {bad[0]}")


def _random_weight(N, K, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    W = (torch.randn(N, K, generator=g) * scale * torch.exp(torch.randn(N, 1, generator=g))
         ).to(torch.bfloat16)
    s = (torch.rand(K, generator=g) * 1.5 + 0.5).to(torch.bfloat16)
    return W, s


@pytest.mark.parametrize("N,K,with_lr", [(8, 64, False), (37, 48, True), (256, 512, True),
                                         (300, 1024, False), (1000, 768, True)])
def test_residual_encoding_bit_exact(N, K, with_lr):
    s_ = H.svdq()
    W, s = _random_weight(N, K, N + K)
    W[3] = 0                                           # an all-zero channel
    W[5, :16] = -0.0
    W[6, 16:32] = 1e-30
    W[7] *= 1e4
    lr = None
    if with_lr:
        g = torch.Generator().manual_seed(K)
        lr = (torch.randn(N, K, generator=g) * 0.1).float()
    got = s_.quantize_weights_residual(W.cuda(), s.cuda(), None if lr is None else lr.cuda())
    s_.check_device_error()
    res = wq.residual_f32(H.bits(W), H.bits(s), None if lr is None else lr.numpy())
    _assert_same_encoding(got, wq.quantize_residual(res), f"{N}x{K}")


def test_grid_weights_round_trip_on_the_gpu():
    s_ = H.svdq()
    W_bits, s_bits, codes, sw, c_bits, a_bits = P._grid_weight(64, 512, 3)
    got = s_.quantize_weights(_t16(W_bits).cuda(), _t16(s_bits).cuda(), R=0)
    s_.check_device_error()
    assert np.array_equal(got["qweight"].cpu().numpy(), nv.pack_nibbles(codes))
    assert np.array_equal(got["wscales"].cpu().numpy(), sw.T)
    assert np.array_equal(H.bits(got["wcscales"].cpu()), c_bits)
    assert np.array_equal(H.bits(got["wtscale"].cpu()), a_bits)


def _effective(q, s_bits):
    d = {k: (H.bits(v.cpu()) if v.dtype == torch.bfloat16 else v.cpu().numpy())
         for k, v in q.items()}
    d["smooth"] = s_bits
    return wq.effective_weight(d)


def test_full_pipeline_against_the_float64_oracle():
    # a weight with a few large singular directions over a dense tail
    s_ = H.svdq()
    N, K, R = 384, 512, 128
    W_bits, s_bits = P._spectral_weight(N, K, 21, top=(300.0, 200.0, 150.0, 100.0), tail=2.0)
    W = nv.bf16_bits_to_f64(W_bits)
    q_gpu = s_.quantize_weights(_t16(W_bits).cuda(), _t16(s_bits).cuda(), R=R)
    s_.check_device_error()
    q_ref = wq.quantize_weights(W_bits, s_bits, R=R)
    q_ref["smooth"] = s_bits
    err_gpu = np.linalg.norm(_effective(q_gpu, s_bits) - W) / np.linalg.norm(W)
    err_ref = np.linalg.norm(wq.effective_weight(q_ref) - W) / np.linalg.norm(W)
    assert err_gpu <= 1.05 * err_ref + 1e-4, (err_gpu, err_ref)
    # Eckart-Young: the low-rank part's truncation error is the discarded
    # spectrum, up to the factors' bf16 rounding and the float32 SVD
    s = nv.bf16_bits_to_f64(s_bits)
    Ws = W / s[None, :]
    LRs = (nv.bf16_bits_to_f64(H.bits(q_gpu["proj_up"].cpu()))
           @ nv.bf16_bits_to_f64(H.bits(q_gpu["proj_down"].cpu())).T) / s[None, :]
    S = q_ref["S"]
    opt = np.sqrt((S[R:] ** 2).sum())
    assert abs(np.linalg.norm(Ws - LRs) - opt) <= 2.0 ** -7 * np.linalg.norm(LRs) + 1e-3 * opt
    # and the layer through the CUDA path with these operands
    M = 96
    x = torch.randn(M, K, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    dev = q_gpu
    wt = s_.repack_weights(dev["wscales"])
    qa, asc, lr = s_.quantize_act(x.cuda(), _t16(s_bits).cuda(), dev["proj_down"])
    y = s_.w4a4_linear(qa, asc, lr, dev["qweight"], wt, dev["wcscales"], dev["wtscale"],
                       dev["proj_up"], None)
    s_.check_device_error()
    xd = nv.bf16_bits_to_f64(H.bits(x))
    y_true = xd @ W.T
    rel = np.linalg.norm(y.cpu().double().numpy() - y_true) / np.linalg.norm(y_true)
    rel_ref = np.linalg.norm(xd @ wq.effective_weight(q_ref).T - y_true) / np.linalg.norm(y_true)
    # activation quantization adds error of its own; the low-rank branch is
    # exact apart from bf16 rounding
    assert rel <= 2.0 * rel_ref + 0.02, (rel, rel_ref)


def test_residual_encoding_bit_exact_at_the_qkv_shape():
    # the full pipeline at N = 11520, K = 3840, R = 128; the device's own
    # float32 low-rank part handed to the oracle, which must then encode
    # the residual identically
    s_ = H.svdq()
    N, K, R = 11520, 3840, 128
    W, s = _random_weight(N, K, 77, scale=0.02)
    q = s_.quantize_weights(W.cuda(), s.cuda(), R=R, return_lowrank=True)
    s_.check_device_error()
    lr = q["lowrank"].cpu().numpy()
    res = wq.residual_f32(H.bits(W), H.bits(s), lr)
    _assert_same_encoding((q["qweight"], q["wscales"], q["wcscales"], q["wtscale"]),
                          wq.quantize_residual(res), "qkv shape")
