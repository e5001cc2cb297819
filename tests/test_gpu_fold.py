"""The folded up-projection (svdq_fold_proj_up) and the layer that uses it.

* The factor is bf16(proj_up / (wtscale * wcscales[n])) with the product
  exact in float32, the quotient correctly rounded to float32 and then
  rounded to nearest-even bf16: checked bit for bit against the same steps
  in NumPy / torch on the CPU, over magnitudes from tiny to huge.
* Elements that cannot be folded (a zero channel scale, a quotient that
  overflows bf16 or falls below its smallest normal) are counted, and a
  prepared weight with such elements keeps the unfolded form; the layer
  then still matches the oracle.
* The layer with the folded factor against the oracle at a ragged shape on
  the CTA-pair GEMM (the other parity tests run both forms everywhere).
"""

import numpy as np
import pytest
import torch

import gpu_helpers as H
from nvfp4_w4a4_quantized_smooth_b200 import synth

pytestmark = pytest.mark.gpu

F32_MIN_NORMAL = np.float32(2.0 ** -126)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from nvfp4_w4a4_quantized_smooth_b200 import build
    build.build()
    torch.cuda.init()
    yield


def _fold_on_cpu(pu, wc, wt):
    """The documented steps with IEEE float32 NumPy arithmetic -> (bf16
    tensor, unfoldable count)."""
    pu32 = pu.float().numpy()
    scale = (np.float32(wt.float().item()) * wc.float().numpy()).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        q = (pu32 / scale[:, None]).astype(np.float32)
    out = torch.from_numpy(q).to(torch.bfloat16)
    f = out.float().numpy()
    bad = ((scale[:, None] == 0) | ~np.isfinite(scale[:, None]) | ~np.isfinite(f)
           | ((f != 0) & (np.abs(f) < F32_MIN_NORMAL)))
    return out, int(bad.sum())


def _bf16(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def test_fold_bit_exact_over_magnitudes():
    s = H.svdq()
    rng = np.random.default_rng(31)
    N, R = 1000, 128
    pu = _bf16(rng.standard_normal((N, R)) * np.exp(rng.uniform(-20, 20, (N, 1))))
    wc = _bf16(np.exp(rng.uniform(-12, 0, N)))
    wt = _bf16([3.1e-4])
    got, bad = s.fold_proj_up(pu.cuda(), wc.cuda(), wt.cuda())
    s.check_device_error()
    want, want_bad = _fold_on_cpu(pu, wc, wt)
    assert bad == want_bad
    assert torch.equal(got.cpu().view(torch.int16), want.view(torch.int16))


def test_fold_counts_what_cannot_be_folded():
    s = H.svdq()
    rng = np.random.default_rng(32)
    N, R = 64, 128
    pu = rng.standard_normal((N, R)).astype(np.float32)
    wc = np.exp(rng.uniform(-3, 0, N)).astype(np.float32)
    wc[3] = 0.0                        # zero channel scale: the whole row
    wc[7], pu[7, :5] = 1.0, 2e-38      # 1e-38: below the smallest normal after the fold
    wc[9], pu[9, 0] = 0.05, 3e38       # 3e39: overflows after the fold
    pu[11, :] = 0.0                    # zeros fold to zeros
    pu, wc, wt = _bf16(pu), _bf16(wc), _bf16([2.0])
    got, bad = s.fold_proj_up(pu.cuda(), wc.cuda(), wt.cuda())
    s.check_device_error()
    want, want_bad = _fold_on_cpu(pu, wc, wt)
    assert want_bad >= R + 5 + 1
    assert bad == want_bad
    ok = torch.ones(N, dtype=torch.bool)
    ok[[3, 7, 9]] = False
    assert torch.equal(got.cpu()[ok].view(torch.int16), want[ok].view(torch.int16))


def test_prepared_weight_keeps_unfolded_form_when_a_channel_cannot_fold():
    s = H.svdq()
    M, K, N = 300, 512, 384
    L = synth.make_layer(M, K, N, seed=33)
    L.wcscales = L.wcscales.clone()
    L.wcscales[5] = 0                  # a channel whose block-scaled part is zero
    d = H.to_dev(L)
    w = s.PreparedWeights(d["qweight"], d["wscales"], d["wcscales"], d["wtscale"], d["smooth"],
                          d["proj_down"], d["proj_up"], d["bias"])
    assert w.proj_up_folded is None
    y = s.svdq_linear(d["x"], w)
    s.check_device_error()
    y_ref, *_ = H.oracle_y(L)
    H.assert_y_close(y.cpu(), y_ref, "unfoldable channel")
    L2 = synth.make_layer(M, K, N, seed=33)
    d2 = H.to_dev(L2)
    w2 = s.PreparedWeights(d2["qweight"], d2["wscales"], d2["wcscales"], d2["wtscale"],
                           d2["smooth"], d2["proj_down"], d2["proj_up"], d2["bias"])
    assert w2.proj_up_folded is not None
    y2 = s.svdq_linear(d2["x"], w2)
    s.check_device_error()
    y2_ref, *_ = H.oracle_y(L2)
    H.assert_y_close(y2.cpu(), y2_ref, "folded")


@pytest.mark.parametrize("M,K,N", [(129, 256, 32), (700, 1280, 800), (1000, 3840, 1056)])
def test_folded_layer_against_oracle(M, K, N):
    L = synth.make_layer(M, K, N, seed=M + K + N)
    r = H.gpu_layer(L)
    y_ref, *_ = H.oracle_y(L)
    H.assert_y_close(r["y_fold"], y_ref, f"folded {M}x{K}x{N}")
    # the folded and unfolded forms differ only by the factor's rounding
    yf = r["y_fold"].double()
    yu = r["y"].double()
    assert (yf - yu).norm() <= 2e-3 * yu.norm()
