"""svdq_silu_mul (the input of the w2 feed-forward linear, silu(a) * b
rounded once to bf16) against the oracle's ``silu_mul``, bit for bit.

The oracle rounds the exact product (float64, refined with 400-digit
decimal arithmetic next to bf16 rounding boundaries); the kernel computes
in float32 and falls back to float64 next to those boundaries.  Inputs:
every finite bf16 a with several b, the large-negative a where exp(-a)
leaves the float range, products in the bf16 subnormal range and near its
smallest normal, planted exact-midpoint products at large a, and a wide
random sample.
"""

import numpy as np
import pytest
import torch

import oracle
from nvfp4_w4a4_quantized_smooth_b200 import synth

import gpu_helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from nvfp4_w4a4_quantized_smooth_b200 import build
    build.build()
    torch.cuda.init()
    yield


def _bits_tensor(values):
    return torch.tensor(values, dtype=torch.float64).to(torch.bfloat16)


def _gpu_vs_oracle(a: torch.Tensor, b: torch.Tensor, what: str):
    s = H.svdq()
    h = s.silu_mul(a.contiguous().cuda(), b.contiguous().cuda())
    s.check_device_error()
    got = synth.bits(h.cpu())
    want = oracle.silu_mul(synth.bits(a), synth.bits(b))
    bad = np.flatnonzero(got.reshape(-1) != want.reshape(-1))
    if bad.size:
        av = a.reshape(-1).float()
        bv = b.reshape(-1).float()
        ex = [(float(av[i]), float(bv[i]), hex(got.reshape(-1)[i]), hex(want.reshape(-1)[i]))
              for i in bad[:6]]
        raise AssertionError(f"{what}: {bad.size} of {got.size} outputs differ, e.g. {ex}")


def _all_finite_bf16():
    pos = torch.arange(0, 0x7F80, dtype=torch.int32)
    u = torch.cat([pos, pos | 0x8000]).to(torch.int16)
    return u.view(torch.bfloat16)


@pytest.mark.parametrize("bv", [1.0, -0.75, 3.140625, 2.0 ** -100, -(2.0 ** 90), 1.0 + 2.0 ** -7])
def test_silu_mul_every_bf16_a(bv):
    a = _all_finite_bf16()
    b = _bits_tensor([bv]).expand(a.shape[0]).contiguous()
    _gpu_vs_oracle(a, b, f"every a, b = {bv}")


def test_silu_mul_edge_inputs():
    rng = np.random.default_rng(31)
    # every bf16 a in [-100, -80] (exp(-a) beyond the float range below
    # -88.7), against many b, products down to the bf16 subnormals
    neg = _all_finite_bf16()
    neg = neg[(neg.float() <= -80) & (neg.float() >= -100)]
    bs = _bits_tensor(np.concatenate([rng.standard_normal(40),
                                      np.exp(rng.uniform(-10, 80, 40)) * rng.choice([-1, 1], 40)]))
    a1 = neg.repeat_interleave(bs.shape[0])
    b1 = bs.repeat(neg.shape[0])
    # |a| > 20 both signs, with b spread over the exponent range
    big = _bits_tensor(np.concatenate([rng.uniform(20, 3000, 20000), -rng.uniform(20, 80, 20000)]))
    b2 = _bits_tensor(np.exp(rng.uniform(-80, 80, 40000)) * rng.choice([-1, 1], 40000))
    # products near the smallest normal 2^-126: b chosen from silu(a)
    a3 = _bits_tensor(rng.standard_normal(40000) * 3)
    s3 = a3.double() / (1 + torch.exp(-a3.double()))
    target = 2.0 ** rng.uniform(-134, -120, 40000)
    b3 = (torch.from_numpy(target) / s3.clamp(min=1e-30) * torch.sign(s3)).to(torch.bfloat16)
    keep = torch.isfinite(b3.float()) & (b3.float() != 0)
    a3, b3 = a3[keep], b3[keep]
    # signed zeros
    a4 = _bits_tensor([0.0, -0.0, 0.0, -0.0, 5.0, -5.0, 0.0, -0.0])
    b4 = _bits_tensor([1.0, 1.0, -1.0, -1.0, 0.0, -0.0, 0.0, -0.0])
    # planted exact midpoints a * b at large a: silu(a) is just below a, so
    # the product rounds toward zero
    a5 = _bits_tensor([48.0, 96.0, 192.0, 384.0, 1536.0, 3072.0, 24576.0, 37888.0] * 2)
    b5 = _bits_tensor([1.0 + 2.0 ** -7] * 8 + [-(1.0 + 2.0 ** -7)] * 8)
    a = torch.cat([a1, big, a3, a4, a5])
    b = torch.cat([b1, b2, b3, b4, b5])
    _gpu_vs_oracle(a, b, "edge inputs")


@pytest.mark.parametrize("n", [1, 7, 8, 9, 1000, 4097, 3 * 1024 * 1024 + 5])
def test_silu_mul_random_and_tails(n):
    g = torch.Generator().manual_seed(n)
    a = (torch.randn(n, generator=g) * 4).to(torch.bfloat16)
    b = (torch.randn(n, generator=g) * torch.exp(torch.randn(n, generator=g) * 8)).to(torch.bfloat16)
    b = torch.where(torch.isfinite(b.float()), b, torch.ones_like(b))
    _gpu_vs_oracle(a, b, f"random n={n}")
