"""The 30-block DiT stack at M = 4352: all 150 linears (qkv, out, w1, w3,
w2 per block, each with its own seeded weights) through the C ABI, checked
against the fp64 oracle.

Blocks 0, 14 and 29: every row and column of every linear, with every
code and scale bit-exact.  Every other linear: 256 seeded rows, all
columns of y, and the codes and scales of those rows.  The w2 input is
silu(y_w1) * y_w3 of the GPU's own bf16 outputs, formed on chip by the
fused activation kernel; its oracle input is the oracle's own silu_mul of
those outputs, so errors do not compound.
"""

import numpy as np
import pytest
import torch

from nvfp4_w4a4_quantized_smooth_b200 import synth

import gpu_helpers as H

pytestmark = pytest.mark.gpu

FULL_BLOCKS = (0, 14, 29)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from nvfp4_w4a4_quantized_smooth_b200 import build
    build.build()
    torch.cuda.init()
    yield


def test_dit_stack_30_blocks():
    import oracle
    s = H.svdq()
    M = synth.TOKENS
    host = synth.make_stack()
    assert len(host) == synth.DIT_BLOCKS
    for b, layers in enumerate(host):
        xd = layers["qkv"].x.cuda()
        y13 = {}
        for i, (name, K, N) in enumerate(synth.DIT_BLOCK_LINEARS):
            L = layers[name]
            assert (L.K, L.N) == (K, N)
            w = s.PreparedWeights(L.qweight.cuda(), L.wscales.cuda(), L.wcscales.cuda(),
                                  L.wtscale.cuda(), L.smooth.cuda(), L.proj_down.cuda(),
                                  L.proj_up.cuda(), L.bias.cuda())
            if name == "w2":
                # w2's input formed on chip from w1's and w3's outputs
                qa, asc, lr = s.silu_mul_quantize_act(y13["w1"], y13["w3"], w.smooth,
                                                      w.proj_down)
            else:
                qa, asc, lr = s.quantize_act(xd, w.smooth, w.proj_down)
            y = s.w4a4_linear(qa, asc, lr, w.qweight, w.wscales_tiled, w.wcscales, w.wtscale,
                              w.proj_up, w.bias)
            s.check_device_error()
            full = b in FULL_BLOCKS
            rows = np.arange(M) if full else H.sample_rows(M, 256, seed=4000 + 10 * b + i)
            rt = torch.from_numpy(rows).cuda()
            what = f"block {b} {name}"
            if name == "w2":
                h_ref = oracle.silu_mul(H.bits(y13["w1"][rt].cpu()), H.bits(y13["w3"][rt].cpu()))
                x_rows = torch.from_numpy(h_ref.view(np.int16)).view(torch.bfloat16)
            else:
                x_rows = L.x[torch.from_numpy(rows)]
            y_ref, q_ref, a_ref, L_ref = H.oracle_y(L, x=x_rows)
            H.assert_quant_exact(qa[rt].cpu(), s.unpack_scales(asc, M, K)[rt].cpu(), q_ref, a_ref,
                                 what)
            H.assert_y_close(y[rt].cpu(), y_ref, what)
            H.assert_lowrank_close(lr[rt].cpu(), L_ref, what)
            if name in ("w1", "w3"):
                y13[name] = y
            del qa, asc, lr, y, w
        del xd, y13
        torch.cuda.empty_cache()
