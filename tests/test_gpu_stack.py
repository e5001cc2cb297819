"""The 30-block DiT stack at M = 4352: all 150 linears (qkv, out, w1, w3,
w2 per block, each with its own seeded weights) through the C ABI, checked
against the fp64 oracle.

Blocks 0, 14 and 29: 16 sampled rows of every linear, all columns, with
their codes and scales bit-exact; block 0's whole input is also quantized
and compared code for code.  Every other linear: 8 sampled rows x 64
sampled columns of y, and the codes and scales of those rows.  The w2
input is silu(y_w1) * y_w3 of the GPU's own bf16 outputs, formed on chip by
the fused activation kernel; its oracle takes that same input (formed by
svdq_silu_mul, bit for bit the same), so errors do not compound.
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
    s = H.svdq()
    M = synth.TOKENS
    host = synth.make_stack()
    assert len(host) == synth.DIT_BLOCKS
    rng = np.random.default_rng(4000)
    records = []
    for b, layers in enumerate(host):
        xd = layers["qkv"].x.cuda()
        y13 = {}
        h = None
        for i, (name, K, N) in enumerate(synth.DIT_BLOCK_LINEARS):
            L = layers[name]
            assert (L.K, L.N) == (K, N)
            w = s.PreparedWeights(L.qweight.cuda(), L.wscales.cuda(), L.wcscales.cuda(),
                                  L.wtscale.cuda(), L.smooth.cuda(), L.proj_down.cuda(),
                                  L.proj_up.cuda(), L.bias.cuda())
            if name == "w2":
                # w2's input formed on chip from w1's and w3's outputs; the
                # oracle takes the same x, formed by svdq_silu_mul
                x_in = h
                qa, asc, lr = s.silu_mul_quantize_act(y13["w1"], y13["w3"], w.smooth,
                                                      w.proj_down)
            else:
                x_in = xd
                qa, asc, lr = s.quantize_act(x_in, w.smooth, w.proj_down)
            y = s.w4a4_linear(qa, asc, lr, w.qweight, w.wscales_tiled, w.wcscales, w.wtscale,
                              w.proj_up, w.bias)
            s.check_device_error()
            full = b in FULL_BLOCKS
            rows = H.sample_rows(M, 16 if full else 8, seed=4000 + 10 * b + i)
            cols = None if full else np.sort(rng.choice(N, 64, replace=False))
            rt = torch.from_numpy(rows).cuda()
            asc_rows = s.unpack_scales(asc, M, K)[rt].cpu()
            y_s = y[rt].cpu() if cols is None else y[rt][:, torch.from_numpy(cols).cuda()].cpu()
            x_rows = x_in[rt].cpu()
            records.append((b, name, L, rows, cols, y_s, qa[rt].cpu(), asc_rows, x_rows))
            if b == 0 and name == "qkv":
                q_ref, a_ref = H.oracle_quant(L.x, L.smooth)
                H.assert_quant_exact(qa.cpu(), s.unpack_scales(asc, M, K).cpu(), q_ref, a_ref,
                                     "block 0 input, every code")
            if name in ("w1", "w3"):
                y13[name] = y
                if name == "w3":
                    h = s.silu_mul(y13["w1"], y13["w3"])
        del xd, y13, h
        torch.cuda.empty_cache()

    for b, name, L, rows, cols, y_s, qa_rows, asc_rows, x_rows in records:
        what = f"block {b} {name}"
        y_ref, q_ref, a_ref, _ = H.oracle_y(L, rows=np.arange(len(rows)), cols=cols, x=x_rows)
        H.assert_quant_exact(qa_rows, asc_rows, q_ref, a_ref, what)
        H.assert_y_close(y_s, y_ref, what)
