"""svdq_quantize_weights_noalloc: the weight encoding for callers that cannot
allocate device memory (code inside a framework or memory pool that owns
all device memory, or a thread that must not call cudaMalloc), with its
scratch in a fixed array inside the library instead of a caller workspace.

Called through the C ABI twice in a row -- a weight with large values, then
one with small values, so that a global amax left over from the first call
would show in the second -- each result must equal, bit for bit, what the
workspace entry point svdq_quantize_weights gives for the same input.  The
file runs last in a collected session and also passes alone in a fresh
process (the first call on the device sets up the array's address).
"""

import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from nvfp4_w4a4_quantized_smooth_b200 import build
    build.build()
    torch.cuda.init()
    from nvfp4_w4a4_quantized_smooth_b200 import svdq
    return svdq


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _outputs(N, K, dev):
    return (torch.empty(N, K // 2, dtype=torch.uint8, device=dev),
            torch.empty(K // 16, N, dtype=torch.uint8, device=dev),
            torch.empty(N, dtype=torch.bfloat16, device=dev),
            torch.empty(1, dtype=torch.bfloat16, device=dev))


def _encode(svdq, W, smooth, lowrank, noalloc):
    N, K = W.shape
    out = _outputs(N, K, W.device)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if noalloc:
        st = svdq._lib.svdq_quantize_weights_noalloc(_ptr(W), _ptr(smooth), _ptr(lowrank), N, K,
                                                    *[_ptr(t) for t in out], stream)
    else:
        ws = torch.empty(svdq._lib.svdq_weight_workspace_bytes(N), dtype=torch.uint8,
                         device=W.device)
        st = svdq._lib.svdq_quantize_weights(_ptr(W), _ptr(smooth), _ptr(lowrank), N, K,
                                            *[_ptr(t) for t in out], _ptr(ws), stream)
    assert st == svdq.SVDQ_OK, st
    svdq.check_device_error()
    return [t.cpu() for t in out]


def _weight(N, K, scale, seed):
    g = torch.Generator().manual_seed(seed)
    W = (torch.randn(N, K, generator=g) * scale).to(torch.bfloat16).cuda()
    s = (torch.rand(K, generator=g) + 0.5).to(torch.bfloat16).cuda()
    lr = (torch.randn(N, K, generator=g) * scale * 0.1).float().cuda()
    return W, s, lr


def test_noalloc_matches_the_workspace_entry_point_on_two_calls_in_a_row(lib):
    for scale, seed in ((100.0, 1), (0.01, 2)):
        W, s, lr = _weight(3840, 1024, scale, seed)
        got = _encode(lib, W, s, lr, noalloc=True)
        want = _encode(lib, W, s, lr, noalloc=False)
        for g, w in zip(got, want):
            assert torch.equal(g.view(torch.uint8) if g.dtype != torch.uint8 else g,
                               w.view(torch.uint8) if w.dtype != torch.uint8 else w), scale


def test_noalloc_rejects_more_rows_than_its_array_holds(lib):
    fake = ctypes.c_void_p(0x1000)
    st = lib._lib.svdq_quantize_weights_noalloc(fake, fake, None, 32769, 64, fake, fake, fake,
                                                fake, None)
    assert st == lib.SVDQ_ERR_UNSUPPORTED
