"""Host-side checks of the C ABI (no GPU needed).

The library must load, export every function include/svdq.h declares,
answer size queries and reject bad arguments before touching the device.
"""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "svdq.h")


@pytest.fixture(scope="module")
def svdq():
    from nvfp4_w4a4_quantized_smooth_b200 import build
    build.build()
    from nvfp4_w4a4_quantized_smooth_b200 import svdq as mod
    return mod


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(svdq_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_path():
    names = declared_functions()
    for n in ("svdq_repack_weights", "svdq_quantize_act", "svdq_w4a4_linear"):
        assert n in names


def test_library_exports_every_declared_symbol(svdq):
    lib = ctypes.CDLL(svdq.LIB_PATH)
    names = declared_functions()
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    # and the binding knows the signature of each one
    assert sorted(svdq.SIGNATURES) == names


def test_abi_version_and_status_strings(svdq):
    assert svdq.abi_version() == 11 == svdq.ABI_VERSION
    for st in range(8):
        s = svdq._lib.svdq_status_string(st).decode()
        assert s.startswith("SVDQ")
    assert "unknown" in svdq._lib.svdq_status_string(99).decode()


def test_size_queries(svdq):
    assert svdq.ascales_tiled_bytes(128, 512) == 1 * 8 * 512
    assert svdq.ascales_tiled_bytes(129, 512) == 2 * 8 * 512
    assert svdq.ascales_tiled_bytes(4352, 3840) == 34 * 60 * 512
    assert svdq.wscales_tiled_bytes(512, 512) == 4 * 8 * 512
    assert svdq.wscales_tiled_bytes(11520, 3840) == 90 * 60 * 512
    assert svdq.wscales_tiled_bytes(100, 64) == 2 * 1 * 512
    assert svdq.lowrank_bytes(4352, 128) == 4352 * 128 * 2
    assert svdq._lib.svdq_weight_workspace_bytes(11520) == 11521 * 4
    assert svdq._lib.svdq_weight_workspace_bytes(0) == 0
    for bad in ((0, 64), (16, 32), (16, 100)):
        assert svdq.ascales_tiled_bytes(*bad) == 0
        assert svdq.wscales_tiled_bytes(*bad) == 0


def test_argument_checks_fail_before_any_device_work(svdq):
    lib = svdq._lib
    P = ctypes.c_void_p
    fake = P(0x1000)            # never dereferenced: checks fail first
    # null pointers
    assert lib.svdq_quantize_act(None, 16, 64, 64, fake, fake, 128, fake, fake, fake,
                                 None) == svdq.SVDQ_ERR_INVALID_ARG
    assert lib.svdq_w4a4_linear(fake, fake, fake, fake, fake, fake, fake, fake, None, None, 16,
                                64, 256, 128, None, 64, None) == svdq.SVDQ_ERR_INVALID_ARG
    assert lib.svdq_repack_weights(None, 64, 64, fake, None) == svdq.SVDQ_ERR_INVALID_ARG
    # shapes
    assert lib.svdq_quantize_act(fake, 0, 64, 64, fake, fake, 128, fake, fake, fake,
                                 None) == svdq.SVDQ_ERR_SHAPE
    assert lib.svdq_quantize_act(fake, 16, 40, 40, fake, fake, 128, fake, fake, fake,
                                 None) == svdq.SVDQ_ERR_SHAPE
    assert lib.svdq_quantize_act(fake, 16, 64, 32, fake, fake, 128, fake, fake, fake,
                                 None) == svdq.SVDQ_ERR_SHAPE
    assert lib.svdq_w4a4_linear(fake, fake, fake, fake, fake, fake, fake, fake, None, None, 16,
                                64, 256, 128, fake, 32, None) == svdq.SVDQ_ERR_SHAPE
    # implemented limits
    assert lib.svdq_quantize_act(fake, 16, 64, 64, fake, fake, 64, fake, fake, fake,
                                 None) == svdq.SVDQ_ERR_UNSUPPORTED
    assert lib.svdq_quantize_act(fake, 16, 80, 80, fake, fake, 128, fake, fake, fake,
                                 None) == svdq.SVDQ_ERR_UNSUPPORTED
    assert lib.svdq_w4a4_linear(fake, fake, fake, fake, fake, fake, fake, fake, None, None, 16,
                                64, 192, 128, fake, 64, None) == svdq.SVDQ_ERR_UNSUPPORTED
    assert lib.svdq_w4a4_linear(fake, fake, fake, fake, fake, fake, fake, fake, None, None, 16,
                                48, 256, 128, fake, 48, None) == svdq.SVDQ_ERR_UNSUPPORTED
    # alignment
    odd = P(0x1001)
    assert lib.svdq_quantize_act(odd, 16, 64, 64, fake, fake, 128, fake, fake, fake,
                                 None) == svdq.SVDQ_ERR_ALIGNMENT
    assert lib.svdq_quantize_act(fake, 16, 64, 68, fake, fake, 128, fake, fake, fake,
                                 None) == svdq.SVDQ_ERR_ALIGNMENT
    assert lib.svdq_w4a4_linear(fake, fake, fake, fake, fake, fake, fake, fake, None, odd, 16,
                                64, 256, 128, fake, 64, None) == svdq.SVDQ_ERR_ALIGNMENT
    assert lib.svdq_w4a4_linear(fake, fake, fake, fake, fake, fake, fake, fake, odd, None, 16,
                                64, 256, 128, fake, 64, None) == svdq.SVDQ_ERR_ALIGNMENT
    # the folded up-projection: arguments, shape, R % 8, alignment
    assert lib.svdq_fold_proj_up(None, fake, fake, 64, 128, fake, fake,
                                 None) == svdq.SVDQ_ERR_INVALID_ARG
    assert lib.svdq_fold_proj_up(fake, fake, fake, 64, 128, fake, None,
                                 None) == svdq.SVDQ_ERR_INVALID_ARG
    assert lib.svdq_fold_proj_up(fake, fake, fake, 0, 128, fake, fake,
                                 None) == svdq.SVDQ_ERR_SHAPE
    assert lib.svdq_fold_proj_up(fake, fake, fake, 64, 12, fake, fake,
                                 None) == svdq.SVDQ_ERR_UNSUPPORTED
    assert lib.svdq_fold_proj_up(odd, fake, fake, 64, 128, fake, fake,
                                 None) == svdq.SVDQ_ERR_ALIGNMENT
    # R = 0 (no low-rank branch): proj_down, lowrank, proj_up and smooth may
    # be null; the other checks still apply
    assert lib.svdq_quantize_act(fake, 0, 64, 64, None, None, 0, fake, fake, None,
                                 None) == svdq.SVDQ_ERR_SHAPE
    assert lib.svdq_quantize_act(fake, 16, 64, 64, None, None, 0, None, fake, None,
                                 None) == svdq.SVDQ_ERR_INVALID_ARG
    assert lib.svdq_quantize_act(fake, 16, 64, 64, None, None, 128, fake, fake, fake,
                                 None) == svdq.SVDQ_ERR_INVALID_ARG      # R = 128 needs proj_down
    assert lib.svdq_w4a4_linear(fake, fake, None, fake, fake, fake, fake, None, None, None, 16,
                                48, 256, 0, fake, 48, None) == svdq.SVDQ_ERR_UNSUPPORTED
    assert lib.svdq_w4a4_linear(fake, fake, None, fake, fake, fake, fake, None, None, None, 16,
                                64, 256, 128, fake, 64, None) == svdq.SVDQ_ERR_INVALID_ARG
    # the fused w2 activation: b is required, the other checks as quantize_act
    assert lib.svdq_silu_mul_quantize_act(fake, None, 16, 64, 64, fake, fake, 128, fake, fake,
                                          fake, None) == svdq.SVDQ_ERR_INVALID_ARG
    assert lib.svdq_silu_mul_quantize_act(fake, fake, 16, 64, 32, fake, fake, 128, fake, fake,
                                          fake, None) == svdq.SVDQ_ERR_SHAPE
    assert lib.svdq_silu_mul_quantize_act(fake, odd, 16, 64, 64, fake, fake, 128, fake, fake,
                                          fake, None) == svdq.SVDQ_ERR_ALIGNMENT
    # the offline weight quantizer: lowrank may be null, the rest may not;
    # K a multiple of 16; 16-byte aligned W and lowrank
    assert lib.svdq_quantize_weights(fake, fake, None, 32, 64, fake, fake, fake, fake, None,
                                     None) == svdq.SVDQ_ERR_INVALID_ARG
    assert lib.svdq_quantize_weights(None, fake, None, 32, 64, fake, fake, fake, fake, fake,
                                     None) == svdq.SVDQ_ERR_INVALID_ARG
    assert lib.svdq_quantize_weights(fake, fake, None, 32, 40, fake, fake, fake, fake, fake,
                                     None) == svdq.SVDQ_ERR_SHAPE
    assert lib.svdq_quantize_weights(fake, fake, None, 0, 64, fake, fake, fake, fake, fake,
                                     None) == svdq.SVDQ_ERR_SHAPE
    assert lib.svdq_quantize_weights(odd, fake, None, 32, 64, fake, fake, fake, fake, fake,
                                     None) == svdq.SVDQ_ERR_ALIGNMENT
    assert lib.svdq_quantize_weights(fake, fake, P(0x1004), 32, 64, fake, fake, fake, fake, fake,
                                     None) == svdq.SVDQ_ERR_ALIGNMENT
    # scale unpack: only the two documented tile orders
    for kind in (-1, 2):
        assert lib.svdq_unpack_scales(fake, 16, 64, kind, fake, None) == svdq.SVDQ_ERR_INVALID_ARG
    assert lib.svdq_unpack_scales(fake, 0, 64, svdq.SCALES_ACT, fake,
                                  None) == svdq.SVDQ_ERR_SHAPE


def test_device_calls_without_a_gpu_report_an_error(svdq):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    P = ctypes.c_void_p
    fake = P(0x1000)
    st = svdq._lib.svdq_quantize_act(fake, 16, 64, 64, fake, fake, 128, fake, fake, fake, None)
    assert st in (svdq.SVDQ_ERR_CUDA, svdq.SVDQ_ERR_ARCH)
