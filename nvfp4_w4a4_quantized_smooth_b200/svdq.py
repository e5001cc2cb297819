"""Thin ctypes binding of libsvdq.so (include/svdq.h), same call names.

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  Tensors are torch CUDA tensors (torch supplies device
memory and streams); each wrapper checks dtypes / contiguity, passes raw
device pointers and the current stream, and raises ``SvdqError`` on a
non-OK status.  There is no CPU fallback: if the library cannot be loaded
the import of this module fails.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsvdq.so")

SVDQ_OK = 0
SVDQ_ERR_INVALID_ARG = 1
SVDQ_ERR_SHAPE = 2
SVDQ_ERR_ALIGNMENT = 3
SVDQ_ERR_UNSUPPORTED = 4
SVDQ_ERR_ARCH = 5
SVDQ_ERR_CUDA = 6
SVDQ_ERR_TIMEOUT = 7

# Constants of include/svdq.h.
ABI_VERSION = 11
SCALES_ACT = 0
SCALES_WEIGHT = 1
GEMM_TOKEN_MAJOR = 0
GEMM_FEW_TOKENS = 1
GEMM_PAIRS = 2

# Every symbol include/svdq.h declares, with (restype, argtypes).
_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t
SIGNATURES = {
    "svdq_status_string": (ctypes.c_char_p, [_I]),
    "svdq_abi_version": (_I, []),
    "svdq_ascales_tiled_bytes": (_SZ, [_I, _I]),
    "svdq_wscales_tiled_bytes": (_SZ, [_I, _I]),
    "svdq_lowrank_bytes": (_SZ, [_I, _I]),
    "svdq_repack_weights": (_I, [_P, _I, _I, _P, _P]),
    "svdq_quantize_act": (_I, [_P, _I, _I, _I, _P, _P, _I, _P, _P, _P, _P]),
    "svdq_w4a4_linear": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _I,
                              _P]),
    "svdq_fold_proj_up": (_I, [_P, _P, _P, _I, _I, _P, _P, _P]),
    "svdq_silu_mul_quantize_act": (_I, [_P, _P, _I, _I, _I, _P, _P, _I, _P, _P, _P, _P]),
    "svdq_quantize_plan": (_I, [_I, _I, ctypes.POINTER(_I), ctypes.POINTER(_I)]),
    "svdq_linear_plan": (_I, [_I, _I, _I, ctypes.POINTER(_I), ctypes.POINTER(_I),
                              ctypes.POINTER(_I)]),
    "svdq_unpack_scales": (_I, [_P, _I, _I, _I, _P, _P]),
    "svdq_silu_mul": (_I, [_P, _P, _P, _SZ, _P]),
    "svdq_weight_workspace_bytes": (_SZ, [_I]),
    "svdq_quantize_weights": (_I, [_P, _P, _P, _I, _I, _P, _P, _P, _P, _P, _P]),
    "svdq_quantize_weights_noalloc": (_I, [_P, _P, _P, _I, _I, _P, _P, _P, _P, _P]),
    "svdq_check_device_error": (_I, [_P]),
    "svdq_set_wait_timeout_ns": (_I, [ctypes.c_uint64]),
    "svdq_wait_probe": (_I, [_I, _P]),
}


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with "
            "`python -m nvfp4_w4a4_quantized_smooth_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if lib.svdq_abi_version() != ABI_VERSION:
        raise ImportError(f"{path} has ABI version {lib.svdq_abi_version()}, this binding "
                          f"expects {ABI_VERSION}: rebuild it")
    return lib


_lib = load_library()


class SvdqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.svdq_status_string(status).decode()
        super().__init__(f"{where}: {msg}")


def _check(status: int, where: str) -> None:
    if status != SVDQ_OK:
        raise SvdqError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, dtype, name: str, dim: Optional[int] = None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if dim is not None and t.dim() != dim:
        raise ValueError(f"{name} must have {dim} dims")


def abi_version() -> int:
    return _lib.svdq_abi_version()


def ascales_tiled_bytes(M: int, K: int) -> int:
    return _lib.svdq_ascales_tiled_bytes(M, K)


def wscales_tiled_bytes(N: int, K: int) -> int:
    return _lib.svdq_wscales_tiled_bytes(N, K)


def lowrank_bytes(M: int, R: int) -> int:
    return _lib.svdq_lowrank_bytes(M, R)


def repack_weights(wscales: torch.Tensor, out: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    """wscales [K/16, N] uint8 (e4m3 codes) -> tiled scale buffer (uint8)."""
    _need(wscales, torch.uint8, "wscales", 2)
    wscales = wscales.contiguous()
    K = wscales.shape[0] * 16
    N = wscales.shape[1]
    nbytes = wscales_tiled_bytes(N, K)
    if out is None:
        out = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=wscales.device)
    _check(_lib.svdq_repack_weights(_ptr(wscales), N, K, _ptr(out), _stream(stream)),
           "svdq_repack_weights")
    return out


def quantize_act(x: torch.Tensor, smooth: Optional[torch.Tensor],
                 proj_down: Optional[torch.Tensor],
                 qact: Optional[torch.Tensor] = None,
                 ascales_tiled: Optional[torch.Tensor] = None,
                 lowrank: Optional[torch.Tensor] = None, stream=None):
    """x [M, K] bf16 (row stride may exceed K) -> (qact, ascales_tiled, lowrank).

    smooth None: no smoothing.  proj_down None: the plain NVFP4 layer
    (R = 0); lowrank is then None."""
    _need(x, torch.bfloat16, "x", 2)
    if smooth is not None:
        _need(smooth, torch.bfloat16, "smooth", 1)
        smooth = smooth.contiguous()
    if proj_down is not None:
        _need(proj_down, torch.bfloat16, "proj_down", 2)
        proj_down = proj_down.contiguous()
    if x.stride(1) != 1:
        raise ValueError("x must have unit stride along K")
    M, K = x.shape
    R = 0 if proj_down is None else proj_down.shape[1]
    dev = x.device
    if qact is None:
        qact = torch.empty(M, K // 2, dtype=torch.uint8, device=dev)
    if ascales_tiled is None:
        ascales_tiled = torch.empty(max(ascales_tiled_bytes(M, K), 1), dtype=torch.uint8,
                                    device=dev)
    if lowrank is None and R:
        lowrank = torch.empty(M, R, dtype=torch.bfloat16, device=dev)
    _check(_lib.svdq_quantize_act(_ptr(x), M, K, x.stride(0), _ptr(smooth), _ptr(proj_down), R,
                                  _ptr(qact), _ptr(ascales_tiled), _ptr(lowrank if R else None),
                                  _stream(stream)),
           "svdq_quantize_act")
    return qact, ascales_tiled, (lowrank if R else None)


def silu_mul_quantize_act(a: torch.Tensor, b: torch.Tensor, smooth: Optional[torch.Tensor],
                          proj_down: Optional[torch.Tensor],
                          qact: Optional[torch.Tensor] = None,
                          ascales_tiled: Optional[torch.Tensor] = None,
                          lowrank: Optional[torch.Tensor] = None, stream=None):
    """quantize_act of x = silu(a) * b (the w2 input of a DiT feed-forward
    block), formed on the device without writing x -> (qact, ascales_tiled,
    lowrank)."""
    _need(a, torch.bfloat16, "a", 2)
    _need(b, torch.bfloat16, "b", 2)
    if a.shape != b.shape or a.stride() != b.stride() or a.stride(1) != 1:
        raise ValueError("a and b must have the same shape and strides, unit stride along K")
    if smooth is not None:
        _need(smooth, torch.bfloat16, "smooth", 1)
        smooth = smooth.contiguous()
    if proj_down is not None:
        _need(proj_down, torch.bfloat16, "proj_down", 2)
        proj_down = proj_down.contiguous()
    M, K = a.shape
    R = 0 if proj_down is None else proj_down.shape[1]
    dev = a.device
    if qact is None:
        qact = torch.empty(M, K // 2, dtype=torch.uint8, device=dev)
    if ascales_tiled is None:
        ascales_tiled = torch.empty(max(ascales_tiled_bytes(M, K), 1), dtype=torch.uint8,
                                    device=dev)
    if lowrank is None and R:
        lowrank = torch.empty(M, R, dtype=torch.bfloat16, device=dev)
    _check(_lib.svdq_silu_mul_quantize_act(_ptr(a), _ptr(b), M, K, a.stride(0), _ptr(smooth),
                                           _ptr(proj_down), R, _ptr(qact), _ptr(ascales_tiled),
                                           _ptr(lowrank if R else None), _stream(stream)),
           "svdq_silu_mul_quantize_act")
    return qact, ascales_tiled, (lowrank if R else None)


def w4a4_linear(qact: torch.Tensor, ascales_tiled: torch.Tensor,
                lowrank: Optional[torch.Tensor], qweight: torch.Tensor,
                wscales_tiled: torch.Tensor, wcscales: torch.Tensor, wtscale: torch.Tensor,
                proj_up: Optional[torch.Tensor], bias: Optional[torch.Tensor],
                y: Optional[torch.Tensor] = None, stream=None,
                proj_up_folded: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The block-scaled FP4 GEMM with the fused epilogue -> y [M, N] bf16.

    lowrank and proj_up None: the plain NVFP4 layer (R = 0).  proj_up_folded:
    fold_proj_up's factor for these proj_up / wcscales / wtscale (the GEMM
    for M > 128 then adds the low-rank product inside its accumulator)."""
    _need(qact, torch.uint8, "qact", 2)
    _need(qweight, torch.uint8, "qweight", 2)
    if (lowrank is None) != (proj_up is None):
        raise ValueError("lowrank and proj_up go together (both None for R = 0)")
    if lowrank is not None:
        _need(lowrank, torch.bfloat16, "lowrank", 2)
        _need(proj_up, torch.bfloat16, "proj_up", 2)
    if proj_up_folded is not None:
        _need(proj_up_folded, torch.bfloat16, "proj_up_folded", 2)
        if proj_up is None or proj_up_folded.shape != proj_up.shape:
            raise ValueError("proj_up_folded needs proj_up of the same shape")
    M = qact.shape[0]
    K = qact.shape[1] * 2
    N = qweight.shape[0]
    R = 0 if proj_up is None else proj_up.shape[1]
    if y is None:
        y = torch.empty(M, N, dtype=torch.bfloat16, device=qact.device)
    _check(_lib.svdq_w4a4_linear(_ptr(qact), _ptr(ascales_tiled), _ptr(lowrank),
                                 _ptr(qweight), _ptr(wscales_tiled), _ptr(wcscales),
                                 _ptr(wtscale), _ptr(proj_up), _ptr(proj_up_folded), _ptr(bias),
                                 M, N, K, R, _ptr(y), y.stride(0), _stream(stream)),
           "svdq_w4a4_linear")
    return y


def fold_proj_up(proj_up: torch.Tensor, wcscales: torch.Tensor, wtscale: torch.Tensor,
                 stream=None):
    """svdq_fold_proj_up -> (proj_up_folded [N, R] bf16, number of elements
    that cannot be folded).  Reads the count back (synchronizes the
    stream); pass the factor to w4a4_linear only when the count is 0."""
    _need(proj_up, torch.bfloat16, "proj_up", 2)
    N, R = proj_up.shape
    out = torch.empty_like(proj_up)
    count = torch.empty(1, dtype=torch.int32, device=proj_up.device)
    _check(_lib.svdq_fold_proj_up(_ptr(proj_up), _ptr(wcscales), _ptr(wtscale), N, R, _ptr(out),
                                  _ptr(count), _stream(stream)),
           "svdq_fold_proj_up")
    if stream is not None:
        stream.synchronize()
    else:
        torch.cuda.current_stream(proj_up.device).synchronize()
    return out, int(count.item())


def quantize_plan(M: int, K: int):
    """(rows per CTA, K split) svdq_quantize_act uses for [M, K] on this device."""
    bm, split = _I(), _I()
    _check(_lib.svdq_quantize_plan(M, K, ctypes.byref(bm), ctypes.byref(split)),
           "svdq_quantize_plan")
    return bm.value, split.value


def linear_plan(M: int, N: int, K: int):
    """(kernel, K split, grid) svdq_w4a4_linear uses for M x N x K on this
    device; kernel is GEMM_PAIRS, GEMM_TOKEN_MAJOR or GEMM_FEW_TOKENS."""
    kernel, split, grid = _I(), _I(), _I()
    _check(_lib.svdq_linear_plan(M, N, K, ctypes.byref(kernel), ctypes.byref(split),
                                 ctypes.byref(grid)),
           "svdq_linear_plan")
    return kernel.value, split.value, grid.value


def unpack_scales(scales_tiled: torch.Tensor, rows: int, K: int, kind: str = "act",
                  stream=None) -> torch.Tensor:
    """Tiled scales -> logical [rows, K/16] uint8 (test / inspection helper).

    kind: "act" for svdq_quantize_act's order, "weight" for
    svdq_repack_weights' order."""
    code = {"act": SCALES_ACT, "weight": SCALES_WEIGHT}[kind]
    out = torch.empty(rows, K // 16, dtype=torch.uint8, device=scales_tiled.device)
    _check(_lib.svdq_unpack_scales(_ptr(scales_tiled), rows, K, code, _ptr(out),
                                   _stream(stream)),
           "svdq_unpack_scales")
    return out


def silu_mul(a: torch.Tensor, b: torch.Tensor, out: Optional[torch.Tensor] = None,
             stream=None) -> torch.Tensor:
    """silu(a) * b elementwise, bf16 (the w2 input of a DiT FFN block)."""
    _need(a, torch.bfloat16, "a")
    _need(b, torch.bfloat16, "b")
    if a.shape != b.shape or not a.is_contiguous() or not b.is_contiguous():
        raise ValueError("a and b must be contiguous with the same shape")
    if out is None:
        out = torch.empty_like(a)
    _check(_lib.svdq_silu_mul(_ptr(a), _ptr(b), _ptr(out), a.numel(), _stream(stream)),
           "svdq_silu_mul")
    return out


def quantize_weights_residual(W: torch.Tensor, smooth: torch.Tensor,
                              lowrank: Optional[torch.Tensor] = None, stream=None):
    """NVFP4 encoding of (W - lowrank) / smooth (svdq_quantize_weights) ->
    (qweight [N, K/2] uint8, wscales [K/16, N] uint8 e4m3 codes, wcscales
    [N] bf16, wtscale [1] bf16)."""
    _need(W, torch.bfloat16, "W", 2)
    _need(smooth, torch.bfloat16, "smooth", 1)
    W = W.contiguous()
    smooth = smooth.contiguous()
    if lowrank is not None:
        _need(lowrank, torch.float32, "lowrank", 2)
        lowrank = lowrank.contiguous()
    N, K = W.shape
    dev = W.device
    qweight = torch.empty(N, K // 2, dtype=torch.uint8, device=dev)
    wscales = torch.empty(K // 16, N, dtype=torch.uint8, device=dev)
    wcscales = torch.empty(N, dtype=torch.bfloat16, device=dev)
    wtscale = torch.empty(1, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(_lib.svdq_weight_workspace_bytes(N), dtype=torch.uint8, device=dev)
    _check(_lib.svdq_quantize_weights(_ptr(W), _ptr(smooth), _ptr(lowrank), N, K, _ptr(qweight),
                                      _ptr(wscales), _ptr(wcscales), _ptr(wtscale), _ptr(ws),
                                      _stream(stream)),
           "svdq_quantize_weights")
    return qweight, wscales, wcscales, wtscale


def quantize_weights(W: torch.Tensor, smooth: torch.Tensor, R: int = 128, stream=None,
                     return_lowrank: bool = False):
    """Offline weight side of the layer: a bf16 weight [N, K] and its
    smoothing factor [K] -> the stored operands (a dict: qweight, wscales,
    wcscales, wtscale, proj_down [K, R], proj_up [N, R]).

    The low-rank factors are the rank-R truncated SVD of W / smooth
    (proj_up = U_R S_R^1/2, proj_down = diag(smooth) V_R S_R^1/2, bf16),
    computed with torch's linear algebra on the device (a library SVD and
    GEMM: this runs once per layer at load time, not on the layer's path);
    the residual and its NVFP4 encoding run in svdq_quantize_weights.
    return_lowrank adds the float32 proj_up @ proj_down^T the encoding
    used (for tests)."""
    _need(W, torch.bfloat16, "W", 2)
    _need(smooth, torch.bfloat16, "smooth", 1)
    N, K = W.shape
    if R > min(N, K):
        raise ValueError("R exceeds the weight's rank bound")
    s = smooth.float()
    if R > 0:
        U, S, Vh = torch.linalg.svd(W.float() / s[None, :], full_matrices=False)
        sq = S[:R].sqrt()
        proj_up = (U[:, :R] * sq[None, :]).to(torch.bfloat16).contiguous()
        proj_down = (Vh[:R].T * sq[None, :] * s[:, None]).to(torch.bfloat16).contiguous()
        lowrank = proj_up.float() @ proj_down.float().T
    else:
        proj_up = torch.zeros(N, 0, dtype=torch.bfloat16, device=W.device)
        proj_down = torch.zeros(K, 0, dtype=torch.bfloat16, device=W.device)
        lowrank = None
    qweight, wscales, wcscales, wtscale = quantize_weights_residual(W, smooth, lowrank,
                                                                    stream=stream)
    out = dict(qweight=qweight, wscales=wscales, wcscales=wcscales, wtscale=wtscale,
               proj_down=proj_down, proj_up=proj_up)
    if return_lowrank:
        out["lowrank"] = lowrank
    return out


def check_device_error(stream=None) -> None:
    """Synchronize the stream and raise if a kernel recorded an error."""
    _check(_lib.svdq_check_device_error(_stream(stream)), "svdq_check_device_error")


def set_wait_timeout_ns(ns: int) -> None:
    _check(_lib.svdq_set_wait_timeout_ns(ns), "svdq_set_wait_timeout_ns")


def wait_probe(arrive: bool, stream=None) -> None:
    """Enqueue one bounded wait that completes only if ``arrive``; without
    it the wait runs out and the next check_device_error raises."""
    _check(_lib.svdq_wait_probe(1 if arrive else 0, _stream(stream)), "svdq_wait_probe")


class PreparedWeights:
    """One layer's device weights with the scales already repacked and (fold
    True, R > 0) the up-projection folded where every element folds."""

    def __init__(self, qweight, wscales, wcscales, wtscale, smooth, proj_down, proj_up,
                 bias=None, stream=None, fold=True):
        self.qweight = qweight
        self.wscales_tiled = repack_weights(wscales, stream=stream)
        self.proj_up_folded = None
        if fold and proj_up is not None and proj_up.shape[1] > 0:
            folded, bad = fold_proj_up(proj_up, wcscales, wtscale, stream=stream)
            self.proj_up_folded = folded if bad == 0 else None
        self.wcscales = wcscales
        self.wtscale = wtscale
        self.smooth = smooth
        self.proj_down = proj_down
        self.proj_up = proj_up
        self.bias = bias
        self.N = qweight.shape[0]
        self.K = qweight.shape[1] * 2


def svdq_linear(x: torch.Tensor, w: PreparedWeights, y: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
    """Whole layer on device tensors: svdq_quantize_act then svdq_w4a4_linear."""
    qact, asc, lr = quantize_act(x, w.smooth, w.proj_down, stream=stream)
    return w4a4_linear(qact, asc, lr, w.qweight, w.wscales_tiled, w.wcscales, w.wtscale,
                       w.proj_up, w.bias, y=y, stream=stream, proj_up_folded=w.proj_up_folded)
