"""Seeded synthetic operands for the SVDQuant W4A4 NVFP4 linear layer.

This module only draws random numbers and casts them with torch's own
dtype conversions; it holds none of the layer's arithmetic, so both the
CUDA path and the CPU oracle can take their inputs from it.

Distributions (one layer of a diffusion transformer, random weights):

* x         bf16 N(0, 1), [M, K]; optionally ``outliers`` distinct input
            channels (drawn from the seed) multiplied by ``outlier_scale``
            for every token before the bf16 cast.
* smooth    bf16 U(0.5, 2), [K].
* qweight   uint8 uniform over 0..255, [N, K/2]: both nibbles uniform over
            the 16 E2M1 codes.
* wscales   float8_e4m3fn of U(0.25, 2), [K/16, N], as raw uint8 codes.
* wcscales  bf16 U(0.5, 1.5), [N].
* wtscale   bf16 0.01, [1].
* proj_down bf16 N(0, 0.02), [K, R]; proj_up bf16 N(0, 0.02), [N, R].
* bias      bf16 N(0, 0.1), [N] (or None).

Seeds: one torch CPU generator per layer, seeded with ``seed``; every
tensor is drawn from it in the fixed order above.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch

R_DEFAULT = 128


@dataclass
class LayerOperands:
    """Host (CPU) operands of one layer, in the on-disk layouts."""
    x: Optional[torch.Tensor]  # [M, K] bfloat16 (None: formed on the device)
    smooth: torch.Tensor       # [K] bfloat16
    qweight: torch.Tensor      # [N, K/2] uint8
    wscales: torch.Tensor      # [K/16, N] uint8 (e4m3fn codes)
    wcscales: torch.Tensor     # [N] bfloat16
    wtscale: torch.Tensor      # [1] bfloat16
    proj_down: torch.Tensor    # [K, R] bfloat16
    proj_up: torch.Tensor      # [N, R] bfloat16
    bias: Optional[torch.Tensor]  # [N] bfloat16 or None

    @property
    def M(self) -> int:
        return self.x.shape[0]

    @property
    def K(self) -> int:
        return self.qweight.shape[1] * 2

    @property
    def N(self) -> int:
        return self.qweight.shape[0]

    @property
    def R(self) -> int:
        return self.proj_down.shape[1]


def make_x(M: int, K: int, gen: torch.Generator, outliers: int = 4,
           outlier_scale: float = 20.0) -> torch.Tensor:
    x = torch.randn(M, K, generator=gen, dtype=torch.float32)
    if outliers:
        ch = torch.randperm(K, generator=gen)[:outliers]
        x[:, ch] *= outlier_scale
    return x.to(torch.bfloat16)


def make_weights(K: int, N: int, R: int, gen: torch.Generator, with_bias: bool = True):
    """One layer's weights, drawn from `gen` in the fixed order of the module
    docstring: (smooth, qweight, wscales, wcscales, wtscale, proj_down,
    proj_up, bias)."""
    smooth = torch.empty(K).uniform_(0.5, 2.0, generator=gen).to(torch.bfloat16)
    qweight = torch.randint(0, 256, (N, K // 2), generator=gen, dtype=torch.uint8)
    wscales = (torch.empty(K // 16, N).uniform_(0.25, 2.0, generator=gen)
               .to(torch.float8_e4m3fn).view(torch.uint8))
    wcscales = torch.empty(N).uniform_(0.5, 1.5, generator=gen).to(torch.bfloat16)
    wtscale = torch.tensor([0.01], dtype=torch.float32).to(torch.bfloat16)
    proj_down = (torch.randn(K, R, generator=gen) * 0.02).to(torch.bfloat16)
    proj_up = (torch.randn(N, R, generator=gen) * 0.02).to(torch.bfloat16)
    bias = ((torch.randn(N, generator=gen) * 0.1).to(torch.bfloat16)
            if with_bias else None)
    return smooth, qweight, wscales, wcscales, wtscale, proj_down, proj_up, bias


def make_layer(M: int, K: int, N: int, R: int = R_DEFAULT, seed: int = 0,
               outliers: int = 4, outlier_scale: float = 20.0,
               with_bias: bool = True) -> LayerOperands:
    """Draw one layer's operands (see the module docstring)."""
    if K % 16 or K < 16:
        raise ValueError("K must be a positive multiple of 16")
    g = torch.Generator().manual_seed(int(seed))
    x = make_x(M, K, g, outliers, outlier_scale)
    return LayerOperands(x, *make_weights(K, N, R, g, with_bias))


# Named workloads: shapes of one Z-Image-class DiT (hidden 3840, FFN 10240,
# 4096 image tokens from a 64x64 latent patch grid + 256 text tokens).
TOKENS = 4352
HIDDEN = 3840
FFN = 10240

WORKLOADS = {
    # name: (M, K, N)
    "layer_m128_k512_n512": (128, 512, 512),
    "qkv_m4352_k3840_n11520": (TOKENS, HIDDEN, 3 * HIDDEN),
    "ffn_w1_m4352_k3840_n10240": (TOKENS, HIDDEN, FFN),
    "ffn_w3_m4352_k3840_n10240": (TOKENS, HIDDEN, FFN),
    "ffn_w2_m4352_k10240_n3840": (TOKENS, FFN, HIDDEN),
}
# The plain NVFP4 layer (no low-rank branch, no smoothing) at the qkv shape.
PLAIN_PREFIX = "nvfp4_"
WORKLOADS[PLAIN_PREFIX + "qkv_m4352_k3840_n11520"] = (TOKENS, HIDDEN, 3 * HIDDEN)

OUT_PROJ_SWEEP_M = (16, 64, 256, 1024, 4352, 17408)
for _m in OUT_PROJ_SWEEP_M:
    WORKLOADS[f"out_m{_m}_k3840_n3840"] = (_m, HIDDEN, HIDDEN)

# Per-block linears of the 30-block stack, in execution order.
DIT_BLOCK_LINEARS = (
    ("qkv", HIDDEN, 3 * HIDDEN),
    ("out", HIDDEN, HIDDEN),
    ("w1", HIDDEN, FFN),
    ("w3", HIDDEN, FFN),
    ("w2", FFN, HIDDEN),
)
DIT_BLOCKS = 30


# The 30-block stack as one workload: every linear of every block, in
# execution order, at TOKENS tokens; and the same stack at 64 tokens, where
# weight streaming and launch overhead dominate.
DIT_STACK = "dit_stack_m4352_30x5"
DIT_STACKS = {DIT_STACK: TOKENS, "dit_stack_m64_30x5": 64}


def make_stack(blocks: int = DIT_BLOCKS, M: int = TOKENS, R: int = R_DEFAULT,
               x_seed_offset: int = 0):
    """Operands of the stack: a list over blocks of {linear name:
    LayerOperands}.  Each block's input is its own seeded plain N(0, 1)
    x [M, HIDDEN] (no outlier channels), shared by qkv, out, w1 and w3 (the
    attention and the norms between them are not part of the layer, so the
    blocks are independent problems of the same shapes).  The w2 operands
    carry x = None: its input is silu(y_w1) * y_w3 of the same block, formed
    from the GPU's own outputs.  Seeds: block input 4000 + 100 b + 5; linear
    i of block b: 4000 + 100 b + 10 i (`x_seed_offset` moves the inputs
    only, for independent token batches on other ranks)."""
    out = []
    for b in range(blocks):
        base = workload_seed("dit_stack", layer=b)
        gx = torch.Generator().manual_seed(base + 5 + x_seed_offset)
        xb = make_x(M, HIDDEN, gx, outliers=0)
        layers = {}
        for i, (name, K, N) in enumerate(DIT_BLOCK_LINEARS):
            g = torch.Generator().manual_seed(base + 10 * i)
            layers[name] = LayerOperands(xb if name != "w2" else None, *make_weights(K, N, R, g))
        out.append(layers)
    return out


def workload_seed(name: str, layer: int = 0) -> int:
    """Deterministic per-workload seed (stable across runs and machines)."""
    base = {
        "layer_m128_k512_n512": 0,
        "qkv_m4352_k3840_n11520": 1000,
        "ffn_w1_m4352_k3840_n10240": 2000,
        "ffn_w3_m4352_k3840_n10240": 2001,
        "ffn_w2_m4352_k10240_n3840": 2002,
    }.get(name)
    if base is None and name.startswith("out_m"):
        base = 3000 + OUT_PROJ_SWEEP_M.index(int(name.split("_")[1][1:]))
    if base is None and name.startswith("dit_"):
        base = 4000
    if base is None and name.startswith(PLAIN_PREFIX):
        base = 5000
    if base is None:
        raise KeyError(name)
    return base + 100 * layer


def bits(t: torch.Tensor):
    """Raw bit patterns of a CPU tensor as a NumPy array (for the oracle).

    bf16 -> uint16, uint8 stays uint8.  Pure reinterpretation, no rounding.
    """
    import numpy as np
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype in (torch.uint8, torch.int8):
        return t.view(torch.uint8).numpy()
    raise TypeError(f"unexpected dtype {t.dtype}")
