"""CPU oracle for the SVDQuant W4A4 NVFP4 linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this
package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It
shares no code with the CUDA library (no kernels, headers, tables or
helpers); the only thing both sides consume is the seeded input generator,
which holds none of the method's arithmetic.

What it computes, and from which passage:

* The runtime formula of the "nunchaku-z-image-turbo-svdq" model card,
  section "What's stored on disk":
  ``y = scaled_mma(quant(x * smooth), qweight, ascales, wscales)
  * wtscale * wcscales + (x @ proj_down) @ proj_up^T + bias``.
* The operand layouts of the same section's table (qweight [N, K/2] FP4
  nibbles with the low nibble holding the even k, wscales [K/16, N]
  float8_e4m3fn, and so on) and the format line of its first paragraph
  (E2M1 elements with one e4m3 scale per 16 elements along K, R = 128).
* The E2M1 bit layout (1 sign, 2 exponent, 1 mantissa bit) of the
  Z-Image NVFP4 blog, section "NVFP4 技术背景 / 什么是 NVFP4？".
* The offline weight side (``weight_quant``): a bf16 weight and smoothing
  factor to the stored operands through a rank-R SVD of the smoothed weight
  and an NVFP4 residual -- the card's "via SVDQuant ... with rank-128 SVD
  residual"; how the operands are derived is not on the pages, so each step
  there is a reading stated in that module.
* The input of the w2 feed-forward linear, silu(w1 x) * (w3 x), for the
  feed-forward linears w1, w2, w3 the same blog names in "Z-Image NVFP4
  模型变体" (``silu_mul``; the gated form is the reading taken).

Everything is decoded to float64 and multiplied with plain NumPy.  Each
function is pinned by ``tests/test_oracle_pins.py`` against closed forms,
hand-worked blocks (``tests/golden/``), an exact rational brute force and
library codecs; there is no function here marked "parity unpinned".
"""

from .nvfp4 import (  # noqa: F401
    E2M1_MAGNITUDES,
    bf16_bits_to_f64,
    f64_to_bf16_bits_rne,
    decode_e2m1,
    decode_e4m3,
    encode_e2m1_rne_sat,
    encode_e4m3_rne_satfinite,
    pack_nibbles,
    unpack_nibbles,
)
from . import weight_quant  # noqa: F401
from .svdq_ref import (  # noqa: F401
    quantize_act,
    lowrank_down,
    dequant_act,
    dequant_weight,
    w4a4_linear,
    svdq_linear_from_x,
    plain_linear_from_x,
    silu_mul,
)
