// kr_scales.cuh -- scale-factor tile order, and two small elementwise
// kernels (scale unpack for tests, SiLU * mul for the feed-forward block).
//
// Tile order of the activation scales: rows are cut into tiles of 128, K
// into blocks of 64 (4 scales of 16).  Each (row tile t, K block b) pair is
// one 512-byte block at offset (t * (K/64) + b) * 512, holding scale
// (row, 4 b + j) at byte (row % 32) * 16 + ((row % 128) / 32) * 4 + j.
// That is the layout tcgen05.cp (32x128b, warpx4) turns into the TMEM
// scale-factor layout of tcgen05.mma kind::mxf4nvf4: TMEM lane row % 32 (in
// every lane quarter), column (row % 128) / 32, byte j.
// The weight scales use the same 512-byte blocks, ordered for 256-row GEMM
// tiles: block ((T * (K/64) + b) * 2 + h) holds rows 256 T + 128 h + [0, 128)
// of K block b, so one tile's scales over a run of K are contiguous.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace svdq {
namespace kr {

__device__ __forceinline__ size_t tiled_offset(int row, int kg, int kblocks) {
  const int t = row >> 7, b = kg >> 2, j = kg & 3;
  return (static_cast<size_t>(t) * kblocks + b) * 512 + (row & 31) * 16 + ((row & 127) >> 5) * 4 + j;
}

__device__ __forceinline__ size_t weight_tiled_offset(int row, int kg, int kblocks) {
  const int T = row >> 8, h = (row >> 7) & 1, b = kg >> 2, j = kg & 3;
  return ((static_cast<size_t>(T) * kblocks + b) * 2 + h) * 512 + (row & 31) * 16 +
         ((row & 127) >> 5) * 4 + j;
}

// Device counter of rejected scale bytes (sign bit set, or NaN 0x7F).
__device__ uint32_t g_bad_scales = 0;

// wscales [K/16, N] (N contiguous) -> weight tile order, rows padded to
// `rows_pad` (a multiple of 256) with zero scales.  One thread per output word (4 scales of one row).
__global__ void repack_weight_scales_kernel(const uint8_t* __restrict__ ws, int N, int K,
                                            int rows_pad, uint8_t* __restrict__ out) {
  const int kblocks = K / 64;
  const size_t words = static_cast<size_t>(rows_pad) * kblocks;  // 4 bytes per (row, block)
  uint32_t bad = 0;
  for (size_t w = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; w < words;
       w += static_cast<size_t>(gridDim.x) * blockDim.x) {
    // w enumerates the tiled buffer word by word: block index, then the
    // word inside the 512-byte block.
    const size_t blk = w >> 7;
    const int wi = static_cast<int>(w & 127);
    const int h = static_cast<int>(blk & 1);
    const int T = static_cast<int>((blk >> 1) / kblocks);
    const int b = static_cast<int>((blk >> 1) % kblocks);
    const int row = T * 256 + h * 128 + ((wi & 3) << 5) + (wi >> 2);
    uint32_t word = 0;
    if (row < N) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t v = ws[static_cast<size_t>(4 * b + j) * N + row];
        if ((v & 0x80u) || v == 0x7Fu) ++bad;
        word |= v << (8 * j);
      }
    }
    reinterpret_cast<uint32_t*>(out)[w] = word;
  }
  if (bad) atomicAdd(&g_bad_scales, bad);
}

// tiled (activation or weight order) -> [rows, K/16] (row-major), the
// logical scale matrix.
__global__ void unpack_scales_kernel(const uint8_t* __restrict__ tiled, int rows, int K,
                                     int weight_order, uint8_t* __restrict__ out) {
  const int kg_n = K / 16;
  const size_t total = static_cast<size_t>(rows) * kg_n;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int row = static_cast<int>(i / kg_n);
    const int kg = static_cast<int>(i % kg_n);
    out[i] = tiled[weight_order ? weight_tiled_offset(row, kg, K / 64)
                                : tiled_offset(row, kg, K / 64)];
  }
}

// proj_up_folded[n, r] = bf16(proj_up[n, r] / (wtscale * wcscales[n])): the
// up-projection in the units of the block-scaled product, so that
//   (acc + L proj_up_folded^T) * wtscale * wcscales[n] + bias
// is the layer's acc * wtscale * wcscales[n] + L proj_up^T + bias up to the
// bf16 rounding of the folded factor (the float32 quotient, correctly
// rounded, then rounded to nearest-even bf16).  An element that cannot be
// folded without losing its precision -- a zero or non-finite scale, a
// quotient that is infinite or below the smallest normal bf16 (and not zero)
// -- is counted in *unfoldable.  One thread per 8 elements.
__global__ void fold_proj_up_kernel(const __nv_bfloat16* __restrict__ proj_up,
                                    const __nv_bfloat16* __restrict__ wcscales,
                                    const __nv_bfloat16* __restrict__ wtscale, int N, int R,
                                    __nv_bfloat16* __restrict__ out,
                                    uint32_t* __restrict__ unfoldable) {
  const float alpha = __bfloat162float(wtscale[0]);
  const size_t total = static_cast<size_t>(N) * R / 8;
  uint32_t bad = 0;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int n = static_cast<int>(i * 8 / R);
    const float scale = __fmul_rn(alpha, __bfloat162float(wcscales[n]));
    const bool scale_ok = scale != 0.0f && isfinite(scale);
    const uint4 v = reinterpret_cast<const uint4*>(proj_up)[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float q0 = __fdiv_rn(__uint_as_float(w[j] << 16), scale);
      const float q1 = __fdiv_rn(__uint_as_float(w[j] & 0xFFFF0000u), scale);
      const __nv_bfloat162 r = __floats2bfloat162_rn(q0, q1);
      o[j] = *reinterpret_cast<const uint32_t*>(&r);
      const float f0 = __low2float(r), f1 = __high2float(r);
      bad += !scale_ok || !isfinite(f0) || (f0 != 0.0f && fabsf(f0) < 1.17549435e-38f);
      bad += !scale_ok || !isfinite(f1) || (f1 != 0.0f && fabsf(f1) < 1.17549435e-38f);
    }
    reinterpret_cast<uint4*>(out)[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (bad) atomicAdd(unfoldable, bad);
}

// out = silu(a) * b = a / (1 + exp(-a)) * b rounded once to bf16
// (silu_mul_words: fp32 with an fp64 path near bf16 rounding boundaries).
__global__ void silu_mul_kernel(const __nv_bfloat16* __restrict__ a,
                                const __nv_bfloat16* __restrict__ b,
                                __nv_bfloat16* __restrict__ out, size_t n) {
  const size_t nvec = n / 8;
  const uint4* a4 = reinterpret_cast<const uint4*>(a);
  const uint4* b4 = reinterpret_cast<const uint4*>(b);
  uint4* o4 = reinterpret_cast<uint4*>(out);
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < nvec;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint4 ua = __ldg(a4 + i), ub = __ldg(b4 + i);
    const uint32_t wa[4] = {ua.x, ua.y, ua.z, ua.w};
    const uint32_t wb[4] = {ub.x, ub.y, ub.z, ub.w};
    uint32_t wo[4];
    silu_mul_words<4>(wa, wb, wo);
    o4[i] = make_uint4(wo[0], wo[1], wo[2], wo[3]);
  }
  // tail
  const size_t tail0 = nvec * 8;
  const size_t tid = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  if (tail0 + tid < n) {
    const float av = __bfloat162float(a[tail0 + tid]);
    const float bv = __bfloat162float(b[tail0 + tid]);
    out[tail0 + tid] = __ushort_as_bfloat16(static_cast<unsigned short>(silu_mul_bf16_rn(av, bv)));
  }
}

}  // namespace kr
}  // namespace svdq
