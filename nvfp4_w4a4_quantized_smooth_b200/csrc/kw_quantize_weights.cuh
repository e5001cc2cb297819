// kw_quantize_weights.cuh -- offline (load-time) weight side of the
// SVDQuant W4A4 layer: the NVFP4 encoding of the residual a bf16 weight
// leaves after its low-rank part.
//
// The "nunchaku-z-image-turbo-svdq" model card stores the layer "via
// SVDQuant ... in NVFP4 ... with rank-128 SVD residual" (first paragraph)
// as the operands of its "What's stored on disk" table; how they are
// derived from a trained weight is not on the pages.  The reading
// implemented here (the low-rank factors come from an SVD of the smoothed
// weight, done with library linear algebra by the caller):
//   res[n, k]  = (W[n, k] - lowrank[n, k]) / smooth[k]
//   A          = max |res|,  a_n = max_k |res[n, k]|
//   wtscale    = bf16(A / (6 * 448))            (bf16 1 if A == 0)
//   wcscales[n]= bf16(a_n / A)                  (0 if A == 0)
//   d_n        = wtscale * wcscales[n]          (exact in fp32)
//   per 16 k:  s = e4m3(a_g / (6 d_n)), S = e4m3value(s) * d_n (exact),
//              code = E2M1(res / S), signed zero codes where S == 0.
// Every float operation is correctly rounded float32 in that order
// (IEEE intrinsics, no contraction), and the float results are encoded
// with the hardware's nearest-even, saturating conversions, so that the
// integer results are a function of the float32 inputs alone.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace svdq {
namespace kw {

constexpr float kSixE4M3Max = 2688.0f;   // 6 * 448

__device__ __forceinline__ float residual_at(const __nv_bfloat16* __restrict__ W,
                                             const float* __restrict__ lowrank,
                                             const __nv_bfloat16* __restrict__ smooth, size_t idx,
                                             int k) {
  const float w = __bfloat162float(W[idx]);
  const float diff = lowrank != nullptr ? __fsub_rn(w, lowrank[idx]) : w;
  return __fdiv_rn(diff, __bfloat162float(smooth[k]));
}

// ws[n] = max_k |res[n, k]| (one block per row); ws[N] = max over all rows,
// as the bit pattern of a non-negative float (ordered like the value), which
// the caller zeroes first.
__global__ void __launch_bounds__(256) weight_residual_amax_kernel(
    const __nv_bfloat16* __restrict__ W, const float* __restrict__ lowrank,
    const __nv_bfloat16* __restrict__ smooth, int N, int K, float* __restrict__ ws) {
  __shared__ float red[8];
  for (int n = blockIdx.x; n < N; n += gridDim.x) {
    float m = 0.0f;
    const size_t row = static_cast<size_t>(n) * K;
    for (int k = threadIdx.x; k < K; k += blockDim.x)
      m = fmaxf(m, fabsf(residual_at(W, lowrank, smooth, row + k, k)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
      float r = red[0];
      for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) r = fmaxf(r, red[w]);
      ws[n] = r;
      atomicMax(reinterpret_cast<unsigned int*>(ws + N), __float_as_uint(r));
    }
    __syncthreads();
  }
}

// One thread per 16-element group of a row: the scales and codes.
__global__ void __launch_bounds__(256) weight_quantize_kernel(
    const __nv_bfloat16* __restrict__ W, const float* __restrict__ lowrank,
    const __nv_bfloat16* __restrict__ smooth, int N, int K, const float* __restrict__ ws,
    uint8_t* __restrict__ qweight, uint8_t* __restrict__ wscales,
    __nv_bfloat16* __restrict__ wcscales, __nv_bfloat16* __restrict__ wtscale) {
  const int G = K / 16;
  const size_t total = static_cast<size_t>(N) * G;
  const float A = __uint_as_float(*reinterpret_cast<const unsigned int*>(ws + N));
  const __nv_bfloat16 alpha_b =
      A > 0.0f ? __float2bfloat16_rn(__fdiv_rn(A, kSixE4M3Max)) : __float2bfloat16_rn(1.0f);
  const float alpha = __bfloat162float(alpha_b);
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    // consecutive threads take consecutive rows of one group column, so
    // that the [K/16, N] scale stores are contiguous
    const int n = static_cast<int>(i % N);
    const int g = static_cast<int>(i / N);
    const __nv_bfloat16 c_b = A > 0.0f ? __float2bfloat16_rn(__fdiv_rn(ws[n], A))
                                       : __float2bfloat16_rn(0.0f);
    const float d = __fmul_rn(alpha, __bfloat162float(c_b));
    const float six_d = __fmul_rn(6.0f, d);
    const size_t base = static_cast<size_t>(n) * K + 16 * g;
    float r[16];
    float ag = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      r[j] = residual_at(W, lowrank, smooth, base + j, 16 * g + j);
      ag = fmaxf(ag, fabsf(r[j]));
    }
    const float t = six_d > 0.0f ? __fdiv_rn(ag, six_d) : 0.0f;
    const uint32_t s = cvt_e4m3x2(t, 0.0f) & 0xFFu;
    const float S = __fmul_rn(e4m3_to_f32(s), d);
    float q[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) q[j] = S > 0.0f ? __fdiv_rn(r[j], S) : 0.0f * r[j];
    const float(&qlo)[8] = *reinterpret_cast<const float(*)[8]>(q);
    const float(&qhi)[8] = *reinterpret_cast<const float(*)[8]>(q + 8);
    *reinterpret_cast<uint2*>(qweight + static_cast<size_t>(n) * (K / 2) + 8 * g) =
        make_uint2(cvt_e2m1x8(qlo), cvt_e2m1x8(qhi));
    wscales[static_cast<size_t>(g) * N + n] = static_cast<uint8_t>(s);
    if (g == 0) wcscales[n] = c_b;
    if (i == 0) wtscale[0] = alpha_b;
  }
}

}  // namespace kw
}  // namespace svdq
