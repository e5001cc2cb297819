// kq_quantize_act.cuh -- activation side of the SVDQuant W4A4 layer for
// sm_100a: reads x once and writes quant(x * smooth) (NVFP4) and the
// low-rank product L = x @ proj_down (nunchaku-z-image-turbo-svdq model
// card, "What's stored on disk", runtime formula).
//
// Quantization of each 16-element group along K (one e4m3 scale per 16 k,
// E2M1 elements, as the card's first paragraph states; rounding to
// nearest-even with saturation):
//   v = x * smooth                  exact in fp32 (bf16 x bf16)
//   s = e4m3(amax|v| / 6)           fp32 division (correctly rounded), then
//                                   the hardware RNE/satfinite conversion
//   q = E2M1(v / s)                 quotient by reciprocal + one FMA
//                                   residual correction, then the hardware
//                                   RNE/satfinite conversion
// Both roundings equal exact rational rounding: a bf16 x bf16 product has
// at most 16 significant bits, every e4m3 midpoint x 6 and every E2M1
// midpoint x s has at most 7, so a quotient that is not exactly on a
// midpoint lies at least 2^-16 (relative) away from it, far more than the
// fp32 error; a quotient exactly on a midpoint is representable, and the
// residual step (r = RN(1/s), q0 = RN(v r), e = v - q0 s exact by FMA,
// q = RN(q0 + e r); Markstein, IBM J. Res. Dev. 34(1), 1990) returns it
// exactly, so the conversion sees the tie.
//
// Layout of one CTA (128 rows x a K range, 10 warps):
//   warp 0      TMA producer: x tile [128 rows x 64 k] bf16 (128-byte
//               swizzle) and proj_down rows [64 k x 128 r] (two 64-column
//               boxes) into a 4-stage ring.
//   warp 1      TMEM owner, MMA issuer: L[128 x 128] += x_tile x pd_chunk
//               with tcgen05.mma kind::f16 (M=128, N=128, K=16), A K-major,
//               B MN-major, fp32 accumulator in 128 TMEM columns.
//   warps 2..9  quantize the same shared-memory x tile (2 groups per
//               thread per stage), write packed codes and tiled scales;
//               afterwards read L out of TMEM.
// The K range is split over a thread-block cluster of `split` CTAs; the
// partial L tiles are summed through distributed shared memory in rank
// order (deterministic) and written once as bf16.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace svdq {
namespace kq {

constexpr int BM = 128;               // rows per CTA
constexpr int BKE = 64;               // k per stage
constexpr int R = 128;                // rank (MMA N)
constexpr int STAGES = 4;
constexpr uint32_t X_BYTES = BM * BKE * 2;         // 16 KB
constexpr uint32_t PD_BYTES = BKE * R * 2;         // 16 KB
constexpr uint32_t PD_HALF = PD_BYTES / 2;         // one 64-column box
constexpr uint32_t STAGE_BYTES = X_BYTES + PD_BYTES;
constexpr int NUM_QWARPS = 8;
constexpr int NUM_QTHREADS = NUM_QWARPS * 32;      // 256
constexpr int NUM_THREADS = 64 + NUM_QTHREADS;     // 320
constexpr uint32_t BAR_BYTES = 128;
constexpr uint32_t SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
constexpr uint32_t TMEM_COLS = 128;
constexpr int PART_STRIDE = 132;  // floats per row of the partial-L buffer
static_assert(BM * PART_STRIDE * 4 <= STAGES * STAGE_BYTES, "partial buffer fits the ring");

constexpr uint32_t SITE_PROD = 0x20, SITE_MMA = 0x21, SITE_QUANT = 0x22, SITE_LFULL = 0x23;

struct Params {
  const __nv_bfloat16* smooth;
  uint8_t* qact;
  uint8_t* ascales_tiled;
  __nv_bfloat16* lowrank;
  int M, K;
  int chunks;  // K / 64
  int split;   // CTAs per cluster along K
};

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Quantize one 16-element group: v[16] (x * smooth, exact) -> 16 E2M1
// codes (64 bits, element 0 in the lowest nibble) and the e4m3 scale byte.
__device__ __forceinline__ uint64_t quantize_group(const float (&v)[16], uint32_t& scale_byte) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t sc = cvt_e4m3x2(__fdiv_rn(amax, 6.0f), 0.0f) & 0xFFu;
  scale_byte = sc;
  const float d = e4m3_to_f32(sc);
  if (d == 0.0f) {
    // Every element rounds to zero; keep each element's sign.
    uint64_t codes = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i)
      codes |= static_cast<uint64_t>(__float_as_uint(v[i]) >> 31) << (4 * i + 3);
    return codes;
  }
  const float r = __frcp_rn(d);
  float lo[8], hi[8];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float q0 = v[i] * r;
    const float e = fmaf(-q0, d, v[i]);
    float q = fmaf(e, r, q0);
    // The correction turns a quotient of -0 into +0: restore v's sign.
    q = __uint_as_float((__float_as_uint(q) & 0x7FFFFFFFu) | (__float_as_uint(v[i]) & 0x80000000u));
    if (i < 8) lo[i] = q; else hi[i - 8] = q;
  }
  return static_cast<uint64_t>(cvt_e2m1x8(lo)) | (static_cast<uint64_t>(cvt_e2m1x8(hi)) << 32);
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
quantize_act_kernel(const __grid_constant__ CUtensorMap tm_x,    // x [M, ldx] bf16
                    const __grid_constant__ CUtensorMap tm_pd,   // proj_down [K, 128] bf16
                    const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t s_ring = smem_u32(smem);
  const uint32_t s_bar = s_ring + STAGES * STAGE_BYTES;
  auto s_x = [&](uint32_t s) { return s_ring + s * STAGE_BYTES; };
  auto s_pd = [&](uint32_t s) { return s_ring + s * STAGE_BYTES + X_BYTES; };
  auto full_bar = [&](uint32_t s) { return s_bar + 8u * s; };
  auto empty_bar = [&](uint32_t s) { return s_bar + 8u * (STAGES + s); };
  const uint32_t lfull_bar = s_bar + 16u * STAGES;
  const uint32_t final_bar = lfull_bar + 8u;
  const uint32_t tmem_slot = lfull_bar + 16u;
  uint32_t* tmem_slot_ptr = reinterpret_cast<uint32_t*>(smem + (tmem_slot - s_ring));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int mb = blockIdx.y;
  const int rank = blockIdx.x;  // == rank in the cluster (cluster dims = (split, 1, 1))
  const int c_begin = rank * p.chunks / p.split;
  const int c_end = (rank + 1) * p.chunks / p.split;
  const int nchunks = c_end - c_begin;  // >= 1 (host guarantees split <= chunks)

  if (threadIdx.x == 0) {
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_pd);
    for (uint32_t s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1 + NUM_QWARPS);
    }
    mbar_init(lfull_bar, 1);
    mbar_init(final_bar, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(tmem_slot_ptr);

  bool l_ready = false;  // quantizer threads: L accumulator readable

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ producer --
      int i = 0;
      bool ok = true;
      for (; i < nchunks; ++i) {
        const uint32_t s = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1u;
        if (!svdq_wait(empty_bar(s), ph ^ 1u, SITE_PROD)) {
          ok = false;
          break;
        }
        const int kc = c_begin + i;
        mbar_arrive_expect_tx(full_bar(s), STAGE_BYTES);
        tma_load_2d(s_x(s), &tm_x, kc * BKE, mb * BM, full_bar(s));
        tma_load_2d(s_pd(s), &tm_pd, 0, kc * BKE, full_bar(s));
        tma_load_2d(s_pd(s) + PD_HALF, &tm_pd, 64, kc * BKE, full_bar(s));
      }
      if (!ok) {
        const int n = i < STAGES ? i : STAGES;
        for (int j = 0; j < n; ++j) {
          const int jt = i - 1 - j;
          drain_wait(full_bar(jt % STAGES), (jt / STAGES) & 1u, 50000000ull);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------- MMA issuer --
      const uint32_t idesc = idesc_bf16_f32(BM, R, 0, 1);
      bool ok = true;
      for (int i = 0; i < nchunks; ++i) {
        const uint32_t s = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1u;
        if (!svdq_wait(full_bar(s), ph, SITE_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BKE / 16; ++kk) {
          // A: 16 k of the x tile = 32 bytes along the swizzled row.
          // B: 16 k rows of proj_down = 2 swizzle atoms of 8 rows (1 KB
          //    each); the two 64-column halves are 8 KB apart.
          mma_f16(tmem_base, smem_desc(s_x(s) + 32 * kk, 16, 1024, kLayoutSwizzle128B),
                  smem_desc(s_pd(s) + 2048 * kk, PD_HALF, 1024, kLayoutSwizzle128B), idesc,
                  (i | kk) != 0 ? 1u : 0u);
        }
        tc_commit(empty_bar(s));
      }
      if (ok) tc_commit(lfull_bar);
      tc_commit(final_bar);
      drain_wait(final_bar, 0, 100000000ull);
    }
  } else {
    // -------------------------------------------------------- quantizers --
    const int qt = threadIdx.x - 64;
    const int half_k = p.K / 2;
    bool ok = true;
    for (int i = 0; i < nchunks; ++i) {
      const uint32_t s = i % STAGES;
      const uint32_t ph = (i / STAGES) & 1u;
      if (!__all_sync(0xFFFFFFFFu, svdq_wait(full_bar(s), ph, SITE_QUANT))) {
        ok = false;
        break;
      }
      const int kc = c_begin + i;
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
        const int gi = pass * NUM_QTHREADS + qt;
        const int r = gi >> 2;  // row in the tile
        const int g = gi & 3;   // group of 16 within the 64-wide chunk
        const uint32_t row_addr = s_x(s) + r * 128;
        const uint4 xa = ld_shared_v4(row_addr + (((2 * g) ^ (r & 7)) << 4));
        const uint4 xb = ld_shared_v4(row_addr + (((2 * g + 1) ^ (r & 7)) << 4));
        const uint4* sp = reinterpret_cast<const uint4*>(p.smooth + kc * BKE + g * 16);
        const uint4 sa = __ldg(sp);
        const uint4 sb = __ldg(sp + 1);
        float xv[16], sv[16], v[16];
        bf16x8_to_f32(xa, xv);
        bf16x8_to_f32(xb, xv + 8);
        bf16x8_to_f32(sa, sv);
        bf16x8_to_f32(sb, sv + 8);
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = xv[e] * sv[e];
        uint32_t scale;
        const uint64_t codes = quantize_group(v, scale);
        const int row = mb * BM + r;
        if (row < p.M) {
          uint2* dst = reinterpret_cast<uint2*>(p.qact + static_cast<size_t>(row) * half_k +
                                                kc * (BKE / 2) + g * 8);
          *dst = make_uint2(static_cast<uint32_t>(codes), static_cast<uint32_t>(codes >> 32));
        }
        // Tiled scales: 512-byte block per (128 rows, 4 groups); byte
        // (r % 32) * 16 + (r / 32) * 4 + g.  Lanes 4i..4i+3 hold one row.
        uint32_t w = scale << (8 * g);
        w |= __shfl_xor_sync(0xFFFFFFFFu, w, 1);
        w |= __shfl_xor_sync(0xFFFFFFFFu, w, 2);
        if (g == 0) {
          uint32_t* sdst = reinterpret_cast<uint32_t*>(
              p.ascales_tiled + (static_cast<size_t>(mb) * p.chunks + kc) * 512 + (r & 31) * 16 +
              (r >> 5) * 4);
          *sdst = w;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_bar(s));
    }
    if (ok) l_ready = __all_sync(0xFFFFFFFFu, svdq_wait(lfull_bar, 0, SITE_LFULL));
  }

  // --------------------------------------------------- low-rank readout --
  // Quantizer warp w reads TMEM lane quarter (w % 4), columns [64 h, 64 h + 64).
  const bool is_q = warp >= 2;
  const int lq = warp & 3;
  const int hcol = (warp - 2) >> 2;
  const int r_out = lq * 32 + lane;
  const int row_out = mb * BM + r_out;
  if (p.split == 1) {
    if (is_q && l_ready) {
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t acc[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(lq * 32) << 16) + 64 * hcol + 32 * c,
                           acc);
        tmem_ld_wait();
        if (row_out < p.M) {
          uint4* dst = reinterpret_cast<uint4*>(p.lowrank + static_cast<size_t>(row_out) * R +
                                                64 * hcol + 32 * c);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(acc[8 * v + 2 * i]),
                                                        __uint_as_float(acc[8 * v + 2 * i + 1]));
              w[i] = *reinterpret_cast<uint32_t*>(&b2);
            }
            dst[v] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    }
  } else {
    // Partial sums: every quantizer warp has finished with the ring before
    // any of them overwrites it with its fp32 partial L rows.
    if (is_q) {
      named_bar_sync(1, NUM_QTHREADS);
      if (l_ready) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t acc[32];
          tmem_ld_32x32b_x32(
              tmem_base + (static_cast<uint32_t>(lq * 32) << 16) + 64 * hcol + 32 * c, acc);
          tmem_ld_wait();
          const uint32_t base = s_ring + (r_out * PART_STRIDE + 64 * hcol + 32 * c) * 4;
#pragma unroll
          for (int v = 0; v < 8; ++v)
            st_shared_v4(base + 16 * v, __uint_as_float(acc[4 * v]),
                         __uint_as_float(acc[4 * v + 1]), __uint_as_float(acc[4 * v + 2]),
                         __uint_as_float(acc[4 * v + 3]));
        }
      }
    }
    __syncwarp();
    cluster_sync_all();
    if (is_q && !error_raised()) {
      const int rows_per = BM / p.split;
      const int row0 = rank * rows_per;
      for (int idx = threadIdx.x - 64; idx < rows_per * (R / 4); idx += NUM_QTHREADS) {
        const int rr = row0 + idx / (R / 4);
        const int c4 = idx % (R / 4);
        const uint32_t off = s_ring + (rr * PART_STRIDE + 4 * c4) * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int src = 0; src < p.split; ++src) {
          const float4 t = ld_dsmem_f4(map_to_rank(off, src));
          acc.x += t.x;
          acc.y += t.y;
          acc.z += t.z;
          acc.w += t.w;
        }
        const int row = mb * BM + rr;
        if (row < p.M) {
          __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
          __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
          uint2* dst = reinterpret_cast<uint2*>(p.lowrank + static_cast<size_t>(row) * R + 4 * c4);
          *dst = make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
        }
      }
    }
    __syncwarp();
    cluster_sync_all();
  }

  // ----------------------------------------------------------- teardown --
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace kq
}  // namespace svdq
