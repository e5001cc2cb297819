// kg_w4a4_linear.cuh -- block-scaled NVFP4 GEMM with the fused SVDQuant
// epilogue, for sm_100a.
//
// Computes (nunchaku-z-image-turbo-svdq model card, "What's stored on
// disk", runtime formula)
//   y[m, n] = acc[m, n] * wtscale * wcscales[n] + (L @ proj_up^T)[m, n] + bias[n]
//   acc[m, n] = sum_k e2m1(qa[m,k]) sa[m,k/16] e2m1(qw[n,k]) sw[k/16,n]
// with L = x @ proj_down from the activation kernel, stored bf16.
//
// Design (one CTA per SM, persistent over 128 x 256 output tiles):
//   warp 0      TMA producer: per K step of 256 it loads the A tile
//               (qact, 128 rows x 128 B), the B tile (qweight, 256 rows x
//               128 B), both 128-byte swizzled, and the matching scale
//               blocks (bulk copies of the tiled scale buffers) into a
//               4-stage shared-memory ring; after the K loop it loads the
//               low-rank operands (L and proj_up, two K halves of 64)
//               through the same ring.
//   warp 1      TMEM owner and MMA issuer (one thread): copies the scale
//               blocks smem -> TMEM (tcgen05.cp), issues
//               tcgen05.mma kind::mxf4nvf4 block16 (M=128, N=256, K=64)
//               into the main accumulator, then tcgen05.mma kind::f16
//               (bf16, K=16) for L @ proj_up^T into a second accumulator.
//   warps 2..9  epilogue (two warps per TMEM lane quarter, one per half
//               of the 256 columns): stage the tile's wcscales / bias in
//               shared memory while the MMAs run, then TMEM -> registers
//               (tcgen05.ld), fp32 acc * wtscale * wcscales + lowrank + bias,
//               packed to bf16 in registers; TMEM is released before the
//               global stores, so the stores overlap the next tile's MMAs.
// TMEM map (512 columns, fp32): main accumulator [0, 256), low-rank
// accumulator [256, 512); the per-step scale factors live in [256, 304)
// while the main K loop runs (the low-rank MMAs start only after every main
// MMA has completed).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace svdq {
namespace kg {

constexpr int BM = 128;          // output rows per tile (MMA M)
constexpr int BN = 256;          // output columns per tile (MMA N)
constexpr int BK_BYTES = 128;    // K step: 256 FP4 values = 128 bytes per row
constexpr int BK = 256;
constexpr int STAGES = 4;
constexpr uint32_t A_BYTES = BM * BK_BYTES;          // 16 KB
constexpr uint32_t B_BYTES = BN * BK_BYTES;          // 32 KB
constexpr uint32_t SFA_BYTES = 4 * 512;              // 128 rows x 16 scales
constexpr uint32_t SFB_BYTES = 2 * 4 * 512;          // 256 rows x 16 scales
constexpr uint32_t LR_A_BYTES = BM * 128;            // 128 rows x 64 bf16
constexpr uint32_t LR_B_BYTES = BN * 128;            // 256 rows x 64 bf16
constexpr uint32_t STAGE_TX = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr uint32_t LR_TX = LR_A_BYTES + LR_B_BYTES;
constexpr uint32_t RING_BYTES = STAGES * (A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES);
constexpr uint32_t BAR_BYTES = 128;
constexpr uint32_t COLV_BYTES = 2 * 2 * BN * 4;      // wcscales, bias (fp32), 2 tile buffers
constexpr uint32_t SMEM_BYTES = RING_BYTES + COLV_BYTES + BAR_BYTES + 1024;  // + alignment
constexpr int NUM_EPI_WARPS = 8;
constexpr int NUM_THREADS = 64 + 32 * NUM_EPI_WARPS;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_ACC = 0;
constexpr uint32_t TM_LR = 256;
constexpr uint32_t TM_SFA = 256;
constexpr uint32_t TM_SFB = 272;

// Wait-site ids recorded in the error word.
constexpr uint32_t SITE_PROD = 0x10, SITE_MMA_TE = 0x11, SITE_MMA_FULL = 0x12,
                   SITE_MMA_DRAIN = 0x13, SITE_EPI = 0x14;

struct Params {
  const uint8_t* ascales_tiled;
  const uint8_t* wscales_tiled;
  const __nv_bfloat16* wcscales;
  const __nv_bfloat16* wtscale;
  const __nv_bfloat16* bias;  // may be null
  __nv_bfloat16* y;
  int M, N, K, ldy;
  int m_tiles, n_tiles;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void unpack_bf16x8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
w4a4_linear_kernel(const __grid_constant__ CUtensorMap tm_a,   // qact   [M, K/2] u8
                   const __grid_constant__ CUtensorMap tm_b,   // qweight[N, K/2] u8
                   const __grid_constant__ CUtensorMap tm_l,   // lowrank[M, 128] bf16
                   const __grid_constant__ CUtensorMap tm_p,   // proj_up[N, 128] bf16
                   const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t s_a = smem_u32(smem);
  const uint32_t s_b = s_a + STAGES * A_BYTES;
  const uint32_t s_sfa = s_b + STAGES * B_BYTES;
  const uint32_t s_sfb = s_sfa + STAGES * SFA_BYTES;
  const uint32_t s_colv = s_sfb + STAGES * SFB_BYTES;
  const uint32_t s_bar = s_colv + COLV_BYTES;
  auto full_bar = [&](uint32_t s) { return s_bar + 8u * s; };
  auto empty_bar = [&](uint32_t s) { return s_bar + 8u * (STAGES + s); };
  const uint32_t tmem_full_bar = s_bar + 16u * STAGES;
  const uint32_t tmem_empty_bar = tmem_full_bar + 8u;
  const uint32_t drain_bar = tmem_full_bar + 16u;
  const uint32_t final_bar = tmem_full_bar + 24u;
  const uint32_t tmem_slot = tmem_full_bar + 32u;
  uint32_t* tmem_slot_ptr = reinterpret_cast<uint32_t*>(smem + (tmem_slot - s_a));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_l);
    prefetch_tmap(&tm_p);
    for (uint32_t s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(tmem_full_bar, 1);
    mbar_init(tmem_empty_bar, NUM_EPI_WARPS);
    mbar_init(drain_bar, 1);
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

  const int num_k = p.K / BK;
  const int tiles = p.m_tiles * p.n_tiles;
  const size_t ka_per_rowtile = static_cast<size_t>(p.K / 64);

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ producer --
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        const int mb = t % p.m_tiles;
        const int nb = t / p.m_tiles;
        for (int kb = 0; kb < num_k + 2; ++kb, ++it) {
          const uint32_t s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!svdq_wait(empty_bar(s), ph ^ 1u, SITE_PROD)) {
            ok = false;
            break;
          }
          if (kb < num_k) {
            mbar_arrive_expect_tx(full_bar(s), STAGE_TX);
            tma_load_2d(s_a + s * A_BYTES, &tm_a, kb * BK_BYTES, mb * BM, full_bar(s));
            tma_load_2d(s_b + s * B_BYTES, &tm_b, kb * BK_BYTES, nb * BN, full_bar(s));
            const uint8_t* sfa_src =
                p.ascales_tiled + (static_cast<size_t>(mb) * ka_per_rowtile + kb * 4) * 512;
            const uint8_t* sfb_src0 =
                p.wscales_tiled + (static_cast<size_t>(2 * nb) * ka_per_rowtile + kb * 4) * 512;
            const uint8_t* sfb_src1 =
                p.wscales_tiled + (static_cast<size_t>(2 * nb + 1) * ka_per_rowtile + kb * 4) * 512;
            bulk_load(s_sfa + s * SFA_BYTES, sfa_src, SFA_BYTES, full_bar(s));
            bulk_load(s_sfb + s * SFB_BYTES, sfb_src0, SFB_BYTES / 2, full_bar(s));
            bulk_load(s_sfb + s * SFB_BYTES + SFB_BYTES / 2, sfb_src1, SFB_BYTES / 2, full_bar(s));
          } else {
            const int j = kb - num_k;  // low-rank K half: r in [64 j, 64 j + 64)
            mbar_arrive_expect_tx(full_bar(s), LR_TX);
            tma_load_2d(s_a + s * A_BYTES, &tm_l, j * 64, mb * BM, full_bar(s));
            tma_load_2d(s_b + s * B_BYTES, &tm_p, j * 64, nb * BN, full_bar(s));
          }
        }
      }
      if (!ok) {
        // Let the copies already issued land before the block exits.
        const uint32_t n = it < STAGES ? it : STAGES;
        for (uint32_t j = 0; j < n; ++j) {
          const uint32_t jt = it - 1 - j;
          drain_wait(full_bar(jt % STAGES), (jt / STAGES) & 1u, 50000000ull);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------- MMA issuer --
      const uint32_t idesc_main = idesc_nvfp4(BM, BN);
      const uint32_t idesc_lr = idesc_bf16_f32(BM, BN, 0, 0);
      uint32_t it = 0, tc = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++tc) {
        if (!svdq_wait(tmem_empty_bar, (tc & 1u) ^ 1u, SITE_MMA_TE)) break;
        tc_fence_after();
        for (int kb = 0; kb < num_k; ++kb, ++it) {
          const uint32_t s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!svdq_wait(full_bar(s), ph, SITE_MMA_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = s_a + s * A_BYTES;
          const uint32_t b0 = s_b + s * B_BYTES;
          const uint32_t sfa0 = s_sfa + s * SFA_BYTES;
          const uint32_t sfb0 = s_sfb + s * SFB_BYTES;
#pragma unroll
          for (int j = 0; j < 4; ++j)
            tmem_cp_32x128b_warpx4(tmem_base + TM_SFA + 4 * j,
                                   smem_desc(sfa0 + 512 * j, 0, 128, kLayoutSwizzleNone));
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tmem_cp_32x128b_warpx4(
                  tmem_base + TM_SFB + 8 * j + 4 * h,
                  smem_desc(sfb0 + (SFB_BYTES / 2) * h + 512 * j, 0, 128, kLayoutSwizzleNone));
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            mma_nvfp4(tmem_base + TM_ACC, smem_desc(a0 + 32 * j, 16, 1024, kLayoutSwizzle128B),
                      smem_desc(b0 + 32 * j, 16, 1024, kLayoutSwizzle128B), idesc_main,
                      tmem_base + TM_SFA + 4 * j, tmem_base + TM_SFB + 8 * j,
                      (kb | j) != 0 ? 1u : 0u);
          }
          tc_commit(empty_bar(s));
        }
        if (!ok) break;
        // The low-rank accumulator overlaps the scale-factor columns: let
        // every main MMA finish before the low-rank MMAs write there.
        tc_commit(drain_bar);
        if (!svdq_wait(drain_bar, tc & 1u, SITE_MMA_DRAIN)) break;
        tc_fence_after();
        for (int j = 0; j < 2; ++j, ++it) {
          const uint32_t s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!svdq_wait(full_bar(s), ph, SITE_MMA_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = s_a + s * A_BYTES;
          const uint32_t b0 = s_b + s * B_BYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            mma_f16(tmem_base + TM_LR, smem_desc(a0 + 32 * kk, 16, 1024, kLayoutSwizzle128B),
                    smem_desc(b0 + 32 * kk, 16, 1024, kLayoutSwizzle128B), idesc_lr,
                    (j | kk) != 0 ? 1u : 0u);
          }
          tc_commit(empty_bar(s));
        }
        if (!ok) break;
        tc_commit(tmem_full_bar);
      }
      // Every MMA this thread issued completes before TMEM is released.
      tc_commit(final_bar);
      drain_wait(final_bar, 0, 100000000ull);
    }
  } else {
    // -------------------------------------------------------- epilogue --
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;    // which 128 of the tile's 256 columns
    const int et = threadIdx.x - 64;     // 0..255
    const float alpha = __bfloat162float(p.wtscale[0]);
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    float* colv = reinterpret_cast<float*>(smem + (s_colv - s_a));
    uint32_t tc = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++tc) {
      const int mb = t % p.m_tiles;
      const int nb = t / p.m_tiles;
      // Per-column factors of this tile -> shared memory (double buffered by
      // tile parity), loaded while the tile's MMAs are still running.
      float* wc_s = colv + (tc & 1u) * (2 * BN);
      float* bs_s = wc_s + BN;
      {
        const int n = nb * BN + et;
        float wcv = 0.f, bsv = 0.f;
        if (n < p.N) {
          wcv = __bfloat162float(p.wcscales[n]);
          if (p.bias != nullptr) bsv = __bfloat162float(p.bias[n]);
        }
        wc_s[et] = wcv * alpha;
        bs_s[et] = bsv;
      }
      named_bar_sync(2, 32 * NUM_EPI_WARPS);
      if (!__all_sync(0xFFFFFFFFu, svdq_wait(tmem_full_bar, tc & 1u, SITE_EPI))) break;
      tc_fence_after();
      const int row = mb * BM + q * 32 + lane;
      uint32_t out[4][16];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int col = half * 128 + 16 * c;
        uint32_t acc[16], lr[16];
        tmem_ld_32x32b_x16(lane_base + TM_ACC + col, acc);
        tmem_ld_32x32b_x16(lane_base + TM_LR + col, lr);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float2 w2 = *reinterpret_cast<const float2*>(wc_s + col + 2 * i);
          const float2 b2 = *reinterpret_cast<const float2*>(bs_s + col + 2 * i);
          const float o0 = fmaf(__uint_as_float(acc[2 * i]), w2.x,
                                __uint_as_float(lr[2 * i]) + b2.x);
          const float o1 = fmaf(__uint_as_float(acc[2 * i + 1]), w2.y,
                                __uint_as_float(lr[2 * i + 1]) + b2.y);
          out[c >> 1][8 * (c & 1) + i] = pack_bf16x2(o0, o1);
        }
      }
      // TMEM is free for the next tile as soon as every warp has its values.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tmem_empty_bar);
      if (row < p.M) {
        __nv_bfloat16* yrow = p.y + static_cast<size_t>(row) * p.ldy;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int n0 = nb * BN + half * 128 + 32 * c;
          if (n0 < p.N) {
            uint4* dst = reinterpret_cast<uint4*>(yrow + n0);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(out[c][4 * v], out[c][4 * v + 1], out[c][4 * v + 2],
                                  out[c][4 * v + 3]);
          }
        }
      }
    }
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

}  // namespace kg
}  // namespace svdq
