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
//   warp 0      operand producer (one thread).  A ring of AB_SLOTS slots; a
//               slot holds one K step of 256: the qact box (128 rows x 128 B,
//               128-byte swizzle) and the qweight box (256 rows x 128 B).
//               After the K steps of a tile two more slots carry the
//               low-rank operands, one 64-wide half of R each (L half in the
//               A place, proj_up half in the B place).
//   warp 1      TMEM owner and MMA issuer (one thread):
//               tcgen05.mma kind::mxf4nvf4 block16 (M=128, N=256, K=64) into
//               the main accumulator, then tcgen05.mma kind::f16 (bf16,
//               K=16) for L @ proj_up^T into a second accumulator.
//   warp 2      scale loader (one thread): a deeper ring of SF_SLOTS slots,
//               each one K step's A and B scale blocks (two contiguous bulk
//               copies, 6 KB), paired with SF_SLOTS TMEM slots; a slot is
//               reloaded as soon as the MMAs that used it have completed.
//   warps 3..10 scale writers during the K loop, epilogue after it (two
//               warps per TMEM lane quarter).
//               Scale writing: the MMA reads each 512-byte scale block
//               replicated in all four lane quarters (lane r % 32 of every
//               quarter, column (r % 128) / 32).  Each warp reads its half
//               of a loaded slot from shared memory (16 B per lane per
//               block) and writes it to its quarter's lanes with
//               tcgen05.st, several steps ahead of the MMAs.  Measured on
//               B200, register stores from eight warps slow the
//               concurrently running MMAs far less than tcgen05.cp copies
//               of the same bytes.
//               Epilogue (one warp per quarter and half of the 256
//               columns): stage the tile's wcscales / bias in
//               shared memory while the MMAs run, then TMEM -> registers
//               (tcgen05.ld), fp32 acc * wtscale * wcscales + lowrank + bias,
//               packed to bf16.  TMEM is released to the next tile right
//               after the reads; the bf16 rows then go through a per-warp
//               swizzled shared-memory buffer to TMA tensor stores, which
//               write whole rows asynchronously and clip the M / N edges.
// TMEM map (512 columns, fp32): main accumulator [0, 256), low-rank
// accumulator [256, 512); the scale-factor slots live in [256, 496) while
// the main K loop runs (the low-rank MMAs start only after every main MMA
// has completed, and no scale copy of the next tile starts before the
// epilogue has read this one).
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
constexpr int AB_SLOTS = 3;
constexpr int SF_SLOTS = 5;
constexpr uint32_t A_BYTES = BM * BK_BYTES;          // 16 KB
constexpr uint32_t B_BYTES = BN * BK_BYTES;          // 32 KB
constexpr uint32_t AB_SLOT_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t SFA_BYTES = 4 * 512;              // 128 rows x 16 scales
constexpr uint32_t SFB_BYTES = 2 * 4 * 512;          // 256 rows x 16 scales
constexpr uint32_t SF_SLOT_BYTES = SFA_BYTES + SFB_BYTES;
constexpr uint32_t LR_A_BYTES = BM * 64 * 2;         // L half: 128 rows x 64 bf16
constexpr uint32_t LR_B_BYTES = BN * 64 * 2;         // proj_up half: 256 rows x 64 bf16
static_assert(LR_A_BYTES <= A_BYTES && LR_B_BYTES <= B_BYTES, "low-rank halves fit a slot");
constexpr uint32_t AB_RING_BYTES = AB_SLOTS * AB_SLOT_BYTES;
constexpr uint32_t SF_RING_BYTES = SF_SLOTS * SF_SLOT_BYTES;
constexpr int NUM_EPI_WARPS = 8;
constexpr int OUT_COLS = 64;                         // columns per TMA store box
constexpr uint32_t OUT_WARP_BYTES = 32 * OUT_COLS * 2;   // 32 rows x 128 B
constexpr uint32_t OUT_BYTES = NUM_EPI_WARPS * OUT_WARP_BYTES;
constexpr uint32_t COLV_BYTES = 2 * 2 * BN * 4;      // wcscales, bias (fp32), 2 tile buffers
constexpr uint32_t BAR_BYTES = 256;
constexpr uint32_t SMEM_BYTES =
    AB_RING_BYTES + SF_RING_BYTES + OUT_BYTES + COLV_BYTES + BAR_BYTES + 1024;
constexpr int EPI_WARP0 = 3;
constexpr int NUM_THREADS = 32 * EPI_WARP0 + 32 * NUM_EPI_WARPS;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_ACC = 0;
constexpr uint32_t TM_LR = 256;
constexpr uint32_t TM_SF = 256;                      // per slot: 16 SFA + 32 SFB columns
constexpr uint32_t TM_SF_SLOT = 48;
static_assert(TM_SF + SF_SLOTS * TM_SF_SLOT <= TMEM_COLS, "scale columns fit");
static_assert(AB_SLOT_BYTES % 1024 == 0 && (AB_RING_BYTES + SF_RING_BYTES) % 1024 == 0,
              "operand slots and the output buffers stay 1024-aligned");

// Wait-site ids recorded in the error word.
constexpr uint32_t SITE_PROD = 0x10, SITE_MMA_TE = 0x11, SITE_MMA_FULL = 0x12,
                   SITE_MMA_DRAIN = 0x13, SITE_EPI = 0x14, SITE_MMA_SF = 0x15,
                   SITE_SF_LOADED = 0x17, SITE_SF_EMPTY = 0x18, SITE_LOAD_EMPTY = 0x19,
                   SITE_EPI_TE = 0x1A;

struct Params {
  const uint8_t* ascales_tiled;
  const uint8_t* wscales_tiled;
  const __nv_bfloat16* wcscales;
  const __nv_bfloat16* wtscale;
  const __nv_bfloat16* bias;  // may be null
  int M, N, K;
  int m_tiles, n_tiles;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// LR: the layer has the low-rank branch (R = 128).  Without it (R = 0, the
// plain NVFP4 layer) a tile has no low-rank slots, drain or MMAs and the
// epilogue reads only the main accumulator.
template <bool LR>
__global__ void __launch_bounds__(NUM_THREADS, 1)
w4a4_linear_kernel(const __grid_constant__ CUtensorMap tm_a,   // qact    [M, K/2] u8, box {128, 128}
                   const __grid_constant__ CUtensorMap tm_b,   // qweight [N, K/2] u8, box {128, 256}
                   const __grid_constant__ CUtensorMap tm_l,   // lowrank [M, 128] bf16, box {64, 128}
                   const __grid_constant__ CUtensorMap tm_p,   // proj_up [N, 128] bf16, box {64, 256}
                   const __grid_constant__ CUtensorMap tm_y,   // y [M, ldy] bf16, box {64, 32}
                   const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t s_ring = smem_u32(smem);
  auto s_a = [&](uint32_t s) { return s_ring + s * AB_SLOT_BYTES; };
  auto s_b = [&](uint32_t s) { return s_ring + s * AB_SLOT_BYTES + A_BYTES; };
  const uint32_t s_sfring = s_ring + AB_RING_BYTES;
  auto s_sfa = [&](uint32_t s) { return s_sfring + s * SF_SLOT_BYTES; };
  auto s_sfb = [&](uint32_t s) { return s_sfring + s * SF_SLOT_BYTES + SFA_BYTES; };
  const uint32_t s_out = s_sfring + SF_RING_BYTES;
  const uint32_t s_colv = s_out + OUT_BYTES;
  const uint32_t s_bar = s_colv + COLV_BYTES;
  // barriers: operand ring full / empty, scale ring loaded / full / empty
  auto full_bar = [&](uint32_t s) { return s_bar + 8u * s; };
  auto empty_bar = [&](uint32_t s) { return s_bar + 8u * (AB_SLOTS + s); };
  auto sf_loaded_bar = [&](uint32_t s) { return s_bar + 8u * (2 * AB_SLOTS + s); };
  auto sf_full_bar = [&](uint32_t s) { return s_bar + 8u * (2 * AB_SLOTS + SF_SLOTS + s); };
  auto sf_empty_bar = [&](uint32_t s) {
    return s_bar + 8u * (2 * AB_SLOTS + 2 * SF_SLOTS + s);
  };
  const uint32_t tmem_full_bar = s_bar + 8u * (2 * AB_SLOTS + 3 * SF_SLOTS);
  const uint32_t tmem_empty_bar = tmem_full_bar + 8u;
  const uint32_t drain_bar = tmem_full_bar + 16u;
  const uint32_t final_bar = tmem_full_bar + 24u;
  const uint32_t tmem_slot = tmem_full_bar + 32u;
  static_assert(8 * (2 * AB_SLOTS + 3 * SF_SLOTS) + 48 <= BAR_BYTES, "barriers fit");
  uint32_t* tmem_slot_ptr = reinterpret_cast<uint32_t*>(smem + (tmem_slot - s_ring));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    if (LR) {
      prefetch_tmap(&tm_l);
      prefetch_tmap(&tm_p);
    }
    prefetch_tmap(&tm_y);
    for (uint32_t s = 0; s < AB_SLOTS; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (uint32_t s = 0; s < SF_SLOTS; ++s) {
      mbar_init(sf_loaded_bar(s), 1);
      mbar_init(sf_full_bar(s), NUM_EPI_WARPS);
      mbar_init(sf_empty_bar(s), 1);
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

  const int num_k = p.K / BK;                  // K steps per tile
  const int tiles = p.m_tiles * p.n_tiles;
  const size_t kblocks = static_cast<size_t>(p.K / 64);   // 512-byte scale blocks per 128 rows
  // The qweight boxes of the first tile's first AB_SLOTS K steps are
  // requested before the wait for the previous kernel, so that the weight
  // stream overlaps it.
  const int t0 = static_cast<int>(blockIdx.x);
  const int pre = t0 < tiles ? (num_k < AB_SLOTS ? num_k : AB_SLOTS) : 0;
  if (warp == 0 && lane == 0) {
    for (int st = 0; st < pre; ++st) {
      const uint32_t s = static_cast<uint32_t>(st);
      mbar_expect_tx(full_bar(s), B_BYTES);
      tma_load_2d(s_b(s), &tm_b, st * BK_BYTES, (t0 / p.m_tiles) * BN, full_bar(s));
    }
  }
  // Set-up above overlaps the previous kernel; what it writes waits for it.
  griddep_wait();
  griddep_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ producer --
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        const int mb = t % p.m_tiles;
        const int nb = t / p.m_tiles;
        for (int st = 0; st < num_k + (LR ? 2 : 0); ++st, ++it) {
          const uint32_t s = it % AB_SLOTS;
          const uint32_t ph = (it / AB_SLOTS) & 1u;
          if (!svdq_wait(empty_bar(s), ph ^ 1u, SITE_PROD)) {
            ok = false;
            break;
          }
          if (st < num_k) {
            const bool weights_in = static_cast<int>(it) < pre;   // requested before the wait
            mbar_arrive_expect_tx(full_bar(s), weights_in ? A_BYTES : AB_SLOT_BYTES);
            tma_load_2d(s_a(s), &tm_a, st * BK_BYTES, mb * BM, full_bar(s));
            if (!weights_in) tma_load_2d(s_b(s), &tm_b, st * BK_BYTES, nb * BN, full_bar(s));
          } else {
            const int hr = st - num_k;           // which 64-wide half of R
            mbar_arrive_expect_tx(full_bar(s), LR_A_BYTES + LR_B_BYTES);
            tma_load_2d(s_a(s), &tm_l, hr * 64, mb * BM, full_bar(s));
            tma_load_2d(s_b(s), &tm_p, hr * 64, nb * BN, full_bar(s));
          }
        }
      }
      if (!ok) {
        // Let the copies already issued land before the block exits.
        const uint32_t n = it < AB_SLOTS ? it : AB_SLOTS;
        for (uint32_t j = 0; j < n; ++j) {
          const uint32_t jt = it - 1 - j;
          drain_wait(full_bar(jt % AB_SLOTS), (jt / AB_SLOTS) & 1u, 50000000ull);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------- MMA issuer --
      const uint32_t idesc_main = idesc_nvfp4(BM, BN);
      const uint32_t idesc_lr = idesc_bf16_f32(BM, BN, 0, 0);
      uint32_t it = 0, ik = 0, tc = 0;   // operand ring uses, K steps, tiles
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++tc) {
        if (!svdq_wait(tmem_empty_bar, (tc & 1u) ^ 1u, SITE_MMA_TE)) break;
        tc_fence_after();
        for (int st = 0; st < num_k; ++st, ++it, ++ik) {
          const uint32_t s = it % AB_SLOTS;
          const uint32_t ph = (it / AB_SLOTS) & 1u;
          const uint32_t sf = ik % SF_SLOTS;
          if (!svdq_wait(full_bar(s), ph, SITE_MMA_FULL) ||
              !svdq_wait(sf_full_bar(sf), (ik / SF_SLOTS) & 1u, SITE_MMA_SF)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfa_t = tmem_base + TM_SF + TM_SF_SLOT * sf;
          const uint32_t sfb_t = sfa_t + 16;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            mma_nvfp4(tmem_base + TM_ACC,
                      smem_desc(s_a(s) + 32 * j, 16, 1024, kLayoutSwizzle128B),
                      smem_desc(s_b(s) + 32 * j, 16, 1024, kLayoutSwizzle128B), idesc_main,
                      sfa_t + 4 * j, sfb_t + 8 * j, (st | j) != 0 ? 1u : 0u);
          }
          tc_commit(empty_bar(s));
          tc_commit(sf_empty_bar(sf));
        }
        if (!ok) break;
        if (!LR) {
          tc_commit(tmem_full_bar);
          continue;
        }
        // The low-rank accumulator overlaps the scale-factor columns: let
        // every main MMA finish before the low-rank MMAs write there.
        tc_commit(drain_bar);
        if (!svdq_wait(drain_bar, tc & 1u, SITE_MMA_DRAIN)) break;
        tc_fence_after();
        for (int hr = 0; hr < 2 && ok; ++hr, ++it) {
          const uint32_t s = it % AB_SLOTS;
          const uint32_t ph = (it / AB_SLOTS) & 1u;
          if (!svdq_wait(full_bar(s), ph, SITE_MMA_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16(tmem_base + TM_LR,
                    smem_desc(s_a(s) + 32 * kk, 16, 1024, kLayoutSwizzle128B),
                    smem_desc(s_b(s) + 32 * kk, 16, 1024, kLayoutSwizzle128B), idesc_lr,
                    (hr | kk) != 0 ? 1u : 0u);
          tc_commit(empty_bar(s));
        }
        if (!ok) break;
        tc_commit(tmem_full_bar);
      }
      // Every MMA this thread issued completes before TMEM is released.
      tc_commit(final_bar);
      drain_wait(final_bar, 0, 100000000ull);
    }
  } else if (warp == 2) {
    if (lane == 0) {
      // -------------------------------------------------- scale loader --
      // K steps of this CTA, in order over its tiles: step i belongs to the
      // tile blockIdx.x + (i / num_k) * gridDim.x, K step i % num_k.
      // Slot i % SF_SLOTS is free once the MMAs of step i - SF_SLOTS (which
      // read its TMEM columns, written from its shared memory) completed.
      const int my_tiles =
          static_cast<int>(blockIdx.x) < tiles ? (tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
      const uint32_t total = static_cast<uint32_t>(my_tiles) * num_k;
      uint32_t i = 0;
      bool ok = true;
      for (; i < total; ++i) {
        const uint32_t s = i % SF_SLOTS;
        const uint32_t ph = (i / SF_SLOTS) & 1u;
        if (i >= SF_SLOTS && !svdq_wait(sf_empty_bar(s), ph ^ 1u, SITE_LOAD_EMPTY)) {
          ok = false;
          break;
        }
        const int t = blockIdx.x + static_cast<int>(i / num_k) * gridDim.x;
        const int st = static_cast<int>(i % num_k);
        const int mb = t % p.m_tiles;
        const int nb = t / p.m_tiles;
        mbar_arrive_expect_tx(sf_loaded_bar(s), SF_SLOT_BYTES);
        bulk_load(s_sfa(s), p.ascales_tiled + (static_cast<size_t>(mb) * kblocks + 4 * st) * 512,
                  SFA_BYTES, sf_loaded_bar(s));
        bulk_load(s_sfb(s),
                  p.wscales_tiled + (static_cast<size_t>(nb) * kblocks + 4 * st) * 1024,
                  SFB_BYTES, sf_loaded_bar(s));
      }
      if (!ok) {
        // Let the scale loads already issued land before the block exits.
        for (uint32_t j = i > SF_SLOTS ? i - SF_SLOTS : 0; j < i; ++j)
          drain_wait(sf_loaded_bar(j % SF_SLOTS), (j / SF_SLOTS) & 1u, 50000000ull);
      }
    }
  } else {
    // -------------------------------------------------------- epilogue --
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int half = (warp - EPI_WARP0) >> 2;     // which 128 of the tile's 256 columns
    const int et = threadIdx.x - 32 * EPI_WARP0;  // 0..255
    const float alpha = __bfloat162float(p.wtscale[0]);
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t s_obuf = s_out + static_cast<uint32_t>(warp - EPI_WARP0) * OUT_WARP_BYTES;
    float* colv = reinterpret_cast<float*>(smem + (s_colv - s_ring));
    uint32_t tc = 0, i = 0;
    bool ok = true;
    // Scale factors of the next n K steps -> TMEM, up to SF_SLOTS steps
    // ahead of the MMAs.  This warp writes blocks 6 * half .. 6 * half + 5
    // of each slot (TMEM columns 4 b .. 4 b + 3 for block b) in its lane
    // quarter.  A tile's steps are written only after every epilogue warp
    // has read the previous tile's low-rank accumulator, which these
    // columns overlap.
    auto write_scales = [&](uint32_t n) {
      for (uint32_t e = i + n; i < e; ++i) {
        const uint32_t s = i % SF_SLOTS;
        const uint32_t ph = (i / SF_SLOTS) & 1u;
        if (ok)
          ok = __all_sync(0xFFFFFFFFu,
                          svdq_wait(sf_loaded_bar(s), ph, SITE_SF_LOADED) &&
                              (i < SF_SLOTS || svdq_wait(sf_empty_bar(s), ph ^ 1u, SITE_SF_EMPTY)));
        if (!ok) continue;
        tc_fence_after();
        const uint32_t src = s_sfa(s) + 16 * lane;
        const uint32_t dst = lane_base + TM_SF + TM_SF_SLOT * s;
#pragma unroll
        for (int k = 0; k < 3; ++k) {
          const int b0 = 6 * half + 2 * k;
          uint32_t v[8];
          ld_shared_v4(src + 512 * b0, v[0], v[1], v[2], v[3]);
          ld_shared_v4(src + 512 * (b0 + 1), v[4], v[5], v[6], v[7]);
          tmem_st_32x32b_x8(dst + 4 * b0, v);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sf_full_bar(s));
      }
    };
    // A tile's first SF_SLOTS steps are written right after the previous
    // tile's TMEM reads, before its output stores, and MID more between the
    // two output pieces, so the MMAs restart soon and do not wait for the
    // stores.
    constexpr uint32_t MID = 2;
    const uint32_t head = num_k < SF_SLOTS ? static_cast<uint32_t>(num_k) : SF_SLOTS;
    const uint32_t mid = num_k - head < MID ? num_k - head : MID;
    if (static_cast<int>(blockIdx.x) < tiles) write_scales(head + mid);
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++tc) {
      const int mb = t % p.m_tiles;
      const int nb = t / p.m_tiles;
      const bool has_next = t + static_cast<int>(gridDim.x) < tiles;
      write_scales(num_k - head - mid);
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
      // Every epilogue warp passes this barrier once per tile, also after a
      // failed wait, so that no warp is left waiting on it.
      named_bar_sync(2, 32 * NUM_EPI_WARPS);
      if (ok) ok = __all_sync(0xFFFFFFFFu, svdq_wait(tmem_full_bar, tc & 1u, SITE_EPI));
      if (!ok) continue;
      tc_fence_after();
      uint32_t out[8][8];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int col = half * 128 + 16 * c;
        uint32_t acc[16], lr[16];
        tmem_ld_32x32b_x16(lane_base + TM_ACC + col, acc);
        if (LR) {
          tmem_ld_32x32b_x16(lane_base + TM_LR + col, lr);
        } else {
#pragma unroll
          for (int z = 0; z < 16; ++z) lr[z] = 0u;   // +0.0f
        }
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float2 w2 = *reinterpret_cast<const float2*>(wc_s + col + 2 * i);
          const float2 b2 = *reinterpret_cast<const float2*>(bs_s + col + 2 * i);
          const float o0 = fmaf(__uint_as_float(acc[2 * i]), w2.x,
                                __uint_as_float(lr[2 * i]) + b2.x);
          const float o1 = fmaf(__uint_as_float(acc[2 * i + 1]), w2.y,
                                __uint_as_float(lr[2 * i + 1]) + b2.y);
          out[c][i] = pack_bf16x2(o0, o1);
        }
      }
      // TMEM is free for the next tile as soon as every warp has its values.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tmem_empty_bar);
      if (has_next) {
        // The other warp of this lane quarter may still be reading low-rank
        // columns that the next scale slots overlap: wait for all readers.
        ok = __all_sync(0xFFFFFFFFu, svdq_wait(tmem_empty_bar, tc & 1u, SITE_EPI_TE));
        write_scales(head);
      }
      // Rows -> swizzled buffer (row = lane, 128 B per row; 16-byte chunk
      // j of row r at chunk j ^ (r % 8), the TMA 128-byte swizzle) -> TMA
      // store of 32 rows x 64 columns, twice per tile.
      const int row0 = mb * BM + q * 32;
#pragma unroll
      for (int pc = 0; pc < 2; ++pc) {
        if (lane == 0) bulk_wait_group_read0();   // previous store has read the buffer
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int c = 4 * pc + (j >> 1);
          const int v = j & 1;
          st_shared_v4(s_obuf + lane * 128 + ((j ^ (lane & 7)) << 4), out[c][4 * v],
                       out[c][4 * v + 1], out[c][4 * v + 2], out[c][4 * v + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        const int x0 = nb * BN + half * 128 + pc * OUT_COLS;
        if (lane == 0 && x0 < p.N && row0 < p.M) {
          tma_store_2d(&tm_y, s_obuf, x0, row0);
          bulk_commit_group();
        }
        if (pc == 0 && has_next) write_scales(mid);
      }
    }
    if (lane == 0) bulk_wait_group0();
  }

  // ----------------------------------------------------------- teardown --
  // Role loops run in one lane of some warps: reconverge every warp first,
  // so that the block barrier waits for all of its threads.
  __syncwarp();
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
