// kg2_w4a4_linear_pair.cuh -- the block-scaled NVFP4 GEMM with the fused
// SVDQuant epilogue on CTA pairs (tcgen05 cta_group::2), for sm_100a.
//
// Same computation as kg_w4a4_linear.cuh (nunchaku-z-image-turbo-svdq model
// card, "What's stored on disk", runtime formula):
//   y[m, n] = acc[m, n] * wtscale * wcscales[n] + (L @ proj_up^T)[m, n] + bias[n]
//   acc[m, n] = sum_k e2m1(qa[m,k]) sa[m,k/16] e2m1(qw[n,k]) sw[k/16,n]
// but each 256 x 256 output tile is computed by a cluster of two CTAs on two
// SMs: the even CTA issues one MMA per 64 k for the pair (M = 256: rows
// [0, 128) of the tile come from its A and land in its TMEM, rows [128, 256)
// from the odd CTA's), and each CTA loads only its own 128 A rows and 128 of
// the tile's 256 B rows.  Per SM and K step of 256 that is 32 KB of operands
// for 128 x 256 x 256 multiply-adds, against 48 KB for the single-SM
// 128 x 256 tile: the L2 -> shared-memory stream per SM, which bounds the
// single-SM kernel's K step, drops by a third, and the same ring holds more
// K steps in flight.
//
// Roles per CTA (both CTAs run all roles; only the even CTA issues MMAs):
//   warps 0, 10 producers (one thread each, taking the stage uses in
//               turn).  A ring of STAGES stages; a stage holds one K step:
//               this CTA's A rows (qact, 128 x 128 B) and
//               B rows (qweight, 128 x 128 B) -- their TMA completions go
//               to the even CTA's full barrier -- and the K step's scale
//               blocks: this CTA's 128 A rows (2 KB) and all 256 B rows of
//               the tile (4 KB: every CTA's TMEM needs all of the tile's B
//               scales), bulk copies completing on this CTA's sf_loaded
//               barrier.  Two more stage uses per tile carry the low-rank
//               operands (a 64-wide half of R each: this CTA's L rows in
//               the A place, its proj_up rows in the B place), after the K
//               steps (LR_SEPARATE) or before them (LR_FOLDED).
//   warp 1      TMEM (512 columns, allocated for the pair); in the even CTA
//               the MMA issuer: tcgen05.mma cta_group::2 kind::mxf4nvf4
//               block16 (M = N = 256, K = 64, four per K step) into the main
//               accumulator, and kind::f16 (K = 16) for the low-rank
//               product; its commits reach both CTAs.
//   warps 2..9  scale writers during the K loop and epilogue after it, in
//               each CTA on its own TMEM (two warps per lane quarter):
//               each stage's 12 scale blocks are written into that stage's
//               TMEM scale slot with tcgen05.st (every block replicated in
//               the four lane quarters, as the block-scaled MMA reads them),
//               and each of the 16 warps of the pair arrives on the even
//               CTA's full barrier of the stage.  Epilogue: TMEM -> registers, TMEM released (to
//               the even CTA), fp32 acc * wtscale * wcscales (+ low-rank
//               accumulator) + bias, bf16, rows through a swizzled per-warp
//               shared-memory buffer to TMA tensor stores.
// The low-rank branch takes one of two forms (template argument LRM):
//   LR_SEPARATE  the formula's order: L @ proj_up^T in a second accumulator,
//                added in the epilogue.  TMEM (each CTA, 512 fp32 columns):
//                main accumulator [0, 256), low-rank accumulator [256, 512);
//                the STAGES scale slots (48 columns each) live in
//                [256, 496) during the K loop, so a tile's low-rank MMAs
//                wait for its main MMAs (drain), and the next tile's first
//                scale slots are written only after every epilogue warp of
//                the CTA has read the low-rank accumulator.
//   LR_FOLDED    proj_up_folded = bf16(proj_up / (wtscale * wcscales[n]))
//                (prepared once per weight): the low-rank product is then in
//                the units of the block-scaled one, and the two low-rank
//                stage uses come first in the tile's K loop, into the main
//                accumulator:  y = (acc + L proj_up_folded^T) * wtscale *
//                wcscales[n] + bias.  TMEM: accumulator [0, 256), scale slots
//                [256, 496) -- disjoint, so the scale writes run ahead of the
//                epilogue, which reads the accumulator once and releases it
//                before its arithmetic.
//   LR_NONE      (R = 0) the folded form's schedule without low-rank uses.
// In every form stage use u writes slot u % STAGES only after the MMAs of
// use u - STAGES completed (the producer reloads the stage's scale bytes
// only then).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace svdq {
namespace kg2 {

constexpr int BM = 256;          // output rows per pair tile (MMA M)
constexpr int BM_CTA = 128;      // rows per CTA
constexpr int BN = 256;          // output columns per tile (MMA N)
constexpr int BN_CTA = 128;      // B rows each CTA loads
constexpr int BK_BYTES = 128;    // K step: 256 FP4 values = 128 bytes per row
constexpr int BK = 256;
constexpr int STAGES = 5;
constexpr uint32_t A_BYTES = BM_CTA * BK_BYTES;      // 16 KB
constexpr uint32_t B_BYTES = BN_CTA * BK_BYTES;      // 16 KB
constexpr uint32_t SFA_BYTES = 4 * 512;              // 128 rows x 16 scales
constexpr uint32_t SFB_BYTES = 2 * 4 * 512;          // 256 rows x 16 scales
constexpr uint32_t SF_BYTES = SFA_BYTES + SFB_BYTES;
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES + SF_BYTES;   // 38 KB
constexpr uint32_t LR_A_BYTES = BM_CTA * 64 * 2;     // L half: 128 rows x 64 bf16
constexpr uint32_t LR_B_BYTES = BN_CTA * 64 * 2;     // proj_up half: 128 rows x 64 bf16
static_assert(LR_A_BYTES <= A_BYTES && LR_B_BYTES <= B_BYTES, "low-rank halves fit a stage");
constexpr uint32_t RING_BYTES = STAGES * STAGE_BYTES;
constexpr int NUM_EPI_WARPS = 8;
constexpr int EPI_WARP0 = 2;
constexpr int PROD1_WARP = EPI_WARP0 + NUM_EPI_WARPS;   // the second producer
constexpr int NUM_THREADS = 32 * (PROD1_WARP + 1);
constexpr int OUT_COLS = 64;                         // columns per TMA store box
constexpr uint32_t OUT_WARP_BYTES = 32 * OUT_COLS * 2;   // 32 rows x 128 B
constexpr uint32_t OUT_BYTES = NUM_EPI_WARPS * OUT_WARP_BYTES;
constexpr uint32_t COLV_BYTES = 2 * BN * 4;          // wcscales * wtscale, bias (fp32)
constexpr uint32_t BAR_BYTES = 256;
constexpr uint32_t SMEM_BYTES = RING_BYTES + OUT_BYTES + COLV_BYTES + BAR_BYTES + 1024;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_ACC = 0;
constexpr uint32_t TM_LR = 256;
constexpr uint32_t TM_SF = 256;                      // per slot: 16 SFA + 32 SFB columns
constexpr uint32_t TM_SF_SLOT = 48;
static_assert(TM_SF + STAGES * TM_SF_SLOT <= TMEM_COLS, "scale columns fit");
static_assert(STAGE_BYTES % 1024 == 0 && RING_BYTES % 1024 == 0,
              "stages and the output buffers stay 1024-aligned");
static_assert(SMEM_BYTES <= 232448, "fits the shared memory of one SM");

// Wait-site ids recorded in the error word.
constexpr uint32_t SITE_PROD = 0x40, SITE_MMA_TE = 0x41, SITE_MMA_FULL = 0x42,
                   SITE_MMA_SF = 0x43, SITE_MMA_DRAIN = 0x44, SITE_SF_LOADED = 0x45,
                   SITE_EPI = 0x46;

struct Params {
  const uint8_t* ascales_tiled;
  const uint8_t* wscales_tiled;
  const __nv_bfloat16* wcscales;
  const __nv_bfloat16* wtscale;
  const __nv_bfloat16* bias;  // may be null
  int M, N, K;
  int m_tiles, n_tiles;       // 256 x 256 pair tiles
  int a_row_tiles;            // 128-row blocks of the activation scales, ceil(M / 128)
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Low-rank forms (see the file comment).
constexpr int LR_NONE = 0, LR_SEPARATE = 1, LR_FOLDED = 2;

template <int LRM>
__global__ void __launch_bounds__(NUM_THREADS, 1)
w4a4_linear_pair_kernel(const __grid_constant__ CUtensorMap tm_a,   // qact    [M, K/2] u8, box {128, 128}
                        const __grid_constant__ CUtensorMap tm_b,   // qweight [N, K/2] u8, box {128, 128}
                        const __grid_constant__ CUtensorMap tm_l,   // lowrank [M, 128] bf16, box {64, 128}
                        const __grid_constant__ CUtensorMap tm_p,   // proj_up [N, 128] bf16, box {64, 128}
                        const __grid_constant__ CUtensorMap tm_y,   // y [M, ldy] bf16, box {64, 32}
                        const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t s_ring = smem_u32(smem);
  auto s_a = [&](uint32_t s) { return s_ring + s * STAGE_BYTES; };
  auto s_b = [&](uint32_t s) { return s_ring + s * STAGE_BYTES + A_BYTES; };
  auto s_sf = [&](uint32_t s) { return s_ring + s * STAGE_BYTES + A_BYTES + B_BYTES; };
  const uint32_t s_out = s_ring + RING_BYTES;
  const uint32_t s_colv = s_out + OUT_BYTES;
  const uint32_t s_bar = s_colv + COLV_BYTES;
  // Per stage: full (even CTA: both CTAs' operand bytes landed and all 16
  // writer warps of the pair wrote the stage's scales into TMEM -- one
  // barrier, so that the MMA thread waits once per stage use), empty (this
  // CTA: the stage's MMAs completed), sf_loaded (this CTA: its scale bytes
  // landed).
  auto full_bar = [&](uint32_t s) { return s_bar + 8u * s; };
  auto empty_bar = [&](uint32_t s) { return s_bar + 8u * (STAGES + s); };
  auto sfl_bar = [&](uint32_t s) { return s_bar + 8u * (2 * STAGES + s); };
  const uint32_t tmem_full_bar = s_bar + 8u * (4 * STAGES);
  const uint32_t tmem_empty_bar = tmem_full_bar + 8u;   // even CTA: 16 epilogue warps
  const uint32_t drain_bar = tmem_full_bar + 16u;
  const uint32_t final_bar = tmem_full_bar + 24u;
  const uint32_t tmem_slot = tmem_full_bar + 32u;
  static_assert(8 * (4 * STAGES) + 40 <= BAR_BYTES, "barriers fit");
  uint32_t* tmem_slot_ptr = reinterpret_cast<uint32_t*>(smem + (tmem_slot - s_ring));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();     // 0: the pair's MMA issuer
  const bool leader = rank == 0;

  constexpr bool LR = LRM != LR_NONE;
  constexpr bool FOLDED = LRM == LR_FOLDED;
  if (threadIdx.x == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    if (LR) {
      prefetch_tmap(&tm_l);
      prefetch_tmap(&tm_p);
    }
    prefetch_tmap(&tm_y);
    for (uint32_t s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1 + 2 * NUM_EPI_WARPS);
      mbar_init(empty_bar(s), 1);
      mbar_init(sfl_bar(s), 1);
    }
    mbar_init(tmem_full_bar, 1);
    mbar_init(tmem_empty_bar, 2 * NUM_EPI_WARPS);
    mbar_init(drain_bar, 1);
    mbar_init(final_bar, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_cg2(tmem_slot, TMEM_COLS);
    tmem_relinquish_cg2();
  }
  // Both CTAs' barriers are initialised (and the TMEM address published)
  // before either CTA touches the other's barriers.
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(tmem_slot_ptr);

  const int num_k = p.K / BK;                  // K steps per tile
  const int uses = num_k + (LR ? 2 : 0);       // stage uses per tile
  // Position of a tile's first K step among its stage uses, and whether
  // stage use `st` of a tile carries low-rank operands.
  const int k0 = FOLDED ? 2 : 0;
  auto lr_use = [&](int st) { return FOLDED ? st < 2 : (LR && st >= num_k); };
  const int tiles = p.m_tiles * p.n_tiles;
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int npairs = static_cast<int>(gridDim.x >> 1);
  const size_t kblocks = static_cast<size_t>(p.K / 64);   // 512-byte scale blocks per 128 rows
  // The weight side of the first tile's first STAGES stage uses (this CTA's
  // qweight rows and the tile's weight scales, or its proj_up half) is
  // requested before the wait for the previous kernel, each use by the
  // producer that owns it, so that the weight stream overlaps that kernel.
  const uint32_t pre = pair < tiles ? (uses < STAGES ? static_cast<uint32_t>(uses) : STAGES) : 0u;
  if ((warp == 0 || warp == PROD1_WARP) && lane == 0) {
    const uint32_t pid = warp == 0 ? 0u : 1u;
    const int nb = pair / p.m_tiles;
    const int brow = nb * BN + static_cast<int>(rank) * BN_CTA;
    for (uint32_t u = pid; u < pre; u += 2) {
      const int st = static_cast<int>(u);
      const uint32_t fb = map_to_rank(full_bar(u), 0);
      if (!lr_use(st)) {
        const int ks = st - k0;
        if (leader) mbar_expect_tx(full_bar(u), 2 * B_BYTES);
        tma_load_2d_cg2(s_b(u), &tm_b, ks * BK_BYTES, brow, fb);
        mbar_expect_tx(sfl_bar(u), SFB_BYTES);
        bulk_load(s_sf(u) + SFA_BYTES,
                  p.wscales_tiled + (static_cast<size_t>(nb) * kblocks + 4 * ks) * 1024, SFB_BYTES,
                  sfl_bar(u));
      } else {
        const int hr = FOLDED ? st : st - num_k;
        if (leader) mbar_expect_tx(full_bar(u), 2 * LR_B_BYTES);
        tma_load_2d_cg2(s_b(u), &tm_p, hr * 64, brow, fb);
      }
    }
  }
  // Set-up above overlaps the previous kernel; what it writes waits for it.
  griddep_wait();
  griddep_launch_dependents();

  if (warp == 0 || warp == PROD1_WARP) {
    if (lane == 0) {
      // ----------------------------------------------------- producers --
      // Two producer threads in two warps take the stage uses in turn (one
      // thread's copies complete about one stage per 0.3 us whatever the
      // ring depth; two keep the SM's operand stream ahead of the MMAs).
      // Each waits on a stage's empty barrier at most one phase ahead of
      // its completion: its previous use waited for the release of the
      // use STAGES + 2 back, and 2 <= STAGES.
      static_assert(STAGES >= 2, "alternating producers need two stages");
      const uint32_t pid = warp == 0 ? 0u : 1u;
      uint32_t it = 0;
      bool ok = true;
      for (int t = pair; t < tiles && ok; t += npairs) {
        const int mb = t % p.m_tiles;
        const int nb = t / p.m_tiles;
        const int arow = mb * BM + static_cast<int>(rank) * BM_CTA;
        const int brow = nb * BN + static_cast<int>(rank) * BN_CTA;
        const int arow_tile = 2 * mb + static_cast<int>(rank);   // 128-row scale block
        // A rows wholly beyond M (odd CTA of a last, half-empty tile): the
        // operand box reads zeros; there is no scale block to copy.
        const bool a_sf = arow_tile < p.a_row_tiles;
        for (int st = 0; st < uses; ++st, ++it) {
          if ((it & 1u) != pid) continue;
          const uint32_t s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!svdq_wait(empty_bar(s), ph ^ 1u, SITE_PROD)) {
            ok = false;
            break;
          }
          const uint32_t fb = map_to_rank(full_bar(s), 0);
          const bool weights_in = it < pre;      // weight side requested before the wait
          if (!lr_use(st)) {
            const int ks = st - k0;              // K step
            if (leader)
              mbar_arrive_expect_tx(full_bar(s), 2 * (A_BYTES + (weights_in ? 0u : B_BYTES)));
            tma_load_2d_cg2(s_a(s), &tm_a, ks * BK_BYTES, arow, fb);
            if (!weights_in) tma_load_2d_cg2(s_b(s), &tm_b, ks * BK_BYTES, brow, fb);
            mbar_arrive_expect_tx(sfl_bar(s),
                                  (a_sf ? SFA_BYTES : 0u) + (weights_in ? 0u : SFB_BYTES));
            if (a_sf)
              bulk_load(s_sf(s),
                        p.ascales_tiled + (static_cast<size_t>(arow_tile) * kblocks + 4 * ks) * 512,
                        SFA_BYTES, sfl_bar(s));
            if (!weights_in)
              bulk_load(s_sf(s) + SFA_BYTES,
                        p.wscales_tiled + (static_cast<size_t>(nb) * kblocks + 4 * ks) * 1024,
                        SFB_BYTES, sfl_bar(s));
          } else {
            const int hr = FOLDED ? st : st - num_k;   // which 64-wide half of R
            if (leader)
              mbar_arrive_expect_tx(full_bar(s),
                                    2 * (LR_A_BYTES + (weights_in ? 0u : LR_B_BYTES)));
            tma_load_2d_cg2(s_a(s), &tm_l, hr * 64, arow, fb);
            if (!weights_in) tma_load_2d_cg2(s_b(s), &tm_p, hr * 64, brow, fb);
            // no scales for the low-rank uses; the barrier keeps its phases
            mbar_arrive(sfl_bar(s));
          }
        }
      }
      if (!ok) {
        // Let the copies already issued land before the block exits: this
        // CTA's scale copies, and (even CTA) the operand copies of both CTAs,
        // which complete on its full barriers.  The teardown's cluster
        // barrier keeps both CTAs alive until then.
        const uint32_t n = it < STAGES ? it : STAGES;
        for (uint32_t j = 0; j < n; ++j) {
          const uint32_t jt = it - 1 - j;
          if ((jt & 1u) != pid) continue;      // the other producer's use
          drain_wait(sfl_bar(jt % STAGES), (jt / STAGES) & 1u, 50000000ull);
          if (leader) drain_wait(full_bar(jt % STAGES), (jt / STAGES) & 1u, 50000000ull);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------------------------------------------- MMA issuer --
      const uint32_t idesc_main = idesc_nvfp4(BM, BN);
      const uint32_t idesc_lr = idesc_bf16_f32(BM, BN, 0, 0);
      uint32_t it = 0, tc = 0;
      bool ok = true;
      for (int t = pair; t < tiles && ok; t += npairs, ++tc) {
        if (!svdq_wait(tmem_empty_bar, (tc & 1u) ^ 1u, SITE_MMA_TE)) break;
        tc_fence_after();
        // LR_FOLDED: the two low-rank uses first (the first MMA starts the
        // accumulator), then the K steps, all into the main accumulator.
        const int main_uses = FOLDED ? uses : num_k;
        for (int st = 0; st < main_uses; ++st, ++it) {
          const uint32_t s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!svdq_wait(full_bar(s), ph, SITE_MMA_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (FOLDED && st < 2) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f16_cg2(tmem_base + TM_ACC,
                          smem_desc(s_a(s) + 32 * kk, 16, 1024, kLayoutSwizzle128B),
                          smem_desc(s_b(s) + 32 * kk, 16, 1024, kLayoutSwizzle128B), idesc_lr,
                          (st | kk) != 0 ? 1u : 0u);
          } else {
            const uint32_t sfa_t = tmem_base + TM_SF + TM_SF_SLOT * s;
            const uint32_t sfb_t = sfa_t + 16;
            const int ks = st - k0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              mma_nvfp4_cg2(tmem_base + TM_ACC,
                            smem_desc(s_a(s) + 32 * j, 16, 1024, kLayoutSwizzle128B),
                            smem_desc(s_b(s) + 32 * j, 16, 1024, kLayoutSwizzle128B), idesc_main,
                            sfa_t + 4 * j, sfb_t + 8 * j, (FOLDED || (ks | j) != 0) ? 1u : 0u);
            }
          }
          tc_commit_cg2_mc(empty_bar(s), 0x3);
        }
        if (!ok) break;
        if (LRM == LR_SEPARATE) {
          // The low-rank accumulator overlaps the scale slots: every main
          // MMA completes before the low-rank MMAs write there.
          tc_commit_cg2(drain_bar);
          if (!svdq_wait(drain_bar, tc & 1u, SITE_MMA_DRAIN)) break;
          tc_fence_after();
          for (int hr = 0; hr < 2 && ok; ++hr, ++it) {
            const uint32_t s = it % STAGES;
            const uint32_t ph = (it / STAGES) & 1u;
            if (!svdq_wait(full_bar(s), ph, SITE_MMA_FULL)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f16_cg2(tmem_base + TM_LR,
                          smem_desc(s_a(s) + 32 * kk, 16, 1024, kLayoutSwizzle128B),
                          smem_desc(s_b(s) + 32 * kk, 16, 1024, kLayoutSwizzle128B), idesc_lr,
                          (hr | kk) != 0 ? 1u : 0u);
            tc_commit_cg2_mc(empty_bar(s), 0x3);
          }
          if (!ok) break;
        }
        tc_commit_cg2_mc(tmem_full_bar, 0x3);
      }
      // Every MMA this thread issued completes before TMEM is released.
      tc_commit_cg2(final_bar);
      drain_wait(final_bar, 0, 100000000ull);
    }
  } else {
    // -------------------------------------- scale writers and epilogue --
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int half = (warp - EPI_WARP0) >> 2;     // which 128 of the tile's 256 columns
    const int et = threadIdx.x - 32 * EPI_WARP0;  // 0..255
    const float alpha = __bfloat162float(p.wtscale[0]);
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t s_obuf = s_out + static_cast<uint32_t>(warp - EPI_WARP0) * OUT_WARP_BYTES;
    const uint32_t full_leader0 = map_to_rank(full_bar(0), 0);
    const uint32_t tmem_empty_leader = map_to_rank(tmem_empty_bar, 0);
    float* wc_s = reinterpret_cast<float*>(smem + (s_colv - s_ring));
    float* bs_s = wc_s + BN;
    uint32_t tc = 0, u = 0;   // tiles, stage uses written
    bool ok = true;
    // Stage uses u .. u + n - 1: wait for the stage's scale bytes, write the
    // K steps' scales into the stage's TMEM slot (this warp: blocks
    // 6 * half .. 6 * half + 5, columns 4 b .. 4 b + 3 for block b, in its
    // lane quarter), and report to the even CTA.  Low-rank uses carry no
    // scales; the arrival keeps the barrier phases in step.
    auto write_uses = [&](uint32_t n) {
      for (uint32_t e = u + n; u < e; ++u) {
        const uint32_t s = u % STAGES;
        const uint32_t ph = (u / STAGES) & 1u;
        if (ok) ok = __all_sync(0xFFFFFFFFu, svdq_wait(sfl_bar(s), ph, SITE_SF_LOADED));
        if (!ok) continue;
        if (!lr_use(static_cast<int>(u % static_cast<uint32_t>(uses)))) {
          const uint32_t src = s_sf(s) + 16 * lane;
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
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(full_leader0 + 8u * s);
      }
    };
    // Per-column factors of tile column nb -> shared memory (every warp has
    // finished the previous tile's arithmetic, which read them).
    auto load_columns = [&](int nb) {
      const int n = nb * BN + et;
      float wcv = 0.f, bsv = 0.f;
      if (n < p.N) {
        wcv = __bfloat162float(p.wcscales[n]);
        if (p.bias != nullptr) bsv = __bfloat162float(p.bias[n]);
      }
      wc_s[et] = wcv * alpha;
      bs_s[et] = bsv;
    };
    // Rows -> swizzled buffer (row = lane, 128 B per row; 16-byte chunk j of
    // row r at chunk j ^ (r % 8), the TMA 128-byte swizzle) -> TMA store of
    // 32 rows x 64 columns, twice per tile; `between` runs after the first.
    auto store_rows = [&](const uint32_t (&out)[8][8], int mb, int nb, auto&& between) {
      const int row0 = mb * BM + static_cast<int>(rank) * BM_CTA + q * 32;
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
        if (pc == 0) between();
      }
    };
    // Every epilogue warp passes the named barriers once per tile, also
    // after a failed wait, so that no warp is left waiting on them.
    if constexpr (LRM == LR_SEPARATE) {
      // A tile's first `head` stage uses are written right after the
      // previous tile's TMEM reads, before its output stores, and `mid` more
      // between the two output pieces, so the MMAs restart soon and do not
      // wait for the stores.
      const uint32_t head = num_k < STAGES ? static_cast<uint32_t>(num_k) : STAGES;
      const uint32_t mid = num_k - head < 2u ? num_k - head : 2u;
      const uint32_t rest = static_cast<uint32_t>(uses) - head - mid;
      if (pair < tiles) write_uses(head + mid);
      for (int t = pair; t < tiles; t += npairs, ++tc) {
        const int mb = t % p.m_tiles;
        const int nb = t / p.m_tiles;
        const bool has_next = t + npairs < tiles;
        write_uses(rest);
        load_columns(nb);
        named_bar_sync(2, 32 * NUM_EPI_WARPS);
        if (ok) ok = __all_sync(0xFFFFFFFFu, svdq_wait(tmem_full_bar, tc & 1u, SITE_EPI));
        uint32_t out[8][8];
        if (ok) {
          tc_fence_after();
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
              out[c][i] = pack_bf16x2(o0, o1);
            }
          }
          tc_fence_before();
        }
        // All TMEM reads of this CTA are done: the low-rank columns (which
        // the next tile's scale slots overlap) and the accumulator are free.
        named_bar_sync(3, 32 * NUM_EPI_WARPS);
        if (!ok) continue;
        if (lane == 0) mbar_arrive_remote(tmem_empty_leader);
        if (has_next) write_uses(head);
        store_rows(out, mb, nb, [&] {
          if (has_next) write_uses(mid);
        });
      }
    } else {
      // Scale slots and accumulator are disjoint, so the scale writes run
      // ahead of the epilogue.  Of the next tile's stage uses, `pre` are
      // written before this tile's accumulator is read (their stages land
      // while this tile's last K steps run), `post` right after it is
      // released, `mid` between the two output pieces and the rest after
      // the stores.  Each warp releases the accumulator as soon as its own
      // reads are done; the arithmetic follows.
      const uint32_t U = static_cast<uint32_t>(uses);
      const uint32_t pre = U < 3u ? U : 3u;
      const uint32_t post = U - pre < 2u ? U - pre : 2u;
      const uint32_t mid = U - pre - post < 2u ? U - pre - post : 2u;
      const uint32_t rest = U - pre - post - mid;
      if (pair < tiles) write_uses(U);
      for (int t = pair; t < tiles; t += npairs, ++tc) {
        const int mb = t % p.m_tiles;
        const int nb = t / p.m_tiles;
        const bool has_next = t + npairs < tiles;
        load_columns(nb);
        named_bar_sync(2, 32 * NUM_EPI_WARPS);
        if (has_next) write_uses(pre);
        if (ok) ok = __all_sync(0xFFFFFFFFu, svdq_wait(tmem_full_bar, tc & 1u, SITE_EPI));
        // Two batches of 64 columns (all 128 would not fit the registers
        // beside the output words); the accumulator is released after the
        // second batch's reads, before its arithmetic.
        uint32_t out[8][8];
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t acc[4][16];
#pragma unroll
            for (int c = 0; c < 4; ++c)
              tmem_ld_32x32b_x16(lane_base + TM_ACC + half * 128 + 64 * h + 16 * c, acc[c]);
            tmem_ld_wait();
            if (h == 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive_remote(tmem_empty_leader);
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int col = half * 128 + 64 * h + 16 * c;
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float2 w2 = *reinterpret_cast<const float2*>(wc_s + col + 2 * i);
                const float2 b2 = *reinterpret_cast<const float2*>(bs_s + col + 2 * i);
                out[4 * h + c][i] =
                    pack_bf16x2(fmaf(__uint_as_float(acc[c][2 * i]), w2.x, b2.x),
                                fmaf(__uint_as_float(acc[c][2 * i + 1]), w2.y, b2.y));
              }
            }
          }
        }
        if (has_next) write_uses(post);
        // Every warp has read this tile's column factors.
        named_bar_sync(3, 32 * NUM_EPI_WARPS);
        if (!ok) continue;
        store_rows(out, mb, nb, [&] {
          if (has_next) write_uses(mid);
        });
        if (has_next) write_uses(rest);
      }
    }
    if (lane == 0) bulk_wait_group0();
  }

  // ----------------------------------------------------------- teardown --
  // Neither CTA releases its TMEM or shared memory while the pair's MMAs,
  // copies or the other CTA's arrivals may still reach them.
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_cg2(tmem_base, TMEM_COLS);
  }
}

}  // namespace kg2
}  // namespace svdq
