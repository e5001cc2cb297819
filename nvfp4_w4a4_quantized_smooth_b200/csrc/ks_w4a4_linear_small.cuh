// ks_w4a4_linear_small.cuh -- the block-scaled NVFP4 GEMM with the fused
// SVDQuant epilogue for few tokens (M <= 64), for sm_100a.
//
// Same computation as kg_w4a4_linear.cuh (nunchaku-z-image-turbo-svdq model
// card, "What's stored on disk", runtime formula), computed transposed:
//   y^T[n, m] = acc^T[n, m] * wtscale * wcscales[n] + (proj_up @ L^T)[n, m] + bias[n]
//   acc^T[n, m] = sum_k e2m1(qw[n,k]) sw[k/16,n] e2m1(qa[m,k]) sa[m,k/16]
// The weights are the MMA's 128-row A operand and the (at most 64) tokens
// its N = 64 operand, so N / 128 CTAs share the weight stream, each over
// its K range (a 128-token x 256-column tile would leave N / 256 CTAs for
// it).  One CTA per 128 weight rows and K range: with `split` > 1 the K
// steps of a tile are divided among the `split` CTAs of a thread-block
// cluster: each rank stores the rows of its fp32 partial tile that rank o
// sums -- rows [o 128 / split, (o + 1) 128 / split) -- into rank o's
// receive buffer (distributed shared memory stores) and keeps its own copy
// of the low-rank tile; after one cluster barrier every rank sums its rows
// over all ranks in rank order from its own shared memory (deterministic),
// applies the epilogue and stores those columns of y.  With `split` = 1 a CTA covers the whole
// K range and loops over tiles when there are more than SMs.
//
// Roles (192 threads):
//   warp 0      producer (one thread): a ring of SLOTS slots, one K step of
//               256 each: the qweight box (128 rows x 128 B), the qact box
//               (64 rows x 128 B; rows beyond M read as zero), the four
//               512-byte scale blocks of the tile's 128 weight rows (one 3-D
//               box out of the 256-row tile order of the repacked weight
//               scales) and the four scale blocks of the tokens (one bulk
//               copy).  A tile's first two slots carry the low-rank halves
//               (proj_up half in the weight place, L half in the token
//               place), so that their latency overlaps the K steps.
//   warp 1      TMEM owner and MMA issuer (one thread): tcgen05.mma
//               kind::f16 (bf16, K = 16) for proj_up @ L^T into the low-rank
//               accumulator, then kind::mxf4nvf4 block16, M = 128, N = 64,
//               K = 64 into the main one.
//   warps 2..5  one per TMEM lane quarter.  During the K loop: slot s's
//               scale blocks -> TMEM scale slot s (tcgen05.st, each block
//               replicated in the four lane quarters, as the MMA reads it).
//               After it, the epilogue: TMEM -> registers, fp32
//               acc * wtscale * wcscales + lr + bias -> bf16, transposed
//               into a [64 tokens][128 columns] shared buffer, then one TMA
//               tensor store, which clips the M and N edges (split > 1:
//               both accumulators -> shared memory for the cluster sum).
// TMEM (512 columns): accumulator [0, 64), low-rank accumulator [64, 128),
// scale slot s at [128 + 32 s, 160 + 32 s): weight scales (4 MMAs x 4
// columns), then token scales (4 x 4).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace svdq {
namespace ks {

constexpr int BMW = 128;         // weight rows per tile (MMA M)
constexpr int NT = 64;           // token columns (MMA N); M <= NT
constexpr int BK_BYTES = 128;    // K step: 256 FP4 values = 128 bytes per row
constexpr int BK = 256;
constexpr int SLOTS = 6;
constexpr uint32_t A_BYTES = BMW * BK_BYTES;         // 16 KB
constexpr uint32_t B_BYTES = NT * BK_BYTES;          // 8 KB
constexpr uint32_t SFA_BYTES = 4 * 512;              // 128 weight rows x 16 scales
constexpr uint32_t SFB_BYTES = 4 * 512;              // one 128-row token block x 16 scales
constexpr uint32_t SLOT_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;   // 28 KB
constexpr uint32_t LR_A_BYTES = BMW * 64 * 2;        // proj_up half: 128 rows x 64 bf16
constexpr uint32_t LR_B_BYTES = NT * 64 * 2;         // L half: 64 rows x 64 bf16
static_assert(LR_A_BYTES <= A_BYTES && LR_B_BYTES <= B_BYTES, "low-rank halves fit a slot");
constexpr uint32_t RING_BYTES = SLOTS * SLOT_BYTES;
constexpr uint32_t OUT_BYTES = NT * BMW * 2;         // [64 tokens][128 columns] bf16
// split > 1: the partial rows every rank sends this one, [rank][token][row]
// fp32 (split ranks x 64 tokens x 128 / split rows)
constexpr uint32_t RECV_BYTES = NT * BMW * 4;
constexpr uint32_t BAR_BYTES = 256;
constexpr uint32_t SMEM_BYTES = RING_BYTES + OUT_BYTES + RECV_BYTES + BAR_BYTES + 1024;
constexpr int EPI_WARP0 = 2;
constexpr int NUM_EPI_WARPS = 4;
constexpr int NUM_THREADS = 32 * (EPI_WARP0 + NUM_EPI_WARPS);
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_ACC = 0;
constexpr uint32_t TM_LR = 64;
constexpr uint32_t TM_SF = 128;
constexpr uint32_t TM_SF_SLOT = 32;
static_assert(TM_SF + SLOTS * TM_SF_SLOT <= TMEM_COLS, "scale columns fit");
static_assert(SLOT_BYTES % 1024 == 0 && RING_BYTES % 1024 == 0,
              "operand boxes stay 1024-aligned");
static_assert(8 * 3 * SLOTS + 32 <= BAR_BYTES, "barriers fit");
static_assert(SMEM_BYTES <= 232448, "fits the shared memory of one SM");

// Wait-site ids recorded in the error word.
constexpr uint32_t SITE_PROD = 0x40, SITE_MMA_TE = 0x41, SITE_MMA_FULL = 0x42,
                   SITE_MMA_SF = 0x43, SITE_SF_FULL = 0x44, SITE_EPI = 0x45;

struct Params {
  const uint8_t* ascales_tiled;      // token scales, 128-row tile order (tile 0)
  const __nv_bfloat16* wcscales;
  const __nv_bfloat16* wtscale;
  const __nv_bfloat16* bias;         // may be null
  __nv_bfloat16* y;                  // [M, ldy], written directly when split > 1
  int M, N, K, ldy;
  int n_tiles;                       // 128-row weight tiles
  int split;                         // K ranges per tile = cluster size (1, 2, 4, 8)
};

// LR: the layer has the low-rank branch (R = 128); without it (R = 0) a
// tile has no low-rank slots or MMAs and the epilogue reads only the main
// accumulator.
template <bool LR>
__global__ void __launch_bounds__(NUM_THREADS, 1)
w4a4_linear_small_kernel(const __grid_constant__ CUtensorMap tm_w,   // qweight [N, K/2] u8, box {128, 128}
                         const __grid_constant__ CUtensorMap tm_x,   // qact [M, K/2] u8, box {128, 64}
                         const __grid_constant__ CUtensorMap tm_sw,  // weight scales, u32 {128, 2, N/256 * K/64}, box {128, 1, 4}
                         const __grid_constant__ CUtensorMap tm_p,   // proj_up [N, 128] bf16, box {64, 128}
                         const __grid_constant__ CUtensorMap tm_l,   // lowrank [M, 128] bf16, box {64, 64}
                         const __grid_constant__ CUtensorMap tm_y,   // y [M, ldy] bf16, box {128, 64}
                         const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t s_ring = smem_u32(smem);
  auto s_a = [&](uint32_t s) { return s_ring + s * SLOT_BYTES; };
  auto s_b = [&](uint32_t s) { return s_ring + s * SLOT_BYTES + A_BYTES; };
  auto s_sf = [&](uint32_t s) { return s_ring + s * SLOT_BYTES + A_BYTES + B_BYTES; };
  const uint32_t s_out = s_ring + RING_BYTES;
  // After the last MMA (split > 1): this rank's low-rank tile, [64 tokens]
  // [128 columns] fp32, over the first ring slots (no copy or MMA uses the
  // ring any more); the receive buffer has its own place, as other ranks
  // may store into it while this one still runs its K loop.
  const uint32_t s_lrt = s_ring;
  static_assert(NT * BMW * 4 <= RING_BYTES, "the low-rank tile fits the ring");
  const uint32_t s_recv = s_out + OUT_BYTES;
  const uint32_t s_bar = s_recv + RECV_BYTES;
  // barriers: slot full (TMA bytes), slot scales in TMEM, slot free
  auto full_bar = [&](uint32_t s) { return s_bar + 8u * s; };
  auto sf_full_bar = [&](uint32_t s) { return s_bar + 8u * (SLOTS + s); };
  auto empty_bar = [&](uint32_t s) { return s_bar + 8u * (2 * SLOTS + s); };
  const uint32_t tmem_full_bar = s_bar + 8u * (3 * SLOTS);
  const uint32_t tmem_empty_bar = tmem_full_bar + 8u;
  const uint32_t final_bar = tmem_full_bar + 16u;
  const uint32_t tmem_slot = tmem_full_bar + 24u;
  uint32_t* tmem_slot_ptr = reinterpret_cast<uint32_t*>(smem + (tmem_slot - s_ring));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_sw);
    if (LR) {
      prefetch_tmap(&tm_p);
      prefetch_tmap(&tm_l);
    }
    prefetch_tmap(&tm_y);
    for (uint32_t s = 0; s < SLOTS; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(sf_full_bar(s), NUM_EPI_WARPS);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(tmem_full_bar, 1);
    mbar_init(tmem_empty_bar, NUM_EPI_WARPS);
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
  const int kblocks = p.K / 64;                // 512-byte scale blocks per 128 rows
  const int split = p.split;
  const int rank = split > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const int k0 = num_k * rank / split;         // this CTA's K steps [k0, k0 + nk)
  const int nk = num_k * (rank + 1) / split - k0;
  const int lr_uses = LR ? 2 : 0;
  const int uses = lr_uses + nk;               // ring slots per tile
  const int tile0 = static_cast<int>(blockIdx.x) / split;
  const int tile_step = static_cast<int>(gridDim.x) / split;
  // The weight side of the first tile's first SLOTS slots (qweight box and
  // weight scales, or the proj_up half) is requested before the wait for
  // the previous kernel, so that the weight stream overlaps it.
  const int pre = tile0 < p.n_tiles ? (uses < SLOTS ? uses : SLOTS) : 0;
  if (warp == 0 && lane == 0) {
    for (int st = 0; st < pre; ++st) {
      const uint32_t s = static_cast<uint32_t>(st);
      if (st < lr_uses) {
        mbar_expect_tx(full_bar(s), LR_A_BYTES);
        tma_load_2d(s_a(s), &tm_p, st * 64, tile0 * BMW, full_bar(s));
      } else {
        const int kk = k0 + st - lr_uses;
        mbar_expect_tx(full_bar(s), A_BYTES + SFA_BYTES);
        tma_load_2d(s_a(s), &tm_w, kk * BK_BYTES, tile0 * BMW, full_bar(s));
        tma_load_3d(s_sf(s), &tm_sw, 0, tile0 & 1, (tile0 >> 1) * kblocks + 4 * kk, full_bar(s));
      }
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
      for (int t = tile0; t < p.n_tiles && ok; t += tile_step) {
        for (int st = 0; st < uses; ++st, ++it) {
          const uint32_t s = it % SLOTS;
          const uint32_t ph = (it / SLOTS) & 1u;
          if (!svdq_wait(empty_bar(s), ph ^ 1u, SITE_PROD)) {
            ok = false;
            break;
          }
          const bool weights_in = static_cast<int>(it) < pre;   // requested before the wait
          if (st < lr_uses) {
            const int hr = st;                   // which 64-wide half of R
            mbar_arrive_expect_tx(full_bar(s), (weights_in ? 0u : LR_A_BYTES) + LR_B_BYTES);
            if (!weights_in) tma_load_2d(s_a(s), &tm_p, hr * 64, t * BMW, full_bar(s));
            tma_load_2d(s_b(s), &tm_l, hr * 64, 0, full_bar(s));
          } else {
            const int kk = k0 + st - lr_uses;    // K step
            mbar_arrive_expect_tx(full_bar(s), weights_in ? B_BYTES + SFB_BYTES : SLOT_BYTES);
            if (!weights_in) {
              tma_load_2d(s_a(s), &tm_w, kk * BK_BYTES, t * BMW, full_bar(s));
              // weight rows [128 t, 128 t + 128) = half (t & 1) of 256-row tile t / 2
              tma_load_3d(s_sf(s), &tm_sw, 0, t & 1, (t >> 1) * kblocks + 4 * kk, full_bar(s));
            }
            tma_load_2d(s_b(s), &tm_x, kk * BK_BYTES, 0, full_bar(s));
            bulk_load(s_sf(s) + SFA_BYTES, p.ascales_tiled + static_cast<size_t>(4 * kk) * 512,
                      SFB_BYTES, full_bar(s));
          }
        }
      }
      if (!ok) {
        // Let the copies already issued land before the block exits.
        const uint32_t n = it < SLOTS ? it : SLOTS;
        for (uint32_t j = 0; j < n; ++j) {
          const uint32_t jt = it - 1 - j;
          drain_wait(full_bar(jt % SLOTS), (jt / SLOTS) & 1u, 50000000ull);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------- MMA issuer --
      const uint32_t idesc_main = idesc_nvfp4(BMW, NT);
      const uint32_t idesc_lr = idesc_bf16_f32(BMW, NT, 0, 0);
      uint32_t it = 0, tc = 0;
      bool ok = true;
      for (int t = tile0; t < p.n_tiles && ok; t += tile_step, ++tc) {
        if (!svdq_wait(tmem_empty_bar, (tc & 1u) ^ 1u, SITE_MMA_TE)) break;
        tc_fence_after();
        if (LR) {
          // The low-rank accumulator has its own columns.
          for (int hr = 0; hr < 2 && ok; ++hr, ++it) {
            const uint32_t s = it % SLOTS;
            const uint32_t ph = (it / SLOTS) & 1u;
            if (!svdq_wait(full_bar(s), ph, SITE_MMA_FULL)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f16(tmem_base + TM_LR, smem_desc(s_a(s) + 32 * kk, 16, 1024, kLayoutSwizzle128B),
                      smem_desc(s_b(s) + 32 * kk, 16, 1024, kLayoutSwizzle128B), idesc_lr,
                      (hr | kk) != 0 ? 1u : 0u);
            tc_commit(empty_bar(s));
          }
          if (!ok) break;
        }
        for (int st = 0; st < nk; ++st, ++it) {
          const uint32_t s = it % SLOTS;
          const uint32_t ph = (it / SLOTS) & 1u;
          if (!svdq_wait(full_bar(s), ph, SITE_MMA_FULL) ||
              !svdq_wait(sf_full_bar(s), ph, SITE_MMA_SF)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sfa_t = tmem_base + TM_SF + TM_SF_SLOT * s;
          const uint32_t sfb_t = sfa_t + 16;
#pragma unroll
          for (int j = 0; j < 4; ++j)
            mma_nvfp4(tmem_base + TM_ACC,
                      smem_desc(s_a(s) + 32 * j, 16, 1024, kLayoutSwizzle128B),
                      smem_desc(s_b(s) + 32 * j, 16, 1024, kLayoutSwizzle128B), idesc_main,
                      sfa_t + 4 * j, sfb_t + 4 * j, (st | j) != 0 ? 1u : 0u);
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
    // ------------------------------------- scale writers, then epilogue --
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const float alpha = __bfloat162float(p.wtscale[0]);
    const int n_local = q * 32 + lane;   // this thread's weight row in the tile
    uint32_t it = 0, tc = 0;
    bool ok = true;
    for (int t = tile0; t < p.n_tiles; t += tile_step, ++tc) {
      // Scale blocks of each K step -> this quarter's lanes of TMEM slot s
      // (block b at columns 4 b .. 4 b + 3: weight blocks 0..3, token
      // blocks 4..7).  The slot's previous MMAs have completed: the
      // producer reloaded the slot only after them.  Every ring use, the
      // low-rank ones included (nothing to write), completes one phase of
      // the slot's scale barrier, so that its phases follow the ring.
      for (int st = 0; st < uses; ++st, ++it) {
        const uint32_t s = it % SLOTS;
        const uint32_t ph = (it / SLOTS) & 1u;
        if (ok) ok = __all_sync(0xFFFFFFFFu, svdq_wait(full_bar(s), ph, SITE_SF_FULL));
        if (!ok) continue;
        if (st >= lr_uses) {
          tc_fence_after();
          const uint32_t src = s_sf(s) + 16 * lane;
          const uint32_t dst = lane_base + TM_SF + TM_SF_SLOT * s;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint32_t v[8];
            ld_shared_v4(src + 512 * (2 * k), v[0], v[1], v[2], v[3]);
            ld_shared_v4(src + 512 * (2 * k + 1), v[4], v[5], v[6], v[7]);
            tmem_st_32x32b_x8(dst + 8 * k, v);
          }
          tmem_st_wait();
          tc_fence_before();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(sf_full_bar(s));
      }
      // Epilogue.  Every epilogue warp passes both named barriers once per
      // tile, also after a failed wait, so that none is left waiting.
      const int n = t * BMW + n_local;
      float wc = 0.f, bs = 0.f;
      if (n < p.N) {
        wc = __bfloat162float(p.wcscales[n]) * alpha;
        if (p.bias != nullptr) bs = __bfloat162float(p.bias[n]);
      }
      if (ok) ok = __all_sync(0xFFFFFFFFu, svdq_wait(tmem_full_bar, tc & 1u, SITE_EPI));
      if (ok && split > 1) {
        // This rank's partial rows -> the receive buffer of the rank that
        // sums them ([rank][token][row - first row of that rank]); its
        // low-rank tile -> its own shared memory ([token][column] fp32).
        tc_fence_after();
        const int r0 = BMW / split;
        const int owner = n_local / r0;
        const uint32_t recv_o =
            map_to_rank(s_recv + static_cast<uint32_t>(rank * NT * r0 + (n_local - owner * r0)) * 4u,
                        static_cast<uint32_t>(owner));
#pragma unroll
        for (int c = 0; c < NT / 16; ++c) {
          uint32_t acc[16], lr[16];
          tmem_ld_32x32b_x16(lane_base + TM_ACC + 16 * c, acc);
          if (LR) {
            tmem_ld_32x32b_x16(lane_base + TM_LR + 16 * c, lr);
          } else {
#pragma unroll
            for (int z = 0; z < 16; ++z) lr[z] = 0u;   // +0.0f
          }
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int m = 16 * c + i;
            st_dsmem_f32(recv_o + static_cast<uint32_t>(m * r0) * 4u, __uint_as_float(acc[i]));
            st_shared_f32(s_lrt + static_cast<uint32_t>(m * BMW + n_local) * 4u,
                          __uint_as_float(lr[i]));
          }
        }
      } else if (ok) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < NT / 16; ++c) {
          uint32_t acc[16], lr[16];
          tmem_ld_32x32b_x16(lane_base + TM_ACC + 16 * c, acc);
          if (LR) {
            tmem_ld_32x32b_x16(lane_base + TM_LR + 16 * c, lr);
          } else {
#pragma unroll
            for (int z = 0; z < 16; ++z) lr[z] = 0u;   // +0.0f
          }
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float o = fmaf(__uint_as_float(acc[i]), wc, __uint_as_float(lr[i]) + bs);
            const __nv_bfloat16 h = __float2bfloat16_rn(o);
            const int m = 16 * c + i;
            st_shared_u16(s_out + static_cast<uint32_t>(m * BMW + n_local) * 2u,
                          *reinterpret_cast<const uint16_t*>(&h));
          }
        }
        // TMEM is free for the next tile as soon as every warp has its values.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tmem_empty_bar);
        fence_proxy_async_smem();
      }
      named_bar_sync(1, 32 * NUM_EPI_WARPS);
      if (warp == EPI_WARP0 && lane == 0) {
        if (ok && split == 1) {
          tma_store_2d(&tm_y, s_out, t * BMW, 0);
          bulk_commit_group();
        }
        bulk_wait_group_read0();    // the buffer may be rewritten
      }
      named_bar_sync(1, 32 * NUM_EPI_WARPS);
    }
    if (warp == EPI_WARP0 && lane == 0) bulk_wait_group0();
  }

  if (split > 1) {
    // ------------------------------------------------- cluster K sum --
    // Every thread of every rank takes the cluster barrier, after which
    // every rank's stores into this rank's receive buffer are visible.
    // Rank r sums rows [r R0, (r + 1) R0) of all ranks' partial tiles in
    // rank order; a unit is 4 consecutive rows of one token (a float4 of
    // each rank's slice), so that a warp reads and writes whole 16-byte
    // pieces.  The low-rank tile is this rank's own copy.  No rank touches
    // another's shared memory after the barrier, so none waits for the
    // others before it exits.
    __syncwarp();
    cluster_sync_all();
    if (warp >= EPI_WARP0 && !error_raised()) {
      const int et = static_cast<int>(threadIdx.x) - 32 * EPI_WARP0;   // 0..127
      const int r0 = BMW / split;                  // rows this rank sums
      const int groups = r0 / 4;
      const int t = tile0;
      for (int u = et; u < groups * NT; u += 32 * NUM_EPI_WARPS) {
        const int m = u / groups;
        const int row = rank * r0 + 4 * (u % groups);
        const int n = t * BMW + row;
        if (m >= p.M || n >= p.N) continue;
        const uint32_t roff = static_cast<uint32_t>(m * r0 + 4 * (u % groups)) * 4u;
        float4 sum = ld_shared_f4(s_recv + roff);
        for (int j = 1; j < split; ++j) {
          const float4 v = ld_shared_f4(s_recv + static_cast<uint32_t>(j * NT * r0) * 4u + roff);
          sum.x += v.x;
          sum.y += v.y;
          sum.z += v.z;
          sum.w += v.w;
        }
        const float4 lr = ld_shared_f4(s_lrt + static_cast<uint32_t>(m * BMW + row) * 4u);
        const float sv[4] = {sum.x, sum.y, sum.z, sum.w};
        const float lv[4] = {lr.x, lr.y, lr.z, lr.w};
        uint32_t packed[2];
#pragma unroll
        for (int k = 0; k < 4; k += 2) {
          float o[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float wc = __bfloat162float(p.wcscales[n + k + e]) * __bfloat162float(p.wtscale[0]);
            const float bs = p.bias != nullptr ? __bfloat162float(p.bias[n + k + e]) : 0.f;
            o[e] = fmaf(sv[k + e], wc, lv[k + e] + bs);
          }
          __nv_bfloat162 h = __floats2bfloat162_rn(o[0], o[1]);
          packed[k / 2] = *reinterpret_cast<uint32_t*>(&h);
        }
        st_global_v2(p.y + static_cast<size_t>(m) * p.ldy + n, packed[0], packed[1]);
      }
    }
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

}  // namespace ks
}  // namespace svdq
