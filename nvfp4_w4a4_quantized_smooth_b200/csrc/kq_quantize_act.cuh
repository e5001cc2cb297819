// kq_quantize_act.cuh -- activation side of the SVDQuant W4A4 layer for
// sm_100a: reads x once and writes quant(x * smooth) (NVFP4) and the
// low-rank product L = x @ proj_down (nunchaku-z-image-turbo-svdq model
// card, "What's stored on disk", runtime formula).
//
// Quantization of each 16-element group along K (one e4m3 scale per 16 k,
// E2M1 elements, as the card's first paragraph states; rounding to
// nearest-even with saturation):
//   v = x * smooth                  exact in fp32 (bf16 x bf16)
//   s = e4m3(amax|v| / 6)           quotient, then the hardware RNE /
//                                   satfinite conversion
//   q = E2M1(v / s)                 quotient, then the hardware RNE /
//                                   satfinite conversion
// Each quotient a / b is formed as r = 1/b (reciprocal), q0 = a r, then one
// residual step e = a - q0 b (exact by FMA), q = q0 + e r (Markstein, IBM J.
// Res. Dev. 34(1), 1990).  Rounding that q equals rounding the exact
// quotient: a bf16 x bf16 product has at most 16 significant bits, and
// every e4m3 midpoint x 6 and every E2M1 midpoint x s at most 7, so a
// quotient that is not exactly a midpoint lies at least 2^-16 (relative)
// from it, far more than q's error (a few ulps of fp32); a quotient that is
// exactly a midpoint is representable and the residual step returns it
// exactly (|1 - b r| <= 2^-22 makes the step's error far below half an
// ulp), so the conversion sees the tie.  A scale that rounds to zero gives
// r = 0 and therefore signed zero codes.
//
// CTA layout: a tile of BM rows (32..256) over a K range, 18 warps.
//   warp 0      TMA producer: per stage of 64 or 128 k, the x tile as
//               [BM rows x 64 k] bf16 boxes (128-byte swizzle), proj_down
//               rows [64 k x 128 r] per box pair (64 x 64 boxes) and the
//               smooth values, into a ring of stages.
//   warp 1      TMEM owner, MMA issuer.  The low-rank product is computed
//               transposed, L^T[128 x BM] += proj_down_chunk^T x_tile^T:
//               tcgen05.mma kind::f16, M = 128 (= R), N = BM, K = 16;
//               A (proj_down) MN-major, B (x tile) K-major, fp32 in BM
//               TMEM columns.  So BM is free (multiple of 32) while the
//               accumulator keeps the full 128-lane layout.
//   warps 2..17 quantize the same shared-memory x tile (four warps per
//               scheduler, one 16-element group per thread per stage for
//               BM = 64), write packed codes and tiled scales; afterwards
//               read L^T out of TMEM.
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

constexpr int R = 128;                 // rank (MMA M)
constexpr int BKE = 64;                // k per chunk (one 128-byte swizzled box row)
constexpr int MAX_BM = 256;
constexpr int MAX_STAGES = 6;
constexpr uint32_t PD_BOX = 64 * 64 * 2;          // [64 k x 64 r] bf16 box, 8 KB
constexpr uint32_t PD_CHUNK = 2 * PD_BOX;         // one chunk of proj_down, 16 KB
constexpr uint32_t SMOOTH_CHUNK = BKE * 2;        // 128 B
constexpr int NUM_QWARPS = 16;
constexpr int NUM_QTHREADS = NUM_QWARPS * 32;
constexpr int NUM_THREADS = 64 + NUM_QTHREADS;
constexpr uint32_t BAR_BYTES = 256;
constexpr uint32_t SMEM_BUDGET = 227 * 1024;
constexpr int PART_STRIDE = R + 4;  // floats per row m of the partial-L buffer

constexpr uint32_t SITE_PROD = 0x20, SITE_MMA = 0x21, SITE_QUANT = 0x22, SITE_LFULL = 0x23;

// A stage holds `cps` chunks of 64 k (1 or 2): x [bm rows x 128 B] per
// chunk, proj_down [64 k x 128 r] per chunk, 128 B of smooth per chunk.
__host__ __device__ constexpr uint32_t x_chunk(int bm) { return static_cast<uint32_t>(bm) * 128u; }
__host__ __device__ constexpr uint32_t x_bytes(int bm, int cps) { return cps * x_chunk(bm); }
__host__ __device__ constexpr uint32_t stage_bytes(int bm, int cps) {
  return (cps * (x_chunk(bm) + PD_CHUNK + SMOOTH_CHUNK) + 1023u) & ~1023u;
}
__host__ __device__ constexpr int num_stages(int bm, int cps) {
  return (SMEM_BUDGET - 1024 - BAR_BYTES) / stage_bytes(bm, cps) < MAX_STAGES
             ? static_cast<int>((SMEM_BUDGET - 1024 - BAR_BYTES) / stage_bytes(bm, cps))
             : MAX_STAGES;
}
__host__ __device__ constexpr uint32_t smem_bytes(int bm, int cps) {
  return num_stages(bm, cps) * stage_bytes(bm, cps) + BAR_BYTES + 1024;
}
// Two chunks per stage when that still leaves three stages in flight.
__host__ __device__ constexpr int chunks_per_stage(int bm) {
  return num_stages(bm, 2) >= 3 ? 2 : 1;
}
__host__ __device__ constexpr uint32_t tmem_cols(int bm) {
  return bm <= 32 ? 32u : bm <= 64 ? 64u : bm <= 128 ? 128u : 256u;
}
static_assert(MAX_BM * PART_STRIDE * 4 <=
                  num_stages(MAX_BM, chunks_per_stage(MAX_BM)) *
                      stage_bytes(MAX_BM, chunks_per_stage(MAX_BM)),
              "partial buffer fits the ring");
static_assert(num_stages(32, chunks_per_stage(32)) >= 3 &&
                  num_stages(MAX_BM, chunks_per_stage(MAX_BM)) >= 3,
              "at least three stages");

struct Params {
  const __nv_bfloat16* smooth;
  uint8_t* qact;
  uint8_t* ascales_tiled;
  __nv_bfloat16* lowrank;
  int M, K;
  int chunks;  // K / 64
  int split;   // CTAs per cluster along K
  int bm;      // rows per CTA (multiple of 32, <= 256)
};

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ void st_shared_f32(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// Packed pairs of fp32 (lo in the low word) and their arithmetic.
__device__ __forceinline__ uint64_t pk(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void upk(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// bf16 pair word -> packed fp32 pair (element 2i in the low word).
__device__ __forceinline__ uint64_t bf16x2_to_pk(uint32_t w) {
  return pk(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// One 16-element group: x (8 bf16x2 words), smooth (8 bf16x2 words) ->
// 16 E2M1 codes (element 0 in the lowest nibble) and the e4m3 scale byte.
__device__ __forceinline__ uint64_t quantize_group(const uint32_t (&xw)[8], const uint32_t (&sw)[8],
                                                   uint32_t& scale_byte) {
  uint64_t v[8];
  float m8[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[i] = mul2(bf16x2_to_pk(xw[i]), bf16x2_to_pk(sw[i]));
    float lo, hi;
    upk(v[i], lo, hi);
    m8[i] = fmaxf(fabsf(lo), fabsf(hi));
  }
  // max is exact, so a tree gives the same amax with a short dependency chain
  const float amax = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                           fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
  // amax / 6 with one residual step; r6 = RN(1/6).
  const float r6 = __uint_as_float(0x3E2AAAABu);
  const float a0 = amax * r6;
  const float a6 = fmaf(fmaf(-a0, 6.0f, amax), r6, a0);
  const uint32_t sc = cvt_e4m3x2(a6, 0.0f) & 0xFFu;
  scale_byte = sc;
  const float d = e4m3_to_f32(sc);
  const float r = d > 0.0f ? rcp_approx(d) : 0.0f;
  const uint64_t r2 = pk(r, r);
  const uint64_t nd2 = pk(-d, -d);
  float q[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint64_t q0 = mul2(v[i], r2);
    const uint64_t e = fma2(q0, nd2, v[i]);
    const uint64_t q1 = fma2(e, r2, q0);
    float lo, hi, vlo, vhi;
    upk(q1, lo, hi);
    upk(v[i], vlo, vhi);
    // The residual step turns a quotient of -0 into +0: restore v's sign.
    q[2 * i] = __uint_as_float((__float_as_uint(lo) & 0x7FFFFFFFu) |
                               (__float_as_uint(vlo) & 0x80000000u));
    q[2 * i + 1] = __uint_as_float((__float_as_uint(hi) & 0x7FFFFFFFu) |
                                   (__float_as_uint(vhi) & 0x80000000u));
  }
  const float(&qlo)[8] = *reinterpret_cast<const float(*)[8]>(q);
  const float(&qhi)[8] = *reinterpret_cast<const float(*)[8]>(q + 8);
  return static_cast<uint64_t>(cvt_e2m1x8(qlo)) | (static_cast<uint64_t>(cvt_e2m1x8(qhi)) << 32);
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
quantize_act_kernel(const __grid_constant__ CUtensorMap tm_x,    // x [M, ldx] bf16, box {64, bm}
                    const __grid_constant__ CUtensorMap tm_pd,   // proj_down [K, 128], box {64, 64}
                    const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int bm = p.bm;
  const int cps = chunks_per_stage(bm);
  const uint32_t sbytes = stage_bytes(bm, cps);
  const uint32_t nst = static_cast<uint32_t>(num_stages(bm, cps));
  const uint32_t s_ring = smem_u32(smem);
  const uint32_t s_bar = s_ring + nst * sbytes;
  // Stage layout: x chunks [cps][bm rows x 128 B], proj_down chunks
  // [cps][r half][64 k x 128 B], smooth chunks [cps][128 B].
  auto s_x = [&](uint32_t s, int c) { return s_ring + s * sbytes + c * x_chunk(bm); };
  auto s_pd = [&](uint32_t s, int c) {
    return s_ring + s * sbytes + x_bytes(bm, cps) + c * PD_CHUNK;
  };
  auto s_sm = [&](uint32_t s, int c) {
    return s_ring + s * sbytes + x_bytes(bm, cps) + cps * PD_CHUNK + c * SMOOTH_CHUNK;
  };
  auto full_bar = [&](uint32_t s) { return s_bar + 8u * s; };
  auto empty_bar = [&](uint32_t s) { return s_bar + 8u * (MAX_STAGES + s); };
  const uint32_t lfull_bar = s_bar + 16u * MAX_STAGES;
  const uint32_t final_bar = lfull_bar + 8u;
  const uint32_t tmem_slot = lfull_bar + 16u;
  uint32_t* tmem_slot_ptr = reinterpret_cast<uint32_t*>(smem + (tmem_slot - s_ring));
  const uint32_t ncols = tmem_cols(bm);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int mb = blockIdx.y;
  const int rank = blockIdx.x;  // == rank in the cluster (cluster dims = (split, 1, 1))
  const int c_begin = rank * p.chunks / p.split;
  const int c_end = (rank + 1) * p.chunks / p.split;
  // >= 1 chunk per CTA (host guarantees split <= chunks); stages of cps
  // chunks, the last one possibly partial.
  const int nstages = (c_end - c_begin + cps - 1) / cps;

  if (threadIdx.x == 0) {
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_pd);
    for (uint32_t s = 0; s < nst; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1 + NUM_QWARPS);
    }
    mbar_init(lfull_bar, 1);
    mbar_init(final_bar, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, ncols);
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
      for (; i < nstages; ++i) {
        const uint32_t s = static_cast<uint32_t>(i) % nst;
        const uint32_t ph = (static_cast<uint32_t>(i) / nst) & 1u;
        if (!svdq_wait(empty_bar(s), ph ^ 1u, SITE_PROD)) {
          ok = false;
          break;
        }
        const int kc0 = c_begin + cps * i;
        const int nc = c_end - kc0 < cps ? c_end - kc0 : cps;
        mbar_arrive_expect_tx(full_bar(s), nc * (x_chunk(bm) + PD_CHUNK + SMOOTH_CHUNK));
        for (int c = 0; c < nc; ++c) {
          const int kc = kc0 + c;
          tma_load_2d(s_x(s, c), &tm_x, kc * BKE, mb * bm, full_bar(s));
          tma_load_2d(s_pd(s, c), &tm_pd, 0, kc * BKE, full_bar(s));
          tma_load_2d(s_pd(s, c) + PD_BOX, &tm_pd, 64, kc * BKE, full_bar(s));
          bulk_load(s_sm(s, c), p.smooth + kc * BKE, SMOOTH_CHUNK, full_bar(s));
        }
      }
      if (!ok) {
        const int n = i < static_cast<int>(nst) ? i : static_cast<int>(nst);
        for (int j = 0; j < n; ++j) {
          const uint32_t jt = static_cast<uint32_t>(i - 1 - j);
          drain_wait(full_bar(jt % nst), (jt / nst) & 1u, 50000000ull);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------- MMA issuer --
      // L^T[r, m] += sum_k proj_down[k, r] x[m, k]: A = proj_down chunk
      // (MN-major: r contiguous; the two 64-r halves are 8 KB apart, 8-row
      // k groups 1 KB apart), B = x chunk (K-major, 128-byte rows).
      const uint32_t idesc = idesc_bf16_f32(R, static_cast<uint32_t>(bm), 1, 0);
      bool ok = true;
      for (int i = 0; i < nstages; ++i) {
        const uint32_t s = static_cast<uint32_t>(i) % nst;
        const uint32_t ph = (static_cast<uint32_t>(i) / nst) & 1u;
        if (!svdq_wait(full_bar(s), ph, SITE_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int kc0 = c_begin + cps * i;
        const int nc = c_end - kc0 < cps ? c_end - kc0 : cps;
        for (int c = 0; c < nc; ++c) {
#pragma unroll
          for (int kk = 0; kk < BKE / 16; ++kk) {
            mma_f16(tmem_base, smem_desc(s_pd(s, c) + 2048 * kk, PD_BOX, 1024, kLayoutSwizzle128B),
                    smem_desc(s_x(s, c) + 32 * kk, 16, 1024, kLayoutSwizzle128B), idesc,
                    (i | c | kk) != 0 ? 1u : 0u);
          }
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
    const int rows_pad = (p.M + 127) & ~127;   // rows the tiled scale buffer holds
    bool ok = true;
    for (int i = 0; i < nstages; ++i) {
      const uint32_t s = static_cast<uint32_t>(i) % nst;
      const uint32_t ph = (static_cast<uint32_t>(i) / nst) & 1u;
      if (!__all_sync(0xFFFFFFFFu, svdq_wait(full_bar(s), ph, SITE_QUANT))) {
        ok = false;
        break;
      }
      const int kc0 = c_begin + cps * i;
      const int nc = c_end - kc0 < cps ? c_end - kc0 : cps;
      // bm rows x (4 cps) groups; consecutive lanes take one row's groups
      // (chunk c, then group g of 16 within it), whole warps together.
      const int gshift = cps == 2 ? 3 : 2;   // log2(groups per row per stage)
      for (int gi = qt; gi < (bm << gshift); gi += NUM_QTHREADS) {
        const int r = gi >> gshift;               // row in the tile
        const int c = (gi >> 2) & (cps - 1);      // chunk within the stage
        const int g = gi & 3;                     // group of 16 within the chunk
        const bool active = c < nc;     // the stage's second chunk may be absent
        const int row = mb * bm + r;
        const int kc = kc0 + c;
        uint32_t scale = 0;
        if (active) {
          const uint32_t row_addr = s_x(s, c) + r * 128;
          const uint4 xa = ld_shared_v4(row_addr + (((2 * g) ^ (r & 7)) << 4));
          const uint4 xb = ld_shared_v4(row_addr + (((2 * g + 1) ^ (r & 7)) << 4));
          const uint4 sa = ld_shared_v4(s_sm(s, c) + g * 32);
          const uint4 sb = ld_shared_v4(s_sm(s, c) + g * 32 + 16);
          const uint32_t xw[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
          const uint32_t sw[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
          const uint64_t codes = quantize_group(xw, sw, scale);
          if (row < p.M) {
            uint2* dst = reinterpret_cast<uint2*>(p.qact + static_cast<size_t>(row) * half_k +
                                                  kc * (BKE / 2) + g * 8);
            *dst = make_uint2(static_cast<uint32_t>(codes), static_cast<uint32_t>(codes >> 32));
          }
        }
        // Tiled scales: 512-byte block per (128 rows, 4 groups); byte
        // (row % 32) * 16 + ((row % 128) / 32) * 4 + g.  Lanes 4j..4j+3 hold
        // one row's four groups of one chunk; every lane takes part in the
        // shuffles.
        uint32_t w = scale << (8 * g);
        w |= __shfl_xor_sync(0xFFFFFFFFu, w, 1);
        w |= __shfl_xor_sync(0xFFFFFFFFu, w, 2);
        if (active && g == 0 && row < rows_pad) {
          uint32_t* sdst = reinterpret_cast<uint32_t*>(
              p.ascales_tiled + (static_cast<size_t>(row >> 7) * p.chunks + kc) * 512 +
              (row & 31) * 16 + ((row & 127) >> 5) * 4);
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
  // TMEM holds L^T: lane r, column m.  The four quantizer warps of lane
  // quarter (w % 4) read its columns in four slices of bm / 4.
  const bool is_q = warp >= 2;
  const int lq = warp & 3;
  const int slice = (warp - 2) >> 2;
  const int r_lane = lq * 32 + lane;
  const int cw = bm >> 2;  // columns per warp (multiple of 8)
  const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(lq * 32) << 16);
  if (p.split == 1) {
    if (is_q && l_ready) {
      tc_fence_after();
      for (int c0 = slice * cw; c0 < (slice + 1) * cw; c0 += 8) {
        uint32_t v[8];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
              "=r"(v[6]), "=r"(v[7])
            : "r"(lane_addr + c0)
            : "memory");
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int row = mb * bm + c0 + j;
          if (row < p.M)
            p.lowrank[static_cast<size_t>(row) * R + r_lane] =
                __float2bfloat16_rn(__uint_as_float(v[j]));
        }
      }
    }
  } else {
    // Partial sums: every quantizer warp has finished with the ring before
    // any of them overwrites it with its fp32 partial (row-major [m][r]).
    if (is_q) {
      named_bar_sync(1, NUM_QTHREADS);
      if (l_ready) {
        tc_fence_after();
        for (int c0 = slice * cw; c0 < (slice + 1) * cw; c0 += 8) {
          uint32_t v[8];
          asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
              : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                "=r"(v[6]), "=r"(v[7])
              : "r"(lane_addr + c0)
              : "memory");
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            st_shared_f32(s_ring + ((c0 + j) * PART_STRIDE + r_lane) * 4, __uint_as_float(v[j]));
        }
      }
    }
    __syncwarp();
    cluster_sync_all();
    if (is_q && !error_raised()) {
      // This rank sums its share of the bm x 32 float4 units over all ranks.
      const int units = bm * (R / 4);
      const int u0 = rank * units / p.split;
      const int u1 = (rank + 1) * units / p.split;
      for (int u = u0 + (threadIdx.x - 64); u < u1; u += NUM_QTHREADS) {
        const int m = u / (R / 4);
        const int c4 = u % (R / 4);
        const uint32_t off = s_ring + (m * PART_STRIDE + 4 * c4) * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int src = 0; src < p.split; ++src) {
          const float4 t = ld_dsmem_f4(map_to_rank(off, src));
          acc.x += t.x;
          acc.y += t.y;
          acc.z += t.z;
          acc.w += t.w;
        }
        const int row = mb * bm + m;
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
  // Role loops run in one lane of some warps: reconverge every warp first,
  // so that the block barrier waits for all of its threads.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, ncols);
  }
}

}  // namespace kq
}  // namespace svdq
