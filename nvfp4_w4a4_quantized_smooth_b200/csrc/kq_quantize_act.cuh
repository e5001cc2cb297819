// kq_quantize_act.cuh -- activation side of the SVDQuant W4A4 layer for
// sm_100a: reads x once and writes quant(x * smooth) (NVFP4) and the
// low-rank product L = x @ proj_down (nunchaku-z-image-turbo-svdq model
// card, "What's stored on disk", runtime formula).
//
// Quantization of each 16-element group along K (one e4m3 scale per 16 k,
// E2M1 elements, as the card's first paragraph states; rounding to
// nearest-even with saturation):
//   v = x * smooth                  exact in fp32 (bf16 x bf16, formed by
//                                   the mixed-precision FMA)
//   s = e4m3(amax|v| / 6)           quotient, then the hardware RNE /
//                                   satfinite conversion
//   q = E2M1(v / s)                 quotient, then the hardware RNE /
//                                   satfinite conversion
// The scale's quotient amax / 6 is one product with RN(1/6): a bf16 x bf16
// product has at most 16 significant bits and every e4m3 midpoint x 6 at
// most 7, so a quotient that is not exactly a midpoint lies at least 2^-16
// (relative) from it, far more than the product's error; at an exact
// midpoint t (at most 5 significant bits) the product is t (1 + 2^-25 or
// so), within half an ulp of t, so it rounds to t and the conversion sees
// the tie.
// An element's quotient v / d takes the reciprocal in two parts: r_hi =
// 1/d rounded down (__frcp_rd), r_lo = (1 - d r_hi) r_hi >= 0 (the residual
// exact by FMA), and q = RN(v r_hi + RN(v r_lo)): within about 2^-46
// (relative) of v / d, so non-midpoints round as the exact quotient does
// (the same 2^-16 argument, the midpoints of E2M1 x d having at most 7
// bits) and an exact midpoint comes out exactly.  Both parts are >= 0, so
// the sign of a zero v is kept (v r_lo and v r_hi carry it, and zeros of
// one sign add to that sign); a scale that rounds to zero gives r_hi =
// r_lo = 0 and therefore signed zero codes.  With the low-rank branch r_hi
// comes from a table of the 128 scale codes, filled once per CTA with the
// same __frcp_rd (the same values; the other instances' rings fill the
// shared memory, so they compute it per group).

// CTA work item: a tile of BM rows (64 or 128, a template parameter) and
// one of `split` ranges of K; the `split` CTAs of a tile form a
// thread-block cluster.  19 warps:
//   warps 0, 18 TMA producers (taking the stages in turn): per stage of
//               128 k, the x tile (one 3-D box:
//               2 chunks x [BM rows x 64 k] bf16, 128-byte swizzle), the
//               proj_down rows (one 3-D box: 2 halves of 64 r x [128 k x
//               128 B]) and 256 B of smooth, into a ring of stages.
//   warp 1      TMEM owner, MMA issuer.  The low-rank product is computed
//               transposed, L^T[128 x BM] += proj_down_stage^T x_tile^T:
//               tcgen05.mma kind::f16, M = 128 (= R), N = BM, K = 16;
//               A (proj_down) MN-major, B (x tile) K-major, fp32
//               accumulator in BM TMEM columns.
//   warps 2..17 quantizers: thread t owns 16-element group (t % 8) of the
//               stage's 128 k and row t / 8 (and t / 8 + 64 when BM = 128,
//               two independent groups side by side); it reads its 16
//               smooth values once per stage; writes packed codes and its
//               scale bytes; afterwards reads L^T out of TMEM.
// Without the low-rank branch (R = 0, the plain NVFP4 layer; template
// parameter LR = false) the same kernel only quantizes: no proj_down, MMA,
// TMEM or cluster, and a deeper ring of x stages.  A null smooth means no
// smoothing (a factor of 1).
// With SILU the input is x = silu(a) * b (bf16) of two [M, K] tensors, the
// w2 input of a DiT feed-forward block: each stage also brings the b tile,
// the quantizer threads form x in place of a (the same function and
// rounding as svdq_silu_mul), and the MMA waits for every quantizer warp's
// part before reading it; x itself is never written to global memory.
// With split == 1 the tile's L is rounded to bf16 and written directly.
// Otherwise (64-row tiles; split a power of two) rank o sums rows
// [o BM / split, (o + 1) BM / split) of the tile: every rank stores those
// rows of its fp32 partial into rank o's receive buffer (distributed
// shared memory stores), and after one cluster barrier each rank sums its
// rows over all ranks in rank order (deterministic) from its own shared
// memory and writes them as bf16.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace svdq {
namespace kq {

constexpr int R = 128;                 // rank (MMA M)
constexpr int BKE = 64;                // k per chunk (one 128-byte swizzled box row)
constexpr int STAGE_K = 128;           // k per stage (2 chunks)
constexpr uint32_t PD_HALF = STAGE_K * 128;        // [128 k x 64 r] bf16, 16 KB
constexpr uint32_t PD_BYTES = 2 * PD_HALF;         // 32 KB
constexpr uint32_t SM_BYTES = STAGE_K * 2;         // 256 B
constexpr int NUM_QWARPS = 16;
constexpr int NUM_QTHREADS = NUM_QWARPS * 32;
constexpr int PROD1_WARP = 2 + NUM_QWARPS;   // the second producer
constexpr int NUM_THREADS = 64 + NUM_QTHREADS + 32;
constexpr uint32_t BAR_BYTES = 256;
constexpr uint32_t SMEM_BUDGET = 227 * 1024;
constexpr int MAX_SPLIT = 16;

// LR: the layer has the low-rank branch (R = 128); without it (R = 0, the
// plain NVFP4 layer) a stage carries only x and smooth, there is no MMA,
// no TMEM and no reduction, and the ring is deeper.
// SILU: the input is silu(a) * b of two [M, K] tensors (w2's input in a
// DiT feed-forward block), formed in shared memory; a stage then also holds
// the b tile.
template <int BM, bool LR = true, bool SILU = false>
struct Shape {
  static constexpr uint32_t X_CHUNK = BM * 128;             // [BM rows x 64 k] bf16
  static constexpr uint32_t X_BYTES = 2 * X_CHUNK;
  static constexpr uint32_t Y_STAGE = SILU ? X_BYTES : 0u;  // the b tile
  static constexpr uint32_t PD_STAGE = LR ? PD_BYTES : 0u;
  // the operand stages (multiples of 1 KB, so every box stays 1024-aligned);
  // each stage's 256 B of smooth in a small ring of its own after them
  static constexpr uint32_t STAGE_BYTES = X_BYTES + Y_STAGE + PD_STAGE;
  // K split (64-row tiles with the low-rank branch): the partial rows the
  // other ranks send, [rank][row][r] fp32 (split ranks x BM / split rows)
  static constexpr uint32_t RECV_BYTES = (LR && BM == 64) ? BM * R * 4 : 0u;
  static constexpr bool CAN_SPLIT = RECV_BYTES > 0;
  // with the low-rank branch: 1/d rounded down for each of the 128 scale
  // codes (the other instances compute it per group: their rings fill the
  // shared memory)
  static constexpr uint32_t RCP_BYTES = LR ? 512u : 0u;
  static constexpr int STAGES_FIT = static_cast<int>(
      (SMEM_BUDGET - BAR_BYTES - 1024 - RECV_BYTES - RCP_BYTES) / (STAGE_BYTES + SM_BYTES));
  static constexpr int MAX_STAGES = LR ? 4 : 8;
  static constexpr int STAGES = STAGES_FIT < MAX_STAGES ? STAGES_FIT : MAX_STAGES;
  static constexpr uint32_t SMEM_BYTES =
      STAGES * (STAGE_BYTES + SM_BYTES) + RECV_BYTES + RCP_BYTES + BAR_BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = BM;                 // 64 or 128 (powers of 2)
  static constexpr int ROWS_PER_THREAD = BM / 64;           // 1 or 2
  static_assert(STAGE_BYTES % 1024 == 0, "stages stay 1024-aligned");
  static_assert(STAGES >= 3, "at least three stages");
  static_assert(SMEM_BYTES <= SMEM_BUDGET, "fits the shared memory of one SM");
  static_assert(24 * STAGES + 24 <= BAR_BYTES, "barriers fit");
};

constexpr uint32_t SITE_PROD = 0x20, SITE_MMA = 0x21, SITE_QUANT = 0x22, SITE_LFULL = 0x23;

struct Params {
  const __nv_bfloat16* smooth;
  uint8_t* qact;
  uint8_t* ascales_tiled;
  __nv_bfloat16* lowrank;
  int M, K;
  int chunks;   // K / 64
  int split;    // K ranges per row tile = cluster size
};

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// x * smooth for one word of each (two bf16 values, element 2i in the low
// half) -> packed fp32 pair: a bf16 x bf16 product is exact in fp32, and
// the mixed-precision FMA forms it straight from the 16-bit halves; the
// addend -0 keeps the product's sign when it is zero (+0 + -0 = +0,
// -0 + -0 = -0).
__device__ __forceinline__ uint64_t mul_bf16x2(uint32_t x, uint32_t s) {
  float lo, hi;
  asm("{\n\t.reg .b16 xl, xh, sl, sh;\n\t"
      "mov.b32 {xl, xh}, %2;\n\t"
      "mov.b32 {sl, sh}, %3;\n\t"
      "fma.rn.f32.bf16 %0, xl, sl, 0f80000000;\n\t"
      "fma.rn.f32.bf16 %1, xh, sh, 0f80000000;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(x), "r"(s));
  return pk(lo, hi);
}

// One 16-element group: x and the smooth values (8 bf16x2 words each) ->
// 16 E2M1 codes (element 0 in the lowest nibble) and the e4m3 scale byte.
__device__ __forceinline__ uint64_t quantize_group(const uint32_t (&xw)[8],
                                                   const uint32_t (&sw)[8],
                                                   uint32_t& scale_byte,
                                                   const float* __restrict__ rhi_tab = nullptr) {
  uint64_t v[8];
  float m8[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[i] = mul_bf16x2(xw[i], sw[i]);
    float lo, hi;
    upk(v[i], lo, hi);
    m8[i] = fmaxf(fabsf(lo), fabsf(hi));
  }
  // max is exact, so a tree gives the same amax with a short dependency chain
  const float amax = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                           fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
  const float r6 = __uint_as_float(0x3E2AAAABu);   // RN(1/6)
  const uint32_t sc = cvt_e4m3x2(amax * r6, 0.0f) & 0xFFu;
  scale_byte = sc;
  const float d = e4m3_to_f32(sc);
  float r_hi = 0.0f, r_lo = 0.0f;
  if (rhi_tab != nullptr) {
    r_hi = rhi_tab[sc];                      // 0 for a zero scale
    r_lo = fmaf(-d, r_hi, 1.0f) * r_hi;
  } else if (d > 0.0f) {
    r_hi = __frcp_rd(d);
    r_lo = fmaf(-d, r_hi, 1.0f) * r_hi;
  }
  const uint64_t rhi2 = pk(r_hi, r_hi);
  const uint64_t rlo2 = pk(r_lo, r_lo);
  float q[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint64_t q1 = fma2(v[i], rhi2, mul2(v[i], rlo2));
    upk(q1, q[2 * i], q[2 * i + 1]);
  }
  const float(&qlo)[8] = *reinterpret_cast<const float(*)[8]>(q);
  const float(&qhi)[8] = *reinterpret_cast<const float(*)[8]>(q + 8);
  return static_cast<uint64_t>(cvt_e2m1x8(qlo)) | (static_cast<uint64_t>(cvt_e2m1x8(qhi)) << 32);
}

template <int BM, bool LR, bool SILU>
__global__ void __launch_bounds__(NUM_THREADS, 1)
quantize_act_kernel(const __grid_constant__ CUtensorMap tm_x,    // x (or a) {64, M, K/64}, box {64, BM, 2}
                    const __grid_constant__ CUtensorMap tm_y,    // b {64, M, K/64} (SILU only)
                    const __grid_constant__ CUtensorMap tm_pd,   // proj_down {64, K, 2}, box {64, 128, 2}
                    const Params p) {
  using S = Shape<BM, LR, SILU>;
  constexpr int STAGES = S::STAGES;
  extern __shared__ uint8_t smem_raw[];
  // 1024-aligned, derived from the shared array so that plain accesses
  // through it stay shared-memory accesses
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t s_ring = smem_u32(smem);
  const uint32_t s_smooth = s_ring + STAGES * S::STAGE_BYTES;
  const uint32_t s_recv = s_smooth + STAGES * SM_BYTES;
  const uint32_t s_rcp = s_recv + S::RECV_BYTES;
  const uint32_t s_bar = s_rcp + S::RCP_BYTES;
  // Stage layout: x [chunk][BM rows x 128 B], (b [chunk][BM rows x 128 B],)
  // proj_down [r half][128 k x 128 B]; the stage's smooth [128 k] bf16 in
  // the smooth ring.
  auto s_x = [&](uint32_t s) { return s_ring + s * S::STAGE_BYTES; };
  auto s_y = [&](uint32_t s) { return s_ring + s * S::STAGE_BYTES + S::X_BYTES; };
  auto s_pd = [&](uint32_t s) { return s_ring + s * S::STAGE_BYTES + S::X_BYTES + S::Y_STAGE; };
  auto s_sm = [&](uint32_t s) { return s_smooth + s * SM_BYTES; };
  auto full_bar = [&](uint32_t s) { return s_bar + 8u * s; };
  auto empty_bar = [&](uint32_t s) { return s_bar + 8u * (STAGES + s); };
  // SILU: the x slot holds silu(a) * b once every quantizer warp has written
  // its part (the MMA reads it then).
  auto h_ready_bar = [&](uint32_t s) { return s_bar + 8u * (2 * STAGES + s); };
  const uint32_t lfull_bar = s_bar + 8u * (3 * STAGES);
  const uint32_t final_bar = lfull_bar + 8u;
  const uint32_t tmem_slot = lfull_bar + 16u;
  uint32_t* tmem_slot_ptr = reinterpret_cast<uint32_t*>(smem + (tmem_slot - s_ring));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int mb = blockIdx.y;
  const int rank = blockIdx.x;   // == rank in the cluster (cluster dims = (split, 1, 1))
  const int c_begin = rank * p.chunks / p.split;      // in chunks of 64 k
  const int c_end = (rank + 1) * p.chunks / p.split;
  // >= 1 chunk per CTA (host guarantees split <= chunks); the last stage of
  // a range may hold one chunk.
  const int nstages = (c_end - c_begin + 1) / 2;

  if (threadIdx.x == 0) {
    prefetch_tmap(&tm_x);
    if (SILU) prefetch_tmap(&tm_y);
    if (LR) prefetch_tmap(&tm_pd);
    for (uint32_t s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), (LR ? 1 : 0) + NUM_QWARPS);
      mbar_init(h_ready_bar(s), NUM_QWARPS);
    }
    mbar_init(lfull_bar, 1);
    mbar_init(final_bar, 1);
    fence_mbar_init();
  }
  if (LR && warp == 1) {
    tmem_alloc(tmem_slot, S::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = LR ? *reinterpret_cast<volatile uint32_t*>(tmem_slot_ptr) : 0u;
  // Set-up above overlaps the previous kernel; global memory waits for it.
  griddep_wait();
  griddep_launch_dependents();

  bool l_ready = false;   // quantizer threads: L^T accumulator readable

  if (warp == 0 || warp == PROD1_WARP) {
    if (lane == 0) {
      // ----------------------------------------------------- producers --
      // Two threads in two warps take the stages in turn (one thread's
      // copies complete about one stage per 0.3 us whatever the ring
      // depth); each waits on a stage's empty barrier at most one phase
      // ahead of its completion, as 2 <= STAGES.
      const int pid = warp == 0 ? 0 : 1;
      int i = pid;
      bool ok = true;
      for (; i < nstages; i += 2) {
        const uint32_t s = static_cast<uint32_t>(i) % STAGES;
        const uint32_t ph = (static_cast<uint32_t>(i) / STAGES) & 1u;
        if (!svdq_wait(empty_bar(s), ph ^ 1u, SITE_PROD)) {
          ok = false;
          break;
        }
        const int kc0 = c_begin + 2 * i;
        const int nc = c_end - kc0 < 2 ? 1 : 2;
        // Boxes are always delivered whole (zero fill past M and K); only
        // the smooth copy is cut to the chunks that exist.
        const uint32_t sm_bytes = p.smooth != nullptr ? nc * 128u : 0u;
        mbar_arrive_expect_tx(full_bar(s), S::X_BYTES + S::Y_STAGE + S::PD_STAGE + sm_bytes);
        tma_load_3d(s_x(s), &tm_x, 0, mb * BM, kc0, full_bar(s));
        if (SILU) tma_load_3d(s_y(s), &tm_y, 0, mb * BM, kc0, full_bar(s));
        if (LR) tma_load_3d(s_pd(s), &tm_pd, 0, kc0 * BKE, 0, full_bar(s));
        if (sm_bytes) bulk_load(s_sm(s), p.smooth + kc0 * BKE, sm_bytes, full_bar(s));
      }
      if (!ok) {
        const int n = i < STAGES ? i : STAGES;
        for (int j = 0; j < n; ++j) {
          const uint32_t jt = static_cast<uint32_t>(i - 1 - j);
          if (static_cast<int>(jt & 1u) != pid) continue;   // the other producer's stage
          drain_wait(full_bar(jt % STAGES), (jt / STAGES) & 1u, 50000000ull);
        }
      }
    }
  } else if (warp == 1) {
    if (LR && lane == 0) {
      // ---------------------------------------------------- MMA issuer --
      // L^T[r, m] += sum_k proj_down[k, r] x[m, k]: A = proj_down stage
      // (MN-major: r contiguous; the two 64-r halves 16 KB apart, 8-row k
      // groups 1 KB apart), B = x chunk (K-major, 128-byte rows).
      const uint32_t idesc = idesc_bf16_f32(R, BM, 1, 0);
      bool ok = true;
      for (int i = 0; i < nstages; ++i) {
        const uint32_t s = static_cast<uint32_t>(i) % STAGES;
        const uint32_t ph = (static_cast<uint32_t>(i) / STAGES) & 1u;
        // SILU: the MMA reads the formed silu(a) * b, after every quantizer
        // warp wrote its part (which it did after the stage landed).
        if (!svdq_wait(SILU ? h_ready_bar(s) : full_bar(s), ph, SITE_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int kc0 = c_begin + 2 * i;
        const int nk = c_end - kc0 < 2 ? 4 : 8;   // K = 16 steps in the stage
        for (int kk = 0; kk < nk; ++kk) {
          mma_f16(tmem_base,
                  smem_desc(s_pd(s) + 2048 * kk, PD_HALF, 1024, kLayoutSwizzle128B),
                  smem_desc(s_x(s) + (kk >> 2) * S::X_CHUNK + 32 * (kk & 3), 16, 1024,
                            kLayoutSwizzle128B),
                  idesc, (i | kk) != 0 ? 1u : 0u);
        }
        tc_commit(empty_bar(s));
      }
      if (ok) tc_commit(lfull_bar);
      tc_commit(final_bar);
      drain_wait(final_bar, 0, 100000000ull);
    }
  } else if (warp < PROD1_WARP) {
    // -------------------------------------------------------- quantizers --
    const int qt = threadIdx.x - 64;
    const int cg = qt & 7;          // group of 16 within the stage's 128 k
    const int c = cg >> 2;          // chunk
    const int g = cg & 3;           // group within the chunk
    const int r0 = qt >> 3;         // row r0 (and r0 + 64) of the tile
    const int half_k = p.K / 2;
    // swizzled 16-byte x chunk positions of this group (same for both rows)
    const uint32_t xo0 =
        static_cast<uint32_t>(c) * S::X_CHUNK + r0 * 128 + ((((2 * g) ^ r0) & 7) << 4);
    const uint32_t xo1 =
        static_cast<uint32_t>(c) * S::X_CHUNK + r0 * 128 + ((((2 * g + 1) ^ r0) & 7) << 4);
    const int m0 = mb * BM + r0;
    const int m1 = m0 + 64;
    uint8_t* q0_row = p.qact + static_cast<size_t>(m0) * half_k + g * 8;
    uint8_t* q1_row = p.qact + static_cast<size_t>(m1) * half_k + g * 8;
    // tiled scales: 512-byte block per (128 rows, 64 k); byte
    // (row % 32) * 16 + ((row % 128) / 32) * 4 + group
    uint8_t* sc0 = p.ascales_tiled + static_cast<size_t>(m0 >> 7) * p.chunks * 512 +
                   (m0 & 31) * 16 + ((m0 & 127) >> 5) * 4;
    uint8_t* sc1 = p.ascales_tiled + static_cast<size_t>(m1 >> 7) * p.chunks * 512 +
                   (m1 & 31) * 16 + ((m1 & 127) >> 5) * 4;
    // rows the tiled scale buffer holds (M rounded up to 128)
    const int rows_pad = (p.M + 127) & ~127;
    // The table of 1/d rounded down, filled once by the first 128
    // quantizer threads with the same operation as the per-group path.
    const float* rhi_tab = nullptr;
    if constexpr (LR) {
      float* tab = reinterpret_cast<float*>(smem + (s_rcp - s_ring));
      if (qt < 128) {
        const float d = e4m3_to_f32(static_cast<uint32_t>(qt));
        tab[qt] = d > 0.0f ? __frcp_rd(d) : 0.0f;
      }
      named_bar_sync(1, NUM_QTHREADS);
      rhi_tab = tab;
    }
    bool ok = true;
    for (int i = 0; i < nstages; ++i) {
      const uint32_t s = static_cast<uint32_t>(i) % STAGES;
      const uint32_t ph = (static_cast<uint32_t>(i) / STAGES) & 1u;
      if (!__all_sync(0xFFFFFFFFu, svdq_wait(full_bar(s), ph, SITE_QUANT))) {
        ok = false;
        break;
      }
      const int kc = c_begin + 2 * i + c;         // this thread's chunk of 64 k
      // In a range's last stage the second chunk may be absent: those lanes
      // compute nothing but still take part in the shuffles below.
      const bool active = kc < c_end;
      // This thread's inputs -> registers: smooth and x for its one or two
      // rows (bf16 pairs).
      uint32_t sw[8];
      uint32_t xv[S::ROWS_PER_THREAD][8];
      uint32_t got = 0;   // depends on every value read from the stage
      if (active) {
        if (p.smooth != nullptr) {
          const uint4 sa = *reinterpret_cast<const uint4*>(smem + (s_sm(s) - s_ring) + cg * 32);
          const uint4 sb =
              *reinterpret_cast<const uint4*>(smem + (s_sm(s) - s_ring) + cg * 32 + 16);
          got ^= sa.x ^ sa.y ^ sa.z ^ sa.w ^ sb.x ^ sb.y ^ sb.z ^ sb.w;
          sw[0] = sa.x; sw[1] = sa.y; sw[2] = sa.z; sw[3] = sa.w;
          sw[4] = sb.x; sw[5] = sb.y; sw[6] = sb.z; sw[7] = sb.w;
        } else {
          // no smoothing: v = x, i.e. a factor of 1 (exact)
#pragma unroll
          for (int j = 0; j < 8; ++j) sw[j] = 0x3F803F80u;
        }
#pragma unroll
        for (int rr = 0; rr < S::ROWS_PER_THREAD; ++rr) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const uint32_t off = (hh ? xo1 : xo0) + rr * 64 * 128;
            uint4 v4 = *reinterpret_cast<const uint4*>(smem + (s_x(s) - s_ring) + off);
            got ^= v4.x ^ v4.y ^ v4.z ^ v4.w;
            if constexpr (SILU) {
              // x = silu(a) * b, written over a in the x slot (same
              // swizzled places) for the MMA
              const uint4 b4 = lds_v4(s_y(s) + off);
              got ^= b4.x ^ b4.y ^ b4.z ^ b4.w;
              const uint32_t wa[4] = {v4.x, v4.y, v4.z, v4.w};
              const uint32_t wb[4] = {b4.x, b4.y, b4.z, b4.w};
              uint32_t wo[4];
              silu_mul_words<4>(wa, wb, wo);
              v4 = make_uint4(wo[0], wo[1], wo[2], wo[3]);
              st_shared_v4(s_x(s) + off, v4.x, v4.y, v4.z, v4.w);
            }
            xv[rr][4 * hh] = v4.x;
            xv[rr][4 * hh + 1] = v4.y;
            xv[rr][4 * hh + 2] = v4.z;
            xv[rr][4 * hh + 3] = v4.w;
          }
        }
      }
      if constexpr (SILU) {
        // x is in place for the MMA, and every lane's reads of the stage
        // have returned (the asm needs their values) and are ordered before
        // the async-proxy copy that refills it: the stage is released now,
        // so the arithmetic below overlaps that copy.
        asm volatile("" ::"r"(got) : "memory");
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(h_ready_bar(s));
          mbar_arrive(empty_bar(s));
        }
      }
      uint32_t sca = 0, scb = 0;
      if (active) {
        const uint64_t ca = quantize_group(xv[0], sw, sca, rhi_tab);
        if (m0 < p.M)
          *reinterpret_cast<uint2*>(q0_row + kc * (BKE / 2)) =
              make_uint2(static_cast<uint32_t>(ca), static_cast<uint32_t>(ca >> 32));
        if constexpr (S::ROWS_PER_THREAD == 2) {
          const uint64_t cb = quantize_group(xv[S::ROWS_PER_THREAD - 1], sw, scb, rhi_tab);
          if (m1 < p.M)
            *reinterpret_cast<uint2*>(q1_row + kc * (BKE / 2)) =
                make_uint2(static_cast<uint32_t>(cb), static_cast<uint32_t>(cb >> 32));
        }
      }
      // Each thread stores its group's scale byte (byte g of the row's
      // word for the chunk).
      if (active && m0 < rows_pad)
        sc0[static_cast<size_t>(kc) * 512 + g] = static_cast<uint8_t>(sca);
      if constexpr (S::ROWS_PER_THREAD == 2) {
        if (active && m1 < rows_pad)
          sc1[static_cast<size_t>(kc) * 512 + g] = static_cast<uint8_t>(scb);
      } else {
        // 64-row tiles may end half way through the last 128-row scale
        // block: the last tile also writes the zero scales of the rows
        // below it that the block holds.
        if (active && g == 0 && m1 >= static_cast<int>(gridDim.y) * BM && m1 < rows_pad)
          *reinterpret_cast<uint32_t*>(sc1 + static_cast<size_t>(kc) * 512) = 0u;
      }
      if constexpr (!SILU) {
        // the stage's values have all been used: release it
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(s));
      }
    }
    if (LR) l_ready = ok && __all_sync(0xFFFFFFFFu, svdq_wait(lfull_bar, 0, SITE_LFULL));
  }

  // ------------------------------------------------- low-rank readout --
  // TMEM holds L^T: lane r, column m.  The four quantizer warps of lane
  // quarter (warp % 4) read BM / 4 columns each.
  const bool is_q = warp >= 2 && warp < PROD1_WARP;
  const int lq = warp & 3;
  const int slice = (warp - 2) >> 2;
  const int r = lq * 32 + lane;
  constexpr int CW = BM / 4;     // 16 or 32 columns per warp
  const int mc = slice * CW;
  const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(lq * 32) << 16) + mc;
  if constexpr (!LR) {
    // no low-rank branch: nothing to read out
  } else if (p.split == 1) {
    if (is_q && l_ready) {
      tc_fence_after();
      uint32_t v[CW];
      if constexpr (CW == 32) {
        tmem_ld_32x32b_x32(lane_addr, v);
      } else {
        tmem_ld_32x32b_x16(lane_addr, v);
      }
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < CW; ++j) {
        const int m = mb * BM + mc + j;
        if (m < p.M) p.lowrank[static_cast<size_t>(m) * R + r] = __float2bfloat16_rn(__uint_as_float(v[j]));
      }
    }
  } else if constexpr (S::CAN_SPLIT) {
    // Rank o sums rows [o RO, (o + 1) RO) of the tile (RO = BM / split):
    // every rank stores those rows of its fp32 partial into rank o's
    // receive buffer ([rank][row - o RO][r]); rank o's buffer is used for
    // nothing else, so the stores may land while o still runs its K loop.
    const int ro = BM / p.split;
    if (is_q && l_ready) {
      tc_fence_after();
      uint32_t v[CW];
      if constexpr (CW == 32) {
        tmem_ld_32x32b_x32(lane_addr, v);
      } else {
        tmem_ld_32x32b_x16(lane_addr, v);
      }
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < CW; ++j) {
        const int m = mc + j;
        const int o = m / ro;
        const uint32_t idx = static_cast<uint32_t>((rank * ro + (m - o * ro)) * R + r);
        st_dsmem_f32(map_to_rank(s_recv + 4u * idx, static_cast<uint32_t>(o)), __uint_as_float(v[j]));
      }
    }
    // After the barrier every rank's stores into this rank's buffer are
    // visible; no rank touches another's shared memory after it, so none
    // waits for the others before it exits.
    __syncwarp();
    cluster_sync_all();
    if (is_q && !error_raised()) {
      // A unit is 4 consecutive r of one row: the float4 of each rank's
      // slice, summed in rank order.
      for (int u = threadIdx.x - 64; u < ro * (R / 4); u += NUM_QTHREADS) {
        const int mr = u / (R / 4);
        const int c4 = u % (R / 4);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int b = 0; b < p.split; ++b) {
          const float4 t = ld_shared_f4(s_recv + 4u * static_cast<uint32_t>((b * ro + mr) * R + 4 * c4));
          acc.x += t.x;
          acc.y += t.y;
          acc.z += t.z;
          acc.w += t.w;
        }
        const int row = mb * BM + rank * ro + mr;
        if (row < p.M) {
          __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
          __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
          uint2* dst = reinterpret_cast<uint2*>(p.lowrank + static_cast<size_t>(row) * R + 4 * c4);
          *dst = make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
        }
      }
    }
  }

  // ----------------------------------------------------------- teardown --
  // Role loops run in one lane of some warps: reconverge every warp first,
  // so that the block barrier waits for all of its threads.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (LR && warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, S::TMEM_COLS);
  }
}

}  // namespace kq
}  // namespace svdq
