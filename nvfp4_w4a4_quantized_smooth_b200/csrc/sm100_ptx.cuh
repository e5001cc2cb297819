// sm100_ptx.cuh -- thin inline-PTX wrappers for the sm_100a features the
// kernels use: mbarriers, TMA (bulk tensor and bulk copies), tcgen05
// (TMEM allocation, MMA, smem->TMEM copy, TMEM loads), clusters and the
// FP8 / FP4 conversions.  Every wait is bounded (see svdq_wait).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace svdq {

// ---------------------------------------------------------------- errors --
// Device error word: bit 0 = a bounded wait ran out.  Bits 8.. hold the
// site id of the first wait that gave up.  Cleared by the host.
__device__ uint32_t g_error_word = 0;
// Limit of every bounded wait, in ns of %globaltimer.
__device__ uint64_t g_wait_limit_ns = 2000000000ull;

constexpr uint32_t kErrTimeout = 1u;

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ bool error_raised() {
  return *(volatile uint32_t*)&g_error_word != 0u;
}

__device__ __forceinline__ void raise_timeout(uint32_t site) {
  atomicOr(&g_error_word, kErrTimeout | (site << 8));
}

// ------------------------------------------------------------ addresses --
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// -------------------------------------------------------------- mbarrier --
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar)
               : "memory");
}

// Raise the barrier's expected transaction bytes without an arrival (for
// copies issued ahead of the arrival that completes the phase's count).
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0u;
}

// Same test, but the thread may sleep in hardware for up to `hint_ns`
// until the phase completes, instead of spinning on the issue slots that
// the working warps of the SM need.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity,
                                                    uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0u;
}

// Bounded wait for the phase with the given parity to complete.  Returns
// false if the limit ran out (the error word is then set) or if another
// thread already raised an error.  `site` identifies the wait.
__device__ __forceinline__ bool svdq_wait(uint32_t bar, uint32_t parity, uint32_t site) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  const uint64_t limit = *(volatile uint64_t*)&g_wait_limit_ns;
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, 200000u)) return true;
    if (error_raised()) return false;
    if (globaltimer_ns() - t0 > limit) {
      raise_timeout(site);
      return false;
    }
  }
}

// Arrive on a barrier given by its shared::cluster address (this CTA's or
// the peer CTA's of a CTA pair, from mapa).  Release at CTA scope, as for a
// local barrier: the writes it publishes are tensor-memory stores ordered by
// tcgen05.wait::st and tcgen05.fence::before_thread_sync before it, and a
// cluster-scope release would fence all of this thread's memory operations
// on every call.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t bar_cluster_addr) {
  asm volatile("mbarrier.arrive.release.cta.shared::cluster.b64 _, [%0];" ::"r"(
                   bar_cluster_addr)
               : "memory");
}

// Bounded wait used on error paths only, to let copies already in flight
// land before the block exits.  Never raises; gives up after `limit_ns`.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) return;
  }
}

// ------------------------------------------------- packed fp32 pairs --
// Two fp32 values in one 64-bit register (lo in the low word) and the
// paired arithmetic sm_100 issues as one instruction.
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
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// ------------------------------------------------------------- SiLU * mul --
// h = silu(a) * b = a / (1 + exp(-a)) * b rounded ONCE to bf16 (nearest,
// ties to even, gradual underflow, overflow to inf): the input of the w2
// linear of a DiT feed-forward block, w2(silu(w1 x) * (w3 x)).  One
// definition for every kernel that forms it, so that a fused and an
// unfused path give the same bits.
//
// Slow path, fp64 (never inlined): v = P sigma(a) with P = a b exact in
// fp64 (two 8-bit significands) and sigma(a) = 1 / (1 + exp(-a)) for
// a >= 0, exp(a) / (1 + exp(a)) below (no overflow), rounded to bf16
// directly.  The exact product is never a bf16 midpoint for a, b != 0 (it
// is transcendental), but the fp64 value can land on one, and then the
// side is decided from the exact value's expansion:
//   |a| < 2^-20: silu(a) b = P (1/2 + a/4 + O(a^3)), so the fp64 value is
//                P / 2 = m and the exact one is beyond m iff a > 0;
//   a > 0:       |v| = |P| - c with c = |P| exp(-a) / (1 + exp(-a)) > 0 and
//                |P| - m exact, so it is beyond m iff |P| - m > c (for
//                a > 37 the fp64 value is P itself and c decides);
//   a < 0:       a coincidence of fp64 rounding; nearest-even is kept.
__device__ __noinline__ uint32_t silu_mul_bf16_f64(float af, float bf) {
  const double a = af, b = bf;
  const double P = a * b;
  const double t = exp(-fabs(a));
  const double v = P * (a >= 0.0 ? 1.0 / (1.0 + t) : t / (1.0 + t));
  const double av = fabs(v);
  if (av == 0.0 || isinf(v)) return __bfloat16_as_ushort(__double2bfloat16(v));
  // spacing of bf16 values at |v|: 2^(e - 7) for 2^e <= |v| (normal), 2^-133 below 2^-126
  const int e = ilogb(av);
  const double q = e < -126 ? 0x1p-133 : ldexp(1.0, e - 7);
  const double x = av / q;   // a power-of-two scaling: exact
  if (x - floor(x) != 0.5 || (a < 0.0 && fabs(a) >= 0x1p-20))
    return __bfloat16_as_ushort(__double2bfloat16(v));
  // v is exactly the midpoint m = |v| between floor(x) q and floor(x) q + q
  const bool away = fabs(a) < 0x1p-20 ? a > 0.0 : (fabs(P) - av) > fabs(P) * (t / (1.0 + t));
  const double r = (floor(x) + (away ? 1.0 : 0.0)) * q;
  return __bfloat16_as_ushort(__double2bfloat16(v < 0.0 ? -r : r));
}

__device__ __forceinline__ float ex2_approx_ftz(float y) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(y));
  return r;
}
__device__ __forceinline__ float rcp_approx_ftz(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Fast path, fp32, one word of two elements (a, b: bf16 pairs, element 0
// in the low half).  t = exp(-|a|) is 2^y with y = -|a| log2(e) split into
// y_hi = fl(-|a| L) and the remainder y_lo (exact by FMA, plus
// -|a| (log2 e - L)) -- the argument reduction of Cody and Waite ("Software
// Manual for the Elementary Functions", 1980) -- so t = ex2(y_hi)
// (1 + y_lo ln 2) with |y_lo| < 2^-16; then silu(a) b = a b / (1 + t) for
// a >= 0 and (a t) b / (1 + t) below, with the reciprocal of 1 + t in
// [1, 2].  With ex2.approx and rcp.approx within 2^-21 and 2^-22
// (relative) and the float roundings, the result is within 2^-20 of the
// exact product, under 16 float ulps, so its nearest-even rounding to bf16
// is that of the exact value unless the float lies within 64 ulps of a bf16
// midpoint (low 16 bits within 64 of 0x8000).  Inputs outside the range of
// that bound show up in the result and are sent to the fp64 path too: for
// |a| > 87 t flushes to zero, which for a < 0 gives a zero product and for
// a > 0 the product a b itself (exact; only a midpoint, caught by the
// window, can round differently from the exact value just inside it); a
// zero, subnormal or infinite bf16 result (zeros, subnormal operands,
// overflow of a b) is sent over as well.  Returns the bf16 pair; bits 0 and
// 1 of `slow` flag the elements the fp64 path must decide.
__device__ __forceinline__ uint32_t silu_mul_fast2(uint32_t a, uint32_t b, uint32_t& slow) {
  const uint64_t kNegL = pk(-1.44269502f, -1.44269502f);     // -log2(e) rounded to float
  const uint64_t kL = pk(1.44269502f, 1.44269502f);
  const uint64_t kLlo = pk(1.92596299e-08f, 1.92596299e-08f); // log2(e) - 1.44269502f
  const uint64_t kNegLn2 = pk(-0.693147182f, -0.693147182f);
  const uint64_t kOne = pk(1.0f, 1.0f);
  const uint64_t av = pk(__uint_as_float(a << 16), __uint_as_float(a & 0xFFFF0000u));
  const uint64_t bv = pk(__uint_as_float(b << 16), __uint_as_float(b & 0xFFFF0000u));
  const uint64_t abs_a = pk(__uint_as_float((a << 17) >> 1), __uint_as_float((a & 0x7FFF0000u)));
  const uint64_t yhi = mul2(abs_a, kNegL);                    // fl(-|a| L)
  const uint64_t r1 = fma2(abs_a, kL, yhi);                   // |a| L + y_hi, exact
  const uint64_t r2 = fma2(abs_a, kLlo, r1);                  // -y_lo
  const uint64_t corr = fma2(r2, kNegLn2, kOne);              // 1 + y_lo ln 2
  float y0, y1;
  upk(yhi, y0, y1);
  const uint64_t t = mul2(pk(ex2_approx_ftz(y0), ex2_approx_ftz(y1)), corr);
  float d0, d1;
  upk(add2(t, kOne), d0, d1);
  const uint64_t rcp = pk(rcp_approx_ftz(d0), rcp_approx_ftz(d1));
  const uint64_t P = mul2(av, bv);                            // a b, exact
  const uint64_t Q = mul2(mul2(av, t), bv);                   // (a t) b
  float p0, p1, q0, q1;
  upk(P, p0, p1);
  upk(Q, q0, q1);
  const uint64_t num = pk((a & 0x8000u) ? q0 : p0, (a & 0x80000000u) ? q1 : p1);
  float v0, v1;
  upk(mul2(num, rcp), v0, v1);
  uint32_t h;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(h) : "f"(v1), "f"(v0));
  const uint32_t u0 = __float_as_uint(v0), u1 = __float_as_uint(v1);
  // result exponent field 0 (zero, subnormal) or 0xFF (inf) in either half
  const uint32_t e = h & 0x7F807F80u;
  const uint32_t zero_sub = ~((e | 0x80008000u) - 0x00800080u) & 0x80008000u;
  const uint32_t inf = (e + 0x00800080u) & 0x80008000u;
  const uint32_t bad = zero_sub | inf;
  slow = (((u0 & 0xFFFFu) - 0x7FC0u) <= 0x80u || (bad & 0x8000u) ? 1u : 0u) |
         (((u1 & 0xFFFFu) - 0x7FC0u) <= 0x80u || (bad & 0x80000000u) ? 2u : 0u);
  return h;
}

// One element, either path.
__device__ __forceinline__ uint32_t silu_mul_bf16_rn(float a, float b) {
  uint32_t slow;
  const uint32_t h = silu_mul_fast2(__float_as_uint(a) >> 16, __float_as_uint(b) >> 16, slow);
  return (slow & 1u) ? silu_mul_bf16_f64(a, b) : (h & 0xFFFFu);
}

// NW words of bf16 pairs (element 0 in the low half): out = silu(a) * b,
// bf16 pairs.  The fast path runs on every element first; the few it cannot
// decide (about one in 500) are redone on the fp64 path afterwards, outside
// the main loop, so that the common path stays a straight line of float
// arithmetic.
template <int NW>
__device__ __forceinline__ void silu_mul_words(const uint32_t (&a)[NW], const uint32_t (&b)[NW],
                                               uint32_t (&out)[NW]) {
  uint32_t need = 0;
#pragma unroll
  for (int i = 0; i < NW; ++i) {
    uint32_t sl;
    out[i] = silu_mul_fast2(a[i], b[i], sl);
    need |= sl << (2 * i);
  }
  if (need != 0u) {
#pragma unroll
    for (int i = 0; i < NW; ++i) {
      if (need & (1u << (2 * i)))
        out[i] = (out[i] & 0xFFFF0000u) |
                 silu_mul_bf16_f64(__uint_as_float(a[i] << 16), __uint_as_float(b[i] << 16));
      if (need & (2u << (2 * i)))
        out[i] = (out[i] & 0xFFFFu) | (silu_mul_bf16_f64(__uint_as_float(a[i] & 0xFFFF0000u),
                                                         __uint_as_float(b[i] & 0xFFFF0000u))
                                       << 16);
    }
  }
}

// ------------------------------------------------- dependent launches --
// A kernel launched with programmatic stream serialization may start while
// the previous kernel in the stream is still running.  griddep_wait blocks
// until that kernel has completed and its memory operations are visible;
// every thread calls it before it touches memory that kernel may write.
// The kernels of this library that let their dependents start early (the
// activation kernel and the GEMMs) never write the weights, so a GEMM may
// issue the copies of its weight operands before its wait.  (No-op for a
// kernel launched without the attribute.)
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Lets the next kernel in the stream begin launching (its blocks run their
// set-up and then wait in griddep_wait).
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------- TMA --
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 2-D tiled bulk tensor load global -> shared (this CTA), completion on bar.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int32_t x, int32_t y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// 3-D tiled bulk tensor load global -> shared (this CTA), completion on bar.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* tmap, int32_t x, int32_t y,
                                            int32_t z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

// 2-D tiled bulk tensor load into this CTA's shared memory whose completion
// is signalled on a barrier of either CTA of the CTA pair (`bar` a
// shared::cluster address): the operand loads of a cta_group::2 MMA.  No
// multicast: each CTA loads its own half from this GPU's memory.
__device__ __forceinline__ void tma_load_2d_cg2(uint32_t dst, const void* tmap, int32_t x,
                                                int32_t y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::"
      "bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// 2-D tiled bulk tensor store shared (this CTA) -> global, tracked by the
// issuing thread's bulk async-group.  Elements outside the tensor map's
// extent are not written.
__device__ __forceinline__ void tma_store_2d(const void* tmap, uint32_t src, int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
          reinterpret_cast<uint64_t>(tmap)),
      "r"(x), "r"(y), "r"(src)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until every committed store of this thread has finished READING its
// shared-memory source (the buffer may then be rewritten).
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}
// 8-byte store to global memory (the address must be 8-byte aligned).
__device__ __forceinline__ void st_global_v2(void* ptr, uint32_t a, uint32_t b) {
  asm volatile("st.global.v2.b32 [%0], {%1, %2};" ::"l"(ptr), "r"(a), "r"(b) : "memory");
}
__device__ __forceinline__ void st_shared_u16(uint32_t addr, uint16_t v) {
  asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}
// Wait until every committed store of this thread has completed.
__device__ __forceinline__ void bulk_wait_group0() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Contiguous bulk copy global -> shared; 16-byte aligned, size % 16 == 0.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// --------------------------------------------------------------- tcgen05 --
// TMEM allocation: executed by one whole warp; the base address is written
// to shared memory at `dst`.
__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// D(tmem) (+)= A(smem) * B(smem), bf16/fp16 inputs (kind::f16).
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D(tmem) (+)= (A * SFA) (B * SFB): FP4 E2M1 operands, ue4m3 scales, one
// scale per 16 K elements (kind::mxf4nvf4, block16), K = 64 per call.
__device__ __forceinline__ void mma_nvfp4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], "
      "p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// ---- CTA pairs (cta_group::2): one MMA over both CTAs' operands ----------
// TMEM allocation / release for the pair: one warp of EACH CTA executes it;
// both CTAs get the same column range.
__device__ __forceinline__ void tmem_alloc_cg2(uint32_t dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_cg2() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_cg2(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// Arrive on the barrier at this offset in every CTA of `cta_mask` once all
// pair MMAs this thread issued so far have completed.
__device__ __forceinline__ void tc_commit_cg2_mc(uint32_t bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
      "[%0], %1;" ::"r"(bar),
      "h"(cta_mask)
      : "memory");
}
// Same, arriving on one barrier of this CTA.
__device__ __forceinline__ void tc_commit_cg2(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}
// Pair MMA, issued by the even CTA: M = 256 rows, rows [0, 128) from this
// CTA's A and into its TMEM, [128, 256) from the odd CTA's; each CTA holds
// half of B's N rows.  Descriptors and TMEM addresses are the same in both.
__device__ __forceinline__ void mma_nvfp4_cg2(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t sfa_tmem,
                                              uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], "
      "p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}
__device__ __forceinline__ void mma_f16_cg2(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Load 32 consecutive 32-bit TMEM columns of this warp's lane quarter: each
// thread gets its own lane's 32 values.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
// Same, 16 consecutive columns.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// Registers -> TMEM: 32 lanes (this warp's lane quarter) x 8 consecutive
// 32-bit columns; lane i stores v[0..7].  Warp-collective.
__device__ __forceinline__ void tmem_st_32x32b_x8(uint32_t taddr, const uint32_t (&v)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void ld_shared_v4(uint32_t addr, uint32_t& a, uint32_t& b, uint32_t& c,
                                             uint32_t& d) {
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
               : "r"(addr)
               : "memory");
}

// ------------------------------------------------------------ descriptors --
// Shared-memory matrix descriptor (sm_100 format): start address, leading
// and stride byte offsets (all in 16-byte units), version 1, layout type.
constexpr uint64_t kLayoutSwizzleNone = 0;
constexpr uint64_t kLayoutSwizzle128B = 2;

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes,
                                              uint32_t sbo_bytes, uint64_t layout) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;  // descriptor version for sm_100
  d |= layout << 61;
  return d;
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 D.
// a_mn_major / b_mn_major: 0 = K-major, 1 = MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(uint32_t M, uint32_t N, uint32_t a_mn_major,
                                                      uint32_t b_mn_major) {
  return (1u << 4)                  // D format: f32
         | (1u << 7)                // A format: bf16
         | (1u << 10)               // B format: bf16
         | (a_mn_major << 15) | (b_mn_major << 16) |
         ((N >> 3) << 17)           // N / 8
         | ((M >> 4) << 24);        // M / 16
}

// Instruction descriptor, kind::mxf4nvf4: E2M1 A/B (K-major), ue4m3 scales,
// scale-factor ids 0, dense K = 64.
__host__ __device__ constexpr uint32_t idesc_nvfp4(uint32_t M, uint32_t N) {
  return (1u << 7)                  // A format: E2M1
         | (1u << 10)               // B format: E2M1
         | ((N >> 3) << 17)         // N / 8
         | (0u << 23)               // scale format: ue4m3
         | ((M >> 4) << 24);        // M / 16
}

// --------------------------------------------------------------- cluster --
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void st_shared_f32(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
// Store to a shared-memory address of this cluster (mapa), possibly another
// CTA's; made visible to that CTA by a later cluster barrier.
__device__ __forceinline__ void st_dsmem_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ float4 ld_shared_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ float4 ld_dsmem_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// Named barrier over `nthreads` threads (multiple of 32).
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ----------------------------------------------------------- conversions --
// Two fp32 -> two e4m3 (nearest-even, saturating to +-448): `lo` goes to
// the low byte of the result.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// e4m3 byte (low byte of `b`) -> fp32, exactly (through f16, which holds
// every e4m3 value).
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
  uint32_t h2;
  uint16_t in = static_cast<uint16_t>(b & 0xFFu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

// Eight fp32 -> eight E2M1 codes (nearest-even, saturating to +-6), packed
// into 32 bits with element 0 in the lowest nibble.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&v)[8]) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return r;
}

}  // namespace svdq
