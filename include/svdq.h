/*
 * svdq.h -- C ABI of libsvdq.so, the SVDQuant W4A4 NVFP4 linear layer for
 * NVIDIA B200 (sm_100a).
 *
 * The layer (nunchaku-z-image-turbo-svdq model card, "What's stored on
 * disk", runtime formula):
 *
 *   y = scaled_mma(quant(x * smooth), qweight, ascales, wscales)
 *       * wtscale * wcscales + (x @ proj_down) @ proj_up^T + bias
 *
 * Operand layouts follow the same section's table: qweight [N, K/2] FP4
 * E2M1 nibble pack with the low nibble holding the even k; wscales
 * [K/16, N] float8_e4m3fn; wcscales [N], wtscale [1], smooth_factor [K]
 * bf16; proj_down [K, R] and proj_up [N, R] bf16 with R = 128.  The NVFP4
 * format (E2M1 elements, one e4m3 scale per 16 elements along K) is the
 * one the card's first paragraph names; the E2M1 bit layout is the one the
 * Z-Image NVFP4 blog gives in "NVFP4 技术背景".
 *
 * The path is three calls: svdq_repack_weights (once per layer),
 * svdq_quantize_act and svdq_w4a4_linear (per forward).
 *
 * Conventions for every call
 * --------------------------
 * - Types: bf16 tensors are passed as raw 16-bit patterns (uint16_t);
 *   FP4 / FP8 tensors as raw bytes.  All matrices are row-major with the
 *   last index contiguous.
 * - Memory: every tensor pointer is a DEVICE pointer on the current CUDA
 *   device, unless a parameter says otherwise.  The caller owns and
 *   allocates every buffer (sizes from the svdq_*_bytes queries); the
 *   library allocates nothing apart from a few static device words (an
 *   error word and a counter).
 * - Streams: `stream` is a cudaStream_t passed as void* (NULL = the
 *   legacy default stream).  Calls only enqueue work and return; nothing
 *   synchronizes the host except where a call says so.
 * - Alignment: tensor pointers must be 16-byte aligned (wtscale: 2 bytes).
 * - Errors: arguments are checked before anything is enqueued; a failing
 *   check returns its status and enqueues nothing.  A launch failure
 *   returns SVDQ_ERR_CUDA.  Every wait inside the kernels is bounded;
 *   a kernel that gives up records it in a device error word and returns,
 *   and svdq_check_device_error reports it as SVDQ_ERR_TIMEOUT.  While an
 *   error is recorded, the waits of later kernels give up at once, so those
 *   kernels stop at their first wait that is not already complete and their
 *   outputs are undefined until svdq_check_device_error has read and
 *   cleared the word.
 * - Device: the calls run only on compute capability 10.0 (B200, sm_100a);
 *   anything else gives SVDQ_ERR_ARCH.
 */
#ifndef SVDQ_H_
#define SVDQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum svdq_status {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,  /* null pointer, bad scale byte, bad value   */
  SVDQ_ERR_SHAPE = 2,        /* M, N < 1, K not a positive multiple of 16 */
  SVDQ_ERR_ALIGNMENT = 3,    /* pointer or leading dimension misaligned   */
  SVDQ_ERR_UNSUPPORTED = 4,  /* valid but not implemented (R, K, N limits)*/
  SVDQ_ERR_ARCH = 5,         /* current device is not sm_100              */
  SVDQ_ERR_CUDA = 6,         /* a CUDA runtime call or launch failed      */
  SVDQ_ERR_TIMEOUT = 7       /* a kernel's bounded wait ran out           */
} svdq_status;

/* Human-readable name of a status code.  Never NULL; static storage. */
const char* svdq_status_string(int status);

/* ABI version of this header (bumped on any signature change). */
#define SVDQ_ABI_VERSION 11
int svdq_abi_version(void);

/* ---- size queries (bytes the caller allocates) ------------------------ */

/* Tiled activation scales written by svdq_quantize_act for an [M, K]
 * input: ceil(M/128) * (K/64) blocks of 512 bytes.  0 on bad arguments. */
size_t svdq_ascales_tiled_bytes(int M, int K);

/* Tiled weight scales written by svdq_repack_weights for N output
 * channels: ceil(N/256)*2 * (K/64) blocks of 512 bytes.  0 on bad args.
 * Block order: 256-row tile, then K block of 64, then 128-row half, so
 * that the scales one GEMM tile needs for a run of K are contiguous. */
size_t svdq_wscales_tiled_bytes(int N, int K);

/* Low-rank activations L = x @ proj_down written by svdq_quantize_act:
 * M * R bf16 values ([M, R] row-major). */
size_t svdq_lowrank_bytes(int M, int R);

/* ---- the path ---------------------------------------------------------- */

/* One-time conversion of the on-disk weight scales into the tile order the
 * GEMM reads (model card, "What's stored on disk": wscales [K/16, N]
 * float8_e4m3fn; the card's "Why row-major" section allows a one-shot
 * load-time pack).
 *   wscales        [K/16, N] e4m3fn codes, device.
 *   N, K           output channels, input channels (K % 64 == 0).
 *   wscales_tiled  device, svdq_wscales_tiled_bytes(N, K) bytes; written
 *                  completely (padding rows get scale 0).
 * The GEMM reads scales as unsigned e4m3, so a byte with the sign bit set,
 * or a NaN code (0x7F), is rejected: the call then returns
 * SVDQ_ERR_INVALID_ARG.  To report that, this call SYNCHRONIZES `stream`.
 * The bad bytes are counted in one device-wide word per device, so
 * concurrent calls (from other host threads, on any stream) are
 * serialized by a process-wide lock held from the counter's reset to its
 * readback; each call reports only its own input. */
int svdq_repack_weights(const uint8_t* wscales, int N, int K,
                        void* wscales_tiled, void* stream);

/* Activation side of the layer (model card runtime formula): reads x once
 * and writes quant(x * smooth) and the low-rank product x @ proj_down.
 * The work is cut into tiles of 64 or 128 rows and, for small M, `split`
 * K ranges per tile handled by a thread-block cluster
 * (svdq_quantize_plan); the K ranges' fp32 partial products of L are
 * summed in K-range order on chip, so results do not depend on timing.
 *   x           [M, ldx] bf16, first K columns used; ldx >= K, ldx % 8 == 0.
 *   smooth      [K] bf16 smoothing factor (multiplied, not divided), or
 *               NULL: no smoothing (a factor of 1).
 *   proj_down   [K, R] bf16 (NULL when R == 0).
 *   R           rank: 128, or 0 for the plain NVFP4 layer without the
 *               low-rank branch (Z-Image NVFP4 blog, the comfy-kitchen
 *               deployment: weights quantized once, activations quantized
 *               dynamically); then proj_down and lowrank are not used and
 *               may be NULL.  Anything else gives SVDQ_ERR_UNSUPPORTED.
 *   qact        out, [M, K/2] bytes: E2M1 codes, low nibble = even k.
 *   ascales_tiled out, svdq_ascales_tiled_bytes(M, K) bytes: one e4m3
 *               scale per 16 k per row, scale = e4m3(amax/6), elements
 *               E2M1(v/scale); both rounded to nearest-even, saturating.
 *               Read its logical [M, K/16] form with svdq_unpack_scales.
 *   lowrank     out, [M, R] bf16: x @ proj_down accumulated in fp32 and
 *               rounded to bf16 (the raw x, not x * smooth); NULL if R == 0.
 * Limits: K % 64 == 0 (else SVDQ_ERR_UNSUPPORTED). */
int svdq_quantize_act(const uint16_t* x, int M, int K, int ldx,
                      const uint16_t* smooth, const uint16_t* proj_down, int R,
                      uint8_t* qact, void* ascales_tiled, uint16_t* lowrank,
                      void* stream);

/* Activation side of the w2 linear of a DiT feed-forward block, whose input
 * is silu(w1 x) * (w3 x): reads a = w1's output and b = w3's output, forms
 * x = silu(a) * b on chip with the same fp32 arithmetic and bf16 rounding
 * as svdq_silu_mul, and writes quant(x * smooth) and x @ proj_down exactly
 * as svdq_quantize_act does for that x (x itself is never written to
 * global memory).  This is the step just before w2 on the feed-forward
 * path of the DiT whose linears the layer replaces (w2(silu(w1 x) * w3 x),
 * as svdq_silu_mul forms it); it saves writing and re-reading x.
 *   a, b        [M, ld] bf16 with the same row stride, first K columns used;
 *               ld >= K, ld % 8 == 0.
 *   the other arguments and the statuses as svdq_quantize_act (R = 128 or
 *   0; smooth may be NULL). */
int svdq_silu_mul_quantize_act(const uint16_t* a, const uint16_t* b, int M, int K, int ld,
                               const uint16_t* smooth, const uint16_t* proj_down, int R,
                               uint8_t* qact, void* ascales_tiled, uint16_t* lowrank,
                               void* stream);

/* Block-scaled FP4 GEMM with the fused epilogue (model card runtime
 * formula):
 *   y[m, n] = acc[m, n] * wtscale * wcscales[n]
 *             + sum_r lowrank[m, r] * proj_up[n, r] + bias[n],
 *   acc[m, n] = sum_k e2m1(qact[m,k]) * sa[m,k/16] * e2m1(qweight[n,k])
 *                     * sw[k/16,n],
 * accumulated in fp32 and stored as bf16 (nearest-even).
 *   qact, ascales_tiled, lowrank  as written by svdq_quantize_act.
 *   qweight        [N, K/2] bytes (on-disk layout).
 *   wscales_tiled  as written by svdq_repack_weights.
 *   wcscales [N], wtscale [1] (read on the device), proj_up [N, R],
 *   bias [N] or NULL: bf16.
 *   proj_up_folded NULL, or svdq_fold_proj_up's output for these proj_up,
 *                  wcscales and wtscale, with no unfoldable element (the
 *                  caller checks the count).  When given, the GEMM for
 *                  M > 128 accumulates the low-rank product in the units
 *                  of the block-scaled one, in the same fp32 accumulator:
 *                    y = (acc + lowrank @ proj_up_folded^T) * wtscale
 *                        * wcscales[n] + bias,
 *                  the same value up to the bf16 rounding of the folded
 *                  factor (relative 2^-9 per element, against the 2^-9 of
 *                  proj_up's own bf16 storage), which lets that GEMM skip
 *                  the second accumulator and its drain.  Other token
 *                  counts use proj_up.  16-byte aligned.
 *   R              128, or 0 without the low-rank branch (then lowrank,
 *                  proj_up and proj_up_folded are not used and may be
 *                  NULL; the term is 0).
 *   y              out, [M, ldy] bf16, ldy >= N, ldy % 8 == 0.
 * Limits: R in {0, 128}, K % 256 == 0, N % 32 == 0 (else
 * SVDQ_ERR_UNSUPPORTED).
 * For M <= 64 the product is computed transposed (the weights as the
 * 128-row MMA operand, one CTA per 128 columns of y and, where such tiles
 * are few, the K steps split over a thread-block cluster whose fp32
 * partials are summed in a fixed rank order); the result is the same
 * sum, accumulated in fp32 in another order.  The split depends on the
 * shape, the device's SM count and the clusters it can co-schedule
 * (svdq_linear_plan), so results repeat bit for bit for the same shape on
 * the same device with the same SMs available; across devices or SM
 * counts they may differ in the last bits of the fp32 sums. */
int svdq_w4a4_linear(const uint8_t* qact, const void* ascales_tiled,
                     const uint16_t* lowrank, const uint8_t* qweight,
                     const void* wscales_tiled, const uint16_t* wcscales,
                     const uint16_t* wtscale, const uint16_t* proj_up,
                     const uint16_t* proj_up_folded, const uint16_t* bias,
                     int M, int N, int K, int R, uint16_t* y, int ldy,
                     void* stream);

/* One-time preparation of the up-projection for svdq_w4a4_linear's folded
 * low-rank form (no counterpart on the pages: it re-associates the model
 * card's runtime formula, "What's stored on disk", so that the low-rank
 * product joins the block-scaled accumulator):
 *   proj_up_folded[n, r] = bf16(proj_up[n, r] / (wtscale * wcscales[n])),
 * the product wtscale * wcscales[n] exact in float32, the quotient
 * correctly rounded to float32, then rounded to nearest-even bf16.
 *   proj_up         [N, R] bf16, device, 16-byte aligned; R % 8 == 0.
 *   wcscales [N], wtscale [1]: bf16, device.
 *   proj_up_folded  out, [N, R] bf16, device, 16-byte aligned.
 *   unfoldable      out, one uint32 in device memory: the number of
 *                   elements that cannot be folded without losing
 *                   precision (a zero or non-finite wtscale * wcscales[n],
 *                   a quotient that is infinite or nonzero below the
 *                   smallest normal bf16).  Zeroed by the call.  When it
 *                   is not 0, do not pass proj_up_folded to
 *                   svdq_w4a4_linear.
 * Enqueues a 4-byte memset and one kernel on `stream`; returns SVDQ_OK or
 * a status for bad arguments. */
int svdq_fold_proj_up(const uint16_t* proj_up, const uint16_t* wcscales,
                      const uint16_t* wtscale, int N, int R,
                      uint16_t* proj_up_folded, uint32_t* unfoldable,
                      void* stream);

/* ---- offline weight side ------------------------------------------------ */

/* Workspace svdq_quantize_weights needs for N output channels: (N + 1)
 * floats.  0 on bad arguments. */
size_t svdq_weight_workspace_bytes(int N);

/* NVFP4 encoding of a weight's residual after its low-rank part, done once
 * at load time (model card "nunchaku-z-image-turbo-svdq", first paragraph:
 * "via SVDQuant, in NVFP4 ... with rank-128 SVD residual"; the operands of
 * "What's stored on disk").  The pages do not say how the operands are
 * derived; this call implements the reading
 *   res[n, k]   = (W[n, k] - lowrank[n, k]) / smooth[k]
 *   wtscale     = bf16(A / 2688), A = max |res|        (bf16 1 if A == 0)
 *   wcscales[n] = bf16(a_n / A), a_n = max_k |res[n, k]| (0 if A == 0)
 *   per 16 k:   wscales[k/16, n] = e4m3(a_g / (6 wtscale wcscales[n])),
 *               qweight codes = E2M1(res / (wscales value * wtscale *
 *               wcscales[n])), signed zero codes where that scale is 0,
 * every float step a correctly rounded float32 operation in that order,
 * every encoding nearest-even and saturating.  lowrank is the low-rank
 * part proj_up @ proj_down^T of the caller's factors (a rank-R SVD of
 * W / smooth, see svdq.py quantize_weights), so that the layer computes
 * x @ W^T as closely as the formats allow.
 *   W          [N, K] bf16, device; K % 16 == 0.
 *   smooth     [K] bf16, device (all ones: no smoothing).
 *   lowrank    [N, K] float32, device, or NULL (no low-rank part).
 *   qweight    out, [N, K/2] bytes (low nibble = even k).
 *   wscales    out, [K/16, N] e4m3 codes (the on-disk layout).
 *   wcscales   out, [N] bf16;  wtscale out, [1] bf16.
 *   workspace  device, svdq_weight_workspace_bytes(N) bytes, caller-owned;
 *              overwritten.
 * Inputs must be finite.  Enqueues three operations on `stream` (a 4-byte
 * memset of the workspace and two kernels); returns SVDQ_OK, or a status
 * for bad arguments. */
int svdq_quantize_weights(const uint16_t* W, const uint16_t* smooth, const float* lowrank, int N,
                          int K, uint8_t* qweight, uint8_t* wscales, uint16_t* wcscales,
                          uint16_t* wtscale, void* workspace, void* stream);

/* The same encoding as svdq_quantize_weights for callers that cannot
 * allocate device memory: code that runs inside a host framework or
 * memory pool which owns all device memory and gives it no allocator, or
 * a latency-critical thread that must not call cudaMalloc (which can
 * synchronize the device).  The pages have no counterpart of this call; it
 * only changes where the scratch lives.
 * The row and global amax words live in one array that the library defines
 * in device memory for at most 32768 output channels (128 KB on every
 * device that loads the library, held until the process exits); N above
 * that gives SVDQ_ERR_UNSUPPORTED and enqueues nothing.  The call
 * allocates nothing: it enqueues a 4-byte memset of the array's global
 * word (the one word that must start at zero; the rest keeps the previous
 * call's values until overwritten) and the two kernels.  The first call on
 * a device also looks up the array's device address on that device
 * (cudaGetSymbolAddress) and keeps it; make that first call before any
 * stream capture begins.  Every call on a device shares the array, so
 * calls that overlap on the GPU (other streams, or other host threads
 * without ordering) race on it: order them, e.g. on one stream.
 * Arguments, outputs and statuses otherwise as svdq_quantize_weights. */
int svdq_quantize_weights_noalloc(const uint16_t* W, const uint16_t* smooth, const float* lowrank,
                                  int N, int K, uint8_t* qweight, uint8_t* wscales,
                                  uint16_t* wcscales, uint16_t* wtscale, void* stream);

/* ---- helpers ------------------------------------------------------------ */

/* Launch shape svdq_quantize_act uses on the current device for an [M, K]
 * input with the low-rank branch (R = 128): rows per tile (*bm, 64 or 128)
 * and the number of K ranges per tile (*split: 1, 2, 4, 8 or 16 CTAs of a
 * cluster, at least 256 k each up to 8 and at least 128 k each with 16; a
 * split always takes 64-row tiles), chosen to occupy the most SMs in one
 * wave.  The K ranges of a tile are
 * [r * (K/64) / split, (r + 1) * (K/64) / split) in units of 64 k, so they
 * differ by at most 64 k when K/64 is not a multiple of split.  The
 * summation order of L (and so its last bits) depends on this plan, which
 * depends on the device's SM count and cluster occupancy.  For inspection
 * and tests; needs a device. */
int svdq_quantize_plan(int M, int K, int* bm, int* split);

/* Launch shape svdq_w4a4_linear uses on the current device for an
 * M x N x K product (N % 32 == 0, K % 256 == 0): *kernel is
 * SVDQ_GEMM_PAIRS (M > 128: persistent 256 x 256 output tiles, each on a
 * pair of CTAs in a 2-CTA cluster sharing one tensor-core MMA, no K
 * split), SVDQ_GEMM_TOKEN_MAJOR (64 < M <= 128: persistent 128 x 256 tiles
 * on single CTAs) or SVDQ_GEMM_FEW_TOKENS (M <= 64: the transposed
 * product, one 128-column tile of y per CTA and *split CTAs of a
 * thread-block cluster per tile, each summing a range of
 * [r * (K/256) / split, (r + 1) * (K/256) / split) K steps of 256); *grid
 * is the number of CTAs launched.  For inspection and tests; needs a
 * device. */
#define SVDQ_GEMM_TOKEN_MAJOR 0
#define SVDQ_GEMM_FEW_TOKENS 1
#define SVDQ_GEMM_PAIRS 2
int svdq_linear_plan(int M, int N, int K, int* kernel, int* split, int* grid);

/* Inverse of the tile order, for tests and inspection: tiled scales of
 * `rows` rows -> out [rows, K/16] bytes, device.  `kind` says which order
 * the buffer has: SVDQ_SCALES_ACT (written by svdq_quantize_act, rows = M)
 * or SVDQ_SCALES_WEIGHT (written by svdq_repack_weights, rows = N; the
 * result is then the transpose of the on-disk wscales [K/16, N]).  Any
 * other kind gives SVDQ_ERR_INVALID_ARG. */
#define SVDQ_SCALES_ACT 0
#define SVDQ_SCALES_WEIGHT 1
int svdq_unpack_scales(const void* scales_tiled, int rows, int K, int kind,
                       uint8_t* out, void* stream);

/* out[i] = silu(a[i]) * b[i] in fp32, rounded to bf16; n elements.  Used
 * to form the w2 input of a DiT feed-forward block (w2(silu(w1 x) * w3 x)). */
int svdq_silu_mul(const uint16_t* a, const uint16_t* b, uint16_t* out,
                  size_t n, void* stream);

/* Synchronizes `stream`, then reads and clears this device's error word.
 * Returns SVDQ_OK, SVDQ_ERR_TIMEOUT (a bounded wait ran out) or
 * SVDQ_ERR_CUDA (a sticky launch / runtime error). */
int svdq_check_device_error(void* stream);

/* Sets the limit of every bounded wait inside the kernels, in nanoseconds
 * of GPU time, for the current device (default 2e9 = 2 s).  0 restores the
 * default.  A short limit is how tests make a wait run out on purpose. */
int svdq_set_wait_timeout_ns(uint64_t ns);

/* Diagnostic with no counterpart in the method: one thread waits, through
 * the same bounded wait the kernels use, on a barrier that completes only
 * if `arrive` is nonzero.  With arrive = 0 the wait runs out after the
 * current limit (svdq_set_wait_timeout_ns) and records SVDQ_ERR_TIMEOUT,
 * which the next svdq_check_device_error returns; the context stays
 * usable.  Enqueues one kernel on `stream`; returns SVDQ_OK, SVDQ_ERR_ARCH
 * or SVDQ_ERR_CUDA. */
int svdq_wait_probe(int arrive, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_H_ */
