// svdq.cu -- the C ABI of libsvdq.so (declared in include/svdq.h):
// argument checks, TMA descriptor encoding, launch configuration.  All
// arithmetic of the layer happens in the kernels included below.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "svdq.h"
#include "sm100_ptx.cuh"
#include "kq_quantize_act.cuh"
#include "kg_w4a4_linear.cuh"
#include "kg2_w4a4_linear_pair.cuh"
#include "ks_w4a4_linear_small.cuh"
#include "kr_scales.cuh"
#include "kw_quantize_weights.cuh"

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool init = false;
  bool sm100 = false;
  int num_sms = 0;
  // Max co-resident clusters of the activation kernel, by (tile height
  // 64 / 128, split 1..8); -1 = not queried yet.
  int kq_clusters[2][svdq::kq::MAX_SPLIT + 1];
  // Max co-resident clusters of the few-token GEMM by K split (1..8).
  int ks_clusters[9];
  // Max co-resident CTA pairs of the pair GEMM; -1 = not queried yet.
  int kg2_pairs = -1;
};

std::mutex g_mu;
// Held by svdq_repack_weights across its reset / kernel / readback of the
// device-wide bad-scale counter, so that concurrent repacks (other host
// threads, other streams) cannot reset or read each other's count.
std::mutex g_repack_mu;
DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Per-device one-time set-up: architecture check, SM count, kernel
// attributes.  Returns SVDQ_OK or an error status.
int device_setup(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SVDQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.init) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return SVDQ_ERR_CUDA;
    d.sm100 = (major == 10 && minor == 0);
    d.num_sms = sms;
    for (auto& row : d.kq_clusters)
      for (int& v : row) v = -1;
    for (int& v : d.ks_clusters) v = -1;
    if (d.sm100) {
      using namespace svdq;
      if (cudaFuncSetAttribute(kq::quantize_act_kernel<64, true, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kq::Shape<64, true>::SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(kq::quantize_act_kernel<128, true, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kq::Shape<128, true>::SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(kq::quantize_act_kernel<64, false, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kq::Shape<64, false>::SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(kq::quantize_act_kernel<128, false, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kq::Shape<128, false>::SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(kq::quantize_act_kernel<64, true, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kq::Shape<64, true, true>::SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(kq::quantize_act_kernel<64, false, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kq::Shape<64, false, true>::SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(kq::quantize_act_kernel<128, false, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kq::Shape<128, false, true>::SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(kg::w4a4_linear_kernel<true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kg::SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(kg::w4a4_linear_kernel<false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kg::SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(ks::w4a4_linear_small_kernel<true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               ks::SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(ks::w4a4_linear_small_kernel<false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               ks::SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(kg2::w4a4_linear_pair_kernel<kg2::LR_NONE>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kg2::SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(kg2::w4a4_linear_pair_kernel<kg2::LR_SEPARATE>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kg2::SMEM_BYTES) != cudaSuccess ||
          cudaFuncSetAttribute(kg2::w4a4_linear_pair_kernel<kg2::LR_FOLDED>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kg2::SMEM_BYTES) != cudaSuccess)
        return SVDQ_ERR_CUDA;
    }
    if (d.sm100) {
      // 16-CTA clusters of the activation kernel (non-portable size); if
      // the device refuses, the occupancy query reports none and the plan
      // keeps to 8.
      using namespace svdq;
      const void* fns[] = {reinterpret_cast<const void*>(kq::quantize_act_kernel<64, true, false>),
                           reinterpret_cast<const void*>(kq::quantize_act_kernel<128, true, false>),
                           reinterpret_cast<const void*>(kq::quantize_act_kernel<64, true, true>)};
      for (const void* fn : fns)
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
            cudaSuccess)
          cudaGetLastError();
    }
    if (g_encode == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                           &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return SVDQ_ERR_CUDA;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    d.init = true;
  }
  if (!d.sm100) return SVDQ_ERR_ARCH;
  *out = &d;
  return SVDQ_OK;
}

// 2-D tensor map over a row-major matrix: `inner` contiguous elements per
// row (row pitch `pitch_bytes`), `outer` rows; box `box_inner` x
// `box_outer`, 128-byte swizzle (or none), zero fill outside the matrix.
int make_tmap(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t inner,
              uint64_t outer, uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer,
              CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SVDQ_OK : SVDQ_ERR_CUDA;
}

// 3-D tensor map: dims {d0 (contiguous), d1, d2} with byte strides s1, s2
// for dims 1 and 2 (any order; the views used here interleave them), box
// {b0, b1, b2}, landing in shared memory as [b2][b1][b0]; 128-byte swizzle
// (or none), zero fill outside the tensor.
int make_tmap3(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t d0, uint64_t d1,
               uint64_t d2, uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2,
               CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SVDQ_OK : SVDQ_ERR_CUDA;
}

int launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

// How many clusters of `split` few-token GEMM CTAs can be resident at once
// on this device (cached).
int ks_max_clusters(DeviceInfo* d, int split) {
  std::lock_guard<std::mutex> lock(g_mu);
  int& slot = d->ks_clusters[split];
  if (slot >= 0) return slot;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(split * 256, 1, 1);
  cfg.blockDim = dim3(svdq::ks::NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = svdq::ks::SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = split;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(
          &n, reinterpret_cast<const void*>(svdq::ks::w4a4_linear_small_kernel<true>), &cfg) !=
      cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  slot = n;
  return n;
}

// K split of the few-token GEMM: the largest of 2, 4, 8 that keeps every
// CTA on its own SM in one wave (all clusters co-resident) and gives each
// CTA at least one K step of 256; else 1 (one CTA per tile, persistent).
int ks_plan(DeviceInfo* d, int n_tiles, int num_k) {
  int best = 1;
  for (int split = 2; split <= 8; split *= 2) {
    if (num_k < split || n_tiles * split > d->num_sms) break;
    if (ks_max_clusters(d, split) < n_tiles) break;
    best = split;
  }
  return best;
}

// Launch shape of the few-token GEMM for N output channels and K: the K
// split (cluster size) and the grid.  svdq_linear_plan reports the same.
void ks_shape(DeviceInfo* d, int N, int K, int* split, int* grid) {
  const int n_tiles = (N + svdq::ks::BMW - 1) / svdq::ks::BMW;
  *split = ks_plan(d, n_tiles, K / svdq::ks::BK);
  *grid = *split > 1 ? n_tiles * *split : (n_tiles < d->num_sms ? n_tiles : d->num_sms);
}

// Grid of the token-major GEMM: one persistent CTA per SM, or one per tile
// when tiles are fewer.
int kg_grid(DeviceInfo* d, int M, int N) {
  const int tiles = ((M + svdq::kg::BM - 1) / svdq::kg::BM) * ((N + svdq::kg::BN - 1) / svdq::kg::BN);
  return tiles < d->num_sms ? tiles : d->num_sms;
}

// The token-major GEMM runs on CTA pairs (256 x 256 tiles) above this many
// tokens; between the few-token limit and it, on single SMs (128 x 256).
constexpr int kPairMinM = 129;

// How many CTA pairs of the pair GEMM can be resident at once (cached).
int kg2_max_pairs(DeviceInfo* d) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (d->kg2_pairs >= 0) return d->kg2_pairs;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(2 * 256, 1, 1);
  cfg.blockDim = dim3(svdq::kg2::NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = svdq::kg2::SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(
          &n, reinterpret_cast<const void*>(
                  svdq::kg2::w4a4_linear_pair_kernel<svdq::kg2::LR_SEPARATE>),
          &cfg) !=
      cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  d->kg2_pairs = n;
  return n;
}

// Grid of the pair GEMM (CTAs, two per pair): one persistent pair per two
// SMs that the device co-schedules, or one per tile when tiles are fewer.
int kg2_grid(DeviceInfo* d, int M, int N) {
  const int tiles = ((M + svdq::kg2::BM - 1) / svdq::kg2::BM) * ((N + svdq::kg2::BN - 1) / svdq::kg2::BN);
  int pairs = kg2_max_pairs(d);
  if (pairs < 1) pairs = 1;
  return 2 * (tiles < pairs ? tiles : pairs);
}

// The GEMM for M <= 64 tokens (ks_w4a4_linear_small.cuh): weights as the
// 128-row MMA operand, one CTA per 128 weight rows and K range.  Arguments
// as checked by svdq_w4a4_linear.
int launch_small(DeviceInfo* d, const uint8_t* qact, const void* ascales_tiled,
                 const uint16_t* lowrank, const uint8_t* qweight, const void* wscales_tiled,
                 const uint16_t* wcscales, const uint16_t* wtscale, const uint16_t* proj_up,
                 const uint16_t* bias, int M, int N, int K, int R, uint16_t* y, int ldy,
                 void* stream) {
  namespace ks = svdq::ks;
  const bool lr = R != 0;
  const uint64_t kb = static_cast<uint64_t>(K) / 2;
  const uint64_t n_tiles256 = (static_cast<uint64_t>(N) + 255) / 256;
  const uint64_t kblocks = static_cast<uint64_t>(K) / 64;
  CUtensorMap tm_w, tm_x, tm_sw, tm_p, tm_l, tm_y;
  // Repacked weight scales: per 256-row tile and 64-k block, 1024 bytes
  // (rows 0..127, then 128..255), viewed as u32 {128, half, tile * kblocks}.
  if (make_tmap(&tm_w, qweight, CU_TENSOR_MAP_DATA_TYPE_UINT8, kb, N, kb, ks::BK_BYTES, ks::BMW) ||
      make_tmap(&tm_x, qact, CU_TENSOR_MAP_DATA_TYPE_UINT8, kb, M, kb, ks::BK_BYTES, ks::NT) ||
      make_tmap3(&tm_sw, wscales_tiled, CU_TENSOR_MAP_DATA_TYPE_UINT32, 128, 2,
                 n_tiles256 * kblocks, 512, 1024, 128, 1, 4, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      make_tmap(&tm_y, y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, static_cast<uint64_t>(ldy) * 2,
                ks::BMW, ks::NT, CU_TENSOR_MAP_SWIZZLE_NONE))
    return SVDQ_ERR_CUDA;
  if (!lr) {
    tm_p = tm_w;   // not read
    tm_l = tm_x;
  } else if (make_tmap(&tm_p, proj_up, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, R, N,
                       static_cast<uint64_t>(R) * 2, 64, ks::BMW) ||
             make_tmap(&tm_l, lowrank, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, R, M,
                       static_cast<uint64_t>(R) * 2, 64, ks::NT)) {
    return SVDQ_ERR_CUDA;
  }
  ks::Params p;
  p.ascales_tiled = static_cast<const uint8_t*>(ascales_tiled);
  p.wcscales = reinterpret_cast<const __nv_bfloat16*>(wcscales);
  p.wtscale = reinterpret_cast<const __nv_bfloat16*>(wtscale);
  p.bias = reinterpret_cast<const __nv_bfloat16*>(bias);
  p.y = reinterpret_cast<__nv_bfloat16*>(y);
  p.M = M;
  p.N = N;
  p.K = K;
  p.ldy = ldy;
  p.n_tiles = (N + ks::BMW - 1) / ks::BMW;
  int grid = 0;
  ks_shape(d, N, K, &p.split, &grid);
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(ks::NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = ks::SMEM_BYTES;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = p.split;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.split > 1 ? 2 : 1;
  const cudaError_t e =
      lr ? cudaLaunchKernelEx(&cfg, ks::w4a4_linear_small_kernel<true>, tm_w, tm_x, tm_sw, tm_p,
                              tm_l, tm_y, p)
         : cudaLaunchKernelEx(&cfg, ks::w4a4_linear_small_kernel<false>, tm_w, tm_x, tm_sw, tm_p,
                              tm_l, tm_y, p);
  if (e != cudaSuccess) return SVDQ_ERR_CUDA;
  return launch_status();
}

// The token-major GEMM on CTA pairs (kg2_w4a4_linear_pair.cuh), 256 x 256
// tiles; the low-rank product in the main accumulator when the folded
// up-projection is given.  Arguments as checked by svdq_w4a4_linear.
int launch_pair(DeviceInfo* d, const uint8_t* qact, const void* ascales_tiled,
                const uint16_t* lowrank, const uint8_t* qweight, const void* wscales_tiled,
                const uint16_t* wcscales, const uint16_t* wtscale, const uint16_t* proj_up,
                const uint16_t* proj_up_folded, const uint16_t* bias, int M, int N, int K, int R,
                uint16_t* y, int ldy, void* stream) {
  namespace kg2 = svdq::kg2;
  const bool lr = R != 0;
  const bool folded = lr && proj_up_folded != nullptr;
  if (folded) proj_up = proj_up_folded;
  const uint64_t kb = static_cast<uint64_t>(K) / 2;
  CUtensorMap tm_a, tm_b, tm_l, tm_p, tm_y;
  if (make_tmap(&tm_a, qact, CU_TENSOR_MAP_DATA_TYPE_UINT8, kb, M, kb, kg2::BK_BYTES,
                kg2::BM_CTA) ||
      make_tmap(&tm_b, qweight, CU_TENSOR_MAP_DATA_TYPE_UINT8, kb, N, kb, kg2::BK_BYTES,
                kg2::BN_CTA) ||
      make_tmap(&tm_y, y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, static_cast<uint64_t>(ldy) * 2,
                kg2::OUT_COLS, 32))
    return SVDQ_ERR_CUDA;
  if (!lr) {
    tm_l = tm_a;   // not read
    tm_p = tm_b;
  } else if (make_tmap(&tm_l, lowrank, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, R, M,
                       static_cast<uint64_t>(R) * 2, 64, kg2::BM_CTA) ||
             make_tmap(&tm_p, proj_up, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, R, N,
                       static_cast<uint64_t>(R) * 2, 64, kg2::BN_CTA)) {
    return SVDQ_ERR_CUDA;
  }
  kg2::Params p;
  p.ascales_tiled = static_cast<const uint8_t*>(ascales_tiled);
  p.wscales_tiled = static_cast<const uint8_t*>(wscales_tiled);
  p.wcscales = reinterpret_cast<const __nv_bfloat16*>(wcscales);
  p.wtscale = reinterpret_cast<const __nv_bfloat16*>(wtscale);
  p.bias = reinterpret_cast<const __nv_bfloat16*>(bias);
  p.M = M;
  p.N = N;
  p.K = K;
  p.m_tiles = (M + kg2::BM - 1) / kg2::BM;
  p.n_tiles = (N + kg2::BN - 1) / kg2::BN;
  p.a_row_tiles = (M + 127) / 128;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(kg2_grid(d, M, N), 1, 1);
  cfg.blockDim = dim3(kg2::NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = kg2::SMEM_BYTES;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e =
      folded ? cudaLaunchKernelEx(&cfg, kg2::w4a4_linear_pair_kernel<kg2::LR_FOLDED>, tm_a, tm_b,
                                  tm_l, tm_p, tm_y, p)
      : lr   ? cudaLaunchKernelEx(&cfg, kg2::w4a4_linear_pair_kernel<kg2::LR_SEPARATE>, tm_a,
                                  tm_b, tm_l, tm_p, tm_y, p)
             : cudaLaunchKernelEx(&cfg, kg2::w4a4_linear_pair_kernel<kg2::LR_NONE>, tm_a, tm_b,
                                  tm_l, tm_p, tm_y, p);
  if (e != cudaSuccess) return SVDQ_ERR_CUDA;
  return launch_status();
}

int grid_for(size_t work, int threads, int num_sms) {
  size_t blocks = (work + threads - 1) / threads;
  size_t cap = static_cast<size_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return static_cast<int>(blocks);
}


// How many clusters of `split` activation-kernel CTAs with tile height
// `bm` can be resident at once on this device (cached).
int kq_max_clusters(DeviceInfo* d, int bm, int split) {
  std::lock_guard<std::mutex> lock(g_mu);
  int& slot = d->kq_clusters[bm == 128 ? 1 : 0][split];
  if (slot >= 0) return slot;
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(split, 1024, 1);
  cfg.blockDim = dim3(svdq::kq::NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes =
      bm == 128 ? svdq::kq::Shape<128>::SMEM_BYTES : svdq::kq::Shape<64>::SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = split;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const void* fn =
      bm == 128 ? reinterpret_cast<const void*>(svdq::kq::quantize_act_kernel<128, true, false>)
                : reinterpret_cast<const void*>(svdq::kq::quantize_act_kernel<64, true, false>);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  slot = n;
  return n;
}

// Tile height (64 or 128 rows) and K split (a cluster of 1, 2, 4 or 8
// CTAs, each with at least two stages of 128 k) of the activation kernel:
// among the grids that run in one wave (at most one CTA per SM, every
// cluster co-resident), the one that occupies the most SMs; ties go to the
// tile height that pads M the least, then to the taller tile (less
// proj_down traffic per row), then to the smaller split.  A split takes
// 64-row tiles (the kernel's receive buffer for the partial sums fits
// beside four stages only there).
// If none fits (very large M), 128-row tiles without a split.
// A K split gives every CTA at least 256 k (4 chunks of 64) up to 8 ranks,
// and at least one 128-k stage with 16 ranks (a non-portable cluster size,
// used where few row tiles leave SMs idle).
bool kq_split_ok(int split, int chunks) {
  return split == 1 || (split <= 8 ? 4 * split <= chunks : 2 * split <= chunks);
}

void kq_plan(DeviceInfo* d, int M, int K, int* bm_out, int* split_out, bool tall_ok = true) {
  const int chunks = K / svdq::kq::BKE;
  int best_bm = tall_ok ? 128 : 64, best_split = 1, best_ctas = -1, best_pad = 0;
  for (int bm : {128, 64}) {
    if (bm == 128 && !tall_ok) continue;
    const int m_tiles = (M + bm - 1) / bm;
    const int pad = m_tiles * bm - M;
    for (int split = 1; split <= svdq::kq::MAX_SPLIT && kq_split_ok(split, chunks);
         split *= 2) {
      const int ctas = m_tiles * split;
      if (ctas > d->num_sms) break;
      if (split > 1 && bm != 64) continue;
      if (split > 1 && m_tiles > kq_max_clusters(d, bm, split)) continue;
      if (ctas > best_ctas || (ctas == best_ctas && pad < best_pad)) {
        best_ctas = ctas;
        best_bm = bm;
        best_split = split;
        best_pad = pad;
      }
    }
  }
  *bm_out = best_bm;
  *split_out = best_split;
}
// Launch shape without the low-rank branch: no cluster and no reduction, so
// the (BM, split) occupying the most SMs in one wave, ties to the tile
// height that pads M least, then the taller tile and the smaller split.
void kq_plan_plain(DeviceInfo* d, int M, int K, int* bm_out, int* split_out) {
  const int chunks = K / svdq::kq::BKE;
  int best_bm = 128, best_split = 1, best_ctas = -1, best_pad = 0;
  for (int bm : {128, 64}) {
    const int m_tiles = (M + bm - 1) / bm;
    const int pad = m_tiles * bm - M;
    for (int split = 1; split <= svdq::kq::MAX_SPLIT && kq_split_ok(split, chunks);
         split *= 2) {
      const int ctas = m_tiles * split;
      if (ctas > d->num_sms) break;
      if (ctas > best_ctas || (ctas == best_ctas && pad < best_pad)) {
        best_ctas = ctas;
        best_bm = bm;
        best_split = split;
        best_pad = pad;
      }
    }
  }
  *bm_out = best_bm;
  *split_out = best_split;
}

// One thread waits, through the same bounded wait the layer's kernels use,
// on an mbarrier that completes only if `arrive` is set.  With arrive = 0
// nothing completes it, so the wait runs out after the current limit and
// records a timeout in the device error word.
__global__ void wait_probe_kernel(int arrive) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t b = svdq::smem_u32(&bar);
  svdq::mbar_init(b, 1);
  svdq::fence_mbar_init();
  if (arrive) svdq::mbar_arrive(b);
  svdq::svdq_wait(b, 0u, 0x01u);
}

}  // namespace

extern "C" {

const char* svdq_status_string(int status) {
  switch (status) {
    case SVDQ_OK: return "SVDQ_OK";
    case SVDQ_ERR_INVALID_ARG: return "SVDQ_ERR_INVALID_ARG: null pointer or invalid value";
    case SVDQ_ERR_SHAPE: return "SVDQ_ERR_SHAPE: invalid M, N or K";
    case SVDQ_ERR_ALIGNMENT: return "SVDQ_ERR_ALIGNMENT: pointer or leading dimension misaligned";
    case SVDQ_ERR_UNSUPPORTED: return "SVDQ_ERR_UNSUPPORTED: shape outside the implemented limits";
    case SVDQ_ERR_ARCH: return "SVDQ_ERR_ARCH: current device is not sm_100 (B200)";
    case SVDQ_ERR_CUDA: return "SVDQ_ERR_CUDA: CUDA runtime or launch error";
    case SVDQ_ERR_TIMEOUT: return "SVDQ_ERR_TIMEOUT: a bounded wait inside a kernel ran out";
    default: return "SVDQ: unknown status";
  }
}

int svdq_abi_version(void) { return SVDQ_ABI_VERSION; }

size_t svdq_ascales_tiled_bytes(int M, int K) {
  if (M < 1 || K < 64 || K % 64) return 0;
  return static_cast<size_t>((M + 127) / 128) * (K / 64) * 512;
}

size_t svdq_wscales_tiled_bytes(int N, int K) {
  if (N < 1 || K < 64 || K % 64) return 0;
  return static_cast<size_t>((N + 255) / 256) * 2 * (K / 64) * 512;
}

size_t svdq_lowrank_bytes(int M, int R) {
  if (M < 1 || R < 1) return 0;
  return static_cast<size_t>(M) * R * 2;
}

int svdq_repack_weights(const uint8_t* wscales, int N, int K, void* wscales_tiled, void* stream) {
  if (!wscales || !wscales_tiled) return SVDQ_ERR_INVALID_ARG;
  if (N < 1 || K < 16 || K % 16) return SVDQ_ERR_SHAPE;
  if (K % 64) return SVDQ_ERR_UNSUPPORTED;
  if (!aligned(wscales_tiled, 16)) return SVDQ_ERR_ALIGNMENT;
  DeviceInfo* d = nullptr;
  if (int st = device_setup(&d)) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int rows_pad = (N + 255) / 256 * 256;
  const size_t words = static_cast<size_t>(rows_pad) * (K / 64);
  uint32_t zero = 0, bad = 0;
  // One repack at a time per process: the counter is shared by every call.
  std::lock_guard<std::mutex> lock(g_repack_mu);
  if (cudaMemcpyToSymbolAsync(svdq::kr::g_bad_scales, &zero, sizeof(zero), 0,
                              cudaMemcpyHostToDevice, s) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  svdq::kr::repack_weight_scales_kernel<<<grid_for(words, 256, d->num_sms), 256, 0, s>>>(
      wscales, N, K, rows_pad, static_cast<uint8_t*>(wscales_tiled));
  if (launch_status()) return SVDQ_ERR_CUDA;
  if (cudaMemcpyFromSymbolAsync(&bad, svdq::kr::g_bad_scales, sizeof(bad), 0,
                                cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  return bad ? SVDQ_ERR_INVALID_ARG : SVDQ_OK;
}

}  // extern "C"

namespace {

using svdq::kq::quantize_act_kernel;
using svdq::kq::Shape;

// One launch of the activation kernel instance <BM, LR, SILU>.
template <int BM, bool LR, bool SILU>
cudaError_t launch_kq(cudaLaunchConfig_t& cfg, const CUtensorMap& tm_x, const CUtensorMap& tm_y,
                      const CUtensorMap& tm_pd, const svdq::kq::Params& p) {
  cfg.dynamicSmemBytes = Shape<BM, LR, SILU>::SMEM_BYTES;
  return cudaLaunchKernelEx(&cfg, quantize_act_kernel<BM, LR, SILU>, tm_x, tm_y, tm_pd, p);
}

// Shared by svdq_quantize_act (b == NULL: the input is a) and
// svdq_silu_mul_quantize_act (the input is silu(a) * b, formed on chip).
int quantize_act_impl(const uint16_t* a, const uint16_t* b, int M, int K, int ld,
                      const uint16_t* smooth, const uint16_t* proj_down, int R, uint8_t* qact,
                      void* ascales_tiled, uint16_t* lowrank, void* stream) {
  const bool lr = R != 0;
  const bool silu = b != nullptr;
  if (!a || !qact || !ascales_tiled || (lr && (!proj_down || !lowrank)))
    return SVDQ_ERR_INVALID_ARG;
  if (M < 1 || K < 16 || K % 16 || ld < K) return SVDQ_ERR_SHAPE;
  if ((R != svdq::kq::R && R != 0) || K % 64) return SVDQ_ERR_UNSUPPORTED;
  if (!aligned(a, 16) || (silu && !aligned(b, 16)) || (smooth && !aligned(smooth, 16)) ||
      !aligned(qact, 16) || !aligned(ascales_tiled, 16) ||
      (lr && (!aligned(proj_down, 16) || !aligned(lowrank, 16))) || ld % 8)
    return SVDQ_ERR_ALIGNMENT;
  DeviceInfo* d = nullptr;
  if (int st = device_setup(&d)) return st;

  const int chunks = K / svdq::kq::BKE;
  int bm = 0, split = 0;
  if (lr)
    kq_plan(d, M, K, &bm, &split, /*tall_ok=*/!silu);
  else
    kq_plan_plain(d, M, K, &bm, &split);
  if (lr && split > 1 && bm != 64) return SVDQ_ERR_UNSUPPORTED;   // the plan never does this
  const int m_tiles = (M + bm - 1) / bm;

  // x (a, b) viewed as {64 k, M rows, K/64 chunks} and proj_down as {64 r,
  // K, 2 halves of R}, so that one box carries a whole 128-k stage.
  CUtensorMap tm_x, tm_y, tm_pd;
  if (make_tmap3(&tm_x, a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, svdq::kq::BKE, M, chunks,
                 static_cast<uint64_t>(ld) * 2, svdq::kq::BKE * 2, svdq::kq::BKE, bm, 2))
    return SVDQ_ERR_CUDA;
  if (!silu)
    tm_y = tm_x;   // not read
  else if (make_tmap3(&tm_y, b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, svdq::kq::BKE, M, chunks,
                      static_cast<uint64_t>(ld) * 2, svdq::kq::BKE * 2, svdq::kq::BKE, bm, 2))
    return SVDQ_ERR_CUDA;
  if (!lr)
    tm_pd = tm_x;   // not read
  else if (make_tmap3(&tm_pd, proj_down, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 64, K, 2,
                      static_cast<uint64_t>(R) * 2, 128, 64, svdq::kq::STAGE_K, 2))
    return SVDQ_ERR_CUDA;

  svdq::kq::Params p;
  p.smooth = reinterpret_cast<const __nv_bfloat16*>(smooth);
  p.qact = qact;
  p.ascales_tiled = static_cast<uint8_t*>(ascales_tiled);
  p.lowrank = reinterpret_cast<__nv_bfloat16*>(lowrank);
  p.M = M;
  p.K = K;
  p.chunks = chunks;
  p.split = split;

  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(split, m_tiles, 1);
  cfg.blockDim = dim3(svdq::kq::NUM_THREADS, 1, 1);
  cfg.stream = static_cast<cudaStream_t>(stream);
  // The K ranges of a tile form a cluster only when their L partials are
  // summed (low-rank branch).
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = split;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = lr ? 2 : 1;
  cudaError_t e;
  if (silu) {
    // (128-row tiles with the low-rank branch do not fit three stages.)
    if (lr)
      e = launch_kq<64, true, true>(cfg, tm_x, tm_y, tm_pd, p);
    else
      e = bm == 128 ? launch_kq<128, false, true>(cfg, tm_x, tm_y, tm_pd, p)
                    : launch_kq<64, false, true>(cfg, tm_x, tm_y, tm_pd, p);
  } else if (lr) {
    e = bm == 128 ? launch_kq<128, true, false>(cfg, tm_x, tm_y, tm_pd, p)
                  : launch_kq<64, true, false>(cfg, tm_x, tm_y, tm_pd, p);
  } else {
    e = bm == 128 ? launch_kq<128, false, false>(cfg, tm_x, tm_y, tm_pd, p)
                  : launch_kq<64, false, false>(cfg, tm_x, tm_y, tm_pd, p);
  }
  if (e != cudaSuccess) return SVDQ_ERR_CUDA;
  return launch_status();
}

}  // namespace

extern "C" {

int svdq_quantize_act(const uint16_t* x, int M, int K, int ldx, const uint16_t* smooth,
                      const uint16_t* proj_down, int R, uint8_t* qact, void* ascales_tiled,
                      uint16_t* lowrank, void* stream) {
  return quantize_act_impl(x, nullptr, M, K, ldx, smooth, proj_down, R, qact, ascales_tiled,
                           lowrank, stream);
}

int svdq_silu_mul_quantize_act(const uint16_t* a, const uint16_t* b, int M, int K, int ld,
                               const uint16_t* smooth, const uint16_t* proj_down, int R,
                               uint8_t* qact, void* ascales_tiled, uint16_t* lowrank,
                               void* stream) {
  if (!b) return SVDQ_ERR_INVALID_ARG;
  return quantize_act_impl(a, b, M, K, ld, smooth, proj_down, R, qact, ascales_tiled, lowrank,
                           stream);
}

int svdq_w4a4_linear(const uint8_t* qact, const void* ascales_tiled, const uint16_t* lowrank,
                     const uint8_t* qweight, const void* wscales_tiled, const uint16_t* wcscales,
                     const uint16_t* wtscale, const uint16_t* proj_up,
                     const uint16_t* proj_up_folded, const uint16_t* bias, int M, int N, int K,
                     int R, uint16_t* y, int ldy, void* stream) {
  const bool lr = R != 0;
  if (!qact || !ascales_tiled || !qweight || !wscales_tiled || !wcscales || !wtscale || !y ||
      (lr && (!lowrank || !proj_up)))
    return SVDQ_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 16 || K % 16 || ldy < N) return SVDQ_ERR_SHAPE;
  if ((R != 128 && R != 0) || K % svdq::kg::BK || N % 32) return SVDQ_ERR_UNSUPPORTED;
  if (!aligned(qact, 16) || !aligned(ascales_tiled, 16) || !aligned(qweight, 16) ||
      !aligned(wscales_tiled, 16) || !aligned(wcscales, 16) || !aligned(wtscale, 2) ||
      (lr && (!aligned(lowrank, 16) || !aligned(proj_up, 16))) ||
      (proj_up_folded && !aligned(proj_up_folded, 16)) || (bias && !aligned(bias, 16)) ||
      !aligned(y, 16) || ldy % 8)
    return SVDQ_ERR_ALIGNMENT;
  DeviceInfo* d = nullptr;
  if (int st = device_setup(&d)) return st;

  const uint64_t kb = static_cast<uint64_t>(K) / 2;
  if (M <= svdq::ks::NT)
    return launch_small(d, qact, ascales_tiled, lowrank, qweight, wscales_tiled, wcscales,
                        wtscale, proj_up, bias, M, N, K, R, y, ldy, stream);
  if (M >= kPairMinM)
    return launch_pair(d, qact, ascales_tiled, lowrank, qweight, wscales_tiled, wcscales,
                       wtscale, proj_up, proj_up_folded, bias, M, N, K, R, y, ldy, stream);
  CUtensorMap tm_a, tm_b, tm_l, tm_p, tm_y;
  if (make_tmap(&tm_a, qact, CU_TENSOR_MAP_DATA_TYPE_UINT8, kb, M, kb, svdq::kg::BK_BYTES,
                svdq::kg::BM) ||
      make_tmap(&tm_b, qweight, CU_TENSOR_MAP_DATA_TYPE_UINT8, kb, N, kb, svdq::kg::BK_BYTES,
                svdq::kg::BN) ||
      make_tmap(&tm_y, y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, static_cast<uint64_t>(ldy) * 2,
                svdq::kg::OUT_COLS, 32))
    return SVDQ_ERR_CUDA;
  if (!lr) {
    tm_l = tm_a;   // not read
    tm_p = tm_b;
  } else if (make_tmap(&tm_l, lowrank, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, R, M,
                       static_cast<uint64_t>(R) * 2, 64, svdq::kg::BM) ||
             make_tmap(&tm_p, proj_up, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, R, N,
                       static_cast<uint64_t>(R) * 2, 64, svdq::kg::BN)) {
    return SVDQ_ERR_CUDA;
  }

  svdq::kg::Params p;
  p.ascales_tiled = static_cast<const uint8_t*>(ascales_tiled);
  p.wscales_tiled = static_cast<const uint8_t*>(wscales_tiled);
  p.wcscales = reinterpret_cast<const __nv_bfloat16*>(wcscales);
  p.wtscale = reinterpret_cast<const __nv_bfloat16*>(wtscale);
  p.bias = reinterpret_cast<const __nv_bfloat16*>(bias);
  p.M = M;
  p.N = N;
  p.K = K;
  p.m_tiles = (M + svdq::kg::BM - 1) / svdq::kg::BM;
  p.n_tiles = (N + svdq::kg::BN - 1) / svdq::kg::BN;
  const int grid = kg_grid(d, M, N);
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(svdq::kg::NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = svdq::kg::SMEM_BYTES;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e =
      lr ? cudaLaunchKernelEx(&cfg, svdq::kg::w4a4_linear_kernel<true>, tm_a, tm_b, tm_l, tm_p,
                              tm_y, p)
         : cudaLaunchKernelEx(&cfg, svdq::kg::w4a4_linear_kernel<false>, tm_a, tm_b, tm_l, tm_p,
                              tm_y, p);
  if (e != cudaSuccess) return SVDQ_ERR_CUDA;
  return launch_status();
}

int svdq_linear_plan(int M, int N, int K, int* kernel, int* split, int* grid) {
  if (!kernel || !split || !grid) return SVDQ_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || K < 16 || K % 16) return SVDQ_ERR_SHAPE;
  if (K % svdq::kg::BK || N % 32) return SVDQ_ERR_UNSUPPORTED;
  DeviceInfo* d = nullptr;
  if (int st = device_setup(&d)) return st;
  if (M <= svdq::ks::NT) {
    *kernel = SVDQ_GEMM_FEW_TOKENS;
    ks_shape(d, N, K, split, grid);
  } else if (M >= kPairMinM) {
    *kernel = SVDQ_GEMM_PAIRS;
    *split = 1;
    *grid = kg2_grid(d, M, N);
  } else {
    *kernel = SVDQ_GEMM_TOKEN_MAJOR;
    *split = 1;
    *grid = kg_grid(d, M, N);
  }
  return SVDQ_OK;
}

int svdq_quantize_plan(int M, int K, int* bm, int* split) {
  if (!bm || !split) return SVDQ_ERR_INVALID_ARG;
  if (M < 1 || K < 16 || K % 16) return SVDQ_ERR_SHAPE;
  if (K % 64) return SVDQ_ERR_UNSUPPORTED;
  DeviceInfo* d = nullptr;
  if (int st = device_setup(&d)) return st;
  kq_plan(d, M, K, bm, split);
  return SVDQ_OK;
}

int svdq_unpack_scales(const void* scales_tiled, int rows, int K, int kind, uint8_t* out,
                       void* stream) {
  if (!scales_tiled || !out) return SVDQ_ERR_INVALID_ARG;
  if (kind != SVDQ_SCALES_ACT && kind != SVDQ_SCALES_WEIGHT) return SVDQ_ERR_INVALID_ARG;
  if (rows < 1 || K < 16 || K % 16) return SVDQ_ERR_SHAPE;
  if (K % 64) return SVDQ_ERR_UNSUPPORTED;
  DeviceInfo* d = nullptr;
  if (int st = device_setup(&d)) return st;
  const size_t total = static_cast<size_t>(rows) * (K / 16);
  svdq::kr::unpack_scales_kernel<<<grid_for(total, 256, d->num_sms), 256, 0,
                                   static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(scales_tiled), rows, K, kind == SVDQ_SCALES_WEIGHT ? 1 : 0,
      out);
  return launch_status();
}

int svdq_silu_mul(const uint16_t* a, const uint16_t* b, uint16_t* out, size_t n, void* stream) {
  if (!a || !b || !out) return SVDQ_ERR_INVALID_ARG;
  if (n == 0) return SVDQ_OK;
  if (!aligned(a, 16) || !aligned(b, 16) || !aligned(out, 16)) return SVDQ_ERR_ALIGNMENT;
  DeviceInfo* d = nullptr;
  if (int st = device_setup(&d)) return st;
  const size_t work = n / 8 > 8 ? n / 8 : 8;
  svdq::kr::silu_mul_kernel<<<grid_for(work, 256, d->num_sms), 256, 0,
                              static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const __nv_bfloat16*>(a), reinterpret_cast<const __nv_bfloat16*>(b),
      reinterpret_cast<__nv_bfloat16*>(out), n);
  return launch_status();
}

int svdq_fold_proj_up(const uint16_t* proj_up, const uint16_t* wcscales, const uint16_t* wtscale,
                      int N, int R, uint16_t* proj_up_folded, uint32_t* unfoldable,
                      void* stream) {
  if (!proj_up || !wcscales || !wtscale || !proj_up_folded || !unfoldable)
    return SVDQ_ERR_INVALID_ARG;
  if (N < 1 || R < 1) return SVDQ_ERR_SHAPE;
  if (R % 8) return SVDQ_ERR_UNSUPPORTED;
  if (!aligned(proj_up, 16) || !aligned(proj_up_folded, 16) || !aligned(wcscales, 2) ||
      !aligned(wtscale, 2) || !aligned(unfoldable, 4))
    return SVDQ_ERR_ALIGNMENT;
  DeviceInfo* d = nullptr;
  if (int st = device_setup(&d)) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(unfoldable, 0, sizeof(uint32_t), s) != cudaSuccess) return SVDQ_ERR_CUDA;
  const size_t work = static_cast<size_t>(N) * R / 8;
  svdq::kr::fold_proj_up_kernel<<<grid_for(work, 256, d->num_sms), 256, 0, s>>>(
      reinterpret_cast<const __nv_bfloat16*>(proj_up),
      reinterpret_cast<const __nv_bfloat16*>(wcscales),
      reinterpret_cast<const __nv_bfloat16*>(wtscale), N, R,
      reinterpret_cast<__nv_bfloat16*>(proj_up_folded), unfoldable);
  return launch_status();
}

size_t svdq_weight_workspace_bytes(int N) {
  if (N < 1) return 0;
  return (static_cast<size_t>(N) + 1) * sizeof(float);
}

int svdq_quantize_weights(const uint16_t* W, const uint16_t* smooth, const float* lowrank, int N,
                          int K, uint8_t* qweight, uint8_t* wscales, uint16_t* wcscales,
                          uint16_t* wtscale, void* workspace, void* stream) {
  if (!W || !smooth || !qweight || !wscales || !wcscales || !wtscale || !workspace)
    return SVDQ_ERR_INVALID_ARG;
  if (N < 1 || K < 16 || K % 16) return SVDQ_ERR_SHAPE;
  if (!aligned(W, 16) || !aligned(smooth, 2) || (lowrank && !aligned(lowrank, 16)) ||
      !aligned(qweight, 8) || !aligned(wcscales, 2) || !aligned(wtscale, 2) ||
      !aligned(workspace, 4))
    return SVDQ_ERR_ALIGNMENT;
  DeviceInfo* d = nullptr;
  if (int st = device_setup(&d)) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* ws = static_cast<float*>(workspace);
  if (cudaMemsetAsync(ws + N, 0, sizeof(float), s) != cudaSuccess) return SVDQ_ERR_CUDA;
  const int rows_grid = N < d->num_sms * 8 ? N : d->num_sms * 8;
  svdq::kw::weight_residual_amax_kernel<<<rows_grid, 256, 0, s>>>(
      reinterpret_cast<const __nv_bfloat16*>(W), lowrank,
      reinterpret_cast<const __nv_bfloat16*>(smooth), N, K, ws);
  if (launch_status()) return SVDQ_ERR_CUDA;
  const size_t groups = static_cast<size_t>(N) * (K / 16);
  svdq::kw::weight_quantize_kernel<<<grid_for(groups, 256, d->num_sms), 256, 0, s>>>(
      reinterpret_cast<const __nv_bfloat16*>(W), lowrank,
      reinterpret_cast<const __nv_bfloat16*>(smooth), N, K, ws, qweight, wscales,
      reinterpret_cast<__nv_bfloat16*>(wcscales), reinterpret_cast<__nv_bfloat16*>(wtscale));
  return launch_status();
}

}  // extern "C"

namespace {

// Scratch of svdq_quantize_weights_noalloc: the per-row and global amax
// words that svdq_quantize_weights keeps in its caller's workspace.  One
// copy per device that loads the library, held until the process exits.
constexpr int kNoAllocMaxRows = 32768;
static __device__ __align__(256) float g_noalloc_weight_scratch[kNoAllocMaxRows + 1];

// Device address of that array for each device, looked up once (with the
// device current) on the first call there.  In host code the array's name
// only stands for the symbol; it is not a device address.
std::mutex g_noalloc_mu;
float* g_noalloc_scratch_addr[kMaxDevices] = {};

}  // namespace

extern "C" {

int svdq_quantize_weights_noalloc(const uint16_t* W, const uint16_t* smooth, const float* lowrank,
                                  int N, int K, uint8_t* qweight, uint8_t* wscales,
                                  uint16_t* wcscales, uint16_t* wtscale, void* stream) {
  if (!W || !smooth || !qweight || !wscales || !wcscales || !wtscale) return SVDQ_ERR_INVALID_ARG;
  if (N < 1 || K < 16 || K % 16) return SVDQ_ERR_SHAPE;
  if (N > kNoAllocMaxRows) return SVDQ_ERR_UNSUPPORTED;
  if (!aligned(W, 16) || !aligned(smooth, 2) || (lowrank && !aligned(lowrank, 16)) ||
      !aligned(qweight, 8) || !aligned(wcscales, 2) || !aligned(wtscale, 2))
    return SVDQ_ERR_ALIGNMENT;
  DeviceInfo* d = nullptr;
  if (int st = device_setup(&d)) return st;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SVDQ_ERR_CUDA;
  float* ws = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_scratch_addr[dev] == nullptr) {
      void* addr = nullptr;
      if (cudaGetSymbolAddress(&addr, g_noalloc_weight_scratch) != cudaSuccess || addr == nullptr)
        return SVDQ_ERR_CUDA;
      g_noalloc_scratch_addr[dev] = static_cast<float*>(addr);
    }
    ws = g_noalloc_scratch_addr[dev];
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The global amax word must start at zero; the per-row words are written
  // before they are read.  Earlier calls' values are otherwise left in place.
  if (cudaMemsetAsync(ws + N, 0, sizeof(float), s) != cudaSuccess) return SVDQ_ERR_CUDA;
  const int rows_grid = N < d->num_sms * 8 ? N : d->num_sms * 8;
  svdq::kw::weight_residual_amax_kernel<<<rows_grid, 256, 0, s>>>(
      reinterpret_cast<const __nv_bfloat16*>(W), lowrank,
      reinterpret_cast<const __nv_bfloat16*>(smooth), N, K, ws);
  if (launch_status()) return SVDQ_ERR_CUDA;
  const size_t groups = static_cast<size_t>(N) * (K / 16);
  svdq::kw::weight_quantize_kernel<<<grid_for(groups, 256, d->num_sms), 256, 0, s>>>(
      reinterpret_cast<const __nv_bfloat16*>(W), lowrank,
      reinterpret_cast<const __nv_bfloat16*>(smooth), N, K, ws, qweight, wscales,
      reinterpret_cast<__nv_bfloat16*>(wcscales), reinterpret_cast<__nv_bfloat16*>(wtscale));
  return launch_status();
}

int svdq_check_device_error(void* stream) {
  DeviceInfo* d = nullptr;
  if (int st = device_setup(&d)) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return SVDQ_ERR_CUDA;
  uint32_t w = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&w, svdq::g_error_word, sizeof(w)) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (w) {
    if (cudaMemcpyToSymbol(svdq::g_error_word, &zero, sizeof(zero)) != cudaSuccess)
      return SVDQ_ERR_CUDA;
    return SVDQ_ERR_TIMEOUT;
  }
  return launch_status();
}

int svdq_wait_probe(int arrive, void* stream) {
  DeviceInfo* d = nullptr;
  if (int st = device_setup(&d)) return st;
  wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(arrive ? 1 : 0);
  return launch_status();
}

int svdq_set_wait_timeout_ns(uint64_t ns) {
  DeviceInfo* d = nullptr;
  if (int st = device_setup(&d)) return st;
  const uint64_t v = ns ? ns : 2000000000ull;
  if (cudaMemcpyToSymbol(svdq::g_wait_limit_ns, &v, sizeof(v)) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  return SVDQ_OK;
}

}  // extern "C"
