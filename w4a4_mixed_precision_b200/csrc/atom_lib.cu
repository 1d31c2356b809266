// atom_lib.cu -- the C ABI declared in include/atom.h: host-side argument
// checks, tensor-map encoding and kernel launches. No allocation, no host
// synchronisation on any compute entry point.
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "atom.h"
#include "gemm.cuh"
#include "gemm_small.cuh"
#include "ptx.cuh"
#include "quant.cuh"
#include "kv.cuh"
#include "probe.cuh"
#include "tiled.cuh"
#include "w8a8.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr int64_t kMaxK = atomk::kQuantMaxK;  // gather offsets are uint16 in shared memory

// Per-device launch facts, filled once. The flags that publish a field read
// outside g_mutex are atomics (written with release after the field, read with
// acquire); everything else is only touched under g_mutex.
struct DeviceState {
  std::atomic<bool> probed{false};   // publishes supported, sm_count, smem_optin
  bool supported = false;
  int sm_count = 0;
  int smem_optin = 0;
  std::atomic<bool> gemm_attr[6] = {};   // by GEMM kernel: mode (Y, partials, quantized Y) + 3 * W4A8
  int gemm_clusters[6] = {};     // co-resident CTA pairs of the GEMM kernel
  bool small_attr = false;       // shared-memory limit set for the small-M GEMM kernels
  bool w8a8_attr = false;
  int w8a8_clusters = 0;          // co-resident CTA pairs of the W8A8 kernel
  uint32_t quant_smem_set = 0;
  std::atomic<void *> noalloc_scratch{nullptr};  // device address of g_noalloc_scratch here
  std::atomic<uint32_t> quant_calls{0};   // picks each quantizer call's row-counter slot
};

DeviceState g_devices[kMaxDevices];
std::mutex g_mutex;

atom_status_t current_device(DeviceState **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATOM_ERR_CUDA;
  DeviceState &d = g_devices[dev];
  if (!d.probed.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!d.probed.load(std::memory_order_relaxed)) {
      int major = 0, minor = 0;
      if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
              cudaSuccess)
        return ATOM_ERR_CUDA;
      d.supported = (major == 10 && minor == 0);  // built for sm_100a only
      d.probed.store(true, std::memory_order_release);
    }
  }
  if (!d.supported) return ATOM_ERR_UNSUPPORTED;
  *out = &d;
  return ATOM_OK;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

atom_status_t check_method_params(int64_t K, int32_t n_outlier, int32_t group) {
  if (group != 128 || n_outlier != 128) return ATOM_ERR_UNSUPPORTED;
  if (K % 128 != 0 || K < 256 || K > kMaxK) return ATOM_ERR_SHAPE;
  return ATOM_OK;
}

// ---------------------------------------------------------------- quantizer

atom_status_t launch_quant(const void *x, int64_t rows, int64_t K, int64_t ld,
                           const int32_t *idx, int32_t n_outlier, int32_t group, uint8_t *q4,
                           int8_t *q8, float *scales, atom_stream_t stream, bool a8 = false) {
  if (rows < 0 || ld < 0) return ATOM_ERR_INVALID_ARG;
  atom_status_t st = check_method_params(K, n_outlier, group);
  if (st != ATOM_OK) return st;
  if (ld < K || ld % 8 != 0) return ATOM_ERR_SHAPE;
  if (rows == 0) return ATOM_OK;
  if (!x || !idx || (!q4 && !a8) || !q8 || !scales) return ATOM_ERR_INVALID_ARG;
  if (!aligned(x, 16) || (!a8 && !aligned(q4, 16)) || !aligned(q8, 16) || !aligned(scales, 4) ||
      !aligned(idx, 4))
    return ATOM_ERR_ALIGN;

  DeviceState *dev = nullptr;
  if ((st = current_device(&dev)) != ATOM_OK) return st;

  // One CTA per SM. Its crews share the rows; each crew has its own ring of
  // 2-4 rows in flight. As many rows as shared memory holds beside the gather
  // table (at most 12), in as many crews (up to 3) as leave each ring >= 2.
  const int64_t fixed = atomk::quant_layout(static_cast<int>(K), 0).total;
  const int64_t row_bytes = 2 * K;
  int64_t fit = (dev->smem_optin - fixed) / row_bytes;
  if (fit > atomk::kQuantMaxStages) fit = atomk::kQuantMaxStages;
  if (fit < 2) return ATOM_ERR_SHAPE;
  const int64_t crews = fit / 2 < atomk::kQuantCrews ? fit / 2 : atomk::kQuantCrews;
  const int64_t stages = fit / crews < 4 ? fit / crews : 4;
  const atomk::QuantLayout L =
      atomk::quant_layout(static_cast<int>(K), static_cast<int>(stages * crews));
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (dev->quant_smem_set < L.total) {
      if (cudaFuncSetAttribute(atomk::reorder_quant_kernel,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(L.total)) != cudaSuccess)
        return ATOM_ERR_CUDA;
      dev->quant_smem_set = L.total;
    }
  }
  const int grid = static_cast<int>(rows < dev->sm_count ? rows : dev->sm_count);
  // The launch's row counter: slots go round in call order, so launches that
  // run at the same time use different slots unless kQuantSlots or more
  // quantizer calls of this device are in flight at once.
  const int slot = static_cast<int>(dev->quant_calls.fetch_add(1, std::memory_order_relaxed) %
                                    static_cast<uint32_t>(atomk::kQuantSlots));
  // programmatic dependent launch: the kernel's set-up may overlap the end of
  // the previous kernel in the stream (it waits for that kernel before it
  // touches its inputs or outputs)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(atomk::kQuantThreads, 1, 1);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  const cudaError_t err = cudaLaunchKernelEx(
      &cfg, atomk::reorder_quant_kernel, static_cast<const __half *>(x), rows, static_cast<int>(K),
      ld, idx, q4, q8, scales, static_cast<int>(stages), static_cast<int>(crews), a8 ? 1 : 0, slot);
  return err == cudaSuccess ? ATOM_OK : ATOM_ERR_CUDA;
}

// ---------------------------------------------------------------- GEMM

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Encoded tensor maps, by their encoding arguments. A map depends only on the
// address, sizes, strides, box and swizzle it is built from (not on the data
// or on the device's state), so an identical request can reuse it; serving
// loops call the same GEMM on the same buffers again and again, and encoding
// the five to seven maps of a call on the host costs more than a decode GEMM
// takes on the GPU. Direct-mapped, guarded by g_map_mutex.
struct MapKey {
  const void *base;
  uint64_t cols, rows, stride;
  uint32_t box_cols, box_rows;
  int dtype, swizzle;
  bool operator==(const MapKey &o) const {
    return base == o.base && cols == o.cols && rows == o.rows && stride == o.stride &&
           box_cols == o.box_cols && box_rows == o.box_rows && dtype == o.dtype &&
           swizzle == o.swizzle;
  }
};
struct MapEntry {
  bool valid = false;
  MapKey key;
  CUtensorMap map;
};
constexpr int kMapCacheSize = 256;
MapEntry g_map_cache[kMapCacheSize];
std::mutex g_map_mutex;

size_t map_slot(const MapKey &k) {
  uint64_t h = reinterpret_cast<uintptr_t>(k.base) * 0x9E3779B97F4A7C15ull;
  for (uint64_t v : {k.cols, k.rows, k.stride, static_cast<uint64_t>(k.box_cols),
                     static_cast<uint64_t>(k.box_rows), static_cast<uint64_t>(k.dtype),
                     static_cast<uint64_t>(k.swizzle)})
    h = (h ^ v) * 0x100000001B3ull;
  return static_cast<size_t>(h >> 32) % kMapCacheSize;
}

// 2-D tensor map over a row-major matrix of `rows` rows, `cols` elements per
// row and a row stride of `stride_bytes`, copied in boxes of box_rows x box_cols;
// reads past the matrix edge fill with zeros.
bool encode_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, uint64_t cols,
               uint64_t rows, uint64_t stride_bytes, uint32_t box_cols, uint32_t box_rows,
               CUtensorMapSwizzle swizzle) {
  const MapKey key{base, cols, rows, stride_bytes, box_cols, box_rows, static_cast<int>(dtype),
                   static_cast<int>(swizzle)};
  const size_t slot = map_slot(key);
  {
    std::lock_guard<std::mutex> lock(g_map_mutex);
    if (g_map_cache[slot].valid && g_map_cache[slot].key == key) {
      *map = g_map_cache[slot].map;
      return true;
    }
  }
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {stride_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  if (fn(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  std::lock_guard<std::mutex> lock(g_map_mutex);
  g_map_cache[slot].key = key;
  g_map_cache[slot].map = *map;
  g_map_cache[slot].valid = true;
  return true;
}

// K splits for a GEMM whose output tiles would leave most CTA pairs idle
// (small M: decode): as many as fill the pairs, at least kMinGroupsPerSplit
// groups of 128 each. 1 = no split.
constexpr int kMinGroupsPerSplit = 4;
constexpr int kMaxSplits = 16;

int gemm_splits(int64_t M, int64_t N, int64_t K, int pairs) {
  using namespace atomk::gemm_cfg;
  const int64_t tiles = ((M + kPairM - 1) / kPairM) * ((N + BN - 1) / BN);
  if (tiles <= 0 || 2 * tiles >= pairs) return 1;
  int64_t s = pairs / tiles;
  const int64_t by_k = (K / 128) / kMinGroupsPerSplit;
  if (s > by_k) s = by_k;
  if (s > kMaxSplits) s = kMaxSplits;
  return s < 2 ? 1 : static_cast<int>(s);
}

// Epilogues of the W4A4 GEMM kernel.
enum GemmMode { kModeY = 0, kModePartials = 1, kModeQuantY = 2 };

atom_status_t gemm_pairs(DeviceState *dev, int mode, int *pairs);   // mode + 3 for W4A8

// K splits of the small-M GEMM (gemm_small.cuh): one 128-row weight tile per
// CTA, as many K ranges (of at least 2 groups, at most 8: they form one
// thread-block cluster of portable size) as keep every SM busy without a
// second wave. 1 = no split.
constexpr int kMaxSmallSplits = atomk::small_cfg::kMaxSplits;
int small_splits(int64_t N, int64_t K, int sms) {
  const int64_t n_tiles = (N + atomk::small_cfg::BW - 1) / atomk::small_cfg::BW;
  if (n_tiles <= 0 || n_tiles >= sms) return 1;
  int64_t s = sms / n_tiles;
  const int64_t by_k = (K / 128) / 2;
  if (s > by_k) s = by_k;
  if (s > kMaxSmallSplits) s = kMaxSmallSplits;
  return s < 2 ? 1 : static_cast<int>(s);
}

// The GEMM for M <= 64 tokens: weights on the MMA's M side (see gemm_small.cuh).
// With `partials` (the debug entry point) K is never split.
atom_status_t launch_gemm_small(DeviceState *dev, const uint8_t *qa4, const int8_t *qa8,
                                const float *sa, const uint8_t *qw4, const int8_t *qw8,
                                const float *sw, void *y, int32_t *partials, int64_t M,
                                int64_t N, int64_t K, void *workspace, size_t workspace_bytes,
                                atom_stream_t stream, bool w_tiled) {
  using namespace atomk::small_cfg;
  const int64_t q4_row = (K - 128) / 2;
  int splits = partials != nullptr ? 1 : small_splits(N, K, dev->sm_count);
  if (splits > 1 && (workspace == nullptr ||
                     workspace_bytes < static_cast<size_t>(splits) * M * N * sizeof(float) ||
                     !aligned(workspace, 16)))
    splits = 1;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!dev->small_attr) {
      const void *fns[6] = {
          reinterpret_cast<const void *>(atomk::w4a4_gemm_small_kernel<16>),
          reinterpret_cast<const void *>(atomk::w4a4_gemm_small_kernel<32>),
          reinterpret_cast<const void *>(atomk::w4a4_gemm_small_kernel<64>),
          reinterpret_cast<const void *>(atomk::w4a4_gemm_small_kernel<16, true>),
          reinterpret_cast<const void *>(atomk::w4a4_gemm_small_kernel<32, true>),
          reinterpret_cast<const void *>(atomk::w4a4_gemm_small_kernel<64, true>)};
      for (const void *fn : fns)
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kSmemBytes)) != cudaSuccess)
          return ATOM_ERR_CUDA;
      dev->small_attr = true;
    }
  }
  atomk::SmallMaps maps;
  const CUtensorMapDataType u8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  // the INT8 group comes in two halves (64 W rows + 32 token rows each)
  // (tiled W: bulk copies of qw4's blocks, no W4 tensor map; the slot is
  // filled with the A4 map, which the kernel then never reads for W)
  if (!encode_2d(&maps.w4, u8, w_tiled ? static_cast<const void *>(qa4) : qw4, q4_row,
                 w_tiled ? M : N, q4_row, 64, w_tiled ? kMaxTokens : BW,
                 CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_2d(&maps.a4, u8, qa4, q4_row, M, q4_row, 64, kMaxTokens,
                 CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_2d(&maps.w8, u8, qw8, 128, N, 128, 128, BW / 2, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&maps.a8, u8, qa8, 128, M, 128, 128, kMaxTokens / 2,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&maps.sw, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, sw, N, K / 128, N * 4, BW, 1,
                 CU_TENSOR_MAP_SWIZZLE_NONE))
    return ATOM_ERR_CUDA;
  atomk::SmallParams p;
  p.sa = sa;
  p.sw = sw;
  p.y = static_cast<__half *>(y);
  p.partials = partials;
  p.qw4t = w_tiled ? qw4 : nullptr;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.G = static_cast<int>(K / 128);
  p.n_tiles = static_cast<int>((N + BW - 1) / BW);
  p.splits = splits;
  p.items = p.n_tiles * splits;
  // with a split, one CTA per (tile, K range) and the K ranges of a tile as
  // one cluster that sums them (no workspace is written)
  const int grid = p.items < dev->sm_count ? p.items : dev->sm_count;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  const int nt = M <= 16 ? 16 : (M <= 32 ? 32 : 64);
  cfg.blockDim = dim3(threads_for(nt), 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  // the K ranges of a tile as one cluster; programmatic dependent launch as
  // for the quantizer
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = static_cast<unsigned>(splits);
  attrs[0].val.clusterDim.y = 1;
  attrs[0].val.clusterDim.z = 1;
  attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 2;
  cudaError_t err;
  if (partials != nullptr) {
    if (M <= 16)
      err = cudaLaunchKernelEx(&cfg, atomk::w4a4_gemm_small_kernel<16, true>, maps, p);
    else if (M <= 32)
      err = cudaLaunchKernelEx(&cfg, atomk::w4a4_gemm_small_kernel<32, true>, maps, p);
    else
      err = cudaLaunchKernelEx(&cfg, atomk::w4a4_gemm_small_kernel<64, true>, maps, p);
  } else if (M <= 16) {
    err = cudaLaunchKernelEx(&cfg, atomk::w4a4_gemm_small_kernel<16>, maps, p);
  } else if (M <= 32) {
    err = cudaLaunchKernelEx(&cfg, atomk::w4a4_gemm_small_kernel<32>, maps, p);
  } else {
    err = cudaLaunchKernelEx(&cfg, atomk::w4a4_gemm_small_kernel<64>, maps, p);
  }
  return err == cudaSuccess ? ATOM_OK : ATOM_ERR_CUDA;
}

atom_status_t launch_gemm(const uint8_t *qa4, const int8_t *qa8, const float *sa,
                          const uint8_t *qw4, const int8_t *qw8, const float *sw, void *y,
                          int32_t *partials, int64_t M, int64_t N, int64_t K, int32_t n_outlier,
                          int32_t group, void *workspace, size_t workspace_bytes,
                          atom_stream_t stream, uint8_t *qy4 = nullptr, int8_t *qy8 = nullptr,
                          float *sy = nullptr, bool a8 = false, bool w_tiled = false) {
  if (M < 0 || N < 0) return ATOM_ERR_INVALID_ARG;
  atom_status_t st = check_method_params(K, n_outlier, group);
  if (st != ATOM_OK) return st;
  if (N < 8 || N % 8 != 0 || M > INT32_MAX || N > INT32_MAX) return ATOM_ERR_SHAPE;
  const bool qmode = qy4 != nullptr || qy8 != nullptr || sy != nullptr;
  // quantized Y: N is the next layer's K (whole groups, the INT8 group last)
  if (qmode && (N % 128 != 0 || N < 256 || N > kMaxK)) return ATOM_ERR_SHAPE;
  // the kernel addresses each packed INT4 matrix with 32-bit byte offsets
  const int64_t q4_row = (K - 128) / 2;
  if (M * q4_row >= (int64_t(1) << 31) || N * q4_row >= (int64_t(1) << 31)) return ATOM_ERR_SHAPE;
  if (M == 0) return ATOM_OK;
  if ((!qa4 && !a8) || !qa8 || !sa || !qw4 || !qw8 || !sw || (!y && !partials && !qmode) ||
      (qmode && (!qy4 || !qy8 || !sy)))
    return ATOM_ERR_INVALID_ARG;
  if ((!a8 && !aligned(qa4, 16)) || !aligned(qa8, 16) || !aligned(qw4, 16) ||
      !aligned(qw8, 16) || !aligned(sa, 4) || !aligned(sw, 4) || (y && !aligned(y, 16)) ||
      (partials && !aligned(partials, 16)) ||
      (qmode && (!aligned(qy4, 16) || !aligned(qy8, 16) || !aligned(sy, 4))))
    return ATOM_ERR_ALIGN;

  DeviceState *dev = nullptr;
  if ((st = current_device(&dev)) != ATOM_OK) return st;

  using namespace atomk::gemm_cfg;
  const bool pmode = partials != nullptr;
  const int mode = pmode ? kModePartials : (qmode ? kModeQuantY : kModeY);
  // A few tokens (decode): the small-M kernel, for Y and for the partials alike.
  if ((mode == kModeY || mode == kModePartials) && !a8 && M <= atomk::small_cfg::kMaxTokens)
    return launch_gemm_small(dev, qa4, qa8, sa, qw4, qw8, sw, y, partials, M, N, K, workspace,
                             workspace_bytes, stream, w_tiled);
  int pairs = 0;
  if ((st = gemm_pairs(dev, mode + (a8 ? 3 : 0), &pairs)) != ATOM_OK) return st;

  const int64_t G = K / 128;
  atomk::GemmMaps maps;
  const bool sa_by_tma = (M % 4) == 0;   // rows of sa must be 16-byte aligned for TMA
  const CUtensorMapDataType u8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const CUtensorMapDataType f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  // W4A8: INT8 activations [M][K], one 128-byte box per row and group; no INT4 A
  if (!encode_2d(&maps.a4, u8, a8 ? static_cast<const void *>(qa8) : qa4, q4_row, M, q4_row, 64,
                 BM, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_2d(&maps.w4, u8, w_tiled ? static_cast<const void *>(qa8) : qw4,
                 w_tiled ? 128 : q4_row, w_tiled ? M : N, w_tiled ? 128 : q4_row, 64, BW,
                 CU_TENSOR_MAP_SWIZZLE_NONE) ||   // (tiled W: bulk copies, this map is unused)
      !encode_2d(&maps.a8, u8, qa8, a8 ? K : 128, M, a8 ? K : 128, 128, BM,
                 CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&maps.w8, u8, qw8, 128, N, 128, 128, BW, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&maps.sw, f32, sw, N, G, N * 4, BN, 1, CU_TENSOR_MAP_SWIZZLE_NONE))
    return ATOM_ERR_CUDA;
  if (y) {
    if (!encode_2d(&maps.y, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, y, N, M, N * 2, 64, 32,
                   CU_TENSOR_MAP_SWIZZLE_128B))
      return ATOM_ERR_CUDA;
  } else {
    maps.y = maps.sw;   // not used by the kernel
  }
  if (sa_by_tma) {
    if (!encode_2d(&maps.sa, f32, sa, M, G, M * 4, BM, 1, CU_TENSOR_MAP_SWIZZLE_NONE))
      return ATOM_ERR_CUDA;
  } else {
    maps.sa = maps.sw;  // not used by the kernel
  }

  atomk::GemmParams p;
  p.qa4 = qa4;
  p.sa = sa;
  p.qw4 = qw4;
  p.sw = sw;
  p.y = static_cast<__half *>(y);
  p.partials = partials;
  p.qy4 = qy4;
  p.qy8 = qy8;
  p.sy = sy;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.G = static_cast<int>(G);
  p.sa_by_tma = sa_by_tma ? 1 : 0;
  p.qw4t = w_tiled ? qw4 : nullptr;
  p.w_tiles = static_cast<int>((N + BW - 1) / BW);
  p.m_tiles = static_cast<int>((M + kPairM - 1) / kPairM);
  p.n_tiles = static_cast<int>((N + BN - 1) / BN);
  const int64_t tiles = static_cast<int64_t>(p.m_tiles) * p.n_tiles;
  // Split K only for fp16 Y, with a workspace large enough for the partials.
  int splits = (mode != kModeY || a8) ? 1 : gemm_splits(M, N, K, pairs);
  if (splits > 1 && (workspace == nullptr ||
                     workspace_bytes < static_cast<size_t>(splits) * M * N * sizeof(float) ||
                     !aligned(workspace, 16)))
    splits = 1;
  if (tiles * splits > INT32_MAX) return ATOM_ERR_SHAPE;
  p.tiles = static_cast<int>(tiles);
  p.splits = splits;
  p.items = static_cast<int>(tiles * splits);
  p.ws = splits > 1 ? static_cast<float *>(workspace) : nullptr;
  const int64_t used = p.items < pairs ? p.items : pairs;
  const int grid = static_cast<int>(2 * used);   // CTA pairs (cluster of 2)
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (a8 && mode == kModePartials)
    atomk::w4a4_gemm_kernel<true, false, true><<<grid, kThreads, kSmemBytes, s>>>(maps, p);
  else if (a8)
    atomk::w4a4_gemm_kernel<false, false, true><<<grid, kThreads, kSmemBytes, s>>>(maps, p);
  else if (mode == kModePartials)
    atomk::w4a4_gemm_kernel<true><<<grid, kThreads, kSmemBytes, s>>>(maps, p);
  else if (mode == kModeQuantY)
    atomk::w4a4_gemm_kernel<false, true><<<grid, kThreads, kSmemBytes, s>>>(maps, p);
  else
    atomk::w4a4_gemm_kernel<false><<<grid, kThreads, kSmemBytes, s>>>(maps, p);
  if (cudaGetLastError() != cudaSuccess) return ATOM_ERR_CUDA;
  if (splits > 1) {
    const int64_t count8 = M * N / 8;
    int64_t blocks = (count8 + 255) / 256;
    const int64_t cap = static_cast<int64_t>(dev->sm_count) * 8;
    if (blocks > cap) blocks = cap;
    atomk::splitk_reduce_kernel<<<static_cast<int>(blocks), 256, 0, s>>>(
        p.ws, static_cast<__half *>(y), count8, M * N, splits);
    if (cudaGetLastError() != cudaSuccess) return ATOM_ERR_CUDA;
  }
  return ATOM_OK;
}

// Co-resident CTA pairs of the GEMM kernel on this device (cached per device).
atom_status_t gemm_pairs(DeviceState *dev, int mode, int *pairs) {
  using namespace atomk::gemm_cfg;
  if (!dev->gemm_attr[mode].load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (dev->gemm_attr[mode].load(std::memory_order_relaxed)) {
      *pairs = dev->gemm_clusters[mode];
      return ATOM_OK;
    }
    const void *fn =
        mode == kModePartials ? reinterpret_cast<const void *>(atomk::w4a4_gemm_kernel<true>)
        : mode == kModeQuantY ? reinterpret_cast<const void *>(atomk::w4a4_gemm_kernel<false, true>)
        : mode == kModeY + 3
            ? reinterpret_cast<const void *>(atomk::w4a4_gemm_kernel<false, false, true>)
        : mode == kModePartials + 3
            ? reinterpret_cast<const void *>(atomk::w4a4_gemm_kernel<true, false, true>)
            : reinterpret_cast<const void *>(atomk::w4a4_gemm_kernel<false>);
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes)) != cudaSuccess)
      return ATOM_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * dev->sm_count, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, fn, &cfg) != cudaSuccess || clusters < 1)
      clusters = dev->sm_count / 2;
    dev->gemm_clusters[mode] = clusters;
    dev->gemm_attr[mode].store(true, std::memory_order_release);
  }
  *pairs = dev->gemm_clusters[mode];
  return ATOM_OK;
}

// Workspace bytes atom_w4a4_gemm asks for on this shape: splits * M * N * 4
// when the kernel that will run (the small-M kernel for M <= 64, the large
// one otherwise) would split K, else 0.
atom_status_t gemm_workspace_need(DeviceState *dev, int64_t M, int64_t N, int64_t K,
                                  size_t *bytes) {
  int splits = 1;
  if (M <= atomk::small_cfg::kMaxTokens) {
    splits = small_splits(N, K, dev->sm_count);
  } else {
    int pairs = 0;
    const atom_status_t st = gemm_pairs(dev, kModeY, &pairs);
    if (st != ATOM_OK) return st;
    splits = gemm_splits(M, N, K, pairs);
  }
  *bytes = splits > 1 ? static_cast<size_t>(splits) * M * N * sizeof(float) : 0;
  return ATOM_OK;
}

}  // namespace

// ---------------------------------------------------------------- W8A8 GEMM

atom_status_t launch_w8a8(const int8_t *qa, const float *sa, const int8_t *qw, const float *sw,
                          void *y, int64_t M, int64_t N, int64_t K, atom_stream_t stream) {
  if (M < 0 || N < 0 || K < 0) return ATOM_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return ATOM_OK;
  // K: rows of 16-byte multiples for the TMA, and an int32 sum that cannot
  // overflow (K * 127 * 127 < 2^31); N: 16-byte rows of fp16 Y.
  if (K < 16 || K % 16 != 0 || K > 131072 || N % 8 != 0 || M > INT32_MAX || N > INT32_MAX)
    return ATOM_ERR_SHAPE;
  if (!qa || !sa || !qw || !sw || !y) return ATOM_ERR_INVALID_ARG;
  if (!aligned(qa, 16) || !aligned(qw, 16) || !aligned(y, 16) || !aligned(sa, 4) ||
      !aligned(sw, 16))
    return ATOM_ERR_ALIGN;

  DeviceState *dev = nullptr;
  atom_status_t st = current_device(&dev);
  if (st != ATOM_OK) return st;
  using namespace atomk::w8a8_cfg;
  int pairs = 0;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!dev->w8a8_attr) {
      const void *fn = reinterpret_cast<const void *>(atomk::w8a8_gemm_kernel);
      if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kSmemBytes)) != cudaSuccess)
        return ATOM_ERR_CUDA;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * dev->sm_count, 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = kSmemBytes;
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = 2;
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, fn, &cfg) != cudaSuccess || clusters < 1)
        clusters = dev->sm_count / 2;
      dev->w8a8_clusters = clusters;
      dev->w8a8_attr = true;
    }
    pairs = dev->w8a8_clusters;
  }

  atomk::W8A8Maps maps;
  const CUtensorMapDataType u8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  if (!encode_2d(&maps.a, u8, qa, K, M, K, 128, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&maps.w, u8, qw, K, N, K, 128, BW, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&maps.y, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, y, N, M, N * 2, 64, 32,
                 CU_TENSOR_MAP_SWIZZLE_128B))
    return ATOM_ERR_CUDA;
  atomk::W8A8Params p;
  p.sa = sa;
  p.sw = sw;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.ksteps = static_cast<int>((K + 127) / 128);
  p.m_tiles = static_cast<int>((M + kPairM - 1) / kPairM);
  const int64_t tiles = static_cast<int64_t>(p.m_tiles) * ((N + BN - 1) / BN);
  if (tiles > INT32_MAX) return ATOM_ERR_SHAPE;
  p.tiles = static_cast<int>(tiles);
  const int64_t used = tiles < pairs ? tiles : pairs;
  atomk::w8a8_gemm_kernel<<<static_cast<int>(2 * used), kThreads, kSmemBytes,
                            reinterpret_cast<cudaStream_t>(stream)>>>(maps, p);
  return cudaGetLastError() == cudaSuccess ? ATOM_OK : ATOM_ERR_CUDA;
}

// ---------------------------------------------------------------- INT4 KV cache

int kv_grid(const DeviceState *dev, int64_t groups) {
  const int64_t want = (groups * 8 + atomk::kKvThreads - 1) / atomk::kKvThreads;
  const int64_t cap = static_cast<int64_t>(dev->sm_count) * 8;
  return static_cast<int>(want < cap ? want : cap);
}

extern "C" {

atom_status_t atom_kv_quant(const void *x, int64_t groups, uint8_t *q4, float *scales,
                            atom_stream_t stream) {
  if (groups < 0) return ATOM_ERR_INVALID_ARG;
  if (groups == 0) return ATOM_OK;
  if (!x || !q4 || !scales) return ATOM_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(q4, 8) || !aligned(scales, 4)) return ATOM_ERR_ALIGN;
  DeviceState *dev = nullptr;
  atom_status_t st = current_device(&dev);
  if (st != ATOM_OK) return st;
  atomk::kv_quant_kernel<<<kv_grid(dev, groups), atomk::kKvThreads, 0,
                           reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const __half *>(x), groups, q4, scales);
  return cudaGetLastError() == cudaSuccess ? ATOM_OK : ATOM_ERR_CUDA;
}

atom_status_t atom_kv_dequant(const uint8_t *q4, const float *scales, int64_t groups, void *out,
                              atom_stream_t stream) {
  if (groups < 0) return ATOM_ERR_INVALID_ARG;
  if (groups == 0) return ATOM_OK;
  if (!q4 || !scales || !out) return ATOM_ERR_INVALID_ARG;
  if (!aligned(q4, 8) || !aligned(scales, 4) || !aligned(out, 16)) return ATOM_ERR_ALIGN;
  DeviceState *dev = nullptr;
  atom_status_t st = current_device(&dev);
  if (st != ATOM_OK) return st;
  atomk::kv_dequant_kernel<<<kv_grid(dev, groups), atomk::kKvThreads, 0,
                             reinterpret_cast<cudaStream_t>(stream)>>>(
      q4, scales, groups, static_cast<__half *>(out));
  return cudaGetLastError() == cudaSuccess ? ATOM_OK : ATOM_ERR_CUDA;
}

atom_status_t atom_w8a8_gemm(const int8_t *qa, const float *sa, const int8_t *qw,
                             const float *sw, void *y, int64_t M, int64_t N, int64_t K,
                             atom_stream_t stream) {
  return launch_w8a8(qa, sa, qw, sw, y, M, N, K, stream);
}

atom_status_t atom_reorder_quant(const void *x, int64_t M, int64_t K, int64_t ld_x,
                                 const int32_t *outlier_idx, int32_t n_outlier, int32_t group,
                                 uint8_t *q4, int8_t *q8, float *scales, atom_stream_t stream) {
  return launch_quant(x, M, K, ld_x, outlier_idx, n_outlier, group, q4, q8, scales, stream);
}

atom_status_t atom_quant_weights(const void *w, int64_t N, int64_t K, int64_t ld_w,
                                 const int32_t *outlier_idx, int32_t n_outlier, int32_t group,
                                 uint8_t *qw4, int8_t *qw8, float *sw, atom_stream_t stream) {
  return launch_quant(w, N, K, ld_w, outlier_idx, n_outlier, group, qw4, qw8, sw, stream);
}

atom_status_t atom_w4a4_gemm(const uint8_t *qa4, const int8_t *qa8, const float *sa,
                             const uint8_t *qw4, const int8_t *qw8, const float *sw, void *y,
                             int64_t M, int64_t N, int64_t K, int32_t n_outlier, int32_t group,
                             void *workspace, size_t workspace_bytes, atom_stream_t stream) {
  if (!y && M > 0) return ATOM_ERR_INVALID_ARG;
  return launch_gemm(qa4, qa8, sa, qw4, qw8, sw, y, nullptr, M, N, K, n_outlier, group, workspace,
                     workspace_bytes, stream);
}

atom_status_t atom_w4a4_gemm_partials(const uint8_t *qa4, const int8_t *qa8, const float *sa,
                                      const uint8_t *qw4, const int8_t *qw8, const float *sw,
                                      int32_t *partials, void *y, int64_t M, int64_t N, int64_t K,
                                      int32_t n_outlier, int32_t group, atom_stream_t stream) {
  if (!partials && M > 0) return ATOM_ERR_INVALID_ARG;
  return launch_gemm(qa4, qa8, sa, qw4, qw8, sw, y, partials, M, N, K, n_outlier, group, nullptr,
                     0, stream);
}

atom_status_t atom_reorder_quant_a8(const void *x, int64_t M, int64_t K, int64_t ld_x,
                                    const int32_t *outlier_idx, int32_t n_outlier, int32_t group,
                                    int8_t *q8, float *scales, atom_stream_t stream) {
  return launch_quant(x, M, K, ld_x, outlier_idx, n_outlier, group, nullptr, q8, scales, stream,
                      true);
}

atom_status_t atom_w4a8_gemm(const int8_t *qa8, const float *sa, const uint8_t *qw4,
                             const int8_t *qw8, const float *sw, void *y, int64_t M, int64_t N,
                             int64_t K, int32_t n_outlier, int32_t group, atom_stream_t stream) {
  if (!y && M > 0) return ATOM_ERR_INVALID_ARG;
  return launch_gemm(nullptr, qa8, sa, qw4, qw8, sw, y, nullptr, M, N, K, n_outlier, group,
                     nullptr, 0, stream, nullptr, nullptr, nullptr, true);
}

atom_status_t atom_w4a8_gemm_partials(const int8_t *qa8, const float *sa, const uint8_t *qw4,
                                      const int8_t *qw8, const float *sw, int32_t *partials,
                                      void *y, int64_t M, int64_t N, int64_t K,
                                      int32_t n_outlier, int32_t group, atom_stream_t stream) {
  if (!partials && M > 0) return ATOM_ERR_INVALID_ARG;
  return launch_gemm(nullptr, qa8, sa, qw4, qw8, sw, y, partials, M, N, K, n_outlier, group,
                     nullptr, 0, stream, nullptr, nullptr, nullptr, true);
}

atom_status_t atom_w4a4_gemm_quant(const uint8_t *qa4, const int8_t *qa8, const float *sa,
                                   const uint8_t *qw4, const int8_t *qw8, const float *sw,
                                   int64_t M, int64_t N, int64_t K, int32_t n_outlier,
                                   int32_t group, uint8_t *qy4, int8_t *qy8, float *sy,
                                   atom_stream_t stream) {
  if ((!qy4 || !qy8 || !sy) && M > 0) return ATOM_ERR_INVALID_ARG;
  return launch_gemm(qa4, qa8, sa, qw4, qw8, sw, nullptr, nullptr, M, N, K, n_outlier, group,
                     nullptr, 0, stream, qy4, qy8, sy);
}

size_t atom_tiled_weights_bytes(int64_t N, int64_t K) {
  if (N <= 0 || K % 128 != 0 || K < 256 || K > kMaxK) return 0;
  return static_cast<size_t>((N + atomk::kTileRows - 1) / atomk::kTileRows) *
         static_cast<size_t>(K / 128 - 1) * atomk::kTileBlock;
}

static atom_status_t tiled_copy(const uint8_t *src, int64_t N, int64_t K, uint8_t *dst,
                                atom_stream_t stream, bool pack) {
  if (N < 0) return ATOM_ERR_INVALID_ARG;
  if (K % 128 != 0 || K < 256 || K > kMaxK || N > INT32_MAX) return ATOM_ERR_SHAPE;
  if (N == 0) return ATOM_OK;
  if (!src || !dst) return ATOM_ERR_INVALID_ARG;
  if (!aligned(src, 16) || !aligned(dst, 16)) return ATOM_ERR_ALIGN;
  DeviceState *dev = nullptr;
  const atom_status_t st = current_device(&dev);
  if (st != ATOM_OK) return st;
  const int64_t g4 = K / 128 - 1;
  const int64_t chunks = static_cast<int64_t>(atom_tiled_weights_bytes(N, K) / 16);
  int64_t blocks = (chunks + 255) / 256;
  const int64_t cap = static_cast<int64_t>(dev->sm_count) * 16;
  if (blocks > cap) blocks = cap;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (pack)
    atomk::pack_weights_tiled_kernel<<<static_cast<int>(blocks), 256, 0, s>>>(src, dst, N,
                                                                               (K - 128) / 2, g4, chunks);
  else
    atomk::unpack_weights_tiled_kernel<<<static_cast<int>(blocks), 256, 0, s>>>(
        src, dst, N, (K - 128) / 2, g4, chunks);
  return cudaGetLastError() == cudaSuccess ? ATOM_OK : ATOM_ERR_CUDA;
}

atom_status_t atom_pack_weights_tiled(const uint8_t *qw4, int64_t N, int64_t K, uint8_t *qw4t,
                                      atom_stream_t stream) {
  return tiled_copy(qw4, N, K, qw4t, stream, true);
}

atom_status_t atom_unpack_weights_tiled(const uint8_t *qw4t, int64_t N, int64_t K, uint8_t *qw4,
                                        atom_stream_t stream) {
  return tiled_copy(qw4t, N, K, qw4, stream, false);
}

atom_status_t atom_w4a4_gemm_tiled(const uint8_t *qa4, const int8_t *qa8, const float *sa,
                                   const uint8_t *qw4t, const int8_t *qw8, const float *sw,
                                   void *y, int64_t M, int64_t N, int64_t K, int32_t n_outlier,
                                   int32_t group, void *workspace, size_t workspace_bytes,
                                   atom_stream_t stream) {
  if (!y && M > 0) return ATOM_ERR_INVALID_ARG;
  return launch_gemm(qa4, qa8, sa, qw4t, qw8, sw, y, nullptr, M, N, K, n_outlier, group,
                     workspace, workspace_bytes, stream, nullptr, nullptr, nullptr, false, true);
}

size_t atom_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K < 256) return 0;
  DeviceState *dev = nullptr;
  if (current_device(&dev) != ATOM_OK) return 0;
  size_t bytes = 0;
  return gemm_workspace_need(dev, M, N, K, &bytes) == ATOM_OK ? bytes : 0;
}

atom_status_t atom_device_status(int clear) {
  if (cudaDeviceSynchronize() != cudaSuccess) return ATOM_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, atomk::g_device_status, sizeof(int)) != cudaSuccess)
    return ATOM_ERR_CUDA;
  if (clear) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(atomk::g_device_status, &zero, sizeof(int)) != cudaSuccess)
      return ATOM_ERR_CUDA;
  }
  return static_cast<atom_status_t>(v);
}

atom_status_t atom_probe_mma_i8(int64_t groups, int32_t *pairs_out, atom_stream_t stream) {
  if (groups < 1 || groups > (int64_t(1) << 20) || pairs_out == nullptr) return ATOM_ERR_INVALID_ARG;
  DeviceState *dev = nullptr;
  atom_status_t st = current_device(&dev);
  if (st != ATOM_OK) return st;
  using namespace atomk::probe_cfg;
  int pairs = 0;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    const void *fn = reinterpret_cast<const void *>(atomk::mma_i8_probe_kernel);
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes)) != cudaSuccess)
      return ATOM_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * dev->sm_count, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&pairs, fn, &cfg) != cudaSuccess || pairs < 1)
      pairs = dev->sm_count / 2;
  }
  atomk::mma_i8_probe_kernel<<<2 * pairs, kThreads, kSmemBytes,
                               reinterpret_cast<cudaStream_t>(stream)>>>(groups);
  if (cudaGetLastError() != cudaSuccess) return ATOM_ERR_CUDA;
  *pairs_out = pairs;
  return ATOM_OK;
}

atom_status_t atom_debug_wait_timeout(uint64_t limit_ns, atom_stream_t stream) {
  if (limit_ns == 0 || limit_ns > atomk::kWaitLimitNs) return ATOM_ERR_INVALID_ARG;
  DeviceState *dev = nullptr;
  const atom_status_t st = current_device(&dev);
  if (st != ATOM_OK) return st;
  atomk::wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns);
  return cudaGetLastError() == cudaSuccess ? ATOM_OK : ATOM_ERR_CUDA;
}

const char *atom_status_string(atom_status_t status) {
  switch (status) {
    case ATOM_OK: return "ATOM_OK";
    case ATOM_ERR_INVALID_ARG: return "ATOM_ERR_INVALID_ARG";
    case ATOM_ERR_SHAPE: return "ATOM_ERR_SHAPE";
    case ATOM_ERR_ALIGN: return "ATOM_ERR_ALIGN";
    case ATOM_ERR_UNSUPPORTED: return "ATOM_ERR_UNSUPPORTED";
    case ATOM_ERR_CUDA: return "ATOM_ERR_CUDA";
    case ATOM_ERR_TIMEOUT: return "ATOM_ERR_TIMEOUT";
  }
  return "ATOM_ERR_UNKNOWN";
}

int atom_version(void) { return 100; }

}  // extern "C"

// ---------------------------------------------------------------- allocation-free GEMM
//
// Some callers cannot allocate device memory around a GEMM call: serving
// runtimes that hand every byte of device memory to a fixed pool at start-up
// (nothing is left to allocate from, and a stray allocation would fragment the
// pool), and C or embedded callers that have no device allocator of their own.
// atom_w4a4_gemm needs scratch only when it splits K (M > 64 with few output
// tiles), and takes it from the caller. This entry point takes it instead from
// a fixed array in the library's device memory.

namespace {

// Scratch of atom_w4a4_gemm_noalloc: the fp32 partial tiles of a split-K call,
// splits * M * N floats. Every GPU that loads the library holds it until exit.
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;   // 8 MiB
__device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

// Device address of the scratch on the current device. In host code the name
// g_noalloc_scratch is a host-side stand-in, not a device address, so the
// address is looked up once per device, with that device current.
atom_status_t noalloc_scratch(DeviceState *dev, void **out) {
  void *p = dev->noalloc_scratch.load(std::memory_order_acquire);
  if (p == nullptr) {
    std::lock_guard<std::mutex> lock(g_mutex);
    p = dev->noalloc_scratch.load(std::memory_order_relaxed);
    if (p == nullptr) {
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
        return ATOM_ERR_CUDA;
      dev->noalloc_scratch.store(p, std::memory_order_release);
    }
  }
  *out = p;
  return ATOM_OK;
}

}  // namespace

extern "C" ATOM_API atom_status_t atom_w4a4_gemm_noalloc(
    const uint8_t *qa4, const int8_t *qa8, const float *sa, const uint8_t *qw4, const int8_t *qw8,
    const float *sw, void *y, int64_t M, int64_t N, int64_t K, int32_t n_outlier, int32_t group,
    atom_stream_t stream) {
  if (M < 0 || N < 0) return ATOM_ERR_INVALID_ARG;
  atom_status_t st = check_method_params(K, n_outlier, group);
  if (st != ATOM_OK) return st;
  if (M == 0) return ATOM_OK;
  if (!y) return ATOM_ERR_INVALID_ARG;
  if (N < 8 || N % 8 != 0 || M > INT32_MAX || N > INT32_MAX) return ATOM_ERR_SHAPE;
  DeviceState *dev = nullptr;
  if ((st = current_device(&dev)) != ATOM_OK) return st;
  // the scratch the split of the kernel that will run needs (the same rule as
  // atom_gemm_workspace_bytes)
  size_t need = 0;
  if ((st = gemm_workspace_need(dev, M, N, K, &need)) != ATOM_OK) return st;
  if (need > kNoAllocScratchBytes)
    return ATOM_ERR_SHAPE;   // the split's partial tiles do not fit in the fixed scratch
  void *scratch = nullptr;
  if ((st = noalloc_scratch(dev, &scratch)) != ATOM_OK) return st;
  return launch_gemm(qa4, qa8, sa, qw4, qw8, sw, y, nullptr, M, N, K, n_outlier, group, scratch,
                     kNoAllocScratchBytes, stream);
}
