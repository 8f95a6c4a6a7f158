// Host side of libhq.so: argument validation, workspace carving, TMA descriptor encoding
// and kernel launches behind the C ABI declared in include/hq.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>

#include "hq.h"
#include "fwht_quant.cuh"
#include "fwht_dual.cuh"
#include "gemm_tcgen05.cuh"
#include "rotate_out.cuh"
#include "prerot_quant.cuh"
#include "mma_peak.cuh"

namespace {

// Per-device status word: written by kernels on a device-side error, read and cleared by
// hq_get_error().
__device__ unsigned int g_hq_status;

constexpr int kMaxDevices = 64;
constexpr int kMaxPartials = 4096;  // upper bound on the absmax pass's grid
constexpr size_t kPartialBytes = kMaxPartials * sizeof(float);
constexpr size_t kAlign = 256;

thread_local int t_last_cuda_error = 0;

struct DeviceInfo {
  bool ready = false;
  bool supported = false;
  int sms = 0;
  unsigned int* status = nullptr;
  unsigned gemm_attr_set = 0;  // bit per GEMM instantiation
  bool cols_attr[5][4][2] = {};  // strided bf16 quantizer instantiations prepared [k][mode][signed]
  unsigned pair_attr_set = 0;  // bit per CTA-pair GEMM instantiation
  bool dual_attr[5][4][2][2] = {};  // fused two-rotation instantiations prepared [k][mode][w32][signed]
  bool dual_onchip_attr[5][2][2][2] = {};  // its single-launch form [k][int8 / fp8][w32][signed]
  bool mn_attr[2] = {};             // MN-major pair GEMM (fp32 output) prepared [int8 / fp8]
  bool rot_attr[3] = {};            // row de-rotation with its 64 KB tile prepared [k = 64, 128, 256]
  bool rotout_attr[2] = {};         // K-major pair GEMM with fp32 rotated output prepared [int8 / fp8]
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

hq_status cuda_fail(cudaError_t e) {
  t_last_cuda_error = static_cast<int>(e);
  return HQ_ERR_CUDA;
}

// Current device's cached properties; fills them on first use.
hq_status device_info(DeviceInfo** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return HQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    int major = 0, sms = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return cuda_fail(e);
    void* p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_hq_status)) != cudaSuccess) return cuda_fail(e);
    d.supported = (major == 10);
    d.sms = sms;
    d.status = static_cast<unsigned int*>(p);
    d.ready = true;
  }
  if (!d.supported) return HQ_ERR_UNSUPPORTED;
  *out = &d;
  return HQ_OK;
}

hq_status tensor_map_encoder(PFN_cuTensorMapEncodeTiled_v12000* fn) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_encode) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                                     cudaEnableDefault, &q);
    if (e != cudaSuccess) return cuda_fail(e);
    if (q != cudaDriverEntryPointSuccess || !p) return cuda_fail(cudaErrorNotSupported);
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  *fn = g_encode;
  return HQ_OK;
}

bool valid_k(int k) { return k == 16 || k == 32 || k == 64 || k == 128 || k == 256; }
bool valid_fmt(int fmt) {
  return fmt == HQ_INT8 || fmt == HQ_FP8_E4M3 || fmt == HQ_FP6_E3M2 || fmt == HQ_FP6_E2M3 || fmt == HQ_FP4_E2M1;
}
// A/B element format field of the kind::f8f6f4 instruction descriptor (0 for INT8's kind::i8).
uint32_t ab_format_code(int fmt) {
  switch (fmt) {
    case HQ_FP6_E2M3: return 3;
    case HQ_FP6_E3M2: return 4;
    case HQ_FP4_E2M1: return 5;
    default: return 0;
  }
}
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

// ------------------------------------------------------------------ quantization launches

// Work units of a quantization pass (warp steps along the contiguous dimension, or tiles).
int64_t quant_units(hq_dtype dt, int64_t rows, int64_t cols, int dim) {
  if (dim == 1) {
    const int64_t units = (rows * cols + hq::kRowsWarpElems - 1) / hq::kRowsWarpElems;
    return (units + hq::kQuantThreads / 32 - 1) / (hq::kQuantThreads / 32);
  }
  if (dt == HQ_BF16)
    return ((rows + hq::kColsTileRows2 - 1) / hq::kColsTileRows2) *
           ((cols + hq::kColsTileCols2 - 1) / hq::kColsTileCols2);
  const int64_t tcols = 8 * (16 / 4);
  return ((rows + hq::kColsTileRows - 1) / hq::kColsTileRows) * ((cols + tcols - 1) / tcols);
}

// Upper bound on the CTAs of any quantization pass (the partial-maxima capacity it needs).
int64_t quant_grid(hq_dtype dt, int64_t rows, int64_t cols, int dim, int sms) {
  return std::max<int64_t>(1, std::min<int64_t>(quant_units(dt, rows, cols, dim),
                                                std::min<int64_t>(int64_t(sms) * 4, kMaxPartials)));
}

// Co-resident CTAs per SM of a kernel (cached): grids never exceed one full wave, so no
// pass ends with a partial second wave.
int blocks_per_sm(const void* fn, size_t smem) {
  static std::mutex mu;
  static const void* keys[512];
  static int vals[512];
  static int n = 0;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n; ++i)
    if (keys[i] == fn) return vals[i];
  int b = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, fn, hq::kQuantThreads, smem) != cudaSuccess || b < 1) b = 1;
  b = std::min(b, 4);
  if (n < 512) {
    keys[n] = fn;
    vals[n] = b;
    ++n;
  }
  return b;
}

template <int K, int MODE, bool SIGNED>
cudaError_t cols_bf16_smem_attr(DeviceInfo& d) {
  constexpr int kIdx = (K == 16 ? 0 : K == 32 ? 1 : K == 64 ? 2 : K == 128 ? 3 : 4);
  std::lock_guard<std::mutex> lock(g_mu);
  bool& done = d.cols_attr[kIdx][MODE][SIGNED ? 1 : 0];
  if (done) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(hq::fwhtq_cols_bf16_kernel<K, MODE, SIGNED>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(hq::kColsSmemBytes2));
  if (e == cudaSuccess) done = true;
  return e;
}

// Launch with programmatic stream serialization: the kernel may be scheduled while the previous
// kernel in the stream is finishing; it waits for that kernel's completion (griddep_wait) before
// touching memory, so the order of results is that of an ordinary launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Launch one pass; returns its grid through *grid (the absmax pass's grid is the number of
// partials the code pass reduces).  SIGNED: the randomized variant with sign flags `neg`.
template <typename SrcT, int K, int MODE, bool SIGNED>
cudaError_t launch_pass_s(const SrcT* src, int64_t rows, int64_t cols, int dim, uint8_t* codes,
                          float* scale, float* partials, int n_partials, int reverse, const uint8_t* neg,
                          int lp_fmt, DeviceInfo& d, cudaStream_t st, int* grid) {
  using namespace hq;
  const int64_t units = quant_units(sizeof(SrcT) == 2 ? HQ_BF16 : HQ_F32, rows, cols, dim);
  auto grid_for = [&](const void* fn, size_t smem) {
    const int64_t cap = std::min<int64_t>(int64_t(d.sms) * blocks_per_sm(fn, smem), kMaxPartials);
    return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(units, cap)));
  };
  int g = 1;
  if (dim == 1) {
    const int64_t n = rows * cols;
    if ((reinterpret_cast<uintptr_t>(src) & 31u) == 0) {
      auto fn = fwhtq_rows_kernel<SrcT, K, MODE, true, SIGNED>;
      g = grid_for(reinterpret_cast<const void*>(fn), 0);
      cudaError_t e = launch_pdl(fn, g, kQuantThreads, 0, st, src, n, codes, partials,
                                 MODE == kModeAbsmax ? g : n_partials, scale, d.status, reverse, neg, cols, lp_fmt);
      if (e != cudaSuccess) return e;
    } else {
      auto fn = fwhtq_rows_kernel<SrcT, K, MODE, false, SIGNED>;
      g = grid_for(reinterpret_cast<const void*>(fn), 0);
      cudaError_t e = launch_pdl(fn, g, kQuantThreads, 0, st, src, n, codes, partials,
                                 MODE == kModeAbsmax ? g : n_partials, scale, d.status, reverse, neg, cols, lp_fmt);
      if (e != cudaSuccess) return e;
    }
  } else if constexpr (sizeof(SrcT) == 2) {
    cudaError_t e = cols_bf16_smem_attr<K, MODE, SIGNED>(d);
    if (e != cudaSuccess) return e;
    auto fn = fwhtq_cols_bf16_kernel<K, MODE, SIGNED>;
    g = grid_for(reinterpret_cast<const void*>(fn), kColsSmemBytes2);
    e = launch_pdl(fn, g, kQuantThreads, kColsSmemBytes2, st, src, rows, cols, codes, partials,
                   MODE == kModeAbsmax ? g : n_partials, scale, d.status, reverse, neg, lp_fmt);
    if (e != cudaSuccess) return e;
  } else {
    auto fn = fwhtq_cols_f32_kernel<SrcT, K, MODE, SIGNED>;
    g = grid_for(reinterpret_cast<const void*>(fn), 0);
    cudaError_t e = launch_pdl(fn, g, kQuantThreads, 0, st, src, rows, cols, codes, partials,
                               MODE == kModeAbsmax ? g : n_partials, scale, d.status, reverse, neg, lp_fmt);
    if (e != cudaSuccess) return e;
  }
  *grid = g;
  return cudaGetLastError();
}

template <typename SrcT, int K, int MODE>
cudaError_t launch_pass(const SrcT* src, int64_t rows, int64_t cols, int dim, uint8_t* codes, float* scale,
                        float* partials, int n_partials, int reverse, const uint8_t* neg, DeviceInfo& d,
                        cudaStream_t st, int* grid, int lp_fmt = 0) {
  return neg ? launch_pass_s<SrcT, K, MODE, true>(src, rows, cols, dim, codes, scale, partials, n_partials, reverse,
                                                  neg, lp_fmt, d, st, grid)
             : launch_pass_s<SrcT, K, MODE, false>(src, rows, cols, dim, codes, scale, partials, n_partials, reverse,
                                                   nullptr, lp_fmt, d, st, grid);
}

// Code pass of a format: INT8 and FP8 have their own instantiations, the FP6 / FP4
// minifloats share one that takes the format at run time.
template <typename SrcT, int K>
cudaError_t launch_code_pass(const SrcT* src, int64_t rows, int64_t cols, int dim, hq_fmt fmt, uint8_t* codes,
                             float* scale, float* partials, int n_partials, int reverse, const uint8_t* neg,
                             DeviceInfo& d, cudaStream_t st) {
  using namespace hq;
  int g = 0;
  if (fmt == HQ_INT8)
    return launch_pass<SrcT, K, kModeInt8>(src, rows, cols, dim, codes, scale, partials, n_partials, reverse, neg, d,
                                           st, &g);
  if (fmt == HQ_FP8_E4M3)
    return launch_pass<SrcT, K, kModeFp8>(src, rows, cols, dim, codes, scale, partials, n_partials, reverse, neg, d,
                                          st, &g);
  return launch_pass<SrcT, K, kModeLowp>(src, rows, cols, dim, codes, scale, partials, n_partials, reverse, neg, d,
                                         st, &g, static_cast<int>(fmt));
}

// One operand, one rotation: absmax pass forward, code pass backward.
template <typename SrcT, int K>
cudaError_t launch_quant(const void* src_v, int64_t rows, int64_t cols, int dim, hq_fmt fmt,
                         uint8_t* codes, float* scale, float* partials, const uint8_t* neg, DeviceInfo& d,
                         cudaStream_t st) {
  const SrcT* src = static_cast<const SrcT*>(src_v);
  using namespace hq;
  int g1 = 0, g2 = 0;
  cudaError_t e = launch_pass<SrcT, K, kModeAbsmax>(src, rows, cols, dim, codes, scale, partials, 0, 0, neg, d, st, &g1);
  if (e != cudaSuccess) return e;
  (void)g2;
  return launch_code_pass<SrcT, K>(src, rows, cols, dim, fmt, codes, scale, partials, g1, 1, neg, d, st);
}

// One operand, both rotations: the four passes run back to back, alternating direction, so
// after the first only what L2 cannot hold is read from HBM again.
template <typename SrcT, int K>
cudaError_t launch_dual(const void* src_v, int64_t rows, int64_t cols, hq_fmt fmt, uint8_t* codes_c,
                        float* scale_c, uint8_t* codes_r, float* scale_r, float* part_c, float* part_r,
                        const uint8_t* neg_c, const uint8_t* neg_r, DeviceInfo& d, cudaStream_t st) {
  const SrcT* src = static_cast<const SrcT*>(src_v);
  using namespace hq;
  int gc = 0, gr = 0, g = 0;
  cudaError_t e = launch_pass<SrcT, K, kModeAbsmax>(src, rows, cols, 1, codes_c, scale_c, part_c, 0, 0, neg_c, d, st, &gc);
  if (e == cudaSuccess) e = launch_pass<SrcT, K, kModeAbsmax>(src, rows, cols, 0, codes_r, scale_r, part_r, 0, 1, neg_r, d, st, &gr);
  if (e != cudaSuccess) return e;
  (void)g;
  e = launch_code_pass<SrcT, K>(src, rows, cols, 1, fmt, codes_c, scale_c, part_c, gc, 0, neg_c, d, st);
  if (e == cudaSuccess) e = launch_code_pass<SrcT, K>(src, rows, cols, 0, fmt, codes_r, scale_r, part_r, gr, 1, neg_r, d, st);
  return e;
}

// Both rotations of a bf16 tensor from one read per pass (fwht_dual.cuh).  The tensor is
// described to TMA as the 3-D view (col, a, b) with row = 64a + b, so it needs rows and
// cols to be multiples of 64; the caller falls back to launch_dual otherwise.
bool fused_dual_ok(int64_t rows, int64_t cols) {
  return rows % 64 == 0 && cols % 64 == 0 && rows / 64 < (int64_t(1) << 31) && cols < (int64_t(1) << 31);
}

hq_status encode_dual_map(CUtensorMap* map, const void* src, int64_t rows, int64_t cols) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  hq_status s = tensor_map_encoder(&enc);
  if (s != HQ_OK) return s;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows / 64), 64};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(64 * cols * 2), static_cast<cuuint64_t>(cols * 2)};
  const cuuint32_t box[3] = {hq::dual::kStripCols, 4, 64};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(src), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
  return HQ_OK;
}

template <int K, int MODE, bool W32, bool SIGNED>
cudaError_t dual_smem_attr(DeviceInfo& d) {
  constexpr int kIdx = (K == 16 ? 0 : K == 32 ? 1 : K == 64 ? 2 : K == 128 ? 3 : 4);
  std::lock_guard<std::mutex> lock(g_mu);
  bool& done = d.dual_attr[kIdx][MODE][W32 ? 1 : 0][SIGNED ? 1 : 0];
  if (done) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(hq::dual::fwhtq_dual_kernel<K, MODE, W32, SIGNED>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(hq::dual::kSmemBytes));
  if (e == cudaSuccess) done = true;
  return e;
}

// The single-launch form (ONCHIP) for tensors of at most one 256 x 256 tile per SM, INT8 / FP8:
// a cooperative launch of one CTA per tile (all resident at once, which the grid barrier
// inside needs); the barrier counter is the last entry of the column rotation's partial array
// (the grid uses entries 0 .. grid - 1), zeroed here before the launch.
template <int K, int MODE, bool W32, bool SIGNED>
hq_status launch_dual_onchip(const CUtensorMap& map, int64_t rows, int64_t cols, uint8_t* codes_c, float* scale_c,
                             uint8_t* codes_r, float* scale_r, float* part_c, float* part_r, const uint8_t* neg_c,
                             const uint8_t* neg_r, DeviceInfo& d, cudaStream_t st, int g) {
  using namespace hq;
  using namespace hq::dual;
  auto kernel = fwhtq_dual_kernel<K, MODE, W32, SIGNED, true>;
  constexpr int kIdx = (K == 16 ? 0 : K == 32 ? 1 : K == 64 ? 2 : K == 128 ? 3 : 4);
  cudaError_t e;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    bool& done = d.dual_onchip_attr[kIdx][MODE == kModeInt8 ? 0 : 1][W32 ? 1 : 0][SIGNED ? 1 : 0];
    if (!done) {
      if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(kSmemBytes))) != cudaSuccess)
        return cuda_fail(e);
      done = true;
    }
  }
  unsigned int* counter = reinterpret_cast<unsigned int*>(part_c + (kMaxPartials - 1));
  if ((e = cudaMemsetAsync(counter, 0, sizeof(unsigned int), st)) != cudaSuccess) return cuda_fail(e);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(g);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kernel, map, rows, cols, codes_c, codes_r, part_c, part_r, g, scale_c, scale_r, d.status,
                         0, neg_c, neg_r, 0, counter);
  return e == cudaSuccess ? HQ_OK : cuda_fail(e);
}

// Pass 1 (both absmax partials, tiles in order) then pass 2 (both code tensors, tiles in
// reverse order), one CTA per SM.  W32: both code buffers are 32-byte aligned, so the code
// stores are whole 32-byte sectors.  SIGNED: the randomized variant (neg_c per column for the
// rotation along the columns, neg_r per row for the rotation along the rows).
template <int K, bool W32, bool SIGNED>
hq_status launch_dual_fused_w(const CUtensorMap& map, int64_t rows, int64_t cols, hq_fmt fmt, uint8_t* codes_c,
                              float* scale_c, uint8_t* codes_r, float* scale_r, float* part_c, float* part_r,
                              const uint8_t* neg_c, const uint8_t* neg_r, DeviceInfo& d, cudaStream_t st) {
  using namespace hq;
  using namespace hq::dual;
  const int64_t n_tiles = ((rows + kTile - 1) / kTile) * ((cols + kTile - 1) / kTile);
  const int g = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(n_tiles, d.sms)));
  // at most one tile per SM: both passes in one launch over tiles resident in shared memory
  if (n_tiles <= d.sms && fmt == HQ_INT8)
    return launch_dual_onchip<K, kModeInt8, W32, SIGNED>(map, rows, cols, codes_c, scale_c, codes_r, scale_r, part_c,
                                                         part_r, neg_c, neg_r, d, st, g);
  if (n_tiles <= d.sms && fmt == HQ_FP8_E4M3)
    return launch_dual_onchip<K, kModeFp8, W32, SIGNED>(map, rows, cols, codes_c, scale_c, codes_r, scale_r, part_c,
                                                        part_r, neg_c, neg_r, d, st, g);
  cudaError_t e = dual_smem_attr<K, kModeAbsmax, W32, SIGNED>(d);
  if (e != cudaSuccess) return cuda_fail(e);
  if ((e = launch_pdl(fwhtq_dual_kernel<K, kModeAbsmax, W32, SIGNED>, g, kThreads, kSmemBytes, st, map, rows, cols,
                      codes_c, codes_r, part_c, part_r, 0, scale_c, scale_r, d.status, 0, neg_c, neg_r, 0, nullptr)) !=
      cudaSuccess)
    return cuda_fail(e);
  if (fmt == HQ_INT8) {
    if ((e = dual_smem_attr<K, kModeInt8, W32, SIGNED>(d)) != cudaSuccess) return cuda_fail(e);
    e = launch_pdl(fwhtq_dual_kernel<K, kModeInt8, W32, SIGNED>, g, kThreads, kSmemBytes, st, map, rows, cols, codes_c,
                   codes_r, part_c, part_r, g, scale_c, scale_r, d.status, 1, neg_c, neg_r, 0, nullptr);
  } else if (fmt == HQ_FP8_E4M3) {
    if ((e = dual_smem_attr<K, kModeFp8, W32, SIGNED>(d)) != cudaSuccess) return cuda_fail(e);
    e = launch_pdl(fwhtq_dual_kernel<K, kModeFp8, W32, SIGNED>, g, kThreads, kSmemBytes, st, map, rows, cols, codes_c,
                   codes_r, part_c, part_r, g, scale_c, scale_r, d.status, 1, neg_c, neg_r, 0, nullptr);
  } else {
    if ((e = dual_smem_attr<K, kModeLowp, W32, SIGNED>(d)) != cudaSuccess) return cuda_fail(e);
    e = launch_pdl(fwhtq_dual_kernel<K, kModeLowp, W32, SIGNED>, g, kThreads, kSmemBytes, st, map, rows, cols, codes_c,
                   codes_r, part_c, part_r, g, scale_c, scale_r, d.status, 1, neg_c, neg_r, static_cast<int>(fmt), nullptr);
  }
  if (e != cudaSuccess) return cuda_fail(e);
  return HQ_OK;
}

template <int K>
hq_status launch_dual_fused(const CUtensorMap& map, int64_t rows, int64_t cols, hq_fmt fmt, uint8_t* codes_c,
                            float* scale_c, uint8_t* codes_r, float* scale_r, float* part_c, float* part_r,
                            const uint8_t* neg_c, const uint8_t* neg_r, DeviceInfo& d, cudaStream_t st) {
  const bool w32 = ((reinterpret_cast<uintptr_t>(codes_c) | reinterpret_cast<uintptr_t>(codes_r)) & 31u) == 0;
  if (neg_c || neg_r) {
    return w32 ? launch_dual_fused_w<K, true, true>(map, rows, cols, fmt, codes_c, scale_c, codes_r, scale_r, part_c,
                                                     part_r, neg_c, neg_r, d, st)
               : launch_dual_fused_w<K, false, true>(map, rows, cols, fmt, codes_c, scale_c, codes_r, scale_r, part_c,
                                                      part_r, neg_c, neg_r, d, st);
  }
  return w32 ? launch_dual_fused_w<K, true, false>(map, rows, cols, fmt, codes_c, scale_c, codes_r, scale_r, part_c,
                                                    part_r, nullptr, nullptr, d, st)
             : launch_dual_fused_w<K, false, false>(map, rows, cols, fmt, codes_c, scale_c, codes_r, scale_r, part_c,
                                                     part_r, nullptr, nullptr, d, st);
}

hq_status launch_dual_fused_k(const void* src, int64_t rows, int64_t cols, int k, hq_fmt fmt, uint8_t* codes_c,
                              float* scale_c, uint8_t* codes_r, float* scale_r, float* part_c, float* part_r,
                              const uint8_t* neg_c, const uint8_t* neg_r, DeviceInfo& d, cudaStream_t st) {
  CUtensorMap map;
  hq_status s = encode_dual_map(&map, src, rows, cols);
  if (s != HQ_OK) return s;
  switch (k) {
    case 16: return launch_dual_fused<16>(map, rows, cols, fmt, codes_c, scale_c, codes_r, scale_r, part_c, part_r, neg_c, neg_r, d, st);
    case 32: return launch_dual_fused<32>(map, rows, cols, fmt, codes_c, scale_c, codes_r, scale_r, part_c, part_r, neg_c, neg_r, d, st);
    case 64: return launch_dual_fused<64>(map, rows, cols, fmt, codes_c, scale_c, codes_r, scale_r, part_c, part_r, neg_c, neg_r, d, st);
    case 128: return launch_dual_fused<128>(map, rows, cols, fmt, codes_c, scale_c, codes_r, scale_r, part_c, part_r, neg_c, neg_r, d, st);
    default: return launch_dual_fused<256>(map, rows, cols, fmt, codes_c, scale_c, codes_r, scale_r, part_c, part_r, neg_c, neg_r, d, st);
  }
}

template <typename SrcT>
cudaError_t launch_dual_k(const void* src, int64_t rows, int64_t cols, int k, hq_fmt fmt, uint8_t* codes_c,
                          float* scale_c, uint8_t* codes_r, float* scale_r, float* part_c, float* part_r,
                          const uint8_t* neg_c, const uint8_t* neg_r, DeviceInfo& d, cudaStream_t st) {
  switch (k) {
    case 16: return launch_dual<SrcT, 16>(src, rows, cols, fmt, codes_c, scale_c, codes_r, scale_r, part_c, part_r, neg_c, neg_r, d, st);
    case 32: return launch_dual<SrcT, 32>(src, rows, cols, fmt, codes_c, scale_c, codes_r, scale_r, part_c, part_r, neg_c, neg_r, d, st);
    case 64: return launch_dual<SrcT, 64>(src, rows, cols, fmt, codes_c, scale_c, codes_r, scale_r, part_c, part_r, neg_c, neg_r, d, st);
    case 128: return launch_dual<SrcT, 128>(src, rows, cols, fmt, codes_c, scale_c, codes_r, scale_r, part_c, part_r, neg_c, neg_r, d, st);
    default: return launch_dual<SrcT, 256>(src, rows, cols, fmt, codes_c, scale_c, codes_r, scale_r, part_c, part_r, neg_c, neg_r, d, st);
  }
}

template <typename SrcT>
cudaError_t launch_quant_k(const void* src, int64_t rows, int64_t cols, int dim, int k, hq_fmt fmt,
                           uint8_t* codes, float* scale, float* partials, const uint8_t* neg, DeviceInfo& d,
                           cudaStream_t st) {
  switch (k) {
    case 16: return launch_quant<SrcT, 16>(src, rows, cols, dim, fmt, codes, scale, partials, neg, d, st);
    case 32: return launch_quant<SrcT, 32>(src, rows, cols, dim, fmt, codes, scale, partials, neg, d, st);
    case 64: return launch_quant<SrcT, 64>(src, rows, cols, dim, fmt, codes, scale, partials, neg, d, st);
    case 128: return launch_quant<SrcT, 128>(src, rows, cols, dim, fmt, codes, scale, partials, neg, d, st);
    default: return launch_quant<SrcT, 256>(src, rows, cols, dim, fmt, codes, scale, partials, neg, d, st);
  }
}

__global__ void set_scale_one_kernel(float* scale) { *scale = 1.0f; }
__global__ void set_zero_kernel(float* v) { *v = 0.0f; }

// Maximum of the absmax pass's per-CTA partials into one device scalar (a non-finite rotated
// value is already +inf in its partial).
__global__ void reduce_partials_kernel(const float* __restrict__ partials, int n, float* __restrict__ out) {
  float m = 0.0f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) m = fmaxf(m, partials[i]);
  __shared__ float scratch[32];
  m = hq::block_max(m, scratch);
  if (threadIdx.x == 0) *out = m;
}

// Split passes for sharded tensors: the absmax pass alone into a device scalar, and the code
// pass from a given absmax (one "partial", e.g. the maximum over ranks).
template <typename SrcT, int K>
cudaError_t launch_absmax_only(const void* src_v, int64_t rows, int64_t cols, int dim, float* partials,
                               const uint8_t* neg, float* absmax, DeviceInfo& d, cudaStream_t st) {
  int g = 0;
  cudaError_t e = launch_pass<SrcT, K, hq::kModeAbsmax>(static_cast<const SrcT*>(src_v), rows, cols, dim, nullptr,
                                                        nullptr, partials, 0, 0, neg, d, st, &g);
  if (e != cudaSuccess) return e;
  reduce_partials_kernel<<<1, 256, 0, st>>>(partials, g, absmax);
  return cudaGetLastError();
}

template <typename SrcT>
cudaError_t split_pass_k(bool codes_pass, const void* src, int64_t rows, int64_t cols, int dim, int k, hq_fmt fmt,
                         const uint8_t* neg, float* partials, float* absmax, uint8_t* codes, float* scale,
                         DeviceInfo& d, cudaStream_t st) {
  const SrcT* sp = static_cast<const SrcT*>(src);
#define HQ_SPLIT_CASE(KK)                                                                                     \
  case KK:                                                                                                    \
    return codes_pass ? launch_code_pass<SrcT, KK>(sp, rows, cols, dim, fmt, codes, scale, absmax, 1, 1, neg, d, st) \
                      : launch_absmax_only<SrcT, KK>(src, rows, cols, dim, partials, neg, absmax, d, st);
  switch (k) {
    HQ_SPLIT_CASE(16)
    HQ_SPLIT_CASE(32)
    HQ_SPLIT_CASE(64)
    HQ_SPLIT_CASE(128)
    default: HQ_SPLIT_CASE(256)
  }
#undef HQ_SPLIT_CASE
}

// The source side of a quantization: dtype, dim, k, sizes, the rotated dim's divisibility.
// `out` is the scalar the call writes (scale or absmax): non-null, 4-byte aligned.
hq_status check_src_args(const void* src, hq_dtype dt, int64_t rows, int64_t cols, int dim, int k, const float* out) {
  if (dt != HQ_F32 && dt != HQ_BF16) return HQ_ERR_DTYPE;
  if ((dim != 0 && dim != 1) || !valid_k(k)) return HQ_ERR_ARG;
  if (rows < 0 || cols < 0 || !out) return HQ_ERR_ARG;
  if (rows == 0 || cols == 0) return HQ_OK;
  if (!src) return HQ_ERR_ARG;
  if (dim == 1 && cols % k != 0) return HQ_ERR_SHAPE;
  if (dim == 0 && (rows % k != 0 || cols % 16 != 0)) return HQ_ERR_SHAPE;
  if (rows > (int64_t(1) << 40) / cols) return HQ_ERR_SHAPE;
  if (!aligned16(src) || (reinterpret_cast<uintptr_t>(out) & 3u)) return HQ_ERR_ALIGN;
  return HQ_OK;
}

hq_status check_quant_args(const void* src, hq_dtype dt, int64_t rows, int64_t cols, int dim, int k,
                           hq_fmt fmt, const void* codes, const float* scale) {
  if (dt != HQ_F32 && dt != HQ_BF16) return HQ_ERR_DTYPE;
  if (!valid_fmt(fmt)) return HQ_ERR_ARG;
  hq_status s = check_src_args(src, dt, rows, cols, dim, k, scale);
  if (s != HQ_OK || rows == 0 || cols == 0) return s;
  if (!codes) return HQ_ERR_ARG;
  if (!aligned16(codes)) return HQ_ERR_ALIGN;
  return HQ_OK;
}

hq_status quantize_impl(const void* src, hq_dtype dt, int64_t rows, int64_t cols, int dim, int k,
                        hq_fmt fmt, void* codes, float* scale, float* partials, DeviceInfo& d,
                        cudaStream_t st, const uint8_t* neg = nullptr) {
  if (rows == 0 || cols == 0) {
    set_scale_one_kernel<<<1, 1, 0, st>>>(scale);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? HQ_OK : cuda_fail(e);
  }
  cudaError_t e = (dt == HQ_BF16)
                      ? launch_quant_k<__nv_bfloat16>(src, rows, cols, dim, k, fmt, static_cast<uint8_t*>(codes), scale, partials, neg, d, st)
                      : launch_quant_k<float>(src, rows, cols, dim, k, fmt, static_cast<uint8_t*>(codes), scale, partials, neg, d, st);
  return e == cudaSuccess ? HQ_OK : cuda_fail(e);
}

// ------------------------------------------------------------------ GEMM launches

hq_status encode_codes_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  hq_status s = tensor_map_encoder(&enc);
  if (s != HQ_OK) return s;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(hq::gemm::BK), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
  return HQ_OK;
}

// bf16 output [rows][cols] as 32-row x 64-column boxes (128-byte rows, 128-byte swizzle) for
// the pair GEMM's TMA-store epilogue.
hq_status encode_out_map(CUtensorMap* map, void* base, int64_t rows, int64_t cols) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  hq_status s = tensor_map_encoder(&enc);
  if (s != HQ_OK) return s;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  const cuuint32_t box[2] = {64, 32};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
  return HQ_OK;
}

template <int FMT, int OUT>
cudaError_t launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const float* sa, const float* sb,
                        void* out, int M, int N, int K, DeviceInfo& d, cudaStream_t st, uint32_t ab_code,
                        int skip_first_load = 0) {
  auto kernel = hq::gemm::gemm_kernel<FMT, OUT>;
  const unsigned bit = 1u << (FMT * 2 + OUT);
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!(d.gemm_attr_set & bit)) {
      cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(hq::gemm::SMEM_BYTES));
      if (e != cudaSuccess) return e;
      d.gemm_attr_set |= bit;
    }
  }
  const int tiles = ((M + hq::gemm::BM - 1) / hq::gemm::BM) * ((N + hq::gemm::BN - 1) / hq::gemm::BN);
  const int grid = std::max(1, std::min(tiles, d.sms));
  kernel<<<grid, hq::gemm::NUM_THREADS, hq::gemm::SMEM_BYTES, st>>>(ta, tb, sa, sb, out, M, N, K, d.status,
                                                                     skip_first_load, ab_code);
  return cudaGetLastError();
}

hq_status check_gemm_args(const void* A, const float* sa, const void* B, const float* sb, int64_t M,
                          int64_t N, int64_t K, hq_fmt fmt, hq_out ok, const void* out) {
  if (!valid_fmt(fmt) || (ok != HQ_OUT_BF16 && ok != HQ_OUT_ACC)) return HQ_ERR_ARG;
  if (M < 0 || N < 0 || K < 0) return HQ_ERR_ARG;
  if (M == 0 || N == 0) return HQ_OK;
  if (!out) return HQ_ERR_ARG;
  if (K > 0 && (!A || !B)) return HQ_ERR_ARG;
  if (ok == HQ_OUT_BF16 && (!sa || !sb)) return HQ_ERR_ARG;
  if (K % 16 != 0 || N % 16 != 0) return HQ_ERR_SHAPE;
  if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31)) return HQ_ERR_SHAPE;
  if (fmt == HQ_INT8 && K > HQ_MAX_K_INT8) return HQ_ERR_SHAPE;
  if (!aligned16(out) || (K > 0 && (!aligned16(A) || !aligned16(B)))) return HQ_ERR_ALIGN;
  if ((sa && (reinterpret_cast<uintptr_t>(sa) & 3u)) || (sb && (reinterpret_cast<uintptr_t>(sb) & 3u))) return HQ_ERR_ALIGN;
  return HQ_OK;
}

// Co-resident 2-CTA clusters of a pair-GEMM instantiation (cached per device).
int pair_clusters(const void* kernel, size_t smem, int sms, int threads) {
  static std::mutex mu;
  static const void* keys[64];
  static int devs[64], vals[64];
  static int n = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n; ++i)
    if (keys[i] == kernel && devs[i] == dev) return vals[i];
  cudaLaunchConfig_t q = {};
  q.gridDim = dim3(2 * (sms / 2));
  q.blockDim = dim3(threads);
  q.dynamicSmemBytes = smem;
  cudaLaunchAttribute qa[1];
  qa[0].id = cudaLaunchAttributeClusterDimension;
  qa[0].val.clusterDim.x = 2;
  qa[0].val.clusterDim.y = 1;
  qa[0].val.clusterDim.z = 1;
  q.attrs = qa;
  q.numAttrs = 1;
  int c = 0;
  if (cudaOccupancyMaxActiveClusters(&c, kernel, &q) != cudaSuccess || c < 1) c = sms / 2;
  if (n < 64) {
    keys[n] = kernel;
    devs[n] = dev;
    vals[n] = c;
    ++n;
  }
  return c;
}

template <int FMT, int OUT, int BN, bool SK, bool MN = false>
cudaError_t launch_gemm_pair(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& to, const float* sa,
                             const float* sb, void* out, int M, int N, int K, int clusters, int split_from,
                             uint32_t* part_ws, int* counters, uint32_t ab_code, DeviceInfo& d, cudaStream_t st,
                             int rot_k = 0) {
  namespace gp = hq::gemm::pair;
  using G = gp::Geo<BN, SK>;
  auto kernel = gp::gemm_pair_kernel<FMT, OUT, BN, SK, MN>;
  const int tiles = ((M + gp::BM - 1) / gp::BM) * ((N + BN - 1) / BN);
  const int f = std::min(split_from, tiles);
  const int items = f + 2 * (tiles - f);  // whole tiles, then both halves of each split one
  const int pairs = std::max(1, std::min(items, clusters));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(G::THREADS);
  cfg.dynamicSmemBytes = G::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see griddep_wait in the kernel
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  (void)d;
  return cudaLaunchKernelEx(&cfg, kernel, ta, tb, to, sa, sb, out, M, N, K, d.status, split_from, part_ws, counters,
                            ab_code, rot_k);
}

// Dynamic shared memory of every pair-GEMM instantiation enabled once per device.
template <int FMT, int OUT, int BN, bool SK>
cudaError_t pair_prepare(DeviceInfo& d, int* clusters) {
  namespace gp = hq::gemm::pair;
  using G = gp::Geo<BN, SK>;
  auto kernel = gp::gemm_pair_kernel<FMT, OUT, BN, SK>;
  const unsigned bit = 1u << (((FMT * 2 + OUT) * 2 + (BN == 256 ? 0 : 1)) * 2 + (SK ? 1 : 0));
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!(d.pair_attr_set & bit)) {
      cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(G::SMEM_BYTES));
      if (e != cudaSuccess) return e;
      d.pair_attr_set |= bit;
    }
  }
  *clusters = pair_clusters(reinterpret_cast<const void*>(kernel), G::SMEM_BYTES, d.sms, G::THREADS);
  return cudaSuccess;
}

// N tile of the pair GEMM: whichever of 256 and 128 finishes in fewer tile-times, counting
// whole waves of `clusters`.  A 128-wide tile takes 0.78 of a 256-wide one's time on B200
// (it needs 1.5x the operand bytes per MAC; measured on the 4096^2 x 11008 dX GEMM: 196 us
// with 128-wide tiles in 7 waves against 126 us with 256-wide tiles in 4), so 128 wins only
// when there are fewer 256-wide tiles than clusters.  Ties keep 256.
int pick_pair_bn(int M, int N, int clusters) {
  const int m_tiles = (M + hq::gemm::pair::BM - 1) / hq::gemm::pair::BM;
  const int64_t w256 = (int64_t(m_tiles) * ((N + 255) / 256) + clusters - 1) / clusters;
  const int64_t w128 = (int64_t(m_tiles) * ((N + 127) / 128) + clusters - 1) / clusters;
  return (double(w128) * 0.78 < double(w256)) ? 128 : 256;
}

// GEMMs with at least one full 256-row pair tile run on CTA pairs; smaller M on single CTAs.
constexpr int64_t kPairMinRows = 256;

// Split contraction for GEMMs with too few 256 x 256 tiles to fill the clusters (the weight
// gradient of a layer with few outputs and many tokens): two halves of the k-blocks per tile,
// when that at least cuts the waves by 30% (so the exchange of fp32/int32 partials pays off)
// and each half keeps 8 or more k-blocks.  Workspace: both halves' partial tiles (fp32/int32)
// and one arrival counter per 32-row slab.
constexpr int kRefClusters = 74;  // workspace sizing: the clusters of a 148-SM B200

int pick_splits(int64_t M, int64_t N, int64_t K, int clusters) {
  if (M < kPairMinRows || clusters <= 0) return 1;
  const int64_t num_kb = (K + hq::gemm::BK - 1) / hq::gemm::BK;
  if (num_kb < 16) return 1;
  const int64_t tiles = ((M + 255) / 256) * ((N + 255) / 256);
  const int64_t w1 = (tiles + clusters - 1) / clusters, w2 = (2 * tiles + clusters - 1) / clusters;
  return double(w2) * 0.5 <= 0.7 * double(w1) ? 2 : 1;
}

// The first tile split in two along the contraction (the pair kernel's split_from; the
// number of 256 x 256 tiles when none is):
//  - every tile, when pick_splits says so;
//  - otherwise the tiles of the last, partial wave, when they fill at most half the clusters,
//    there are at most three full waves before them and the contraction has 64 or more
//    k-blocks. The halves then all run in one wave of half a tile-time.
// The exchange of partials and the counter reset cost about 8 us. Measured with INT8 on a
// B200 (74 clusters), plain -> split:
//   4096 x 4096 x 11008 (3.46 waves):  121.2 -> 116.6 us;
//   4096 x 4096 x 4096 (3.46 waves):    53.5 -> 57.3 us;
//   4096 x 11008 x 4096 (9.3 waves):   116.0 -> 118.9 us.
// Hence the limits above.
int64_t pick_split_from(int64_t M, int64_t N, int64_t K, int clusters) {
  const int64_t tiles = ((M + 255) / 256) * ((N + 255) / 256);
  if (M < kPairMinRows || clusters <= 0) return tiles;
  if (pick_splits(M, N, K, clusters) == 2) return 0;
  const int64_t num_kb = (K + hq::gemm::BK - 1) / hq::gemm::BK;
  if (num_kb < 64) return tiles;
  const int64_t full = tiles / clusters, tail = tiles - full * clusters;
  return (full >= 1 && full <= 3 && tail > 0 && 2 * tail <= clusters) ? tiles - tail : tiles;
}

// Partial accumulators of t split tiles (both halves, fp32 / int32) and their arrival
// counters (one per 32-row slab).
size_t split_part_bytes(int64_t t) { return size_t(2) * size_t(t) * 256 * 256 * 4; }
size_t split_counter_bytes(int64_t t) { return align_up(size_t(t) * 8 * sizeof(int)); }

// Workspace a GEMM of the layer may use for a split contraction (0 when it never splits).
size_t split_ws_bytes(int64_t M, int64_t N, int64_t K) {
  const int64_t tiles = ((M + 255) / 256) * ((N + 255) / 256);
  const int64_t t = tiles - pick_split_from(M, N, K, kRefClusters);
  if (t <= 0) return 0;
  return split_part_bytes(t) + split_counter_bytes(t);
}

hq_status gemm_impl(const void* A, const float* sa, const void* B, const float* sb, int64_t M, int64_t N,
                    int64_t K, hq_fmt fmt, hq_out ok, void* out, DeviceInfo& d, cudaStream_t st,
                    void* split_ws = nullptr, size_t split_ws_len = 0) {
  if (M == 0 || N == 0) return HQ_OK;
  if (K == 0) {
    const size_t elem = ok == HQ_OUT_BF16 ? 2 : 4;
    cudaError_t e = cudaMemsetAsync(out, 0, size_t(M) * size_t(N) * elem, st);
    return e == cudaSuccess ? HQ_OK : cuda_fail(e);
  }
  const bool pair = M >= kPairMinRows;
  const int m = static_cast<int>(M), n = static_cast<int>(N), kk = static_cast<int>(K);
  const uint32_t ab = ab_format_code(fmt);
  using namespace hq::gemm;
  cudaError_t e;
  int bn = 256, clusters = 0;
  // short contractions whose output is bf16 use the SHORT_K shape (fewer operand stages, the
  // whole output tile staged for TMA stores)
  const bool sk = pair && ok == HQ_OUT_BF16 && (K + hq::gemm::BK - 1) / hq::gemm::BK <= hq::gemm::pair::kShortKBlocks;
  if (pair) {
    // both N tiles of the chosen instantiation are prepared; the cluster counts are equal in
    // practice (one CTA per SM either way)
#define HQ_PAIR_PREP(F, O, SKV)                                        \
  e = pair_prepare<F, O, 256, SKV>(d, &clusters);                      \
  if (e == cudaSuccess) { int c2; e = pair_prepare<F, O, 128, SKV>(d, &c2); }
    if (fmt == HQ_INT8) {
      if (ok == HQ_OUT_ACC) { HQ_PAIR_PREP(kInt8, kOutAcc, false) }
      else if (sk) { HQ_PAIR_PREP(kInt8, kOutBf16, true) }
      else { HQ_PAIR_PREP(kInt8, kOutBf16, false) }
    } else {
      if (ok == HQ_OUT_ACC) { HQ_PAIR_PREP(kFp8, kOutAcc, false) }
      else if (sk) { HQ_PAIR_PREP(kFp8, kOutBf16, true) }
      else { HQ_PAIR_PREP(kFp8, kOutBf16, false) }
    }
#undef HQ_PAIR_PREP
    if (e != cudaSuccess) return cuda_fail(e);
    bn = pick_pair_bn(m, n, clusters);
  }
  const int64_t tiles256 = ((M + 255) / 256) * ((N + 255) / 256);
  int split_from = INT_MAX;  // no split
  uint32_t* part_ws = nullptr;
  int* counters = nullptr;
  if (pair && !sk && ok == HQ_OUT_BF16 && split_ws) {
    const int64_t f = pick_split_from(M, N, K, clusters), t = tiles256 - f;
    if (t > 0 && split_ws_len >= split_part_bytes(t) + split_counter_bytes(t)) {
      split_from = static_cast<int>(f);
      bn = 256;
      counters = static_cast<int*>(split_ws);
      part_ws = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(split_ws) + split_counter_bytes(t));
      e = cudaMemsetAsync(counters, 0, split_counter_bytes(t), st);
      if (e != cudaSuccess) return cuda_fail(e);
    }
  }
  CUtensorMap ta, tb;
  hq_status s = encode_codes_map(&ta, A, M, K, pair ? hq::gemm::pair::HALF : hq::gemm::BM);
  if (s != HQ_OK) return s;
  if ((s = encode_codes_map(&tb, B, N, K, pair ? uint32_t(bn / 2) : uint32_t(hq::gemm::BN))) != HQ_OK) return s;
  if (pair) {
    CUtensorMap to;  // read by the bf16 epilogue only
    std::memset(&to, 0, sizeof(to));
    if (ok == HQ_OUT_BF16 && (s = encode_out_map(&to, out, M, N)) != HQ_OK) return s;
#define HQ_PAIR_LAUNCH(F, O, SKV)                                                                       \
  (bn == 256 ? launch_gemm_pair<F, O, 256, SKV>(ta, tb, to, sa, sb, out, m, n, kk, clusters, split_from, part_ws, \
                                                counters, ab, d, st)                                         \
             : launch_gemm_pair<F, O, 128, SKV>(ta, tb, to, sa, sb, out, m, n, kk, clusters, split_from, part_ws, \
                                                counters, ab, d, st))
    if (fmt == HQ_INT8)
      e = ok == HQ_OUT_ACC ? HQ_PAIR_LAUNCH(kInt8, kOutAcc, false)
          : sk             ? HQ_PAIR_LAUNCH(kInt8, kOutBf16, true)
                           : HQ_PAIR_LAUNCH(kInt8, kOutBf16, false);
    else
      e = ok == HQ_OUT_ACC ? HQ_PAIR_LAUNCH(kFp8, kOutAcc, false)
          : sk             ? HQ_PAIR_LAUNCH(kFp8, kOutBf16, true)
                           : HQ_PAIR_LAUNCH(kFp8, kOutBf16, false);
#undef HQ_PAIR_LAUNCH
  } else {
    if (fmt == HQ_INT8)
      e = ok == HQ_OUT_BF16 ? launch_gemm<kInt8, kOutBf16>(ta, tb, sa, sb, out, m, n, kk, d, st, 0)
                            : launch_gemm<kInt8, kOutAcc>(ta, tb, sa, sb, out, m, n, kk, d, st, 0);
    else
      e = ok == HQ_OUT_BF16 ? launch_gemm<kFp8, kOutBf16>(ta, tb, sa, sb, out, m, n, kk, d, st, ab)
                            : launch_gemm<kFp8, kOutAcc>(ta, tb, sa, sb, out, m, n, kk, d, st, ab);
  }
  return e == cudaSuccess ? HQ_OK : cuda_fail(e);
}

// ------------------------------------------------------------------ rotated-output placement

// out[M][N] fp32 = fp32(sum_l A[l][i] B[l][j]) * fp32(s_a * s_b) with both operands stored
// contraction-outermost: A as [K][M], B as [K][N] (the token-rotated output-gradient codes and
// the forward's K-rotated weight codes); CTA pairs, 256 x 256 tiles.  rot_k != 0: the output
// leaves the epilogue rotated along its columns in blocks of rot_k (N % rot_k == 0).
hq_status gemm_mn_f32_impl(const void* A, const float* sa, const void* B, const float* sb, int64_t M, int64_t N,
                           int64_t K, hq_fmt fmt, float* out, DeviceInfo& d, cudaStream_t st, int rot_k) {
  namespace gp = hq::gemm::pair;
  using G = gp::Geo<256, false>;
  const int f = fmt == HQ_INT8 ? 0 : 1;
  const void* kernel = f == 0 ? reinterpret_cast<const void*>(gp::gemm_pair_kernel<hq::gemm::kInt8, hq::gemm::kOutF32, 256, false, true>)
                              : reinterpret_cast<const void*>(gp::gemm_pair_kernel<hq::gemm::kFp8, hq::gemm::kOutF32, 256, false, true>);
  cudaError_t e;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!d.mn_attr[f]) {
      if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(G::SMEM_BYTES))) != cudaSuccess)
        return cuda_fail(e);
      d.mn_attr[f] = true;
    }
  }
  const int clusters = pair_clusters(kernel, G::SMEM_BYTES, d.sms, G::THREADS);
  CUtensorMap ta, tb, to;
  std::memset(&to, 0, sizeof(to));
  // boxes of 128 contraction rows x 128 bytes along M (N): the K-major map with the roles of
  // its two dimensions exchanged
  hq_status s = encode_codes_map(&ta, A, K, M, gp::HALF);
  if (s != HQ_OK) return s;
  if ((s = encode_codes_map(&tb, B, K, N, G::B_ROWS)) != HQ_OK) return s;
  const int m = static_cast<int>(M), n = static_cast<int>(N), kk = static_cast<int>(K);
  e = f == 0 ? launch_gemm_pair<hq::gemm::kInt8, hq::gemm::kOutF32, 256, false, true>(
                   ta, tb, to, sa, sb, out, m, n, kk, clusters, INT_MAX, nullptr, nullptr, 0u, d, st, rot_k)
             : launch_gemm_pair<hq::gemm::kFp8, hq::gemm::kOutF32, 256, false, true>(
                   ta, tb, to, sa, sb, out, m, n, kk, clusters, INT_MAX, nullptr, nullptr, 0u, d, st, rot_k);
  return e == cudaSuccess ? HQ_OK : cuda_fail(e);
}

template <int K>
cudaError_t launch_derotate_k(float* z, int64_t rows, int64_t cols, __nv_bfloat16* out, DeviceInfo& d,
                              cudaStream_t st) {
  const float c = static_cast<float>(1.0 / std::sqrt(static_cast<double>(K)));  // fp32(1/sqrt(k)), one rounding
  cudaError_t e;
  namespace hr = hq::rot;
  const size_t smem = K >= 64 ? hr::kRowsSmemBytes : 0;
  if (K >= 64) {
    std::lock_guard<std::mutex> lock(g_mu);
    const int ki = K == 64 ? 0 : K == 128 ? 1 : 2;
    if (!d.rot_attr[ki]) {
      if ((e = cudaFuncSetAttribute(hr::rot_rows_f32_bf16_kernel<K>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(smem))) != cudaSuccess)
        return e;
      d.rot_attr[ki] = true;
    }
  }
  const int64_t blocks_r = ((rows + hr::kRowTile - 1) / hr::kRowTile) * ((cols + hr::kColTile - 1) / hr::kColTile);
  hr::rot_rows_f32_bf16_kernel<K><<<static_cast<unsigned>(blocks_r), hr::kThreads, smem, st>>>(z, rows, cols, c, out);
  return cudaGetLastError();
}

// out = bf16(H Z) for Z already rotated along its columns (by the GEMM's epilogue): the rows'
// rotation, rounded to bf16.
hq_status derotate_impl(float* z, int64_t rows, int64_t cols, int k, void* out, DeviceInfo& d, cudaStream_t st) {
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out);
  cudaError_t e;
  switch (k) {
    case 16: e = launch_derotate_k<16>(z, rows, cols, o, d, st); break;
    case 32: e = launch_derotate_k<32>(z, rows, cols, o, d, st); break;
    case 64: e = launch_derotate_k<64>(z, rows, cols, o, d, st); break;
    case 128: e = launch_derotate_k<128>(z, rows, cols, o, d, st); break;
    default: e = launch_derotate_k<256>(z, rows, cols, o, d, st); break;
  }
  return e == cudaSuccess ? HQ_OK : cuda_fail(e);
}

// Shape rules of the reuse placement's dX: M and K are rotated (multiples of k and below 2^31),
// N is the contraction.
hq_status check_dx_reuse_shape(int64_t M, int64_t K, int64_t N, int k, hq_fmt fmt) {
  if (!valid_k(k) || (fmt != HQ_INT8 && fmt != HQ_FP8_E4M3)) return HQ_ERR_ARG;
  if (M < 0 || K < 0 || N < 0) return HQ_ERR_ARG;
  if (M == 0 || K == 0 || N == 0) return HQ_ERR_SHAPE;
  if (M % k || K % k) return HQ_ERR_SHAPE;
  if (fmt == HQ_INT8 && N > HQ_MAX_K_INT8) return HQ_ERR_SHAPE;
  if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31)) return HQ_ERR_SHAPE;
  return HQ_OK;
}

hq_status dx_reuse_impl(const void* g_codes, const float* g_scale, const void* wq_codes, const float* wq_scale,
                        int64_t M, int64_t K, int64_t N, int k, hq_fmt fmt, void* dX, float* z, DeviceInfo& d,
                        cudaStream_t st) {
  hq_status s = gemm_mn_f32_impl(g_codes, g_scale, wq_codes, wq_scale, M, K, N, fmt, z, d, st, k);
  if (s != HQ_OK) return s;
  return derotate_impl(z, M, K, k, dX, d, st);
}

// ------------------------------------------------------------------ next layer's rotation in the epilogue

// out[M][N] fp32 = blockdiag(H_k / sqrt(k)) applied along the columns of
// fp32(sum_l A[i][l] B[j][l]) * fp32(s_a * s_b): both operands K-major, CTA pairs, 256-wide tiles.
hq_status gemm_rotout_impl(const void* A, const float* sa, const void* B, const float* sb, int64_t M, int64_t N,
                           int64_t K, int k, hq_fmt fmt, float* out, DeviceInfo& d, cudaStream_t st) {
  namespace gp = hq::gemm::pair;
  using G = gp::Geo<256, false>;
  const int f = fmt == HQ_INT8 ? 0 : 1;
  const void* kernel = f == 0 ? reinterpret_cast<const void*>(gp::gemm_pair_kernel<hq::gemm::kInt8, hq::gemm::kOutF32, 256, false, false>)
                              : reinterpret_cast<const void*>(gp::gemm_pair_kernel<hq::gemm::kFp8, hq::gemm::kOutF32, 256, false, false>);
  cudaError_t e;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!d.rotout_attr[f]) {
      if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(G::SMEM_BYTES))) != cudaSuccess)
        return cuda_fail(e);
      d.rotout_attr[f] = true;
    }
  }
  const int clusters = pair_clusters(kernel, G::SMEM_BYTES, d.sms, G::THREADS);
  CUtensorMap ta, tb, to;
  std::memset(&to, 0, sizeof(to));
  hq_status s = encode_codes_map(&ta, A, M, K, gp::HALF);
  if (s != HQ_OK) return s;
  if ((s = encode_codes_map(&tb, B, N, K, G::B_ROWS)) != HQ_OK) return s;
  const int m = static_cast<int>(M), n = static_cast<int>(N), kk = static_cast<int>(K);
  e = f == 0 ? launch_gemm_pair<hq::gemm::kInt8, hq::gemm::kOutF32, 256, false>(
                   ta, tb, to, sa, sb, out, m, n, kk, clusters, INT_MAX, nullptr, nullptr, 0u, d, st, k)
             : launch_gemm_pair<hq::gemm::kFp8, hq::gemm::kOutF32, 256, false>(
                   ta, tb, to, sa, sb, out, m, n, kk, clusters, INT_MAX, nullptr, nullptr, 0u, d, st, k);
  return e == cudaSuccess ? HQ_OK : cuda_fail(e);
}

// Tensor-wise INT8 / e4m3 codes of n already-rotated fp32 values (n % 4 == 0, n > 0).
hq_status prerot_quant_impl(const float* y, int64_t n, hq_fmt fmt, void* codes, float* scale, float* partials,
                            DeviceInfo& d, cudaStream_t st) {
  namespace pr = hq::prerot;
  const int64_t n4 = n / 4;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((n4 + pr::kThreads - 1) / pr::kThreads,
                                                                           int64_t(d.sms) * 4)));
  uint8_t* c = static_cast<uint8_t*>(codes);
  pr::prerot_quant_kernel<hq::kModeAbsmax><<<grid, pr::kThreads, 0, st>>>(y, n4, c, partials, grid, scale, d.status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  if (fmt == HQ_INT8)
    pr::prerot_quant_kernel<hq::kModeInt8><<<grid, pr::kThreads, 0, st>>>(y, n4, c, partials, grid, scale, d.status);
  else
    pr::prerot_quant_kernel<hq::kModeFp8><<<grid, pr::kThreads, 0, st>>>(y, n4, c, partials, grid, scale, d.status);
  e = cudaGetLastError();
  return e == cudaSuccess ? HQ_OK : cuda_fail(e);
}

// ------------------------------------------------------------------ the linear layer

struct LinearWs {
  uint8_t* codes_a;
  uint8_t* codes_b;
  float* scale_a;
  float* scale_b;
  float* partials;
  void* split;  // split-contraction scratch of the GEMM (split_len bytes, may be 0)
  size_t split_len;
};

size_t linear_ws_bytes(int64_t a_bytes, int64_t b_bytes, size_t split_bytes) {
  return align_up(size_t(a_bytes)) + align_up(size_t(b_bytes)) + kAlign + kPartialBytes + align_up(split_bytes);
}

hq_status carve_linear_ws(void* ws, size_t ws_bytes, int64_t a_bytes, int64_t b_bytes, size_t split_bytes,
                          LinearWs* out) {
  if (!ws || ws_bytes < linear_ws_bytes(a_bytes, b_bytes, split_bytes)) return HQ_ERR_WORKSPACE;
  if (!aligned16(ws)) return HQ_ERR_ALIGN;
  uint8_t* p = static_cast<uint8_t*>(ws);
  out->codes_a = p;
  p += align_up(size_t(a_bytes));
  out->codes_b = p;
  p += align_up(size_t(b_bytes));
  out->scale_a = reinterpret_cast<float*>(p);
  out->scale_b = reinterpret_cast<float*>(p) + 4;
  p += kAlign;
  out->partials = reinterpret_cast<float*>(p);
  p += kPartialBytes;
  out->split = split_bytes ? p : nullptr;
  out->split_len = split_bytes;
  return HQ_OK;
}

struct Operand {
  const void* src;
  int64_t rows, cols;
  int dim;
};

// Quantize both operands along the shared contraction dimension, then run the GEMM.
hq_status linear_gemm(Operand a, Operand b, int64_t gm, int64_t gn, int64_t gk, hq_dtype dt, int k,
                      hq_fmt fmt, void* out, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (dt != HQ_F32 && dt != HQ_BF16) return HQ_ERR_DTYPE;
  if (!valid_k(k) || !valid_fmt(fmt)) return HQ_ERR_ARG;
  if (gm < 0 || gn < 0 || gk < 0) return HQ_ERR_ARG;
  if (gm % k || gn % k || gk % k) return HQ_ERR_SHAPE;
  if (gm == 0 || gn == 0) return HQ_OK;
  if (!out) return HQ_ERR_ARG;
  if (gk > 0 && (!a.src || !b.src)) return HQ_ERR_ARG;
  if (fmt == HQ_INT8 && gk > HQ_MAX_K_INT8) return HQ_ERR_SHAPE;
  if (gm >= (int64_t(1) << 31) || gn >= (int64_t(1) << 31) || gk >= (int64_t(1) << 31)) return HQ_ERR_SHAPE;
  if (!aligned16(out) || (gk > 0 && (!aligned16(a.src) || !aligned16(b.src)))) return HQ_ERR_ALIGN;
  LinearWs w;
  hq_status s = carve_linear_ws(ws, ws_bytes, gm * gk, gn * gk, split_ws_bytes(gm, gn, gk), &w);
  if (s != HQ_OK) return s;
  DeviceInfo* d = nullptr;
  if ((s = device_info(&d)) != HQ_OK) return s;
  if (gk > 0) {
    if ((s = quantize_impl(a.src, dt, a.rows, a.cols, a.dim, k, fmt, w.codes_a, w.scale_a, w.partials, *d, st)) != HQ_OK) return s;
    if ((s = quantize_impl(b.src, dt, b.rows, b.cols, b.dim, k, fmt, w.codes_b, w.scale_b, w.partials, *d, st)) != HQ_OK) return s;
  }
  return gemm_impl(w.codes_a, w.scale_a, w.codes_b, w.scale_b, gm, gn, gk, fmt, HQ_OUT_BF16, out, *d, st,
                   w.split, w.split_len);
}

// ------------------------------------------------------------------ quantize once, both rotations

hq_status check_dual_args(const void* src, hq_dtype dt, int64_t rows, int64_t cols, int k, hq_fmt fmt,
                          const void* codes_c, const float* scale_c, const void* codes_r, const float* scale_r) {
  if (dt != HQ_F32 && dt != HQ_BF16) return HQ_ERR_DTYPE;
  if (!valid_k(k) || !valid_fmt(fmt)) return HQ_ERR_ARG;
  if (rows < 0 || cols < 0 || !scale_c || !scale_r) return HQ_ERR_ARG;
  if (rows == 0 || cols == 0) return HQ_OK;
  if (!src || !codes_c || !codes_r) return HQ_ERR_ARG;
  if (rows % k != 0 || cols % k != 0) return HQ_ERR_SHAPE;
  if (rows > (int64_t(1) << 40) / cols) return HQ_ERR_SHAPE;
  if (!aligned16(src) || !aligned16(codes_c) || !aligned16(codes_r)) return HQ_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(scale_c) & 3u) || (reinterpret_cast<uintptr_t>(scale_r) & 3u)) return HQ_ERR_ALIGN;
  return HQ_OK;
}

hq_status dual_impl(const void* src, hq_dtype dt, int64_t rows, int64_t cols, int k, hq_fmt fmt, void* codes_c,
                    float* scale_c, void* codes_r, float* scale_r, float* part_c, float* part_r, DeviceInfo& d,
                    cudaStream_t st, const uint8_t* neg_c = nullptr, const uint8_t* neg_r = nullptr) {
  if (rows == 0 || cols == 0) {
    set_scale_one_kernel<<<1, 1, 0, st>>>(scale_c);
    set_scale_one_kernel<<<1, 1, 0, st>>>(scale_r);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? HQ_OK : cuda_fail(e);
  }
  uint8_t* cc = static_cast<uint8_t*>(codes_c);
  uint8_t* cr = static_cast<uint8_t*>(codes_r);
  if (dt == HQ_BF16 && fused_dual_ok(rows, cols))
    return launch_dual_fused_k(src, rows, cols, k, fmt, cc, scale_c, cr, scale_r, part_c, part_r, neg_c, neg_r, d, st);
  cudaError_t e = dt == HQ_BF16
                      ? launch_dual_k<__nv_bfloat16>(src, rows, cols, k, fmt, cc, scale_c, cr, scale_r, part_c, part_r, neg_c, neg_r, d, st)
                      : launch_dual_k<float>(src, rows, cols, k, fmt, cc, scale_c, cr, scale_r, part_c, part_r, neg_c, neg_r, d, st);
  return e == cudaSuccess ? HQ_OK : cuda_fail(e);
}

// Per-device side stream of hq_linear_fwd_bwd (created on first use, kept until exit) and the
// events that fork it from / join it to the caller's stream.  Enqueueing is serialised by a
// mutex, so concurrent callers on one device interleave correctly (their side work shares
// the one side stream).
struct SideStream {
  bool ready = false;
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join_dx = nullptr, join_dw = nullptr;
};
SideStream g_side[kMaxDevices];
std::mutex g_side_mu;

hq_status side_stream(SideStream** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return HQ_ERR_UNSUPPORTED;
  SideStream& ss = g_side[dev];
  if (!ss.ready) {
    if ((e = cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking)) != cudaSuccess) return cuda_fail(e);
    for (cudaEvent_t* ev : {&ss.fork, &ss.join_dx, &ss.join_dw})
      if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess) return cuda_fail(e);
    ss.ready = true;
  }
  *out = &ss;
  return HQ_OK;
}

// Workspace of hq_linear_fwd_bwd: six code tensors, six scales, four partial buffers (one
// pair per stream).
struct StepWs {
  uint8_t *xq, *xqt, *wq, *wqt, *dyq, *dyqt;
  float* scales;  // x_c, x_r, w_c, w_r, dy_c, dy_r
  float *part_c, *part_r;    // caller's stream
  float *spart_c, *spart_r;  // side stream
  void* split;  // split-contraction scratch shared by the GEMMs (they run in stream order)
  size_t split_len;
};

// The layer step quantizes X and W with the two-rotation kernel when both are bf16 tensors
// with dimensions of at least 2048 (multiples of 64) and k <= 128: there one call was measured
// 4-25 % faster than the two single-rotation calls (each of which reads the source twice).  At
// k = 256 the two were within a few percent of each other, the single-rotation calls ahead on
// tensors up to 50 M elements, and on narrow tensors (768-wide ViT layers) the single-rotation
// calls were faster at every k.
bool step_dual_ok(hq_dtype dt, int64_t rows, int64_t cols, int k) {
  return dt == HQ_BF16 && fused_dual_ok(rows, cols) && rows >= 2048 && cols >= 2048 && k <= 128;
}

size_t step_split_bytes(int64_t M, int64_t K, int64_t N) {
  return std::max({split_ws_bytes(M, N, K), split_ws_bytes(M, K, N), split_ws_bytes(N, K, M)});
}

size_t step_ws_bytes(int64_t M, int64_t K, int64_t N) {
  return 2 * (align_up(size_t(M * K)) + align_up(size_t(N * K)) + align_up(size_t(M * N))) + kAlign +
         4 * kPartialBytes + align_up(step_split_bytes(M, K, N));
}

hq_status carve_step_ws(void* ws, size_t ws_bytes, int64_t M, int64_t K, int64_t N, StepWs* w) {
  if (!ws || ws_bytes < step_ws_bytes(M, K, N)) return HQ_ERR_WORKSPACE;
  if (!aligned16(ws)) return HQ_ERR_ALIGN;
  uint8_t* p = static_cast<uint8_t*>(ws);
  auto take = [&](size_t n) { uint8_t* r = p; p += align_up(n); return r; };
  w->xq = take(size_t(M * K));
  w->xqt = take(size_t(M * K));
  w->wq = take(size_t(N * K));
  w->wqt = take(size_t(N * K));
  w->dyq = take(size_t(M * N));
  w->dyqt = take(size_t(M * N));
  w->scales = reinterpret_cast<float*>(take(kAlign));
  w->part_c = reinterpret_cast<float*>(take(kPartialBytes));
  w->part_r = reinterpret_cast<float*>(take(kPartialBytes));
  w->spart_c = reinterpret_cast<float*>(take(kPartialBytes));
  w->spart_r = reinterpret_cast<float*>(take(kPartialBytes));
  w->split_len = step_split_bytes(M, K, N);
  w->split = w->split_len ? take(w->split_len) : nullptr;
  return HQ_OK;
}

// Shape and format checks shared by the multi-GEMM layer calls (every one of M, K, N is a
// contraction length of one of the layer's GEMMs and a rotated dimension).
hq_status check_step_shape(hq_dtype dt, int64_t M, int64_t K, int64_t N, int k, hq_fmt fmt) {
  if (dt != HQ_F32 && dt != HQ_BF16) return HQ_ERR_DTYPE;
  if (!valid_k(k) || !valid_fmt(fmt)) return HQ_ERR_ARG;
  if (M < 0 || K < 0 || N < 0) return HQ_ERR_ARG;
  if (M % k || K % k || N % k) return HQ_ERR_SHAPE;
  if (M == 0 || K == 0 || N == 0) return HQ_ERR_SHAPE;
  if (fmt == HQ_INT8 && (M > HQ_MAX_K_INT8 || K > HQ_MAX_K_INT8 || N > HQ_MAX_K_INT8)) return HQ_ERR_SHAPE;
  if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31)) return HQ_ERR_SHAPE;
  return HQ_OK;
}

// Workspace of hq_linear_fwd_save (X along K, W along K) and hq_linear_bwd (dY along N,
// W along N, dY along M): up to three code tensors, scales, four partial buffers (one pair
// per stream).
size_t codes_ws_bytes(int64_t b0, int64_t b1, int64_t b2, size_t split_bytes) {
  return align_up(size_t(b0)) + align_up(size_t(b1)) + align_up(size_t(b2)) + kAlign + 4 * kPartialBytes +
         align_up(split_bytes);
}

struct CodesWs {
  uint8_t* c[3];
  float* scales;
  float *part_c, *part_r;    // caller's stream
  float *spart_c, *spart_r;  // side stream
  void* split;  // split-contraction scratch of the GEMMs (they run in stream order)
  size_t split_len;
};

hq_status carve_codes_ws(void* ws, size_t ws_bytes, int64_t b0, int64_t b1, int64_t b2, size_t split_bytes,
                         CodesWs* w) {
  if (!ws || ws_bytes < codes_ws_bytes(b0, b1, b2, split_bytes)) return HQ_ERR_WORKSPACE;
  if (!aligned16(ws)) return HQ_ERR_ALIGN;
  uint8_t* p = static_cast<uint8_t*>(ws);
  auto take = [&](size_t n) { uint8_t* r = p; p += align_up(n); return r; };
  w->c[0] = take(size_t(b0));
  w->c[1] = take(size_t(b1));
  w->c[2] = take(size_t(b2));
  w->scales = reinterpret_cast<float*>(take(kAlign));
  w->part_c = reinterpret_cast<float*>(take(kPartialBytes));
  w->part_r = reinterpret_cast<float*>(take(kPartialBytes));
  w->spart_c = reinterpret_cast<float*>(take(kPartialBytes));
  w->spart_r = reinterpret_cast<float*>(take(kPartialBytes));
  w->split_len = split_bytes;
  w->split = split_bytes ? take(split_bytes) : nullptr;
  return HQ_OK;
}

// ------------------------------------------------------------------ allocation-free quantize

// Scratch for hq_quantize_noalloc: the absmax pass's per-CTA partial maxima, in a fixed
// array every device that loads the library keeps until exit.  Host code never uses the name
// as an address: the device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) float g_noalloc_partials[HQ_NOALLOC_MAX_PARTIALS];
// The quantizer's grids are capped at kMaxPartials CTAs (one partial each); the array must hold
// that many, whatever the launch-time check below derives.
static_assert(kMaxPartials <= HQ_NOALLOC_MAX_PARTIALS, "the no-allocation scratch holds every partial maximum");

struct NoAllocSlot {
  bool ready = false;
  float* partials = nullptr;
};
NoAllocSlot g_noalloc[kMaxDevices];

hq_status noalloc_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return HQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  NoAllocSlot& s = g_noalloc[dev];
  if (!s.ready) {
    void* p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_noalloc_partials)) != cudaSuccess) return cuda_fail(e);
    s.partials = static_cast<float*>(p);
    s.ready = true;
  }
  *out = s.partials;
  return HQ_OK;
}

}  // namespace

// ====================================================================== exported C ABI

extern "C" {

size_t hq_quantize_workspace_bytes(void) { return kPartialBytes; }

hq_status hq_quantize_rht(const void* src, hq_dtype dt, int64_t rows, int64_t cols, int dim, int k, hq_fmt fmt,
                          const uint8_t* neg, void* codes, float* scale, void* workspace, size_t ws_bytes,
                          hq_stream_t stream) {
  hq_status s = check_quant_args(src, dt, rows, cols, dim, k, fmt, codes, scale);
  if (s != HQ_OK) return s;
  if (neg && !aligned16(neg)) return HQ_ERR_ALIGN;
  if (rows > 0 && cols > 0) {
    if (!workspace || ws_bytes < kPartialBytes) return HQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return HQ_ERR_ALIGN;
  }
  DeviceInfo* d = nullptr;
  if ((s = device_info(&d)) != HQ_OK) return s;
  return quantize_impl(src, dt, rows, cols, dim, k, fmt, codes, scale, static_cast<float*>(workspace), *d,
                       reinterpret_cast<cudaStream_t>(stream), neg);
}

hq_status hq_quantize(const void* src, hq_dtype dt, int64_t rows, int64_t cols, int dim, int k,
                      hq_fmt fmt, void* codes, float* scale, void* workspace, size_t ws_bytes,
                      hq_stream_t stream) {
  return hq_quantize_rht(src, dt, rows, cols, dim, k, fmt, nullptr, codes, scale, workspace, ws_bytes, stream);
}

hq_status hq_gemm(const void* A, const float* scale_a, const void* B, const float* scale_b, int64_t M,
                  int64_t N, int64_t K, hq_fmt fmt, hq_out out_kind, void* out, hq_stream_t stream) {
  hq_status s = check_gemm_args(A, scale_a, B, scale_b, M, N, K, fmt, out_kind, out);
  if (s != HQ_OK || M == 0 || N == 0) return s;
  DeviceInfo* d = nullptr;
  if ((s = device_info(&d)) != HQ_OK) return s;
  return gemm_impl(A, scale_a, B, scale_b, M, N, K, fmt, out_kind, out, *d, reinterpret_cast<cudaStream_t>(stream));
}

size_t hq_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 0 || K < 0) return 0;
  return split_ws_bytes(M, N, K);
}

hq_status hq_gemm_ws(const void* A, const float* scale_a, const void* B, const float* scale_b, int64_t M, int64_t N,
                     int64_t K, hq_fmt fmt, hq_out out_kind, void* out, void* workspace, size_t ws_bytes,
                     hq_stream_t stream) {
  hq_status s = check_gemm_args(A, scale_a, B, scale_b, M, N, K, fmt, out_kind, out);
  if (s != HQ_OK || M == 0 || N == 0) return s;
  if (workspace && !aligned16(workspace)) return HQ_ERR_ALIGN;
  DeviceInfo* d = nullptr;
  if ((s = device_info(&d)) != HQ_OK) return s;
  return gemm_impl(A, scale_a, B, scale_b, M, N, K, fmt, out_kind, out, *d, reinterpret_cast<cudaStream_t>(stream),
                   workspace, workspace ? ws_bytes : 0);
}

size_t hq_linear_workspace_bytes(int64_t M, int64_t K, int64_t N) {
  if (M < 0 || K < 0 || N < 0) return 0;
  size_t best = 0;
  best = std::max(best, linear_ws_bytes(M * K, N * K, split_ws_bytes(M, N, K)));  // forward
  best = std::max(best, linear_ws_bytes(M * N, K * N, split_ws_bytes(M, K, N)));  // dX
  best = std::max(best, linear_ws_bytes(N * M, K * M, split_ws_bytes(N, K, M)));  // dW
  return best;
}

hq_status hq_linear_fwd(const void* X, const void* W, hq_dtype dt, int64_t M, int64_t K, int64_t N, int k,
                        hq_fmt fmt, void* Y, void* workspace, size_t ws_bytes, hq_stream_t stream) {
  return linear_gemm(Operand{X, M, K, 1}, Operand{W, N, K, 1}, M, N, K, dt, k, fmt, Y, workspace, ws_bytes,
                     reinterpret_cast<cudaStream_t>(stream));
}

hq_status hq_linear_bwd_dx(const void* dY, const void* W, hq_dtype dt, int64_t M, int64_t K, int64_t N, int k,
                           hq_fmt fmt, void* dX, void* workspace, size_t ws_bytes, hq_stream_t stream) {
  return linear_gemm(Operand{dY, M, N, 1}, Operand{W, N, K, 0}, M, K, N, dt, k, fmt, dX, workspace, ws_bytes,
                     reinterpret_cast<cudaStream_t>(stream));
}

hq_status hq_linear_bwd_dw(const void* dY, const void* X, hq_dtype dt, int64_t M, int64_t K, int64_t N, int k,
                           hq_fmt fmt, void* dW, void* workspace, size_t ws_bytes, hq_stream_t stream) {
  return linear_gemm(Operand{dY, M, N, 0}, Operand{X, M, K, 0}, N, K, M, dt, k, fmt, dW, workspace, ws_bytes,
                     reinterpret_cast<cudaStream_t>(stream));
}

size_t hq_quantize_dual_workspace_bytes(void) { return 2 * kPartialBytes; }

hq_status hq_quantize_dual_rht(const void* src, hq_dtype dt, int64_t rows, int64_t cols, int k, hq_fmt fmt,
                               const uint8_t* neg_c, const uint8_t* neg_r, void* codes_c, float* scale_c,
                               void* codes_r, float* scale_r, void* workspace, size_t ws_bytes,
                               hq_stream_t stream) {
  hq_status s = check_dual_args(src, dt, rows, cols, k, fmt, codes_c, scale_c, codes_r, scale_r);
  if (s != HQ_OK) return s;
  if ((neg_c && !aligned16(neg_c)) || (neg_r && !aligned16(neg_r))) return HQ_ERR_ALIGN;
  if (rows > 0 && cols > 0) {
    if (!workspace || ws_bytes < 2 * kPartialBytes) return HQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return HQ_ERR_ALIGN;
  }
  DeviceInfo* d = nullptr;
  if ((s = device_info(&d)) != HQ_OK) return s;
  float* part = static_cast<float*>(workspace);
  return dual_impl(src, dt, rows, cols, k, fmt, codes_c, scale_c, codes_r, scale_r, part, part + kMaxPartials,
                   *d, reinterpret_cast<cudaStream_t>(stream), neg_c, neg_r);
}

hq_status hq_quantize_dual(const void* src, hq_dtype dt, int64_t rows, int64_t cols, int k, hq_fmt fmt,
                           void* codes_c, float* scale_c, void* codes_r, float* scale_r, void* workspace,
                           size_t ws_bytes, hq_stream_t stream) {
  return hq_quantize_dual_rht(src, dt, rows, cols, k, fmt, nullptr, nullptr, codes_c, scale_c, codes_r, scale_r,
                              workspace, ws_bytes, stream);
}

size_t hq_linear_fwd_bwd_workspace_bytes(int64_t M, int64_t K, int64_t N) {
  if (M < 0 || K < 0 || N < 0) return 0;
  return step_ws_bytes(M, K, N);
}

hq_status hq_linear_fwd_bwd_rht(const void* X, const void* W, const void* dY, hq_dtype dt, int64_t M, int64_t K,
                                int64_t N, int k, hq_fmt fmt, const uint8_t* neg_k, const uint8_t* neg_n,
                                const uint8_t* neg_m, void* Y, void* dX, void* dW, void* workspace,
                                size_t ws_bytes, hq_stream_t stream) {
  hq_status s = check_step_shape(dt, M, K, N, k, fmt);
  if (s != HQ_OK) return s;
  if ((neg_k && !aligned16(neg_k)) || (neg_n && !aligned16(neg_n)) || (neg_m && !aligned16(neg_m)))
    return HQ_ERR_ALIGN;
  if (!X || !W || !dY || !Y || !dX || !dW) return HQ_ERR_ARG;
  if (!aligned16(X) || !aligned16(W) || !aligned16(dY) || !aligned16(Y) || !aligned16(dX) || !aligned16(dW))
    return HQ_ERR_ALIGN;
  StepWs w;
  s = carve_step_ws(workspace, ws_bytes, M, K, N, &w);
  if (s != HQ_OK) return s;
  DeviceInfo* d = nullptr;
  if ((s = device_info(&d)) != HQ_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  float* sc = w.scales;  // x_K, x_M, w_K, w_N, dy_N, dy_M
  std::lock_guard<std::mutex> lock(g_side_mu);
  SideStream* ss = nullptr;
  if ((s = side_stream(&ss)) != HQ_OK) return s;
  cudaError_t e;
  if ((e = cudaEventRecord(ss->fork, st)) != cudaSuccess) return cuda_fail(e);
  if ((e = cudaStreamWaitEvent(ss->s, ss->fork, 0)) != cudaSuccess) return cuda_fail(e);
  // side stream: the rotations only the backward GEMMs need, alongside the forward operands
  // and GEMM: dY in both rotations (one read per pass), W along N, X along M
  if ((s = dual_impl(dY, dt, M, N, k, fmt, w.dyq, sc + 4, w.dyqt, sc + 5, w.spart_c, w.spart_r, *d, ss->s, neg_n,
                     neg_m)) != HQ_OK)
    return s;
  if (step_dual_ok(dt, M, K, k) && step_dual_ok(dt, N, K, k)) {
    // large X and W: both rotations of each by the two-rotation kernel on the caller's stream
    // (one read of the source per pass, measured faster than two single-rotation calls on
    // these shapes), then the three GEMMs; the backward GEMMs wait for dY's codes
    if ((e = cudaEventRecord(ss->join_dx, ss->s)) != cudaSuccess) return cuda_fail(e);
    if ((s = dual_impl(X, dt, M, K, k, fmt, w.xq, sc + 0, w.xqt, sc + 1, w.part_c, w.part_r, *d, st, neg_k, neg_m)) !=
        HQ_OK)
      return s;
    if ((s = dual_impl(W, dt, N, K, k, fmt, w.wq, sc + 2, w.wqt, sc + 3, w.part_c, w.part_r, *d, st, neg_k, neg_n)) !=
        HQ_OK)
      return s;
    if ((s = gemm_impl(w.xq, sc + 0, w.wq, sc + 2, M, N, K, fmt, HQ_OUT_BF16, Y, *d, st, w.split, w.split_len)) !=
        HQ_OK)
      return s;
    if ((e = cudaStreamWaitEvent(st, ss->join_dx, 0)) != cudaSuccess) return cuda_fail(e);
    if ((s = gemm_impl(w.dyq, sc + 4, w.wqt, sc + 3, M, K, N, fmt, HQ_OUT_BF16, dX, *d, st, w.split,
                       w.split_len)) != HQ_OK)
      return s;
    return gemm_impl(w.dyqt, sc + 5, w.xqt, sc + 1, N, K, M, fmt, HQ_OUT_BF16, dW, *d, st, w.split, w.split_len);
  }
  if ((s = quantize_impl(W, dt, N, K, 0, k, fmt, w.wqt, sc + 3, w.spart_c, *d, ss->s, neg_n)) != HQ_OK) return s;
  if ((e = cudaEventRecord(ss->join_dx, ss->s)) != cudaSuccess) return cuda_fail(e);  // dX's operands
  if ((s = quantize_impl(X, dt, M, K, 0, k, fmt, w.xqt, sc + 1, w.spart_c, *d, ss->s, neg_m)) != HQ_OK) return s;
  if ((e = cudaEventRecord(ss->join_dw, ss->s)) != cudaSuccess) return cuda_fail(e);  // dW's
  // caller's stream: the forward operands (X and W along K) first, so the forward GEMM starts
  // as early as possible, then the backward GEMMs once the side stream's codes have landed
  if ((s = quantize_impl(X, dt, M, K, 1, k, fmt, w.xq, sc + 0, w.part_c, *d, st, neg_k)) != HQ_OK) return s;
  if ((s = quantize_impl(W, dt, N, K, 1, k, fmt, w.wq, sc + 2, w.part_c, *d, st, neg_k)) != HQ_OK) return s;
  if ((s = gemm_impl(w.xq, sc + 0, w.wq, sc + 2, M, N, K, fmt, HQ_OUT_BF16, Y, *d, st, w.split, w.split_len)) !=
      HQ_OK)
    return s;
  if ((e = cudaStreamWaitEvent(st, ss->join_dx, 0)) != cudaSuccess) return cuda_fail(e);
  if ((s = gemm_impl(w.dyq, sc + 4, w.wqt, sc + 3, M, K, N, fmt, HQ_OUT_BF16, dX, *d, st, w.split,
                     w.split_len)) != HQ_OK)
    return s;
  // X along M lands while the dX GEMM runs
  if ((e = cudaStreamWaitEvent(st, ss->join_dw, 0)) != cudaSuccess) return cuda_fail(e);
  return gemm_impl(w.dyqt, sc + 5, w.xqt, sc + 1, N, K, M, fmt, HQ_OUT_BF16, dW, *d, st, w.split, w.split_len);
}

hq_status hq_linear_fwd_bwd(const void* X, const void* W, const void* dY, hq_dtype dt, int64_t M, int64_t K,
                            int64_t N, int k, hq_fmt fmt, void* Y, void* dX, void* dW, void* workspace,
                            size_t ws_bytes, hq_stream_t stream) {
  return hq_linear_fwd_bwd_rht(X, W, dY, dt, M, K, N, k, fmt, nullptr, nullptr, nullptr, Y, dX, dW, workspace,
                               ws_bytes, stream);
}

size_t hq_linear_fwd_save_workspace_bytes(int64_t M, int64_t K, int64_t N) {
  if (M < 0 || K < 0 || N < 0) return 0;
  return codes_ws_bytes(M * K, N * K, 0, split_ws_bytes(M, N, K));
}

}  // extern "C"

namespace {

// hq_linear_fwd_save, and with wq_codes / wq_scale non-null hq_linear_fwd_keep (W's K-rotated
// codes and scale go to the caller's buffers instead of the workspace).
hq_status fwd_save_impl(const void* X, const void* W, hq_dtype dt, int64_t M, int64_t K, int64_t N, int k,
                        hq_fmt fmt, void* Y, void* xqt_codes, float* xqt_scale, void* wq_codes, float* wq_scale,
                        void* workspace, size_t ws_bytes, hq_stream_t stream) {
  hq_status s = check_step_shape(dt, M, K, N, k, fmt);
  if (s != HQ_OK) return s;
  if (!X || !W || !Y || !xqt_codes || !xqt_scale) return HQ_ERR_ARG;
  if (!aligned16(X) || !aligned16(W) || !aligned16(Y) || !aligned16(xqt_codes) ||
      (reinterpret_cast<uintptr_t>(xqt_scale) & 3u))
    return HQ_ERR_ALIGN;
  if (wq_codes && (!aligned16(wq_codes) || (reinterpret_cast<uintptr_t>(wq_scale) & 3u))) return HQ_ERR_ALIGN;
  CodesWs w;
  if ((s = carve_codes_ws(workspace, ws_bytes, M * K, wq_codes ? 0 : N * K, 0, split_ws_bytes(M, N, K), &w)) != HQ_OK)
    return s;
  uint8_t* wc = wq_codes ? static_cast<uint8_t*>(wq_codes) : w.c[1];
  float* ws_ = wq_codes ? wq_scale : w.scales + 1;
  DeviceInfo* d = nullptr;
  if ((s = device_info(&d)) != HQ_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(g_side_mu);
  SideStream* ss = nullptr;
  if ((s = side_stream(&ss)) != HQ_OK) return s;
  cudaError_t e;
  if ((e = cudaEventRecord(ss->fork, st)) != cudaSuccess) return cuda_fail(e);
  if ((e = cudaStreamWaitEvent(ss->s, ss->fork, 0)) != cudaSuccess) return cuda_fail(e);
  // side stream: W along K
  if ((s = quantize_impl(W, dt, N, K, 1, k, fmt, wc, ws_, w.spart_c, *d, ss->s)) != HQ_OK) return s;
  if ((e = cudaEventRecord(ss->join_dw, ss->s)) != cudaSuccess) return cuda_fail(e);
  // caller's stream: X in both rotations (along K for the forward GEMM, along M kept for the
  // weight gradient), then the forward GEMM once W's codes have landed
  if ((s = dual_impl(X, dt, M, K, k, fmt, w.c[0], w.scales + 0, xqt_codes, xqt_scale, w.part_c, w.part_r, *d,
                     st)) != HQ_OK)
    return s;
  if ((e = cudaStreamWaitEvent(st, ss->join_dw, 0)) != cudaSuccess) return cuda_fail(e);
  return gemm_impl(w.c[0], w.scales + 0, wc, ws_, M, N, K, fmt, HQ_OUT_BF16, Y, *d, st, w.split, w.split_len);
}

}  // namespace

extern "C" {

hq_status hq_linear_fwd_save(const void* X, const void* W, hq_dtype dt, int64_t M, int64_t K, int64_t N, int k,
                             hq_fmt fmt, void* Y, void* xqt_codes, float* xqt_scale, void* workspace,
                             size_t ws_bytes, hq_stream_t stream) {
  return fwd_save_impl(X, W, dt, M, K, N, k, fmt, Y, xqt_codes, xqt_scale, nullptr, nullptr, workspace, ws_bytes,
                       stream);
}

size_t hq_linear_fwd_keep_workspace_bytes(int64_t M, int64_t K, int64_t N) {
  if (M < 0 || K < 0 || N < 0) return 0;
  return codes_ws_bytes(M * K, 0, 0, split_ws_bytes(M, N, K));
}

hq_status hq_linear_fwd_keep(const void* X, const void* W, hq_dtype dt, int64_t M, int64_t K, int64_t N, int k,
                             hq_fmt fmt, void* Y, void* xqt_codes, float* xqt_scale, void* wq_codes, float* wq_scale,
                             void* workspace, size_t ws_bytes, hq_stream_t stream) {
  if (!wq_codes || !wq_scale) return HQ_ERR_ARG;
  return fwd_save_impl(X, W, dt, M, K, N, k, fmt, Y, xqt_codes, xqt_scale, wq_codes, wq_scale, workspace, ws_bytes,
                       stream);
}

size_t hq_linear_bwd_workspace_bytes(int64_t M, int64_t K, int64_t N) {
  if (M < 0 || K < 0 || N < 0) return 0;
  return codes_ws_bytes(M * N, K * N, N * M, std::max(split_ws_bytes(M, K, N), split_ws_bytes(N, K, M)));
}

hq_status hq_linear_bwd(const void* dY, const void* W, const void* xqt_codes, const float* xqt_scale, hq_dtype dt,
                        int64_t M, int64_t K, int64_t N, int k, hq_fmt fmt, void* dX, void* dW, void* workspace,
                        size_t ws_bytes, hq_stream_t stream) {
  hq_status s = check_step_shape(dt, M, K, N, k, fmt);
  if (s != HQ_OK) return s;
  if (!dY || !W || !xqt_codes || !xqt_scale || !dX || !dW) return HQ_ERR_ARG;
  if (!aligned16(dY) || !aligned16(W) || !aligned16(xqt_codes) || !aligned16(dX) || !aligned16(dW) ||
      (reinterpret_cast<uintptr_t>(xqt_scale) & 3u))
    return HQ_ERR_ALIGN;
  CodesWs w;
  if ((s = carve_codes_ws(workspace, ws_bytes, M * N, K * N, N * M,
                          std::max(split_ws_bytes(M, K, N), split_ws_bytes(N, K, M)), &w)) != HQ_OK)
    return s;
  DeviceInfo* d = nullptr;
  if ((s = device_info(&d)) != HQ_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  float* sc = w.scales;  // dy_N, w_N, dy_M
  std::lock_guard<std::mutex> lock(g_side_mu);
  SideStream* ss = nullptr;
  if ((s = side_stream(&ss)) != HQ_OK) return s;
  cudaError_t e;
  if ((e = cudaEventRecord(ss->fork, st)) != cudaSuccess) return cuda_fail(e);
  if ((e = cudaStreamWaitEvent(ss->s, ss->fork, 0)) != cudaSuccess) return cuda_fail(e);
  // side stream: W along N
  if ((s = quantize_impl(W, dt, N, K, 0, k, fmt, w.c[1], sc + 1, w.spart_r, *d, ss->s)) != HQ_OK) return s;
  if ((e = cudaEventRecord(ss->join_dx, ss->s)) != cudaSuccess) return cuda_fail(e);
  // caller's stream: dY in both rotations, then dX once W's codes have landed, then dW
  if ((s = dual_impl(dY, dt, M, N, k, fmt, w.c[0], sc + 0, w.c[2], sc + 2, w.part_c, w.part_r, *d, st)) != HQ_OK)
    return s;
  if ((e = cudaStreamWaitEvent(st, ss->join_dx, 0)) != cudaSuccess) return cuda_fail(e);
  if ((s = gemm_impl(w.c[0], sc + 0, w.c[1], sc + 1, M, K, N, fmt, HQ_OUT_BF16, dX, *d, st, w.split,
                     w.split_len)) != HQ_OK)
    return s;
  return gemm_impl(w.c[2], sc + 2, xqt_codes, xqt_scale, N, K, M, fmt, HQ_OUT_BF16, dW, *d, st, w.split,
                   w.split_len);
}

hq_status hq_gemm_rotout(const void* A, const float* scale_a, const void* B, const float* scale_b, int64_t M,
                         int64_t N, int64_t K, int k, hq_fmt fmt, float* out, hq_stream_t stream) {
  if (!valid_k(k) || (fmt != HQ_INT8 && fmt != HQ_FP8_E4M3)) return HQ_ERR_ARG;
  hq_status s = check_gemm_args(A, scale_a, B, scale_b, M, N, K, fmt, HQ_OUT_BF16, out);
  if (s != HQ_OK) return s;
  if (N % k) return HQ_ERR_SHAPE;
  if (M == 0 || N == 0) return HQ_OK;
  DeviceInfo* d = nullptr;
  if ((s = device_info(&d)) != HQ_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (K == 0) {
    cudaError_t e = cudaMemsetAsync(out, 0, size_t(M) * size_t(N) * 4, st);
    return e == cudaSuccess ? HQ_OK : cuda_fail(e);
  }
  return gemm_rotout_impl(A, scale_a, B, scale_b, M, N, K, k, fmt, out, *d, st);
}

size_t hq_quantize_prerotated_workspace_bytes(void) { return kPartialBytes; }

hq_status hq_quantize_prerotated(const float* y, int64_t rows, int64_t cols, hq_fmt fmt, void* codes, float* scale,
                                 void* workspace, size_t ws_bytes, hq_stream_t stream) {
  if (fmt != HQ_INT8 && fmt != HQ_FP8_E4M3) return HQ_ERR_ARG;
  if (rows < 0 || cols < 0) return HQ_ERR_ARG;
  if (!scale) return HQ_ERR_ARG;
  if (cols % 16) return HQ_ERR_SHAPE;
  if (reinterpret_cast<uintptr_t>(scale) & 3u) return HQ_ERR_ALIGN;
  const bool empty = rows == 0 || cols == 0;
  if (!empty && (!y || !codes)) return HQ_ERR_ARG;
  if (!empty && (!aligned16(y) || !aligned16(codes))) return HQ_ERR_ALIGN;
  if (!workspace || ws_bytes < kPartialBytes) return HQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return HQ_ERR_ALIGN;
  DeviceInfo* d = nullptr;
  hq_status s = device_info(&d);
  if (s != HQ_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (empty) {
    set_scale_one_kernel<<<1, 1, 0, st>>>(scale);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? HQ_OK : cuda_fail(e);
  }
  return prerot_quant_impl(y, rows * cols, fmt, codes, scale, static_cast<float*>(workspace), *d, st);
}

size_t hq_linear_bwd_dx_reuse_workspace_bytes(int64_t M, int64_t K, int64_t N) {
  (void)N;
  if (M < 0 || K < 0) return 0;
  return align_up(size_t(M) * size_t(K) * 4);
}

hq_status hq_linear_bwd_dx_reuse(const void* g_codes, const float* g_scale, const void* wq_codes,
                                 const float* wq_scale, int64_t M, int64_t K, int64_t N, int k, hq_fmt fmt, void* dX,
                                 void* workspace, size_t ws_bytes, hq_stream_t stream) {
  hq_status s = check_dx_reuse_shape(M, K, N, k, fmt);
  if (s != HQ_OK) return s;
  if (!g_codes || !g_scale || !wq_codes || !wq_scale || !dX) return HQ_ERR_ARG;
  if (!aligned16(g_codes) || !aligned16(wq_codes) || !aligned16(dX) ||
      (reinterpret_cast<uintptr_t>(g_scale) & 3u) || (reinterpret_cast<uintptr_t>(wq_scale) & 3u))
    return HQ_ERR_ALIGN;
  if (!workspace || ws_bytes < hq_linear_bwd_dx_reuse_workspace_bytes(M, K, N)) return HQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return HQ_ERR_ALIGN;
  DeviceInfo* d = nullptr;
  if ((s = device_info(&d)) != HQ_OK) return s;
  return dx_reuse_impl(g_codes, g_scale, wq_codes, wq_scale, M, K, N, k, fmt, dX, static_cast<float*>(workspace), *d,
                       reinterpret_cast<cudaStream_t>(stream));
}

size_t hq_linear_bwd_reuse_workspace_bytes(int64_t M, int64_t K, int64_t N) {
  if (M < 0 || K < 0 || N < 0) return 0;
  return align_up(size_t(N) * size_t(M)) + kAlign + kPartialBytes + align_up(size_t(M) * size_t(K) * 4) +
         align_up(split_ws_bytes(N, K, M));
}

hq_status hq_linear_bwd_reuse(const void* dY, hq_dtype dt, const void* xqt_codes, const float* xqt_scale,
                              const void* wq_codes, const float* wq_scale, int64_t M, int64_t K, int64_t N, int k,
                              hq_fmt fmt, void* dX, void* dW, void* workspace, size_t ws_bytes, hq_stream_t stream) {
  hq_status s = check_step_shape(dt, M, K, N, k, fmt);
  if (s != HQ_OK) return s;
  if ((s = check_dx_reuse_shape(M, K, N, k, fmt)) != HQ_OK) return s;
  if (!dY || !xqt_codes || !xqt_scale || !wq_codes || !wq_scale || !dX || !dW) return HQ_ERR_ARG;
  if (!aligned16(dY) || !aligned16(xqt_codes) || !aligned16(wq_codes) || !aligned16(dX) || !aligned16(dW) ||
      (reinterpret_cast<uintptr_t>(xqt_scale) & 3u) || (reinterpret_cast<uintptr_t>(wq_scale) & 3u))
    return HQ_ERR_ALIGN;
  if (!workspace || ws_bytes < hq_linear_bwd_reuse_workspace_bytes(M, K, N)) return HQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return HQ_ERR_ALIGN;
  uint8_t* p = static_cast<uint8_t*>(workspace);
  auto take = [&](size_t n) { uint8_t* r = p; p += align_up(n); return r; };
  uint8_t* g = take(size_t(N) * size_t(M));
  float* g_scale = reinterpret_cast<float*>(take(kAlign));
  float* partials = reinterpret_cast<float*>(take(kPartialBytes));
  float* z = reinterpret_cast<float*>(take(size_t(M) * size_t(K) * 4));
  const size_t split_len = split_ws_bytes(N, K, M);
  void* split = split_len ? take(split_len) : nullptr;
  DeviceInfo* d = nullptr;
  if ((s = device_info(&d)) != HQ_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // dY once, rotated along the tokens: [N][M], the weight gradient's operand as it is and the
  // input gradient's MN-major operand
  if ((s = quantize_impl(dY, dt, M, N, 0, k, fmt, g, g_scale, partials, *d, st)) != HQ_OK) return s;
  // the dX GEMM first (its output rotated along the columns, fp32), then its row de-rotation
  // (HBM-bound) on the side stream while the dW GEMM (tensor-bound) runs on `stream`
  if ((s = gemm_mn_f32_impl(g, g_scale, wq_codes, wq_scale, M, K, N, fmt, z, *d, st, k)) != HQ_OK) return s;
  std::lock_guard<std::mutex> lock(g_side_mu);
  SideStream* ss = nullptr;
  if ((s = side_stream(&ss)) != HQ_OK) return s;
  cudaError_t e;
  if ((e = cudaEventRecord(ss->fork, st)) != cudaSuccess) return cuda_fail(e);
  if ((e = cudaStreamWaitEvent(ss->s, ss->fork, 0)) != cudaSuccess) return cuda_fail(e);
  if ((s = derotate_impl(z, M, K, k, dX, *d, ss->s)) != HQ_OK) return s;
  if ((e = cudaEventRecord(ss->join_dx, ss->s)) != cudaSuccess) return cuda_fail(e);
  if ((s = gemm_impl(g, g_scale, xqt_codes, xqt_scale, N, K, M, fmt, HQ_OUT_BF16, dW, *d, st, split, split_len)) != HQ_OK)
    return s;
  if ((e = cudaStreamWaitEvent(st, ss->join_dx, 0)) != cudaSuccess) return cuda_fail(e);
  return HQ_OK;
}

hq_status hq_quantize_noalloc(const void* src, hq_dtype dt, int64_t rows, int64_t cols, int dim, int k,
                              hq_fmt fmt, void* codes, float* scale, hq_stream_t stream) {
  hq_status s = check_quant_args(src, dt, rows, cols, dim, k, fmt, codes, scale);
  if (s != HQ_OK) return s;
  DeviceInfo* d = nullptr;
  if ((s = device_info(&d)) != HQ_OK) return s;
  float* partials = nullptr;
  if ((s = noalloc_scratch(&partials)) != HQ_OK) return s;
  if (rows > 0 && cols > 0 && quant_grid(dt, rows, cols, dim, d->sms) > HQ_NOALLOC_MAX_PARTIALS)
    return HQ_ERR_WORKSPACE;
  return quantize_impl(src, dt, rows, cols, dim, k, fmt, codes, scale, partials, *d,
                       reinterpret_cast<cudaStream_t>(stream));
}

hq_status hq_quantize_absmax(const void* src, hq_dtype dt, int64_t rows, int64_t cols, int dim, int k,
                             const uint8_t* neg, float* absmax, void* workspace, size_t ws_bytes, hq_stream_t stream) {
  hq_status s = check_src_args(src, dt, rows, cols, dim, k, absmax);
  if (s != HQ_OK) return s;
  if (neg && !aligned16(neg)) return HQ_ERR_ALIGN;
  DeviceInfo* d = nullptr;
  if ((s = device_info(&d)) != HQ_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (rows == 0 || cols == 0) {
    set_zero_kernel<<<1, 1, 0, st>>>(absmax);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? HQ_OK : cuda_fail(e);
  }
  if (!workspace || ws_bytes < kPartialBytes) return HQ_ERR_WORKSPACE;
  if (!aligned16(workspace)) return HQ_ERR_ALIGN;
  float* part = static_cast<float*>(workspace);
  cudaError_t e = dt == HQ_BF16
                      ? split_pass_k<__nv_bfloat16>(false, src, rows, cols, dim, k, HQ_INT8, neg, part, absmax, nullptr,
                                                    nullptr, *d, st)
                      : split_pass_k<float>(false, src, rows, cols, dim, k, HQ_INT8, neg, part, absmax, nullptr, nullptr,
                                            *d, st);
  return e == cudaSuccess ? HQ_OK : cuda_fail(e);
}

hq_status hq_quantize_codes(const void* src, hq_dtype dt, int64_t rows, int64_t cols, int dim, int k, hq_fmt fmt,
                            const uint8_t* neg, const float* absmax, void* codes, float* scale, hq_stream_t stream) {
  hq_status s = check_quant_args(src, dt, rows, cols, dim, k, fmt, codes, scale);
  if (s != HQ_OK) return s;
  if (!absmax) return HQ_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(absmax) & 3u) || (neg && !aligned16(neg))) return HQ_ERR_ALIGN;
  DeviceInfo* d = nullptr;
  if ((s = device_info(&d)) != HQ_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (rows == 0 || cols == 0) {
    set_scale_one_kernel<<<1, 1, 0, st>>>(scale);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? HQ_OK : cuda_fail(e);
  }
  float* a = const_cast<float*>(absmax);  // read only: the code pass reduces it as one partial
  cudaError_t e = dt == HQ_BF16
                      ? split_pass_k<__nv_bfloat16>(true, src, rows, cols, dim, k, fmt, neg, nullptr, a,
                                                    static_cast<uint8_t*>(codes), scale, *d, st)
                      : split_pass_k<float>(true, src, rows, cols, dim, k, fmt, neg, nullptr, a,
                                            static_cast<uint8_t*>(codes), scale, *d, st);
  return e == cudaSuccess ? HQ_OK : cuda_fail(e);
}

hq_status hq_selftest_gemm_timeout(const void* A, const void* B, void* out, int64_t M, int64_t N, int64_t K,
                                   hq_stream_t stream) {
  hq_status s = check_gemm_args(A, nullptr, B, nullptr, M, N, K, HQ_INT8, HQ_OUT_ACC, out);
  if (s != HQ_OK) return s;
  if (M <= 0 || N <= 0 || K <= 0 || M > 4096 || N > 4096 || K > 4096) return HQ_ERR_SHAPE;
  DeviceInfo* d = nullptr;
  if ((s = device_info(&d)) != HQ_OK) return s;
  CUtensorMap ta, tb;
  if ((s = encode_codes_map(&ta, A, M, K, hq::gemm::BM)) != HQ_OK) return s;
  if ((s = encode_codes_map(&tb, B, N, K, hq::gemm::BN)) != HQ_OK) return s;
  cudaError_t e = launch_gemm<hq::gemm::kInt8, hq::gemm::kOutAcc>(ta, tb, nullptr, nullptr, out, int(M), int(N),
                                                                  int(K), *d, reinterpret_cast<cudaStream_t>(stream), 0,
                                                                  1);
  return e == cudaSuccess ? HQ_OK : cuda_fail(e);
}

size_t hq_workspace_bytes(int64_t M, int64_t K, int64_t N, hq_fmt fmt) {
  if (M < 0 || K < 0 || N < 0) return 0;
  if (fmt != HQ_INT8 && fmt != HQ_FP8_E4M3 && fmt != HQ_FP6_E3M2 && fmt != HQ_FP6_E2M3 && fmt != HQ_FP4_E2M1) return 0;
  const size_t sizes[] = {hq_linear_workspace_bytes(M, K, N), hq_linear_fwd_bwd_workspace_bytes(M, K, N),
                          hq_linear_fwd_save_workspace_bytes(M, K, N), hq_linear_bwd_workspace_bytes(M, K, N),
                          hq_linear_fwd_keep_workspace_bytes(M, K, N), hq_linear_bwd_reuse_workspace_bytes(M, K, N),
                          hq_linear_bwd_dx_reuse_workspace_bytes(M, K, N)};
  size_t m = 0;
  for (size_t v : sizes) m = std::max(m, v);
  return m;
}

hq_status hq_mma_peak(hq_fmt fmt, int64_t n_blocks, int* pairs_out, hq_stream_t stream) {
  if (fmt != HQ_INT8 && fmt != HQ_FP8_E4M3) return HQ_ERR_ARG;
  if (n_blocks < 1 || n_blocks > (int64_t(1) << 24)) return HQ_ERR_ARG;
  DeviceInfo* d = nullptr;
  hq_status s = device_info(&d);
  if (s != HQ_OK) return s;
  const int pairs = d->sms / 2;
  if (pairs_out) *pairs_out = pairs;
  auto kernel = fmt == HQ_INT8 ? hq::peak::mma_peak_kernel<hq::gemm::kInt8> : hq::peak::mma_peak_kernel<hq::gemm::kFp8>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(hq::peak::kSmemBytes));
  if (e != cudaSuccess) return cuda_fail(e);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(hq::peak::kThreads);
  cfg.dynamicSmemBytes = hq::peak::kSmemBytes;
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kernel, n_blocks, d->status);
  return e == cudaSuccess ? HQ_OK : cuda_fail(e);
}

hq_status hq_get_error(hq_stream_t stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e);
  DeviceInfo* d = nullptr;
  hq_status s = device_info(&d);
  if (s != HQ_OK) return s;
  unsigned int v = 0;
  if ((e = cudaMemcpyAsync(&v, d->status, sizeof(v), cudaMemcpyDeviceToHost, st)) != cudaSuccess) return cuda_fail(e);
  if ((e = cudaMemsetAsync(d->status, 0, sizeof(v), st)) != cudaSuccess) return cuda_fail(e);
  if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return cuda_fail(e);
  return static_cast<hq_status>(v);
}

int hq_last_cuda_error(void) { return t_last_cuda_error; }

const char* hq_status_string(hq_status status) {
  switch (status) {
    case HQ_OK: return "ok";
    case HQ_ERR_ARG: return "invalid argument";
    case HQ_ERR_SHAPE: return "unsupported shape";
    case HQ_ERR_DTYPE: return "unsupported dtype";
    case HQ_ERR_ALIGN: return "pointer not 16-byte aligned";
    case HQ_ERR_NONFINITE: return "non-finite value in a rotated operand";
    case HQ_ERR_TIMEOUT: return "a bounded wait inside a kernel expired";
    case HQ_ERR_CUDA: return "CUDA runtime error";
    case HQ_ERR_WORKSPACE: return "workspace missing or too small";
    case HQ_ERR_UNSUPPORTED: return "device is not sm_100";
  }
  return "unknown status";
}

int hq_version(void) { return 100; }

}  // extern "C"
