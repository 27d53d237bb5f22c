// fp8train.cu — the C ABI declared in include/fp8train.h: host-side validation, launch
// configuration and tensor-map encoding for the four kernels of the FP8 delayed-scaling Linear
// step. Every argument is checked before the first CUDA call, so invalid input returns an error
// status and launches nothing; there is no fallback path.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "fp8train.h"
#include "cast_transpose_amax.cuh"
#include "current_scaling.cuh"
#include "fused_adamw.cuh"
#include "gemm_tcgen05.cuh"
#include "gemm_mx_wide.cuh"
#include "mx_cast.cuh"
#include "scale_update.cuh"

namespace {

thread_local std::string t_last_error;

fp8t_status fail(fp8t_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return s;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  int state = 0;               // 0 unknown, 1 sm_100, 2 other
  int sms = 0;
  int adamw_blocks_per_sm = 0;
  int adamw_cast_blocks_per_sm = 0;
  int gemm_clusters = 0;       // co-resident 2-CTA clusters of the GEMM kernel
  int gemm_wide_clusters = 0;  // ... of its wide-tile form
  int gemm_mx_clusters = 0;    // ... of its MXFP8 variant
  int gemm_mxw_clusters = 0;   // ... of the MXFP8 256 x 384 kernel
  int mx_cast_blocks_per_sm = 0;
  int cast_blocks_per_sm = 0;
  int cast_rowmajor_blocks_per_sm = 0;
  void* noalloc_scratch = nullptr;   // device address of g_adamw_noalloc_scratch
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mutex;

// Current device must be compute capability 10.0 (sm_100a code runs there only).
fp8t_status current_device(DeviceInfo** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(FP8T_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(FP8T_ERR_UNSUPPORTED_DEVICE, "device index %d", dev);
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  DeviceInfo& d = g_dev[dev];
  if (d.state == 0) {
    int major = 0, minor = 0, sms = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return fail(FP8T_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
    d.sms = sms;
    d.state = (major == 10 && minor == 0) ? 1 : 2;
    if (d.state == 1) {
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.adamw_blocks_per_sm,
                                                        fp8t::adamw::k_adamw_update<false>,
                                                        fp8t::adamw::kThreads, 0);
      if (e != cudaSuccess || d.adamw_blocks_per_sm < 1) d.adamw_blocks_per_sm = 1;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.adamw_cast_blocks_per_sm,
                                                        fp8t::adamw::k_adamw_update<true>,
                                                        fp8t::adamw::kThreads, 0);
      if (e != cudaSuccess || d.adamw_cast_blocks_per_sm < 1) d.adamw_cast_blocks_per_sm = 1;
      e = cudaFuncSetAttribute(fp8t::gemm::k_fp8_gemm<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               fp8t::gemm::kSmemBytes);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fp8t::gemm::k_fp8_gemm<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 fp8t::gemm::kSmemBytesMX);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fp8t::gemm::k_fp8_gemm_wide, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 fp8t::gemm::kSmemBytesW);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fp8t::mx::k_mx_cast, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 fp8t::mx::kSmemBytes);
      if (e != cudaSuccess) {
        d.state = 0;
        return fail(FP8T_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
      }
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
      cfg.blockDim = dim3(fp8t::gemm::kThreads, 1, 1);
      cfg.dynamicSmemBytes = fp8t::gemm::kSmemBytes;
      int clusters = 0;
      e = cudaOccupancyMaxActiveClusters(&clusters, fp8t::gemm::k_fp8_gemm<false>, &cfg);
      if (e != cudaSuccess || clusters < 1) {
        (void)cudaGetLastError();
        clusters = sms / 2;
      }
      d.gemm_clusters = clusters;
      cfg.blockDim = dim3(fp8t::gemm::kThreadsW, 1, 1);
      cfg.dynamicSmemBytes = fp8t::gemm::kSmemBytesW;
      clusters = 0;
      e = cudaOccupancyMaxActiveClusters(&clusters, fp8t::gemm::k_fp8_gemm_wide, &cfg);
      if (e != cudaSuccess || clusters < 1) {
        (void)cudaGetLastError();
        clusters = sms / 2;
      }
      d.gemm_wide_clusters = clusters;
      cfg.blockDim = dim3(fp8t::gemm::kThreads, 1, 1);
      cfg.dynamicSmemBytes = fp8t::gemm::kSmemBytesMX;
      clusters = 0;
      e = cudaOccupancyMaxActiveClusters(&clusters, fp8t::gemm::k_fp8_gemm<true>, &cfg);
      if (e != cudaSuccess || clusters < 1) {
        (void)cudaGetLastError();
        clusters = sms / 2;
      }
      d.gemm_mx_clusters = clusters;
      e = cudaFuncSetAttribute(fp8t::gemm::k_fp8_gemm_mx_wide,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, fp8t::gemm::kSmemBytesX);
      if (e != cudaSuccess) {
        d.state = 0;
        return fail(FP8T_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
      }
      cfg.blockDim = dim3(fp8t::gemm::kThreadsX, 1, 1);
      cfg.dynamicSmemBytes = fp8t::gemm::kSmemBytesX;
      clusters = 0;
      e = cudaOccupancyMaxActiveClusters(&clusters, fp8t::gemm::k_fp8_gemm_mx_wide, &cfg);
      if (e != cudaSuccess || clusters < 1) {
        (void)cudaGetLastError();
        clusters = sms / 2;
      }
      d.gemm_mxw_clusters = clusters;
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.mx_cast_blocks_per_sm, fp8t::mx::k_mx_cast,
                                                        fp8t::mx::kThreads, fp8t::mx::kSmemBytes);
      if (e != cudaSuccess || d.mx_cast_blocks_per_sm < 1) {
        (void)cudaGetLastError();
        d.mx_cast_blocks_per_sm = 1;
      }
      e = cudaFuncSetAttribute(fp8t::cast::k_cast_transpose_amax<false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, fp8t::cast::kSmemBytes);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(fp8t::cast::k_cast_transpose_amax<true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, fp8t::cast::kSmemBytes);
      if (e != cudaSuccess) {
        d.state = 0;
        return fail(FP8T_ERR_CUDA, "cudaFuncSetAttribute(cast): %s", cudaGetErrorString(e));
      }
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.cast_rowmajor_blocks_per_sm,
                                                        fp8t::cast::k_cast_rowmajor<true>,
                                                        fp8t::cast::kThreads, 0);
      if (e != cudaSuccess || d.cast_rowmajor_blocks_per_sm < 1) {
        (void)cudaGetLastError();
        d.cast_rowmajor_blocks_per_sm = 1;
      }
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&d.cast_blocks_per_sm,
                                                        fp8t::cast::k_cast_transpose_amax<true>,
                                                        fp8t::cast::kThreads, fp8t::cast::kSmemBytes);
      if (e != cudaSuccess || d.cast_blocks_per_sm < 1) {
        (void)cudaGetLastError();
        d.cast_blocks_per_sm = 1;
      }
    }
  }
  if (d.state != 1) return fail(FP8T_ERR_UNSUPPORTED_DEVICE, "device %d is not sm_100", dev);
  *out = &d;
  return FP8T_OK;
}

fp8t_status after_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(FP8T_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return FP8T_OK;
}

// ------------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// rows x K bytes, row-major: boxes of box_rows rows x 128 bytes, 128-byte swizzle, zero fill.
fp8t_status encode_kmajor(CUtensorMap* map, const void* ptr, int64_t rows, int64_t K,
                          uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(FP8T_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(fp8t::gemm::kBK), box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box,
                  es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FP8T_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return FP8T_OK;
}

// K rows x N bytes, row-major, read as an MN-major operand in boxes of 64 columns x 128 K rows with
// the 64-byte swizzle, zero fill.
fp8t_status encode_mn64(CUtensorMap* map, const void* ptr, int64_t K, int64_t N) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(FP8T_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(K)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(N)};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(fp8t::gemm::kBK)};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box,
                  es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FP8T_ERR_CUDA, "cuTensorMapEncodeTiled (64-column box) failed (%d)", (int)r);
  return FP8T_OK;
}

// ------------------------------------------------------------------ AdamW helpers
struct AdamWPlan {
  int nbatches = 0;
  int64_t nparts = 0;
};

int64_t chunks_of(int64_t numel) { return (numel + fp8t::adamw::kChunk - 1) / fp8t::adamw::kChunk; }

AdamWPlan plan_adamw(const fp8t_adamw_tensor* t, int32_t n) {
  AdamWPlan p;
  for (int32_t b0 = 0; b0 < n; b0 += fp8t::adamw::kMaxTensors) {
    int64_t chunks = 0;
    const int32_t b1 = std::min<int32_t>(n, b0 + fp8t::adamw::kMaxTensors);
    for (int32_t i = b0; i < b1; ++i) chunks += chunks_of(t[i].numel);
    p.nparts += std::min<int64_t>(chunks, fp8t::adamw::kSumsqBlocks);
    ++p.nbatches;
  }
  return p;
}

// One double per norm partial, then one int64 slot for the step a device-counted call performs.
size_t workspace_for(const AdamWPlan& p) {
  return static_cast<size_t>(((p.nparts + 1) * 8 + 255) / 256 * 256);
}

}  // namespace

// Scratch of fused_adamw_multi_tensor_noalloc, for callers that cannot allocate: a file-scope
// device array, present on every GPU that loads the library until the process exits. In host
// code this name is only a stand-in; its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_adamw_noalloc_scratch[FP8T_NOALLOC_SCRATCH_BYTES];

extern "C" {

int32_t fp8t_abi_version(void) { return 2; }

const char* fp8t_last_error_message(void) { return t_last_error.c_str(); }

const char* fp8t_status_string(fp8t_status s) {
  switch (s) {
    case FP8T_OK: return "FP8T_OK";
    case FP8T_ERR_INVALID_ARG: return "FP8T_ERR_INVALID_ARG";
    case FP8T_ERR_UNSUPPORTED_SHAPE: return "FP8T_ERR_UNSUPPORTED_SHAPE";
    case FP8T_ERR_MISALIGNED: return "FP8T_ERR_MISALIGNED";
    case FP8T_ERR_UNSUPPORTED_DEVICE: return "FP8T_ERR_UNSUPPORTED_DEVICE";
    case FP8T_ERR_CUDA: return "FP8T_ERR_CUDA";
    case FP8T_ERR_TIMEOUT: return "FP8T_ERR_TIMEOUT";
  }
  return "FP8T_UNKNOWN_STATUS";
}

// ------------------------------------------------------------------ cast / transpose / amax
}  // extern "C"

namespace {

// Casts of n tensors in launches of up to eight; with `updates`, the last CTA of each launch also
// performs the delayed-scaling update of that launch's tensors; with `current_ws`, each launch
// is preceded by the current-scaling amax pass that sets the scales it uses.
fp8t_status cast_multi(const fp8t_cast_tensor* tensors, const fp8t_cast_update* updates,
                       int32_t n_tensors, int32_t history_len, fp8t_amax_algo algo, int32_t margin,
                       unsigned int* d_ticket, unsigned int* current_ws, void* stream) {
  t_last_error.clear();
  if (!tensors || n_tensors < 1 || n_tensors > 4096)
    return fail(FP8T_ERR_INVALID_ARG, "fp8_cast_transpose_amax: tensors NULL or n_tensors out of range");
  if (current_ws && (!aligned(current_ws, 4) || margin < 0 || margin > 126))
    return fail(FP8T_ERR_INVALID_ARG, "fp8_cast_transpose_amax_current: misaligned workspace or margin outside 0..126");
  if (updates) {
    if (!d_ticket || !aligned(d_ticket, 4))
      return fail(FP8T_ERR_INVALID_ARG, "fp8_cast_transpose_amax_update: NULL or misaligned ticket");
    if (history_len < 1 || history_len > 65536)
      return fail(FP8T_ERR_INVALID_ARG, "fp8_cast_transpose_amax_update: history_len in 1..65536");
    if (algo != FP8T_AMAX_MAX && algo != FP8T_AMAX_MOST_RECENT)
      return fail(FP8T_ERR_INVALID_ARG, "fp8_cast_transpose_amax_update: unknown amax algorithm %d", (int)algo);
    if (margin < 0 || margin > 126)
      return fail(FP8T_ERR_INVALID_ARG, "fp8_cast_transpose_amax_update: margin in 0..126");
    for (int32_t i = 0; i < n_tensors; ++i) {
      const fp8t_cast_update& u = updates[i];
      if (!u.d_amax_history || !u.d_scale_inv_next)
        return fail(FP8T_ERR_INVALID_ARG, "fp8_cast_transpose_amax_update: tensor %d: NULL history or scale_inv_next", i);
      if (!aligned(u.d_amax_history, 4) || !aligned(u.d_scale_inv_next, 4))
        return fail(FP8T_ERR_MISALIGNED, "fp8_cast_transpose_amax_update: tensor %d: misaligned pointer", i);
      if (u.d_scale_inv_next == tensors[i].d_scale_inv_out)
        return fail(FP8T_ERR_INVALID_ARG,
                    "fp8_cast_transpose_amax_update: tensor %d: scale_inv_next must differ from the cast's scale_inv_out", i);
    }
  }
  for (int32_t i = 0; i < n_tensors; ++i) {
    const fp8t_cast_tensor& t = tensors[i];
    if (updates && !t.x_bf16 && t.rows == 0 && t.cols == 0 && !t.q_rowmajor && !t.q_transposed &&
        !t.d_counters && t.d_scale && t.d_amax_inout && aligned(t.d_scale, 4) &&
        aligned(t.d_amax_inout, 4) && aligned(t.d_scale_inv_out, 4) &&
        (t.fmt == FP8T_E4M3 || t.fmt == FP8T_E5M2))
      continue;                       // scale update only: the amax was accumulated elsewhere
    if (!t.x_bf16 || !t.d_scale || !t.d_amax_inout)
      return fail(FP8T_ERR_INVALID_ARG, "fp8_cast_transpose_amax: tensor %d: NULL input, scale or amax pointer", i);
    if (t.fmt != FP8T_E4M3 && t.fmt != FP8T_E5M2)
      return fail(FP8T_ERR_INVALID_ARG, "fp8_cast_transpose_amax: tensor %d: unknown format %d", i, (int)t.fmt);
    if (t.rows <= 0 || t.cols <= 0)
      return fail(FP8T_ERR_INVALID_ARG, "fp8_cast_transpose_amax: tensor %d: rows and cols must be > 0", i);
    if (t.rows % 16 || t.cols % 16 || t.rows > (int64_t(1) << 31) || t.cols > (int64_t(1) << 31) ||
        t.rows * t.cols >= (int64_t(1) << 40))
      return fail(FP8T_ERR_UNSUPPORTED_SHAPE,
                  "fp8_cast_transpose_amax: tensor %d: rows and cols must be multiples of 16, rows*cols < 2^40", i);
    if (!aligned(t.x_bf16, 16) || !aligned(t.q_rowmajor, 16) || !aligned(t.q_transposed, 16) ||
        !aligned(t.d_scale, 4) || !aligned(t.d_amax_inout, 4) || !aligned(t.d_scale_inv_out, 4) ||
        !aligned(t.d_counters, 8))
      return fail(FP8T_ERR_MISALIGNED, "fp8_cast_transpose_amax: tensor %d: misaligned pointer", i);
  }
  DeviceInfo* dev = nullptr;
  fp8t_status st = current_device(&dev);
  if (st != FP8T_OK) return st;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(FP8T_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");

  using namespace fp8t::cast;
  static thread_local Group group;
  for (int32_t b0 = 0; b0 < n_tensors; b0 += kMaxTensors) {
    const int32_t b1 = std::min<int32_t>(n_tensors, b0 + kMaxTensors);
    std::memset(&group, 0, sizeof(group));
    group.n = b1 - b0;
    int64_t tiles = 0;
    for (int32_t i = b0; i < b1; ++i) {
      const fp8t_cast_tensor& t = tensors[i];
      Tensor& T = group.t[i - b0];
      if (t.x_bf16) {
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(t.cols), static_cast<cuuint64_t>(t.rows)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(t.cols) * 2};
        cuuint32_t box[2] = {kTile, kTile};
        cuuint32_t es[2] = {1, 1};
        CUresult r = fn(&T.x_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(t.x_bf16),
                        dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return fail(FP8T_ERR_CUDA, "cuTensorMapEncodeTiled (cast input) failed (%d)", (int)r);
      }
      if (t.q_transposed) {
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(t.rows), static_cast<cuuint64_t>(t.cols)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(t.rows)};
        cuuint32_t box[2] = {kTile, kTile};
        cuuint32_t es[2] = {1, 1};
        CUresult r = fn(&T.qt_map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, t.q_transposed, dims, strides,
                        box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return fail(FP8T_ERR_CUDA, "cuTensorMapEncodeTiled (q^T store) failed (%d)", (int)r);
      }
      T.scale = const_cast<float*>(t.d_scale);      // written only by the update
      T.x = static_cast<const uint4*>(t.x_bf16);
      T.amax_bits = reinterpret_cast<unsigned int*>(t.d_amax_inout);
      T.scale_inv = t.d_scale_inv_out;
      if (updates) {
        T.hist = updates[i].d_amax_history;
        T.scale_inv_next = updates[i].d_scale_inv_next;
      }
      T.counters = t.d_counters;
      T.q = static_cast<uint8_t*>(t.q_rowmajor);
      T.rows = t.rows;
      T.cols = t.cols;
      T.tiles_c = (t.cols + kTile - 1) / kTile;
      T.tile_start = tiles;
      T.fmt = t.fmt;
      T.has_qt = t.q_transposed ? 1 : 0;
      tiles += ((t.rows + kTile - 1) / kTile) * T.tiles_c;
    }
    group.total_tiles = tiles;
    if (updates) {
      group.update = 1;
      group.ticket = d_ticket;
      group.H = history_len;
      group.algo_max = algo == FP8T_AMAX_MAX ? 1 : 0;
      group.margin = margin;
    }
    bool count = false, any_qt = false;
    for (int32_t i = b0; i < b1; ++i) {
      count |= tensors[i].d_counters != nullptr;
      any_qt |= tensors[i].q_transposed != nullptr;
    }
    int64_t grid = std::min<int64_t>(tiles, static_cast<int64_t>(dev->sms) * dev->cast_blocks_per_sm);
    if (grid < 1) grid = 1;           // update-only entries: one CTA does the update
    if (current_ws) {                  // the scales of this group, from its own amax
      fp8t::current::Group cg;
      std::memset(&cg, 0, sizeof(cg));
      cg.n = b1 - b0;
      cg.margin = margin;
      cg.ws = current_ws;
      int64_t vecs = 0;
      for (int32_t i = b0; i < b1; ++i) {
        cg.x[i - b0] = static_cast<const uint4*>(tensors[i].x_bf16);
        cg.nvec[i - b0] = tensors[i].rows * tensors[i].cols / 8;
        cg.scale[i - b0] = const_cast<float*>(tensors[i].d_scale);
        cg.fp8_max[i - b0] = tensors[i].fmt == FP8T_E4M3 ? 448.0f : 57344.0f;
        vecs += cg.nvec[i - b0];
      }
      const int64_t cgrid = std::max<int64_t>(1, std::min<int64_t>(
          (vecs + fp8t::current::kThreads - 1) / fp8t::current::kThreads, 4 * static_cast<int64_t>(dev->sms)));
      fp8t::current::k_current_amax<<<static_cast<unsigned>(cgrid), fp8t::current::kThreads, 0,
                                      as_stream(stream)>>>(cg);
      if ((st = after_launch("current-scaling amax launch")) != FP8T_OK) return st;
    }
    if (!any_qt) {                     // row-major codes only: the streaming kernel
      int64_t segs = 0;
      for (int32_t i = b0; i < b1; ++i) segs += tensors[i].rows * tensors[i].cols / 16;
      const int64_t rgrid = std::max<int64_t>(1, std::min<int64_t>(
          (segs + kThreads - 1) / kThreads, static_cast<int64_t>(dev->sms) * dev->cast_rowmajor_blocks_per_sm));
      if (count)
        k_cast_rowmajor<true><<<static_cast<unsigned>(rgrid), kThreads, 0, as_stream(stream)>>>(group);
      else
        k_cast_rowmajor<false><<<static_cast<unsigned>(rgrid), kThreads, 0, as_stream(stream)>>>(group);
    } else if (count) {
      k_cast_transpose_amax<true><<<static_cast<unsigned>(grid), kThreads, kSmemBytes, as_stream(stream)>>>(group);
    } else {
      k_cast_transpose_amax<false><<<static_cast<unsigned>(grid), kThreads, kSmemBytes, as_stream(stream)>>>(group);
    }
    if ((st = after_launch("fp8_cast_transpose_amax launch")) != FP8T_OK) return st;
  }
  return FP8T_OK;
}

}  // namespace

extern "C" {

fp8t_status fp8_cast_transpose_amax_multi(const fp8t_cast_tensor* tensors, int32_t n_tensors,
                                          void* stream) {
  return cast_multi(tensors, nullptr, n_tensors, 0, FP8T_AMAX_MAX, 0, nullptr, nullptr, stream);
}

fp8t_status fp8_cast_transpose_amax_update_multi(const fp8t_cast_tensor* tensors,
                                                 const fp8t_cast_update* updates, int32_t n_tensors,
                                                 int32_t history_len, fp8t_amax_algo algo,
                                                 int32_t margin, unsigned int* d_ticket,
                                                 void* stream) {
  if (!updates) {
    t_last_error.clear();
    return fail(FP8T_ERR_INVALID_ARG, "fp8_cast_transpose_amax_update: updates NULL");
  }
  return cast_multi(tensors, updates, n_tensors, history_len, algo, margin, d_ticket, nullptr,
                    stream);
}

fp8t_status fp8_cast_transpose_amax_current_multi(const fp8t_cast_tensor* tensors,
                                                  int32_t n_tensors, int32_t margin,
                                                  unsigned int* d_workspace, void* stream) {
  if (!d_workspace) {
    t_last_error.clear();
    return fail(FP8T_ERR_INVALID_ARG, "fp8_cast_transpose_amax_current: workspace NULL");
  }
  return cast_multi(tensors, nullptr, n_tensors, 0, FP8T_AMAX_MAX, margin, nullptr, d_workspace,
                    stream);
}

fp8t_status fp8_cast_transpose_amax(const void* x_bf16, int64_t rows, int64_t cols, fp8t_format fmt,
                                    const float* d_scale, void* q_rowmajor, void* q_transposed,
                                    float* d_amax_inout, float* d_scale_inv_out,
                                    unsigned long long* d_counters, void* stream) {
  const fp8t_cast_tensor t = {x_bf16, rows, cols, fmt, d_scale, q_rowmajor, q_transposed,
                              d_amax_inout, d_scale_inv_out, d_counters};
  return fp8_cast_transpose_amax_multi(&t, 1, stream);
}

// ------------------------------------------------------------------ GEMM
}  // extern "C"

namespace {

constexpr size_t kSumsqHeader = 256;    // ticket and abort words, then the partial slots

// Tile lists of a grouped GEMM launch: every tile costs its problem's K / 128 k-blocks (twice
// that for a wide tile); tiles are handed out longest first, each to the least-loaded cluster.
// A wide launch then splits tiles into their two 256-column halves, one half moving to the least
// busy cluster, while that lowers the busiest cluster's load. A half tile is costed at 0.58 of a
// whole one, not 0.5: it runs half the MMAs but loads all of A, the operand-starved pattern the
// wide tile avoids. (On the 4096 step this takes the busiest cluster from 704 to 678 k-block
// units with 28 splits, and the launch from ~0.295 to ~0.292 ms; costing halves at 0.5 split
// more and gained less. Timed per cluster, a half tile's k-block costs 0.76 of a whole one's and
// wgrad's k-blocks 8% more than dgrad's; costing the items that way, or running halves last,
// changed the launch by less than its run-to-run spread.) Every cluster then runs its items in
// index order. Items are 3 * tile + part.
// Launches with more tiles than the table holds keep round-robin (with thousands of tiles it is
// balanced already).
void build_schedule(fp8t::gemm::Group& g, int clusters, bool wide, bool mx_wide = false) {
  using namespace fp8t::gemm;
  g.scheduled = 0;
  if (g.total_tiles > kMaxSchedTiles || clusters > kMaxClusters || clusters < 2) return;
  struct Item { int64_t cost; int tile, part; };
  std::vector<Item> items;
  items.reserve(g.total_tiles);
  for (int p = 0; p < g.n; ++p) {
    const int end = p + 1 < g.n ? g.p[p + 1].tile_start : g.total_tiles;
    const int64_t kbs = (g.p[p].K + kBK - 1) / kBK;
    const int64_t cost = kbs * (wide ? 2 : 1);
    for (int t = g.p[p].tile_start; t < end; ++t) {
      // MX 256 x 384 tiles: three 128-column MMAs per k-step, two where N ends within the tile
      const int nt = (t - g.p[p].tile_start) % g.p[p].tiles_n;
      const int64_t c = mx_wide ? kbs * (nt * kBNx + 256 < g.p[p].N ? 3 : 2) : cost;
      items.push_back({c, t, 0});
    }
  }
  std::stable_sort(items.begin(), items.end(),
                   [](const Item& a, const Item& b) { return a.cost > b.cost; });
  std::vector<int64_t> load(clusters, 0);
  std::vector<std::vector<Item>> own(clusters);
  for (const auto& it : items) {
    int best = 0;
    for (int c = 1; c < clusters; ++c)
      if (load[c] < load[best]) best = c;
    load[best] += it.cost;
    own[best].push_back(it);
  }
  // a half tile runs about 0.58 of a whole one: half the MMAs, but all of A's loads
  auto half_cost = [](int64_t whole) { return (whole * 29 + 49) / 50; };
  int n_items = g.total_tiles;
  while (wide && n_items < kMaxSchedTiles) {
    int hi = 0, lo = 0;
    for (int c = 1; c < clusters; ++c) {
      if (load[c] > load[hi]) hi = c;
      if (load[c] < load[lo]) lo = c;
    }
    int pick = -1;                    // the whole tile of `hi` whose split lowers `hi` most
    int64_t best = load[hi];
    for (int k = 0; k < static_cast<int>(own[hi].size()); ++k) {
      const Item& it = own[hi][k];
      if (it.part != 0) continue;
      const int64_t h = half_cost(it.cost);
      const int64_t after = std::max(load[hi] - it.cost + h, load[lo] + h);
      if (after < best) {
        best = after;
        pick = k;
      }
    }
    if (pick < 0) break;
    Item& it = own[hi][pick];
    const int64_t h = half_cost(it.cost);
    load[hi] += h - it.cost;
    load[lo] += h;
    it.cost = h;
    it.part = 1;
    own[lo].push_back({h, it.tile, 2});
    ++n_items;
  }
  int k = 0;
  for (int c = 0; c < clusters; ++c) {
    std::sort(own[c].begin(), own[c].end(), [](const Item& a, const Item& b) {
      return a.tile != b.tile ? a.tile < b.tile : a.part < b.part;
    });
    g.start[c] = static_cast<uint16_t>(k);
    for (const auto& it : own[c]) g.order[k++] = static_cast<uint16_t>(3 * it.tile + it.part);
  }
  g.start[clusters] = static_cast<uint16_t>(k);
  g.scheduled = 1;
}

// Wide tiles (256 x 512 per pair) when every problem of the call is at least 512 wide; the choice
// is made for the whole call, so every launch of it numbers its sum-of-squares slots alike.
bool use_wide(const fp8t_gemm_desc* gemms, int32_t n) {
  for (int32_t i = 0; i < n; ++i)
    if (gemms[i].N < fp8t::gemm::kBNw) return false;
  return true;
}

int64_t gemm_tiles(const fp8t_gemm_desc& d, bool wide) {
  using namespace fp8t::gemm;
  const int64_t bn = wide ? kBNw : kBN;
  return ((d.M + kBM - 1) / kBM) * ((d.N + bn - 1) / bn);
}

int64_t sumsq_slots(const fp8t_gemm_desc* gemms, int32_t n, const int32_t* sumsq_of) {
  const bool wide = use_wide(gemms, n);
  const int64_t per_tile = wide ? fp8t::gemm::kSumsqPerTileW : fp8t::gemm::kSumsqPerTile;
  int64_t slots = 0;
  for (int32_t i = 0; i < n; ++i)
    if (sumsq_of[i]) slots += gemm_tiles(gemms[i], wide) * per_tile;
  return slots;
}

fp8t_status gemm_multi(const fp8t_gemm_desc* gemms, int32_t n_gemms, const int32_t* sumsq_of,
                       double* d_sumsq_out, void* d_workspace, size_t workspace_bytes,
                       void* stream) {
  t_last_error.clear();
  if (!gemms || n_gemms < 1 || n_gemms > 4096)
    return fail(FP8T_ERR_INVALID_ARG, "fp8_gemm: gemms NULL or n_gemms out of range");
  const int64_t lim = int64_t(1) << 31;
  for (int32_t i = 0; i < n_gemms; ++i) {
    const fp8t_gemm_desc& d = gemms[i];
    if (!d.A || !d.B || !d.D_bf16 || !d.d_a_scale_inv || !d.d_b_scale_inv)
      return fail(FP8T_ERR_INVALID_ARG, "fp8_gemm: problem %d: NULL pointer", i);
    if ((d.a_fmt != FP8T_E4M3 && d.a_fmt != FP8T_E5M2) || (d.b_fmt != FP8T_E4M3 && d.b_fmt != FP8T_E5M2))
      return fail(FP8T_ERR_INVALID_ARG, "fp8_gemm: problem %d: unknown format", i);
    if ((d.a_layout != FP8T_K_MAJOR && d.a_layout != FP8T_MN_MAJOR) ||
        (d.b_layout != FP8T_K_MAJOR && d.b_layout != FP8T_MN_MAJOR))
      return fail(FP8T_ERR_INVALID_ARG, "fp8_gemm: problem %d: unknown operand layout", i);
    if (d.M <= 0 || d.N <= 0 || d.K <= 0)
      return fail(FP8T_ERR_INVALID_ARG, "fp8_gemm: problem %d: M, N, K must be > 0", i);
    if (d.M % 16 || d.N % 16 || d.K % 16 || d.M >= lim || d.N >= lim || d.K >= lim)
      return fail(FP8T_ERR_UNSUPPORTED_SHAPE, "fp8_gemm: problem %d: M, N, K must be multiples of 16 below 2^31", i);
    if (!aligned(d.A, 16) || !aligned(d.B, 16) || !aligned(d.D_bf16, 16) ||
        !aligned(d.d_a_scale_inv, 4) || !aligned(d.d_b_scale_inv, 4))
      return fail(FP8T_ERR_MISALIGNED, "fp8_gemm: problem %d: misaligned pointer", i);
  }
  int64_t n_slots = 0;
  if (sumsq_of) {
    if (!d_sumsq_out || !aligned(d_sumsq_out, 8) || !d_workspace || !aligned(d_workspace, 256))
      return fail(FP8T_ERR_INVALID_ARG, "fp8_gemm_multi_sumsq: NULL or misaligned sumsq_out or workspace");
    n_slots = sumsq_slots(gemms, n_gemms, sumsq_of);
    if (n_slots < 1 || n_slots >= (int64_t(1) << 31))
      return fail(FP8T_ERR_INVALID_ARG, "fp8_gemm_multi_sumsq: no problem (or too many tiles) selected");
    const size_t need = kSumsqHeader + static_cast<size_t>(n_slots) * 8;
    if (workspace_bytes < need)
      return fail(FP8T_ERR_INVALID_ARG, "fp8_gemm_multi_sumsq: workspace of %zu bytes needed", need);
  }
  DeviceInfo* dev = nullptr;
  fp8t_status st = current_device(&dev);
  if (st != FP8T_OK) return st;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(FP8T_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");

  using namespace fp8t::gemm;
  static thread_local Group group;
  int64_t slot = 0;
  const bool wide = use_wide(gemms, n_gemms);
  const int bn = wide ? kBNw : kBN;
  for (int32_t b0 = 0; b0 < n_gemms; b0 += kMaxProblems) {
    const int32_t b1 = std::min<int32_t>(n_gemms, b0 + kMaxProblems);
    std::memset(&group, 0, sizeof(group));
    group.n = b1 - b0;
    if (sumsq_of) {
      group.ticket = static_cast<unsigned int*>(d_workspace);
      group.abort_word = static_cast<unsigned int*>(d_workspace) + 1;
      group.partials = reinterpret_cast<double*>(static_cast<char*>(d_workspace) + kSumsqHeader);
      group.sumsq_out = d_sumsq_out;
      group.n_partials = static_cast<int32_t>(n_slots);
      group.last_launch = b1 == n_gemms ? 1 : 0;
    }
    int64_t tiles = 0;
    for (int32_t i = b0; i < b1; ++i) {
      const fp8t_gemm_desc& d = gemms[i];
      Problem& P = group.p[i - b0];
      // 128 x 128-byte boxes either way: [rows][K] (K-major) or [K][rows] (MN-major)
      const bool a_mn = d.a_layout == FP8T_MN_MAJOR, b_mn = d.b_layout == FP8T_MN_MAJOR;
      if ((st = a_mn ? encode_kmajor(&P.a, d.A, d.K, d.M, kBK)
                     : encode_kmajor(&P.a, d.A, d.M, d.K, kHalf)) != FP8T_OK) return st;
      if ((st = b_mn ? encode_kmajor(&P.b, d.B, d.K, d.N, kBK)
                     : encode_kmajor(&P.b, d.B, d.N, d.K, kHalf)) != FP8T_OK) return st;
      P.a_mn = a_mn ? 1 : 0;
      P.b_mn = b_mn ? 1 : 0;
      // D (BF16 M x N): 32 x 32 boxes, 64-byte swizzle, written by the epilogue's TMA stores
      cuuint64_t dims[2] = {static_cast<cuuint64_t>(d.N), static_cast<cuuint64_t>(d.M)};
      cuuint64_t strides[1] = {static_cast<cuuint64_t>(d.N) * 2};
      cuuint32_t box[2] = {32, 32};
      cuuint32_t es[2] = {1, 1};
      CUresult r = fn(&P.d, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d.D_bf16, dims, strides, box, es,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                      CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (r != CUDA_SUCCESS) return fail(FP8T_ERR_CUDA, "cuTensorMapEncodeTiled (D) failed (%d)", (int)r);
      P.sa = d.d_a_scale_inv;
      P.sb = d.d_b_scale_inv;
      P.M = static_cast<int32_t>(d.M);
      P.N = static_cast<int32_t>(d.N);
      P.K = static_cast<int32_t>(d.K);
      P.idesc = make_idesc(d.a_fmt, d.b_fmt, P.a_mn, P.b_mn);
      P.tiles_n = static_cast<int32_t>((d.N + bn - 1) / bn);
      P.tile_start = static_cast<int32_t>(tiles);
      P.sumsq_slot = -1;
      if (sumsq_of && sumsq_of[i]) {
        P.sumsq_slot = static_cast<int32_t>(slot);
        slot += gemm_tiles(d, wide) * (wide ? kSumsqPerTileW : kSumsqPerTile);
      }
      tiles += ((d.M + kBM - 1) / kBM) * P.tiles_n;            // one tile per pair
      if (tiles >= (int64_t(1) << 30))
        return fail(FP8T_ERR_UNSUPPORTED_SHAPE, "fp8_gemm: too many tiles in one launch");
    }
    group.total_tiles = static_cast<int32_t>(tiles);
    // persistent pairs: wide tiles may be split in two, so a wide launch may use up to twice as
    // many clusters as it has tiles
    const int64_t grid = wide ? 2 * std::min<int64_t>(2 * tiles, dev->gemm_wide_clusters)
                              : 2 * std::min<int64_t>(tiles, dev->gemm_clusters);
    build_schedule(group, static_cast<int>(grid / 2), wide);   // round-robin: extra pairs idle
    if (wide)
      k_fp8_gemm_wide<<<static_cast<unsigned>(grid), kThreadsW, kSmemBytesW, as_stream(stream)>>>(group);
    else
      k_fp8_gemm<false><<<static_cast<unsigned>(grid), kThreads, kSmemBytes, as_stream(stream)>>>(group);
    if ((st = after_launch("fp8_gemm launch")) != FP8T_OK) return st;
  }
  return FP8T_OK;
}

}  // namespace

extern "C" {

fp8t_status fp8_gemm_multi(const fp8t_gemm_desc* gemms, int32_t n_gemms, void* stream) {
  return gemm_multi(gemms, n_gemms, nullptr, nullptr, nullptr, 0, stream);
}

size_t fp8_gemm_sumsq_workspace_bytes(const fp8t_gemm_desc* gemms, int32_t n_gemms,
                                      const int32_t* sumsq_of) {
  if (!gemms || !sumsq_of || n_gemms < 1 || n_gemms > 4096) return 0;
  for (int32_t i = 0; i < n_gemms; ++i)
    if (gemms[i].M <= 0 || gemms[i].N <= 0) return 0;
  const int64_t slots = sumsq_slots(gemms, n_gemms, sumsq_of);
  if (slots < 1) return 0;
  return kSumsqHeader + static_cast<size_t>(slots) * 8;
}

fp8t_status fp8_gemm_multi_sumsq(const fp8t_gemm_desc* gemms, int32_t n_gemms,
                                 const int32_t* sumsq_of, double* d_sumsq_out, void* d_workspace,
                                 size_t workspace_bytes, void* stream) {
  if (!sumsq_of) {
    t_last_error.clear();
    return fail(FP8T_ERR_INVALID_ARG, "fp8_gemm_multi_sumsq: sumsq_of NULL");
  }
  return gemm_multi(gemms, n_gemms, sumsq_of, d_sumsq_out, d_workspace, workspace_bytes, stream);
}

// ------------------------------------------------------------------ MXFP8
fp8t_status fp8_mx_cast_multi(const fp8t_mx_cast_tensor* tensors, int32_t n_tensors, void* stream) {
  t_last_error.clear();
  if (!tensors || n_tensors < 1 || n_tensors > 4096)
    return fail(FP8T_ERR_INVALID_ARG, "fp8_mx_cast: tensors NULL or n_tensors out of range");
  for (int32_t i = 0; i < n_tensors; ++i) {
    const fp8t_mx_cast_tensor& t = tensors[i];
    if (!t.x_bf16 || (!t.q_row && !t.q_col) || (t.q_row && !t.scales_row) || (t.q_col && !t.scales_col))
      return fail(FP8T_ERR_INVALID_ARG, "fp8_mx_cast: tensor %d: NULL input, or an output without its scales", i);
    if (t.fmt != FP8T_E4M3 && t.fmt != FP8T_E5M2)
      return fail(FP8T_ERR_INVALID_ARG, "fp8_mx_cast: tensor %d: unknown format", i);
    if (t.rows <= 0 || t.cols <= 0 || t.rows % 128 || t.cols % 128 || t.rows >= (int64_t(1) << 31) ||
        t.cols >= (int64_t(1) << 31))
      return fail(FP8T_ERR_UNSUPPORTED_SHAPE, "fp8_mx_cast: tensor %d: rows and cols must be positive multiples of 128", i);
    if (!aligned(t.x_bf16, 16) || !aligned(t.q_row, 16) || !aligned(t.q_col, 16) ||
        !aligned(t.scales_row, 16) || !aligned(t.scales_col, 16))
      return fail(FP8T_ERR_MISALIGNED, "fp8_mx_cast: tensor %d: pointers must be 16-byte aligned", i);
  }
  DeviceInfo* dev = nullptr;
  fp8t_status st = current_device(&dev);
  if (st != FP8T_OK) return st;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(FP8T_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  using namespace fp8t::mx;
  static thread_local Group group;
  for (int32_t b0 = 0; b0 < n_tensors; b0 += kMaxTensors) {
    const int32_t b1 = std::min<int32_t>(n_tensors, b0 + kMaxTensors);
    std::memset(&group, 0, sizeof(group));
    group.n = b1 - b0;
    int64_t tiles = 0;
    for (int32_t i = b0; i < b1; ++i) {
      const fp8t_mx_cast_tensor& t = tensors[i];
      Tensor& T = group.t[i - b0];
      // BF16 [rows][cols] read as 128-row x 64-column boxes (128 bytes per row: 128-byte swizzle)
      cuuint64_t dims[2] = {static_cast<cuuint64_t>(t.cols), static_cast<cuuint64_t>(t.rows)};
      cuuint64_t strides[1] = {static_cast<cuuint64_t>(t.cols) * 2};
      cuuint32_t box[2] = {64, static_cast<cuuint32_t>(kTile)};
      cuuint32_t es[2] = {1, 1};
      CUresult r = fn(&T.x_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(t.x_bf16),
                      dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (r != CUDA_SUCCESS) return fail(FP8T_ERR_CUDA, "cuTensorMapEncodeTiled (MX cast input) failed (%d)", (int)r);
      T.q_row = static_cast<uint8_t*>(t.q_row);
      T.sf_row = static_cast<uint8_t*>(t.scales_row);
      T.q_col = static_cast<uint8_t*>(t.q_col);
      T.sf_col = static_cast<uint8_t*>(t.scales_col);
      T.rows = t.rows;
      T.cols = t.cols;
      T.tiles_c = t.cols / kTile;
      T.tile_start = tiles;
      T.fmt = t.fmt;
      tiles += (t.rows / kTile) * T.tiles_c;
    }
    group.total_tiles = tiles;
    const int64_t grid = std::min<int64_t>(tiles, static_cast<int64_t>(dev->sms) * dev->mx_cast_blocks_per_sm);
    k_mx_cast<<<static_cast<unsigned>(grid), kThreads, kSmemBytes, as_stream(stream)>>>(group);
    if ((st = after_launch("fp8_mx_cast launch")) != FP8T_OK) return st;
  }
  return FP8T_OK;
}

}  // extern "C"

namespace {

// MX launches use 256 x 384 tiles when every output is at least 512 wide (for the whole call).
bool mx_use_wide(const fp8t_mx_gemm_desc* gemms, int32_t n) {
  for (int32_t i = 0; i < n; ++i)
    if (gemms[i].N < 512) return false;
  return true;
}

int64_t mx_sumsq_slots(const fp8t_mx_gemm_desc* gemms, int32_t n, const int32_t* sumsq_of) {
  using namespace fp8t::gemm;
  const bool wide = mx_use_wide(gemms, n);
  const int64_t bn = wide ? kBNx : kBN, per_tile = wide ? kSumsqPerTileW : kSumsqPerTile;
  int64_t slots = 0;
  for (int32_t i = 0; i < n; ++i)
    if (sumsq_of[i]) slots += ((gemms[i].M + kBM - 1) / kBM) * ((gemms[i].N + bn - 1) / bn) * per_tile;
  return slots;
}

fp8t_status mx_gemm_multi(const fp8t_mx_gemm_desc* gemms, int32_t n_gemms, const int32_t* sumsq_of,
                          double* d_sumsq_out, void* d_workspace, size_t workspace_bytes,
                          void* stream) {
  t_last_error.clear();
  if (!gemms || n_gemms < 1 || n_gemms > 4096)
    return fail(FP8T_ERR_INVALID_ARG, "fp8_mx_gemm: gemms NULL or n_gemms out of range");
  const int64_t lim = int64_t(1) << 31;
  for (int32_t i = 0; i < n_gemms; ++i) {
    const fp8t_mx_gemm_desc& d = gemms[i];
    if (!d.A || !d.B || !d.A_scales || !d.B_scales || !d.D_bf16)
      return fail(FP8T_ERR_INVALID_ARG, "fp8_mx_gemm: problem %d: NULL pointer", i);
    if ((d.a_fmt != FP8T_E4M3 && d.a_fmt != FP8T_E5M2) || (d.b_fmt != FP8T_E4M3 && d.b_fmt != FP8T_E5M2) ||
        (d.a_layout != FP8T_K_MAJOR && d.a_layout != FP8T_MN_MAJOR) ||
        (d.b_layout != FP8T_K_MAJOR && d.b_layout != FP8T_MN_MAJOR))
      return fail(FP8T_ERR_INVALID_ARG, "fp8_mx_gemm: problem %d: unknown format or layout", i);
    if (d.M <= 0 || d.N <= 0 || d.K <= 0 || d.M % 128 || d.N % 128 || d.K % 128 || d.M >= lim ||
        d.N >= lim || d.K >= lim)
      return fail(FP8T_ERR_UNSUPPORTED_SHAPE, "fp8_mx_gemm: problem %d: M, N, K must be positive multiples of 128", i);
    if (!aligned(d.A, 16) || !aligned(d.B, 16) || !aligned(d.D_bf16, 16) || !aligned(d.A_scales, 16) ||
        !aligned(d.B_scales, 16))
      return fail(FP8T_ERR_MISALIGNED, "fp8_mx_gemm: problem %d: pointers must be 16-byte aligned", i);
  }
  int64_t n_slots = 0;
  if (sumsq_of) {
    if (!d_sumsq_out || !aligned(d_sumsq_out, 8) || !d_workspace || !aligned(d_workspace, 256))
      return fail(FP8T_ERR_INVALID_ARG, "fp8_mx_gemm_multi_sumsq: NULL or misaligned sumsq_out or workspace");
    n_slots = mx_sumsq_slots(gemms, n_gemms, sumsq_of);
    if (n_slots < 1 || n_slots >= (int64_t(1) << 31))
      return fail(FP8T_ERR_INVALID_ARG, "fp8_mx_gemm_multi_sumsq: no problem (or too many tiles) selected");
    const size_t need = kSumsqHeader + static_cast<size_t>(n_slots) * 8;
    if (workspace_bytes < need)
      return fail(FP8T_ERR_INVALID_ARG, "fp8_mx_gemm_multi_sumsq: workspace of %zu bytes needed", need);
  }
  DeviceInfo* dev = nullptr;
  fp8t_status st = current_device(&dev);
  if (st != FP8T_OK) return st;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(FP8T_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  using namespace fp8t::gemm;
  // 256 x 384 tiles when every output is at least 512 wide (the choice holds for the whole call)
  const bool mxw = mx_use_wide(gemms, n_gemms);
  int64_t slot = 0;
  // scale atoms viewed as [atoms][512] bytes, read one atom at a time
  auto encode_sf = [&](CUtensorMap* map, const void* ptr, int64_t atoms) -> fp8t_status {
    cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(atoms)};
    cuuint64_t strides[1] = {512};
    cuuint32_t box[2] = {128, 1};
    cuuint32_t es[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(ptr), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(FP8T_ERR_CUDA, "cuTensorMapEncodeTiled (scales) failed (%d)", (int)r);
    return FP8T_OK;
  };
  static thread_local Group group;
  for (int32_t b0 = 0; b0 < n_gemms; b0 += kMaxProblems) {
    const int32_t b1 = std::min<int32_t>(n_gemms, b0 + kMaxProblems);
    std::memset(&group, 0, sizeof(group));
    group.n = b1 - b0;
    if (sumsq_of) {
      group.ticket = static_cast<unsigned int*>(d_workspace);
      group.abort_word = static_cast<unsigned int*>(d_workspace) + 1;
      group.partials = reinterpret_cast<double*>(static_cast<char*>(d_workspace) + kSumsqHeader);
      group.sumsq_out = d_sumsq_out;
      group.n_partials = static_cast<int32_t>(n_slots);
      group.last_launch = b1 == n_gemms ? 1 : 0;
    }
    int64_t tiles = 0;
    for (int32_t i = b0; i < b1; ++i) {
      const fp8t_mx_gemm_desc& d = gemms[i];
      Problem& P = group.p[i - b0];
      const bool a_mn = d.a_layout == FP8T_MN_MAJOR, b_mn = d.b_layout == FP8T_MN_MAJOR;
      if ((st = a_mn ? encode_kmajor(&P.a, d.A, d.K, d.M, kBK)
                     : encode_kmajor(&P.a, d.A, d.M, d.K, kHalf)) != FP8T_OK) return st;
      if ((st = b_mn ? encode_kmajor(&P.b, d.B, d.K, d.N, kBK)
                     : encode_kmajor(&P.b, d.B, d.N, d.K, kHalf)) != FP8T_OK) return st;
      if ((st = encode_sf(&P.sfa, d.A_scales, (d.M / 128) * (d.K / 128))) != FP8T_OK) return st;
      if ((st = encode_sf(&P.sfb, d.B_scales, (d.N / 128) * (d.K / 128))) != FP8T_OK) return st;
      cuuint64_t dims[2] = {static_cast<cuuint64_t>(d.N), static_cast<cuuint64_t>(d.M)};
      cuuint64_t strides[1] = {static_cast<cuuint64_t>(d.N) * 2};
      cuuint32_t box[2] = {32, 32};
      cuuint32_t es[2] = {1, 1};
      CUresult r = fn(&P.d, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d.D_bf16, dims, strides, box, es,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                      CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (r != CUDA_SUCCESS) return fail(FP8T_ERR_CUDA, "cuTensorMapEncodeTiled (D) failed (%d)", (int)r);
      P.sa = nullptr;                          // block scales only: alpha = 1
      P.sb = nullptr;
      P.M = static_cast<int32_t>(d.M);
      P.N = static_cast<int32_t>(d.N);
      P.K = static_cast<int32_t>(d.K);
      P.a_mn = a_mn ? 1 : 0;
      P.b_mn = b_mn ? 1 : 0;
      P.a_fmt = d.a_fmt;
      P.b_fmt = d.b_fmt;
      P.kb128 = static_cast<int32_t>(d.K / 128);
      P.sumsq_slot = -1;
      if (mxw && (st = b_mn ? encode_mn64(&P.b64, d.B, d.K, d.N)
                            : encode_kmajor(&P.b64, d.B, d.N, d.K, kHalf / 2)) != FP8T_OK) return st;
      P.tiles_n = static_cast<int32_t>((d.N + (mxw ? kBNx : kBN) - 1) / (mxw ? kBNx : kBN));
      P.tile_start = static_cast<int32_t>(tiles);
      const int64_t p_tiles = ((d.M + kBM - 1) / kBM) * P.tiles_n;
      if (sumsq_of && sumsq_of[i]) {
        P.sumsq_slot = static_cast<int32_t>(slot);
        slot += p_tiles * (mxw ? kSumsqPerTileW : kSumsqPerTile);
      }
      tiles += p_tiles;
      if (tiles >= (int64_t(1) << 30))
        return fail(FP8T_ERR_UNSUPPORTED_SHAPE, "fp8_mx_gemm: too many tiles in one launch");
    }
    group.total_tiles = static_cast<int32_t>(tiles);
    const int64_t grid = 2 * std::min<int64_t>(tiles, mxw ? dev->gemm_mxw_clusters : dev->gemm_mx_clusters);
    build_schedule(group, static_cast<int>(grid / 2), false, mxw);
    if (mxw)
      k_fp8_gemm_mx_wide<<<static_cast<unsigned>(grid), kThreadsX, kSmemBytesX, as_stream(stream)>>>(group);
    else
      k_fp8_gemm<true><<<static_cast<unsigned>(grid), kThreads, kSmemBytesMX, as_stream(stream)>>>(group);
    if ((st = after_launch("fp8_mx_gemm launch")) != FP8T_OK) return st;
  }
  return FP8T_OK;
}

}  // namespace

extern "C" {

fp8t_status fp8_mx_gemm_multi(const fp8t_mx_gemm_desc* gemms, int32_t n_gemms, void* stream) {
  return mx_gemm_multi(gemms, n_gemms, nullptr, nullptr, nullptr, 0, stream);
}

size_t fp8_mx_gemm_sumsq_workspace_bytes(const fp8t_mx_gemm_desc* gemms, int32_t n_gemms,
                                         const int32_t* sumsq_of) {
  if (!gemms || !sumsq_of || n_gemms < 1 || n_gemms > 4096) return 0;
  for (int32_t i = 0; i < n_gemms; ++i)
    if (gemms[i].M <= 0 || gemms[i].N <= 0) return 0;
  const int64_t slots = mx_sumsq_slots(gemms, n_gemms, sumsq_of);
  if (slots < 1) return 0;
  return kSumsqHeader + static_cast<size_t>(slots) * 8;
}

fp8t_status fp8_mx_gemm_multi_sumsq(const fp8t_mx_gemm_desc* gemms, int32_t n_gemms,
                                    const int32_t* sumsq_of, double* d_sumsq_out,
                                    void* d_workspace, size_t workspace_bytes, void* stream) {
  if (!sumsq_of) {
    t_last_error.clear();
    return fail(FP8T_ERR_INVALID_ARG, "fp8_mx_gemm_multi_sumsq: sumsq_of NULL");
  }
  return mx_gemm_multi(gemms, n_gemms, sumsq_of, d_sumsq_out, d_workspace, workspace_bytes, stream);
}

fp8t_status fp8_gemm(const void* A, fp8t_format a_fmt, const void* B, fp8t_format b_fmt, int64_t M,
                     int64_t N, int64_t K, const float* d_a_scale_inv, const float* d_b_scale_inv,
                     void* D_bf16, void* stream) {
  const fp8t_gemm_desc d = {A, a_fmt, B, b_fmt, M, N, K, d_a_scale_inv, d_b_scale_inv, D_bf16};
  return fp8_gemm_multi(&d, 1, stream);
}

// ------------------------------------------------------------------ scale update
fp8t_status fp8_scale_update(int32_t n_tensors, float* d_amax, float* d_amax_history,
                             int32_t history_len, const float* d_fp8_max, fp8t_amax_algo algo,
                             int32_t margin, float* d_scale, float* d_scale_inv, void* stream) {
  t_last_error.clear();
  if (!d_amax || !d_amax_history || !d_fp8_max || !d_scale || !d_scale_inv)
    return fail(FP8T_ERR_INVALID_ARG, "fp8_scale_update: NULL pointer");
  if (n_tensors < 1 || n_tensors > 65535 || history_len < 1 || history_len > 65536)
    return fail(FP8T_ERR_INVALID_ARG, "fp8_scale_update: n_tensors in 1..65535, history_len in 1..65536");
  if (algo != FP8T_AMAX_MAX && algo != FP8T_AMAX_MOST_RECENT)
    return fail(FP8T_ERR_INVALID_ARG, "fp8_scale_update: unknown amax algorithm %d", (int)algo);
  if (margin < 0 || margin > 126) return fail(FP8T_ERR_INVALID_ARG, "fp8_scale_update: margin in 0..126");
  if (!aligned(d_amax, 4) || !aligned(d_amax_history, 4) || !aligned(d_fp8_max, 4) ||
      !aligned(d_scale, 4) || !aligned(d_scale_inv, 4))
    return fail(FP8T_ERR_MISALIGNED, "fp8_scale_update: misaligned pointer");
  DeviceInfo* dev = nullptr;
  fp8t_status st = current_device(&dev);
  if (st != FP8T_OK) return st;
  fp8t::scale::k_scale_update<<<n_tensors, fp8t::scale::kThreads, 0, as_stream(stream)>>>(
      d_amax, d_amax_history, history_len, d_fp8_max, algo == FP8T_AMAX_MAX ? 1 : 0, margin,
      d_scale, d_scale_inv);
  return after_launch("fp8_scale_update launch");
}

// ------------------------------------------------------------------ fused AdamW
size_t fused_adamw_workspace_bytes(const fp8t_adamw_tensor* tensors, int32_t n_tensors) {
  if (!tensors || n_tensors < 1 || n_tensors > (1 << 20)) return 0;
  for (int32_t i = 0; i < n_tensors; ++i)
    if (tensors[i].numel <= 0) return 0;
  return workspace_for(plan_adamw(tensors, n_tensors));
}

}  // extern "C"

namespace {

// The AdamW call; with d_presummed the norm pass is skipped and its sum of squares read there.
fp8t_status adamw_call(const fp8t_adamw_tensor* tensors, const fp8t_adamw_cast* casts,
                       int32_t n_tensors, float lr, float beta1,
                       float beta2, float eps, float weight_decay, int64_t step,
                       int64_t* d_step_inout, float loss_scale, float max_grad_norm,
                       float* d_grad_norm_out, int32_t* d_skipped_out, void* d_workspace,
                       size_t workspace_bytes, const double* d_presummed, unsigned int* d_ticket,
                       void* stream) {
  t_last_error.clear();
  if (!tensors || n_tensors < 1 || n_tensors > (1 << 20))
    return fail(FP8T_ERR_INVALID_ARG, "fused_adamw_multi_tensor: tensors NULL or n_tensors out of range");
  for (int32_t i = 0; i < n_tensors; ++i) {
    const fp8t_adamw_tensor& t = tensors[i];
    if (!t.master || !t.m || !t.v || !t.grad_bf16 || !t.weight_bf16 || t.numel <= 0)
      return fail(FP8T_ERR_INVALID_ARG, "fused_adamw_multi_tensor: tensor %d has a NULL pointer or numel <= 0", i);
    if (!aligned(t.master, 16) || !aligned(t.m, 16) || !aligned(t.v, 16) ||
        !aligned(t.grad_bf16, 16) || !aligned(t.weight_bf16, 16))
      return fail(FP8T_ERR_MISALIGNED, "fused_adamw_multi_tensor: tensor %d is not 16-byte aligned", i);
  }
  if (casts) {
    for (int32_t i = 0; i < n_tensors; ++i) {
      const fp8t_adamw_cast& c = casts[i];
      if (c.rows == 0 && c.cols == 0) continue;                     // no cast for this tensor
      if (c.rows <= 0 || c.cols <= 0 || c.rows % 16 || c.cols % 16 || c.rows >= (int64_t(1) << 31) ||
          c.cols >= (int64_t(1) << 31) || c.rows * c.cols != tensors[i].numel)
        return fail(FP8T_ERR_UNSUPPORTED_SHAPE,
                    "fused_adamw_multi_tensor_presummed: cast %d: rows x cols must equal numel, multiples of 16", i);
      if (c.fmt != FP8T_E4M3 && c.fmt != FP8T_E5M2)
        return fail(FP8T_ERR_INVALID_ARG, "fused_adamw_multi_tensor_presummed: cast %d: unknown format", i);
      if (!c.d_scale || !c.d_amax_inout)
        return fail(FP8T_ERR_INVALID_ARG, "fused_adamw_multi_tensor_presummed: cast %d: NULL scale or amax", i);
      if (!aligned(c.d_scale, 4) || !aligned(c.d_amax_inout, 4) || !aligned(c.d_scale_inv_out, 4) ||
          !aligned(c.q_rowmajor, 16))
        return fail(FP8T_ERR_MISALIGNED, "fused_adamw_multi_tensor_presummed: cast %d: misaligned pointer", i);
    }
  }
  if (!d_step_inout && step < 1)
    return fail(FP8T_ERR_INVALID_ARG, "fused_adamw_multi_tensor: step must be >= 1");
  if (!(loss_scale > 0.0f) || !std::isfinite(loss_scale) || !std::isfinite(lr) ||
      !std::isfinite(beta1) || !std::isfinite(beta2) || !std::isfinite(eps) ||
      !std::isfinite(weight_decay) || !std::isfinite(max_grad_norm))
    return fail(FP8T_ERR_INVALID_ARG, "fused_adamw_multi_tensor: non-finite hyperparameter or loss_scale <= 0");
  if (!aligned(d_grad_norm_out, 4) || !aligned(d_skipped_out, 4) || !aligned(d_workspace, 16) ||
      !aligned(d_step_inout, 8))
    return fail(FP8T_ERR_MISALIGNED, "fused_adamw_multi_tensor: misaligned output or workspace");
  const AdamWPlan plan = plan_adamw(tensors, n_tensors);
  const size_t need = workspace_for(plan);
  if (d_presummed) {
    if (!aligned(d_presummed, 8))
      return fail(FP8T_ERR_MISALIGNED, "fused_adamw_multi_tensor_presummed: misaligned sum of squares");
    if (d_step_inout && (!d_ticket || !aligned(d_ticket, 4)))
      return fail(FP8T_ERR_INVALID_ARG, "fused_adamw_multi_tensor_presummed: a device step counter needs a ticket");
  } else if (!d_workspace || workspace_bytes < need) {
    return fail(FP8T_ERR_INVALID_ARG, "fused_adamw_multi_tensor: workspace of %zu bytes needed", need);
  }
  DeviceInfo* dev = nullptr;
  fp8t_status st = current_device(&dev);
  if (st != FP8T_OK) return st;

  using namespace fp8t::adamw;
  Scalars k;
  k.beta1 = beta1;
  k.beta2 = beta2;
  k.omb1 = static_cast<float>(1.0 - static_cast<double>(beta1));
  k.omb2 = static_cast<float>(1.0 - static_cast<double>(beta2));
  k.decay = static_cast<float>(1.0 - static_cast<double>(lr) * static_cast<double>(weight_decay));
  k.d_step = d_step_inout;
  k.step_slot = d_presummed ? nullptr
                            : reinterpret_cast<const int64_t*>(static_cast<double*>(d_workspace) + plan.nparts);
  k.step_ticket = d_ticket;
  k.lr_d = lr;
  k.beta1_d = beta1;
  k.beta2_d = beta2;
  if (!d_step_inout) {
    k.step_size = static_cast<float>(static_cast<double>(lr) /
                                     (1.0 - std::pow(static_cast<double>(beta1), static_cast<double>(step))));
    k.bc2_sqrt = static_cast<float>(std::sqrt(1.0 - std::pow(static_cast<double>(beta2), static_cast<double>(step))));
  } else {
    k.step_size = 0.0f;      // formed on the device from the counter
    k.bc2_sqrt = 0.0f;
  }
  k.eps = eps;
  k.inv_s_d = 1.0 / static_cast<double>(loss_scale);
  k.inv_s = static_cast<float>(k.inv_s_d);
  k.max_norm = max_grad_norm;

  cudaStream_t s = as_stream(stream);
  double* partials = static_cast<double*>(d_workspace);
  static thread_local Batch batch;   // ~17 KB: kept off the stack
  // a batch ends at kMaxTensors tensors or kMaxCasts casts
  auto has_cast = [&](int32_t i) { return casts && casts[i].rows > 0; };
  auto batch_end = [&](int32_t b0) {
    int32_t b1 = b0, nc = 0;
    while (b1 < n_tensors && b1 - b0 < kMaxTensors) {
      if (has_cast(b1)) {
        if (nc == kMaxCasts) break;
        ++nc;
      }
      ++b1;
    }
    return b1;
  };
  int64_t off = 0;
  for (int pass = d_presummed ? 1 : 0; pass < 2; ++pass) {
    off = 0;
    for (int32_t b0 = 0, bi = 0, b1 = 0; b0 < n_tensors; b0 = b1, ++bi) {
      b1 = batch_end(b0);
      batch.n = b1 - b0;
      batch.first = bi == 0 ? 1 : 0;
      batch.last = b1 == n_tensors ? 1 : 0;
      int64_t acc = 0;
      int32_t nc = 0;
      for (int32_t i = b0; i < b1; ++i) {
        const int j = i - b0;
        batch.chunk_start[j] = acc;
        batch.cast_of[j] = -1;
        if (has_cast(i)) {
          const fp8t_adamw_cast& c = casts[i];
          CastInfo& ci = batch.cast[nc];
          ci.scale = c.d_scale;
          ci.amax_bits = reinterpret_cast<unsigned int*>(c.d_amax_inout);
          ci.scale_inv = c.d_scale_inv_out;
          ci.q = static_cast<uint8_t*>(c.q_rowmajor);
          ci.fmt = c.fmt;
          batch.cast_of[j] = static_cast<int8_t>(nc++);
        }
        acc += chunks_of(tensors[i].numel);
        batch.numel[j] = tensors[i].numel;
        batch.master[j] = tensors[i].master;
        batch.m[j] = tensors[i].m;
        batch.v[j] = tensors[i].v;
        batch.g[j] = static_cast<const uint16_t*>(tensors[i].grad_bf16);
        batch.w[j] = static_cast<uint16_t*>(tensors[i].weight_bf16);
      }
      batch.chunk_start[batch.n] = acc;
      if (pass == 0) {
        const int64_t grid = std::min<int64_t>(acc, kSumsqBlocks);
        k_adamw_sumsq<<<static_cast<unsigned>(grid), kThreads, 0, s>>>(
            batch, partials + off, bi == 0 ? d_step_inout : nullptr,
            reinterpret_cast<int64_t*>(partials + plan.nparts));
        off += grid;
        if ((st = after_launch("adamw norm pass launch")) != FP8T_OK) return st;
      } else {
        const double* parts = d_presummed ? d_presummed : partials;
        const int np = d_presummed ? 1 : static_cast<int>(plan.nparts);
        if (nc) {
          const int64_t grid = std::min<int64_t>(acc, static_cast<int64_t>(dev->sms) * dev->adamw_cast_blocks_per_sm);
          k_adamw_update<true><<<static_cast<unsigned>(grid), kThreads, 0, s>>>(
              batch, k, parts, np, d_grad_norm_out, d_skipped_out);
        } else {
          const int64_t grid = std::min<int64_t>(acc, static_cast<int64_t>(dev->sms) * dev->adamw_blocks_per_sm);
          k_adamw_update<false><<<static_cast<unsigned>(grid), kThreads, 0, s>>>(
              batch, k, parts, np, d_grad_norm_out, d_skipped_out);
        }
        if ((st = after_launch("adamw update launch")) != FP8T_OK) return st;
      }
    }
  }
  return FP8T_OK;
}

}  // namespace

extern "C" {

fp8t_status fused_adamw_multi_tensor(const fp8t_adamw_tensor* tensors, int32_t n_tensors, float lr,
                                     float beta1, float beta2, float eps, float weight_decay,
                                     int64_t step, int64_t* d_step_inout, float loss_scale,
                                     float max_grad_norm, float* d_grad_norm_out,
                                     int32_t* d_skipped_out, void* d_workspace,
                                     size_t workspace_bytes, void* stream) {
  return adamw_call(tensors, nullptr, n_tensors, lr, beta1, beta2, eps, weight_decay, step,
                    d_step_inout, loss_scale, max_grad_norm, d_grad_norm_out, d_skipped_out,
                    d_workspace, workspace_bytes, nullptr, nullptr, stream);
}

fp8t_status fused_adamw_multi_tensor_presummed(const fp8t_adamw_tensor* tensors,
                                               const fp8t_adamw_cast* casts, int32_t n_tensors,
                                               float lr, float beta1, float beta2, float eps,
                                               float weight_decay, int64_t step,
                                               int64_t* d_step_inout, float loss_scale,
                                               float max_grad_norm, const double* d_grad_sumsq,
                                               float* d_grad_norm_out, int32_t* d_skipped_out,
                                               unsigned int* d_ticket, void* stream) {
  if (!d_grad_sumsq) {
    t_last_error.clear();
    return fail(FP8T_ERR_INVALID_ARG, "fused_adamw_multi_tensor_presummed: d_grad_sumsq NULL");
  }
  return adamw_call(tensors, casts, n_tensors, lr, beta1, beta2, eps, weight_decay, step,
                    d_step_inout, loss_scale, max_grad_norm, d_grad_norm_out, d_skipped_out,
                    nullptr, 0, d_grad_sumsq, d_ticket, stream);
}

// Same step as fused_adamw_multi_tensor, with the built-in scratch array as its workspace.
fp8t_status fused_adamw_multi_tensor_noalloc(const fp8t_adamw_tensor* tensors, int32_t n_tensors,
                                             float lr, float beta1, float beta2, float eps,
                                             float weight_decay, int64_t step,
                                             int64_t* d_step_inout, float loss_scale,
                                             float max_grad_norm, float* d_grad_norm_out,
                                             int32_t* d_skipped_out, void* stream) {
  t_last_error.clear();
  const size_t need = fused_adamw_workspace_bytes(tensors, n_tensors);
  if (need == 0)   // invalid tensor table: the regular entry point reports it, launching nothing
    return fused_adamw_multi_tensor(tensors, n_tensors, lr, beta1, beta2, eps, weight_decay, step,
                                    d_step_inout, loss_scale, max_grad_norm, d_grad_norm_out,
                                    d_skipped_out, nullptr, 0, stream);
  if (need > FP8T_NOALLOC_SCRATCH_BYTES)
    return fail(FP8T_ERR_UNSUPPORTED_SHAPE,
                "fused_adamw_multi_tensor_noalloc: needs %zu bytes of scratch, the built-in array "
                "holds %d; split the tensors over several calls or use fused_adamw_multi_tensor",
                need, FP8T_NOALLOC_SCRATCH_BYTES);
  DeviceInfo* dev = nullptr;
  fp8t_status st = current_device(&dev);
  if (st != FP8T_OK) return st;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (!dev->noalloc_scratch) {       // once per device, with that device current
      void* p = nullptr;
      cudaError_t e = cudaGetSymbolAddress(&p, g_adamw_noalloc_scratch);
      if (e != cudaSuccess || !p)
        return fail(FP8T_ERR_CUDA, "cudaGetSymbolAddress(noalloc scratch): %s", cudaGetErrorString(e));
      dev->noalloc_scratch = p;
    }
    scratch = dev->noalloc_scratch;
  }
  return fused_adamw_multi_tensor(tensors, n_tensors, lr, beta1, beta2, eps, weight_decay, step,
                                  d_step_inout, loss_scale, max_grad_norm, d_grad_norm_out,
                                  d_skipped_out, scratch, FP8T_NOALLOC_SCRATCH_BYTES, stream);
}

// ------------------------------------------------------------------ device error word
fp8t_status fp8t_check_device_error(void* stream) {
  t_last_error.clear();
  cudaError_t e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return fail(FP8T_ERR_CUDA, "stream: %s", cudaGetErrorString(e));
  unsigned int word = 0;
  e = cudaMemcpyFromSymbol(&word, fp8t::g_error_word, sizeof(word));
  if (e != cudaSuccess) return fail(FP8T_ERR_CUDA, "reading the error word: %s", cudaGetErrorString(e));
  if (word) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(fp8t::g_error_word, &zero, sizeof(zero));
    if (e != cudaSuccess) return fail(FP8T_ERR_CUDA, "clearing the error word: %s", cudaGetErrorString(e));
    if (word & fp8t::kErrTimeout) return fail(FP8T_ERR_TIMEOUT, "a bounded wait in a kernel expired");
  }
  return FP8T_OK;
}

fp8t_status fp8t_debug_expire_waits(int32_t mode) {
  t_last_error.clear();
  if (mode < 0 || mode > 2) return fail(FP8T_ERR_INVALID_ARG, "fp8t_debug_expire_waits: mode in 0..2");
  cudaError_t e = cudaMemcpyToSymbol(fp8t::g_expire_waits, &mode, sizeof(mode));
  if (e != cudaSuccess) return fail(FP8T_ERR_CUDA, "setting the test hook: %s", cudaGetErrorString(e));
  return FP8T_OK;
}

fp8t_status fp8t_set_wait_timeout_ns(uint64_t ns) {
  t_last_error.clear();
  const unsigned long long v = ns;
  cudaError_t e = cudaMemcpyToSymbol(fp8t::g_wait_timeout_ns, &v, sizeof(v));
  if (e != cudaSuccess) return fail(FP8T_ERR_CUDA, "setting the wait limit: %s", cudaGetErrorString(e));
  return FP8T_OK;
}

}  // extern "C"
