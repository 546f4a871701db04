// Outlier-column detection that allocates no device memory.
//
// Some callers cannot allocate device memory at the point where they need
// the outlier set of an activation matrix: an inference engine's plugin whose
// enqueue step is forbidden to allocate, a serving loop that must not
// allocate after warm-up, or a process whose caching allocator has already
// reserved nearly all of the device memory, so that a fresh cudaMalloc (or a
// stream-ordered allocation) fails or fragments the pool.  For them this file
// runs the outlier-detection kernel with its scratch (epoch-tagged column
// maxima, the completion ticket, the column bitmask and its word prefix) in a
// fixed static device array instead of a handle-owned workspace.
//
// The array is kNoAllocScratchBytes (1 MiB) per device.  It is part of the
// library's device image, so every GPU that loads the library holds it until
// the process exits.  All calls share it: two calls whose kernels overlap on
// the GPU (for example on two streams without ordering between them) race
// on it and give wrong results.
#include "int8mm.h"
#include "kernels.cuh"

#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <mutex>
#include <string>

namespace {

constexpr size_t kNoAllocScratchBytes = INT8MM_NOALLOC_SCRATCH_BYTES;
// Layout of the array (byte offsets): ticket and epoch, then the column keys,
// the bitmask, its word prefix, and column maxima for callers that pass none.
constexpr size_t kTicketOffset = 0;                       // u32, cleared by every call
constexpr size_t kEpochOffset = 8;                        // u64, grows from call to call
constexpr size_t kColkeyOffset = 256;                     // 65536 u64
constexpr size_t kMaskOffset = kColkeyOffset + 65536 * 8; // 2048 u32
constexpr size_t kPreOffset = kMaskOffset + 2048 * 4;     // 2048 i32
constexpr size_t kColmaxOffset = kPreOffset + 2048 * 4;   // 65536 fp32
constexpr size_t kScratchUsed = kColmaxOffset + 65536 * 4;
static_assert(kScratchUsed <= kNoAllocScratchBytes, "layout fits the static array");

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
// Per device: the context the address was looked up in, and the address.
// A context that is destroyed and re-created (cudaDeviceReset, or a primary
// context released and retained again) reloads the library's device image,
// so the array may move: the address is looked up again for a new context.
unsigned long long g_scratch_ctx[kMaxDevices] = {};
void* g_scratch_ptr[kMaxDevices] = {};

int8mm_status setup_error(int8mm_status s, const std::string& msg) {
  i8mm::set_last_error(msg);  // reported by int8mm_last_error()
  return s;
}

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (0 if there is none or
// the driver cannot say); ids are never reused within a process.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Once per device and context, with that device current: the device address
// of the static scratch array (its host-side name is only a stand-in).
int8mm_status device_scratch(int dev, void** ptr) {
  std::lock_guard<std::mutex> g(g_setup_mu);
  const unsigned long long ctx = current_context_id();
  if (g_scratch_ptr[dev] == nullptr || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess)
      return setup_error(INT8MM_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
    // the lookup makes the device's primary context current if none was
    g_scratch_ctx[dev] = ctx != 0 ? ctx : current_context_id();
  }
  *ptr = g_scratch_ptr[dev];
  return INT8MM_OK;
}

}  // namespace

extern "C" {

int8mm_status int8mm_outlier_columns_noalloc(const void* X_fp16_dev, int64_t M, int64_t K, float alpha,
                                             int32_t* idx_dev, int32_t* count_dev, float* colmax_dev,
                                             void* stream) {
  if (idx_dev == nullptr || count_dev == nullptr || (M > 0 && X_fp16_dev == nullptr))
    return setup_error(INT8MM_ERR_INVALID_ARG, "idx and count, and X when M > 0, must not be NULL");
  if (std::isnan(alpha)) return setup_error(INT8MM_ERR_INVALID_ARG, "alpha is NaN");
  if (M < 0 || M >= (int64_t(1) << 31))
    return setup_error(INT8MM_ERR_INVALID_ARG, "M must be in [0, 2^31)");
  if (K < 16 || K % 16 != 0 || K > INT8MM_MAX_K)
    return setup_error(INT8MM_ERR_UNSUPPORTED_SHAPE,
                       "K=" + std::to_string(K) + ": the no-allocation detection needs 16 <= K <= " +
                           std::to_string(INT8MM_MAX_K) + ", a multiple of 16");
  if (((K + 255) / 256) * ((M + 63) / 64) >= (int64_t(1) << 31))
    return setup_error(INT8MM_ERR_UNSUPPORTED_SHAPE, "M is too large for one detection launch");
  if ((reinterpret_cast<uintptr_t>(X_fp16_dev) & 15u) != 0)
    return setup_error(INT8MM_ERR_ALIGNMENT, "X must be 16-byte aligned");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return setup_error(INT8MM_ERR_CUDA, "no usable current CUDA device");
  void* base = nullptr;
  int8mm_status st = device_scratch(dev, &base);
  if (st != INT8MM_OK) return st;

  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (M == 0) {  // no rows: no outlier columns, and every column maximum is 0
    if ((e = cudaMemsetAsync(count_dev, 0, sizeof(int32_t), cs)) != cudaSuccess ||
        (colmax_dev != nullptr &&
         (e = cudaMemsetAsync(colmax_dev, 0, static_cast<size_t>(K) * sizeof(float), cs)) != cudaSuccess))
      return setup_error(INT8MM_ERR_CUDA, std::string("output reset: ") + cudaGetErrorString(e));
    return INT8MM_OK;
  }
  unsigned char* s = static_cast<unsigned char*>(base);
  // The array keeps the previous call's contents.  The ticket must start at
  // zero; the column keys need no clearing (each call raises the epoch that
  // its keys carry).
  if ((e = cudaMemsetAsync(s + kTicketOffset, 0, sizeof(unsigned), cs)) != cudaSuccess)
    return setup_error(INT8MM_ERR_CUDA, std::string("ticket reset: ") + cudaGetErrorString(e));
  i8mm::OutlierScratch sc;
  sc.ticket = reinterpret_cast<unsigned*>(s + kTicketOffset);
  sc.epoch = reinterpret_cast<unsigned long long*>(s + kEpochOffset);
  sc.colkey = reinterpret_cast<unsigned long long*>(s + kColkeyOffset);
  sc.mask = reinterpret_cast<uint32_t*>(s + kMaskOffset);
  sc.pre = reinterpret_cast<int32_t*>(s + kPreOffset);
  sc.colmax = colmax_dev ? colmax_dev : reinterpret_cast<float*>(s + kColmaxOffset);
  sc.idx = idx_dev;
  sc.count = count_dev;
  if ((e = i8mm::launch_outlier_detect(static_cast<const __half*>(X_fp16_dev), M, K, alpha, sc, cs)) !=
      cudaSuccess)
    return setup_error(INT8MM_ERR_CUDA, std::string("outlier detection launch: ") + cudaGetErrorString(e));
  return INT8MM_OK;
}

}  // extern "C"
