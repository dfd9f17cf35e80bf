// mx_noalloc.cu -- mx_error_stats_noalloc: the three-term error reduction without a caller
// workspace.
//
// mx_error_stats needs a device workspace for its per-CTA partial sums.  Some callers cannot
// provide one: code that runs where allocation is not allowed or not available (a host framework
// that owns every device allocation and hands the library only the tensors, a real-time loop that
// must not enter the allocator, C callers with no device allocator of their own).  This entry point
// takes its scratch from a fixed array in the library's own device memory instead.  It allocates
// nothing: no cudaMalloc, cudaFree or allocating library routine.
//
// The array lives in every device's copy of this library's module for as long as the process keeps
// the library loaded.  Host code cannot use the array's name as a device address, so the first call
// on each device resolves the address with cudaGetSymbolAddress (with that device current) and
// keeps it; later calls on that device reuse it.  A lookup that fails is not kept: the call
// reports MX_ERR_CUDA and the next call tries again.
#include <atomic>
#include <mutex>

#include "../../include/mx.h"
#include "mx_launch.h"

namespace {

// Largest scratch mx_error_stats can use: one 64-byte partial per CTA of its capped grid.  It does
// not depend on the tensor size.
constexpr size_t kNoAllocScratchBytes = (size_t)mxk::kMaxReduceCtas * 64;  // 256 KiB

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_resolve_mutex[kMaxDevices];
std::atomic<void*> g_scratch_ptr[kMaxDevices];  // nullptr until resolved on that device

// Device address of the scratch array on the current device.  Only a successful lookup is kept:
// a failure (for example an error left pending by unrelated earlier work) is returned to this
// caller, and the next call on the device tries again.
cudaError_t scratch_on_current_device(void** out) {
  int dev = 0;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    std::lock_guard<std::mutex> lock(g_resolve_mutex[dev]);
    p = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (p == nullptr) {
      const cudaError_t r = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (r != cudaSuccess || p == nullptr) return r != cudaSuccess ? r : cudaErrorUnknown;
      g_scratch_ptr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return cudaSuccess;
}

}  // namespace

extern "C" MX_API mx_status mx_error_stats_noalloc(const void* x, mx_dtype xt, int64_t rows,
                                                    int64_t cols, int block, mx_scale_fmt fmt,
                                                    uint16_t global_scale_fp16,
                                                    const uint8_t* packed, const uint8_t* scales,
                                                    mx_error_stats_t* out_dev,
                                                    cudaStream_t stream) {
  // the same size rule as the workspace entry point; beyond the static array the call is refused
  if (mx_error_stats_workspace_size(rows, cols, block) > kNoAllocScratchBytes)
    return MX_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (scratch_on_current_device(&scratch) != cudaSuccess || scratch == nullptr) return MX_ERR_CUDA;
  return mx_error_stats(x, xt, rows, cols, block, fmt, global_scale_fp16, packed, scales, out_dev,
                        scratch, kNoAllocScratchBytes, stream);
}
