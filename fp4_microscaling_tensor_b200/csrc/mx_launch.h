// mx_launch.h -- host-side launch helpers and the internal kernel entry points.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace mxk {

// Upper bound on the CTAs of any reduction kernel; sizes the workspaces.
constexpr int kMaxReduceCtas = 4096;

// Persistent grid for a grid-stride kernel with kThreads threads: enough CTAs to fill every SM
// at the kernel's occupancy, never more than the work needs (items / (threads * items_per_iter)).
inline int persistent_grid(const void* kern, int64_t nitems, int items_per_iter,
                           int cap = 1 << 30) {
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, 0);
  if (per_sm < 1) per_sm = 1;
  const int64_t full = (int64_t)sms * per_sm;
  const int64_t need = (nitems + 256LL * items_per_iter - 1) / (256LL * items_per_iter);
  int64_t g = need < full ? need : full;
  if (g > cap) g = cap;
  return (int)(g < 1 ? 1 : g);
}

// Launch with programmatic stream serialization: the kernel may be scheduled while the previous
// kernel in the stream is still finishing.  Every kernel launched this way executes
// griddep_wait() (mx_device.cuh) before its first global-memory access, which returns once the
// previous grid has completed and its writes are visible; so ordering is as for a plain launch and
// only the launch latency and the shared-memory setup overlap the previous kernel's tail.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), int grid, int block, cudaStream_t stream,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)block);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

cudaError_t run_quantize(const void* x, bool bf16, int64_t numel, int block, int fmt,
                         uint16_t g_bits, uint8_t* packed, uint8_t* scales, cudaStream_t stream,
                         int* launches);
cudaError_t run_dequantize(const uint8_t* packed, const uint8_t* scales, int64_t numel, int block,
                           int fmt, uint16_t g_bits, void* y, bool bf16, cudaStream_t stream,
                           int* launches);
// out: device mx_error_stats_t (layout-compatible struct defined in mx.h)
cudaError_t run_error_stats(const void* x, bool bf16, int64_t numel, int block, int fmt,
                            uint16_t g_bits, const uint8_t* packed, const uint8_t* scales,
                            void* out, void* workspace, cudaStream_t stream, int* launches);
// Quantize + pack with the three-term error reduction fused into the same pass (bf16 input; fp32
// input runs quantize then the reduction from the stored codes).
cudaError_t run_quantize_stats(const void* x, bool bf16, int64_t numel, int block, int fmt,
                               uint16_t g_bits, uint8_t* packed, uint8_t* scales, void* out,
                               void* workspace, cudaStream_t stream, int* launches);
// The last 4 elements of an N = 4 tensor whose size is not a multiple of 8 (from element `first`).
cudaError_t run_quantize_tail4(const void* x, bool bf16, int64_t first, int fmt, uint16_t g_bits,
                               uint8_t* packed, uint8_t* scales, cudaStream_t stream,
                               int* launches);
cudaError_t run_global_scale(const void* x, bool bf16, int64_t numel, int fmt, uint16_t* out,
                             void* workspace, cudaStream_t stream, int* launches);

}  // namespace mxk
