// mx_launch.h -- host-side launch helpers and the internal kernel entry points.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace mxk {

// Upper bound on the CTAs of any reduction kernel; sizes the workspaces.
constexpr int kMaxReduceCtas = 4096;

// Tensors per grouped launch (one persistent grid split among them).
constexpr int kMaxGroup = 16;

// Static split of a grid among the tensors of a group: CTAs [begin[t], begin[t + 1]) work on
// tensor t (an empty range for an empty tensor).  Passed by value in the kernel parameters.
struct CtaSplit {
  int count;
  int begin[kMaxGroup + 1];
#ifdef __CUDACC__
  // The tensor of CTA `cta` (a linear scan over at most kMaxGroup entries, once per CTA).
  __device__ __forceinline__ int find(int cta) const {
    int t = 0;
    while (t + 1 < count && cta >= begin[t + 1]) ++t;
    return t;
  }
#endif
};

// Resident CTAs of 256 threads on the whole device for `kern` (SMs x occupancy), with `smem`
// bytes of dynamic shared memory per CTA.
inline int64_t resident_ctas_smem(const void* kern, int smem) {
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem);
  if (per_sm < 1) per_sm = 1;
  return (int64_t)sms * per_sm;
}
inline int64_t resident_ctas(const void* kern) { return resident_ctas_smem(kern, 0); }

// Dynamic shared memory above 48 KiB must be enabled per kernel and per device: flags[dev] (one
// array per kernel) is set once the attribute call has succeeded on that device; a failed call is
// retried on the next launch.
constexpr int kMaxDevices = 64;
template <typename K>
inline cudaError_t allow_dynamic_smem(std::atomic<bool>* flags, K* kern, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < kMaxDevices && flags[dev].load(std::memory_order_acquire))
    return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev >= 0 && dev < kMaxDevices)
    flags[dev].store(true, std::memory_order_release);
  return e;
}

// Persistent grid for a grid-stride kernel with kThreads threads: enough CTAs to fill every SM
// at the kernel's occupancy, never more than the work needs (items / (threads * items_per_iter)).
inline int persistent_grid(const void* kern, int64_t nitems, int items_per_iter,
                           int cap = 1 << 30) {
  const int64_t full = resident_ctas(kern);
  const int64_t need = (nitems + 256LL * items_per_iter - 1) / (256LL * items_per_iter);
  int64_t g = need < full ? need : full;
  if (g > cap) g = cap;
  return (int)(g < 1 ? 1 : g);
}

// Split one persistent grid among `count` tensors of nitems[t] items: at most the resident CTAs
// (and `cap`) in total, each tensor with work at least one CTA and at most what its items need,
// the rest in proportion to the items.  Returns the total grid (0 when there is no work).
inline int split_grid(const void* kern, const int64_t* nitems, int count, int items_per_iter,
                      int cap, CtaSplit* split) {
  int64_t full = resident_ctas(kern);
  if (full > cap) full = cap;
  int64_t need[kMaxGroup], total = 0, nonempty = 0;
  for (int t = 0; t < count; ++t) {
    need[t] = (nitems[t] + 256LL * items_per_iter - 1) / (256LL * items_per_iter);
    total += nitems[t];
    nonempty += nitems[t] > 0;
  }
  if (full < nonempty) full = nonempty;
  int64_t share[kMaxGroup], used = 0;
  for (int t = 0; t < count; ++t) {
    share[t] = nitems[t] > 0 ? (int64_t)((double)full * (double)nitems[t] / (double)total) : 0;
    if (nitems[t] > 0 && share[t] < 1) share[t] = 1;
    if (share[t] > need[t]) share[t] = need[t];
    used += share[t];
  }
  // hand out what is left, one CTA at a time, to the tensors with the most items per CTA
  while (used < full) {
    int best = -1;
    double best_load = 0.0;
    for (int t = 0; t < count; ++t) {
      if (share[t] >= need[t]) continue;
      const double load = (double)nitems[t] / (double)share[t];
      if (best < 0 || load > best_load) { best = t; best_load = load; }
    }
    if (best < 0) break;
    ++share[best];
    ++used;
  }
  split->count = count;
  split->begin[0] = 0;
  for (int t = 0; t < count; ++t) split->begin[t + 1] = split->begin[t] + (int)share[t];
  for (int t = count + 1; t <= kMaxGroup; ++t) split->begin[t] = split->begin[count];
  return split->begin[count];
}

// Launch with programmatic stream serialization: the kernel may be scheduled while the previous
// kernel in the stream is still finishing.  Every kernel launched this way executes
// griddep_wait() (mx_device.cuh) before its first global-memory access, which returns once the
// previous grid has completed and its writes are visible; so ordering is as for a plain launch and
// only the launch latency and the shared-memory setup overlap the previous kernel's tail.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_smem(void (*kern)(KArgs...), int grid, int block, size_t smem,
                                   cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), int grid, int block, cudaStream_t stream,
                              Args... args) {
  return launch_pdl_smem(kern, grid, block, 0, stream, args...);
}

// One tensor of a grouped call (all pointers device memory; numel = rows * cols).
struct TensorArgs {
  const void* x;      // input of quantize / the error reduction
  void* y;            // output of dequantize
  uint8_t* packed;    // codes: written by quantize, read by dequantize / given-code reduction
  uint8_t* scales;    // scale codes, likewise
  void* stats;        // device mx_error_stats_t of the error reduction
  int64_t numel;
  uint16_t g_bits;
  uint16_t* g_dev;    // when set: g is read from here when the kernel runs (g_bits unused); the
                      // global-scale group launch writes it
  int64_t rows, cols; // the shape (used for tensors whose rows the block size does not divide)
};

// What the error-reduction pass does with the codes (see mx_error_stats.cu).
enum StatsMode { kGiven = 0, kRecompute = 1, kStore = 2 };

// Grouped launches: count <= kMaxGroup tensors sharing block size, format and dtype, one
// persistent grid split among them.
cudaError_t run_quantize_group(const TensorArgs* t, int count, bool bf16, int block, int fmt,
                               cudaStream_t stream, int* launches);
cudaError_t run_dequantize_group(const TensorArgs* t, int count, bool bf16out, int block, int fmt,
                                 cudaStream_t stream, int* launches);
cudaError_t run_stats_group(const TensorArgs* t, int count, bool bf16, int block, int fmt,
                            StatsMode mode, void* workspace, cudaStream_t stream, int* launches);

// Fake quantization (the round trip quantize -> dequantize in one pass): y = E2M1 * S * g of the
// codes mx_quantize would store, as bf16 (ybf16) or fp32; nothing else is written.
cudaError_t run_fake_quantize(const void* x, bool bf16, int64_t numel, int block, int fmt,
                              uint16_t g_bits, void* y, bool ybf16, cudaStream_t stream,
                              int* launches);

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
// The `count` elements from `first` on (a multiple of the block size N <= 8, fewer than an item of
// the calling kernel): quantize + pack them with plain per-element code.
cudaError_t run_quantize_tail(const void* x, bool bf16, int64_t first, int count, int N, int fmt,
                              uint16_t g_bits, const uint16_t* g_dev, uint8_t* packed,
                              uint8_t* scales, cudaStream_t stream, int* launches);
// One CTA's partial sums of the error reduction (64 bytes; the workspace holds one per CTA after
// a header of kMaxGroup 64-byte counters).
struct StatsPartial {
  double sse_elem, sse_max, sse_zero, pad;
  unsigned long long n_zero_blocks, n_scale_sat, n_elem_sat, pad2;
};
// One CTA adds nparts partials in a fixed order and writes the mx_error_stats_t record.
cudaError_t launch_stats_final(const StatsPartial* part, int nparts, int64_t numel,
                               int64_t nblocks, void* out, cudaStream_t stream, int* launches);

// Ragged tensors (cols % block != 0): one thread per block with plain per-element code.  Outputs
// that are null are not produced: codes + scales (packed / scales), the round trip (y), the error
// record (out, with workspace; from stored codes when packed_in is given).
// g_dev: when set, g is read from device memory when the kernel runs (g_bits unused).
cudaError_t run_ragged(const void* x, bool bf16, int64_t rows, int64_t cols, int block, int fmt,
                       uint16_t g_bits, const uint16_t* g_dev, const uint8_t* packed_in,
                       const uint8_t* scales_in, uint8_t* packed, uint8_t* scales, void* y,
                       bool y_bf16, void* out, void* workspace, cudaStream_t stream,
                       int* launches);
cudaError_t run_ragged_dequantize(const uint8_t* packed, const uint8_t* scales, int64_t rows,
                                  int64_t cols, int block, int fmt, uint16_t g_bits,
                                  const uint16_t* g_dev, void* y, bool y_bf16,
                                  cudaStream_t stream, int* launches);

// Row-pitched modes of the whole-block kernels: bf16 tensors whose rows start on 16-byte
// boundaries (cols % 8 == 0) and whose length the block size does not divide; one tensor per
// launch.  Quantize (N >= 16): codes and scales (y null), or the round trip to y (bf16 or fp32;
// packed / scales unused).
bool rows_quantize_supported(bool bf16, int64_t rows, int64_t cols, int block);
cudaError_t run_rows_quantize(const void* x, int64_t rows, int64_t cols, int block, int fmt,
                              uint16_t g_bits, const uint16_t* g_dev, uint8_t* packed,
                              uint8_t* scales, void* y, bool y_bf16, cudaStream_t stream,
                              int* launches);
// The error reduction with recomputed codes (N >= 32), fused with quantize + pack when packed /
// scales are set; out: device mx_error_stats_t; workspace as for the error reduction.
bool rows_stats_supported(bool bf16, int64_t rows, int64_t cols, int block);
cudaError_t run_rows_stats(const void* x, int64_t rows, int64_t cols, int block, int fmt,
                           uint16_t g_bits, const uint16_t* g_dev, uint8_t* packed,
                           uint8_t* scales, void* out, void* workspace, cudaStream_t stream,
                           int* launches);
// Dequantize to bf16 (N >= 16) through row tiles written by TMA (mx_tma.cuh).
bool tile_dequantize_supported(bool y_bf16, int64_t rows, int64_t cols, int block);
cudaError_t run_tile_dequantize(const uint8_t* packed, const uint8_t* scales, int64_t rows,
                                int64_t cols, int block, int fmt, uint16_t g_bits,
                                const uint16_t* g_dev, void* y, cudaStream_t stream,
                                int* launches);

// Zeroes one last-CTA counter once the previous kernel in the stream is done with it (a one-thread
// kernel launched with programmatic serialization).
cudaError_t launch_counter_reset(unsigned int* counter, cudaStream_t stream, int* launches);

// C (m x n, fp32 or bf16) = alpha * dequant(A) dequant(B)^T for A (m x k) and B (n x k) stored
// with blocks of 16 along k and E4M3 scales; k a positive multiple of 256; scales in the
// tensor-core order written by run_scales_to_mma.  cta_pairs: 256 x 256 tiles of C computed by
// CTA pairs (tcgen05 cta_group::2) when m > 128, else 128 x 256 tiles, one per CTA.
cudaError_t run_matmul_nvfp4(const uint8_t* a_packed, const uint8_t* a_scales,
                             const uint8_t* b_packed, const uint8_t* b_scales, int64_t m,
                             int64_t n, int64_t k, float alpha, void* c, bool c_bf16,
                             bool cta_pairs, cudaStream_t stream, int* launches);
// C (m x n, fp32 or bf16) = A dequant(W)^T for bf16 activations A (m x k) and weights W (n x k)
// stored by the quantizer with blocks of `block` along k, E4M3 or UE5M3 scales and global scale g
// (g_bits, or read from g_dev when that is set); k a positive multiple of 64 and of block.
cudaError_t run_dequant_matmul(const void* a, int64_t m, int64_t k, const uint8_t* w_packed,
                               const uint8_t* w_scales, int64_t n, int block, int fmt,
                               uint16_t g_bits, const uint16_t* g_dev, void* c, bool c_bf16,
                               cudaStream_t stream, int* launches);
// Bytes of an operand's scales in tensor-core order, and the reordering kernel.
int64_t mma_scales_bytes(int64_t rows, int64_t k);
cudaError_t run_scales_to_mma(const uint8_t* scales, int64_t rows, int64_t k, uint8_t* out,
                              cudaStream_t stream, int* launches);
// Reads and clears the count of matmul CTAs whose bounded waits ran out (synchronizes).
cudaError_t matmul_gave_up(unsigned int* count);
// Test hook: marks the most recent matmul launch as abandoned on the current device, as a CTA
// whose waits ran out does (synchronizes).
cudaError_t matmul_abandon_last();

// Per-tensor FP16 scale of every tensor of a group: t[k].x -> *t[k].g_dev.
cudaError_t run_global_scale_group(const TensorArgs* t, int count, bool bf16, int fmt,
                                   void* workspace, cudaStream_t stream, int* launches);
cudaError_t run_global_scale(const void* x, bool bf16, int64_t numel, int fmt, uint16_t* out,
                             void* workspace, cudaStream_t stream, int* launches);
// Zeroes n last-CTA counters 64 bytes apart (counters[16 k], k < n <= 32) once the previous kernel
// in the stream is done with them (a one-warp kernel launched with programmatic serialization).
cudaError_t launch_counters_reset(unsigned int* counters, int n, cudaStream_t stream,
                                  int* launches);

}  // namespace mxk
