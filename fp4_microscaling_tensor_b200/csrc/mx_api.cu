// mx_api.cu -- the C ABI declared in include/mx.h: argument checks on the host, then the kernel
// launches of mx_quantize.cu, mx_dequantize.cu, mx_error_stats.cu and mx_global_scale.cu on the
// caller's stream.  Nothing is allocated and nothing is synchronized here.
#include <atomic>
#include <cmath>

#include "../../include/mx.h"
#include "mx_device.cuh"
#include "mx_launch.h"

static_assert(sizeof(mx_error_stats_t) == 64, "mx_error_stats_t layout");
static_assert(sizeof(mx_tensor_t) == 72, "mx_tensor_t layout");
static_assert(MX_MAX_GROUP == mxk::kMaxGroup, "group size");

namespace {

std::atomic<long long> g_launches{0};  // diagnostic: kernels enqueued by this library
std::atomic<int> g_fail_next{0};       // test hook: calls still to fail with MX_ERR_CUDA

// True when an armed test failure is consumed by this call (nothing is enqueued then).
bool injected_failure() {
  int n = g_fail_next.load();
  while (n > 0) {
    if (g_fail_next.compare_exchange_weak(n, n - 1)) return true;
  }
  return false;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_block(int block) {
  return block == 4 || block == 8 || block == 16 || block == 32 || block == 64 || block == 128 ||
         block == 256;
}

// g must be a finite, positive binary16 (subnormals allowed).
bool valid_g(uint16_t g) {
  const unsigned e = (g >> 10) & 31u;
  return (g & 0x8000u) == 0 && e != 31u && (g & 0x7FFFu) != 0;
}

bool valid_dtype(int t) { return t == MX_F32 || t == MX_BF16; }
bool valid_fmt(int f) { return f == MX_SCALE_E4M3 || f == MX_SCALE_UE5M3; }

// rows, cols >= 0, product representable; returns false on overflow.
bool shape_ok(int64_t rows, int64_t cols) {
  if (rows < 0 || cols < 0) return false;
  if (rows != 0 && cols > (int64_t(1) << 62) / rows) return false;
  return true;
}

mx_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MX_OK : MX_ERR_CUDA; }

size_t stats_ws_bytes() { return (size_t)mxk::kMaxReduceCtas * 64; }
size_t amax_ws_bytes() { return (size_t)mxk::kMaxReduceCtas * 4; }

}  // namespace

extern "C" {

mx_status mx_quantize(const void* x, mx_dtype xt, int64_t rows, int64_t cols, int block,
                      mx_scale_fmt fmt, uint16_t global_scale_fp16, uint8_t* packed,
                      uint8_t* scales, cudaStream_t stream) {
  if (!valid_dtype(xt) || !valid_fmt(fmt) || !valid_g(global_scale_fp16) || !shape_ok(rows, cols))
    return MX_ERR_INVALID_ARG;
  if (!valid_block(block)) return MX_ERR_UNSUPPORTED;
  const int64_t numel = rows * cols;
  if (numel == 0) return MX_OK;
  if (!x || !packed || !scales) return MX_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed) || !aligned16(scales)) return MX_ERR_MISALIGNED;
  if (injected_failure()) return MX_ERR_CUDA;
  int n = 0;
  const cudaError_t e =
      cols % block != 0
          ? mxk::run_ragged(x, xt == MX_BF16, rows, cols, block, (int)fmt, global_scale_fp16,
                            nullptr, nullptr, nullptr, packed, scales, nullptr, false, nullptr,
                            nullptr, stream, &n)
          : mxk::run_quantize(x, xt == MX_BF16, numel, block, (int)fmt, global_scale_fp16, packed,
                              scales, stream, &n);
  g_launches += n;
  return from_cuda(e);
}

mx_status mx_dequantize(const uint8_t* packed, const uint8_t* scales, int64_t rows, int64_t cols,
                        int block, mx_scale_fmt fmt, uint16_t global_scale_fp16, void* y,
                        mx_dtype yt, cudaStream_t stream) {
  if (!valid_dtype(yt) || !valid_fmt(fmt) || !valid_g(global_scale_fp16) || !shape_ok(rows, cols))
    return MX_ERR_INVALID_ARG;
  if (!valid_block(block)) return MX_ERR_UNSUPPORTED;
  const int64_t numel = rows * cols;
  if (numel == 0) return MX_OK;
  if (!packed || !scales || !y) return MX_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(scales) || !aligned16(y)) return MX_ERR_MISALIGNED;
  if (injected_failure()) return MX_ERR_CUDA;
  int n = 0;
  const cudaError_t e =
      cols % block != 0
          ? mxk::run_ragged_dequantize(packed, scales, rows, cols, block, (int)fmt,
                                       global_scale_fp16, nullptr, y, yt == MX_BF16, stream, &n)
          : mxk::run_dequantize(packed, scales, numel, block, (int)fmt, global_scale_fp16, y,
                                yt == MX_BF16, stream, &n);
  g_launches += n;
  return from_cuda(e);
}

mx_status mx_fake_quantize(const void* x, mx_dtype xt, int64_t rows, int64_t cols, int block,
                           mx_scale_fmt fmt, uint16_t global_scale_fp16, void* y, mx_dtype yt,
                           cudaStream_t stream) {
  if (!valid_dtype(xt) || !valid_dtype(yt) || !valid_fmt(fmt) || !valid_g(global_scale_fp16) ||
      !shape_ok(rows, cols))
    return MX_ERR_INVALID_ARG;
  if (!valid_block(block)) return MX_ERR_UNSUPPORTED;
  const int64_t numel = rows * cols;
  if (numel == 0) return MX_OK;
  if (!x || !y) return MX_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return MX_ERR_MISALIGNED;
  if (injected_failure()) return MX_ERR_CUDA;
  int n = 0;
  const cudaError_t e =
      cols % block != 0
          ? mxk::run_ragged(x, xt == MX_BF16, rows, cols, block, (int)fmt, global_scale_fp16,
                            nullptr, nullptr, nullptr, nullptr, nullptr, y, yt == MX_BF16,
                            nullptr, nullptr, stream, &n)
          : mxk::run_fake_quantize(x, xt == MX_BF16, numel, block, (int)fmt, global_scale_fp16,
                                   y, yt == MX_BF16, stream, &n);
  g_launches += n;
  return from_cuda(e);
}

size_t mx_error_stats_workspace_size(int64_t rows, int64_t cols, int block) {
  (void)rows;
  (void)cols;
  (void)block;
  return stats_ws_bytes();
}

mx_status mx_error_stats(const void* x, mx_dtype xt, int64_t rows, int64_t cols, int block,
                         mx_scale_fmt fmt, uint16_t global_scale_fp16, const uint8_t* packed,
                         const uint8_t* scales, mx_error_stats_t* out_dev, void* workspace,
                         size_t ws_bytes, cudaStream_t stream) {
  if (!valid_dtype(xt) || !valid_fmt(fmt) || !valid_g(global_scale_fp16) || !shape_ok(rows, cols))
    return MX_ERR_INVALID_ARG;
  if (!valid_block(block)) return MX_ERR_UNSUPPORTED;
  if ((packed == nullptr) != (scales == nullptr)) return MX_ERR_INVALID_ARG;
  if (!out_dev) return MX_ERR_INVALID_ARG;
  const int64_t numel = rows * cols;
  if (numel != 0 && !x) return MX_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < stats_ws_bytes()) return MX_ERR_WORKSPACE;
  if ((numel != 0 && !aligned16(x)) || !aligned16(out_dev) || !aligned16(workspace) ||
      (packed && (!aligned16(packed) || !aligned16(scales))))
    return MX_ERR_MISALIGNED;
  if (injected_failure()) return MX_ERR_CUDA;
  int n = 0;
  const cudaError_t e =
      numel != 0 && cols % block != 0
          ? mxk::run_ragged(x, xt == MX_BF16, rows, cols, block, (int)fmt, global_scale_fp16,
                            nullptr, packed, scales, nullptr, nullptr, nullptr, false, out_dev,
                            workspace, stream, &n)
          : mxk::run_error_stats(numel ? x : nullptr, xt == MX_BF16, numel, block, (int)fmt,
                                 global_scale_fp16, packed, scales, out_dev, workspace, stream,
                                 &n);
  g_launches += n;
  return from_cuda(e);
}

mx_status mx_quantize_stats(const void* x, mx_dtype xt, int64_t rows, int64_t cols, int block,
                            mx_scale_fmt fmt, uint16_t global_scale_fp16, uint8_t* packed,
                            uint8_t* scales, mx_error_stats_t* out_dev, void* workspace,
                            size_t ws_bytes, cudaStream_t stream) {
  if (!valid_dtype(xt) || !valid_fmt(fmt) || !valid_g(global_scale_fp16) || !shape_ok(rows, cols))
    return MX_ERR_INVALID_ARG;
  if (!valid_block(block)) return MX_ERR_UNSUPPORTED;
  if (!out_dev) return MX_ERR_INVALID_ARG;
  const int64_t numel = rows * cols;
  if (numel != 0 && (!x || !packed || !scales)) return MX_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < stats_ws_bytes()) return MX_ERR_WORKSPACE;
  if ((numel != 0 && (!aligned16(x) || !aligned16(packed) || !aligned16(scales))) ||
      !aligned16(out_dev) || !aligned16(workspace))
    return MX_ERR_MISALIGNED;
  if (injected_failure()) return MX_ERR_CUDA;
  int n = 0;
  const cudaError_t e =
      numel != 0 && cols % block != 0
          ? mxk::run_ragged(x, xt == MX_BF16, rows, cols, block, (int)fmt, global_scale_fp16,
                            nullptr, nullptr, nullptr, packed, scales, nullptr, false, out_dev,
                            workspace, stream, &n)
          : mxk::run_quantize_stats(numel ? x : nullptr, xt == MX_BF16, numel, block, (int)fmt,
                                    global_scale_fp16, packed, scales, out_dev, workspace, stream,
                                    &n);
  g_launches += n;
  return from_cuda(e);
}

mx_status mx_error_stats_means(const mx_error_stats_t* record, double* mse4) {
  if (!record || !mse4) return MX_ERR_INVALID_ARG;
  if (record->numel <= 0) {
    mse4[0] = mse4[1] = mse4[2] = mse4[3] = 0.0;
    return MX_OK;
  }
  const double n = (double)record->numel;
  mse4[0] = record->sse_elem / n;
  mse4[1] = record->sse_max / n;
  mse4[2] = record->sse_zero / n;
  mse4[3] = mse4[0] + mse4[1] + mse4[2];
  return MX_OK;
}

size_t mx_global_scale_workspace_size(int64_t rows, int64_t cols) {
  (void)rows;
  (void)cols;
  return amax_ws_bytes();
}

mx_status mx_global_scale(const void* x, mx_dtype xt, int64_t rows, int64_t cols, mx_scale_fmt fmt,
                          uint16_t* out_fp16_dev, void* workspace, size_t ws_bytes,
                          cudaStream_t stream) {
  if (!valid_dtype(xt) || !valid_fmt(fmt) || !shape_ok(rows, cols)) return MX_ERR_INVALID_ARG;
  if (!out_fp16_dev) return MX_ERR_INVALID_ARG;
  const int64_t numel = rows * cols;
  if (numel != 0 && !x) return MX_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < amax_ws_bytes()) return MX_ERR_WORKSPACE;
  if ((numel != 0 && !aligned16(x)) || !aligned16(workspace)) return MX_ERR_MISALIGNED;
  if (injected_failure()) return MX_ERR_CUDA;
  int n = 0;
  const cudaError_t e = mxk::run_global_scale(x, xt == MX_BF16, numel, (int)fmt, out_fp16_dev,
                                              workspace, stream, &n);
  g_launches += n;
  return from_cuda(e);
}

}  // extern "C"

namespace {

// Value of a finite binary16 bit pattern (exact in float).
float half_value(uint16_t h) {
  const int e = (h >> 10) & 31, m = h & 1023;
  const float v = e == 0 ? std::ldexp((float)m, -24) : std::ldexp((float)(1024 + m), e - 25);
  return (h & 0x8000u) ? -v : v;
}

mx_status matmul_impl(const uint8_t* a_packed, const uint8_t* a_scales, uint16_t a_g,
                      const uint8_t* b_packed, const uint8_t* b_scales, uint16_t b_g, int64_t m,
                      int64_t n, int64_t k, int block, mx_scale_fmt fmt, void* c, mx_dtype ct,
                      bool cta_pairs, cudaStream_t stream) {
  if (!valid_fmt(fmt) || !valid_dtype(ct) || !valid_g(a_g) || !valid_g(b_g)) return MX_ERR_INVALID_ARG;
  if (m < 0 || n < 0 || k < 0 || m >= (int64_t(1) << 31) || n >= (int64_t(1) << 31) ||
      k > (int64_t(1) << 40))
    return MX_ERR_INVALID_ARG;
  if (block != 16 || fmt != MX_SCALE_E4M3 || k == 0 || k % 256 != 0) return MX_ERR_UNSUPPORTED;
  if (m == 0 || n == 0) return MX_OK;
  // TMA coordinates are 32-bit: k / 2 bytes per row and the prepared scales as 256-byte rows
  if (k >= (int64_t(1) << 31) || mxk::mma_scales_bytes(m, k) / 256 >= (int64_t(1) << 31) ||
      mxk::mma_scales_bytes(n, k) / 256 >= (int64_t(1) << 31))
    return MX_ERR_UNSUPPORTED;
  if (!a_packed || !a_scales || !b_packed || !b_scales || !c) return MX_ERR_INVALID_ARG;
  if (!aligned16(a_packed) || !aligned16(a_scales) || !aligned16(b_packed) ||
      !aligned16(b_scales) || !aligned16(c))
    return MX_ERR_MISALIGNED;
  if (injected_failure()) return MX_ERR_CUDA;
  int launches = 0;
  const cudaError_t e = mxk::run_matmul_nvfp4(a_packed, a_scales, b_packed, b_scales, m, n, k,
                                              half_value(a_g) * half_value(b_g), c, ct == MX_BF16,
                                              cta_pairs, stream, &launches);
  g_launches += launches;
  return from_cuda(e);
}

}  // namespace

extern "C" {

mx_status mx_matmul(const uint8_t* a_packed, const uint8_t* a_scales, uint16_t a_g,
                    const uint8_t* b_packed, const uint8_t* b_scales, uint16_t b_g, int64_t m,
                    int64_t n, int64_t k, int block, mx_scale_fmt fmt, void* c, mx_dtype ct,
                    cudaStream_t stream) {
  return matmul_impl(a_packed, a_scales, a_g, b_packed, b_scales, b_g, m, n, k, block, fmt, c, ct,
                     false, stream);
}

mx_status mx_matmul_pair(const uint8_t* a_packed, const uint8_t* a_scales, uint16_t a_g,
                         const uint8_t* b_packed, const uint8_t* b_scales, uint16_t b_g,
                         int64_t m, int64_t n, int64_t k, int block, mx_scale_fmt fmt, void* c,
                         mx_dtype ct, cudaStream_t stream) {
  return matmul_impl(a_packed, a_scales, a_g, b_packed, b_scales, b_g, m, n, k, block, fmt, c, ct,
                     true, stream);
}

mx_status mx_dequant_matmul(const void* a, int64_t m, int64_t k, const uint8_t* w_packed,
                            const uint8_t* w_scales, int64_t n, int block, mx_scale_fmt fmt,
                            uint16_t w_global_scale_fp16, const uint16_t* w_global_scale_dev,
                            void* c, mx_dtype ct, cudaStream_t stream) {
  if (!valid_fmt(fmt) || !valid_dtype(ct)) return MX_ERR_INVALID_ARG;
  if (!w_global_scale_dev && !valid_g(w_global_scale_fp16)) return MX_ERR_INVALID_ARG;
  if (m < 0 || n < 0 || k < 0 || m >= (int64_t(1) << 31) || n >= (int64_t(1) << 31) ||
      k >= (int64_t(1) << 31))
    return MX_ERR_INVALID_ARG;
  if (!valid_block(block) || k == 0 || k % 64 != 0 || k % block != 0) return MX_ERR_UNSUPPORTED;
  if (m == 0 || n == 0) return MX_OK;
  if (!a || !w_packed || !w_scales || !c) return MX_ERR_INVALID_ARG;
  if (!aligned16(a) || !aligned16(w_packed) || !aligned16(w_scales) || !aligned16(c) ||
      (reinterpret_cast<uintptr_t>(w_global_scale_dev) & 1u) != 0)
    return MX_ERR_MISALIGNED;
  if (injected_failure()) return MX_ERR_CUDA;
  int launches = 0;
  const cudaError_t e = mxk::run_dequant_matmul(a, m, k, w_packed, w_scales, n, block, (int)fmt,
                                                w_global_scale_fp16, w_global_scale_dev, c,
                                                ct == MX_BF16, stream, &launches);
  g_launches += launches;
  return from_cuda(e);
}

size_t mx_matmul_scales_size(int64_t rows, int64_t k) {
  if (rows < 0 || rows >= (int64_t(1) << 31) || k <= 0 || k % 256 != 0 || k > (int64_t(1) << 40))
    return 0;
  return (size_t)mxk::mma_scales_bytes(rows, k);
}

mx_status mx_matmul_prepare_scales(const uint8_t* scales, int64_t rows, int64_t k, uint8_t* out,
                                   size_t out_bytes, cudaStream_t stream) {
  if (rows < 0 || rows >= (int64_t(1) << 31) || k < 0 || k > (int64_t(1) << 40))
    return MX_ERR_INVALID_ARG;
  if (k == 0 || k % 256 != 0) return MX_ERR_UNSUPPORTED;
  if (rows == 0) return MX_OK;
  if (!scales || !out) return MX_ERR_INVALID_ARG;
  if (out_bytes < mx_matmul_scales_size(rows, k)) return MX_ERR_WORKSPACE;
  if (!aligned16(scales) || !aligned16(out)) return MX_ERR_MISALIGNED;
  if (injected_failure()) return MX_ERR_CUDA;
  int launches = 0;
  const cudaError_t e = mxk::run_scales_to_mma(scales, rows, k, out, stream, &launches);
  g_launches += launches;
  return from_cuda(e);
}

mx_status mx_matmul_gave_up(unsigned int* count) {
  if (!count) return MX_ERR_INVALID_ARG;
  return from_cuda(mxk::matmul_gave_up(count));
}

mx_status mx_test_matmul_abandon_last(void) { return from_cuda(mxk::matmul_abandon_last()); }

namespace {

// Checks shared by the grouped calls: per tensor shape, pointers (`need` says which) and g.
enum : unsigned { kNeedX = 1, kNeedY = 2, kNeedCodes = 4, kNeedStats = 8, kNeedGOut = 16 };

mx_status check_group(const mx_tensor_t* t, int count, int block, unsigned need,
                      mxk::TensorArgs* args) {
  if (!t || count < 1 || count > MX_MAX_GROUP) return MX_ERR_INVALID_ARG;
  for (int k = 0; k < count; ++k) {
    const mx_tensor_t& d = t[k];
    // g: an output (kNeedGOut), read from device memory (global_scale_dev), or the bit pattern
    const bool g_ok = (need & kNeedGOut) ? d.global_scale_dev != nullptr
                                         : (d.global_scale_dev != nullptr ||
                                            valid_g(d.global_scale_fp16));
    if (!shape_ok(d.rows, d.cols) || !g_ok || d.reserved[0] || d.reserved[1] || d.reserved[2])
      return MX_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(d.global_scale_dev) & 1u) != 0) return MX_ERR_MISALIGNED;
    const int64_t numel = d.rows * d.cols;
    if ((need & kNeedStats) && !d.stats) return MX_ERR_INVALID_ARG;
    if ((need & kNeedStats) && !aligned16(d.stats)) return MX_ERR_MISALIGNED;
    if (numel != 0) {
      if (((need & kNeedX) && !d.x) || ((need & kNeedY) && !d.y) ||
          ((need & kNeedCodes) && (!d.packed || !d.scales)))
        return MX_ERR_INVALID_ARG;
      if (((need & kNeedX) && !aligned16(d.x)) || ((need & kNeedY) && !aligned16(d.y)) ||
          ((need & kNeedCodes) && (!aligned16(d.packed) || !aligned16(d.scales))))
        return MX_ERR_MISALIGNED;
    }
    args[k] = {d.x, d.y, d.packed, d.scales, d.stats, numel, d.global_scale_fp16,
               d.global_scale_dev, d.rows, d.cols};
  }
  return MX_OK;
}

// Splits checked tensors into those of whole blocks (one grouped launch) and ragged ones (cols %
// block != 0, non-empty: the row-wise kernels, one launch each, after the grouped one).
int split_ragged(const mxk::TensorArgs* args, int count, int block, mxk::TensorArgs* whole,
                 mxk::TensorArgs* ragged, int* nragged) {
  int nw = 0;
  *nragged = 0;
  for (int k = 0; k < count; ++k) {
    if (args[k].numel != 0 && args[k].cols % block != 0) ragged[(*nragged)++] = args[k];
    else whole[nw++] = args[k];
  }
  return nw;
}

}  // namespace

mx_status mx_quantize_group(const mx_tensor_t* tensors, int count, mx_dtype xt, int block,
                            mx_scale_fmt fmt, cudaStream_t stream) {
  if (!valid_dtype(xt) || !valid_fmt(fmt)) return MX_ERR_INVALID_ARG;
  if (!valid_block(block)) return MX_ERR_UNSUPPORTED;
  mxk::TensorArgs args[MX_MAX_GROUP], whole[MX_MAX_GROUP], ragged[MX_MAX_GROUP];
  const mx_status st = check_group(tensors, count, block, kNeedX | kNeedCodes, args);
  if (st != MX_OK) return st;
  if (injected_failure()) return MX_ERR_CUDA;
  int n = 0, nr = 0;
  const int nw = split_ragged(args, count, block, whole, ragged, &nr);
  cudaError_t e = nw ? mxk::run_quantize_group(whole, nw, xt == MX_BF16, block, (int)fmt, stream,
                                               &n)
                     : cudaSuccess;
  for (int k = 0; k < nr && e == cudaSuccess; ++k) {
    const mxk::TensorArgs& t = ragged[k];
    e = mxk::run_ragged(t.x, xt == MX_BF16, t.rows, t.cols, block, (int)fmt, t.g_bits, t.g_dev,
                        nullptr, nullptr, t.packed, t.scales, nullptr, false, nullptr, nullptr,
                        stream, &n);
  }
  g_launches += n;
  return from_cuda(e);
}

mx_status mx_dequantize_group(const mx_tensor_t* tensors, int count, int block, mx_scale_fmt fmt,
                              mx_dtype yt, cudaStream_t stream) {
  if (!valid_dtype(yt) || !valid_fmt(fmt)) return MX_ERR_INVALID_ARG;
  if (!valid_block(block)) return MX_ERR_UNSUPPORTED;
  mxk::TensorArgs args[MX_MAX_GROUP], whole[MX_MAX_GROUP], ragged[MX_MAX_GROUP];
  const mx_status st = check_group(tensors, count, block, kNeedY | kNeedCodes, args);
  if (st != MX_OK) return st;
  if (injected_failure()) return MX_ERR_CUDA;
  int n = 0, nr = 0;
  const int nw = split_ragged(args, count, block, whole, ragged, &nr);
  cudaError_t e = nw ? mxk::run_dequantize_group(whole, nw, yt == MX_BF16, block, (int)fmt,
                                                 stream, &n)
                     : cudaSuccess;
  for (int k = 0; k < nr && e == cudaSuccess; ++k) {
    const mxk::TensorArgs& t = ragged[k];
    e = mxk::run_ragged_dequantize(t.packed, t.scales, t.rows, t.cols, block, (int)fmt, t.g_bits,
                                   t.g_dev, t.y, yt == MX_BF16, stream, &n);
  }
  g_launches += n;
  return from_cuda(e);
}

mx_status mx_quantize_stats_group(const mx_tensor_t* tensors, int count, mx_dtype xt, int block,
                                  mx_scale_fmt fmt, void* workspace, size_t ws_bytes,
                                  cudaStream_t stream) {
  if (!valid_dtype(xt) || !valid_fmt(fmt)) return MX_ERR_INVALID_ARG;
  if (!valid_block(block)) return MX_ERR_UNSUPPORTED;
  mxk::TensorArgs args[MX_MAX_GROUP];
  const mx_status st = check_group(tensors, count, block, kNeedX | kNeedCodes | kNeedStats, args);
  if (st != MX_OK) return st;
  if (!workspace || ws_bytes < stats_ws_bytes()) return MX_ERR_WORKSPACE;
  if (!aligned16(workspace)) return MX_ERR_MISALIGNED;
  if (injected_failure()) return MX_ERR_CUDA;
  mxk::TensorArgs whole[MX_MAX_GROUP], ragged[MX_MAX_GROUP];
  int n = 0, nr = 0;
  const int nw = split_ragged(args, count, block, whole, ragged, &nr);
  // the ragged tensors reuse the workspace after the grouped launch (same stream, in order)
  cudaError_t e = nw ? mxk::run_stats_group(whole, nw, xt == MX_BF16, block, (int)fmt,
                                            mxk::kStore, workspace, stream, &n)
                     : cudaSuccess;
  for (int k = 0; k < nr && e == cudaSuccess; ++k) {
    const mxk::TensorArgs& t = ragged[k];
    e = mxk::run_ragged(t.x, xt == MX_BF16, t.rows, t.cols, block, (int)fmt, t.g_bits, t.g_dev,
                        nullptr, nullptr, t.packed, t.scales, nullptr, false, t.stats, workspace,
                        stream, &n);
  }
  g_launches += n;
  return from_cuda(e);
}

mx_status mx_global_scale_group(const mx_tensor_t* tensors, int count, mx_dtype xt,
                                 mx_scale_fmt fmt, void* workspace, size_t ws_bytes,
                                 cudaStream_t stream) {
  if (!valid_dtype(xt) || !valid_fmt(fmt)) return MX_ERR_INVALID_ARG;
  mxk::TensorArgs args[MX_MAX_GROUP];
  const mx_status st = check_group(tensors, count, 1, kNeedX | kNeedGOut, args);
  if (st != MX_OK) return st;
  if (!workspace || ws_bytes < amax_ws_bytes()) return MX_ERR_WORKSPACE;
  if (!aligned16(workspace)) return MX_ERR_MISALIGNED;
  if (injected_failure()) return MX_ERR_CUDA;
  int n = 0;
  const cudaError_t e =
      mxk::run_global_scale_group(args, count, xt == MX_BF16, (int)fmt, workspace, stream, &n);
  g_launches += n;
  return from_cuda(e);
}

const char* mx_status_string(mx_status status) {
  switch (status) {
    case MX_OK: return "MX_OK";
    case MX_ERR_INVALID_ARG: return "MX_ERR_INVALID_ARG: invalid argument";
    case MX_ERR_UNSUPPORTED: return "MX_ERR_UNSUPPORTED: block size not in {4,8,16,32,64,128,256}";
    case MX_ERR_MISALIGNED: return "MX_ERR_MISALIGNED: pointer not 16-byte aligned";
    case MX_ERR_WORKSPACE: return "MX_ERR_WORKSPACE: workspace missing or too small";
    case MX_ERR_CUDA: return "MX_ERR_CUDA: CUDA runtime error while enqueueing";
    default: return "unknown mx_status";
  }
}

long long mx_kernel_launches(void) { return g_launches.load(); }

int mx_test_fail_next_calls(int count) { return g_fail_next.exchange(count > 0 ? count : 0); }

}  // extern "C"
