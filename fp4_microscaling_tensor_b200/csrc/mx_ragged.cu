// mx_ragged.cu -- tensors whose rows the block size N does not divide.
//
// Method: the microscaling article (hotelren.com/news/2192771) §1 cuts a tensor into blocks of
// 4-256 values and §3.1 item 2 quantizes each block; a row of cols values whose length N does not
// divide ends in a block of cols mod N values, quantized by the same rule with its own absmax and
// scale.  Layout: a row's codes take ceil(cols/2) bytes (element 2k in the low nibble of byte k;
// an odd last element leaves the high nibble 0), its scales ceil(cols/N) bytes, rows one after
// another.  For cols % N == 0 this is the layout of the whole-block kernels, which handle that
// case; these kernels cover the rest.
//
// One thread per block, grid-stride, with plain per-element code: absmax (first index of the
// largest |x|), scale s = RNE_fmt(a / (6 g)) and quotients x / (S g) by IEEE division (a correctly
// rounded quotient lands on a rounding midpoint only when the exact quotient does), E2M1 codes by
// the hardware RNE-saturating conversion.  Errors are formed and summed in double; each CTA
// writes one partial and one CTA adds the partials in a fixed order.
#include "mx_device.cuh"
#include "mx_launch.h"

namespace mxk {
namespace {

struct RaggedArgs {
  const void* x;
  int64_t rows, cols;
  int N;
  uint32_t g_bits;
  const uint8_t* packed_in;  // stored codes (error reduction from codes), or null
  const uint8_t* scales_in;
  uint8_t* packed;           // codes written, or null
  uint8_t* scales;
  void* y;                   // round trip written (fake quantize), or null
  int y_bf16;
  StatsPartial* part;        // per-CTA partial sums, or null
};

template <typename T>
__device__ __forceinline__ float load_x(const T* p) {
  if constexpr (sizeof(T) == 2)
    return __uint_as_float((uint32_t)*reinterpret_cast<const uint16_t*>(p) << 16);
  else
    return *reinterpret_cast<const float*>(p);
}

__device__ __forceinline__ void store_y(void* y, int64_t i, float v, int bf16) {
  if (bf16)
    static_cast<__nv_bfloat16*>(y)[i] = __float2bfloat16_rn(v);
  else
    static_cast<float*>(y)[i] = v;
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ unsigned long long warp_sum_u(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <typename T, int FMT>
__global__ void __launch_bounds__(kThreads) k_ragged_blocks(const __grid_constant__ RaggedArgs a) {
  const float g = fp16_bits_to_float((uint16_t)a.g_bits);
  const float g6 = __fmul_rn(6.0f, g);                   // exact
  const float sat_thr = __fmul_rn(g6, scale_max<FMT>());  // exact
  const int64_t nb = (a.cols + a.N - 1) / a.N, pb = (a.cols + 1) / 2;
  const int64_t total = a.rows * nb;
  double e_elem = 0.0, e_max = 0.0, e_zero = 0.0;
  unsigned long long c_zero = 0, c_ssat = 0, c_esat = 0;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / nb, b = i - r * nb, j0 = b * a.N;  // j0 even: whole bytes
    const int len = (int)(a.cols - j0 < a.N ? a.cols - j0 : a.N);
    const T* xr = static_cast<const T*>(a.x) + r * a.cols + j0;
    float amax = 0.0f;
    int imax = 0;
    for (int k = 0; k < len; ++k) {
      const float v = fabsf(load_x(xr + k));
      if (v > amax) { amax = v; imax = k; }
    }
    const uint32_t s = a.packed_in ? (uint32_t)a.scales_in[r * nb + b]
                                   : encode_scale<FMT>(__fdiv_rn(amax, g6));
    const float D = __fmul_rn(scale_value((int)s, FMT), g);  // exact
    if (a.scales) a.scales[r * nb + b] = (uint8_t)s;
    const int64_t byte0 = r * pb + j0 / 2;
    for (int k = 0; k < len; k += 2) {
      const bool two = k + 1 < len;
      const float v0 = load_x(xr + k), v1 = two ? load_x(xr + k + 1) : 0.0f;
      uint32_t c;
      if (a.packed_in) {
        c = a.packed_in[byte0 + k / 2];
      } else {
        const float q0 = D > 0.0f ? __fdiv_rn(v0, D) : __fmul_rn(v0, 0.0f);
        const float q1 = D > 0.0f ? __fdiv_rn(v1, D) : __fmul_rn(v1, 0.0f);
        c = cvt_e2m1x8(q0, q1, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f) & (two ? 0xFFu : 0xFu);
      }
      if (a.packed) a.packed[byte0 + k / 2] = (uint8_t)c;
      if (a.y) {
        store_y(a.y, r * a.cols + j0 + k, __fmul_rn(e2m1_to_float(c & 0xF), D), a.y_bf16);
        if (two) store_y(a.y, r * a.cols + j0 + k + 1, __fmul_rn(e2m1_to_float(c >> 4), D),
                         a.y_bf16);
      }
      if (a.part) {
        for (int t = 0; t < 1 + (int)two; ++t) {
          const float v = t ? v1 : v0;
          const double yv = (double)__fmul_rn(e2m1_to_float((c >> (4 * t)) & 0xF), D);  // exact
          const double d = (double)v - yv;                                           // exact
          if (!(D > 0.0f)) e_zero += (double)v * (double)v;
          else if (k + t == imax) e_max += d * d;
          else e_elem += d * d;
          if (D > 0.0f && fabsf(v) > __fmul_rn(6.0f, D)) ++c_esat;
        }
      }
    }
    if (a.part) {
      c_zero += D > 0.0f ? 0 : 1;
      c_ssat += amax > sat_thr ? 1 : 0;
    }
  }
  if (!a.part) return;
  // CTA partial, fixed order (lanes, then warps)
  __shared__ double sd[3][kThreads / 32];
  __shared__ unsigned long long su[3][kThreads / 32];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  e_elem = warp_sum_d(e_elem); e_max = warp_sum_d(e_max); e_zero = warp_sum_d(e_zero);
  c_zero = warp_sum_u(c_zero); c_ssat = warp_sum_u(c_ssat); c_esat = warp_sum_u(c_esat);
  if (lane == 0) {
    sd[0][w] = e_elem; sd[1][w] = e_max; sd[2][w] = e_zero;
    su[0][w] = c_zero; su[1][w] = c_ssat; su[2][w] = c_esat;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    StatsPartial p{};
    for (int k = 0; k < kThreads / 32; ++k) {
      p.sse_elem += sd[0][k]; p.sse_max += sd[1][k]; p.sse_zero += sd[2][k];
      p.n_zero_blocks += su[0][k]; p.n_scale_sat += su[1][k]; p.n_elem_sat += su[2][k];
    }
    a.part[blockIdx.x] = p;
  }
}

// One thread per code byte: y = E2M1 x S x g (exact), bf16 = its round to nearest even.
template <int FMT>
__global__ void __launch_bounds__(kThreads)
    k_ragged_dequantize(const uint8_t* __restrict__ packed, const uint8_t* __restrict__ scales,
                        int64_t rows, int64_t cols, int N, uint16_t g_bits, void* y, int y_bf16) {
  const float g = fp16_bits_to_float(g_bits);
  const int64_t nb = (cols + N - 1) / N, pb = (cols + 1) / 2, total = rows * pb;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / pb, j = 2 * (i - r * pb);
    const uint32_t c = packed[i];
    const float D = __fmul_rn(scale_value((int)scales[r * nb + j / N], FMT), g);  // one block
    store_y(y, r * cols + j, __fmul_rn(e2m1_to_float(c & 0xF), D), y_bf16);
    if (j + 1 < cols) store_y(y, r * cols + j + 1, __fmul_rn(e2m1_to_float(c >> 4), D), y_bf16);
  }
}

constexpr int kMaxRaggedGrid = kMaxReduceCtas - 2 * kMaxGroup;  // partials after the header

template <typename T, int FMT>
cudaError_t launch_ragged(const RaggedArgs& args, int64_t nblocks, void* out, cudaStream_t stream,
                          int* launches) {
  const int grid = persistent_grid((const void*)k_ragged_blocks<T, FMT>, nblocks, 1,
                                   kMaxRaggedGrid);
  k_ragged_blocks<T, FMT><<<grid, kThreads, 0, stream>>>(args);
  ++*launches;
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess && args.part)
    e = launch_stats_final(args.part, grid, args.rows * args.cols, nblocks, out, stream, launches);
  return e;
}

}  // namespace

cudaError_t run_ragged(const void* x, bool bf16, int64_t rows, int64_t cols, int block, int fmt,
                       uint16_t g_bits, const uint8_t* packed_in, const uint8_t* scales_in,
                       uint8_t* packed, uint8_t* scales, void* y, bool y_bf16, void* out,
                       void* workspace, cudaStream_t stream, int* launches) {
  RaggedArgs args{x, rows, cols, block, g_bits, packed_in, scales_in, packed, scales, y,
                  y_bf16 ? 1 : 0, nullptr};
  if (out)  // partials after the workspace's 64-byte counter headers
    args.part = reinterpret_cast<StatsPartial*>(static_cast<char*>(workspace) + 64 * kMaxGroup);
  const int64_t nblocks = rows * ((cols + block - 1) / block);
  if (bf16)
    return fmt == kUE5M3 ? launch_ragged<uint16_t, kUE5M3>(args, nblocks, out, stream, launches)
                         : launch_ragged<uint16_t, kE4M3>(args, nblocks, out, stream, launches);
  return fmt == kUE5M3 ? launch_ragged<float, kUE5M3>(args, nblocks, out, stream, launches)
                       : launch_ragged<float, kE4M3>(args, nblocks, out, stream, launches);
}

cudaError_t run_ragged_dequantize(const uint8_t* packed, const uint8_t* scales, int64_t rows,
                                  int64_t cols, int block, int fmt, uint16_t g_bits, void* y,
                                  bool y_bf16, cudaStream_t stream, int* launches) {
  const int64_t bytes = rows * ((cols + 1) / 2);
  if (fmt == kUE5M3) {
    const int grid = persistent_grid((const void*)k_ragged_dequantize<kUE5M3>, bytes, 1);
    k_ragged_dequantize<kUE5M3><<<grid, kThreads, 0, stream>>>(packed, scales, rows, cols, block,
                                                               g_bits, y, y_bf16 ? 1 : 0);
  } else {
    const int grid = persistent_grid((const void*)k_ragged_dequantize<kE4M3>, bytes, 1);
    k_ragged_dequantize<kE4M3><<<grid, kThreads, 0, stream>>>(packed, scales, rows, cols, block,
                                                              g_bits, y, y_bf16 ? 1 : 0);
  }
  ++*launches;
  return cudaGetLastError();
}

}  // namespace mxk
