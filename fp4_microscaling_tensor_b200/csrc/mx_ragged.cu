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
// bf16 tensors whose rows start on 16-byte boundaries (cols % 8 == 0) go to the row-pitched modes
// of the whole-block kernels (quantize and fake quantize for N >= 16, the error reduction with
// recomputed codes, fused or not, for N >= 32) and to the row-tile dequantize kernel (bf16 output,
// N >= 16; tiles written by TMA, mx_tma.cuh).  The rest runs here:
// one warp per row, lanes over consecutive element pairs (coalesced loads and byte stores), block
// maxima by segmented warp reductions; scale s = RNE_fmt(a / (6 g)) and quotients x / (S g) by
// IEEE division (a correctly rounded quotient lands on a rounding midpoint only when the exact
// quotient does), E2M1 codes by the hardware RNE-saturating conversion.  Errors are formed and
// summed in double; each CTA writes one partial and one CTA adds the partials in a fixed order.
#include "mx_device.cuh"
#include "mx_launch.h"

namespace mxk {
namespace {

struct RaggedArgs {
  const void* x;
  int64_t rows, cols;
  int N;
  uint32_t g_bits;
  const uint16_t* g_dev;     // g in device memory when set (g_bits unused)
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

// One warp per row (grid-stride over rows).  A warp step covers 256 elements of the row: lane l
// holds the 8 consecutive elements 8 l .. 8 l + 7 of the step (one 16-byte load when the row
// start allows it, else element loads), i.e. two blocks of 4, one block of 8, or 1 / G of a block
// of N = 8 G; a block's absmax and first max index are in-lane or segmented warp reductions over
// G lanes.  Elements past the row end are absent (zero for the absmax, nothing stored or summed).
// bf16 inputs use the exact reciprocal-multiply quotients of the whole-block kernels (snap21 for
// the scale, snap_quotient2 for the elements); fp32 inputs the IEEE division.
template <typename T, int FMT, int N>
__global__ void __launch_bounds__(kThreads) k_ragged_rows(const __grid_constant__ RaggedArgs a) {
  constexpr bool BF16 = sizeof(T) == 2;
  constexpr int BPL = N == 4 ? 2 : 1;          // blocks per lane
  constexpr int G = N <= 8 ? 1 : N / 8;        // lanes per block
  constexpr int EB = N == 4 ? 4 : 8;           // elements of a lane in one block
  const float g = fp16_bits_to_float(tensor_g_bits(a.g_bits, a.g_dev));
  const float g6 = __fmul_rn(6.0f, g);                   // exact
  const float r6 = __frcp_rn(g6);
  const float sat_thr = __fmul_rn(g6, scale_max<FMT>());  // exact
  const int cols = (int)a.cols;
  const int nb = (cols + N - 1) / N, pb = (cols + 1) / 2;
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  double e_elem = 0.0, e_max = 0.0, e_zero = 0.0;
  unsigned long long c_zero = 0, c_ssat = 0, c_esat = 0;
  for (int64_t r = warp; r < a.rows; r += nwarps) {
    const T* xr = static_cast<const T*>(a.x) + r * a.cols;
    const bool x_aligned = ((r * a.cols) & (BF16 ? 7 : 3)) == 0;  // 16-byte row start
    const int64_t prow = r * pb, srow = r * nb;
    // the 8 elements of this lane in the step from e0 (zero past the row end); the next step's
    // are loaded before the current step's work
    auto load_step = [&](int e0, float (&v)[8]) {
      const int j0 = e0 + 8 * lane;
      const int nv = max(0, min(8, cols - j0));
      if (nv == 8 && x_aligned) {
        if constexpr (BF16) {
          const uint4 w = ld_stream16(xr + j0);
          v[0] = bf16lo(w.x); v[1] = bf16hi(w.x); v[2] = bf16lo(w.y); v[3] = bf16hi(w.y);
          v[4] = bf16lo(w.z); v[5] = bf16hi(w.z); v[6] = bf16lo(w.w); v[7] = bf16hi(w.w);
        } else {
          const uint4 u0 = ld_stream16(xr + j0), u1 = ld_stream16(xr + j0 + 4);
          v[0] = __uint_as_float(u0.x); v[1] = __uint_as_float(u0.y);
          v[2] = __uint_as_float(u0.z); v[3] = __uint_as_float(u0.w);
          v[4] = __uint_as_float(u1.x); v[5] = __uint_as_float(u1.y);
          v[6] = __uint_as_float(u1.z); v[7] = __uint_as_float(u1.w);
        }
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = k < nv ? load_x(xr + j0 + k) : 0.0f;
      }
    };
    float vn[8];
    load_step(0, vn);
    for (int e0 = 0; e0 < cols; e0 += 256) {
      const int j0 = e0 + 8 * lane;  // this lane's first element
      const int nv = max(0, min(8, cols - j0));
      float v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) v[k] = vn[k];
      if (e0 + 256 < cols) load_step(e0 + 256, vn);
      uint32_t codes = 0;  // 8 codes, element k in nibble k
#pragma unroll
      for (int h = 0; h < BPL; ++h) {
        const float* vb = v + EB * h;
        const int jb0 = j0 + EB * h;           // this lane's first element of the block
        float m = 0.0f;
#pragma unroll
        for (int k = 0; k < EB; ++k) m = fmaxf(m, fabsf(vb[k]));
#pragma unroll
        for (int off = 1; off < G; off <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        const int jb = N >= 16 ? jb0 - EB * (lane & (G - 1)) : jb0;  // first element of the block
        const int b = jb / N;
        const bool block_here = jb < cols;
        const bool leader = (lane & (G - 1)) == 0;
        uint32_t s = 0;
        if (a.packed_in) {
          if (block_here) s = a.scales_in[srow + b];
        } else {
          s = BF16 ? encode_scale<FMT>(snap21(__fmul_rn(m, r6)))
                   : encode_scale<FMT>(__fdiv_rn(m, g6));
        }
        const float D = __fmul_rn(scale_value((int)s, FMT), g);  // exact
        if (a.scales && leader && block_here) a.scales[srow + b] = (uint8_t)s;
        uint32_t cb;  // this block's codes of this lane (EB nibbles)
        if (a.packed_in) {
          cb = 0;
#pragma unroll
          for (int k = 0; k < EB; k += 2)
            if (k < nv - EB * h) cb |= (uint32_t)a.packed_in[prow + (jb0 + k) / 2] << (4 * k);
        } else {
          float q[8];
          if constexpr (BF16) {
            const float rD = D > 0.0f ? __frcp_rn(D) : 0.0f;
#pragma unroll
            for (int k = 0; k < EB; k += 2) {
              const float2 qq =
                  snap_quotient2(__float_as_uint(vb[k]), __float_as_uint(vb[k + 1]), rD);
              q[k] = qq.x;
              q[k + 1] = qq.y;
            }
          } else {
#pragma unroll
            for (int k = 0; k < EB; ++k)
              q[k] = D > 0.0f ? __fdiv_rn(vb[k], D) : __fmul_rn(vb[k], 0.0f);
          }
          if constexpr (EB == 8) cb = cvt_e2m1x8(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]);
          else cb = cvt_e2m1x8(q[0], q[1], q[2], q[3], 0.f, 0.f, 0.f, 0.f) & 0xFFFFu;
        }
        codes |= cb << (4 * EB * h);
        if (a.part) {
          // first index of the block maximum: in-lane, then over the block's lanes
          int imax = INT_MAX;
#pragma unroll
          for (int k = EB - 1; k >= 0; --k)
            if (k < nv - EB * h && fabsf(vb[k]) == m) imax = jb0 + k;
#pragma unroll
          for (int off = 1; off < G; off <<= 1) imax = min(imax, __shfl_xor_sync(0xffffffffu, imax, off));
#pragma unroll
          for (int k = 0; k < EB; ++k) {
            if (k >= nv - EB * h) break;
            const float xv = vb[k];
            const double yv = (double)__fmul_rn(e2m1_to_float((cb >> (4 * k)) & 0xF), D);
            const double d = (double)xv - yv;  // exact
            if (!(D > 0.0f)) e_zero += (double)xv * (double)xv;
            else if (jb0 + k == imax) e_max += d * d;
            else e_elem += d * d;
            if (D > 0.0f && fabsf(xv) > __fmul_rn(6.0f, D)) ++c_esat;
          }
          if (leader && block_here) {
            c_zero += D > 0.0f ? 0 : 1;
            c_ssat += m > sat_thr ? 1 : 0;
          }
        }
        if (a.y) {
#pragma unroll
          for (int k = 0; k < EB; ++k)
            if (k < nv - EB * h)
              store_y(a.y, r * a.cols + jb0 + k,
                      __fmul_rn(e2m1_to_float((cb >> (4 * k)) & 0xF), D), a.y_bf16);
        }
      }
      if (a.packed && nv > 0) {
        if (nv & 1) codes &= ~(0xFu << (4 * nv));  // an odd row end leaves the high nibble 0
        if (nv == 8 && ((prow + j0 / 2) & 3) == 0) {
          *reinterpret_cast<uint32_t*>(a.packed + prow + j0 / 2) = codes;
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if (2 * k < nv) a.packed[prow + j0 / 2 + k] = (uint8_t)(codes >> (8 * k));
        }
      }
    }
  }
  if (!a.part) return;
  // CTA partial, fixed order (lanes, then warps)
  __shared__ double sd[3][kThreads / 32];
  __shared__ unsigned long long su[3][kThreads / 32];
  const int w = threadIdx.x >> 5;
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

// One warp per row, a warp step of 256 elements: lane l takes the 8 consecutive elements
// 8 l .. 8 l + 7 of the step (4 code bytes: one 4-byte load where the row's code bytes are
// aligned, else byte loads; one scale byte, two for N = 4), y = E2M1 x S x g (exact; S g from a
// per-CTA table), bf16 = its round to nearest even, stored as one 16-byte vector (fp32: two)
// where the row start allows, else element by element.  The next step's loads are issued before
// the current step's stores.  Elements past the row end are neither read nor written.
template <int FMT, int LOGN>
__global__ void __launch_bounds__(kThreads)
    k_ragged_dequantize(const uint8_t* __restrict__ packed, const uint8_t* __restrict__ scales,
                        int64_t rows, int64_t cols, uint16_t g_bits, const uint16_t* g_dev,
                        void* y, int y_bf16) {
  constexpr int N = 1 << LOGN;
  __shared__ float s_D[256];
  const float g = fp16_bits_to_float(tensor_g_bits(g_bits, g_dev));
  for (int c = threadIdx.x; c < 256; c += blockDim.x) s_D[c] = __fmul_rn(scale_value(c, FMT), g);
  __syncthreads();
  const int64_t nb = (cols + N - 1) >> LOGN, pb = (cols + 1) / 2;
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int icols = (int)cols;
  struct Step {
    uint32_t codes, sc;  // 8 codes (element k in nibble k); scale byte(s), N = 4: two
    int nv;              // elements of this lane in the step (0..8)
  };
  auto load = [&](int64_t r, int e0) {
    Step st{0u, 0u, 0};
    const int j0 = e0 + 8 * lane;
    st.nv = max(0, min(8, icols - j0));
    if (st.nv == 0) return st;
    const int64_t cb = r * pb + j0 / 2;  // first code byte
    if (st.nv == 8 && (cb & 3) == 0) {
      st.codes = __ldg(reinterpret_cast<const unsigned int*>(packed + cb));
    } else {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (2 * k < st.nv) st.codes |= (uint32_t)__ldg(packed + cb + k) << (8 * k);
    }
    const int64_t sb = r * nb + (j0 >> LOGN);
    st.sc = __ldg(scales + sb);
    if (N == 4 && st.nv > 4) st.sc |= (uint32_t)__ldg(scales + sb + 1) << 8;
    return st;
  };
  for (int64_t r = warp; r < rows; r += nwarps) {
    const int64_t y0 = r * cols;  // first element of the row in y
    const bool vec = y_bf16 ? (y0 & 7) == 0 : (y0 & 3) == 0;
    Step cur = load(r, 0);
    for (int e0 = 0; e0 < icols; e0 += 256) {
      const Step nxt = e0 + 256 < icols ? load(r, e0 + 256) : Step{0u, 0u, 0};
      if (cur.nv > 0) {
        const int j0 = e0 + 8 * lane;
        float v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float D = s_D[N == 4 && k >= 4 ? (cur.sc >> 8) & 0xFF : cur.sc & 0xFF];
          v[k] = __fmul_rn(__fmul_rn(__uint_as_float(e2m1_scaled_bits_at(cur.codes, 4 * k)),
                                     0x1p126f),
                           D);  // exact
        }
        if (cur.nv == 8 && vec) {
          if (y_bf16) {
            *reinterpret_cast<uint4*>(static_cast<uint16_t*>(y) + y0 + j0) =
                make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                           pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
          } else {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(y) + y0 + j0);
            dst[0] = make_float4(v[0], v[1], v[2], v[3]);
            dst[1] = make_float4(v[4], v[5], v[6], v[7]);
          }
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            if (k < cur.nv) store_y(y, y0 + j0 + k, v[k], y_bf16);
        }
      }
      cur = nxt;
    }
  }
}

constexpr int kMaxRaggedGrid = kMaxReduceCtas - 2 * kMaxGroup;  // partials after the header

template <typename T, int FMT, int N>
cudaError_t launch_rows(const RaggedArgs& args, int64_t nblocks, void* out, cudaStream_t stream,
                        int* launches) {
  // one warp per row: rows / 8 CTAs, at most the resident CTAs (and the partial slots)
  const int grid = persistent_grid((const void*)k_ragged_rows<T, FMT, N>, args.rows * 32, 1,
                                   kMaxRaggedGrid);
  k_ragged_rows<T, FMT, N><<<grid, kThreads, 0, stream>>>(args);
  ++*launches;
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess && args.part)
    e = launch_stats_final(args.part, grid, args.rows * args.cols, nblocks, out, stream, launches);
  return e;
}

template <typename T, int FMT>
cudaError_t launch_ragged(const RaggedArgs& args, int64_t nblocks, void* out, cudaStream_t stream,
                          int* launches) {
  switch (args.N) {
    case 4: return launch_rows<T, FMT, 4>(args, nblocks, out, stream, launches);
    case 8: return launch_rows<T, FMT, 8>(args, nblocks, out, stream, launches);
    case 16: return launch_rows<T, FMT, 16>(args, nblocks, out, stream, launches);
    case 32: return launch_rows<T, FMT, 32>(args, nblocks, out, stream, launches);
    case 64: return launch_rows<T, FMT, 64>(args, nblocks, out, stream, launches);
    case 128: return launch_rows<T, FMT, 128>(args, nblocks, out, stream, launches);
    default: return launch_rows<T, FMT, 256>(args, nblocks, out, stream, launches);
  }
}

template <int FMT, int LOGN>
cudaError_t launch_dq(const uint8_t* packed, const uint8_t* scales, int64_t rows, int64_t cols,
                      uint16_t g_bits, const uint16_t* g_dev, void* y, bool y_bf16,
                      cudaStream_t stream) {
  const int grid = persistent_grid((const void*)k_ragged_dequantize<FMT, LOGN>, rows * 32, 1);
  k_ragged_dequantize<FMT, LOGN><<<grid, kThreads, 0, stream>>>(packed, scales, rows, cols,
                                                                 g_bits, g_dev, y, y_bf16 ? 1 : 0);
  return cudaGetLastError();
}

template <int FMT>
cudaError_t launch_dq_fmt(const uint8_t* packed, const uint8_t* scales, int64_t rows,
                          int64_t cols, int block, uint16_t g_bits, const uint16_t* g_dev,
                          void* y, bool y_bf16, cudaStream_t stream) {
  switch (block) {
    case 4: return launch_dq<FMT, 2>(packed, scales, rows, cols, g_bits, g_dev, y, y_bf16,
                                             stream);
    case 8: return launch_dq<FMT, 3>(packed, scales, rows, cols, g_bits, g_dev, y, y_bf16,
                                             stream);
    case 16: return launch_dq<FMT, 4>(packed, scales, rows, cols, g_bits, g_dev, y, y_bf16,
                                             stream);
    case 32: return launch_dq<FMT, 5>(packed, scales, rows, cols, g_bits, g_dev, y, y_bf16,
                                             stream);
    case 64: return launch_dq<FMT, 6>(packed, scales, rows, cols, g_bits, g_dev, y, y_bf16,
                                             stream);
    case 128: return launch_dq<FMT, 7>(packed, scales, rows, cols, g_bits, g_dev, y, y_bf16,
                                             stream);
    default: return launch_dq<FMT, 8>(packed, scales, rows, cols, g_bits, g_dev, y, y_bf16, stream);
  }
}

}  // namespace

cudaError_t run_ragged(const void* x, bool bf16, int64_t rows, int64_t cols, int block, int fmt,
                       uint16_t g_bits, const uint16_t* g_dev, const uint8_t* packed_in,
                       const uint8_t* scales_in,
                       uint8_t* packed, uint8_t* scales, void* y, bool y_bf16, void* out,
                       void* workspace, cudaStream_t stream, int* launches) {
  if (cols > (int64_t(1) << 30)) return cudaErrorInvalidValue;  // in-row indices are 32-bit
  // bf16 rows on 16-byte boundaries with recomputed codes: the row-pitched whole-block kernels
  if (!packed_in && out && !y && rows_stats_supported(bf16, rows, cols, block))
    return run_rows_stats(x, rows, cols, block, fmt, g_bits, g_dev, packed, scales, out, workspace,
                          stream, launches);
  if (!packed_in && !out && rows_quantize_supported(bf16, rows, cols, block))
    return run_rows_quantize(x, rows, cols, block, fmt, g_bits, g_dev, packed, scales, y, y_bf16,
                             stream, launches);
  RaggedArgs args{x, rows, cols, block, g_bits, g_dev, packed_in, scales_in, packed, scales, y,
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
                                  int64_t cols, int block, int fmt, uint16_t g_bits,
                                  const uint16_t* g_dev, void* y,
                                  bool y_bf16, cudaStream_t stream, int* launches) {
  if (tile_dequantize_supported(y_bf16, rows, cols, block))
    return run_tile_dequantize(packed, scales, rows, cols, block, fmt, g_bits, g_dev, y, stream,
                               launches);
  ++*launches;
  return fmt == kUE5M3
             ? launch_dq_fmt<kUE5M3>(packed, scales, rows, cols, block, g_bits, g_dev, y, y_bf16,
                                     stream)
             : launch_dq_fmt<kE4M3>(packed, scales, rows, cols, block, g_bits, g_dev, y, y_bf16,
                                    stream);
}

}  // namespace mxk
