// mx_quantize.cu -- quantize + pack kernel (sm_100a).
//
// Method: the microscaling article (hotelren.com/news/2192771) §3.1 item 2, quantize_block:
//   abs_max = max|block|; scale = Q_fp8(abs_max / 6); q = Q_fp4(block / scale)
// with the FP16 per-tensor factor g of §3.1 item 3 (abs_max / (6 g), block / (scale g)), and two
// FP4 codes per byte (4-bit float article, gtnt.cn/news/16247, §4.3).
//
// Layout: the tensor is contiguous row-major and cols % N == 0, so blocks never straddle rows and
// the whole tensor is one flat run of blocks.  A thread owns EPT consecutive elements (an "item"):
// EPT = 16 bf16 (32 bytes, two 16-byte loads) when N >= 16 so a block spans N/16 lanes of a warp
// and its absmax is finished with warp shuffles; EPT = 8 for N in {4, 8} (one or two blocks per
// item, no shuffles).  fp32 input uses EPT = 8.  Every CTA first builds a 256-entry table of
// per-scale-code constants in shared memory (1/(S g) for bf16, S g for fp32), so the per-block work
// is: absmax, one multiply + snap + FP8 encode, one shared-memory lookup.  The grid is persistent
// (a multiple of the SM count) and walks the items with a grid stride, two items per thread in
// flight.  No kernel here waits on another CTA.
//
// Rows whose length the block size does not divide (cols % N != 0, bf16, cols % 8 == 0) use the
// same kernel in its row-pitched mode (ROWS): each row's blocks rounded up to whole items, a
// RowCursor turning the item index into (row, item), the chunks past a row's end neither read nor
// written.
#include "mx_device.cuh"
#include "mx_launch.h"

namespace mxk {

// Item shape (compile-time; the defaults are the tuned values): elements per item for bf16 input
// when N >= 16 (8 or 16), and items in flight per thread.
#ifndef MX_Q_EPT_BF16
#define MX_Q_EPT_BF16 16
#endif
#ifndef MX_Q_U
#define MX_Q_U 2
#endif

template <int N, typename T>
struct QShape {
  static constexpr int EPT = (sizeof(T) == 2 && N >= 16) ? MX_Q_EPT_BF16 : 8;  // elements per item
  static constexpr int L = (N >= EPT) ? N / EPT : 1;                          // lanes per block
  static constexpr int BPI = (N >= EPT) ? 1 : EPT / N;                        // blocks per item
  static constexpr int U = (sizeof(T) == 2) ? MX_Q_U : 2;                    // items in flight
};

// Kernel parameters: up to kMaxGroup tensors and the split of the grid among them.  A CTA works
// on one tensor with a grid stride of its own range of CTAs.
struct QTensor {
  const void* x;
  uint8_t* packed;
  uint8_t* scales;
  void* y;  // round trip (OUT != kCodes): the dequantized output instead of codes and scales
  int64_t nitems;
  uint32_t g_bits;
  const uint16_t* g_dev;  // g in device memory (written by the previous kernel) when set
  // Row-pitched mode (rows whose length cols the block size does not divide): ipr items per row,
  // the row's blocks rounded up to whole items (the last ones hold zeros past the row's end);
  // row pitches of x / y (cols elements), codes (pb bytes) and scales (nb bytes).
  int64_t cols, ipr, pb, nb;
};

// What a quantize kernel writes: codes and scales, or (the fake-quantize round trip) the
// dequantized value E2M1(code) * S * g of every element, as bf16 (round to nearest even of the
// exact product) or fp32 (exact).
enum QOut { kCodes = 0, kRoundTripBf16 = 1, kRoundTripF32 = 2 };

// Round trip: the 8 codes of each code word times the scale of its block, stored to y at item i.
template <int EPT, int BPI, int OUT>
__device__ __forceinline__ void store_round_trip(void* y, int64_t i, const uint32_t* codes,
                                                 uint32_t sc, const float* s_D) {
  constexpr int BE = EPT / BPI;
  float out[EPT];
#pragma unroll
  for (int b = 0; b < BPI; ++b) {
    const float D = s_D[(sc >> (8 * b)) & 0xFF];
#pragma unroll
    for (int k = 0; k < BE; ++k) {
      const int e = b * BE + k;  // nibble e % 8 of code word e / 8
      const float f = __uint_as_float(e2m1_scaled_bits_at(codes[e / 8], 4 * (e % 8)));
      out[e] = __fmul_rn(__fmul_rn(f, 0x1p126f), D);  // exact
    }
  }
  if constexpr (OUT == kRoundTripBf16) {
    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(y) + i * EPT);
#pragma unroll
    for (int h = 0; h < EPT / 8; ++h)
      __stcs(dst + h, make_uint4(pack_bf16x2(out[8 * h], out[8 * h + 1]),
                                 pack_bf16x2(out[8 * h + 2], out[8 * h + 3]),
                                 pack_bf16x2(out[8 * h + 4], out[8 * h + 5]),
                                 pack_bf16x2(out[8 * h + 6], out[8 * h + 7])));
  } else {
    float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(y) + i * EPT);
#pragma unroll
    for (int h = 0; h < EPT / 4; ++h)
      __stcs(dst + h, make_float4(out[4 * h], out[4 * h + 1], out[4 * h + 2], out[4 * h + 3]));
  }
}
struct QGroup {
  QTensor t[kMaxGroup];
  CtaSplit split;
};

// This CTA's tensor, its index among the tensor's CTAs and their number.
struct QWork {
  QTensor t;
  int cta, nctas;
};
__device__ __forceinline__ QWork q_work(const QGroup& grp) {
  const int ti = grp.split.find((int)blockIdx.x);
  return {grp.t[ti], (int)blockIdx.x - grp.split.begin[ti],
          grp.split.begin[ti + 1] - grp.split.begin[ti]};
}

// ------------------------------------------------------------------------------------------------
// bf16 input
// ------------------------------------------------------------------------------------------------

// Absmax (as non-negative bf16 bits) of words w[k0 .. k0+nw).
template <int NW>
__device__ __forceinline__ uint32_t absmax_bits(const uint32_t* w) {
  uint32_t t = w[0];
#pragma unroll
  for (int k = 1; k < NW; ++k) t = bf16x2_absmax(t, w[k]);
  if (NW == 1) t = bf16x2_absmax(t, t);
  t &= 0x7FFF7FFFu;
  return max(t & 0xFFFFu, t >> 16);
}

// ROWS: the row-pitched mode (QTensor) for rows of cols % 8 == 0 elements that the block size does
// not divide: item i of the padded item space is item j of row i / ipr (a RowCursor per item in
// flight, no division per item); x and the round trip at row * cols + j * EPT (16-byte aligned),
// codes at row * pb + j * EPT / 2 as 4-byte words, scales at row * nb; an item's 8-element chunks
// past the row's end are neither read (zeros: they do not change the block maximum) nor written.
template <int N, int FMT, int OUT = kCodes, bool ROWS = false>
__global__ void __launch_bounds__(kThreads) k_quantize_bf16(const __grid_constant__ QGroup grp) {
  using S = QShape<N, uint16_t>;
  constexpr int EPT = S::EPT, L = S::L, BPI = S::BPI, U = S::U, NW = EPT / 2;
  static_assert(!ROWS || (N >= 16 && BPI == 1), "row-pitched mode: blocks of 16 and more");
  const QWork wk = q_work(grp);
  const uint16_t* __restrict__ x = static_cast<const uint16_t*>(wk.t.x);
  uint8_t* __restrict__ packed = wk.t.packed;
  uint8_t* __restrict__ scales = wk.t.scales;
  const int64_t nitems = wk.t.nitems;
  __shared__ float s_rcp[256];
  __shared__ float s_D[OUT == kCodes ? 1 : 256];
  const float g = fp16_bits_to_float(tensor_g_bits(wk.t.g_bits, wk.t.g_dev));
  for (int c = threadIdx.x; c < 256; c += blockDim.x) {
    const float D = __fmul_rn(scale_value(c, FMT), g);  // exact (<= 15 significant bits)
    s_rcp[c] = D > 0.0f ? __frcp_rn(D) : 0.0f;          // zero scale -> every code is +-0
    if constexpr (OUT != kCodes) s_D[c] = D;
  }
  const float r6 = __frcp_rn(__fmul_rn(6.0f, g));
  __syncthreads();
  griddep_wait();  // inputs may come from the previous kernel in the stream
  griddep_launch_next();

  const int64_t T = (int64_t)wk.nctas * blockDim.x;
  const int64_t tid = (int64_t)wk.cta * blockDim.x + threadIdx.x;
  const int64_t warp0 = tid - (threadIdx.x & 31);
  const int lane = threadIdx.x & 31;
  RowCursor rc[U];  // ROWS: row and item of each item in flight
  if constexpr (ROWS) {
#pragma unroll
    for (int u = 0; u < U; ++u) rc[u].init(tid + (int64_t)u * T, T * U, wk.t.ipr);
  }

  for (int64_t base = 0; warp0 + base < nitems; base += T * U) {
    uint32_t w[U][NW];
    bool ok[U];
    int nval[U];      // ROWS: elements of the item inside its row (a multiple of 8; <= 0: none)
    int64_t off[U];   // ROWS: the item's first element in x
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = tid + base + (int64_t)u * T;
      ok[u] = i < nitems;
      if constexpr (ROWS) {
        nval[u] = (int)min((int64_t)EPT, wk.t.cols - rc[u].j * EPT);
        off[u] = rc[u].row * wk.t.cols + rc[u].j * EPT;
        ok[u] = ok[u] && nval[u] > 0;
      }
#pragma unroll
      for (int h = 0; h < NW / 4; ++h) {
        uint4 v = make_uint4(0, 0, 0, 0);
        if constexpr (ROWS) {
          if (ok[u] && 8 * h < nval[u]) v = ld_stream16(x + off[u] + h * 8);
        } else {
          if (ok[u]) v = ld_stream16(x + i * EPT + h * 8);
        }
        w[u][4 * h + 0] = v.x;
        w[u][4 * h + 1] = v.y;
        w[u][4 * h + 2] = v.z;
        w[u][4 * h + 3] = v.w;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = tid + base + (int64_t)u * T;
      float qv[EPT];
      uint32_t sc = 0;
#pragma unroll
      for (int b = 0; b < BPI; ++b) {
        constexpr int BW = NW / BPI;  // words per block inside this item
        uint32_t m = absmax_bits<BW>(&w[u][b * BW]);
#pragma unroll
        for (int off = 1; off < L; off <<= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
        const float a = __uint_as_float(m << 16);
        const uint32_t s = encode_scale<FMT>(snap21(__fmul_rn(a, r6)));
        const float r = s_rcp[s];
        sc |= s << (8 * b);
#pragma unroll
        for (int k = 0; k < BW; ++k) {
          const uint32_t wk = w[u][b * BW + k];
          const float2 q = snap_quotient2(wk << 16, wk & 0xFFFF0000u, r);
          qv[2 * (b * BW + k)] = q.x;
          qv[2 * (b * BW + k) + 1] = q.y;
        }
      }
      uint32_t codes[EPT / 8];
#pragma unroll
      for (int j = 0; j < EPT / 8; ++j)
        codes[j] = cvt_e2m1x8(qv[8 * j], qv[8 * j + 1], qv[8 * j + 2], qv[8 * j + 3], qv[8 * j + 4],
                              qv[8 * j + 5], qv[8 * j + 6], qv[8 * j + 7]);
      if (!ok[u]) continue;
      if constexpr (ROWS) {
        const int64_t row = rc[u].row, j = rc[u].j;
        if constexpr (OUT != kCodes) {
          const float D = s_D[sc & 0xFF];
#pragma unroll
          for (int h = 0; h < EPT / 8; ++h) {
            if (8 * h >= nval[u]) continue;
            float out[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              out[e] = __fmul_rn(__fmul_rn(__uint_as_float(e2m1_scaled_bits_at(codes[h], 4 * e)),
                                           0x1p126f),
                                 D);  // exact
            if constexpr (OUT == kRoundTripBf16) {
              __stcs(reinterpret_cast<uint4*>(static_cast<uint16_t*>(wk.t.y) + off[u] + 8 * h),
                     make_uint4(pack_bf16x2(out[0], out[1]), pack_bf16x2(out[2], out[3]),
                                pack_bf16x2(out[4], out[5]), pack_bf16x2(out[6], out[7])));
            } else {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(wk.t.y) + off[u] + 8 * h);
              __stcs(dst, make_float4(out[0], out[1], out[2], out[3]));
              __stcs(dst + 1, make_float4(out[4], out[5], out[6], out[7]));
            }
          }
        } else {
          uint8_t* prow = packed + row * wk.t.pb + j * (EPT / 2);
#pragma unroll
          for (int h = 0; h < EPT / 8; ++h)
            if (8 * h < nval[u]) *reinterpret_cast<uint32_t*>(prow + 4 * h) = codes[h];
          if ((lane & (L - 1)) == 0) scales[row * wk.t.nb + (j * EPT) / N] = (uint8_t)sc;
        }
        continue;
      }
      if constexpr (OUT != kCodes) {
        store_round_trip<EPT, BPI, OUT>(wk.t.y, i, codes, sc, s_D);
        continue;
      }
      if constexpr (NW == 8) {
        *reinterpret_cast<uint2*>(packed + i * 8) = make_uint2(codes[0], codes[1]);
      } else {
        *reinterpret_cast<uint32_t*>(packed + i * 4) = codes[0];
      }
      if constexpr (BPI == 1) {
        if ((lane & (L - 1)) == 0) scales[i / L] = (uint8_t)sc;
      } else {
        *reinterpret_cast<uint16_t*>(scales + i * 2) = (uint16_t)sc;
      }
    }
    if constexpr (ROWS) {
#pragma unroll
      for (int u = 0; u < U; ++u) rc[u].advance();
    }
  }
}

// ------------------------------------------------------------------------------------------------
// fp32 input: IEEE division (see mx_device.cuh for why the multiply shortcut is not used here)
// ------------------------------------------------------------------------------------------------

template <int N, int FMT, int OUT = kCodes>
__global__ void __launch_bounds__(kThreads) k_quantize_f32(const __grid_constant__ QGroup grp) {
  using S = QShape<N, float>;
  constexpr int EPT = S::EPT, L = S::L, BPI = S::BPI, U = S::U;
  const QWork wk = q_work(grp);
  const float* __restrict__ x = static_cast<const float*>(wk.t.x);
  uint8_t* __restrict__ packed = wk.t.packed;
  uint8_t* __restrict__ scales = wk.t.scales;
  const int64_t nitems = wk.t.nitems;
  __shared__ float s_D[256];
  const float g = fp16_bits_to_float(tensor_g_bits(wk.t.g_bits, wk.t.g_dev));
  for (int c = threadIdx.x; c < 256; c += blockDim.x) s_D[c] = __fmul_rn(scale_value(c, FMT), g);
  const float g6 = __fmul_rn(6.0f, g);
  __syncthreads();
  griddep_wait();  // inputs may come from the previous kernel in the stream
  griddep_launch_next();

  const int64_t T = (int64_t)wk.nctas * blockDim.x;
  const int64_t tid = (int64_t)wk.cta * blockDim.x + threadIdx.x;
  const int64_t warp0 = tid - (threadIdx.x & 31);
  const int lane = threadIdx.x & 31;

  for (int64_t base = 0; warp0 + base < nitems; base += T * U) {
    float v[U][EPT];
    bool ok[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = tid + base + (int64_t)u * T;
      ok[u] = i < nitems;
#pragma unroll
      for (int h = 0; h < EPT / 4; ++h) {
        uint4 t = make_uint4(0, 0, 0, 0);
        if (ok[u]) t = ld_stream16(x + i * EPT + h * 4);
        v[u][4 * h + 0] = __uint_as_float(t.x);
        v[u][4 * h + 1] = __uint_as_float(t.y);
        v[u][4 * h + 2] = __uint_as_float(t.z);
        v[u][4 * h + 3] = __uint_as_float(t.w);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = tid + base + (int64_t)u * T;
      float q[EPT];
      uint32_t sc = 0;
#pragma unroll
      for (int b = 0; b < BPI; ++b) {
        constexpr int BE = EPT / BPI;  // elements per block inside this item
        float a = 0.0f;
#pragma unroll
        for (int k = 0; k < BE; ++k) a = fmaxf(a, fabsf(v[u][b * BE + k]));
#pragma unroll
        for (int off = 1; off < L; off <<= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
        const uint32_t s = encode_scale<FMT>(__fdiv_rn(a, g6));
        const float D = s_D[s];
        sc |= s << (8 * b);
#pragma unroll
        for (int k = 0; k < BE; ++k) {
          const float xv = v[u][b * BE + k];
          q[b * BE + k] = D > 0.0f ? __fdiv_rn(xv, D) : __fmul_rn(xv, 0.0f);
        }
      }
      if (!ok[u]) continue;
      const uint32_t code = cvt_e2m1x8(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]);
      if constexpr (OUT != kCodes) {
        store_round_trip<EPT, BPI, OUT>(wk.t.y, i, &code, sc, s_D);
        continue;
      }
      *reinterpret_cast<uint32_t*>(packed + i * 4) = code;
      if constexpr (BPI == 1) {
        if ((lane & (L - 1)) == 0) scales[i / L] = (uint8_t)sc;
      } else {
        *reinterpret_cast<uint16_t*>(scales + i * 2) = (uint16_t)sc;
      }
    }
  }
}

// ------------------------------------------------------------------------------------------------
// tail: the elements after the last whole item (a multiple of N <= 8, fewer than an item).  One
// thread finishes them block by block with plain per-element code (IEEE division).
// ------------------------------------------------------------------------------------------------

template <int FMT, typename T, int OUT = kCodes>
__global__ void k_quantize_tail(const T* __restrict__ x, int64_t first, int count, int N,
                                uint16_t g_bits, const uint16_t* g_dev,
                                uint8_t* __restrict__ packed, uint8_t* __restrict__ scales,
                                void* __restrict__ y = nullptr) {
  if (threadIdx.x != 0) return;
  const float g = fp16_bits_to_float(tensor_g_bits(g_bits, g_dev));
  for (int b0 = 0; b0 < count; b0 += N) {
    const int64_t f = first + b0;
    float v[16], a = 0.0f;  // N <= 16
    for (int k = 0; k < N; ++k) {
      if constexpr (sizeof(T) == 2)
        v[k] = __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(x)[f + k] << 16);
      else
        v[k] = reinterpret_cast<const float*>(x)[f + k];
      a = fmaxf(a, fabsf(v[k]));
    }
    const uint32_t s = encode_scale<FMT>(__fdiv_rn(a, __fmul_rn(6.0f, g)));
    const float D = __fmul_rn(scale_value((int)s, FMT), g);
    for (int k0 = 0; k0 < N; k0 += 2) {  // one byte (two codes) at a time
      float q[2];
      for (int k = 0; k < 2; ++k)
        q[k] = D > 0.0f ? __fdiv_rn(v[k0 + k], D) : __fmul_rn(v[k0 + k], 0.0f);
      const uint32_t c = cvt_e2m1x8(q[0], q[1], 0.f, 0.f, 0.f, 0.f, 0.f, 0.f) & 0xFF;
      if constexpr (OUT != kCodes) {
        for (int k = 0; k < 2; ++k) {
          const float yv = __fmul_rn(e2m1_to_float(c >> (4 * k)), D);  // exact
          if constexpr (OUT == kRoundTripBf16)
            reinterpret_cast<__nv_bfloat16*>(y)[f + k0 + k] = __float2bfloat16_rn(yv);
          else
            reinterpret_cast<float*>(y)[f + k0 + k] = yv;
        }
      } else {
        packed[(f + k0) / 2] = (uint8_t)c;
      }
    }
    if constexpr (OUT == kCodes) scales[f / N] = (uint8_t)s;
  }
}

// ------------------------------------------------------------------------------------------------
// launcher
// ------------------------------------------------------------------------------------------------

template <int N, int FMT, typename T, int OUT>
static cudaError_t launch_q(const TensorArgs* ta, int count, cudaStream_t stream, int* launches) {
  using S = QShape<N, T>;
  QGroup grp = {};
  int64_t nitems[kMaxGroup];
  for (int k = 0; k < count; ++k) {
    nitems[k] = ta[k].numel / S::EPT;
    grp.t[k] = {ta[k].x, ta[k].packed, ta[k].scales, ta[k].y, nitems[k], ta[k].g_bits,
                ta[k].g_dev};
  }
  auto kern = (sizeof(T) == 2) ? (void*)k_quantize_bf16<N, FMT, OUT>
                               : (void*)k_quantize_f32<N, FMT, OUT>;
  const int grid = split_grid(kern, nitems, count, S::U, 1 << 30, &grp.split);
  if (grid > 0) {
    const cudaError_t e =
        (sizeof(T) == 2) ? launch_pdl(k_quantize_bf16<N, FMT, OUT>, grid, kThreads, stream, grp)
                         : launch_pdl(k_quantize_f32<N, FMT, OUT>, grid, kThreads, stream, grp);
    if (e != cudaSuccess) return e;
    ++*launches;
  }
  for (int k = 0; k < count; ++k) {
    if (ta[k].numel % S::EPT != 0) {  // only N = 4 leaves a remainder (of exactly 4 elements)
      k_quantize_tail<FMT, T, OUT><<<1, 32, 0, stream>>>(
          (const T*)ta[k].x, nitems[k] * S::EPT, (int)(ta[k].numel % S::EPT), N, ta[k].g_bits,
          ta[k].g_dev, ta[k].packed, ta[k].scales, ta[k].y);
      ++*launches;
    }
  }
  return cudaGetLastError();
}

template <int FMT, typename T, int OUT>
static cudaError_t dispatch_block(int block, const TensorArgs* t, int count, cudaStream_t st,
                                  int* n) {
  switch (block) {
    case 4: return launch_q<4, FMT, T, OUT>(t, count, st, n);
    case 8: return launch_q<8, FMT, T, OUT>(t, count, st, n);
    case 16: return launch_q<16, FMT, T, OUT>(t, count, st, n);
    case 32: return launch_q<32, FMT, T, OUT>(t, count, st, n);
    case 64: return launch_q<64, FMT, T, OUT>(t, count, st, n);
    case 128: return launch_q<128, FMT, T, OUT>(t, count, st, n);
    default: return launch_q<256, FMT, T, OUT>(t, count, st, n);
  }
}

// Row-pitched mode of k_quantize_bf16 (rows whose length the block size N >= 16 does not divide,
// cols % 8 == 0): one tensor per launch.
template <int N, int FMT, int OUT>
static cudaError_t launch_q_rows(const void* x, int64_t rows, int64_t cols, uint16_t g_bits,
                                 const uint16_t* g_dev, uint8_t* packed, uint8_t* scales, void* y,
                                 cudaStream_t stream, int* launches) {
  using S = QShape<N, uint16_t>;
  static_assert(N >= S::EPT, "whole items per block");
  const int64_t nb = (cols + N - 1) / N, ipr = nb * (N / S::EPT);
  const int64_t nitems = rows * ipr;
  QGroup grp = {};
  grp.t[0] = {x, packed, scales, y, nitems, g_bits, g_dev, cols, ipr, (cols + 1) / 2, nb};
  const int grid = split_grid((const void*)k_quantize_bf16<N, FMT, OUT, true>, &nitems, 1, S::U,
                              1 << 30, &grp.split);
  if (grid == 0) return cudaSuccess;
  const cudaError_t e = launch_pdl(k_quantize_bf16<N, FMT, OUT, true>, grid, kThreads, stream, grp);
  if (e == cudaSuccess) ++*launches;
  return e;
}

template <int FMT, int OUT>
static cudaError_t q_rows_block(int block, const void* x, int64_t rows, int64_t cols,
                                uint16_t g_bits, const uint16_t* g_dev, uint8_t* packed,
                                uint8_t* scales, void* y, cudaStream_t st, int* n) {
  switch (block) {
    case 16: return launch_q_rows<16, FMT, OUT>(x, rows, cols, g_bits, g_dev, packed, scales, y, st, n);
    case 32: return launch_q_rows<32, FMT, OUT>(x, rows, cols, g_bits, g_dev, packed, scales, y, st, n);
    case 64: return launch_q_rows<64, FMT, OUT>(x, rows, cols, g_bits, g_dev, packed, scales, y, st, n);
    case 128: return launch_q_rows<128, FMT, OUT>(x, rows, cols, g_bits, g_dev, packed, scales, y, st, n);
    default: return launch_q_rows<256, FMT, OUT>(x, rows, cols, g_bits, g_dev, packed, scales, y, st, n);
  }
}

template <int OUT>
static cudaError_t q_rows_fmt(int fmt, int block, const void* x, int64_t rows, int64_t cols,
                              uint16_t g_bits, const uint16_t* g_dev, uint8_t* packed,
                              uint8_t* scales, void* y, cudaStream_t st, int* n) {
  return fmt == kUE5M3
             ? q_rows_block<kUE5M3, OUT>(block, x, rows, cols, g_bits, g_dev, packed, scales, y, st, n)
             : q_rows_block<kE4M3, OUT>(block, x, rows, cols, g_bits, g_dev, packed, scales, y, st, n);
}

bool rows_quantize_supported(bool bf16, int64_t rows, int64_t cols, int block) {
  return bf16 && block >= 16 && cols % 8 == 0 && rows >= 1;
}

cudaError_t run_rows_quantize(const void* x, int64_t rows, int64_t cols, int block, int fmt,
                              uint16_t g_bits, const uint16_t* g_dev, uint8_t* packed,
                              uint8_t* scales, void* y, bool y_bf16, cudaStream_t stream,
                              int* launches) {
  if (!y)
    return q_rows_fmt<kCodes>(fmt, block, x, rows, cols, g_bits, g_dev, packed, scales, nullptr,
                              stream, launches);
  return y_bf16 ? q_rows_fmt<kRoundTripBf16>(fmt, block, x, rows, cols, g_bits, g_dev, nullptr,
                                             nullptr, y, stream, launches)
                : q_rows_fmt<kRoundTripF32>(fmt, block, x, rows, cols, g_bits, g_dev, nullptr,
                                            nullptr, y, stream, launches);
}

cudaError_t run_quantize_tail(const void* x, bool bf16, int64_t first, int count, int N, int fmt,
                              uint16_t g_bits, const uint16_t* g_dev, uint8_t* packed,
                              uint8_t* scales, cudaStream_t stream, int* launches) {
  if (bf16) {
    if (fmt == kUE5M3)
      k_quantize_tail<kUE5M3, uint16_t><<<1, 32, 0, stream>>>((const uint16_t*)x, first, count, N,
                                                              g_bits, g_dev, packed, scales);
    else
      k_quantize_tail<kE4M3, uint16_t><<<1, 32, 0, stream>>>((const uint16_t*)x, first, count, N,
                                                             g_bits, g_dev, packed, scales);
  } else {
    if (fmt == kUE5M3)
      k_quantize_tail<kUE5M3, float><<<1, 32, 0, stream>>>((const float*)x, first, count, N,
                                                           g_bits, g_dev, packed, scales);
    else
      k_quantize_tail<kE4M3, float><<<1, 32, 0, stream>>>((const float*)x, first, count, N,
                                                          g_bits, g_dev, packed, scales);
  }
  ++*launches;
  return cudaGetLastError();
}

template <int OUT>
static cudaError_t quantize_out(const TensorArgs* t, int count, bool bf16, int block, int fmt,
                                cudaStream_t stream, int* launches) {
  if (bf16)
    return fmt == kUE5M3
               ? dispatch_block<kUE5M3, uint16_t, OUT>(block, t, count, stream, launches)
               : dispatch_block<kE4M3, uint16_t, OUT>(block, t, count, stream, launches);
  return fmt == kUE5M3 ? dispatch_block<kUE5M3, float, OUT>(block, t, count, stream, launches)
                       : dispatch_block<kE4M3, float, OUT>(block, t, count, stream, launches);
}

cudaError_t run_quantize_group(const TensorArgs* t, int count, bool bf16, int block, int fmt,
                               cudaStream_t stream, int* launches) {
  return quantize_out<kCodes>(t, count, bf16, block, fmt, stream, launches);
}

cudaError_t run_fake_quantize(const void* x, bool bf16, int64_t numel, int block, int fmt,
                              uint16_t g_bits, void* y, bool ybf16, cudaStream_t stream,
                              int* launches) {
  const TensorArgs t = {x, y, nullptr, nullptr, nullptr, numel, g_bits};
  return ybf16 ? quantize_out<kRoundTripBf16>(&t, 1, bf16, block, fmt, stream, launches)
               : quantize_out<kRoundTripF32>(&t, 1, bf16, block, fmt, stream, launches);
}

cudaError_t run_quantize(const void* x, bool bf16, int64_t numel, int block, int fmt,
                         uint16_t g_bits, uint8_t* packed, uint8_t* scales, cudaStream_t stream,
                         int* launches) {
  const TensorArgs t = {x, nullptr, packed, scales, nullptr, numel, g_bits};
  return run_quantize_group(&t, 1, bf16, block, fmt, stream, launches);
}

}  // namespace mxk
