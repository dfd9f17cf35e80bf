// mx_dequantize.cu -- dequantize kernel (sm_100a).
//
// Method: the microscaling article (hotelren.com/news/2192771) §1 and §3.1 item 3: the stored value
// is FP4 x FP8_scale x FP16_scale.  The product of an E2M1 value (<= 2 significant bits), an FP8
// scale (<= 4) and the FP16 g (<= 11) has at most 17 significant bits and stays inside the fp32
// normal range, so y = e2m1 * (S g) is exact in fp32; bf16 output is its round-to-nearest-even.
//
// Layout mirrors the quantize kernel: a thread owns EPT consecutive codes (16 for bf16 output with
// N >= 16, else 8), reads EPT/2 packed bytes and the scale byte(s) of its block(s), decodes the
// codes, multiplies by the per-code constant S g from a
// shared-memory table and writes 16-byte vectors.  Codes are decoded with exact bit arithmetic
// (e2m1_scaled_bits_at), not with a conversion instruction.
#include <cuda_fp16.h>

#include "mx_device.cuh"
#include "mx_launch.h"

namespace mxk {

// Item shape (compile-time; the defaults are the tuned values).
#ifndef MX_DQ_EPT_BF16
#define MX_DQ_EPT_BF16 8
#endif
#ifndef MX_DQ_U
#define MX_DQ_U 2
#endif

#ifndef MX_DQ_HWDEC
#define MX_DQ_HWDEC 1
#endif

// The eight codes of a loaded word w (code k in nibble k) decoded to f16x2 values h[0..3] (word k:
// codes 2k, 2k+1) by the E2M1x2 -> f16x2 conversion; exact (E2M1 values are f16 values).  The word
// comes from memory and is split into its bytes inside the same asm block.
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t* h) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(w));
}

template <int N, bool BF16OUT>
struct DShape {
  static constexpr int EPT = (BF16OUT && N >= 16) ? MX_DQ_EPT_BF16 : 8;
  static constexpr int L = (N >= EPT) ? N / EPT : 1;
  static constexpr int BPI = (N >= EPT) ? 1 : EPT / N;
  static constexpr int U = MX_DQ_U;
};

// Kernel parameters: up to kMaxGroup tensors and the split of the grid among them.
struct DTensor {
  const uint8_t* packed;
  const uint8_t* scales;
  void* y;
  int64_t nitems;
  uint32_t g_bits;
  const uint16_t* g_dev;  // g in device memory (written by the previous kernel) when set
};
struct DGroup {
  DTensor t[kMaxGroup];
  CtaSplit split;
};

template <int N, int FMT, bool BF16OUT>
__global__ void __launch_bounds__(kThreads) k_dequantize(const __grid_constant__ DGroup grp) {
  using S = DShape<N, BF16OUT>;
  constexpr int EPT = S::EPT, L = S::L, BPI = S::BPI, U = S::U;
  const int ti = grp.split.find((int)blockIdx.x);
  const DTensor tt = grp.t[ti];
  const int cta = (int)blockIdx.x - grp.split.begin[ti];
  const int nctas = grp.split.begin[ti + 1] - grp.split.begin[ti];
  const uint8_t* __restrict__ packed = tt.packed;
  const uint8_t* __restrict__ scales = tt.scales;
  void* __restrict__ y = tt.y;
  const int64_t nitems = tt.nitems;
  __shared__ float s_D[256];
  const float g = fp16_bits_to_float(tensor_g_bits(tt.g_bits, tt.g_dev));
  for (int c = threadIdx.x; c < 256; c += blockDim.x) s_D[c] = __fmul_rn(scale_value(c, FMT), g);
  __syncthreads();
  griddep_wait();  // inputs may come from the previous kernel in the stream
  griddep_launch_next();

  const int64_t T = (int64_t)nctas * blockDim.x;
  const int64_t tid = (int64_t)cta * blockDim.x + threadIdx.x;
  for (int64_t base = tid; base < nitems; base += T * U) {
    uint32_t cw[U][EPT / 8];
    uint32_t sc[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = base + (int64_t)u * T;
      cw[u][0] = 0;
      if (EPT == 16) cw[u][EPT / 8 - 1] = 0;
      sc[u] = 0;
      if (i < nitems) {
        if constexpr (EPT == 16) {
          const uint2 p = __ldcs(reinterpret_cast<const uint2*>(packed) + i);
          cw[u][0] = p.x;
          cw[u][EPT / 8 - 1] = p.y;
        } else {
          cw[u][0] = __ldcs(reinterpret_cast<const unsigned int*>(packed) + i);
        }
        if constexpr (BPI == 1)
          sc[u] = __ldg(scales + i / L);
        else if constexpr (BPI == 2)
          sc[u] = __ldg(reinterpret_cast<const unsigned short*>(scales) + i);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = base + (int64_t)u * T;
      if (i >= nitems) continue;
      float out[EPT];
#if MX_DQ_HWDEC
      uint32_t hv[EPT / 2];
#pragma unroll
      for (int j = 0; j < EPT / 8; ++j) e2m1x8_to_f16x2(cw[u][j], &hv[4 * j]);
#pragma unroll
      for (int b = 0; b < BPI; ++b) {
        const float D = s_D[(sc[u] >> (8 * b)) & 0xFF];
        constexpr int BE = EPT / BPI;
#pragma unroll
        for (int k = 0; k < BE / 2; ++k) {
          const int e = b * BE + 2 * k;  // elements e, e + 1: word e / 2 of hv
          const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&hv[e / 2]));
          const float2 y2 = __fmul2_rn(v, make_float2(D, D));  // exact
          out[e] = y2.x;
          out[e + 1] = y2.y;
        }
      }
#else
#pragma unroll
      for (int b = 0; b < BPI; ++b) {
        const float D = s_D[(sc[u] >> (8 * b)) & 0xFF];
        constexpr int BE = EPT / BPI;
#pragma unroll
        for (int k = 0; k < BE; ++k) {
          const int e = b * BE + k;  // element index in the item: nibble e % 8 of word e / 8
          const float f = __uint_as_float(e2m1_scaled_bits_at(cw[u][e / 8], 4 * (e % 8)));
          out[e] = __fmul_rn(__fmul_rn(f, 0x1p126f), D);
        }
      }
#endif
      if constexpr (BF16OUT) {
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
  }
}

// The last 4 codes when N = 4 and numel % 8 == 4.
template <int FMT, bool BF16OUT>
__global__ void k_dequantize_tail4(const uint8_t* __restrict__ packed,
                                   const uint8_t* __restrict__ scales, int64_t first,
                                   uint16_t g_bits, const uint16_t* g_dev, void* __restrict__ y) {
  if (threadIdx.x >= 4) return;
  const int64_t e = first + threadIdx.x;
  const float D = __fmul_rn(scale_value(scales[first / 4], FMT),
                            fp16_bits_to_float(tensor_g_bits(g_bits, g_dev)));
  const uint32_t nib = (uint32_t)(packed[e / 2] >> (4 * (e & 1))) & 0xFu;
  const float v = __fmul_rn(e2m1_to_float(nib), D);
  if (BF16OUT)
    reinterpret_cast<__nv_bfloat16*>(y)[e] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float*>(y)[e] = v;
}

template <int N, int FMT, bool BF16OUT>
static cudaError_t launch_dq(const TensorArgs* ta, int count, cudaStream_t stream,
                             int* launches) {
  using S = DShape<N, BF16OUT>;
  DGroup grp = {};
  int64_t nitems[kMaxGroup];
  for (int k = 0; k < count; ++k) {
    nitems[k] = ta[k].numel / S::EPT;
    grp.t[k] = {ta[k].packed, ta[k].scales, ta[k].y, nitems[k], ta[k].g_bits, ta[k].g_dev};
  }
  const int grid = split_grid((const void*)k_dequantize<N, FMT, BF16OUT>, nitems, count, S::U,
                              1 << 30, &grp.split);
  if (grid > 0) {
    const cudaError_t e =
        launch_pdl(k_dequantize<N, FMT, BF16OUT>, grid, kThreads, stream, grp);
    if (e != cudaSuccess) return e;
    ++*launches;
  }
  for (int k = 0; k < count; ++k) {
    if (ta[k].numel % S::EPT != 0) {
      k_dequantize_tail4<FMT, BF16OUT><<<1, 32, 0, stream>>>(ta[k].packed, ta[k].scales,
                                                              nitems[k] * S::EPT, ta[k].g_bits,
                                                              ta[k].g_dev, ta[k].y);
      ++*launches;
    }
  }
  return cudaGetLastError();
}

template <int FMT, bool BF16OUT>
static cudaError_t dq_block(int block, const TensorArgs* t, int count, cudaStream_t st, int* n) {
  switch (block) {
    case 4: return launch_dq<4, FMT, BF16OUT>(t, count, st, n);
    case 8: return launch_dq<8, FMT, BF16OUT>(t, count, st, n);
    case 16: return launch_dq<16, FMT, BF16OUT>(t, count, st, n);
    case 32: return launch_dq<32, FMT, BF16OUT>(t, count, st, n);
    case 64: return launch_dq<64, FMT, BF16OUT>(t, count, st, n);
    case 128: return launch_dq<128, FMT, BF16OUT>(t, count, st, n);
    default: return launch_dq<256, FMT, BF16OUT>(t, count, st, n);
  }
}

cudaError_t run_dequantize_group(const TensorArgs* t, int count, bool bf16, int block, int fmt,
                                 cudaStream_t stream, int* launches) {
  if (fmt == kUE5M3)
    return bf16 ? dq_block<kUE5M3, true>(block, t, count, stream, launches)
                : dq_block<kUE5M3, false>(block, t, count, stream, launches);
  return bf16 ? dq_block<kE4M3, true>(block, t, count, stream, launches)
              : dq_block<kE4M3, false>(block, t, count, stream, launches);
}

cudaError_t run_dequantize(const uint8_t* packed, const uint8_t* scales, int64_t numel, int block,
                           int fmt, uint16_t g_bits, void* y, bool bf16, cudaStream_t stream,
                           int* launches) {
  const TensorArgs t = {nullptr, y, const_cast<uint8_t*>(packed), const_cast<uint8_t*>(scales),
                        nullptr, numel, g_bits};
  return run_dequantize_group(&t, 1, bf16, block, fmt, stream, launches);
}

}  // namespace mxk
