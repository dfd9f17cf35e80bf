// mx_global_scale.cu -- per-tensor FP16 scale (sm_100a).
//
// The microscaling article (hotelren.com/news/2192771) §3.1 item 3 adds a per-tensor FP16 factor
// (value = FP4 x FP8_scale x FP16_scale) without saying how it is chosen.  This library takes the
// smallest binary16 value g with g * 6 * Smax >= A, A = max|x| (no block scale can saturate), 1.0 when
// A = 0, 65504 when even that is too small.
//
// Pass 1 (k_amax): persistent grid; max|x| as the integer maximum of the magnitude bit patterns
// (non-negative IEEE values order like their bit patterns), one partial per CTA.
// Pass 2 (k_amax_final): one CTA takes the maximum of the partials and picks g: RU(A / K) as a first
// guess, then one exact step either way using h * K, which is exact in fp32 (h has <= 11 and K =
// 6 * Smax <= 6 significant bits).
#include "mx_device.cuh"
#include "mx_launch.h"

namespace mxk {

template <bool BF16>
__global__ void __launch_bounds__(kThreads) k_amax(const void* __restrict__ x, int64_t nvec,
                                                   uint32_t* __restrict__ part) {
  // a "vector" is 16 bytes: 8 bf16 or 4 fp32 values
  const int64_t T = (int64_t)gridDim.x * blockDim.x;
  uint32_t m = 0;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nvec; i += 2 * T) {
    const uint4 v0 = ld_stream16(reinterpret_cast<const uint4*>(x) + i);
    uint4 v1 = make_uint4(0, 0, 0, 0);
    if (i + T < nvec) v1 = ld_stream16(reinterpret_cast<const uint4*>(x) + i + T);
    if constexpr (BF16) {
      uint32_t t = bf16x2_absmax(bf16x2_absmax(v0.x, v0.y), bf16x2_absmax(v0.z, v0.w));
      t = bf16x2_absmax(t, bf16x2_absmax(bf16x2_absmax(v1.x, v1.y), bf16x2_absmax(v1.z, v1.w)));
      t &= 0x7FFF7FFFu;
      m = max(m, max(t & 0xFFFFu, t >> 16) << 16);  // as fp32 bits
    } else {
      const uint32_t a = max(max(v0.x & 0x7FFFFFFFu, v0.y & 0x7FFFFFFFu),
                             max(v0.z & 0x7FFFFFFFu, v0.w & 0x7FFFFFFFu));
      const uint32_t b = max(max(v1.x & 0x7FFFFFFFu, v1.y & 0x7FFFFFFFu),
                             max(v1.z & 0x7FFFFFFFu, v1.w & 0x7FFFFFFFu));
      m = max(m, max(a, b));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ uint32_t sm[kThreads / 32];
  if ((threadIdx.x & 31) == 0) sm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t r = 0;
    for (int k = 0; k < kThreads / 32; ++k) r = max(r, sm[k]);
    part[blockIdx.x] = r;
  }
}

// Remaining elements that do not fill a 16-byte vector (at most 7 bf16 or 3 fp32).
template <bool BF16>
__global__ void k_amax_tail(const void* __restrict__ x, int64_t first, int64_t numel,
                            uint32_t* __restrict__ part) {
  if (threadIdx.x != 0) return;
  uint32_t m = 0;
  for (int64_t i = first; i < numel; ++i) {
    const uint32_t b = BF16 ? ((uint32_t)reinterpret_cast<const uint16_t*>(x)[i] << 16)
                            : reinterpret_cast<const uint32_t*>(x)[i];
    m = max(m, b & 0x7FFFFFFFu);
  }
  part[0] = m;
}

template <int FMT>
__global__ void __launch_bounds__(kThreads) k_amax_final(const uint32_t* __restrict__ part,
                                                         int nparts, uint16_t* __restrict__ out) {
  uint32_t m = 0;
  for (int k = threadIdx.x; k < nparts; k += blockDim.x) m = max(m, part[k]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ uint32_t sm[kThreads / 32];
  if ((threadIdx.x & 31) == 0) sm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x != 0) return;
  for (int k = 0; k < kThreads / 32; ++k) m = max(m, sm[k]);
  const float A = __uint_as_float(m);
  if (A == 0.0f) {
    *out = 0x3C00;  // 1.0
    return;
  }
  const float K = __fmul_rn(6.0f, scale_max<FMT>());
  const float q = __fdiv_rn(A, K);
  uint32_t h = __half_as_ushort(__float2half_ru(q));
  if (h > 0x7BFFu) h = 0x7BFFu;  // RU overflowed to inf: clamp at 65504
  if (h < 1u) h = 1u;
  auto val = [](uint32_t b) { return __half2float(__ushort_as_half((unsigned short)b)); };
  // exact corrections: h * K is exact in fp32
  if (h > 1u && __fmul_rn(val(h - 1), K) >= A) h -= 1;
  if (__fmul_rn(val(h), K) < A && h < 0x7BFFu) h += 1;
  *out = (uint16_t)h;
}

cudaError_t run_global_scale(const void* x, bool bf16, int64_t numel, int fmt, uint16_t* out,
                             void* workspace, cudaStream_t stream, int* launches) {
  uint32_t* part = reinterpret_cast<uint32_t*>(workspace);
  const int per_vec = bf16 ? 8 : 4;
  const int64_t nvec = numel / per_vec;
  int nparts = 0;
  if (nvec > 0) {
    const void* kern = bf16 ? (const void*)k_amax<true> : (const void*)k_amax<false>;
    const int grid = persistent_grid(kern, nvec, 2, kMaxReduceCtas - 1);
    if (bf16)
      k_amax<true><<<grid, kThreads, 0, stream>>>(x, nvec, part);
    else
      k_amax<false><<<grid, kThreads, 0, stream>>>(x, nvec, part);
    ++*launches;
    nparts = grid;
  }
  if (nvec * per_vec < numel) {
    if (bf16)
      k_amax_tail<true><<<1, 32, 0, stream>>>(x, nvec * per_vec, numel, part + nparts);
    else
      k_amax_tail<false><<<1, 32, 0, stream>>>(x, nvec * per_vec, numel, part + nparts);
    ++*launches;
    ++nparts;
  }
  if (fmt == kUE5M3)
    k_amax_final<kUE5M3><<<1, kThreads, 0, stream>>>(part, nparts, out);
  else
    k_amax_final<kE4M3><<<1, kThreads, 0, stream>>>(part, nparts, out);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace mxk
