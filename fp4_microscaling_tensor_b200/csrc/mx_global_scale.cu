// mx_global_scale.cu -- per-tensor FP16 scale (sm_100a).
//
// The microscaling article (hotelren.com/news/2192771) §3.1 item 3 adds a per-tensor FP16 factor
// (value = FP4 x FP8_scale x FP16_scale) without saying how it is chosen.  This library takes the
// smallest binary16 value g with g * 6 * Smax >= A, A = max|x| (no block scale can saturate), 1.0 when
// A = 0, 65504 when even that is too small.
//
// One pass (k_global_scale): persistent grid (split among up to kMaxGroup tensors), max|x| per
// CTA, the last CTA of each tensor to finish picks that tensor's g.
#include "mx_device.cuh"
#include "mx_launch.h"

namespace mxk {

// The smallest binary16 g with g * 6 * Smax >= A (1.0 for A = 0, 65504 when none is large enough):
// RU(A / K) as a first guess, then one exact step either way (h * K is exact in fp32: h has <= 11
// and K = 6 * Smax <= 6 significant bits).
template <int FMT>
__device__ uint16_t pick_g(float A) {
  if (A == 0.0f) return 0x3C00;  // 1.0
  const float K = __fmul_rn(6.0f, scale_max<FMT>());
  const float q = __fdiv_rn(A, K);
  uint32_t h = __half_as_ushort(__float2half_ru(q));
  if (h > 0x7BFFu) h = 0x7BFFu;  // RU overflowed to inf: clamp at 65504
  if (h < 1u) h = 1u;
  auto val = [](uint32_t b) { return __half2float(__ushort_as_half((unsigned short)b)); };
  if (h > 1u && __fmul_rn(val(h - 1), K) >= A) h -= 1;
  if (__fmul_rn(val(h), K) < A && h < 0x7BFFu) h += 1;
  return (uint16_t)h;
}

// One tensor of a grouped launch and the split of the grid among the tensors.
struct GTensor {
  const void* x;
  int64_t nvec, numel;     // 16-byte vectors, elements
  uint16_t* out;           // where g goes (device)
  uint32_t* part;          // this tensor's CTAs' partial maxima
  unsigned int* counter;   // last-CTA counter, zeroed before the launch
};
struct GGroup {
  GTensor t[kMaxGroup];
  CtaSplit split;
};

// max|x| as the integer maximum of the magnitude bit patterns (non-negative IEEE values order like
// their bit patterns) over 16-byte vectors (8 bf16 or 4 fp32), MX_GS_U vectors in flight per thread;
// one partial per CTA.  The tensor's CTA that finishes last (one atomic counter per tensor, zeroed
// before the launch) takes the maximum of the partials and of the elements after the last whole
// vector, and writes g.  No CTA waits for another.
#ifndef MX_GS_U  // 16-byte vectors in flight per thread (8: 1.00 of the measured copy peak on a
#define MX_GS_U 8  // 70B-shaped layer, against 0.87 with 2 and 0.84 with 4)
#endif
template <bool BF16, int FMT>
__global__ void __launch_bounds__(kThreads) k_global_scale(const __grid_constant__ GGroup grp) {
  constexpr int U = MX_GS_U;
  const int ti = grp.split.find((int)blockIdx.x);
  const GTensor& t = grp.t[ti];
  const int cta = (int)blockIdx.x - grp.split.begin[ti];
  const int nctas = grp.split.begin[ti + 1] - grp.split.begin[ti];
  const void* __restrict__ x = t.x;
  const int64_t nvec = t.nvec;
  griddep_wait();  // x may come from the previous kernel in the stream
  griddep_launch_next();
  const int64_t T = (int64_t)nctas * blockDim.x;
  uint32_t m = 0;
  for (int64_t i = (int64_t)cta * blockDim.x + threadIdx.x; i < nvec; i += U * T) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      v[u] = make_uint4(0, 0, 0, 0);
      if (i + u * T < nvec) v[u] = ld_stream16(reinterpret_cast<const uint4*>(x) + i + u * T);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if constexpr (BF16) {
        uint32_t w = bf16x2_absmax(bf16x2_absmax(v[u].x, v[u].y), bf16x2_absmax(v[u].z, v[u].w));
        w &= 0x7FFF7FFFu;
        m = max(m, max(w & 0xFFFFu, w >> 16) << 16);  // as fp32 bits
      } else {
        m = max(m, max(max(v[u].x & 0x7FFFFFFFu, v[u].y & 0x7FFFFFFFu),
                       max(v[u].z & 0x7FFFFFFFu, v[u].w & 0x7FFFFFFFu)));
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ uint32_t sm[kThreads / 32];
  __shared__ unsigned int s_last;
  if ((threadIdx.x & 31) == 0) sm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t r = 0;
    for (int k = 0; k < kThreads / 32; ++k) r = max(r, sm[k]);
    t.part[cta] = r;
    __threadfence();
    s_last = atomicAdd(t.counter, 1u) == (unsigned)nctas - 1u;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  m = 0;
  for (int k = threadIdx.x; k < nctas; k += blockDim.x) m = max(m, __ldcg(t.part + k));
  const int64_t first = nvec * (BF16 ? 8 : 4);  // elements after the last whole vector
  for (int64_t k = first + threadIdx.x; k < t.numel; k += blockDim.x) {
    const uint32_t b = BF16 ? ((uint32_t)reinterpret_cast<const uint16_t*>(x)[k] << 16)
                            : reinterpret_cast<const uint32_t*>(x)[k];
    m = max(m, b & 0x7FFFFFFFu);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) sm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int k = 0; k < kThreads / 32; ++k) m = max(m, sm[k]);
    *t.out = pick_g<FMT>(__uint_as_float(m));
    *t.counter = 0;
  }
}

// Workspace: kMaxGroup 64-byte headers (the last-CTA counter of tensor k in header k), then one
// 4-byte partial per CTA of the launch.
constexpr int kGsHeader = 64 * kMaxGroup;
constexpr int kMaxGsGrid = kMaxReduceCtas - kGsHeader / 4;

template <bool BF16, int FMT>
static cudaError_t launch_gs(const TensorArgs* ta, int count, void* workspace, cudaStream_t stream,
                             int* launches) {
  unsigned int* counters = reinterpret_cast<unsigned int*>(workspace);
  uint32_t* part = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(workspace) + kGsHeader);
  GGroup grp = {};
  int64_t nitems[kMaxGroup];
  for (int k = 0; k < count; ++k) {
    const int64_t nvec = ta[k].numel / (BF16 ? 8 : 4);
    nitems[k] = nvec > 0 ? nvec : 1;  // every tensor gets a CTA: it writes g (1.0 when empty)
    grp.t[k] = {ta[k].x, nvec, ta[k].numel, ta[k].g_dev, nullptr, counters + 16 * k};
  }
  const int grid = split_grid((const void*)k_global_scale<BF16, FMT>, nitems, count, MX_GS_U, kMaxGsGrid,
                              &grp.split);
  for (int k = 0; k < count; ++k) grp.t[k].part = part + grp.split.begin[k];
  cudaError_t e = launch_counters_reset(counters, count, stream, launches);
  if (e != cudaSuccess) return e;
  e = launch_pdl(k_global_scale<BF16, FMT>, grid, kThreads, stream, grp);
  if (e != cudaSuccess) return e;
  ++*launches;
  return cudaGetLastError();
}

cudaError_t run_global_scale_group(const TensorArgs* t, int count, bool bf16, int fmt,
                                   void* workspace, cudaStream_t stream, int* launches) {
  if (bf16)
    return fmt == kUE5M3 ? launch_gs<true, kUE5M3>(t, count, workspace, stream, launches)
                         : launch_gs<true, kE4M3>(t, count, workspace, stream, launches);
  return fmt == kUE5M3 ? launch_gs<false, kUE5M3>(t, count, workspace, stream, launches)
                       : launch_gs<false, kE4M3>(t, count, workspace, stream, launches);
}

cudaError_t run_global_scale(const void* x, bool bf16, int64_t numel, int fmt, uint16_t* out,
                             void* workspace, cudaStream_t stream, int* launches) {
  TensorArgs t = {};
  t.x = x;
  t.numel = numel;
  t.g_dev = out;
  return run_global_scale_group(&t, 1, bf16, fmt, workspace, stream, launches);
}

}  // namespace mxk
