// mx_dequantize.cu -- dequantize kernel (sm_100a).
//
// Method: the microscaling article (hotelren.com/news/2192771) §1 and §3.1 item 3: the stored value
// is FP4 x FP8_scale x FP16_scale.  The product of an E2M1 value (<= 2 significant bits), an FP8
// scale (<= 4) and the FP16 g (<= 11) has at most 17 significant bits and stays inside the fp32
// normal range, so y = e2m1 * (S g) is exact in fp32; bf16 output is its round-to-nearest-even.
//
// Layout mirrors the quantize kernel: a thread owns EPT = 8 consecutive codes (MX_DQ_EPT_BF16 = 16
// for bf16 output with N >= 16 was measured slower: 0.64 against 0.85 of the copy peak), two items
// in flight, reads EPT/2 packed bytes and the scale byte(s) of its block(s), decodes the codes with
// the E2M1x2 -> f16x2 conversion on the loaded word (exact: E2M1 values are f16 values; bit
// arithmetic with MX_DQ_HWDEC = 0), multiplies by the per-code constant S g from a shared-memory
// table and writes 16-byte vectors.  Ragged rows with bf16 output go through k_tile_dequantize
// below: row tiles assembled in shared memory and written by TMA.
#include <cuda_fp16.h>

#include <atomic>

#include "mx_device.cuh"
#include "mx_launch.h"
#include "mx_tma.cuh"

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

// ------------------------------------------------------------------------------------------------
// Row tiles written by TMA: bf16 output whose rows start on 16-byte boundaries (cols % 8 == 0),
// any cols otherwise (mx_tma.cuh)
// ------------------------------------------------------------------------------------------------
// Each warp walks tiles of 4 rows x 256 columns of y (a stride of all the grid's warps).  A lane
// takes one 32-element slice of one row (tma::tile_lane): it loads the slice's 16 code bytes as
// four 4-byte words (a row's code bytes start on a 4-byte boundary; register word c is word c ^ rot
// of the slice) and its scale byte(s), the next tile's before the current tile's arithmetic;
// decodes them (E2M1x2 -> f16x2 conversion, times S g from a per-CTA table: exact; bf16 = its round
// to nearest even) into the warp's shared-memory copy of the tile (chunk c ^ rot at step c: eight
// bank groups per row); then lane 0 writes the tile with a 2-D tensor store, which leaves out the
// part of the box past the tensor's last row or column -- so a ragged last block needs nothing
// special.  Each warp alternates two tile buffers; a buffer is rewritten only after its previous
// store has finished reading it.  Warps never wait for one another.
namespace dqtiles {
constexpr int kBuffers = 2;
constexpr int kSmem = 8 * kBuffers * tma::kTileBytes + 128;  // 8 warps' buffers + slack
}  // namespace dqtiles

struct TileDqArgs {
  const uint8_t* packed;  // row pitch pb bytes
  const uint8_t* scales;  // row pitch nb bytes
  int rows, cols, pb, nb;
  int ntc, ntr;  // tiles per row of tiles, rows of tiles
  uint32_t g_bits;
  const uint16_t* g_dev;
};

template <int N, int FMT>
__global__ void __launch_bounds__(kThreads)
    k_tile_dequantize(const __grid_constant__ CUtensorMap ymap, const __grid_constant__ TileDqArgs a) {
  static_assert(N >= 16, "blocks of 16 and more");
  constexpr int BPL = N == 16 ? 2 : 1;  // blocks in a lane's slice
  extern __shared__ uint8_t tdq_smem_raw[];
  uint8_t* bufs = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(tdq_smem_raw) + 127) & ~uintptr_t(127));
  __shared__ float s_D[256];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float g = fp16_bits_to_float(tensor_g_bits(a.g_bits, a.g_dev));
  for (int c = threadIdx.x; c < 256; c += blockDim.x) s_D[c] = __fmul_rn(scale_value(c, FMT), g);
  __syncthreads();
  griddep_wait();  // codes and scales may come from the previous kernel in the stream
  griddep_launch_next();

  const tma::TileLane tl = tma::tile_lane();
  uint8_t* wbuf = bufs + warp * (dqtiles::kBuffers * tma::kTileBytes);
  struct Slice {
    uint32_t cw[4];  // register word c: code word c ^ rot of the slice
    uint32_t sc;     // scale byte(s): byte b = register block b
    int nvalid;
  };
  auto load = [&](const tma::TileCursor& at) {
    Slice v{{0u, 0u, 0u, 0u}, 0u, 0};
    if (at.tr >= a.ntr) return v;
    const int row = at.tr * tma::kTileRows + tl.row;
    const int col0 = at.tc * tma::kTileCols + tl.slice * 32;
    v.nvalid = row < a.rows ? max(0, min(32, a.cols - col0)) : 0;  // a multiple of 8
    if (v.nvalid == 0) return v;
    const uint8_t* prow = a.packed + (int64_t)row * a.pb + (col0 >> 1);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int cc = c ^ tl.rot;
      if (8 * cc < v.nvalid) v.cw[c] = __ldcs(reinterpret_cast<const unsigned int*>(prow + 4 * cc));
    }
    const uint8_t* srow = a.scales + (int64_t)row * a.nb;
    if constexpr (BPL == 2) {
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const int bb = b ^ (tl.rot >> 1);  // register block b is block bb of the slice
        if (16 * bb < v.nvalid) v.sc |= (uint32_t)__ldg(srow + col0 / 16 + bb) << (8 * b);
      }
    } else {
      v.sc = __ldg(srow + col0 / N);
    }
    return v;
  };

  const int64_t gwarp = (int64_t)blockIdx.x * 8 + warp, nwarps = (int64_t)gridDim.x * 8;
  tma::TileCursor at, ahead;  // the current tile and the next one
  at.init(gwarp, nwarps, a.ntc);
  ahead = at;
  ahead.advance();
  Slice cur = load(at);
  for (int k = 0; at.tr < a.ntr; ++k, at = ahead, ahead.advance()) {
    const Slice nxt = load(ahead);
    uint4 out[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t hv[4];
      e2m1x8_to_f16x2(cur.cw[c], hv);
      const float D = s_D[(cur.sc >> (8 * (BPL == 2 ? c / 2 : 0))) & 0xFF];
      uint32_t o[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&hv[h]));
        const float2 y2 = __fmul2_rn(v, make_float2(D, D));  // exact
        o[h] = pack_bf16x2(y2.x, y2.y);
      }
      out[c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    uint8_t* buf = wbuf + (k % dqtiles::kBuffers) * tma::kTileBytes;
    if (lane == 0) tma::store_wait_read<dqtiles::kBuffers - 1>();  // the buffer's last store
    __syncwarp();
    if (cur.nvalid > 0) {
      uint8_t* dst = buf + tl.off;
#pragma unroll
      for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4*>(dst + 16 * (c ^ tl.rot)) = out[c];
    }
    tma::fence_smem_to_async();  // the writes come before the store reads them
    __syncwarp();
    if (lane == 0) {
      tma::store_2d(&ymap, at.tc * tma::kTileCols, at.tr * tma::kTileRows, tma::smem_addr(buf));
      tma::store_commit();
    }
    cur = nxt;
  }
  if (lane == 0) tma::store_wait_all();
}

// Row-tile dequantize (k_tile_dequantize) of one tensor with bf16 output, cols % 8 == 0, N >= 16.
template <int N, int FMT>
static cudaError_t launch_tile_dq(const uint8_t* packed, const uint8_t* scales, int64_t rows,
                                  int64_t cols, uint16_t g_bits, const uint16_t* g_dev, void* y,
                                  cudaStream_t stream, int* launches) {
  static std::atomic<bool> smem_ok[kMaxDevices];
  auto kern = k_tile_dequantize<N, FMT>;
  CUtensorMap map;
  if (!tma::map_row_tiles(&map, y, rows, cols, 2)) return cudaErrorInvalidValue;
  cudaError_t e = allow_dynamic_smem(smem_ok, kern, dqtiles::kSmem);
  if (e != cudaSuccess) return e;
  const int ntc = (int)((cols + tma::kTileCols - 1) / tma::kTileCols);
  const int ntr = (int)((rows + tma::kTileRows - 1) / tma::kTileRows);
  int64_t grid = resident_ctas_smem((const void*)kern, dqtiles::kSmem);
  const int64_t need = ((int64_t)ntc * ntr + 7) / 8;  // one tile per warp at least
  if (grid > need) grid = need;
  const TileDqArgs args{packed, scales, (int)rows, (int)cols, (int)((cols + 1) / 2),
                        (int)((cols + N - 1) / N), ntc, ntr, g_bits, g_dev};
  e = launch_pdl_smem(kern, (int)grid, kThreads, dqtiles::kSmem, stream, map, args);
  if (e == cudaSuccess) ++*launches;
  return e;
}

template <int FMT>
static cudaError_t tile_dq_block(int block, const uint8_t* packed, const uint8_t* scales,
                                 int64_t rows, int64_t cols, uint16_t g_bits,
                                 const uint16_t* g_dev, void* y, cudaStream_t st, int* n) {
  switch (block) {
    case 16: return launch_tile_dq<16, FMT>(packed, scales, rows, cols, g_bits, g_dev, y, st, n);
    case 32: return launch_tile_dq<32, FMT>(packed, scales, rows, cols, g_bits, g_dev, y, st, n);
    case 64: return launch_tile_dq<64, FMT>(packed, scales, rows, cols, g_bits, g_dev, y, st, n);
    case 128: return launch_tile_dq<128, FMT>(packed, scales, rows, cols, g_bits, g_dev, y, st, n);
    default: return launch_tile_dq<256, FMT>(packed, scales, rows, cols, g_bits, g_dev, y, st, n);
  }
}

bool tile_dequantize_supported(bool y_bf16, int64_t rows, int64_t cols, int block) {
  return y_bf16 && block >= 16 && cols % 8 == 0 && rows >= 1 && rows <= 0x7FFFFFFF &&
         cols <= 0x7FFFFFFF;
}

cudaError_t run_tile_dequantize(const uint8_t* packed, const uint8_t* scales, int64_t rows,
                                int64_t cols, int block, int fmt, uint16_t g_bits,
                                const uint16_t* g_dev, void* y, cudaStream_t stream,
                                int* launches) {
  return fmt == kUE5M3
             ? tile_dq_block<kUE5M3>(block, packed, scales, rows, cols, g_bits, g_dev, y, stream,
                                     launches)
             : tile_dq_block<kE4M3>(block, packed, scales, rows, cols, g_bits, g_dev, y, stream,
                                    launches);
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
