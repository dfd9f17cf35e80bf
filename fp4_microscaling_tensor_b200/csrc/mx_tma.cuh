// mx_tma.cuh -- tensor-copy (TMA) helpers of the row-tile kernels, and the host-side tensor-map
// encoder.
//
// A row-tile kernel writes a row-major tensor as tiles of kTileRows rows x kTileCols columns, one
// tile per warp at a time: the warp assembles its tile in shared memory and its lane 0 stores it
// with a 2-D tensor copy (cp.async.bulk.tensor, shared -> this GPU's global memory), which writes
// only the part of the box inside the tensor -- rows and columns past the end are left out, so a
// ragged last block needs nothing special.  Warps never wait for one another.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mxk {
namespace tma {

constexpr int kTileRows = 4;               // rows of a warp's tile (8 lanes per row)
constexpr int kTileCols = 256;             // columns of a tile (8 lanes x 32 elements per row)
constexpr int kTileBytes = kTileRows * kTileCols * 2;  // one bf16 tile: 2 KiB

#ifdef __CUDACC__
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
// 2-D tensor copy shared -> global of the box at (x, y) (x a multiple of 8, y >= 0); the part of
// the box outside the tensor is not written.
__device__ __forceinline__ void store_2d(const CUtensorMap* map, int x, int y, uint32_t src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(src)
               : "memory");
}
__device__ __forceinline__ void store_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Waits until at most N committed store groups are still reading their shared-memory source.
template <int N>
__device__ __forceinline__ void store_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Waits until every committed store group has completed.
__device__ __forceinline__ void store_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// Orders this thread's shared-memory writes before later tensor-copy reads of them.
__device__ __forceinline__ void fence_smem_to_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// A lane's place in its warp's tile: row (0..3), slice (0..7: 32 columns each) within the row, and
// the XOR that staggers its four 16-byte chunks so that the eight lanes of a row (one
// shared-memory wavefront of 16-byte accesses) touch eight different bank groups; `off` is the
// slice's byte offset in the tile.
struct TileLane {
  int row, slice, rot, off;
};
__device__ __forceinline__ TileLane tile_lane() {
  const int lane = threadIdx.x & 31;
  TileLane t;
  t.row = lane >> 3;
  t.slice = lane & 7;
  t.rot = (t.slice >> 1) & 3;
  t.off = t.row * (kTileCols * 2) + t.slice * 64;
  return t;
}

// Position of a warp's current tile among the tiles (rows of tiles x ntc tiles per row), walked
// with a stride of all the grid's warps: the stride is split once into whole rows of tiles and a
// column step, so moving on costs two adds and a compare (no division per tile).
struct TileCursor {
  int tr, tc;      // tile row, tile column
  int dr, dc, ntc;
  __device__ __forceinline__ void init(int64_t first, int64_t stride, int ntiles_per_row) {
    ntc = ntiles_per_row;
    tr = (int)(first / ntc);
    tc = (int)(first % ntc);
    dr = (int)(stride / ntc);
    dc = (int)(stride % ntc);
  }
  __device__ __forceinline__ void advance() {
    tc += dc;
    tr += dr;
    if (tc >= ntc) {
      tc -= ntc;
      ++tr;
    }
  }
};

#endif  // __CUDACC__

// ------------------------------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link-time libcuda).
inline EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// Map of a rows x cols row-major tensor of `esize`-byte elements (bf16 or fp32; the row pitch
// cols * esize a multiple of 16 bytes, the base 16-byte aligned) in boxes of kTileRows rows x
// kTileCols columns, no swizzle; a store writes only the part of a box inside the tensor.
inline bool map_row_tiles(CUtensorMap* map, const void* base, int64_t rows, int64_t cols,
                          int esize) {
  const EncodeTiledFn enc = encode_tiled();
  if (!enc || rows < 1 || cols < 1 || (cols * esize) % 16 != 0 || rows > 0x7FFFFFFF ||
      cols > 0x7FFFFFFF)
    return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(cols * esize)};
  const cuuint32_t box[2] = {(cuuint32_t)kTileCols, (cuuint32_t)kTileRows};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt =
      esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  return enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tma
}  // namespace mxk
