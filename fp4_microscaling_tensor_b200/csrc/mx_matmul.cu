// mx_matmul.cu -- C = gA gB * dequant(A) dequant(B)^T on the fifth-generation tensor cores.
//
// Method: the 4-bit float quantization article (gtnt.cn/news/16247) §3.1 runs inference by
// dequantizing stored FP4 weights and multiplying; here both operands are stored by this library
// (E2M1 codes, two per byte, low nibble first; one E4M3 scale per block of 16 along the reduction
// dimension k; an FP16 global scale per operand) and the tensor core applies the block scales
// inside the multiply (tcgen05.mma kind::mxf4nvf4, block16, E4M3 scales), so nothing is
// dequantized to memory.  A is m x k and B is n x k, both row-major with k contiguous ("K-major"),
// which is the layout the quantizer writes; C is m x n row-major, float32 or bfloat16.
//
// One CTA per 128 x BN tile of C (MMA N = BN), 4 warps.  BN = 128 with 3 stages by default: the
// CTA then needs 108 KiB of shared memory and 256 TMEM columns, so two CTAs share an SM and one
// CTA's prologue and epilogue overlap the other's main loop (measured 3127 TFLOP/s at 8192^3
// against 2830 for BN = 256, whose 216 KiB and 512 columns allow one CTA per SM):
//   * warp 0, one thread, produces: for each 256-element step of k, one TMA load per operand
//     (128 or BN rows x 128 bytes, 128-byte swizzle) and one bulk copy per 128-row tile of the
//     step's scales, which mx_matmul_prepare_scales has already put into tensor-core order (2048
//     contiguous bytes per 128 rows and step), all completing on the stage's full mbarrier;
//   * warp 1, one thread, issues per step the tcgen05.cp copies of the scale groups into TMEM
//     (rotating through MX_MM_SFBUF buffers) and 4 tcgen05.mma (128 x BN x 64 each, fp32
//     accumulator in TMEM), then a tcgen05.commit that frees the stage;
//   * all 4 warps then read the accumulator (tcgen05.ld, one row per thread), multiply by gA gB
//     and store C.
// Every wait is bounded: a CTA that gives up records it in a device counter and marks its launch
// (a generation number passed per launch) so that the launch's other CTAs stop waiting too; it
// lets its issued copies and MMAs finish (bounded again), frees its TMEM and returns.  Later
// launches carry other generation numbers and are not affected.
#include <cuda.h>

#include <atomic>

#include "mx_device.cuh"
#include "mx_launch.h"
#include "mx_tma.cuh"

namespace mxk {
namespace {

#ifndef MX_MM_PAIR_STAGES  // pipeline stages of the CTA-pair kernel
#define MX_MM_PAIR_STAGES 5
#endif
#ifndef MX_MM_PROD_SLEEP  // ns slept between polls of an empty barrier by a producer
#define MX_MM_PROD_SLEEP 20
#endif

#ifndef MX_MM_SFBUF  // TMEM copies of the scales in rotation: a step's scale copies never wait
#define MX_MM_SFBUF 2  // for the previous step's MMAs to finish reading the same columns
#endif
#ifndef MX_MM_BN  // columns of C per CTA in the one-CTA kernel: 128 or 256 (MMA N)
#define MX_MM_BN 128
#endif
#ifndef MX_MM_STAGES128  // pipeline stages of the one-CTA kernel with 128-column tiles: 3 keeps
#define MX_MM_STAGES128 3  // two CTAs per SM (shared memory and TMEM), so that one CTA's epilogue
                           // overlaps the other's main loop
#endif

constexpr int kBM = 128;              // rows of C per CTA (MMA M)
constexpr int kBK = 256;              // k elements per stage (128 bytes of codes per row)
constexpr int kRowBytes = kBK / 2;
constexpr uint32_t kWaitLimit = 1u << 20;  // polls of one mbarrier before a CTA gives up

// Tile geometry for BN columns of C per CTA.
template <int BN>
struct Tile {
  static constexpr int kHalves = BN / 128;                     // 128-row scale atoms of B per step
  static constexpr int kStages = BN == 256 ? 4 : MX_MM_STAGES128;
  static constexpr int kABytes = kBM * kRowBytes;             // 16 KiB
  static constexpr int kBBytes = BN * kRowBytes;              // 16 or 32 KiB
  static constexpr int kSfaBytes = kBM * (kBK / 16);          // four 512-byte atoms
  static constexpr int kSfbBytes = BN * (kBK / 16);           // 4 x kHalves atoms
  static constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
  static_assert(kStageBytes % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
  static constexpr int kSmemBytes = kStages * kStageBytes + 256 + 1024;  // + barriers, alignment
  // TMEM: accumulator BN columns, then MX_MM_SFBUF scale buffers of kSfCols columns each: A's
  // scales (4 per MMA step), then B's (4 kHalves per step); column w of a step's scales serves
  // rows 32 w .. 32 w + 31 of its operand tile.
  static constexpr uint32_t kSfCols = 16 + 16 * kHalves;
  static constexpr uint32_t kSfaCol = BN, kSfbCol = BN + 16;
  static constexpr uint32_t kTmemCols = BN == 256 ? 512 : 256;
  static_assert(BN + MX_MM_SFBUF * kSfCols <= kTmemCols, "TMEM columns");
  // Instruction descriptor of kind::mxf4nvf4 (block-scaled): A and B E2M1 (format 1), K-major,
  // E4M3 scales (scale format 0), N = BN (bits 17..22: N / 8), M = 128 (bits 24..28: M / 16),
  // scale-factor ids 0, dense, K = 64.
  static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                     ((uint32_t)(kBM >> 4) << 24);
};

__device__ unsigned int g_mm_gave_up;  // CTAs that stopped waiting (bounded waits ran out)
// Generation number of the last launch one of whose CTAs gave up: the launch's other CTAs stop
// waiting too.  Every launch gets a new number (from 1), so a launch that gave up leaves later
// launches alone.
__device__ volatile unsigned int g_mm_abandon_gen;

struct MmArgs {
  const uint8_t* a_scales;
  const uint8_t* b_scales;
  void* c;
  int64_t m, n, k;
  float alpha;
  int c_bf16;
  unsigned int gen;  // this launch's generation number (never 0)
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
// True once the phase with the given parity has completed; false after kWaitLimit polls, or
// earlier once another CTA has given up.  SLEEP_NS > 0 sleeps between polls: waits off the
// critical path must not flood the shared-memory pipe that the TMA and the tensor core use.
// CLUSTER: acquire at cluster scope (the phase was completed by the other CTA of a pair).
template <int SLEEP_NS = 0, bool CLUSTER = false>
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, unsigned int gen) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if ((i & 1023u) == 1023u && g_mm_abandon_gen == gen) return false;
    if (SLEEP_NS > 0 && i > 0) __nanosleep(SLEEP_NS);
    uint32_t ok;
    if constexpr (CLUSTER)
      asm volatile(
          "{\n\t.reg .pred p;\n\t"
          "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
          "selp.u32 %0, 1, 0, p;\n\t}"
          : "=r"(ok)
          : "r"(bar), "r"(parity)
          : "memory");
    else
      asm volatile(
          "{\n\t.reg .pred p;\n\t"
          "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
          "selp.u32 %0, 1, 0, p;\n\t}"
          : "=r"(ok)
          : "r"(bar), "r"(parity)
          : "memory");
    if (ok) return true;
  }
  return false;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor, K-major operand with 128-byte swizzle: rows of 128 bytes,
// 8-row groups 1024 bytes apart (stride byte offset), version 1, layout type 2.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Descriptor of one 512-byte scale atom for tcgen05.cp: 32 rows of 16 bytes, no swizzle, 8-row
// groups 128 bytes apart.
__device__ __forceinline__ uint64_t desc_sf(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(128 >> 4) << 32) |
         ((uint64_t)1 << 46);
}

__device__ __forceinline__ void tc_copy_sf(uint32_t taddr, uint64_t desc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc)
               : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], "
      "p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// 32 consecutive accumulator columns of this warp's 32 lanes (one row per thread).
__device__ __forceinline__ void tc_load32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// One contiguous block of global memory into shared memory (bulk copy engine), completing on bar.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Scale bytes in tensor-core order: for each 128-row tile t of an operand and each 256-element
// step kt of k, 2048 contiguous bytes = four 512-byte atoms (one per 64-element MMA step j); in
// atom j, row 32 q + r of the tile has its four scales at byte 16 r + 4 q.  The tile count is
// rounded up to even (a 256-column tile of C reads two), and rows past the end of the operand
// give zero scales.  One thread per (t, kt, r) reads the 16 scale bytes of rows 32 q + r
// (q = 0..3) and writes 16 bytes to each atom.
__global__ void k_scales_to_mma(const uint8_t* __restrict__ scales, int64_t rows, int64_t k,
                                uint8_t* __restrict__ out) {
  const int64_t KT = k / kBK, pitch = k / 16;
  const int64_t tiles = 2 * ((rows + 2 * kBM - 1) / (2 * kBM));
  const int64_t total = tiles * KT * 32;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int r = (int)(i & 31);
    const int64_t tk = i >> 5, t = tk / KT, kt = tk - t * KT;
    uint4 v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int64_t row = t * kBM + 32 * q + r;
      v[q] = row < rows ? __ldg(reinterpret_cast<const uint4*>(scales + row * pitch + kt * 16))
                        : make_uint4(0, 0, 0, 0);
    }
    uint8_t* dst = out + tk * 2048 + 16 * r;
    *reinterpret_cast<uint4*>(dst + 0) = make_uint4(v[0].x, v[1].x, v[2].x, v[3].x);
    *reinterpret_cast<uint4*>(dst + 512) = make_uint4(v[0].y, v[1].y, v[2].y, v[3].y);
    *reinterpret_cast<uint4*>(dst + 1024) = make_uint4(v[0].z, v[1].z, v[2].z, v[3].z);
    *reinterpret_cast<uint4*>(dst + 1536) = make_uint4(v[0].w, v[1].w, v[2].w, v[3].w);
  }
}

// Epilogue of one CTA: accumulator rows row0 + 32 w + lane (one per thread; warp w reads TMEM
// lanes 32 w ..), NC columns from n0, times alpha, stored to C as float32 or bfloat16.
template <int NC>
__device__ __forceinline__ void store_rows(uint32_t tmem, int warp, int lane, int64_t row0,
                                           int64_t n0, const MmArgs& args) {
  const int64_t row = row0 + 32 * warp + lane;
  const bool row_ok = row < args.m;
#pragma unroll 1
  for (int cb = 0; cb < NC / 32; ++cb) {
    uint32_t r[32];
    tc_load32(tmem + ((uint32_t)(32 * warp) << 16) + 32 * cb, r);
    const int64_t col = n0 + 32 * cb;
    if (!row_ok || col >= args.n) continue;
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __fmul_rn(__uint_as_float(r[i]), args.alpha);
    const bool whole = col + 32 <= args.n;
    if (args.c_bf16) {
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(args.c) + row * args.n + col;
      if (whole && (args.n % 8) == 0) {
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          uint4 pk;
          pk.x = pack_bf16x2(v[i], v[i + 1]);
          pk.y = pack_bf16x2(v[i + 2], v[i + 3]);
          pk.z = pack_bf16x2(v[i + 4], v[i + 5]);
          pk.w = pack_bf16x2(v[i + 6], v[i + 7]);
          *reinterpret_cast<uint4*>(out + i) = pk;
        }
      } else {
        for (int i = 0; i < 32 && col + i < args.n; ++i) out[i] = __float2bfloat16_rn(v[i]);
      }
    } else {
      float* out = static_cast<float*>(args.c) + row * args.n + col;
      if (whole && (args.n % 4) == 0) {
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(out + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
      } else {
        for (int i = 0; i < 32 && col + i < args.n; ++i) out[i] = v[i];
      }
    }
  }
}

template <int BN>
__global__ void __launch_bounds__(128, 1)
    k_matmul_nvfp4(const __grid_constant__ CUtensorMap tma_a,
                   const __grid_constant__ CUtensorMap tma_b, const __grid_constant__ MmArgs args) {
  using T = Tile<BN>;
  constexpr int kStages = T::kStages, kStageBytes = T::kStageBytes, kABytes = T::kABytes,
                kBBytes = T::kBBytes, kSfaBytes = T::kSfaBytes, kSfbBytes = T::kSfbBytes,
                kH = T::kHalves;
  constexpr uint32_t kTmemCols = T::kTmemCols, kSfaCol = T::kSfaCol, kSfbCol = T::kSfbCol;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* done = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* gave_up = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t m0 = (int64_t)blockIdx.y * kBM, n0 = (int64_t)blockIdx.x * BN;
  const int KT = (int)(args.k / kBK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(full + s), 1);
      mbar_init(smem_u32(empty + s), 1);
    }
    mbar_init(smem_u32(done), 1);
    *gave_up = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- producer (one thread) ----------------
    if (lane == 0) {
      const int64_t KTl = KT;
      const uint8_t* sfa_src = args.a_scales + (m0 / kBM) * KTl * 2048;
      const uint8_t* sfb_src = args.b_scales + (n0 / kBM) * KTl * 2048;
      int issued = 0;
      for (int kt = 0; kt < KT; ++kt) {
        const int s = kt % kStages;
        if (*gave_up ||
            (kt >= kStages && !mbar_wait<MX_MM_PROD_SLEEP>(smem_u32(empty + s), ((kt / kStages) + 1) & 1,
                                                     args.gen))) {
          *gave_up = 1;
          break;
        }
        const uint32_t st = smem_u32(smem + s * kStageBytes), bar = smem_u32(full + s);
        mbar_expect_tx(bar, kABytes + kBBytes + kSfaBytes + kSfbBytes);  // OOB rows included
        tma_load_2d(st, &tma_a, kt * kRowBytes, (int)m0, bar);
        tma_load_2d(st + kABytes, &tma_b, kt * kRowBytes, (int)n0, bar);
        // scales: A's tile, then each 128-row half of B's (2048 bytes per tile and step)
        bulk_load(st + kABytes + kBBytes, sfa_src + (int64_t)kt * 2048, 2048, bar);
#pragma unroll
        for (int h = 0; h < kH; ++h)
          bulk_load(st + kABytes + kBBytes + kSfaBytes + 2048 * h,
                    sfb_src + ((int64_t)h * KTl + kt) * 2048, 2048, bar);
        mbar_arrive(bar);
        issued = kt + 1;
      }
      if (*gave_up) {
        // let the copies already issued land before the CTA can exit (bounded)
        for (int kt = issued - kStages < 0 ? 0 : issued - kStages; kt < issued; ++kt)
          mbar_wait<100>(smem_u32(full + kt % kStages), (kt / kStages) & 1, args.gen);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer (one thread) ----------------
    if (lane == 0) {
      for (int kt = 0; kt < KT; ++kt) {
        const int s = kt % kStages;
        if (!mbar_wait(smem_u32(full + s), (kt / kStages) & 1, args.gen)) {
          *gave_up = 1;
          break;
        }
        tc_fence_after();
        const uint32_t st = smem_u32(smem + s * kStageBytes);
        const uint32_t sfa = st + kABytes + kBBytes, sfb = sfa + kSfaBytes;
        const uint32_t tsf = tmem + (kt % MX_MM_SFBUF) * T::kSfCols;  // this step's buffer
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          tc_copy_sf(tsf + kSfaCol + 4 * j, desc_sf(sfa + 512 * j));
#pragma unroll
          for (int h = 0; h < kH; ++h)
            tc_copy_sf(tsf + kSfbCol + 4 * (kH * j + h), desc_sf(sfb + 2048 * h + 512 * j));
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
          tc_mma(tmem, desc_sw128(st + 32 * j), desc_sw128(st + kABytes + 32 * j), T::kIdesc,
                 tsf + kSfaCol + 4 * j, tsf + kSfbCol + 4 * kH * j, (kt | j) != 0);
        tc_commit(smem_u32(empty + s));
      }
      tc_commit(smem_u32(done));  // also after giving up: the epilogue waits for issued MMAs
    }
    __syncwarp();
  }

  // ---------------- epilogue: all 4 warps, one accumulator row per thread ----------------
  __syncwarp();
  bool ok = true;
  if (lane == 0) {
    ok = mbar_wait<200>(smem_u32(done), 0, args.gen);  // sleeps through the main loop
    if (!ok) *gave_up = 1;
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  tc_fence_after();
  if (__all_sync(0xffffffffu, ok && !*gave_up)) store_rows<BN>(tmem, warp, lane, m0, n0, args);
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *gave_up) {
    atomicAdd(&g_mm_gave_up, 1u);
    g_mm_abandon_gen = args.gen;
  }
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}


// ------------------------------------------------------------------------------------------------
// CTA pair (tcgen05 cta_group::2): a cluster of two CTAs on one TPC computes a 256 x 256 tile of
// C with 256 x 256 x 64 MMAs issued by the even CTA (the leader).  CTA r holds rows 128 r .. of
// the tile's A rows and rows 128 r .. of its 256 B rows (the MMA reads both CTAs' shared memory
// at the same offsets), A's scales for its own rows and B's scales for all 256 rows; the
// accumulator of CTA r (its 128 rows x 256 columns) is in its own TMEM.  Per SM that is 32 KiB
// of codes per 256-element step for 128 x 256 outputs, against 48 KiB in the one-CTA kernel.
// Both CTAs' tile and scale copies (TMA, cta_group::2 form, no multicast) complete on the
// leader's full barrier, which expects the bytes of both; the leader commits its MMAs to its own
// and to the peer's empty / done barriers with separate single-target commits.
// ------------------------------------------------------------------------------------------------
// Geometry of the CTA-pair kernel: 256 x PN tiles of C, each CTA of the pair holding 128 rows of A
// and PN / 2 rows of B per stage.  PN = 256: 5 stages, 512 TMEM columns, one CTA per SM; PN = 128:
// 3 stages of 28 KiB and 256 TMEM columns, so two CTAs (of different pairs) share an SM.
#ifndef MX_MM_PAIR_N
#define MX_MM_PAIR_N 128
#endif
template <int PN>
struct PairT {
  static constexpr int kStages = PN == 256 ? MX_MM_PAIR_STAGES : 3;
  static constexpr int kBRows = PN / 2;              // this CTA's rows of B
  static constexpr int kGroups = PN / 128;           // 128-row scale groups of B
  static constexpr int kABytes = kBM * kRowBytes;    // this CTA's 128 rows of A
  static constexpr int kBBytes = kBRows * kRowBytes;
  static constexpr int kSfaBytes = 2048;             // A's scales, this CTA's rows
  static constexpr int kSfbBytes = 2048 * kGroups;   // B's scales, all PN rows
  static constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
  static_assert(kStageBytes % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
  static constexpr int kSmemBytes = kStages * kStageBytes + 256 + 1024;
  static constexpr uint32_t kTmemCols = PN == 256 ? 512 : 256, kSfaCol = PN, kSfbCol = PN + 16,
                            kSfCols = 16 + 16 * kGroups;
  static_assert(PN + MX_MM_SFBUF * kSfCols <= kTmemCols, "TMEM columns");
  // M = 256 (bits 24..28: 16), N = PN (bits 17..22: PN / 8), otherwise as the one-CTA descriptor
  static constexpr uint32_t kIdesc =
      (1u << 7) | (1u << 10) | ((uint32_t)(PN >> 3) << 17) | (16u << 24);
};
using Pair = PairT<MX_MM_PAIR_N>;

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_to(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
                   "memory");
}
// TMA 2-D load into this CTA's shared memory whose completion is counted on an mbarrier of
// either CTA of the pair (here: the leader's).
__device__ __forceinline__ void tma2_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                             uint32_t cluster_bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(cluster_bar)
      : "memory");
}
__device__ __forceinline__ void tc2_copy_sf(uint32_t taddr, uint64_t desc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc)
               : "memory");
}
__device__ __forceinline__ void tc2_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                        uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], "
      "p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}
// Arrive on one mbarrier (this CTA's or the peer's, shared::cluster address) when the pair's
// MMAs issued so far are complete.
__device__ __forceinline__ void tc2_commit(uint32_t cluster_addr) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   cluster_addr)
               : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(128, 1)
    k_matmul_nvfp4_pair(const __grid_constant__ CUtensorMap tma_a,
                        const __grid_constant__ CUtensorMap tma_b,
                        const __grid_constant__ CUtensorMap tma_sfa,
                        const __grid_constant__ CUtensorMap tma_sfb,
                        const __grid_constant__ MmArgs args) {
  using P = Pair;
  constexpr int kStages = P::kStages, kStageBytes = P::kStageBytes, kABytes = P::kABytes,
                kBBytes = P::kBBytes, kSfaBytes = P::kSfaBytes, kSfbBytes = P::kSfbBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* done = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* gave_up = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  constexpr int PN = MX_MM_PAIR_N;
  const int64_t pair = blockIdx.x >> 1, NT = (args.n + PN - 1) / PN;
  const int64_t mt = pair / NT, nt = pair - mt * NT;
  const int64_t m0 = mt * 256 + 128 * rank;  // this CTA's rows of A and of C
  const int64_t n0 = nt * PN;                // the pair's columns of C
  const int KT = (int)(args.k / kBK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(full + s), 1);
      mbar_init(smem_u32(empty + s), 1);
    }
    mbar_init(smem_u32(done), 1);
    *gave_up = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(P::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers initialized and TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------- producer (one thread per CTA) ----------------
    // Both CTAs' copies complete on the leader's full barrier; the leader expects both.
    if (lane == 0) {
      const uint32_t full0 = map_to(smem_u32(full), 0);
      const int sfa_row = (int)((m0 / kBM) * KT * 8), sfb_row = (int)((n0 / kBM) * KT * 8);
      int issued = 0;
      for (int kt = 0; kt < KT; ++kt) {
        const int s = kt % kStages;
        if (*gave_up ||
            (kt >= kStages && !mbar_wait<MX_MM_PROD_SLEEP>(smem_u32(empty + s), ((kt / kStages) + 1) & 1,
                                                     args.gen))) {
          *gave_up = 1;
          break;
        }
        const uint32_t st = smem_u32(smem + s * kStageBytes), bar = full0 + 8 * s;
        if (rank == 0)
          mbar_expect_tx(smem_u32(full + s), 2 * (kABytes + kBBytes + kSfaBytes + kSfbBytes));
        tma2_load_2d(st, &tma_a, kt * kRowBytes, (int)m0, bar);
        tma2_load_2d(st + kABytes, &tma_b, kt * kRowBytes, (int)(n0 + P::kBRows * rank), bar);
        // scale groups: 2048 bytes = 8 rows of 256 in the scale maps
        tma2_load_2d(st + kABytes + kBBytes, &tma_sfa, 0, sfa_row + 8 * kt, bar);
#pragma unroll
        for (int h = 0; h < P::kGroups; ++h)
          tma2_load_2d(st + kABytes + kBBytes + kSfaBytes + 2048 * h, &tma_sfb, 0,
                       sfb_row + 8 * (h * KT + kt), bar);
        if (rank == 0) mbar_arrive(smem_u32(full + s));
        issued = kt + 1;
      }
      if (*gave_up && issued > 0) {
        // this CTA cannot see its copies complete (they count on the leader's barrier): give
        // them time to land before the CTA may exit (bounded)
        for (int i = 0; i < 4096; ++i) __nanosleep(1000);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------- MMA issuer (leader, one thread) ----------------
      const uint32_t empty1 = map_to(smem_u32(empty), 1), done1 = map_to(smem_u32(done), 1);
      for (int kt = 0; kt < KT; ++kt) {
        const int s = kt % kStages;
        if (!mbar_wait(smem_u32(full + s), (kt / kStages) & 1, args.gen)) {
          *gave_up = 1;
          break;
        }
        tc_fence_after();
        const uint32_t st = smem_u32(smem + s * kStageBytes);
        const uint32_t sfa = st + kABytes + kBBytes, sfb = sfa + kSfaBytes;
        const uint32_t tsf = tmem + (kt % MX_MM_SFBUF) * P::kSfCols;  // this step's buffer
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          tc2_copy_sf(tsf + P::kSfaCol + 4 * j, desc_sf(sfa + 512 * j));
#pragma unroll
          for (int h = 0; h < P::kGroups; ++h)
            tc2_copy_sf(tsf + P::kSfbCol + 4 * (P::kGroups * j + h),
                        desc_sf(sfb + 2048 * h + 512 * j));
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
          tc2_mma(tmem, desc_sw128(st + 32 * j), desc_sw128(st + kABytes + 32 * j), P::kIdesc,
                  tsf + P::kSfaCol + 4 * j, tsf + P::kSfbCol + 4 * P::kGroups * j, (kt | j) != 0);
        tc2_commit(smem_u32(empty + s));
        tc2_commit(empty1 + 8 * s);
      }
      tc2_commit(smem_u32(done));  // also after giving up: both epilogues wait for issued MMAs
      tc2_commit(done1);
    }
    __syncwarp();
  }

  // ---------------- epilogue: this CTA's 128 rows x 256 columns ----------------
  __syncwarp();
  bool ok = true;
  if (lane == 0) {
    ok = mbar_wait<200>(smem_u32(done), 0, args.gen);
    if (!ok) *gave_up = 1;
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  tc_fence_after();
  if (__all_sync(0xffffffffu, ok && !*gave_up)) store_rows<PN>(tmem, warp, lane, m0, n0, args);
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *gave_up) {
    atomicAdd(&g_mm_gave_up, 1u);
    g_mm_abandon_gen = args.gen;
  }
  cluster_sync();  // neither CTA releases TMEM or exits while the pair still signals it
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(P::kTmemCols)
                 : "memory");
  }
}


// Map of one operand's codes: rows x (k / 2) bytes, row pitch k / 2, boxes of box_rows x 128
// bytes loaded with the 128-byte swizzle; rows past the end read as zero.
bool make_map(CUtensorMap* map, const uint8_t* codes, int64_t rows, int64_t k, int box_rows) {
  const tma::EncodeTiledFn enc = tma::encode_tiled();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)(k / 2), (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(k / 2)};
  const cuuint32_t box[2] = {(cuuint32_t)kRowBytes, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Map of a prepared scale array seen as rows of 256 bytes, boxes of 8 rows (one 2048-byte group).
bool make_rows_map(CUtensorMap* map, const uint8_t* scales, int64_t rows) {
  const tma::EncodeTiledFn enc = tma::encode_tiled();
  if (!enc) return false;
  const cuuint64_t dims[2] = {256, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {256};
  const cuuint32_t box[2] = {256, 8};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(scales), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


// ------------------------------------------------------------------------------------------------
// bf16 activations x stored FP4 weights: C = A dequant(W)^T (the inference step of the 4-bit float
// quantization article, gtnt.cn/news/16247, §3.1: the stored weights are dequantized to the
// activations' type, then multiplied).  W is n x k as mx_quantize stores it, with any block size
// N, E4M3 or UE5M3 scales ([MX] §3.1 item 1) and an FP16 global scale; the tensor core has no
// block-scaled form for UE5M3 or for most of these N, so each CTA dequantizes its tile of W into
// shared memory itself -- RN_bf16(E2M1 * S * g), the values mx_dequantize writes as bf16 -- and
// multiplies bf16 x bf16 with tcgen05.mma kind::f16 (fp32 accumulator in TMEM).  Nothing is
// dequantized to global memory: per element of W the kernel reads 1/2 + 1/N bytes.
//
// One CTA per 256 x 256 tile of C (two 128-row accumulators side by side in TMEM, 512 columns),
// 11 warps:
//   * warp 0, one thread: per 64-element step of k, TMA loads of the step's two 128 x 64 tiles of
//     A (128-byte swizzle), completing on the stage's A barrier;
//   * warp 10, one thread: TMA loads of the step's code bytes of the W tile (256 rows x 32 bytes)
//     into a ring of 4 code tiles, up to 4 steps ahead of their use;
//   * warps 2..9 (256 threads, one row of the W tile each): read the step's 32 code bytes from the
//     ring (every lane acquires the ring's barrier), take the 64 / N scale bytes loaded two steps
//     earlier, decode the codes (E2M1x2 -> f16x2), multiply by the block's S g (exact in fp32),
//     round to bf16 and write the 128-byte row into the stage's W tile in the same 128-byte-swizzled
//     K-major layout the TMA writes for A; then a proxy fence and one arrival per warp on the
//     stage's W barrier;
//   * warp 1, one thread: waits for both barriers, issues 4 (or 8) tcgen05.mma of 128 x 256 x 16,
//     commits to the stage's empty barrier;
//   * warps 2..9 then read the accumulators back (tcgen05.ld; warp w serves TMEM lanes 32 (w % 4)
//     of accumulator (w - 2) / 4) and store C.
// Every wait is bounded, as in the kernels above.
// ------------------------------------------------------------------------------------------------
namespace dqmm {
constexpr int kBN = 256;                      // columns of C per CTA (MMA N)
constexpr int kBK = 64;                       // k elements per stage
constexpr int kStages = 3;
constexpr int kATile = 128 * 128;             // one 128-row half of A: 128 x 64 bf16
constexpr int kABytes = 2 * kATile;
constexpr int kBBytes = kBN * 128;            // the W tile: 256 x 64 bf16
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kCStages = 4;                   // ring of the W tile's code bytes (TMA)
constexpr int kCBytes = kBN * (kBK / 2);      // 256 rows x 32 bytes
constexpr int kThreads = 352;  // warp 0: A, warp 1: MMA, warps 2..9: W, warp 10: W codes
constexpr int kDqWarps = 8;
constexpr int kSmemBytes = kStages * kStageBytes + kCStages * kCBytes + 256 * 4 + 256 + 1024;
static_assert(kSmemBytes <= 232448, "dynamic shared memory per CTA");
constexpr uint32_t kTmemCols = 512;
// Instruction descriptor of kind::f16: fp32 accumulator (bits 4..5 = 1), A and B bf16 (bits 7..9
// and 10..12 = 1), both K-major, N = 256 (bits 17..22: N / 8), M = 128 (bits 24..28: M / 16).
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) |
                            ((uint32_t)(128 >> 4) << 24);
static_assert(kStageBytes % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
}  // namespace dqmm

struct DqArgs {
  const uint8_t* w_packed;
  const uint8_t* w_scales;
  const uint16_t* g_dev;  // when set, the global scale is read here (device)
  void* c;
  int64_t m, n, k;
  uint32_t g_bits;
  int c_bf16;
  unsigned int gen;
};

__device__ __forceinline__ void tc_mma_f16(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void st_shared16(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                            uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// The scale bytes of one 64-element step of a row, packed little-endian (64 / N of them for
// N <= 64, the one covering the step otherwise).
template <int N>
struct StepScales {
  static constexpr int kBytes = N >= 64 ? 1 : 64 / N;
  uint32_t v[kBytes > 4 ? kBytes / 4 : 1];
};

template <int N>
__device__ __forceinline__ void load_scales(const uint8_t* srow, int kt, bool ok,
                                            StepScales<N>& sc) {
#pragma unroll
  for (int i = 0; i < (int)(sizeof(sc.v) / 4); ++i) sc.v[i] = 0;
  if (!ok) return;
  if constexpr (N == 4) {
    const uint4 t = __ldg(reinterpret_cast<const uint4*>(srow + 16 * (int64_t)kt));
    sc.v[0] = t.x; sc.v[1] = t.y; sc.v[2] = t.z; sc.v[3] = t.w;
  } else if constexpr (N == 8) {
    const uint2 t = __ldg(reinterpret_cast<const uint2*>(srow + 8 * (int64_t)kt));
    sc.v[0] = t.x; sc.v[1] = t.y;
  } else if constexpr (N == 16) {
    sc.v[0] = __ldg(reinterpret_cast<const unsigned int*>(srow + 4 * (int64_t)kt));
  } else if constexpr (N == 32) {
    sc.v[0] = __ldg(reinterpret_cast<const unsigned short*>(srow + 2 * (int64_t)kt));
  } else {
    sc.v[0] = __ldg(srow + (64 * (int64_t)kt) / N);
  }
}

// Scale byte of block b inside the step (b < 64 / N; 0 for N >= 64).
template <int N>
__device__ __forceinline__ uint32_t step_scale(const StepScales<N>& sc, int b) {
  if constexpr (N >= 64) return sc.v[0] & 0xFFu;
  else return (sc.v[b >> 2] >> (8 * (b & 3))) & 0xFFu;
}

// One code word (elements 8 w .. 8 w + 7 of the step) -> 8 bf16 = one 16-byte chunk of the row.
template <int N>
__device__ __forceinline__ void dq_word(uint32_t cw, int w, const StepScales<N>& sc,
                                        const float* s_D, uint32_t (&out)[4]) {
  uint32_t h[4];
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(cw));
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = 8 * w + 2 * i;  // element index in the step
    const float D = s_D[step_scale<N>(sc, N >= 64 ? 0 : e / N)];
    const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&h[i]));
    const float2 y = __fmul2_rn(v, make_float2(D, D));  // exact
    out[i] = pack_bf16x2(y.x, y.y);                    // round to nearest even
  }
}

template <int N, int FMT>
__global__ void __launch_bounds__(dqmm::kThreads, 1)
    k_dequant_matmul(const __grid_constant__ CUtensorMap tma_a,
                     const __grid_constant__ CUtensorMap tma_w, const __grid_constant__ DqArgs args) {
  using namespace dqmm;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* codes = smem + kStages * kStageBytes;  // kCStages code tiles
  float* s_D = reinterpret_cast<float*>(codes + kCStages * kCBytes);
  uint64_t* a_full = reinterpret_cast<uint64_t*>(s_D + 256);
  uint64_t* b_full = a_full + kStages;
  uint64_t* empty = b_full + kStages;
  uint64_t* c_full = empty + kStages;
  uint64_t* c_empty = c_full + kCStages;
  uint64_t* done = c_empty + kCStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* gave_up = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t NT = (args.n + kBN - 1) / kBN;  // tiles of C: n fastest (one 1-D grid)
  const int64_t m0 = ((int64_t)blockIdx.x / NT) * 256, n0 = ((int64_t)blockIdx.x % NT) * kBN;
  const bool two = m0 + 128 < args.m;  // the second 128-row half has rows
  const int KT = (int)(args.k / dqmm::kBK);
  const uint16_t gb = args.g_dev ? __ldg(args.g_dev) : (uint16_t)args.g_bits;
  const float g = fp16_bits_to_float(gb);
  for (int c = threadIdx.x; c < 256; c += blockDim.x) s_D[c] = __fmul_rn(scale_value(c, FMT), g);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(a_full + s), 1);
      mbar_init(smem_u32(b_full + s), kDqWarps);
      mbar_init(smem_u32(empty + s), 1);
    }
    for (int c = 0; c < kCStages; ++c) {
      mbar_init(smem_u32(c_full + c), 1);
      mbar_init(smem_u32(c_empty + c), kDqWarps);
    }
    mbar_init(smem_u32(done), 1);
    *gave_up = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 10) {
    // ---------------- code producer (one thread): the W tile's code bytes, kCStages ahead ----
    // (a warp of its own: two spinning producers in one warp need not both make progress)
    if (lane == 0) {
      int issued = 0;
      for (int kt = 0; kt < KT; ++kt) {
        const int c = kt % kCStages;
        if (*gave_up ||
            (kt >= kCStages && !mbar_wait<MX_MM_PROD_SLEEP>(smem_u32(c_empty + c),
                                                            ((kt / kCStages) + 1) & 1, args.gen))) {
          *gave_up = 1;
          break;
        }
        const uint32_t bar = smem_u32(c_full + c);
        mbar_expect_tx(bar, kCBytes);  // OOB rows included
        tma_load_2d(smem_u32(codes + c * kCBytes), &tma_w, kt * (dqmm::kBK / 2), (int)n0, bar);
        mbar_arrive(bar);
        issued = kt + 1;
      }
      if (*gave_up) {
        for (int kt = issued - kCStages < 0 ? 0 : issued - kCStages; kt < issued; ++kt)
          mbar_wait<100>(smem_u32(c_full + kt % kCStages), (kt / kCStages) & 1, args.gen);
      }
    }
    __syncwarp();
  } else if (warp == 0) {
    // ---------------- A producer (one thread) ----------------
    if (lane == 0) {
      int issued = 0;
      for (int kt = 0; kt < KT; ++kt) {
        const int s = kt % kStages;
        if (*gave_up ||
            (kt >= kStages && !mbar_wait<MX_MM_PROD_SLEEP>(smem_u32(empty + s),
                                                           ((kt / kStages) + 1) & 1, args.gen))) {
          *gave_up = 1;
          break;
        }
        const uint32_t st = smem_u32(smem + s * kStageBytes), bar = smem_u32(a_full + s);
        mbar_expect_tx(bar, two ? 2 * kATile : kATile);  // OOB rows included
        tma_load_2d(st, &tma_a, kt * dqmm::kBK, (int)m0, bar);
        if (two) tma_load_2d(st + kATile, &tma_a, kt * dqmm::kBK, (int)(m0 + 128), bar);
        mbar_arrive(bar);  // the barrier's one arrival; the phase completes when the bytes land
        issued = kt + 1;
      }
      if (*gave_up) {
        for (int kt = issued - kStages < 0 ? 0 : issued - kStages; kt < issued; ++kt)
          mbar_wait<100>(smem_u32(a_full + kt % kStages), (kt / kStages) & 1, args.gen);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer (one thread) ----------------
    if (lane == 0) {
      for (int kt = 0; kt < KT; ++kt) {
        const int s = kt % kStages;
        if (!mbar_wait(smem_u32(a_full + s), (kt / kStages) & 1, args.gen) ||
            !mbar_wait(smem_u32(b_full + s), (kt / kStages) & 1, args.gen)) {
          *gave_up = 1;
          break;
        }
        tc_fence_after();
        const uint32_t st = smem_u32(smem + s * kStageBytes), wt = st + kABytes;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t bdesc = desc_sw128(wt + 32 * j);
          tc_mma_f16(tmem, desc_sw128(st + 32 * j), bdesc, kIdesc, (kt | j) != 0);
          if (two) tc_mma_f16(tmem + 256, desc_sw128(st + kATile + 32 * j), bdesc, kIdesc,
                              (kt | j) != 0);
        }
        tc_commit(smem_u32(empty + s));
      }
      tc_commit(smem_u32(done));  // also after giving up: the epilogue waits for issued MMAs
    }
    __syncwarp();
  } else {
    // ---------------- W dequantization (warps 2..9, one row of the tile per thread) ----------
    // codes from the TMA ring (row d at byte 32 d of a code tile), scales by plain loads two steps
    // ahead
    const int d = threadIdx.x - 64;
    const int64_t row = n0 + d;
    const bool row_ok = row < args.n;
    const uint8_t* srow = args.w_scales + (row_ok ? row : 0) * (args.k / N);
    const uint32_t r8 = (uint32_t)(d & 7);
    const uint32_t row_off = (uint32_t)(d >> 3) * 1024u + r8 * 128u;
    StepScales<N> sc0, sc1;
    load_scales<N>(srow, 0, row_ok && 0 < KT, sc0);
    load_scales<N>(srow, 1, row_ok && 1 < KT, sc1);
    for (int kt = 0; kt < KT; ++kt) {
      const int s = kt % kStages, c = kt % kCStages;
      StepScales<N> sc2;
      load_scales<N>(srow, kt + 2, row_ok && kt + 2 < KT, sc2);
      // every lane that reads the tile acquires the barrier the TMA completes
      bool ok = !*gave_up && mbar_wait(smem_u32(c_full + c), (kt / kCStages) & 1, args.gen);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        *gave_up = 1;
        break;
      }
      uint4 c0, c1;
      const uint32_t caddr = smem_u32(codes + c * kCBytes) + 32u * (uint32_t)d;
      asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(c0.x), "=r"(c0.y), "=r"(c0.z), "=r"(c0.w) : "r"(caddr) : "memory");
      asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(c1.x), "=r"(c1.y), "=r"(c1.z), "=r"(c1.w) : "r"(caddr + 16u) : "memory");
      if (kt >= kStages && lane == 0)
        ok = mbar_wait<MX_MM_PROD_SLEEP>(smem_u32(empty + s), ((kt / kStages) + 1) & 1, args.gen);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        *gave_up = 1;
        break;
      }
      const uint32_t base = smem_u32(smem + s * kStageBytes + kABytes) + row_off;
      const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        uint32_t o[4];
        dq_word<N>(cw[w], w, sc0, s_D, o);
        st_shared16(base + (((uint32_t)w ^ r8) << 4), o[0], o[1], o[2], o[3]);
      }
      // the tensor core reads this tile through the async proxy
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(b_full + s));
        // the code tile's slot is released only now that every lane has used the values it read
        // (released right after the loads were issued, the next TMA into the slot was measured
        // to overwrite codes some lanes had not read yet)
        mbar_arrive(smem_u32(c_empty + c));
      }
      sc0 = sc1;
      sc1 = sc2;
    }
  }

  // ---------------- epilogue: warps 2..9 ----------------
  if (warp >= 2 && warp <= 9) {
    const int q = warp & 3, h = (warp - 2) >> 2;
    bool ok = true;
    if (lane == 0) {
      ok = mbar_wait<200>(smem_u32(done), 0, args.gen);
      if (!ok) *gave_up = 1;
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    tc_fence_after();
    if (__all_sync(0xffffffffu, ok && !*gave_up) && (h == 0 || two)) {
      MmArgs ea{nullptr, nullptr, args.c, args.m, args.n, args.k, 1.0f, args.c_bf16, args.gen};
      store_rows<kBN>(tmem + (uint32_t)(256 * h), q, lane, m0 + 128 * h, n0, ea);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *gave_up) {
    atomicAdd(&g_mm_gave_up, 1u);
    g_mm_abandon_gen = args.gen;
  }
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// Map of the weights' codes: n rows of k / 2 bytes, boxes of 256 rows x 32 bytes (one 64-element
// step), no swizzle; rows past the end read as zero.
bool make_codes_map(CUtensorMap* map, const uint8_t* codes, int64_t n, int64_t k) {
  const tma::EncodeTiledFn enc = tma::encode_tiled();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)(k / 2), (cuuint64_t)n};
  const cuuint64_t strides[1] = {(cuuint64_t)(k / 2)};
  const cuuint32_t box[2] = {(cuuint32_t)(dqmm::kBK / 2), (cuuint32_t)dqmm::kBN};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Map of the bf16 activations: m x k, row pitch 2 k bytes, boxes of 128 rows x 64 elements loaded
// with the 128-byte swizzle; rows past the end read as zero.
bool make_bf16_map(CUtensorMap* map, const void* a, int64_t m, int64_t k) {
  const tma::EncodeTiledFn enc = tma::encode_tiled();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)k, (cuuint64_t)m};
  const cuuint64_t strides[1] = {(cuuint64_t)(2 * k)};
  const cuuint32_t box[2] = {(cuuint32_t)dqmm::kBK, 128};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace

int64_t mma_scales_bytes(int64_t rows, int64_t k);

// Dynamic shared memory above 48 KiB is enabled per kernel and per device (allow_dynamic_smem).
static std::atomic<bool> g_smem_one[kMaxDevices], g_smem_pair[kMaxDevices];
static std::atomic<unsigned int> g_launch_gen{0};


// A new generation number for a launch (never 0, the flag's initial value).
static unsigned int next_gen() {
  unsigned int g = g_launch_gen.fetch_add(1u) + 1u;
  if (g == 0) g = g_launch_gen.fetch_add(1u) + 1u;
  return g;
}

cudaError_t run_matmul_nvfp4(const uint8_t* a_packed, const uint8_t* a_scales,
                             const uint8_t* b_packed, const uint8_t* b_scales, int64_t m,
                             int64_t n, int64_t k, float alpha, void* c, bool c_bf16,
                             bool cta_pairs, cudaStream_t stream, int* launches) {
  MmArgs args{a_scales, b_scales, c, m, n, k, alpha, c_bf16 ? 1 : 0, next_gen()};
  CUtensorMap ma, mb;
  if (m > kBM && cta_pairs) {
    // CTA pairs: 256 x 256 tiles of C
    cudaError_t e = allow_dynamic_smem(g_smem_pair, k_matmul_nvfp4_pair, Pair::kSmemBytes);
    if (e != cudaSuccess) return e;
    CUtensorMap msa, msb;
    if (!make_map(&ma, a_packed, m, k, kBM) || !make_map(&mb, b_packed, n, k, Pair::kBRows) ||
        !make_rows_map(&msa, a_scales, mma_scales_bytes(m, k) / 256) ||
        !make_rows_map(&msb, b_scales, mma_scales_bytes(n, k) / 256))
      return cudaErrorInvalidValue;
    const int64_t pairs = ((m + 255) / 256) * ((n + MX_MM_PAIR_N - 1) / MX_MM_PAIR_N);
    k_matmul_nvfp4_pair<<<(unsigned)(2 * pairs), 128, Pair::kSmemBytes, stream>>>(ma, mb, msa, msb,
                                                                                 args);
  } else {
    constexpr int BN = MX_MM_BN;
    static_assert(BN == 128 || BN == 256, "tile width");
    using T = Tile<BN>;
    cudaError_t e = allow_dynamic_smem(g_smem_one, k_matmul_nvfp4<BN>, T::kSmemBytes);
    if (e != cudaSuccess) return e;
    if (!make_map(&ma, a_packed, m, k, kBM) || !make_map(&mb, b_packed, n, k, BN))
      return cudaErrorInvalidValue;
    const dim3 grid((unsigned)((n + BN - 1) / BN), (unsigned)((m + kBM - 1) / kBM));
    k_matmul_nvfp4<BN><<<grid, 128, T::kSmemBytes, stream>>>(ma, mb, args);
  }
  ++*launches;
  return cudaGetLastError();
}

template <int N, int FMT>
static cudaError_t launch_dqmm(const CUtensorMap& ma, const CUtensorMap& mw, const DqArgs& args,
                               cudaStream_t stream) {
  static std::atomic<bool> attr[kMaxDevices];
  const cudaError_t e = allow_dynamic_smem(attr, k_dequant_matmul<N, FMT>, dqmm::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int64_t tiles = ((args.n + dqmm::kBN - 1) / dqmm::kBN) * ((args.m + 255) / 256);
  if (tiles >= (int64_t(1) << 31)) return cudaErrorInvalidConfiguration;
  k_dequant_matmul<N, FMT><<<(unsigned)tiles, dqmm::kThreads, dqmm::kSmemBytes, stream>>>(ma, mw,
                                                                                        args);
  return cudaGetLastError();
}

template <int FMT>
static cudaError_t dqmm_block(int block, const CUtensorMap& ma, const CUtensorMap& mw,
                              const DqArgs& args, cudaStream_t st) {
  switch (block) {
    case 4: return launch_dqmm<4, FMT>(ma, mw, args, st);
    case 8: return launch_dqmm<8, FMT>(ma, mw, args, st);
    case 16: return launch_dqmm<16, FMT>(ma, mw, args, st);
    case 32: return launch_dqmm<32, FMT>(ma, mw, args, st);
    case 64: return launch_dqmm<64, FMT>(ma, mw, args, st);
    case 128: return launch_dqmm<128, FMT>(ma, mw, args, st);
    default: return launch_dqmm<256, FMT>(ma, mw, args, st);
  }
}

cudaError_t run_dequant_matmul(const void* a, int64_t m, int64_t k, const uint8_t* w_packed,
                               const uint8_t* w_scales, int64_t n, int block, int fmt,
                               uint16_t g_bits, const uint16_t* g_dev, void* c, bool c_bf16,
                               cudaStream_t stream, int* launches) {
  CUtensorMap ma, mw;
  if (!make_bf16_map(&ma, a, m, k) || !make_codes_map(&mw, w_packed, n, k))
    return cudaErrorInvalidValue;
  const DqArgs args{w_packed, w_scales, g_dev, c, m, n, k, g_bits, c_bf16 ? 1 : 0, next_gen()};
  const cudaError_t e = fmt == kUE5M3 ? dqmm_block<kUE5M3>(block, ma, mw, args, stream)
                                      : dqmm_block<kE4M3>(block, ma, mw, args, stream);
  if (e == cudaSuccess) ++*launches;
  return e;
}

int64_t mma_scales_bytes(int64_t rows, int64_t k) {
  return 2 * ((rows + 2 * kBM - 1) / (2 * kBM)) * kBM * (k / 16);
}

cudaError_t run_scales_to_mma(const uint8_t* scales, int64_t rows, int64_t k, uint8_t* out,
                              cudaStream_t stream, int* launches) {
  const int64_t threads = mma_scales_bytes(rows, k) / 64;  // 64 bytes written per thread
  const int64_t blocks = (threads + 255) / 256;
  k_scales_to_mma<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, stream>>>(scales, rows, k,
                                                                                  out);
  ++*launches;
  return cudaGetLastError();
}

cudaError_t matmul_gave_up(unsigned int* count) {
  const unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(count, g_mm_gave_up, sizeof(unsigned int));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_mm_gave_up, &zero, sizeof(unsigned int));
  return e;
}

cudaError_t matmul_abandon_last() {
  const unsigned int gen = g_launch_gen.load();
  return cudaMemcpyToSymbol(g_mm_abandon_gen, &gen, sizeof(unsigned int));
}

}  // namespace mxk
