// mx_error_stats.cu -- three-term block-error reduction, alone or fused with quantize + pack.
//
// Method: the microscaling article (hotelren.com/news/2192771) §2.2 items 1-3.  Per block with a
// non-zero scale: the max element (first index of max|x|) contributes (x - y)^2 to SSE_max (the
// scale-rounding error of item 2), every other element to SSE_elem (item 1).  A block whose scale
// is zero contributes sum x^2 to SSE_zero (item 3).  y is the exact E2M1 * S * g.
//
// Main pass: persistent grid; each thread walks items of 8, 16 or 32 elements with the next item's
// loads issued before the current item's arithmetic.  The codes are read (kGiven), recomputed in
// registers with the quantize rule (kRecompute), or recomputed and stored (kStore: the fused
// quantize + pack + reduction pass, x read once).  Blocks of 4, 8 and 16 with recomputed codes run
// on k_qstats_small (block pairs, per-item sums; see there), everything else on k_error_stats_bf16
// (bf16) or k_error_stats_f32.  Per block slice held by a lane of k_error_stats_bf16:
//   * Scaling.  s = 2^k brings the block maximum a into [1, 2).  d' = x s - code * (S g s) is one
//     FMA (the code's bits are its value times 2^-126; S g s 2^126 is a per-block constant) and
//     exact; squares are summed in fp32 (at most 32 terms) and scaled back exactly in double.
//   * Recomputed codes (blocks of 32 and more): every element's square goes into the slice sum;
//     all max-valued elements of a block share one error dmax, computed once per block, and the
//     lane holding the block's first max element moves dmax^2 to SSE_max (slice_finish_closed).
//     Clipped elements (|x| > 6 S g) are counted with one bf16x2 compare per word.
//   * Stored codes: two bf16x2 compares per word, |x| >= a (the max-valued elements, whose codes
//     may differ) and |x| > 6 S g; the max-valued squares are summed apart, and a lane holding a
//     tie of the maximum redoes them in double.  The block's first max element (lowest lane,
//     lowest index) goes to SSE_max, everything else to SSE_elem.
//   * Underflow.  A slice whose scaled sum is below 2^-80 (squares below 2^-126 could be lost),
//     or whose stored scale is far from a, redoes its slice in double.
// Final sum: the CTA that finishes last (one atomic counter per launch) adds the per-CTA partials
// in a fixed order, so results are deterministic for a given device and grid; with a tail (N <= 16) a
// separate one-CTA pass does it.  No CTA waits on another.
#include "mx_device.cuh"
#include "mx_launch.h"

// Item shape (compile-time; the defaults are the tuned values).
#ifndef MX_ST_EPT_BF16
#define MX_ST_EPT_BF16 32
#endif
#ifndef MX_ST_U
#define MX_ST_U 1
#endif
#ifndef MX_ST_MINB  // minimum resident CTAs per SM for the bf16 pass (register cap)
#define MX_ST_MINB 2
#endif
#ifndef MX_ST_EPT_SMALL  // elements per item of the bf16 pass for N <= 8 (a multiple of 8)
#define MX_ST_EPT_SMALL 16
#endif
#ifndef MX_ST_MINB_SMALL  // the same for N <= 8 (short per-block work: more warps hide the latency)
#define MX_ST_MINB_SMALL 3
#endif
#ifndef MX_QS_MINB  // the same for the small-block kernel with recomputed codes
#define MX_QS_MINB 2
#endif

namespace mxk {

struct StatsOut {  // layout of mx_error_stats_t
  double sse_elem, sse_max, sse_zero;
  long long numel, n_blocks, n_zero_blocks, n_scale_sat, n_elem_sat;
};

template <int N, typename T>
struct SShape {
  static constexpr int EPT = sizeof(T) != 2 ? 8
                             : N >= 16 ? (N < MX_ST_EPT_BF16 ? N : MX_ST_EPT_BF16)
                                       : MX_ST_EPT_SMALL;
  static constexpr int L = (N >= EPT) ? N / EPT : 1;
  static constexpr int BPI = (N >= EPT) ? 1 : EPT / N;
  static constexpr int U = (sizeof(T) == 2) ? MX_ST_U : 1;
};

struct Acc {
  double elem = 0.0, mx = 0.0, zero = 0.0;
  unsigned n_zero = 0, n_ssat = 0;
  float n_esat = 0.0f;  // clipped elements (exact: a thread sees far fewer than 2^24)
  float n_zero_f = 0.0f, n_ssat_f = 0.0f;  // the same counts kept in fp32 (small-block kernel)
};

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ unsigned long long warp_sum(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// CTA-wide reduction of the accumulators into *slot (fixed order).
__device__ void write_partial(const Acc& acc, StatsPartial* slot) {
  __shared__ double sd[3][kThreads / 32];
  __shared__ unsigned long long su[3][kThreads / 32];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const double a0 = warp_sum(acc.elem), a1 = warp_sum(acc.mx), a2 = warp_sum(acc.zero);
  const unsigned long long c0 = warp_sum((unsigned long long)acc.n_zero +
                                         (unsigned long long)acc.n_zero_f);
  const unsigned long long c1 = warp_sum((unsigned long long)acc.n_ssat +
                                         (unsigned long long)acc.n_ssat_f);
  const unsigned long long c2 = warp_sum((unsigned long long)acc.n_esat);
  if (lane == 0) {
    sd[0][w] = a0; sd[1][w] = a1; sd[2][w] = a2;
    su[0][w] = c0; su[1][w] = c1; su[2][w] = c2;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    StatsPartial p{};
    for (int k = 0; k < kThreads / 32; ++k) {
      p.sse_elem += sd[0][k]; p.sse_max += sd[1][k]; p.sse_zero += sd[2][k];
      p.n_zero_blocks += su[0][k]; p.n_scale_sat += su[1][k]; p.n_elem_sat += su[2][k];
    }
    *slot = p;
  }
}

// One tensor of a grouped error-reduction launch, and the grid split among the tensors.
struct STensor {
  const void* x;
  const uint8_t* packed;   // stored codes (kGiven)
  const uint8_t* scales;
  uint8_t* packed_out;     // codes written (kStore)
  uint8_t* scales_out;
  StatsPartial* part;      // this tensor's CTAs' partials: part[0 .. its CTA count)
  unsigned int* counter;   // last-CTA counter, zeroed before the launch; nullptr: a separate pass
                           // adds the partials (a tail, N <= 16)
  StatsOut* out;
  int64_t nitems, numel, nblocks;
  uint32_t g_bits;
  const uint16_t* g_dev;   // g in device memory (written by the previous kernel) when set
  // Row-pitched mode (rows whose length cols the block size does not divide): ipr items per row,
  // the row's blocks rounded up to whole items (the last ones hold zeros past the row's end); row
  // pitches of x (cols elements), codes (pb bytes) and scales (nb bytes).
  int64_t cols, ipr, pb, nb;
};
struct SGroup {
  STensor t[kMaxGroup];
  CtaSplit split;
};

// This CTA's tensor, its index among the tensor's CTAs and their number.
struct SWork {
  STensor t;
  int cta, nctas;
};
__device__ __forceinline__ SWork s_work(const SGroup& grp) {
  const int ti = grp.split.find((int)blockIdx.x);
  return {grp.t[ti], (int)blockIdx.x - grp.split.begin[ti],
          grp.split.begin[ti + 1] - grp.split.begin[ti]};
}

__device__ void final_reduce(const StatsPartial* part, int nparts, const StatsPartial* extra,
                             int64_t numel, int64_t nblocks, StatsOut* out);

// Writes this CTA's partial; the tensor's CTA that finishes last (counted with one atomic per CTA
// after a fence) then adds the tensor's partials in a fixed order and resets the counter.  No CTA
// waits for another.
__device__ void finish_cta(const Acc& acc, const SWork& wk) {
  write_partial(acc, wk.t.part + wk.cta);
  if (wk.t.counter == nullptr) return;
  __shared__ unsigned int s_last;
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(wk.t.counter, 1u) == (unsigned)wk.nctas - 1u;
  }
  __syncthreads();
  if (s_last) {
    __threadfence();
    final_reduce(wk.t.part, wk.nctas, nullptr, wk.t.numel, wk.t.nblocks, wk.t.out);
    if (threadIdx.x == 0) *wk.t.counter = 0;
  }
}

// v * 2^(2E - 254) in double for a non-negative fp32 v that is zero or normal, built with integer
// operations: the fp32 exponent and mantissa move into the double's fields and the block's scale
// factor is added to the exponent (no conversion or double multiply instructions).
__device__ __forceinline__ double scaled_to_double(float v, int E) {
  const uint32_t b = __float_as_uint(v);
  const uint32_t hi = (b >> 3) + ((uint32_t)(642 + 2 * E) << 20);
  const uint32_t lo = b << 29;
  return b ? __hiloint2double((int)hi, (int)lo) : 0.0;
}

// Per-block constants of one block slice (see the file comment for the scaling).
struct SliceSetup {
  int E;           // biased exponent of the block maximum a, clamped to [1, 253]
  float sc;        // 2^(127 - E), a normal number: a * sc in [1, 2) (in [2, 4) for the top
                   // binade, where the clamp keeps sc normal: the mixed-precision FMAs that
                   // apply it take it as a bf16 operand, and a subnormal one would be lost)
  float sat6s;     // 6 S g sc, the scaled clip level
  float nDq;       // -S g sc 2^126: one FMA with a code's bits gives -y sc
  float tiny;      // a 2^-30: below it a scaled square could lose digits
  bool zero_blk;   // S == 0
  bool scale_ok;   // S g sc in [2^-30, 2] (always true for recomputed codes)
};

__device__ __forceinline__ SliceSetup slice_setup(float a, float D) {
  SliceSetup st;
  st.E = min(max((int)((__float_as_uint(a) >> 23) & 0xFFu), 1), 253);
  st.sc = __uint_as_float((uint32_t)(254 - st.E) << 23);
  const float Ds = __fmul_rn(D, st.sc);
  st.sat6s = __fmul_rn(6.0f, Ds);
  st.nDq = -__fmul_rn(Ds, 0x1p126f);
  st.tiny = __fmul_rn(a, 0x1p-30f);
  st.zero_blk = !(D > 0.0f);
  st.scale_ok = st.zero_blk || (Ds <= 2.0f && Ds >= 0x1p-30f);
  return st;
}

// Core of a bf16 block slice, one word (two elements) at a time, in PTX so that every step is one
// instruction: scaled values (f32x2 multiply), scaled errors (f32x2 FMA with the code bits),
// |x| >= a and |x| > 6 S g as bf16x2 compares (x is bf16, so |x| > 6 S g holds exactly when |x| is
// above 6 S g rounded down to bf16), predicated sums and counters (fp32 adds: the counters stay
// exact and the integer pipe stays free for the decode).  MS: also sum the squares of the
// max-valued elements (stored codes); with recomputed codes their error is known per block.
//   w: the word, lo / hi: its elements as fp32 bits; cw: the code word holding the word's code
//   byte at byte J; A2 = {a, a}, S2 = {RD(6 S g), same} as bf16x2.  The left shifts are written as
//   multiplies by 2^k.
template <int J, bool MS>
__device__ __forceinline__ void pair_step(uint32_t w, uint32_t lo, uint32_t hi, uint32_t cw,
                                          float sc, float nDq, uint32_t A2, uint32_t S2, float& lt,
                                          float& ms, float& cnt, float& nsat) {
  static_assert(J >= 0 && J < 4, "byte index");
  // The decode of code byte J is bit arithmetic: each code's bits become its value times 2^-126
  // (sign to bit 31, exponent and mantissa to bits 24..22), and %7 is -S g s 2^126.  (The
  // E2M1x2 -> f16x2 conversion instruction was tried instead and gave wrong values for some
  // inputs when its byte came straight from the encoding conversion in registers.)
#define MX_PAIR_HEAD                            \
  "{\n\t"                                      \
  ".reg .b32 blo, bhi, aw, t;\n\t"             \
  ".reg .b64 x2, s2, b2, q2, d2;\n\t"          \
  ".reg .f32 dlo, dhi;\n\t"                    \
  ".reg .pred pl, ph, ql, qh;\n\t"             \
  "mov.b64 x2, {%12, %13};\n\t"                \
  "mov.b64 s2, {%6, %6};\n\t"                  \
  "mul.rn.f32x2 x2, x2, s2;\n\t"               \
  "mul.lo.u32 t, %5, %10;\n\t"                 \
  "shr.s32 t, t, 6;\n\t"                       \
  "and.b32 blo, t, 0x81c00000;\n\t"            \
  "mul.lo.u32 t, %5, %11;\n\t"                 \
  "shr.s32 t, t, 6;\n\t"                       \
  "and.b32 bhi, t, 0x81c00000;\n\t"            \
  "mov.b64 b2, {blo, bhi};\n\t"                \
  "mov.b64 q2, {%7, %7};\n\t"                  \
  "fma.rn.f32x2 d2, b2, q2, x2;\n\t"           \
  "mov.b64 {dlo, dhi}, d2;\n\t"                \
  "and.b32 aw, %4, 0x7fff7fff;\n\t"            \
  "setp.ge.bf16x2 pl|ph, aw, %8;\n\t"          \
  "setp.gt.bf16x2 ql|qh, aw, %9;\n\t"          \
  "@!pl fma.rn.f32 %0, dlo, dlo, %0;\n\t"      \
  "@!ph fma.rn.f32 %0, dhi, dhi, %0;\n\t"
#define MX_PAIR_TAIL                            \
  "@pl add.f32 %2, %2, 0f3F800000;\n\t"        \
  "@ph add.f32 %2, %2, 0f3F800000;\n\t"        \
  "@ql add.f32 %3, %3, 0f3F800000;\n\t"        \
  "@qh add.f32 %3, %3, 0f3F800000;\n\t"        \
  "}"
  if constexpr (MS) {
    asm(MX_PAIR_HEAD
        "@pl fma.rn.f32 %1, dlo, dlo, %1;\n\t"
        "@ph fma.rn.f32 %1, dhi, dhi, %1;\n\t" MX_PAIR_TAIL
        : "+f"(lt), "+f"(ms), "+f"(cnt), "+f"(nsat)
        : "r"(w), "r"(cw), "f"(sc), "f"(nDq), "r"(A2), "r"(S2), "n"(1u << (28 - 8 * J)),
          "n"(1u << (24 - 8 * J)), "r"(lo), "r"(hi));
  } else {
    asm(MX_PAIR_HEAD MX_PAIR_TAIL
        : "+f"(lt), "+f"(ms), "+f"(cnt), "+f"(nsat)
        : "r"(w), "r"(cw), "f"(sc), "f"(nDq), "r"(A2), "r"(S2), "n"(1u << (28 - 8 * J)),
          "n"(1u << (24 - 8 * J)), "r"(lo), "r"(hi));
  }
#undef MX_PAIR_HEAD
#undef MX_PAIR_TAIL
}

// Error step of one word (two elements) whose codes were computed beforehand (the signed form of
// qs_word8's error part, used where the codes of a whole item are converted first): every
// element's scaled error d goes into the f32x2 sum of squares lt2 -- the max-valued ones included,
// the first of them is taken out per block, see slice_finish_closed -- and the clipped elements
// (|x| above S2 = RD_bf16(6 S g)) are counted per half in nsat2 as bf16x2 integers.
template <int J>
__device__ __forceinline__ void pair_step_all(uint32_t w, uint32_t lo, uint32_t hi, uint32_t cw,
                                              float sc, float nDq, uint32_t S2,
                                              unsigned long long& lt2, uint32_t& nsat2) {
  static_assert(J >= 0 && J < 4, "byte index");
  asm("{\n\t"
      ".reg .b32 blo, bhi, aw, t, m;\n\t"
      ".reg .b64 x2, s2, b2, q2, d2;\n\t"
      "mov.b64 x2, {%8, %9};\n\t"
      "mov.b64 s2, {%3, %3};\n\t"
      "mul.rn.f32x2 x2, x2, s2;\n\t"
      "mul.lo.u32 t, %2, %6;\n\t"
      "shr.s32 t, t, 6;\n\t"
      "and.b32 blo, t, 0x81c00000;\n\t"
      "mul.lo.u32 t, %2, %7;\n\t"
      "shr.s32 t, t, 6;\n\t"
      "and.b32 bhi, t, 0x81c00000;\n\t"
      "mov.b64 b2, {blo, bhi};\n\t"
      "mov.b64 q2, {%4, %4};\n\t"
      "fma.rn.f32x2 d2, b2, q2, x2;\n\t"
      "fma.rn.f32x2 %0, d2, d2, %0;\n\t"
      "and.b32 aw, %10, 0x7fff7fff;\n\t"
      "set.gt.bf16x2.bf16x2 m, aw, %5;\n\t"
      "add.rn.bf16x2 %1, %1, m;\n\t"
      "}"
      : "+l"(lt2), "+r"(nsat2)
      : "r"(cw), "f"(sc), "f"(nDq), "r"(S2), "n"(1u << (28 - 8 * J)), "n"(1u << (24 - 8 * J)),
        "r"(lo), "r"(hi), "r"(w));
}

// |x| s for the two bf16 halves of aw, s a power of two given as its bf16 bit pattern sc16: two
// mixed-precision FMAs (bf16 operands, fp32 result) take the halves straight from the word, so the
// word needs no split into two fp32 values first.  Exact (a power-of-two scaling of a bf16 value).
__device__ __forceinline__ float2 mag_scaled2(uint32_t aw, uint32_t sc16) {
  float lo, hi;
  asm("{\n\t.reg .b16 l, h, s;\n\t"
      "mov.b32 {l, h}, %2;\n\t"
      "cvt.u16.u32 s, %3;\n\t"
      "fma.rn.f32.bf16 %0, l, s, 0f00000000;\n\t"
      "fma.rn.f32.bf16 %1, h, s, 0f00000000;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(aw), "r"(sc16));
  return make_float2(lo, hi);
}

// Code word of four bf16 words w0..w3 from their magnitude codes cm (byte k: word k's two codes,
// sign bits clear): each code takes its element's sign bit.  Per word, bytes 1 and 3 (the halves'
// high bytes) with their sign bit replicated over the byte (prmt selector nibbles with the top bit
// set), then regrouped so that byte k of hs / ls holds the sign of word k's high / low half.
__device__ __forceinline__ uint32_t put_signs(uint32_t cm, uint32_t w0, uint32_t w1, uint32_t w2,
                                              uint32_t w3) {
  uint32_t x01, x23, hs, ls;
  asm("prmt.b32 %0, %1, %2, 0xFDB9;" : "=r"(x01) : "r"(w0), "r"(w1));
  asm("prmt.b32 %0, %1, %2, 0xFDB9;" : "=r"(x23) : "r"(w2), "r"(w3));
  asm("prmt.b32 %0, %1, %2, 0x7531;" : "=r"(hs) : "r"(x01), "r"(x23));
  asm("prmt.b32 %0, %1, %2, 0x6420;" : "=r"(ls) : "r"(x01), "r"(x23));
  return (cm | (hs & 0x80808080u)) | (ls & 0x08080808u);
}

// One code word's eight elements (words w[0..3], all in one block) with recomputed codes,
// quantized and reduced in one go.  The scaled magnitudes xs = |x| s (s = 2^k, the slice scaling)
// come straight from the bf16 words (mag_scaled2).  The quotients are taken of them with the
// rescaled reciprocal r / s (x r = xs (r / s) exactly: s is a power of two), rounded onto the
// 2^-18 grid by adding and subtracting 48 (see snap_quotient2; a magnitude needs no sign fix for
// zero), so the E2M1 conversion gives magnitude codes whose decode is one shift and one mask; x's
// sign bits are put into the codes afterwards (byte permutes that replicate each half's sign, two
// masked ORs).  Errors use the magnitudes too: (xs - |q| S g s)^2 is the element's scaled square.
// A block far beyond its saturation (S g s below 2^-64: possible only with a caller's g far below
// the tensor's) would overflow r / s; for it the quotients are taken of the unscaled |x| with r,
// from the fp32 split of the words.  MODE says how that case is found: kFast / kDeep when the
// caller has decided it for the whole item (deep_item), kCheck per call (where two inlined copies
// of the item's work would cost registers).  r, nDq, S2: the block's reciprocal, -S g s 2^126 and
// clip level RD_bf16(6 S g) (twice); lt2 collects the squares, nsat2 the clipped elements.
enum QsMode { kFast = 0, kDeep = 1, kCheck = 2 };
template <int PB, int MODE>
__device__ __forceinline__ uint32_t qs_word8(const uint32_t* w, const float* r, const float* nDq,
                                              const uint32_t* S2, float sc, float2* lt2,
                                              uint32_t& nsat2) {
  static_assert(PB == 4, "the code word's four words lie in one block");
  uint32_t aw[4];
  float2 xs[4];
  float q[8];
  const uint32_t sc16 = __float_as_uint(sc) >> 16;  // a power of two: exact as a bf16
  const float rs = __fmul_rn(r[0], __frcp_rn(sc));  // r / s, exact unless it overflows
  const bool deep = MODE == kDeep || (MODE == kCheck && !(rs <= 0x1p64f));
#pragma unroll
  for (int k = 0; k < 4; ++k) aw[k] = w[k] & 0x7FFF7FFFu;
  if (!deep) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      xs[k] = mag_scaled2(aw[k], sc16);
      const float2 y = __ffma2_rn(xs[k], make_float2(rs, rs), make_float2(48.0f, 48.0f));
      const float2 qq = __fadd2_rn(y, make_float2(-48.0f, -48.0f));
      q[2 * k] = qq.x;
      q[2 * k + 1] = qq.y;
    }
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 xa = make_float2(__uint_as_float(aw[k] << 16),
                                    __uint_as_float(aw[k] & 0xFFFF0000u));
      xs[k] = __fmul2_rn(xa, make_float2(sc, sc));
      const float2 y = __ffma2_rn(xa, make_float2(r[0], r[0]), make_float2(48.0f, 48.0f));
      const float2 qq = __fadd2_rn(y, make_float2(-48.0f, -48.0f));
      q[2 * k] = qq.x;
      q[2 * k + 1] = qq.y;
    }
  }
  const uint32_t cm = cvt_e2m1x8(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    // magnitude bits of byte k's two codes moved to bits 22..24: the value times 2^-126
    const uint32_t blo = (k < 3 ? cm << (22 - 8 * k) : cm >> 2) & 0x01C00000u;
    const uint32_t bhi = (k < 3 ? cm << (18 - 8 * k) : cm >> 6) & 0x01C00000u;
    const float nd = nDq[k / PB];
    const float2 d = __ffma2_rn(make_float2(__uint_as_float(blo), __uint_as_float(bhi)),
                                make_float2(nd, nd), xs[k]);
    lt2[k / PB] = __ffma2_rn(d, d, lt2[k / PB]);
    uint32_t m;
    asm("set.gt.bf16x2.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(aw[k]), "r"(S2[k / PB]));
    asm("add.rn.bf16x2 %0, %0, %1;" : "+r"(nsat2) : "r"(m));
  }
  return put_signs(cm, w[0], w[1], w[2], w[3]);
}

// True when one of the blocks (reciprocals r[0..nb)) is so far beyond its saturation that r / s
// would overflow (see qs_word8): the item then takes the unscaled quotients.
template <int NBL>
__device__ __forceinline__ bool deep_item(const float* r, float sc) {
  float mr = r[0];
#pragma unroll
  for (int b = 1; b < NBL; ++b) mr = fmaxf(mr, r[b]);
  return __fmul_rn(mr, __frcp_rn(sc)) > 0x1p64f;
}

// One E2M1 conversion of two values: the code of lo in bits 0..3, of hi in bits 4..7.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float hi, float lo) {
  uint32_t r;
  asm("{\n\t.reg .b8 b;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\t"
      "cvt.u32.u8 %0, b;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

// Tail of a block slice: lt / ms are the scaled squares of the other / the max-valued elements,
// cnt the number of max-valued elements, nsat the clipped elements.  xval(k) / code(k) (k a
// compile-time constant) serve the exact path: ties of the maximum in this lane, or a slice that
// could lose digits to fp32 underflow.
template <int NE, int L, typename XF, typename CF>
__device__ __forceinline__ void slice_finish(Acc& acc, int lane, bool ok, float a, float D,
                                             float sat_thr, bool exact, const SliceSetup& st,
                                             float lt, float ms, float cnt, float nsat,
                                             XF xval, CF code) {
  if (!ok) cnt = nsat = 0.0f;
  const bool has_max = cnt != 0.0f;
  exact |= !st.scale_ok;
  double lt_d, first, others = 0.0;
  if (!exact && cnt <= 1.0f) {
    // common case: at most one max-valued element in this lane
    lt_d = scaled_to_double(lt, st.E);
    first = scaled_to_double(ms, st.E);
  } else {
    // ties of the maximum or the exact path: every element in double, lowest max apart
    lt_d = first = 0.0;
    bool seen = false;
#pragma unroll
    for (int k = 0; k < NE; ++k) {
      const float y = __fmul_rn(e2m1_to_float(code(k)), D);  // exact
      const double dd = (double)xval(k) - (double)y;          // exact
      const double e2 = dd * dd;
      if (fabsf(xval(k)) != a) {
        lt_d += e2;
      } else if (!seen) {
        first = e2;
        seen = true;
      } else {
        others += e2;
      }
    }
  }
  bool is_first_lane = has_max;
  if constexpr (L > 1) {
    const unsigned gmask = (L == 32) ? 0xffffffffu : (((1u << L) - 1u) << (lane & ~(L - 1)));
    const unsigned has = __ballot_sync(0xffffffffu, has_max) & gmask;
    is_first_lane = has != 0 && (__ffs(has) - 1) == lane;
  }
  if (!ok) lt_d = first = others = 0.0;
  if (st.zero_blk) {
    acc.zero += lt_d + first + others;
  } else {
    acc.elem += lt_d + others + (is_first_lane ? 0.0 : first);
    if (is_first_lane) acc.mx += first;
    acc.n_esat += nsat;
  }
  if (ok && (lane & (L - 1)) == 0) {
    acc.n_zero += st.zero_blk ? 1u : 0u;
    acc.n_ssat += (a > sat_thr) ? 1u : 0u;
  }
}

// 2^(2E - 254) as a double: the factor that undoes the slice scaling of a sum of squares.
__device__ __forceinline__ double unscale_sq(int E) {
  return __hiloint2double((2 * E + 769) << 20, 0);
}

// Exact errors of a slice in double: every element, or (ONLY_MAX) only the max-valued ones.
// first: the lowest-index max-valued element; others: the other max-valued ones; rest: the rest.
template <int NE, bool ONLY_MAX, typename XF, typename CF>
__device__ __forceinline__ void exact_slice(float a, float D, XF xval, CF code, double& rest,
                                            double& first, double& others) {
  bool seen = false;
#pragma unroll
  for (int k = 0; k < NE; ++k) {
    const bool is_max = fabsf(xval(k)) == a;
    if (ONLY_MAX && !is_max) continue;
    const float y = __fmul_rn(e2m1_to_float(code(k)), D);  // exact
    const double dd = (double)xval(k) - (double)y;          // exact
    const double e2 = dd * dd;
    if (!is_max) {
      rest += e2;
    } else if (!seen) {
      first = e2;
      seen = true;
    } else {
      others += e2;
    }
  }
}

// Tail of a bf16 block slice: lt is the sum of the scaled squares of the elements below the
// maximum, cnt the number of max-valued elements, nsat the clipped elements.  Without CLOSED, ms
// sums the scaled squares of the max-valued elements and a lane with ties of the maximum redoes
// those elements in double; with stored codes (!RC) a slice whose stored scale is far from a
// redoes everything.  CLOSED (recomputed codes): every max-valued element has the same error,
// dmax (scaled), computed once per block.  Either way a slice whose lt is below 2^-80 may have lost squares below 2^-126
// and is redone in double (any loss in a larger sum is below 2^-40 of it).  Items past the end
// hold zeros and an all-zero scale, so they add zeros (their block counters are skipped via ok).
template <int NE, int L, bool RC, bool CLOSED, typename XF, typename CF>
__device__ __forceinline__ void slice_finish_bf16(Acc& acc, int lane, bool ok, float a, float D,
                                                  float sat_thr, const SliceSetup& st, float lt,
                                                  float ms, float dmax, float cnt, float nsat,
                                                  XF xval, CF code) {
  const bool has_max = cnt != 0.0f;
  bool is_first_lane = has_max;
  if constexpr (L > 1) {
    const unsigned gmask = (L == 32) ? 0xffffffffu : (((1u << L) - 1u) << (lane & ~(L - 1)));
    const unsigned has = __ballot_sync(0xffffffffu, has_max) & gmask;
    is_first_lane = has != 0 && (__ffs(has) - 1) == lane;
  }
  double rest = 0.0, first = 0.0, others = 0.0;
  bool all_exact = lt < 0x1p-80f;
  if constexpr (!RC) all_exact |= !st.scale_ok;
  if (all_exact) {
    exact_slice<NE, false>(a, D, xval, code, rest, first, others);
  } else {
    const double sd = unscale_sq(st.E);
    rest = (double)lt * sd;
    if constexpr (CLOSED) {
      if (has_max) {
        first = (double)dmax * (double)dmax * sd;  // exact
        others = (double)(cnt - 1.0f) * first;
      }
    } else {
      if (cnt <= 1.0f) first = (double)ms * sd;
      else exact_slice<NE, true>(a, D, xval, code, rest, first, others);
    }
  }
  if (st.zero_blk) {
    acc.zero += rest + first + others;
  } else {
    acc.elem += rest + others + (is_first_lane ? 0.0 : first);
    if (is_first_lane) acc.mx += first;
    acc.n_esat += nsat;
  }
  if (ok && (lane & (L - 1)) == 0) {
    acc.n_zero += st.zero_blk ? 1u : 0u;
    acc.n_ssat += (a > sat_thr) ? 1u : 0u;
  }
}

// Tail of a bf16 block slice with recomputed codes (blocks of 16 and more).  lt2 sums the scaled
// squares of all the slice's elements; every max-valued element has the error dmax (scaled), so
// the lane holding the block's first max element moves dmax^2 (exact in double) from that sum to
// SSE_max and the rest stays in SSE_elem (other max-valued elements included, as they should).
// The subtraction only loses digits when dmax^2 dominates the slice's sum; a slice whose remainder
// is below dmax^2 / 8, or whose sum is below 2^-80 (squares below 2^-126 could be lost), is redone
// exactly in double -- unless every element of the slice is zero (lane_zero: zeros of a block's
// padding past a row's end, or of an all-zero block), whose errors are exactly zero.  has_max:
// this lane holds a max-valued element.
template <int NE, int L, typename XF, typename CF>
__device__ __forceinline__ void slice_finish_closed(Acc& acc, int lane, bool ok, bool has_max,
                                                    bool lane_zero, float a, float D,
                                                    float sat_thr, const SliceSetup& st,
                                                    float2 lt2, float dmax, uint32_t nsat2,
                                                    XF xval, CF code) {
  bool is_first_lane = has_max;
  if constexpr (L > 1) {
    const unsigned gmask = (L == 32) ? 0xffffffffu : (((1u << L) - 1u) << (lane & ~(L - 1)));
    const unsigned has = __ballot_sync(0xffffffffu, has_max) & gmask;
    is_first_lane = has != 0 && (__ffs(has) - 1) == lane;
  }
  const float lt = __fadd_rn(lt2.x, lt2.y);
  double rest = 0.0, first = 0.0, others = 0.0;
  bool exact = lt < 0x1p-80f && !lane_zero;
  if (!exact) {
    rest = (double)lt * unscale_sq(st.E);
    if (is_first_lane && !st.zero_blk) {
      first = (double)dmax * (double)dmax * unscale_sq(st.E);  // exact
      rest -= first;
      exact = rest < 0.125 * first;
    }
  }
  if (exact) {
    rest = first = others = 0.0;
    exact_slice<NE, false>(a, D, xval, code, rest, first, others);
    rest += others;
    if (!is_first_lane) rest += first, first = 0.0;
  }
  if (st.zero_blk) {
    acc.zero += rest + first;
  } else {
    acc.elem += rest;
    acc.mx += first;
    float c0, c1;
    asm("{\n\t.reg .b16 h0, h1;\n\t"
        "mov.b32 {h0, h1}, %2;\n\t"
        "cvt.f32.bf16 %0, h0;\n\t"
        "cvt.f32.bf16 %1, h1;\n\t}"
        : "=f"(c0), "=f"(c1) : "r"(nsat2));
    acc.n_esat += c0 + c1;
  }
  if (ok && (lane & (L - 1)) == 0) {
    acc.n_zero += st.zero_blk ? 1u : 0u;
    acc.n_ssat += (a > sat_thr) ? 1u : 0u;
  }
}

// Generic block slice of NE elements (fp32 input): xval(k) value, code(k) a word whose low nibble
// is element k's code (k a compile-time constant after unrolling).  min_abs: the slice's min|x|
// (zeros included); a nonzero value below 2^-30 a could lose digits to fp32 underflow.
template <int NE, int L, typename XF, typename CF>
__device__ __forceinline__ void block_slice(Acc& acc, int lane, bool ok, float a, float D,
                                            float sat_thr, float min_abs, XF xval, CF code) {
  const SliceSetup st = slice_setup(a, D);
  const float as = __fmul_rn(a, st.sc);
  float lt = 0.0f, ms = 0.0f, cnt = 0.0f, nsat = 0.0f;
#pragma unroll
  for (int k = 0; k < NE; ++k) {
    const float xs = __fmul_rn(xval(k), st.sc);
    const float d = __fmaf_rn(__uint_as_float(e2m1_scaled_bits_at(code(k), 0)), st.nDq, xs);
    const float ax = fabsf(xs);
    if (ax >= as) {
      ms = __fmaf_rn(d, d, ms);
      cnt += 1.0f;
    } else {
      lt = __fmaf_rn(d, d, lt);
    }
    if (ax > st.sat6s) nsat += 1.0f;
  }
  bool exact = false;
  if (min_abs < st.tiny) {
#pragma unroll
    for (int k = 0; k < NE; ++k) {
      const float ax = fabsf(xval(k));
      exact |= (ax != 0.0f) && (ax < st.tiny);
    }
  }
  slice_finish<NE, L>(acc, lane, ok, a, D, sat_thr, exact, st, lt, ms, cnt, nsat, xval, code);
}

// ------------------------------------------------------------------------------------------------
// bf16 input
// ------------------------------------------------------------------------------------------------

// What the bf16 pass does with the codes (StatsMode): read them (kGiven), recompute them in
// registers with the quantize kernel's rule (kRecompute), or recompute and also write them to
// packed_out / scales_out (kStore: the fused quantize + pack + reduction pass).

// One thread's item: EPT consecutive elements (NW words), their code words and scale bytes.
template <int NW, int NCW>
struct StatsItem {
  uint32_t w[NW];
  uint32_t cw[NCW];
  uint32_t scw;
  int64_t row, j;  // row-pitched mode: the item's row and its item index in the row
  int nval;        // row-pitched mode: its elements inside the row (a multiple of 8; <= 0: none)
};

// ROWS: the row-pitched mode (STensor) for rows of cols % 8 == 0 elements that the block size
// N >= 32 does not divide (recomputed codes): item i of the padded item space is item j of row
// i / ipr (a RowCursor that follows the loads, no division per item); x at row * cols + 32 j
// (16-byte aligned), codes at row * pb + 16 j as 4-byte words, scales at row * nb; an item's
// 8-element chunks past the row's end are neither read (zeros: they change neither the block
// maximum nor the sums) nor written.
template <int N, int FMT, int MODE, bool ROWS = false>
__global__ void __launch_bounds__(kThreads, N <= 8 ? MX_ST_MINB_SMALL : MX_ST_MINB)
    k_error_stats_bf16(
    const __grid_constant__ SGroup grp) {
  const SWork wk = s_work(grp);
  const uint16_t* __restrict__ x = static_cast<const uint16_t*>(wk.t.x);
  const uint8_t* __restrict__ packed = wk.t.packed;
  const uint8_t* __restrict__ scales = wk.t.scales;
  uint8_t* __restrict__ packed_out = wk.t.packed_out;
  uint8_t* __restrict__ scales_out = wk.t.scales_out;
  const int64_t nitems = wk.t.nitems;
  const uint16_t g_bits = tensor_g_bits(wk.t.g_bits, wk.t.g_dev);
  constexpr bool RECOMPUTE = MODE != kGiven, STORE = MODE == kStore;
  // Recomputed codes (blocks of 32 and more; smaller blocks run on k_qstats_small): the
  // max-valued elements' error in closed form per block.
  static_assert(!RECOMPUTE || N >= 32, "recomputed codes with N <= 16 run on k_qstats_small");
  constexpr bool CLOSED = RECOMPUTE;
  using S = SShape<N, uint16_t>;
  constexpr int EPT = S::EPT, L = S::L, BPI = S::BPI, NW = EPT / 2, NCW = EPT / 8;
  constexpr int BW = NW / BPI;  // words per block inside an item
  constexpr int BE = 2 * BW;    // elements per block inside an item
  using Item = StatsItem<NW, NCW>;
  static_assert(NCW == 1 || NCW == 2 || NCW == 4, "items of 8, 16 or 32 elements");
  static_assert(!ROWS || (RECOMPUTE && BPI == 1 && NCW == 4), "row-pitched mode: N >= 32");
  __shared__ float s_rcp[256], s_D[256];
  const float g = fp16_bits_to_float(g_bits);
  for (int c = threadIdx.x; c < 256; c += blockDim.x) {
    const float D = __fmul_rn(scale_value(c, FMT), g);
    s_D[c] = D;
    s_rcp[c] = D > 0.0f ? __frcp_rn(D) : 0.0f;
  }
  const float r6 = __frcp_rn(__fmul_rn(6.0f, g));
  const float sat_thr = __fmul_rn(__fmul_rn(6.0f, g), scale_max<FMT>());  // exact
  __syncthreads();
  griddep_wait();  // inputs may come from the previous kernel in the stream
  griddep_launch_next();

  Acc acc;
  const int64_t T = (int64_t)wk.nctas * blockDim.x;
  const int64_t tid = (int64_t)wk.cta * blockDim.x + threadIdx.x;
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = tid - lane;

  RowCursor lc;  // ROWS: row and item of the next item loaded (loads go tid, tid + T, ...)
  if constexpr (ROWS) lc.init(tid, T, wk.t.ipr);

  // Loads of one item (zeros past the end).  Issued one item ahead of the arithmetic.
  auto load = [&](Item& it, int64_t i) {
    bool ok = i < nitems;
    int64_t off = 0;
    if constexpr (ROWS) {
      it.row = lc.row;
      it.j = lc.j;
      it.nval = (int)min((int64_t)EPT, wk.t.cols - lc.j * EPT);
      off = lc.row * wk.t.cols + lc.j * EPT;
      ok = ok && it.nval > 0;
      lc.advance();
    }
#pragma unroll
    for (int h = 0; h < NW / 4; ++h) {
      uint4 v = make_uint4(0, 0, 0, 0);
      if constexpr (ROWS) {
        if (ok && 8 * h < it.nval) v = ld_stream16(x + off + h * 8);
      } else {
        if (ok) v = ld_stream16(x + i * EPT + h * 8);
      }
      it.w[4 * h + 0] = v.x; it.w[4 * h + 1] = v.y; it.w[4 * h + 2] = v.z; it.w[4 * h + 3] = v.w;
    }
    it.scw = 0;
#pragma unroll
    for (int j = 0; j < NCW; ++j) it.cw[j] = 0;
    if constexpr (!RECOMPUTE) {
      if (ok) {
        if constexpr (NCW == 4) {
          const uint4 p = __ldcs(reinterpret_cast<const uint4*>(packed) + i);
          it.cw[0] = p.x; it.cw[1] = p.y; it.cw[2] = p.z; it.cw[3] = p.w;
        } else if constexpr (NCW == 2) {
          const uint2 p = __ldcs(reinterpret_cast<const uint2*>(packed) + i);
          it.cw[0] = p.x; it.cw[1] = p.y;
        } else {
          it.cw[0] = __ldcs(reinterpret_cast<const unsigned int*>(packed) + i);
        }
        if constexpr (BPI == 1) it.scw = __ldg(scales + i / L);
        else if constexpr (BPI == 2) it.scw = __ldg(reinterpret_cast<const unsigned short*>(scales) + i);
        else it.scw = __ldg(reinterpret_cast<const unsigned int*>(scales) + i);
      }
    }
  };

  auto process = [&](Item& it, int64_t i) {
    bool ok = i < nitems;
    if constexpr (ROWS) ok = ok && it.nval > 0;
    float a_b[BPI], D_b[BPI], r_b[BPI];
    uint32_t m_b[BPI];
    bool own_b[BPI];      // this lane holds a max-valued element of block b
    bool zero_b[BPI];     // this lane's elements of block b are all zero
    uint32_t sc_all = 0;  // scale codes of the item's blocks, byte b = block b
#pragma unroll
    for (int b = 0; b < BPI; ++b) {
      const uint32_t* wb = &it.w[b * BW];
      uint32_t t = wb[0];
#pragma unroll
      for (int k = 1; k < BW; ++k) t = bf16x2_absmax(t, wb[k]);
      t &= 0x7FFF7FFFu;
      uint32_t m = max(t & 0xFFFFu, t >> 16);
      const uint32_t m_lane = m;
#pragma unroll
      for (int off = 1; off < L; off <<= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
      const float a = __uint_as_float(m << 16);
      uint32_t s;
      if constexpr (RECOMPUTE) {
        s = encode_scale<FMT>(snap21(__fmul_rn(a, r6)));
        r_b[b] = s_rcp[s];
      } else {
        s = (it.scw >> (8 * b)) & 0xFF;
      }
      a_b[b] = a;
      m_b[b] = m;
      own_b[b] = m_lane == m;
      zero_b[b] = m_lane == 0;
      D_b[b] = s_D[s];
      sc_all |= s << (8 * b);
    }
    // closed form (one block slice per item): codes and squares together, per code word (also
    // where a block spans several lanes, N >= 64: measured 0.68 -> 0.74 of the copy peak there
    // against converting the item's codes first and reducing them afterwards)
    SliceSetup st0;
    float2 lt0 = make_float2(0.0f, 0.0f);
    uint32_t nsat0 = 0u;
    constexpr bool W8 = CLOSED;
    if constexpr (W8) {
      static_assert(!CLOSED || BPI == 1, "one block slice per item");
      st0 = slice_setup(a_b[0], D_b[0]);
      const uint32_t S2 = (__float_as_uint(__fmul_rn(6.0f, D_b[0])) >> 16) * 0x10001u;
      // (measured: deciding the saturation case once per item is faster where a lane holds a
      // whole block; where a block spans lanes the two inlined copies spill, so each code word
      // checks it itself)
      if constexpr (L > 1) {
#pragma unroll
        for (int j = 0; j < NCW; ++j)
          it.cw[j] = qs_word8<4, kCheck>(&it.w[4 * j], &r_b[0], &st0.nDq, &S2, st0.sc, &lt0,
                                         nsat0);
      } else if (!deep_item<1>(&r_b[0], st0.sc)) {
#pragma unroll
        for (int j = 0; j < NCW; ++j)
          it.cw[j] = qs_word8<4, kFast>(&it.w[4 * j], &r_b[0], &st0.nDq, &S2, st0.sc, &lt0, nsat0);
      } else {
#pragma unroll
        for (int j = 0; j < NCW; ++j)
          it.cw[j] = qs_word8<4, kDeep>(&it.w[4 * j], &r_b[0], &st0.nDq, &S2, st0.sc, &lt0, nsat0);
      }
    }
    if constexpr (STORE && ROWS) {
      if (ok) {
        uint8_t* prow = packed_out + it.row * wk.t.pb + it.j * 16;
#pragma unroll
        for (int h = 0; h < 4; ++h)
          if (8 * h < it.nval) *reinterpret_cast<uint32_t*>(prow + 4 * h) = it.cw[h];
        if ((lane & (L - 1)) == 0)
          scales_out[it.row * wk.t.nb + (it.j * EPT) / N] = (uint8_t)sc_all;
      }
    } else if constexpr (STORE) {
      if (ok) {
        if constexpr (NCW == 4)
          *reinterpret_cast<uint4*>(packed_out + i * 16) =
              make_uint4(it.cw[0], it.cw[1], it.cw[2], it.cw[3]);
        else if constexpr (NCW == 2)
          *reinterpret_cast<uint2*>(packed_out + i * 8) = make_uint2(it.cw[0], it.cw[1]);
        else
          *reinterpret_cast<uint32_t*>(packed_out + i * 4) = it.cw[0];
        if constexpr (BPI == 1) {
          if ((lane & (L - 1)) == 0) scales_out[i / L] = (uint8_t)sc_all;
        } else if constexpr (BPI == 2) {
          *reinterpret_cast<uint16_t*>(scales_out + i * 2) = (uint16_t)sc_all;
        } else {
          *reinterpret_cast<uint32_t*>(scales_out + i * 4) = sc_all;
        }
      }
    }
#pragma unroll
    for (int b = 0; b < BPI; ++b) {
      const float a = a_b[b], D = D_b[b];
      const SliceSetup st = W8 ? st0 : slice_setup(a, D);
      const uint32_t sb = __float_as_uint(__fmul_rn(6.0f, D)) >> 16;  // 6 S g rounded down
      const uint32_t A2 = m_b[b] * 0x10001u, S2 = sb * 0x10001u;
      float lt = 0.0f, ms = 0.0f, cnt = 0.0f, nsat = 0.0f, dmax = 0.0f;
      const float nD = st.nDq;
#pragma unroll
      for (int k = 0; k < BW && !CLOSED; ++k) {
        const int wi = b * BW + k;
        const uint32_t w = it.w[wi], lo = w << 16, hi = w & 0xFFFF0000u, cw = it.cw[wi >> 2];
        constexpr bool MS = !CLOSED;
        switch (wi & 3) {
          case 0: pair_step<0, MS>(w, lo, hi, cw, st.sc, nD, A2, S2, lt, ms, cnt, nsat); break;
          case 1: pair_step<1, MS>(w, lo, hi, cw, st.sc, nD, A2, S2, lt, ms, cnt, nsat); break;
          case 2: pair_step<2, MS>(w, lo, hi, cw, st.sc, nD, A2, S2, lt, ms, cnt, nsat); break;
          default: pair_step<3, MS>(w, lo, hi, cw, st.sc, nD, A2, S2, lt, ms, cnt, nsat); break;
        }
      }
      if constexpr (CLOSED) {
        // the max-valued elements' code magnitude is that of a; their scaled error, as above
        const float qa = snap_quotient2(__float_as_uint(a), 0u, r_b[b]).x;
        const uint32_t ca = cvt_e2m1x8(qa, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f);
        dmax = __fmaf_rn(__uint_as_float(e2m1_scaled_bits_at(ca, 0)), st.nDq,
                         __fmul_rn(a, st.sc));
      }
      const int e0 = b * BE;
      auto xval = [&](int k) {
        const uint32_t wd = it.w[(e0 + k) >> 1];
        return ((e0 + k) & 1) ? bf16hi(wd) : bf16lo(wd);
      };
      auto code = [&](int k) { return it.cw[(e0 + k) >> 3] >> (4 * ((e0 + k) & 7)); };
      if constexpr (CLOSED)
        slice_finish_closed<BE, L>(acc, lane, ok, own_b[b], zero_b[b], a, D, sat_thr, st, lt0,
                                   dmax, nsat0,
                                   xval, code);
      else
        slice_finish_bf16<BE, L, RECOMPUTE, false>(acc, lane, ok, a, D, sat_thr, st, lt, ms, dmax,
                                                   cnt, nsat, xval, code);
    }
  };

  // Two items in flight per thread: the loads of the next item are issued before the arithmetic
  // of the current one.  The trip test is warp-uniform (lanes of a block share shuffles).
  Item A, B;
  int64_t i = tid;
  load(A, i);
  while (warp0 + (i - tid) < nitems) {
    load(B, i + T);
    process(A, i);
    i += T;
    if (!(warp0 + (i - tid) < nitems)) break;
    load(A, i + T);
    process(B, i);
    i += T;
  }
  finish_cta(acc, wk);
}

// ------------------------------------------------------------------------------------------------
// bf16 input, small blocks (N = 4, 8, 16) with recomputed codes
// ------------------------------------------------------------------------------------------------
// The per-block work dominates at these sizes, so it is done for two blocks at once where the
// hardware has paired forms: block maxima as one bf16x2 word per block pair, two scale quotients
// per f32x2 multiply, two E4M3 codes per conversion, the max elements' errors per f32x2 FMA.  The
// whole item (16 or 32 elements) shares one scaling s = 2^(127 - E), E the exponent of the item's
// largest block maximum, so the three sums are kept in fp32 per item and turned into double once
// per item.  Every element's square goes into its block's sum; each non-zero block then moves its
// first max element's square (dmax^2: all max-valued elements of a block share that error) to
// SSE_max.  Where dmax^2 dominates a block so much (remainder below dmax^2 / 64) that the
// subtraction would cost digits, that block's elements below the maximum are summed apart.  An
// item is redone exactly in double when squares could have been lost to fp32 underflow: a non-zero
// block maximum with a sum below 2^-80, or (in a block summed apart) a non-zero scaled error below
// 2^-63.
// N = 4 with UE5M3 scales goes further: each block pair's two blocks sit side by side in f32x2
// form through the whole item (qs4_pair), a block's reciprocal, scale value and clip level come
// from one 16-byte shared-memory entry, and the split of the sums is made for both blocks of a
// pair with one test (the per-block handling above runs only where a pair has a zero block, a
// dominating max element or a possibly underflowed sum).  N = 4 with E4M3 scales keeps the
// per-block form: without a global scale, data of small magnitude puts E4M3 scales in its coarse
// subnormal range, where a block's max element often dominates its sum; some lane of nearly every
// warp then needs the per-block handling, and the pair test only adds to it (measured: 0.41 of the
// copy peak per-block against 0.37 paired on a 70B-shaped layer, while UE5M3 goes from 0.44 to
// 0.52).  N = 8 and 16 reduce one code word at a time (qs_word8).

// Quotients of two elements with their own reciprocals (see snap_quotient2).
__device__ __forceinline__ float2 snap_quotient2v(float2 x, float2 r) {
  const float2 y = __ffma2_rn(x, r, make_float2(48.0f, 48.0f));
  const float2 q = __fadd2_rd(y, make_float2(-48.0f, -48.0f));
  return __ffma2_rn(x, make_float2(0x1p-60f, 0x1p-60f), q);
}

__device__ __forceinline__ uint32_t bf16x2_set_gt(uint32_t a, uint32_t b) {  // 1.0 where a > b
  uint32_t d;
  asm("set.gt.bf16x2.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bf16x2_set_eq(uint32_t a, uint32_t b) {  // 1.0 where a == b
  uint32_t d;
  asm("set.eq.bf16x2.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bf16x2_add(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bf16x2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
// Sum of the two halves of a bf16x2 word of small integers, as fp32.
__device__ __forceinline__ float bf16x2_hsum(uint32_t v) {
  return __fadd_rn(__uint_as_float(v << 16), __uint_as_float(v & 0xFFFF0000u));
}

// Blocks of 4 (UE5M3): one block pair (words w[0], w[1]: block 2j; w[2], w[3]: block 2j + 1)
// quantized and reduced with the two blocks side by side in f32x2 form -- .x an element of block
// 2j, .y the element at the same place in block 2j + 1 -- so that each pair operand (the
// reciprocals rq, the code scalings nDq = -S g s 2^126, the sums lt) is the two blocks' own values
// and needs no copy.
// As in qs_word8 the quotients are taken of magnitudes, xs = |x| s from the mixed-precision FMAs
// with rq = r / s (DEEP: of the unscaled |x| with rq = r, for an item with a block so far beyond
// its saturation that r / s would overflow), the magnitude codes decode with one shift and one
// mask, and x's signs are put into the code word at the end.  S2a / S2b: the two blocks' clip
// levels RD_bf16(6 S g), twice; clipped elements are counted in nsat2 (bf16x2 integers).
template <bool DEEP>
__device__ __forceinline__ uint32_t qs4_pair(const uint32_t* w, float2 rq, float2 nDq,
                                             uint32_t S2a, uint32_t S2b, float sc, uint32_t sc16,
                                             float2& lt, uint32_t& nsat2) {
  uint32_t aw[4];
  float2 xs[4], xq[4];  // per word: (low half, high half) scaled, and the quotients' operands
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    aw[k] = w[k] & 0x7FFF7FFFu;
    if constexpr (!DEEP) {
      xs[k] = mag_scaled2(aw[k], sc16);
      xq[k] = xs[k];
    } else {
      xq[k] = make_float2(__uint_as_float(aw[k] << 16), __uint_as_float(aw[k] & 0xFFFF0000u));
      xs[k] = __fmul2_rn(xq[k], make_float2(sc, sc));
    }
  }
  // element pair p: half p & 1 of word p >> 1 in each block
  float2 X[4], Q[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int m = p >> 1;
    X[p] = (p & 1) ? make_float2(xs[m].y, xs[m + 2].y) : make_float2(xs[m].x, xs[m + 2].x);
    const float2 o =
        (p & 1) ? make_float2(xq[m].y, xq[m + 2].y) : make_float2(xq[m].x, xq[m + 2].x);
    const float2 y = __ffma2_rn(o, rq, make_float2(48.0f, 48.0f));
    Q[p] = __fadd2_rn(y, make_float2(-48.0f, -48.0f));
  }
  // byte k of cm: word k's two magnitude codes (words 0, 1 from the .x lanes, 2, 3 from the .y)
  const uint32_t cm = cvt_e2m1x8(Q[0].x, Q[1].x, Q[2].x, Q[3].x, Q[0].y, Q[1].y, Q[2].y, Q[3].y);
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    // nibble 4p holds pair p's .x code, nibble 16 + 4p its .y code: magnitude bits to 22..24
    const uint32_t bx = (cm << (22 - 4 * p)) & 0x01C00000u;
    const uint32_t by = (p < 2 ? cm << (6 - 4 * p) : cm >> (4 * p - 6)) & 0x01C00000u;
    const float2 d = __ffma2_rn(make_float2(__uint_as_float(bx), __uint_as_float(by)), nDq, X[p]);
    lt = __ffma2_rn(d, d, lt);
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) nsat2 = bf16x2_add(nsat2, bf16x2_set_gt(aw[k], k < 2 ? S2a : S2b));
  return put_signs(cm, w[0], w[1], w[2], w[3]);
}

// Item shape of the small-block kernel: 16 elements for N = 4 (four blocks), 32 for N = 8 and 16
// (four or two blocks), so that blocks always come in pairs.
#ifndef MX_QS_EPT8  // elements per item of the small-block kernel for N = 8 (16 or 32)
#define MX_QS_EPT8 32
#endif
template <int N>
struct QSShape {
  static constexpr int EPT = N == 16 ? 32 : N == 8 ? MX_QS_EPT8 : MX_ST_EPT_SMALL;
};

template <int N, int FMT, int MODE>
__global__ void __launch_bounds__(kThreads, MX_QS_MINB)
    k_qstats_small(const __grid_constant__ SGroup grp) {
  static_assert(N == 4 || N == 8 || N == 16, "small blocks only");
  static_assert(MODE != kGiven, "codes are recomputed");
  const SWork wk = s_work(grp);
  const uint16_t* __restrict__ x = static_cast<const uint16_t*>(wk.t.x);
  uint8_t* __restrict__ packed_out = wk.t.packed_out;
  uint8_t* __restrict__ scales_out = wk.t.scales_out;
  const int64_t nitems = wk.t.nitems;
  constexpr bool STORE = MODE == kStore;
  constexpr int EPT = QSShape<N>::EPT, NW = EPT / 2, NCW = EPT / 8, NB = EPT / N, BW = N / 2;
  constexpr int NP = NB / 2;
  static_assert(NB % 2 == 0 && NB <= 4 && (NCW == 2 || NCW == 4), "2 or 4 blocks per item");
  // Blocks of 4 with UE5M3 scales take the block-pair form (qs4_pair); E4M3 keeps the per-block
  // form, which measured faster there (see the note above qs4_pair)
  constexpr bool PAIRS4 = N == 4 && FMT == kUE5M3;
  __shared__ float s_rcp[256], s_D[256];
  // PAIRS4: per scale code {1 / (S g) (0 for S = 0), S g, the clip level RD_bf16(6 S g) twice as
  // bf16x2 bits (the largest finite bf16 for S = 0, which no finite |x| exceeds), unused}
  __shared__ float4 s_tab[PAIRS4 ? 256 : 1];
  const float g = fp16_bits_to_float(tensor_g_bits(wk.t.g_bits, wk.t.g_dev));
  for (int c = threadIdx.x; c < 256; c += blockDim.x) {
    const float D = __fmul_rn(scale_value(c, FMT), g);
    const float rcp = D > 0.0f ? __frcp_rn(D) : 0.0f;
    if constexpr (PAIRS4) {
      uint32_t thr = __float_as_uint(__fmul_rn(6.0f, D)) >> 16;  // exact product, truncated
      if (thr == 0u) thr = 0x7F7Fu;
      s_tab[c] = make_float4(rcp, D, __uint_as_float(thr * 0x10001u), 0.0f);
    } else {
      s_D[c] = D;
      s_rcp[c] = rcp;
    }
  }
  const float r6 = __frcp_rn(__fmul_rn(6.0f, g));
  const float sat_thr = __fmul_rn(__fmul_rn(6.0f, g), scale_max<FMT>());  // exact
  const uint32_t SAT2 = (__float_as_uint(sat_thr) >> 16) * 0x10001u;      // RD to bf16, twice
  __syncthreads();
  griddep_wait();  // inputs may come from the previous kernel in the stream
  griddep_launch_next();

  Acc acc;
  const int64_t T = (int64_t)wk.nctas * blockDim.x;
  const int64_t tid = (int64_t)wk.cta * blockDim.x + threadIdx.x;
  using Item = StatsItem<NW, NCW>;

  auto load = [&](Item& it, int64_t i) {
    const bool ok = i < nitems;
#pragma unroll
    for (int h = 0; h < NW / 4; ++h) {
      uint4 v = make_uint4(0, 0, 0, 0);
      if (ok) v = ld_stream16(x + i * EPT + h * 8);
      it.w[4 * h + 0] = v.x; it.w[4 * h + 1] = v.y; it.w[4 * h + 2] = v.z; it.w[4 * h + 3] = v.w;
    }
  };

  auto process = [&](Item& it, int64_t i) {
    const bool ok = i < nitems;
    // block maxima, two blocks per bf16x2 word: M[j] = {a_2j, a_2j+1}
    uint32_t M[NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) {
      uint32_t t0 = it.w[2 * j * BW], t1 = it.w[(2 * j + 1) * BW];
#pragma unroll
      for (int k = 1; k < BW; ++k) {
        t0 = bf16x2_absmax(t0, it.w[2 * j * BW + k]);
        t1 = bf16x2_absmax(t1, it.w[(2 * j + 1) * BW + k]);
      }
      M[j] = bf16x2_absmax(__byte_perm(t0, t1, 0x5410), __byte_perm(t0, t1, 0x7632)) & 0x7FFF7FFFu;
    }
    // the item's scaling
    uint32_t mm = M[0];
#pragma unroll
    for (int j = 1; j < NP; ++j) mm = bf16x2_absmax(mm, M[j]);
    // E clamped to [1, 253]: sc = 2^(127 - E) stays a normal number (see SliceSetup)
    const int E = min(max((int)(max(mm & 0x7FFFu, (mm >> 16) & 0x7FFFu) >> 7), 1), 253);
    const float sc = __uint_as_float((uint32_t)(254 - E) << 23);
    if constexpr (PAIRS4) {
      // Blocks of 4: the item's two block pairs, each with its blocks side by side in f32x2 form
      // (qs4_pair); the per-block split of the sums is made for both blocks of a pair at once
      // where neither needs the special handling below (a zero block, a block whose max element
      // dominates its sum, or a sum that could have lost squares to underflow).
      const float rcs = __uint_as_float((uint32_t)E << 23);  // 1 / sc, exact
      const uint32_t sc16 = __float_as_uint(sc) >> 16;       // sc as a bf16 (a power of two)
      float2 af[2], r2[2], D2[2], nDq2[2], rs2[2];
      uint32_t S2[4];
      uint32_t sc_all = 0, ss2 = 0;  // scale bytes; saturated-scale count
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        af[j] = make_float2(__uint_as_float(M[j] << 16), __uint_as_float(M[j] & 0xFFFF0000u));
        const float2 u = __fmul2_rn(af[j], make_float2(r6, r6));
        uint32_t s0, s1;
        if constexpr (FMT == kE4M3) {
          unsigned short h;
          asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
              : "=h"(h) : "f"(snap21(u.y)), "f"(snap21(u.x)));
          s0 = h & 0xFFu;
          s1 = (uint32_t)h >> 8;
        } else {
          s0 = encode_scale<FMT>(snap21(u.x));
          s1 = encode_scale<FMT>(snap21(u.y));
        }
        sc_all |= (s0 | (s1 << 8)) << (16 * j);
        const float4 t0 = s_tab[s0], t1 = s_tab[s1];
        r2[j] = make_float2(t0.x, t1.x);
        D2[j] = make_float2(t0.y, t1.y);
        S2[2 * j] = __float_as_uint(t0.z);
        S2[2 * j + 1] = __float_as_uint(t1.z);
        nDq2[j] = __fmul2_rn(__fmul2_rn(D2[j], make_float2(sc, sc)),
                             make_float2(-0x1p126f, -0x1p126f));
        rs2[j] = __fmul2_rn(r2[j], make_float2(rcs, rcs));  // r / s (see qs_word8)
        ss2 = bf16x2_add(ss2, bf16x2_set_gt(M[j], SAT2));
      }
      const bool deep = fmaxf(fmaxf(rs2[0].x, rs2[0].y), fmaxf(rs2[1].x, rs2[1].y)) > 0x1p64f;
      uint32_t cw[2];
      float2 lt[2] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
      uint32_t nsat2 = 0u;
      if (!deep) {
#pragma unroll
        for (int j = 0; j < 2; ++j)
          cw[j] = qs4_pair<false>(&it.w[4 * j], rs2[j], nDq2[j], S2[2 * j], S2[2 * j + 1], sc,
                                  sc16, lt[j], nsat2);
      } else {
#pragma unroll
        for (int j = 0; j < 2; ++j)
          cw[j] = qs4_pair<true>(&it.w[4 * j], r2[j], nDq2[j], S2[2 * j], S2[2 * j + 1], sc,
                                 sc16, lt[j], nsat2);
      }
      if constexpr (STORE) {
        if (ok) {
          *reinterpret_cast<uint2*>(packed_out + i * 8) = make_uint2(cw[0], cw[1]);
          *reinterpret_cast<uint32_t*>(scales_out + i * 4) = sc_all;
        }
      }
      float2 ae2 = make_float2(0.0f, 0.0f), am2 = make_float2(0.0f, 0.0f);
      float az = 0.0f, nz = 0.0f;  // zero blocks' sums and their count
      bool exact = false;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        // the two blocks' max elements: code of a / (S g) (unscaled quotients, which never
        // overflow), scaled error, square
        const float2 y = __ffma2_rn(af[j], r2[j], make_float2(48.0f, 48.0f));
        const float2 qa = __fadd2_rn(y, make_float2(-48.0f, -48.0f));
        const uint32_t ca = cvt_e2m1x2(qa.y, qa.x);
        const float2 dec = make_float2(__uint_as_float((ca << 22) & 0x01C00000u),
                                       __uint_as_float((ca << 18) & 0x01C00000u));
        const float2 dm = __ffma2_rn(dec, nDq2[j], __fmul2_rn(af[j], make_float2(sc, sc)));
        const float2 f2 = __fmul2_rn(dm, dm);
        const float2 rest = __ffma2_rn(f2, make_float2(-1.0f, -1.0f), lt[j]);
        const float2 lim = __fmul2_rn(f2, make_float2(0x1p-6f, 0x1p-6f));
        const bool plain = D2[j].x > 0.0f && D2[j].y > 0.0f && !(rest.x < lim.x) &&
                           !(rest.y < lim.y) && !(lt[j].x < 0x1p-80f) && !(lt[j].y < 0x1p-80f);
        if (plain) {
          ae2 = __fadd2_rn(ae2, rest);
          am2 = __fadd2_rn(am2, f2);
        } else {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int b = 2 * j + h;
            const float tb = h ? lt[j].y : lt[j].x;
            const float first = h ? f2.y : f2.x;
            const float ab = h ? af[j].y : af[j].x;
            const float Db = h ? D2[j].y : D2[j].x;
            const float nDqb = h ? nDq2[j].y : nDq2[j].x;
            exact |= ab > 0.0f && tb < 0x1p-80f;
            if (Db > 0.0f) {
              float rb = __fsub_rn(tb, first);
              if (rb < __fmul_rn(first, 0x1p-6f)) {
                // dmax^2 dominates the block: sum the elements below the maximum apart (no
                // cancellation) and add the other max-valued elements' copies of dmax^2
                float rs = 0.0f, nt = 0.0f;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const int e = b * 4 + k;
                  const uint32_t wd = it.w[e >> 1];
                  const float xv = (e & 1) ? bf16hi(wd) : bf16lo(wd);
                  const float dq = __uint_as_float(e2m1_scaled_bits_at(cw[e >> 3], 4 * (e & 7)));
                  const float d = __fmaf_rn(dq, nDqb, __fmul_rn(xv, sc));
                  if (fabsf(xv) != ab) rs = __fmaf_rn(d, d, rs);
                  else nt += 1.0f;
                  exact |= d != 0.0f && fabsf(d) < 0x1p-63f;  // its square would be lost
                }
                rb = __fmaf_rn(nt - 1.0f, first, rs);
              }
              if (h) {
                ae2.y = __fadd_rn(ae2.y, rb);
                am2.y = __fadd_rn(am2.y, first);
              } else {
                ae2.x = __fadd_rn(ae2.x, rb);
                am2.x = __fadd_rn(am2.x, first);
              }
            } else {
              az = __fadd_rn(az, tb);
              nz += 1.0f;
            }
          }
        }
      }
      if (!exact) {
        const double us = unscale_sq(E);
        acc.elem += (double)__fadd_rn(ae2.x, ae2.y) * us;
        acc.mx += (double)__fadd_rn(am2.x, am2.y) * us;
        acc.zero += (double)az * us;
      } else {
        // exact in double, block by block (first max element by index)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int e0 = b * 4;
          auto xval = [&](int k) {
            const uint32_t wd = it.w[(e0 + k) >> 1];
            return ((e0 + k) & 1) ? bf16hi(wd) : bf16lo(wd);
          };
          auto code = [&](int k) { return cw[(e0 + k) >> 3] >> (4 * ((e0 + k) & 7)); };
          const float ab = (b & 1) ? af[b >> 1].y : af[b >> 1].x;
          const float Db = (b & 1) ? D2[b >> 1].y : D2[b >> 1].x;
          double rest = 0.0, first = 0.0, others = 0.0;
          exact_slice<4, false>(ab, Db, xval, code, rest, first, others);
          if (Db > 0.0f) {
            acc.elem += rest + others;
            acc.mx += first;
          } else {
            acc.zero += rest + first + others;
          }
        }
      }
      if (ok) {
        acc.n_esat += bf16x2_hsum(nsat2);
        acc.n_zero_f += nz;
        acc.n_ssat_f += bf16x2_hsum(ss2);
      }
      return;
    }
    // scale codes, reciprocals and per-block constants, two blocks at a time
    float r_b[NB], D_b[NB], nDq_b[NB];
    uint32_t S2_b[NB];
    uint32_t sc_all = 0, zc2 = 0, ss2 = 0;  // scale bytes; zero-block and saturated-scale counts
    float2 af[NP];
#pragma unroll
    for (int j = 0; j < NP; ++j) {
      af[j] = make_float2(__uint_as_float(M[j] << 16), __uint_as_float(M[j] & 0xFFFF0000u));
      const float2 u = __fmul2_rn(af[j], make_float2(r6, r6));
      uint32_t s0, s1;
      if constexpr (FMT == kE4M3) {
        unsigned short h;
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
            : "=h"(h) : "f"(snap21(u.y)), "f"(snap21(u.x)));
        s0 = h & 0xFFu;
        s1 = (uint32_t)h >> 8;
      } else {
        s0 = encode_scale<FMT>(snap21(u.x));
        s1 = encode_scale<FMT>(snap21(u.y));
      }
      sc_all |= (s0 | (s1 << 8)) << (16 * j);
      r_b[2 * j] = s_rcp[s0];
      r_b[2 * j + 1] = s_rcp[s1];
      const float2 D2 = make_float2(s_D[s0], s_D[s1]);
      D_b[2 * j] = D2.x;
      D_b[2 * j + 1] = D2.y;
      const float2 nDq = __fmul2_rn(__fmul2_rn(D2, make_float2(sc, sc)),
                                    make_float2(-0x1p126f, -0x1p126f));
      nDq_b[2 * j] = nDq.x;
      nDq_b[2 * j + 1] = nDq.y;
      // clip levels RD_bf16(6 S g) (exact products, truncated); a zero block gets the largest
      // finite bf16, which no finite |x| exceeds
      const float2 six = __fmul2_rn(D2, make_float2(6.0f, 6.0f));
      uint32_t thr = __byte_perm(__float_as_uint(six.x), __float_as_uint(six.y), 0x7632);
      const uint32_t z2 = bf16x2_set_eq(thr, 0u);
      thr = bf16x2_fma(z2, 0x7F7F7F7Fu, thr);
      S2_b[2 * j] = __byte_perm(thr, thr, 0x1010);
      S2_b[2 * j + 1] = __byte_perm(thr, thr, 0x3232);
      zc2 = bf16x2_add(zc2, z2);
      ss2 = bf16x2_add(ss2, bf16x2_set_gt(M[j], SAT2));
    }
    // codes and every element's scaled square (into its block's sum), one code word at a time;
    // clipped elements counted
    // (measured: for N = 4, converting the item's codes first and then reducing is faster)
    constexpr int PB = BW < 4 ? BW : 4;  // pairs per block inside a code word
    uint32_t cw[NCW];
    float2 lt[NB];
    uint32_t nsat2 = 0u;
#pragma unroll
    for (int b = 0; b < NB; ++b) lt[b] = make_float2(0.0f, 0.0f);
    if constexpr (N >= 8) {
      if (!deep_item<NB>(r_b, sc)) {
#pragma unroll
        for (int c = 0; c < NCW; ++c) {
          const int b0 = (4 * c) / BW;  // block of the code word's first pair
          cw[c] = qs_word8<PB, kFast>(&it.w[4 * c], &r_b[b0], &nDq_b[b0], &S2_b[b0], sc, &lt[b0],
                                      nsat2);
        }
      } else {
#pragma unroll
        for (int c = 0; c < NCW; ++c) {
          const int b0 = (4 * c) / BW;
          cw[c] = qs_word8<PB, kDeep>(&it.w[4 * c], &r_b[b0], &nDq_b[b0], &S2_b[b0], sc, &lt[b0],
                                      nsat2);
        }
      }
    } else {
#pragma unroll
      for (int c = 0; c < NCW; ++c) {
        float q[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int wi = 4 * c + k;
          const uint32_t w = it.w[wi];
          const float2 qq = snap_quotient2(w << 16, w & 0xFFFF0000u, r_b[wi / BW]);
          q[2 * k] = qq.x;
          q[2 * k + 1] = qq.y;
        }
        cw[c] = cvt_e2m1x8(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]);
      }
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        unsigned long long l2 = 0ull;
#pragma unroll
        for (int k = 0; k < BW; ++k) {
          const int wi = b * BW + k;
          const uint32_t w = it.w[wi], lo = w << 16, hi = w & 0xFFFF0000u, c = cw[wi >> 2];
          switch (wi & 3) {
            case 0: pair_step_all<0>(w, lo, hi, c, sc, nDq_b[b], S2_b[b], l2, nsat2); break;
            case 1: pair_step_all<1>(w, lo, hi, c, sc, nDq_b[b], S2_b[b], l2, nsat2); break;
            case 2: pair_step_all<2>(w, lo, hi, c, sc, nDq_b[b], S2_b[b], l2, nsat2); break;
            default: pair_step_all<3>(w, lo, hi, c, sc, nDq_b[b], S2_b[b], l2, nsat2); break;
          }
        }
        asm("mov.b64 {%0, %1}, %2;" : "=f"(lt[b].x), "=f"(lt[b].y) : "l"(l2));
      }
    }
    if constexpr (STORE) {
      if (ok) {
        if constexpr (NCW == 4)
          *reinterpret_cast<uint4*>(packed_out + i * 16) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
        else
          *reinterpret_cast<uint2*>(packed_out + i * 8) = make_uint2(cw[0], cw[1]);
        if constexpr (NB == 2) *reinterpret_cast<uint16_t*>(scales_out + i * 2) = (uint16_t)sc_all;
        else *reinterpret_cast<uint32_t*>(scales_out + i * 4) = sc_all;
      }
    }
    // per block pair: the max elements' errors, then each block's split of its sum
    float ae = 0.0f, am = 0.0f, az = 0.0f;
    bool exact = false;
#pragma unroll
    for (int j = 0; j < NP; ++j) {
      // the two blocks' max elements: code of a / (S g), scaled error, square
      const float2 qa = snap_quotient2v(af[j], make_float2(r_b[2 * j], r_b[2 * j + 1]));
      const uint32_t ca = cvt_e2m1x8(qa.x, qa.y, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f);
      const float2 dec = make_float2(__uint_as_float(e2m1_scaled_bits_at(ca, 0)),
                                     __uint_as_float(e2m1_scaled_bits_at(ca, 4)));
      const float2 dm = __ffma2_rn(dec, make_float2(nDq_b[2 * j], nDq_b[2 * j + 1]),
                                   __fmul2_rn(af[j], make_float2(sc, sc)));
      const float2 f2 = __fmul2_rn(dm, dm);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int b = 2 * j + h;
        const float tb = __fadd_rn(lt[b].x, lt[b].y);
        const float first = h ? f2.y : f2.x;
        const float ab = h ? af[j].y : af[j].x;
        exact |= ab > 0.0f && tb < 0x1p-80f;
        if (D_b[b] > 0.0f) {
          float rest = __fsub_rn(tb, first);
          if (rest < __fmul_rn(first, 0x1p-6f)) {
            // dmax^2 dominates the block: sum the elements below the maximum apart (no
            // cancellation) and add the other max-valued elements' copies of dmax^2
            float rs = 0.0f, nt = 0.0f;
#pragma unroll
            for (int k = 0; k < N; ++k) {
              const int e = b * N + k;
              const uint32_t wd = it.w[e >> 1];
              const float xv = (e & 1) ? bf16hi(wd) : bf16lo(wd);
              const float dq = __uint_as_float(e2m1_scaled_bits_at(cw[e >> 3], 4 * (e & 7)));
              const float d = __fmaf_rn(dq, nDq_b[b], __fmul_rn(xv, sc));
              if (fabsf(xv) != ab) rs = __fmaf_rn(d, d, rs);
              else nt += 1.0f;
              exact |= d != 0.0f && fabsf(d) < 0x1p-63f;  // its square would be lost
            }
            rest = __fmaf_rn(nt - 1.0f, first, rs);
          }
          ae = __fadd_rn(ae, rest);
          am = __fadd_rn(am, first);
        } else {
          az = __fadd_rn(az, tb);
        }
      }
    }
    if (!exact) {
      const double us = unscale_sq(E);
      acc.elem += (double)ae * us;
      acc.mx += (double)am * us;
      acc.zero += (double)az * us;
    } else {
      // exact in double, block by block (first max element by index)
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const int e0 = b * N;
        auto xval = [&](int k) {
          const uint32_t wd = it.w[(e0 + k) >> 1];
          return ((e0 + k) & 1) ? bf16hi(wd) : bf16lo(wd);
        };
        auto code = [&](int k) { return cw[(e0 + k) >> 3] >> (4 * ((e0 + k) & 7)); };
        const float ab = (b & 1) ? af[b >> 1].y : af[b >> 1].x;
        double rest = 0.0, first = 0.0, others = 0.0;
        exact_slice<N, false>(ab, D_b[b], xval, code, rest, first, others);
        if (D_b[b] > 0.0f) {
          acc.elem += rest + others;
          acc.mx += first;
        } else {
          acc.zero += rest + first + others;
        }
      }
    }
    if (ok) {
      acc.n_esat += bf16x2_hsum(nsat2);
      acc.n_zero_f += bf16x2_hsum(zc2);
      acc.n_ssat_f += bf16x2_hsum(ss2);
    }
  };

  Item A, B;
  int64_t i = tid;
  load(A, i);
  while (i < nitems) {
    load(B, i + T);
    process(A, i);
    i += T;
    if (!(i < nitems)) break;
    load(A, i + T);
    process(B, i);
    i += T;
  }
  finish_cta(acc, wk);
}

// ------------------------------------------------------------------------------------------------
// fp32 input (codes recomputed with IEEE division, or read)
// ------------------------------------------------------------------------------------------------

template <int N, int FMT, bool RECOMPUTE>
__global__ void __launch_bounds__(kThreads) k_error_stats_f32(const __grid_constant__ SGroup grp) {
  const SWork wk = s_work(grp);
  const float* __restrict__ x = static_cast<const float*>(wk.t.x);
  const uint8_t* __restrict__ packed = wk.t.packed;
  const uint8_t* __restrict__ scales = wk.t.scales;
  const int64_t nitems = wk.t.nitems;
  const uint16_t g_bits = tensor_g_bits(wk.t.g_bits, wk.t.g_dev);
  using S = SShape<N, float>;
  constexpr int EPT = S::EPT, L = S::L, BPI = S::BPI;
  constexpr int BE = EPT / BPI;
  __shared__ float s_D[256];
  const float g = fp16_bits_to_float(g_bits);
  for (int c = threadIdx.x; c < 256; c += blockDim.x) s_D[c] = __fmul_rn(scale_value(c, FMT), g);
  const float g6 = __fmul_rn(6.0f, g);
  const float sat_thr = __fmul_rn(g6, scale_max<FMT>());
  __syncthreads();
  griddep_wait();  // inputs may come from the previous kernel in the stream
  griddep_launch_next();

  Acc acc;
  const int64_t T = (int64_t)wk.nctas * blockDim.x;
  const int64_t tid = (int64_t)wk.cta * blockDim.x + threadIdx.x;
  const int64_t warp0 = tid - (threadIdx.x & 31);
  const int lane = threadIdx.x & 31;

  for (int64_t base = 0; warp0 + base < nitems; base += T) {
    const int64_t i = tid + base;
    const bool ok = i < nitems;
    float v[EPT];
#pragma unroll
    for (int h = 0; h < EPT / 4; ++h) {
      uint4 t = make_uint4(0, 0, 0, 0);
      if (ok) t = ld_stream16(x + i * EPT + h * 4);
      v[4 * h] = __uint_as_float(t.x); v[4 * h + 1] = __uint_as_float(t.y);
      v[4 * h + 2] = __uint_as_float(t.z); v[4 * h + 3] = __uint_as_float(t.w);
    }
    uint32_t cw = 0, scw = 0;
    if (!RECOMPUTE && ok) {
      cw = reinterpret_cast<const unsigned int*>(packed)[i];
      scw = (BPI == 1) ? scales[i / L] : reinterpret_cast<const unsigned short*>(scales)[i];
    }
#pragma unroll
    for (int b = 0; b < BPI; ++b) {
      const float* vb = &v[b * BE];
      float a = 0.0f;
      uint32_t mn = 0x7FFFFFFFu;
#pragma unroll
      for (int k = 0; k < BE; ++k) {
        a = fmaxf(a, fabsf(vb[k]));
        mn = min(mn, __float_as_uint(vb[k]) & 0x7FFFFFFFu);
      }
#pragma unroll
      for (int off = 1; off < L; off <<= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
      uint32_t s, bc = 0;
      if constexpr (RECOMPUTE) {
        s = encode_scale<FMT>(__fdiv_rn(a, g6));
        const float D0 = s_D[s];
        float q[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
          q[k] = (k < BE && D0 > 0.0f) ? __fdiv_rn(vb[k < BE ? k : 0], D0)
                                       : __fmul_rn(k < BE ? vb[k < BE ? k : 0] : 0.0f, 0.0f);
        bc = cvt_e2m1x8(q[0], q[1], q[2], q[3], q[4], q[5], q[6], q[7]);
      } else {
        s = (scw >> (8 * b)) & 0xFF;
        bc = cw >> (4 * b * BE);
      }
      const float D = s_D[s];
      auto xval = [&](int k) { return vb[k]; };
      auto code = [&](int k) { return bc >> (4 * k); };
      block_slice<BE, L>(acc, lane, ok, a, D, sat_thr, __uint_as_float(mn), xval, code);
    }
  }
  finish_cta(acc, wk);
}

// ------------------------------------------------------------------------------------------------
// N = 4 tail (4 elements) and the final reduction
// ------------------------------------------------------------------------------------------------

// The elements after the last whole item (count of them, a multiple of the block size N <= 16):
// one thread, block by block, in double; codes recomputed (packed == nullptr) or read.
template <int FMT, typename T>
__global__ void k_error_stats_tail(const T* __restrict__ x, int64_t first, int count, int N,
                                   uint16_t g_bits, const uint16_t* g_dev,
                                   const uint8_t* __restrict__ packed,
                                   const uint8_t* __restrict__ scales, StatsPartial* part) {
  if (threadIdx.x != 0) return;
  const float g = fp16_bits_to_float(tensor_g_bits(g_bits, g_dev));
  StatsPartial p{};
  for (int b0 = 0; b0 < count; b0 += N) {
    const int64_t f = first + b0;
    float v[16], a = 0.0f;
    int imax = 0;
    for (int k = 0; k < N; ++k) {
      if constexpr (sizeof(T) == 2)
        v[k] = __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(x)[f + k] << 16);
      else
        v[k] = reinterpret_cast<const float*>(x)[f + k];
      if (fabsf(v[k]) > a) { a = fabsf(v[k]); imax = k; }
    }
    uint32_t s, codes[16];
    if (packed == nullptr) {
      s = encode_scale<FMT>(__fdiv_rn(a, __fmul_rn(6.0f, g)));
      const float D0 = __fmul_rn(scale_value((int)s, FMT), g);
      for (int k = 0; k < N; ++k) {
        const float q = D0 > 0.0f ? __fdiv_rn(v[k], D0) : __fmul_rn(v[k], 0.0f);
        codes[k] = cvt_e2m1x8(q, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f) & 0xF;
      }
    } else {
      s = scales[f / N];
      for (int k = 0; k < N; ++k) codes[k] = (packed[(f + k) / 2] >> (4 * ((f + k) & 1))) & 0xF;
    }
    const float D = __fmul_rn(scale_value((int)s, FMT), g);
    for (int k = 0; k < N; ++k) {
      const double y = (double)__fmul_rn(e2m1_to_float(codes[k]), D);
      const double d = (double)v[k] - y;
      if (!(D > 0.0f)) p.sse_zero += (double)v[k] * (double)v[k];
      else if (k == imax) p.sse_max += d * d;
      else p.sse_elem += d * d;
      if (D > 0.0f && fabsf(v[k]) > __fmul_rn(6.0f, D)) p.n_elem_sat += 1;
    }
    p.n_zero_blocks += (D > 0.0f) ? 0 : 1;
    p.n_scale_sat += (a > __fmul_rn(__fmul_rn(6.0f, g), scale_max<FMT>())) ? 1 : 0;
  }
  part[0] = p;
}

// Adds nparts partials in a fixed order (thread t takes t, t + 256, ...; then warps, then the 8
// warp sums in order) and writes the result record.  Run by all threads of one CTA.
__device__ void final_reduce(const StatsPartial* part, int nparts, const StatsPartial* extra,
                             int64_t numel, int64_t nblocks, StatsOut* out) {
  double e = 0.0, m = 0.0, z = 0.0;
  unsigned long long c0 = 0, c1 = 0, c2 = 0;
  const int n = nparts + (extra != nullptr);
  for (int k = threadIdx.x; k < n; k += blockDim.x) {
    const StatsPartial* src = k < nparts ? part + k : extra;
    const double* pd = reinterpret_cast<const double*>(src);
    const unsigned long long* pu = reinterpret_cast<const unsigned long long*>(src);
    e += __ldcg(pd + 0); m += __ldcg(pd + 1); z += __ldcg(pd + 2);
    c0 += __ldcg(pu + 4); c1 += __ldcg(pu + 5); c2 += __ldcg(pu + 6);
  }
  __shared__ double sd[3][kThreads / 32];
  __shared__ unsigned long long su[3][kThreads / 32];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  e = warp_sum(e); m = warp_sum(m); z = warp_sum(z);
  c0 = warp_sum(c0); c1 = warp_sum(c1); c2 = warp_sum(c2);
  if (lane == 0) {
    sd[0][w] = e; sd[1][w] = m; sd[2][w] = z;
    su[0][w] = c0; su[1][w] = c1; su[2][w] = c2;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    StatsOut o{};
    for (int k = 0; k < kThreads / 32; ++k) {
      o.sse_elem += sd[0][k]; o.sse_max += sd[1][k]; o.sse_zero += sd[2][k];
      o.n_zero_blocks += (long long)su[0][k]; o.n_scale_sat += (long long)su[1][k];
      o.n_elem_sat += (long long)su[2][k];
    }
    o.numel = numel;
    o.n_blocks = nblocks;
    *out = o;
  }
}

__global__ void __launch_bounds__(kThreads) k_error_stats_final(const StatsPartial* __restrict__ part,
                                                                int nparts,
                                                                const StatsPartial* extra,
                                                                int64_t numel, int64_t nblocks,
                                                                StatsOut* __restrict__ out) {
  final_reduce(part, nparts, extra, numel, nblocks, out);
}

// ------------------------------------------------------------------------------------------------
// launcher
// ------------------------------------------------------------------------------------------------

// Workspace layout: kMaxGroup 64-byte headers (the last-CTA counter of tensor t of a group in
// header t), then 64-byte partials: the main pass's CTAs in grid order, then one slot per tensor
// for an N = 4 tail.
struct Workspace {
  unsigned int* counters;
  StatsPartial* part;
  explicit Workspace(void* ws)
      : counters(reinterpret_cast<unsigned int*>(ws)),
        part(reinterpret_cast<StatsPartial*>(reinterpret_cast<char*>(ws) + 64 * kMaxGroup)) {}
  unsigned int* counter(int t) const { return counters + 16 * t; }
};
constexpr int kMaxStatsGrid = kMaxReduceCtas - 2 * kMaxGroup;  // headers + tail slots

cudaError_t launch_stats_final(const StatsPartial* part, int nparts, int64_t numel,
                               int64_t nblocks, void* out, cudaStream_t stream, int* launches) {
  k_error_stats_final<<<1, kThreads, 0, stream>>>(part, nparts, nullptr, numel, nblocks,
                                                  static_cast<StatsOut*>(out));
  ++*launches;
  return cudaGetLastError();
}

// Zeroes the last-CTA counters of a group once the previous kernel in the stream is done with
// them (launched with programmatic serialization, so its launch overlaps that kernel's tail and
// the main pass's launch overlaps it).
__global__ void k_stats_reset(unsigned int* counters, int n) {
  griddep_wait();
  if ((int)threadIdx.x < n) counters[16 * threadIdx.x] = 0;
  griddep_launch_next();
}

cudaError_t launch_counter_reset(unsigned int* counter, cudaStream_t stream, int* launches) {
  return launch_counters_reset(counter, 1, stream, launches);
}

cudaError_t launch_counters_reset(unsigned int* counters, int n, cudaStream_t stream,
                                  int* launches) {
  const cudaError_t e = launch_pdl(k_stats_reset, 1, 32, stream, counters, n);
  if (e == cudaSuccess) ++*launches;
  return e;
}

// Main pass over the group; then, for each tensor the main pass does not finish, its tail (the
// elements after the last whole item: N <= 16 only) and a one-CTA final pass, or (no items) the
// final pass alone.  Without a tail the main pass adds a tensor's partials itself.
template <int N, int FMT, typename T, int MODE>
static cudaError_t launch_stats(const TensorArgs* ta, int count, int block, Workspace ws,
                                cudaStream_t stream, int* launches) {
  using S = SShape<N, T>;
  constexpr bool RC = MODE != kGiven;
  // bf16 with recomputed codes and N <= 16: the small-block kernel
  constexpr bool SMALL = sizeof(T) == 2 && RC && N <= 16;
  constexpr int EPT = SMALL ? QSShape<N>::EPT : S::EPT;
  SGroup grp = {};
  int64_t nitems[kMaxGroup];
  bool tail[kMaxGroup];
  for (int k = 0; k < count; ++k) {
    nitems[k] = ta[k].numel / EPT;
    tail[k] = ta[k].numel % EPT != 0;
  }
  const void* kern;
  if constexpr (SMALL) kern = (const void*)k_qstats_small<N, FMT, MODE>;
  else if constexpr (sizeof(T) == 2) kern = (const void*)k_error_stats_bf16<N, FMT, MODE>;
  else kern = (const void*)k_error_stats_f32<N, FMT, RC>;
  const int grid = split_grid(kern, nitems, count, S::U, kMaxStatsGrid, &grp.split);
  bool any_counter = false;
  for (int k = 0; k < count; ++k) {
    const bool counted = !tail[k] && nitems[k] > 0;
    any_counter |= counted;
    grp.t[k] = {ta[k].x,
                MODE == kGiven ? ta[k].packed : nullptr,
                MODE == kGiven ? ta[k].scales : nullptr,
                MODE == kStore ? ta[k].packed : nullptr,
                MODE == kStore ? ta[k].scales : nullptr,
                ws.part + grp.split.begin[k],
                counted ? ws.counter(k) : nullptr,
                (StatsOut*)ta[k].stats,
                nitems[k],
                ta[k].numel,
                ta[k].numel / block,
                ta[k].g_bits,
                ta[k].g_dev};
  }
  if (grid > 0) {
    if (any_counter) {
      const cudaError_t e = launch_pdl(k_stats_reset, 1, 32, stream, ws.counters, count);
      if (e != cudaSuccess) return e;
      ++*launches;
    }
    cudaError_t e;
    if constexpr (SMALL)
      e = launch_pdl(k_qstats_small<N, FMT, MODE>, grid, kThreads, stream, grp);
    else if constexpr (sizeof(T) == 2)
      e = launch_pdl(k_error_stats_bf16<N, FMT, MODE>, grid, kThreads, stream, grp);
    else
      e = launch_pdl(k_error_stats_f32<N, FMT, RC>, grid, kThreads, stream, grp);
    if (e != cudaSuccess) return e;
    ++*launches;
  }
  for (int k = 0; k < count; ++k) {
    if (!tail[k] && nitems[k] > 0) continue;
    StatsPartial* extra = nullptr;
    if (tail[k]) {
      extra = ws.part + grid + k;
      const int64_t first = nitems[k] * EPT;
      const int count = (int)(ta[k].numel - first);  // < EPT, a multiple of N <= 16
      if (MODE == kStore) {  // quantize the last elements, then reduce them from the codes
        const cudaError_t e = run_quantize_tail(ta[k].x, sizeof(T) == 2, first, count, N, FMT,
                                                ta[k].g_bits, ta[k].g_dev, ta[k].packed,
                                                ta[k].scales, stream, launches);
        if (e != cudaSuccess) return e;
      }
      k_error_stats_tail<FMT, T><<<1, 32, 0, stream>>>(
          (const T*)ta[k].x, first, count, N, ta[k].g_bits, ta[k].g_dev,
          MODE == kRecompute ? nullptr : ta[k].packed, ta[k].scales, extra);
      ++*launches;
    }
    const int nparts = nitems[k] > 0 ? grp.split.begin[k + 1] - grp.split.begin[k] : 0;
    k_error_stats_final<<<1, kThreads, 0, stream>>>(ws.part + grp.split.begin[k], nparts, extra,
                                                    ta[k].numel, ta[k].numel / block,
                                                    (StatsOut*)ta[k].stats);
    ++*launches;
  }
  return cudaGetLastError();
}

template <int FMT, typename T, int MODE>
static cudaError_t stats_block(int block, const TensorArgs* t, int count, Workspace ws,
                               cudaStream_t st, int* n) {
  switch (block) {
    case 4: return launch_stats<4, FMT, T, MODE>(t, count, block, ws, st, n);
    case 8: return launch_stats<8, FMT, T, MODE>(t, count, block, ws, st, n);
    case 16: return launch_stats<16, FMT, T, MODE>(t, count, block, ws, st, n);
    case 32: return launch_stats<32, FMT, T, MODE>(t, count, block, ws, st, n);
    case 64: return launch_stats<64, FMT, T, MODE>(t, count, block, ws, st, n);
    case 128: return launch_stats<128, FMT, T, MODE>(t, count, block, ws, st, n);
    default: return launch_stats<256, FMT, T, MODE>(t, count, block, ws, st, n);
  }
}

template <int FMT, typename T>
static cudaError_t stats_mode(StatsMode mode, int block, const TensorArgs* t, int count,
                              Workspace ws, cudaStream_t st, int* n) {
  switch (mode) {
    case kGiven: return stats_block<FMT, T, kGiven>(block, t, count, ws, st, n);
    case kRecompute: return stats_block<FMT, T, kRecompute>(block, t, count, ws, st, n);
    default: return stats_block<FMT, T, kStore>(block, t, count, ws, st, n);
  }
}

// Row-pitched mode of k_error_stats_bf16 over one bf16 tensor (rows whose length the block size
// N >= 32 does not divide, cols % 8 == 0), recomputed codes, stored (STORE) or not.
template <int N, int FMT, bool STORE>
static cudaError_t launch_stats_rows(const void* x, int64_t rows, int64_t cols, uint16_t g_bits,
                                     const uint16_t* g_dev, uint8_t* packed, uint8_t* scales,
                                     void* out, Workspace ws, cudaStream_t stream,
                                     int* launches) {
  constexpr int MODE = STORE ? kStore : kRecompute;
  using S = SShape<N, uint16_t>;
  static_assert(N >= S::EPT, "whole items per block");
  const int64_t nb = (cols + N - 1) / N, ipr = nb * (N / S::EPT);
  const int64_t nitems = rows * ipr;
  SGroup grp = {};
  grp.t[0] = {x, nullptr, nullptr, STORE ? packed : nullptr, STORE ? scales : nullptr, ws.part,
              ws.counter(0), static_cast<StatsOut*>(out), nitems, rows * cols, rows * nb,
              g_bits, g_dev, cols, ipr, (cols + 1) / 2, nb};
  const int grid = split_grid((const void*)k_error_stats_bf16<N, FMT, MODE, true>, &nitems, 1,
                              S::U, kMaxStatsGrid, &grp.split);
  cudaError_t e = launch_pdl(k_stats_reset, 1, 32, stream, ws.counters, 1);
  if (e != cudaSuccess) return e;
  ++*launches;
  e = launch_pdl(k_error_stats_bf16<N, FMT, MODE, true>, grid, kThreads, stream, grp);
  if (e == cudaSuccess) ++*launches;
  return e;
}

template <int FMT, bool STORE>
static cudaError_t stats_rows_block(int block, const void* x, int64_t rows, int64_t cols,
                                    uint16_t g_bits, const uint16_t* g_dev, uint8_t* packed,
                                    uint8_t* scales, void* out, Workspace ws, cudaStream_t st,
                                    int* n) {
  switch (block) {
    case 32: return launch_stats_rows<32, FMT, STORE>(x, rows, cols, g_bits, g_dev, packed, scales, out, ws, st, n);
    case 64: return launch_stats_rows<64, FMT, STORE>(x, rows, cols, g_bits, g_dev, packed, scales, out, ws, st, n);
    case 128: return launch_stats_rows<128, FMT, STORE>(x, rows, cols, g_bits, g_dev, packed, scales, out, ws, st, n);
    default: return launch_stats_rows<256, FMT, STORE>(x, rows, cols, g_bits, g_dev, packed, scales, out, ws, st, n);
  }
}

bool rows_stats_supported(bool bf16, int64_t rows, int64_t cols, int block) {
  return bf16 && block >= 32 && cols % 8 == 0 && rows >= 1;
}

cudaError_t run_rows_stats(const void* x, int64_t rows, int64_t cols, int block, int fmt,
                           uint16_t g_bits, const uint16_t* g_dev, uint8_t* packed,
                           uint8_t* scales, void* out, void* workspace, cudaStream_t stream,
                           int* launches) {
  const Workspace ws(workspace);
  if (packed)
    return fmt == kUE5M3 ? stats_rows_block<kUE5M3, true>(block, x, rows, cols, g_bits, g_dev, packed, scales, out, ws, stream, launches)
                         : stats_rows_block<kE4M3, true>(block, x, rows, cols, g_bits, g_dev, packed, scales, out, ws, stream, launches);
  return fmt == kUE5M3 ? stats_rows_block<kUE5M3, false>(block, x, rows, cols, g_bits, g_dev, nullptr, nullptr, out, ws, stream, launches)
                       : stats_rows_block<kE4M3, false>(block, x, rows, cols, g_bits, g_dev, nullptr, nullptr, out, ws, stream, launches);
}

cudaError_t run_stats_group(const TensorArgs* t, int count, bool bf16, int block, int fmt,
                            StatsMode mode, void* workspace, cudaStream_t stream, int* launches) {
  const Workspace ws(workspace);
  if (!bf16 && mode == kStore) {  // fp32 input: quantize, then reduce from the stored codes
    const cudaError_t e = run_quantize_group(t, count, false, block, fmt, stream, launches);
    if (e != cudaSuccess) return e;
    mode = kGiven;
  }
  if (bf16)
    return fmt == kUE5M3 ? stats_mode<kUE5M3, uint16_t>(mode, block, t, count, ws, stream, launches)
                         : stats_mode<kE4M3, uint16_t>(mode, block, t, count, ws, stream, launches);
  return fmt == kUE5M3 ? stats_mode<kUE5M3, float>(mode, block, t, count, ws, stream, launches)
                       : stats_mode<kE4M3, float>(mode, block, t, count, ws, stream, launches);
}

cudaError_t run_quantize_stats(const void* x, bool bf16, int64_t numel, int block, int fmt,
                               uint16_t g_bits, uint8_t* packed, uint8_t* scales, void* out,
                               void* workspace, cudaStream_t stream, int* launches) {
  const TensorArgs t = {x, nullptr, packed, scales, out, numel, g_bits};
  return run_stats_group(&t, 1, bf16, block, fmt, kStore, workspace, stream, launches);
}

cudaError_t run_error_stats(const void* x, bool bf16, int64_t numel, int block, int fmt,
                            uint16_t g_bits, const uint8_t* packed, const uint8_t* scales,
                            void* out, void* workspace, cudaStream_t stream, int* launches) {
  const TensorArgs t = {x, nullptr, const_cast<uint8_t*>(packed), const_cast<uint8_t*>(scales),
                        out, numel, g_bits};
  return run_stats_group(&t, 1, bf16, block, fmt, packed ? kGiven : kRecompute, workspace, stream,
                         launches);
}

}  // namespace mxk
