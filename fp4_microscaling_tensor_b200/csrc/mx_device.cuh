// mx_device.cuh -- device helpers of the sm_100a FP4 microscaling kernels.
//
// Exactness argument used by the bf16 fast path (the microscaling article, hotelren.com/news/
// 2192771, §3.1 item 2 divides by the scale; these helpers replace the division):
//   Let D be a divisor with at most 15 significant bits (6g, or S*g with S an FP8 value and g an
//   FP16 value), r = RN(1/D) in fp32 and x a bf16 value (8 significant bits).  q0 = RN(x*r) is within
//   2^-23 (relative) of the exact quotient q = x/D.  Every rounding midpoint t of the E2M1 grid and
//   of the FP8 grids has at most 5 significant bits, so t*D has at most 18 and, when q != t,
//   |x - t*D| is at least one unit in the 18th place: |q - t| > t * 2^-18.  Rounding q0 to 21
//   significant bits (snap21) therefore lands exactly on t when q == t, and on the same side of
//   every midpoint as q otherwise.  RNE of snap21(q0) to the narrow grid equals RNE of q.
// The fp32 input path has 24-bit x, where that margin does not hold; it uses the IEEE division
// (correctly rounded), whose result is a midpoint only when q is (the quotient of a 24-bit and a
// 15-bit number is never within half an fp32 ulp of a short midpoint without being equal to it).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace mxk {

constexpr int kThreads = 256;  // threads per CTA of every streaming kernel
constexpr int kE4M3 = 0;
constexpr int kUE5M3 = 1;

// Largest finite scale value of a format (E4M3: 0x7E = 448, UE5M3: 0xFF = 122880).
template <int FMT>
__host__ __device__ constexpr float scale_max() {
  return FMT == kUE5M3 ? 122880.0f : 448.0f;
}

// Exact fp32 value of an 8-bit scale code (all 256 codes; E4M3 keeps its sign bit, 0x7F/0xFF NaN).
__device__ __forceinline__ float scale_value(int code, int fmt) {
  if (fmt == kUE5M3) {
    const int e = code >> 3, m = code & 7;
    if (e == 0) return __fmul_rn((float)m, 0x1p-17f);
    return __uint_as_float(((uint32_t)(e + 112) << 23) | ((uint32_t)m << 20));
  }
  const int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
  float v;
  if (e == 15 && m == 7)
    v = __uint_as_float(0x7fc00000u);
  else if (e == 0)
    v = __fmul_rn((float)m, 0x1p-9f);
  else
    v = __uint_as_float(((uint32_t)(e + 120) << 23) | ((uint32_t)m << 20));
  return s ? -v : v;
}

__device__ __forceinline__ float fp16_bits_to_float(uint16_t b) {
  return __half2float(__ushort_as_half(b));
}

// Round an fp32 value to 21 significant bits (drop 3 mantissa bits, half-up on the magnitude).
__device__ __forceinline__ float snap21(float v) {
  return __uint_as_float((__float_as_uint(v) + 4u) & ~7u);
}

// Quotients x / (S g) of two elements (lo / hi: their fp32 bits) for the E2M1 conversion, on the
// FMA pipe.  r = RN(1 / (S g)), so x r is within 2^-21 of the true quotient t when |t| <= 8.
// Adding 48 (whose binade [32, 64) has spacing 2^-18) and subtracting it again rounds x r onto that
// grid exactly (Sterbenz for the subtraction).  A midpoint of the E2M1 grid (a multiple of 1/4) is
// then hit exactly when t is one.  Otherwise (x is bf16 with 8 significant bits, S g has at most
// 15) t lies more than 2^-18 from every midpoint: at least 1.25 * 2^-18 from the 3-significant-bit
// midpoints 1.25, 1.75, 2.5, 3.5 and 5, at least 2^-17 from the others.  That margin exceeds half
// the grid spacing (2^-19) plus the product error (2^-21), so the rounded value stays on t's side.
// Larger |t| only has to stay above 6, which it does.
// Signs: the subtraction rounds toward -inf, so a quotient that cancels to zero is -0; the final
// FMA adds x 2^-60, which leaves any non-zero quotient unchanged (|x| 2^-60 is below a quarter of
// its unit in the last place, since r >= 2^-33) and gives a zero quotient the sign of x (+0 + -0 is
// +0, -0 + -0 is -0): the E2M1 code's sign bit always follows x.
__device__ __forceinline__ float2 snap_quotient2(uint32_t lo, uint32_t hi, float r) {
  const float2 x = make_float2(__uint_as_float(lo), __uint_as_float(hi));
  const float2 y = __ffma2_rn(x, make_float2(r, r), make_float2(48.0f, 48.0f));
  const float2 q = __fadd2_rd(y, make_float2(-48.0f, -48.0f));
  return __ffma2_rn(x, make_float2(0x1p-60f, 0x1p-60f), q);
}

// FP8 code of u >= 0 (already exact or snapped), nearest-even, saturating.
template <int FMT>
__device__ __forceinline__ uint32_t encode_scale(float u) {
  if constexpr (FMT == kE4M3) {
    unsigned short h;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(h) : "f"(0.0f), "f"(u));
    return (uint32_t)(h & 0xFFu);
  } else {
    // UE5M3 normal range (u >= 2^-14): rebias the fp32 exponent by -112, round the 23-bit
    // mantissa to 3 bits (nearest, ties to even; a carry moves into the exponent), clamp at 0xFF.
    const uint32_t b = __float_as_uint(u);
    uint32_t t = b - (112u << 23);
    t += 0x7FFFFu + ((t >> 20) & 1u);
    const uint32_t cn = min(t >> 20, 255u);
    // subnormal range: the code is u / 2^-17 rounded to an integer (8 = the smallest normal)
    const uint32_t cs = __float2uint_rn(__fmul_rn(u, 131072.0f));
    return b >= (113u << 23) ? cn : cs;
  }
}

// Four element pairs -> four bytes of E2M1 codes in one word; v[2k] goes to the low nibble of
// byte k.  The converter rounds to nearest even and saturates at +-6; the sign is kept for zeros.
__device__ __forceinline__ uint32_t cvt_e2m1x8(float v0, float v1, float v2, float v3, float v4,
                                              float v5, float v6, float v7) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
  return r;
}

// E2M1 decode by bit arithmetic (exact; no conversion instruction).  The three magnitude bits of a
// code placed at bits 22..24 form a binary32 whose exponent field is the code's exponent field and
// whose top mantissa bit is the code's mantissa bit (code 1 lands in the subnormal range), i.e. the
// code's value times 2^-126; the sign goes to bit 31.  e2m1_scaled_bits gives that pattern for the
// nibble at bit position P of w; multiplying by 2^126 restores the value.
template <int P>
__device__ __forceinline__ uint32_t e2m1_scaled_bits(uint32_t w) {
  // move the nibble to bits 28..31, then an arithmetic shift by 6 copies the sign over bits 25..31
  // and leaves the magnitude at 22..24
  const int32_t t = (int32_t)(P <= 28 ? (w << (28 - P)) : w);
  return (uint32_t)(t >> 6) & 0x81C00000u;
}

// Same, for a nibble position p that is a compile-time constant after unrolling.
__device__ __forceinline__ uint32_t e2m1_scaled_bits_at(uint32_t w, int p) {
  return (uint32_t)((int32_t)(w << (28 - p)) >> 6) & 0x81C00000u;
}

__device__ __forceinline__ float e2m1_to_float(uint32_t nib) {
  return __fmul_rn(__uint_as_float(e2m1_scaled_bits<0>(nib)), 0x1p126f);
}

// max(|a|, |b|) per bf16 half (the sign of the result is meaningless; callers mask it).
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Programmatic dependent launch: wait until the previous grid in the stream has completed and its
// memory is visible (a no-op without such a dependency); then allow the next grid to be scheduled.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_next() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// g of one tensor: its binary16 bit pattern, or, when g_dev is set, the value the previous kernel
// in the stream wrote there (the global-scale launch); that read first waits for that kernel.
__device__ __forceinline__ uint16_t tensor_g_bits(uint32_t g_bits, const uint16_t* g_dev) {
  if (g_dev == nullptr) return (uint16_t)g_bits;
  griddep_wait();
  return __ldcg(g_dev);
}

// Row and item of a linear item index in a space of rows x ipr items (a row-pitched tensor seen as
// whole items per row), moved on by a fixed stride without a division per step: the stride is
// split once into whole rows and an item step.
struct RowCursor {
  int64_t row, j;  // current row and item within the row
  int64_t dr, dj, ipr;
  __device__ __forceinline__ void init(int64_t i, int64_t stride, int64_t items_per_row) {
    ipr = items_per_row;
    row = i / ipr;
    j = i - row * ipr;
    dr = stride / ipr;
    dj = stride - dr * ipr;
  }
  __device__ __forceinline__ void advance() {
    j += dj;
    row += dr;
    if (j >= ipr) {
      j -= ipr;
      ++row;
    }
  }
};

// Streaming 16-byte load of read-only data (not kept in L1).
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // round to nearest even
  return *reinterpret_cast<uint32_t*>(&h);
}

}  // namespace mxk
