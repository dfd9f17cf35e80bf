/*
 * mx_oracle.h -- plain CPU definition of block-wise FP4 microscaling (test infrastructure).
 *
 * THIS IS TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.  Only the test-suite, the smoke check and
 * the CPU-baseline leg of the benchmark may load it.  It shares no code, header, table or constant
 * with the CUDA library: it decodes every number format from its closed form and rounds by
 * searching the decoded code table for the nearest value, in double precision.
 *
 * Sources (the method is defined only in prose and formulas):
 *   [MX]  the microscaling article at hotelren.com/news/2192771 (page titled
 *         "企业官网建设流程全解析"; the body is about FP4 + FP8 microscaling):
 *         §1 (FP4 E2M1 elements, FP8 block scales, blocks of 4-256 values),
 *         §2.2 items 1-3 (the three error sources), §3.1 item 1 (E4M3 vs UE5M3 exponent widths),
 *         §3.1 item 2 (quantize_block: scale = Q_fp8(absmax/6), q = Q_fp4(block/scale)),
 *         §3.1 item 3 (value = FP4 x FP8_scale x FP16_scale).
 *   [F4]  the 4-bit float quantization article at gtnt.cn/news/16247: §1 (sign/2-bit exponent/
 *         1-bit mantissa layout), §4.3 (two FP4 values stored per byte).
 *
 * Readings where the pages are silent or garbled (each is listed with its reason in the design
 * notes of the repository):
 *   - rounding is round-to-nearest, ties to the even code, saturating at the largest finite value;
 *   - E2M1 has no inf/NaN (all 16 codes finite); E4M3 is the OCP "FN" variant (bias 7, max 448,
 *     0x7F/0xFF NaN, never produced); UE5M3 is unsigned, bias 15, subnormals, every code finite,
 *     max 122880;
 *   - blocks are N consecutive elements of a row, from its first element; when N does not divide
 *     cols the last block of each row holds the cols mod N remaining elements (its own absmax and
 *     scale, the same element rule);
 *   - element 2k of a row goes to the low nibble of byte k, element 2k+1 to the high nibble; a
 *     row's codes take ceil(cols/2) bytes (an odd last element leaves the high nibble 0) and its
 *     scales ceil(cols/N) bytes;
 *   - the code's sign bit is the sign bit of x, also in zero-scale blocks and for -0.0;
 *   - the error terms are sums over the tensor; each MSE is its sum divided by rows*cols;
 *   - the per-tensor FP16 scale chosen by orc_global_scale is the smallest FP16 value g with
 *     g * 6 * Smax >= max|x| (1.0 for an all-zero tensor, clamped to 65504).
 */
#ifndef MX_ORACLE_H
#define MX_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* element dtypes of x / y */
#define ORC_F32 0
#define ORC_BF16 1
/* scale formats */
#define ORC_E4M3 0
#define ORC_UE5M3 1

typedef struct {
  double sse_elem;  /* [MX] §2.2 item 1: squared error of the non-max elements of blocks with S>0 */
  double sse_max;   /* [MX] §2.2 item 2: squared error of the max element of blocks with S>0 */
  double sse_zero;  /* [MX] §2.2 item 3: sum of x^2 over blocks whose scale is zero */
  int64_t numel, n_blocks, n_zero_blocks, n_scale_sat, n_elem_sat;
} orc_stats;

/* closed-form decoders (return NaN for NaN codes) */
double orc_e2m1_value(int code);   /* 4-bit code, sign in bit 3 */
double orc_e4m3_value(int code);   /* 8-bit code */
double orc_ue5m3_value(int code);  /* 8-bit code */
double orc_scale_value(int code, int fmt);
double orc_fp16_value(uint16_t bits);
double orc_bf16_value(uint16_t bits);

/* nearest-value rounding (ties to the even code, saturating); u, v >= 0 */
int orc_round_scale(double u, int fmt);
int orc_round_e2m1_mag(double v);
/* largest finite scale value and smallest positive one of a format */
double orc_scale_max(int fmt);
double orc_scale_min(int fmt);

/* Quantize a row-major rows x cols tensor (bf16 bits or float32) in blocks of `block` columns.
 * packed: rows*cols/2 bytes; scales: rows*cols/block bytes.  Returns 0, or -1 on bad arguments. */
int orc_quantize(const void* x, int xdtype, int64_t rows, int64_t cols, int block, int fmt,
                 uint16_t g_bits, uint8_t* packed, uint8_t* scales, int nthreads);

/* Reconstruct y = E2M1(code) * S(scale) * g, written as float32 or bf16 (round to nearest even). */
int orc_dequantize(const uint8_t* packed, const uint8_t* scales, int64_t rows, int64_t cols,
                   int block, int fmt, uint16_t g_bits, void* y, int ydtype, int nthreads);

/* Three-term error reduction.  packed/scales NULL: quantize x first (same rule as orc_quantize);
 * otherwise use the given codes.  The reconstruction used is the exact value E2M1*S*g. */
int orc_error_stats(const void* x, int xdtype, int64_t rows, int64_t cols, int block, int fmt,
                    uint16_t g_bits, const uint8_t* packed, const uint8_t* scales, orc_stats* out,
                    int nthreads);

/* Per-tensor FP16 scale (bit pattern), see the reading above. */
uint16_t orc_global_scale(const void* x, int xdtype, int64_t numel, int fmt);

#ifdef __cplusplus
}
#endif
#endif
