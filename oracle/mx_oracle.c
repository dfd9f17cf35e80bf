/*
 * mx_oracle.c -- plain CPU definition of block-wise FP4 microscaling (TEST INFRASTRUCTURE).
 *
 * Only the test-suite, the smoke check and the benchmark's CPU-baseline leg may load this file's
 * library.  Nothing here is shared with the CUDA library.  The method is followed step by step as
 * the microscaling article states it ([MX], hotelren.com/news/2192771, §3.1 item 2):
 *
 *     abs_max = max|block|;  scale = Q_fp8(abs_max / 6);  q = Q_fp4(block / scale)
 *
 * with the per-tensor FP16 factor of [MX] §3.1 item 3 folded in (abs_max / (6 g), block / (scale g)).
 * Every quotient is formed in double.  Because x has at most 24 significant bits and every divisor
 * (6 g, S g) at most 15, a double quotient is never rounded onto, or off, a rounding midpoint of
 * the 4- or 8-bit target grids, so the nearest-value search below sees the exact real quotient's
 * position.  Rounding is a scan over the decoded code table: the code with the smallest distance
 * wins, and of two equidistant codes the even one.  Threads only split rows, for speed.
 */
#include "mx_oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------------------ */
/* number formats, from their closed forms                                                     */
/* ------------------------------------------------------------------------------------------ */

/* FP4 E2M1 ([MX] §1; [F4] §1): sign | 2-bit exponent (bias 1) | 1-bit mantissa, no inf/NaN. */
double orc_e2m1_value(int code) {
  int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  double mag = (e == 0) ? 0.5 * m : (1.0 + 0.5 * m) * ldexp(1.0, e - 1);
  return s ? -mag : mag;
}

/* FP8 E4M3, OCP "FN" variant ([MX] §3.1 item 1 "standard E4M3"): bias 7, subnormals, NaN at
 * exponent 15 / mantissa 7, no inf. */
double orc_e4m3_value(int code) {
  int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
  double mag;
  if (e == 15 && m == 7) return NAN;
  mag = (e == 0) ? m * ldexp(1.0, -9) : (1.0 + m / 8.0) * ldexp(1.0, e - 7);
  return s ? -mag : mag;
}

/* FP8 UE5M3 ([MX] §3.1 item 1: the sign bit becomes a fifth exponent bit): unsigned, bias 15,
 * subnormals, every one of the 256 codes finite. */
double orc_ue5m3_value(int code) {
  int e = (code >> 3) & 31, m = code & 7;
  return (e == 0) ? m * ldexp(1.0, -17) : (1.0 + m / 8.0) * ldexp(1.0, e - 15);
}

double orc_scale_value(int code, int fmt) {
  return fmt == ORC_UE5M3 ? orc_ue5m3_value(code & 255) : orc_e4m3_value(code & 255);
}

double orc_scale_max(int fmt) { return fmt == ORC_UE5M3 ? orc_ue5m3_value(0xFF) : orc_e4m3_value(0x7E); }
double orc_scale_min(int fmt) { return fmt == ORC_UE5M3 ? orc_ue5m3_value(0x01) : orc_e4m3_value(0x01); }

/* IEEE binary16: sign | 5-bit exponent (bias 15) | 10-bit mantissa. */
double orc_fp16_value(uint16_t bits) {
  int s = (bits >> 15) & 1, e = (bits >> 10) & 31, m = bits & 1023;
  double mag;
  if (e == 31) return m ? NAN : (s ? -INFINITY : INFINITY);
  mag = (e == 0) ? m * ldexp(1.0, -24) : (1.0 + m / 1024.0) * ldexp(1.0, e - 15);
  return s ? -mag : mag;
}

/* bfloat16 is the top half of an IEEE binary32. */
double orc_bf16_value(uint16_t bits) {
  uint32_t w = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &w, 4);
  return (double)f;
}

static double load_x(const void* x, int xdtype, int64_t i) {
  if (xdtype == ORC_BF16) return orc_bf16_value(((const uint16_t*)x)[i]);
  return (double)((const float*)x)[i];
}

/* ------------------------------------------------------------------------------------------ */
/* rounding by nearest-value search                                                            */
/* ------------------------------------------------------------------------------------------ */

/* Scale code for u >= 0: nearest finite non-negative code of the format; of two equidistant codes
 * the even one; anything above the largest value gets the largest value (saturation). */
int orc_round_scale(double u, int fmt) {
  int last = (fmt == ORC_UE5M3) ? 0xFF : 0x7E; /* non-negative finite codes, increasing values */
  int best = 0, c;
  double bestd = fabs(u - orc_scale_value(0, fmt));
  /* saturation first: far above the table a double distance can no longer separate two codes */
  if (u >= orc_scale_value(last, fmt)) return last;
  for (c = 1; c <= last; ++c) {
    double d = fabs(u - orc_scale_value(c, fmt));
    if (d < bestd || (d == bestd && (c & 1) == 0)) {
      best = c;
      bestd = d;
    }
  }
  return best;
}

/* E2M1 magnitude code (0..7) for v >= 0, same rule over {0, .5, 1, 1.5, 2, 3, 4, 6}. */
int orc_round_e2m1_mag(double v) {
  int best = 0, c;
  double bestd = fabs(v);
  if (v >= 6.0) return 7; /* saturation at the largest magnitude, see orc_round_scale */
  for (c = 1; c <= 7; ++c) {
    double d = fabs(v - orc_e2m1_value(c));
    if (d < bestd || (d == bestd && (c & 1) == 0)) {
      best = c;
      bestd = d;
    }
  }
  return best;
}

/* ------------------------------------------------------------------------------------------ */
/* argument checks shared by the entry points of this file                                     */
/* ------------------------------------------------------------------------------------------ */

static int bad_shape(int64_t rows, int64_t cols, int block) {
  if (rows < 0 || cols < 0) return 1;
  if (block < 4 || block > 256 || (block & (block - 1)) != 0) return 1; /* [MX] §1: 4..256 */
  return 0;
}

/* Row layout (any cols): a row is cut into blocks of N from its first element, the last block
 * holding cols mod N elements when N does not divide cols; a row's codes take ceil(cols / 2)
 * bytes (element 2k low nibble, 2k + 1 high nibble of byte k; an odd last element leaves the high
 * nibble 0) and its scales ceil(cols / N) bytes. */
static int64_t row_bytes(int64_t cols) { return (cols + 1) / 2; }
static int64_t row_blocks(int64_t cols, int block) { return (cols + block - 1) / block; }

static int bad_g(uint16_t g_bits) {
  double g = orc_fp16_value(g_bits);
  return !(g > 0.0) || isinf(g) || isnan(g);
}

/* ------------------------------------------------------------------------------------------ */
/* threading helper: rows are split into contiguous ranges                                      */
/* ------------------------------------------------------------------------------------------ */

typedef struct {
  void (*fn)(void* ctx, int64_t r0, int64_t r1, int tid);
  void* ctx;
  int64_t r0, r1;
  int tid;
} orc_job;

static void* orc_job_run(void* p) {
  orc_job* j = (orc_job*)p;
  j->fn(j->ctx, j->r0, j->r1, j->tid);
  return NULL;
}

static int clamp_threads(int nthreads, int64_t rows) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (rows < nthreads) nthreads = rows > 0 ? (int)rows : 1;
  return nthreads;
}

static void parallel_rows(int64_t rows, int nthreads, void (*fn)(void*, int64_t, int64_t, int),
                          void* ctx) {
  orc_job jobs[256];
  pthread_t th[256];
  int t;
  nthreads = clamp_threads(nthreads, rows);
  for (t = 0; t < nthreads; ++t) {
    jobs[t].fn = fn;
    jobs[t].ctx = ctx;
    jobs[t].r0 = rows * t / nthreads;
    jobs[t].r1 = rows * (t + 1) / nthreads;
    jobs[t].tid = t;
  }
  if (nthreads == 1) {
    orc_job_run(&jobs[0]);
    return;
  }
  for (t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, orc_job_run, &jobs[t]);
  for (t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
}

/* ------------------------------------------------------------------------------------------ */
/* one block: [MX] §3.1 item 2 (quantize_block), with the FP16 factor of §3.1 item 3           */
/* ------------------------------------------------------------------------------------------ */

/* xs: N values; writes N 4-bit codes and returns the scale code. */
static int quantize_block(const double* xs, int n, int fmt, double g, uint8_t* codes) {
  double a = 0.0, S;
  int i, s;
  for (i = 0; i < n; ++i)
    if (fabs(xs[i]) > a) a = fabs(xs[i]);      /* abs_max = max|block| */
  s = orc_round_scale(a / (6.0 * g), fmt);     /* scale = Q_fp8(abs_max / 6)  (per g) */
  S = orc_scale_value(s, fmt);
  for (i = 0; i < n; ++i) {                    /* q = Q_fp4(block / scale)  (per g) */
    int mag = (S > 0.0) ? orc_round_e2m1_mag(fabs(xs[i]) / (S * g)) : 0; /* zero scale: zero block */
    codes[i] = (uint8_t)((signbit(xs[i]) ? 8 : 0) | mag);
  }
  return s;
}

/* code of element j of row r */
static int get_code(const uint8_t* packed, int64_t cols, int64_t r, int64_t j) {
  uint8_t b = packed[r * row_bytes(cols) + (j >> 1)];
  return (j & 1) ? (b >> 4) : (b & 15); /* even element in the low nibble */
}

/* ------------------------------------------------------------------------------------------ */
/* quantize                                                                                     */
/* ------------------------------------------------------------------------------------------ */

typedef struct {
  const void* x;
  int xdtype, block, fmt;
  int64_t cols;
  double g;
  uint8_t *packed, *scales;
} q_ctx;

static void q_rows(void* p, int64_t r0, int64_t r1, int tid) {
  q_ctx* c = (q_ctx*)p;
  double xs[256];
  uint8_t codes[256];
  int64_t r, b, nb = row_blocks(c->cols, c->block), pb = row_bytes(c->cols);
  int i;
  (void)tid;
  for (r = r0; r < r1; ++r) {
    for (b = 0; b < nb; ++b) {
      const int64_t j0 = b * c->block; /* even: blocks start on byte boundaries */
      const int len = (int)(c->cols - j0 < c->block ? c->cols - j0 : c->block);
      for (i = 0; i < len; ++i) xs[i] = load_x(c->x, c->xdtype, r * c->cols + j0 + i);
      c->scales[r * nb + b] = (uint8_t)quantize_block(xs, len, c->fmt, c->g, codes);
      for (i = 0; i < len; i += 2)
        c->packed[r * pb + ((j0 + i) >> 1)] =
            (uint8_t)(codes[i] | (i + 1 < len ? codes[i + 1] << 4 : 0));
    }
  }
}

int orc_quantize(const void* x, int xdtype, int64_t rows, int64_t cols, int block, int fmt,
                 uint16_t g_bits, uint8_t* packed, uint8_t* scales, int nthreads) {
  q_ctx c;
  if (bad_shape(rows, cols, block) || bad_g(g_bits)) return -1;
  if (rows * cols == 0) return 0;
  if (!x || !packed || !scales) return -1;
  c.x = x;
  c.xdtype = xdtype;
  c.block = block;
  c.fmt = fmt;
  c.cols = cols;
  c.g = orc_fp16_value(g_bits);
  c.packed = packed;
  c.scales = scales;
  parallel_rows(rows, nthreads, q_rows, &c);
  return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* dequantize: [MX] §1 and §3.1 item 3, value = FP4 x FP8_scale x FP16_scale                  */
/* ------------------------------------------------------------------------------------------ */

/* Round a double to bfloat16 (8 significant bits, nearest, ties to even) and return its bits. */
static uint16_t to_bf16_bits(double v) {
  float f;
  uint32_t w;
  if (isnan(v)) return 0x7FC0;
  if (v == 0.0 || isinf(v)) {
    f = (float)v; /* keeps the sign of zero */
  } else {
    int e;
    double fr = frexp(fabs(v), &e);                   /* |v| = fr * 2^e, fr in [0.5, 1) */
    double r = ldexp(nearbyint(ldexp(fr, 8)), e - 8); /* 8 significant bits, ties to even */
    f = (float)(signbit(v) ? -r : r);
  }
  memcpy(&w, &f, 4);
  return (uint16_t)(w >> 16);
}

typedef struct {
  const uint8_t *packed, *scales;
  int block, fmt, ydtype;
  int64_t cols;
  double g;
  void* y;
} dq_ctx;

static void dq_rows(void* p, int64_t r0, int64_t r1, int tid) {
  dq_ctx* c = (dq_ctx*)p;
  int64_t r, j, nb = row_blocks(c->cols, c->block);
  (void)tid;
  for (r = r0; r < r1; ++r) {
    for (j = 0; j < c->cols; ++j) {
      int64_t idx = r * c->cols + j;
      double S = orc_scale_value(c->scales[r * nb + j / c->block], c->fmt);
      double v = orc_e2m1_value(get_code(c->packed, c->cols, r, j)) * S * c->g;
      if (c->ydtype == ORC_BF16)
        ((uint16_t*)c->y)[idx] = to_bf16_bits(v);
      else
        ((float*)c->y)[idx] = (float)v; /* exact: at most 17 significant bits */
    }
  }
}

int orc_dequantize(const uint8_t* packed, const uint8_t* scales, int64_t rows, int64_t cols,
                   int block, int fmt, uint16_t g_bits, void* y, int ydtype, int nthreads) {
  dq_ctx c;
  if (bad_shape(rows, cols, block) || bad_g(g_bits)) return -1;
  if (rows * cols == 0) return 0;
  if (!packed || !scales || !y) return -1;
  c.packed = packed;
  c.scales = scales;
  c.block = block;
  c.fmt = fmt;
  c.ydtype = ydtype;
  c.cols = cols;
  c.g = orc_fp16_value(g_bits);
  c.y = y;
  parallel_rows(rows, nthreads, dq_rows, &c);
  return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* three-term error reduction, [MX] §2.2 items 1-3                                              */
/* ------------------------------------------------------------------------------------------ */

typedef struct {
  const void* x;
  int xdtype, block, fmt;
  int64_t cols;
  double g;
  const uint8_t *packed, *scales;
  orc_stats part[256];
} st_ctx;

static void st_rows(void* p, int64_t r0, int64_t r1, int tid) {
  st_ctx* c = (st_ctx*)p;
  orc_stats* o = &c->part[tid];
  double xs[256];
  uint8_t codes[256];
  int64_t r, b, nb = row_blocks(c->cols, c->block);
  double smax = orc_scale_max(c->fmt);
  int i;
  memset(o, 0, sizeof(*o));
  for (r = r0; r < r1; ++r) {
    for (b = 0; b < nb; ++b) {
      const int64_t j0 = b * c->block;
      const int len = (int)(c->cols - j0 < c->block ? c->cols - j0 : c->block);
      double a = 0.0, S;
      int s, imax = 0;
      for (i = 0; i < len; ++i) {
        xs[i] = load_x(c->x, c->xdtype, r * c->cols + j0 + i);
        if (fabs(xs[i]) > a) { /* strict: the first index of the largest |x| is "the max element" */
          a = fabs(xs[i]);
          imax = i;
        }
      }
      if (c->packed) {
        s = c->scales[r * nb + b];
        for (i = 0; i < len; ++i) codes[i] = (uint8_t)get_code(c->packed, c->cols, r, j0 + i);
      } else {
        s = quantize_block(xs, len, c->fmt, c->g, codes);
      }
      S = orc_scale_value(s, c->fmt);
      o->n_blocks += 1;
      if (a > 6.0 * c->g * smax) o->n_scale_sat += 1; /* a/(6g) above the largest scale */
      if (S == 0.0) {
        /* item 3: the whole block is stored as zero; its error is sum x^2 */
        o->n_zero_blocks += 1;
        for (i = 0; i < len; ++i) o->sse_zero += xs[i] * xs[i];
        continue;
      }
      for (i = 0; i < len; ++i) {
        double y = orc_e2m1_value(codes[i]) * S * c->g;
        double d = xs[i] - y;
        if (i == imax)
          o->sse_max += d * d;  /* item 2: the max element (scale-rounding error) */
        else
          o->sse_elem += d * d; /* item 1: the other N-1 elements */
        if (fabs(xs[i]) > 6.0 * S * c->g) o->n_elem_sat += 1; /* clipped at the top code */
      }
    }
  }
}

int orc_error_stats(const void* x, int xdtype, int64_t rows, int64_t cols, int block, int fmt,
                    uint16_t g_bits, const uint8_t* packed, const uint8_t* scales, orc_stats* out,
                    int nthreads) {
  st_ctx* c;
  int t, nt;
  if (bad_shape(rows, cols, block) || bad_g(g_bits) || !out) return -1;
  if ((packed == NULL) != (scales == NULL)) return -1;
  memset(out, 0, sizeof(*out));
  out->numel = rows * cols;
  if (rows * cols == 0) return 0;
  if (!x) return -1;
  c = (st_ctx*)calloc(1, sizeof(st_ctx));
  if (!c) return -1;
  c->x = x;
  c->xdtype = xdtype;
  c->block = block;
  c->fmt = fmt;
  c->cols = cols;
  c->g = orc_fp16_value(g_bits);
  c->packed = packed;
  c->scales = scales;
  nt = clamp_threads(nthreads, rows);
  parallel_rows(rows, nt, st_rows, c);
  for (t = 0; t < nt; ++t) { /* fixed order */
    out->sse_elem += c->part[t].sse_elem;
    out->sse_max += c->part[t].sse_max;
    out->sse_zero += c->part[t].sse_zero;
    out->n_blocks += c->part[t].n_blocks;
    out->n_zero_blocks += c->part[t].n_zero_blocks;
    out->n_scale_sat += c->part[t].n_scale_sat;
    out->n_elem_sat += c->part[t].n_elem_sat;
  }
  free(c);
  return 0;
}

/* ------------------------------------------------------------------------------------------ */
/* per-tensor FP16 scale: smallest FP16 value g with g * 6 * Smax >= max|x|                     */
/* ------------------------------------------------------------------------------------------ */

uint16_t orc_global_scale(const void* x, int xdtype, int64_t numel, int fmt) {
  double A = 0.0, K = 6.0 * orc_scale_max(fmt);
  int64_t i;
  uint16_t h;
  for (i = 0; i < numel; ++i) {
    double v = fabs(load_x(x, xdtype, i));
    if (v > A) A = v;
  }
  if (A == 0.0) return 0x3C00; /* nothing to scale: 1.0 */
  /* positive finite binary16 patterns 0x0001..0x7BFF are increasing in value */
  for (h = 0x0001; h <= 0x7BFF; ++h)
    if (orc_fp16_value(h) * K >= A) return h; /* product exact: <= 17 significant bits */
  return 0x7BFF; /* clamp at 65504 */
}
