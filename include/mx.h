/*
 * mx.h -- C ABI of the B200 (sm_100a) FP4 microscaling library (libmxfp4_b200.so).
 *
 * The method (microscaling article, hotelren.com/news/2192771, page titled "企业官网建设流程全解析";
 * cited below as [MX]):
 *   - a tensor is cut into blocks of N consecutive values, N in 4..256 ([MX] §1); here a block is
 *     N consecutive columns of one row; when N does not divide cols, the last block of every row
 *     holds the cols mod N remaining values (its own absmax and scale, the same rule);
 *   - each block gets one FP8 scale s = Q_fp8(absmax / (6 g)) in E4M3 or UE5M3 ([MX] §3.1 items 1-2);
 *   - each value becomes the FP4 E2M1 code q = Q_fp4(x / (s g)) ([MX] §1, §3.1 item 2);
 *   - g is an optional per-tensor FP16 factor, value = FP4 x FP8_scale x FP16_scale ([MX] §3.1 item 3);
 *   - the quantization error splits into three sums ([MX] §2.2 items 1-3).
 * Q_* rounds to the nearest representable value, ties to the even code, and saturates at the largest
 * finite value.  E2M1 has no inf/NaN.  E4M3 is the OCP "FN" variant (bias 7, max 448; 0x7F never
 * produced).  UE5M3 is unsigned, bias 15, with subnormals, every code finite, max 122880.
 *
 * Conventions shared by every entry point:
 *   - All tensors are caller-owned DEVICE memory, contiguous and row-major.  The library never
 *     allocates and never synchronizes (except the calls documented as synchronizing).  State that
 *     outlives a call: the diagnostic launch counter (mx_kernel_launches), the scratch array of
 *     mx_error_stats_noalloc (shared by its calls on a device, see there), the test hook's armed
 *     failures (mx_test_fail_next_calls), and for mx_matmul a per-device count of thread blocks
 *     whose bounded waits ran out plus the generation number of the last launch that gave up
 *     (see mx_matmul_gave_up; later launches are not affected by it).
 *   - Everything is enqueued on `stream` (0 = the legacy default stream); results are valid after
 *     the caller synchronizes that stream.
 *   - Arguments are checked on the host before anything is enqueued; a non-OK status means nothing
 *     was launched.  MX_ERR_CUDA reports a launch error (cudaGetLastError); faults that happen while
 *     a kernel runs surface at the caller's next synchronization, as usual in CUDA.
 *   - Every pointer argument must be 16-byte aligned (MX_ERR_MISALIGNED otherwise).
 *   - Layout of codes and scales: row-major, a row's codes in ceil(cols/2) bytes (element 2k in
 *     the low nibble of byte k, 2k+1 in the high nibble; an odd last element leaves the high
 *     nibble 0) and its scales in ceil(cols/N) bytes.  For cols % N == 0 that is rows*cols/2 and
 *     rows*cols/N bytes.  Tensors with cols % N != 0 ("ragged"; cols up to 2^30, else
 *     MX_ERR_CUDA) run on ragged paths: bf16 rows on 16-byte boundaries (cols % 8 == 0) on the
 *     whole-block kernels in a row-pitched mode (quantize and fake quantize for N >= 16, the error
 *     reduction with recomputed codes for N >= 32) or through row tiles written by TMA
 *     (dequantize to bf16, N >= 16); everything else on a row-wise kernel (one warp per row).  In
 *     a grouped call they run after the group's one launch over its whole-block tensors.
 *   - rows == 0 or cols == 0 is an empty tensor: quantize / dequantize enqueue nothing,
 *     mx_error_stats writes an all-zero result and mx_global_scale writes 1.0.
 *   - x must be finite: NaN or Inf in x gives unspecified codes (no kernel faults or hangs).
 *   - global_scale_fp16 is the IEEE binary16 bit pattern of g; it must be finite and > 0
 *     (0x3C00 = 1.0 = no global scale); anything else is MX_ERR_INVALID_ARG.
 */
#ifndef MX_H
#define MX_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define MX_API __attribute__((visibility("default")))
#else
#define MX_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MX_OK = 0,
  MX_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad enum, bad g */
  MX_ERR_UNSUPPORTED = 2, /* block not one of 4, 8, 16, 32, 64, 128, 256 */
  MX_ERR_MISALIGNED = 3,  /* a pointer is not 16-byte aligned */
  MX_ERR_WORKSPACE = 4,   /* workspace pointer NULL or smaller than the *_workspace_size() value */
  MX_ERR_CUDA = 5         /* the CUDA runtime reported an error while enqueueing */
} mx_status;

typedef enum { MX_F32 = 0, MX_BF16 = 1 } mx_dtype;
typedef enum { MX_SCALE_E4M3 = 0, MX_SCALE_UE5M3 = 1 } mx_scale_fmt;

/* Result of mx_error_stats ([MX] §2.2).  The SSE fields are sums over the tensor; the pages' mean
 * squared errors are sse_* / numel, and the three sum to the total MSE. */
typedef struct {
  double sse_elem;       /* item 1: (x - y)^2 over every non-max element of blocks with s > 0 */
  double sse_max;        /* item 2: (x - y)^2 of the max element (first index of max|x|) of blocks
                            with s > 0, i.e. the error left by rounding the scale */
  double sse_zero;       /* item 3: x^2 over every element of blocks whose scale is zero */
  int64_t numel;         /* rows * cols */
  int64_t n_blocks;      /* rows * cols / block */
  int64_t n_zero_blocks; /* blocks whose scale code decodes to 0 */
  int64_t n_scale_sat;   /* blocks with absmax / (6 g) above the largest scale value */
  int64_t n_elem_sat;    /* elements of blocks with s > 0 and |x| > 6 s g (clipped at +-6) */
} mx_error_stats_t;

/* Quantize + pack ([MX] §3.1 item 2, with g from §3.1 item 3; packing from the 4-bit float
 * article, gtnt.cn/news/16247, §4.3, two FP4 values per byte).
 *   x       rows x cols values of type xt (MX_BF16 or MX_F32), device.
 *   block   N, one of 4, 8, 16, 32, 64, 128, 256 (any cols: a ragged last block per row when N
 *           does not divide cols).
 *   fmt     scale format of the block scales.
 *   packed  OUT rows*ceil(cols/2) bytes, device: element 2k of a row in the low nibble of the row's
 *           byte k, element 2k+1 in the high nibble.  Nibble = sign<<3 | E2M1 magnitude code; the
 *           sign bit is x's sign bit (also for -0.0 and in zero-scale blocks).
 *   scales  OUT rows*ceil(cols/block) bytes, device: the FP8 code of each block, row-major.
 * A block whose scale rounds to zero (absmax <= 3 g smin) stores magnitude 0 in every element. */
MX_API mx_status mx_quantize(const void* x, mx_dtype xt, int64_t rows, int64_t cols, int block,
                      mx_scale_fmt fmt, uint16_t global_scale_fp16, uint8_t* packed,
                      uint8_t* scales, cudaStream_t stream);

/* Dequantize ([MX] §1 and §3.1 item 3: value = FP4 x FP8_scale x FP16_scale).
 *   packed, scales  as written by mx_quantize (any byte values are accepted; E4M3 codes with the
 *                   sign bit decode to negative scales, 0x7F / 0xFF to NaN).
 *   y       OUT rows x cols values of type yt, device.  MX_F32 holds the exact product
 *           E2M1 * S * g; MX_BF16 holds its round-to-nearest-even. */
MX_API mx_status mx_dequantize(const uint8_t* packed, const uint8_t* scales, int64_t rows, int64_t cols,
                        int block, mx_scale_fmt fmt, uint16_t global_scale_fp16, void* y,
                        mx_dtype yt, cudaStream_t stream);

/* Fake quantization for quantization-aware training ([MX] §5.2 item 1: the forward pass injects
 * the quantization noise, x -> dequant(quant(x))): y is, bit for bit, what mx_dequantize writes
 * for the codes and scales mx_quantize would store, computed in one pass that reads x and writes
 * only y (4 bytes per element for bf16 -> bf16).  Arguments as mx_quantize (x, xt, rows, cols,
 * block, fmt, global scale) and mx_dequantize (y, yt).  The gradient (straight-through) belongs to
 * the caller's autograd; the Python binding provides it. */
MX_API mx_status mx_fake_quantize(const void* x, mx_dtype xt, int64_t rows, int64_t cols,
                                  int block, mx_scale_fmt fmt, uint16_t global_scale_fp16, void* y,
                                  mx_dtype yt, cudaStream_t stream);

/* Bytes of device workspace mx_error_stats needs (a bound that holds for any device). */
MX_API size_t mx_error_stats_workspace_size(int64_t rows, int64_t cols, int block);

/* Three-term error reduction ([MX] §2.2 items 1-3).
 *   packed, scales  NULL, NULL: the codes are recomputed from x in registers (same rule as
 *                   mx_quantize, nothing is written); otherwise the given codes are used and only
 *                   scale codes the quantizer can produce are meaningful (E4M3 0x00..0x7E).
 *   out_dev  OUT one mx_error_stats_t in device memory (written by the last kernel).
 *   workspace, ws_bytes  device scratch of at least mx_error_stats_workspace_size() bytes; its
 *                   contents need no initialisation and are overwritten (a counter, reset by the
 *                   call, and one partial sum per CTA).  Two calls that share a workspace must
 *                   not run concurrently (order them on one stream).
 * The reconstruction used for the errors is the exact E2M1 * S * g.  Each thread sums the squared
 * errors of at most 32 elements in fp32 and adds those partial sums in double; the partials are
 * combined in a fixed order for a given device, so repeated calls give identical results.  The
 * three sums are within 1e-5 relative of the exact sums; the counts are exact. */
MX_API mx_status mx_error_stats(const void* x, mx_dtype xt, int64_t rows, int64_t cols, int block,
                         mx_scale_fmt fmt, uint16_t global_scale_fp16, const uint8_t* packed,
                         const uint8_t* scales, mx_error_stats_t* out_dev, void* workspace,
                         size_t ws_bytes, cudaStream_t stream);

/* Quantize + pack with the three-term error reduction fused into the same pass over x ([MX] §3.1
 * item 2 and §2.2 items 1-3).  packed and scales are what mx_quantize writes; out_dev is what
 * mx_error_stats reports for them.  x is read once instead of twice.  Arguments are those of
 * mx_quantize plus out_dev, workspace and ws_bytes of mx_error_stats (same size rule). */
MX_API mx_status mx_quantize_stats(const void* x, mx_dtype xt, int64_t rows, int64_t cols,
                                   int block, mx_scale_fmt fmt, uint16_t global_scale_fp16,
                                   uint8_t* packed, uint8_t* scales, mx_error_stats_t* out_dev,
                                   void* workspace, size_t ws_bytes, cudaStream_t stream);

/* The pages' mean squared errors from a record copied to host memory ([MX] §2.2: each sum over
 * the tensor's element count, so the three means add up to the total MSE):
 * mse4[0..3] = sse_elem / numel, sse_max / numel, sse_zero / numel and their sum (all zero for an
 * empty tensor).  record and mse4 are host memory; NULL gives MX_ERR_INVALID_ARG. */
MX_API mx_status mx_error_stats_means(const mx_error_stats_t* record, double* mse4);

/* Bytes of device workspace mx_global_scale needs. */
MX_API size_t mx_global_scale_workspace_size(int64_t rows, int64_t cols);

/* Per-tensor FP16 scale for [MX] §3.1 item 3.  The pages do not say how g is chosen; this library
 * takes the smallest binary16 value g with g * 6 * Smax >= max|x| (so no block scale saturates),
 * 1.0 when x is all zero, and 65504 when even that is too small.
 *   out_fp16_dev  OUT one uint16_t (binary16 bit pattern) in device memory. */
MX_API mx_status mx_global_scale(const void* x, mx_dtype xt, int64_t rows, int64_t cols, mx_scale_fmt fmt,
                          uint16_t* out_fp16_dev, void* workspace, size_t ws_bytes,
                          cudaStream_t stream);

/* mx_error_stats without a caller workspace (no counterpart in the pages: a library convenience).
 * For callers that cannot allocate device memory for a workspace -- a host framework that owns all
 * device allocations and passes the library only tensors, a real-time loop that must not enter an
 * allocator, a C caller without a device allocator.  The scratch is a fixed 256 KiB array in this
 * library's device memory (every GPU that loads the library holds it until the process exits); the
 * call allocates nothing (no cudaMalloc, cudaFree or allocating library routine).  Arguments,
 * results and errors are those of mx_error_stats; any rows x cols fits, because the scratch need
 * does not grow with the tensor (a call that needed more than the array would get MX_ERR_WORKSPACE).
 *   - The first call on a device resolves the array's device address (cudaGetSymbolAddress, with
 *     that device current) and keeps it; make that first call before any stream capture.
 *   - Every call on a device shares the one array and leaves its contents behind.  Nothing in it
 *     needs to start at zero (each call overwrites what it reads), but calls whose kernels overlap
 *     on the GPU (different streams, no ordering between them) race on it: order them. */
MX_API mx_status mx_error_stats_noalloc(const void* x, mx_dtype xt, int64_t rows, int64_t cols,
                                        int block, mx_scale_fmt fmt, uint16_t global_scale_fp16,
                                        const uint8_t* packed, const uint8_t* scales,
                                        mx_error_stats_t* out_dev, cudaStream_t stream);

/* ---- Grouped calls (no counterpart in the pages: a launch-level batching of the calls above).
 * Up to MX_MAX_GROUP tensors that share dtype, block size and scale format are processed by one
 * persistent kernel launch whose grid is split among them (in proportion to their sizes), instead
 * of one launch per tensor -- for example every weight matrix of a transformer layer.  Results are
 * those of the per-tensor calls, tensor by tensor (the error sums up to the order of the
 * additions).  The descriptor array is host memory, read during the call only.  Arguments are
 * checked for every tensor before anything is enqueued; count outside [1, MX_MAX_GROUP] gives
 * MX_ERR_INVALID_ARG. */
#define MX_MAX_GROUP 16

/* One tensor of a grouped call: rows x cols, row-major (any cols; the layout of codes and scales
 * is the one described above). */
typedef struct {
  const void* x;              /* input of mx_quantize_group / mx_quantize_stats_group /
                                 mx_global_scale_group */
  void* y;                    /* output of mx_dequantize_group */
  uint8_t* packed;            /* rows*cols/2 codes: written by quantize, read by dequantize */
  uint8_t* scales;            /* rows*cols/block scale codes, likewise */
  mx_error_stats_t* stats;    /* mx_quantize_stats_group: this tensor's record (device) */
  uint16_t* global_scale_dev; /* NULL, or the device address (2-byte aligned) of this tensor's g
                                 as a binary16 bit pattern: written by mx_global_scale_group, read
                                 by the other grouped calls when their kernels run (so g never
                                 visits the host; global_scale_fp16 is then ignored) */
  int64_t rows, cols;
  uint16_t global_scale_fp16; /* per-tensor g, as in mx_quantize (used when global_scale_dev is
                                 NULL) */
  uint16_t reserved[3];       /* must be zero */
} mx_tensor_t;

/* mx_quantize of every tensor (x -> packed, scales). */
MX_API mx_status mx_quantize_group(const mx_tensor_t* tensors, int count, mx_dtype xt, int block,
                                   mx_scale_fmt fmt, cudaStream_t stream);

/* mx_dequantize of every tensor (packed, scales -> y of type yt). */
MX_API mx_status mx_dequantize_group(const mx_tensor_t* tensors, int count, int block,
                                     mx_scale_fmt fmt, mx_dtype yt, cudaStream_t stream);

/* mx_quantize_stats of every tensor (x -> packed, scales, stats) with one workspace of
 * mx_error_stats_workspace_size() bytes for the whole group. */
MX_API mx_status mx_quantize_stats_group(const mx_tensor_t* tensors, int count, mx_dtype xt,
                                         int block, mx_scale_fmt fmt, void* workspace,
                                         size_t ws_bytes, cudaStream_t stream);

/* mx_global_scale of every tensor (x -> *global_scale_dev, which must be non-NULL) with one
 * workspace of mx_global_scale_workspace_size() bytes for the whole group; global_scale_fp16 is
 * not read.  The same descriptors can then drive mx_quantize_stats_group and mx_dequantize_group
 * on the same stream: the per-tensor g stays in device memory ([MX] §3.1 item 3, a per-tensor
 * FP16 factor; how it is chosen is this library's rule, see mx_global_scale). */
MX_API mx_status mx_global_scale_group(const mx_tensor_t* tensors, int count, mx_dtype xt,
                                       mx_scale_fmt fmt, void* workspace, size_t ws_bytes,
                                       cudaStream_t stream);

/* ---- Block-scaled matrix product on the tensor cores.
 * C = dequant(A) * dequant(B)^T, the dequantize-then-multiply step of inference in the 4-bit float
 * quantization article (gtnt.cn/news/16247, §3.1), with both operands stored by mx_quantize and
 * the block scales applied inside the tensor-core multiply (nothing is dequantized to memory).
 *
 * Operands: A is m x k (a_packed: m*k/2 bytes, as mx_quantize writes a row-major m x k tensor with
 * block = 16 and MX_SCALE_E4M3), B is n x k (b_packed: n*k/2 bytes, likewise); a_g / b_g are the
 * global scales they were quantized with.  Their scale arrays are first put into tensor-core
 * order by mx_matmul_prepare_scales (for weights, once), and mx_matmul reads the prepared arrays.
 *
 * mx_matmul_scales_size(rows, k): bytes of a prepared scale array for a rows x k operand,
 * 2 * ceil(rows / 256) * 128 * k / 16 (rows padded with zero scales); 0 when rows < 0 or k is not
 * a positive multiple of 256. */
MX_API size_t mx_matmul_scales_size(int64_t rows, int64_t k);

/* scales (rows * k / 16 bytes, the mx_quantize layout, block 16) -> out (out_bytes >=
 * mx_matmul_scales_size(rows, k), device memory): for each 128-row tile and each 256-element step
 * of k, 2048 contiguous bytes holding four 512-byte groups (one per 64-element tensor-core step);
 * in group j, row 32 q + r of the tile has its four scales at byte 16 r + 4 q.  Errors: k not a
 * positive multiple of 256 -> MX_ERR_UNSUPPORTED; rows < 0 -> MX_ERR_INVALID_ARG; out_bytes too
 * small -> MX_ERR_WORKSPACE; rows == 0 enqueues nothing. */
MX_API mx_status mx_matmul_prepare_scales(const uint8_t* scales, int64_t rows, int64_t k,
                                          uint8_t* out, size_t out_bytes, cudaStream_t stream);

/* C (m x n, row-major, float32 for ct = MX_F32 or bfloat16 rounded to nearest even for MX_BF16)
 *   C[i][j] = a_g b_g sum_t E2M1(A[i][t]) S(A)[i][t/16] E2M1(B[j][t]) S(B)[j][t/16],
 * accumulated in float32 by the tensor core (order unspecified), then multiplied by a_g b_g (one
 * rounding).  a_scales_mma / b_scales_mma are the prepared arrays of A (m rows) and B (n rows).
 * block != 16 or fmt != MX_SCALE_E4M3 (no native tensor-core form), k == 0 or k % 256 != 0:
 * MX_ERR_UNSUPPORTED; m, n or k negative, or m, n >= 2^31: MX_ERR_INVALID_ARG; m == 0 or n == 0:
 * nothing is enqueued.  Every wait inside the kernel is bounded; a launch whose waits ran out
 * leaves C unspecified and is counted by mx_matmul_gave_up (it does not affect later launches).
 * Kernel: one CTA per 128 x 256 tile of C. */
MX_API mx_status mx_matmul(const uint8_t* a_packed, const uint8_t* a_scales_mma, uint16_t a_g,
                           const uint8_t* b_packed, const uint8_t* b_scales_mma, uint16_t b_g,
                           int64_t m, int64_t n, int64_t k, int block, mx_scale_fmt fmt, void* c,
                           mx_dtype ct, cudaStream_t stream);

/* mx_matmul computed by CTA pairs (tcgen05 cta_group::2): a cluster of two CTAs per 256 x 256
 * tile of C when m > 128 (else the one-CTA kernel).  Same arguments, results and errors as
 * mx_matmul; an alternative kernel for the same product (slower than mx_matmul on the shapes
 * measured so far). */
MX_API mx_status mx_matmul_pair(const uint8_t* a_packed, const uint8_t* a_scales_mma, uint16_t a_g,
                                const uint8_t* b_packed, const uint8_t* b_scales_mma, uint16_t b_g,
                                int64_t m, int64_t n, int64_t k, int block, mx_scale_fmt fmt,
                                void* c, mx_dtype ct, cudaStream_t stream);

/* bf16 activations times stored FP4 weights on the tensor cores: the inference step of the 4-bit
 * float quantization article (gtnt.cn/news/16247, §3.1, dequantize the stored weights, then
 * multiply), for weights in any of this library's formats ([MX] §3.1 items 1-3: blocks of
 * 4..256, E4M3 or UE5M3 scales, FP16 global scale):
 *   C[i][j] = sum_t A[i][t] * Wq[j][t],  Wq = RN_bf16(E2M1 * S * g), the values mx_dequantize
 *   writes as bf16,
 * accumulated in float32 by the tensor core (order unspecified; every product is exact).  Each
 * weight tile is dequantized into shared memory inside the kernel, nothing to global memory.
 *   a        m x k bf16, row-major (device).
 *   w_packed, w_scales  n x k weights exactly as mx_quantize stores them with this block / fmt
 *            (n*k/2 code bytes, n*k/block scale bytes).
 *   w_global_scale_fp16 / w_global_scale_dev  g as a bit pattern, or (dev non-NULL, 2-byte
 *            aligned) read from device memory when the kernel runs (e.g. mx_global_scale output).
 *   c        OUT m x n, row-major, float32 (ct = MX_F32) or bfloat16 rounded to nearest even.
 * Errors: k not a positive multiple of 64 and of block, or block not one of 4..256:
 * MX_ERR_UNSUPPORTED; m, n or k negative or >= 2^31, bad fmt / ct / g: MX_ERR_INVALID_ARG;
 * m == 0 or n == 0: nothing is enqueued.  Kernel: one CTA per 256 x 256 tile of C, tcgen05.mma
 * kind::f16; its waits are bounded and counted by mx_matmul_gave_up like mx_matmul's. */
MX_API mx_status mx_dequant_matmul(const void* a, int64_t m, int64_t k, const uint8_t* w_packed,
                                   const uint8_t* w_scales, int64_t n, int block,
                                   mx_scale_fmt fmt, uint16_t w_global_scale_fp16,
                                   const uint16_t* w_global_scale_dev, void* c, mx_dtype ct,
                                   cudaStream_t stream);

/* Number of mx_matmul thread blocks that stopped waiting since the previous call (0 in normal
 * operation), written to *count (host memory); clears the count.  Synchronizes the device. */
MX_API mx_status mx_matmul_gave_up(unsigned int* count);

/* Test hook (no counterpart in the pages): marks the most recent mx_matmul / mx_matmul_pair launch
 * on the current device as abandoned, as a thread block whose waits ran out would.  Later
 * launches must not be affected.  Synchronizes the device. */
MX_API mx_status mx_test_matmul_abandon_last(void);

/* Test hook for error paths (no counterpart in the pages).  The next `count` calls that pass
 * their argument checks and would enqueue work return MX_ERR_CUDA instead, as a failed launch is
 * reported, without enqueueing anything or touching any buffer.  count <= 0 disarms the hook.
 * Returns the number of armed failures that were still pending. */
MX_API int mx_test_fail_next_calls(int count);

/* Static description of a status code (never NULL). */
MX_API const char* mx_status_string(mx_status status);

/* Diagnostic: number of kernels this library has enqueued in this process so far (all calls,
 * all threads).  It never affects results. */
MX_API long long mx_kernel_launches(void);

#ifdef __cplusplus
}
#endif
#endif /* MX_H */
