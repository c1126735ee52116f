/*
 * fp8sm — FP8 (e4m3) scaled matrix multiply and dynamic quantizer for
 * NVIDIA B200 (sm_100a).  C ABI.
 *
 *   out = (A_fp8 * s_A) @ (B_fp8 * s_B)^T (+ bias)
 *
 * Sources for the operations (public pull-request pages):
 *   [P1] "Fix: Handle LowLevelZeroPlugin with use_fp8=True" (ColossalAI PR
 *        #6419), Solution: the FP8 linear forward calls a scaled matmul
 *        whose result equals dequantize-then-matmul plus bias; scales are
 *        dequantization multipliers; tensorwise scales presented as (1, 1).
 *   [P2] "Add _grouped_mm dispatch handler to Float8Tensor" (torchao PR
 *        #4390): MoE expert weights (E, N, K) used as weight.transpose(-2,-1);
 *        rowwise activation scales and (E, N) weight scales; offs required;
 *        an unsupported granularity must raise, never fall back silently.
 *   [P3] "per-token scaling for fp8 linear" (DiffSynth-Engine PR #160),
 *        Highlights: per-row amax -> scale, input pre-scaled (epsilon guard)
 *        and cast to fp8 before one scaled matmul.
 *   [P4] "Add _scaled_mm_v2 API" (PyTorch PR #164141): explicit (declared,
 *        not inferred) scaling recipes per operand; A and B fp8 with fp32
 *        scales; Blockwise_1x128 (A) x Blockwise_128x128 (B); argument errors
 *        are ValueError-class, unimplemented combinations NotImplementedError-
 *        class, everything else RuntimeError-class.
 *   [P5] "improve fp8 blockwise gemm perf" (torchao PR #2784): the
 *        1x128_128x128 GEMM (output = input @ weight.t()) and the
 *        1x128_128x1 GEMM (grad_weight = grad_output_t @ input).
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE memory owned by the caller; the library
 *     never allocates, frees or keeps them.  Calls are asynchronous on the
 *     given stream and return once the work is enqueued.
 *   - Matrices are row-major.  A is (M, K) with K contiguous; B is stored
 *     (N, K) with K contiguous (i.e. the GEMM computes input @ weight.t()).
 *     FP8 tensors are e4m3 bytes; bf16 tensors are raw 16-bit patterns.
 *   - Argument errors (null pointers, bad sizes, misaligned pointers, a scale
 *     layout that does not fit the recipe) return FP8_ERR_VALUE before
 *     anything is launched.  A recipe / dtype combination that is not
 *     implemented returns FP8_ERR_UNSUPPORTED; there is no fallback path of
 *     any kind.  A failed CUDA launch returns FP8_ERR_CUDA.  fp8_last_error()
 *     then describes the problem (per host thread).
 *   - Errors found on the device (a malformed offs array, a pipeline wait
 *     that ran past its time limit) are recorded in a per-device status word
 *     and read back with fp8_get_device_status().
 */
#ifndef FP8SM_H
#define FP8SM_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FP8SM_API __attribute__((visibility("default")))
#else
#define FP8SM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* fp8_stream_t;

/* Status codes: [P4] error classes (ValueError / NotImplementedError /
 * RuntimeError) mapped to codes; TIMEOUT is a device wait that gave up. */
typedef enum {
  FP8_OK = 0,
  FP8_ERR_VALUE = 1,        /* invalid argument (user error)                */
  FP8_ERR_UNSUPPORTED = 2,  /* valid request, not implemented: no fallback  */
  FP8_ERR_CUDA = 3,         /* CUDA runtime / launch failure                */
  FP8_ERR_TIMEOUT = 4       /* a device-side wait ran past its limit        */
} fp8_status;

/* Quantization group shapes ([P3] per-row, [P4]/[P5] 1x128 and 128x128,
 * [P1] per-tensor). */
typedef enum {
  FP8_SCALE_TENSOR = 0,         /* one scale for the whole matrix           */
  FP8_SCALE_ROW = 1,            /* one scale per row                        */
  FP8_SCALE_BLOCK_1x128 = 2,    /* one scale per row per 128 columns        */
  FP8_SCALE_BLOCK_128x128 = 3   /* one scale per 128x128 tile               */
} fp8_quant_recipe;

/* GEMM scaling recipes, named A-recipe_B-recipe as in [P4]; B orientation as
 * in [P5] (the B operand is stored (N, K), so "128x1" means one scale per
 * output column n per 128-wide K block). */
typedef enum {
  FP8_MM_TENSOR_TENSOR = 0,     /* s_A[0] * s_B[0]                           */
  FP8_MM_ROW_ROW = 1,           /* s_A[m] * s_B[n]                           */
  FP8_MM_1x128_128x128 = 2,     /* s_A[kb*M + m] * s_B[kb*ceil(N/128) + n/128] */
  FP8_MM_1x128_128x1 = 3        /* s_A[kb*M + m] * s_B[kb*N + n]             */
} fp8_mm_recipe;

typedef enum {
  FP8_OUT_BF16 = 0,   /* round to nearest even from the fp32 result        */
  FP8_OUT_F32 = 1     /* the fp32 result before any bf16 cast              */
} fp8_out_dtype;

/*
 * Dynamic quantization ([P3] Highlights; scale = max(amax, 1e-12)/448).
 *
 * For every group G of x (shape set by `recipe`):
 *   amax = max |x| over G;  a = max(amax, 1e-12f)
 *   scale[G] = a / 448 (fp32, IEEE division)   -- the dequantization multiplier
 *   q = e4m3_rn_satfinite(x * (448 / a))        -- one fp32 multiply, then the
 *                                                  RNE cast saturating at +-448
 *
 *   x_bf16     (rows, cols) bf16, row stride ld_x elements; 16-byte aligned,
 *              ld_x % 8 == 0, cols % 8 == 0.
 *   out_fp8    (rows, cols) e4m3, row stride cols; 16-byte aligned.
 *   out_scales fp32, 4-byte aligned:
 *                TENSOR:   1 value
 *                ROW:      rows values, scale[r]
 *                1x128:    (cols/128) * rows values, scale[kb*rows + r]
 *                          (K-block-major: one block's scales for consecutive
 *                          rows are contiguous)
 *                128x128:  (cols/128) * ceil(rows/128) values,
 *                          scale[kb*ceil(rows/128) + r/128]
 *              Blockwise recipes need cols % 128 == 0 (rows may be ragged).
 *   workspace  device scratch of fp8_quantize_workspace_bytes() bytes (may be
 *              NULL when that is 0).  TENSOR needs 16 bytes; the library
 *              clears it on the stream before use.  Calls that share one
 *              workspace must not overlap on the GPU.
 * Empty inputs are valid: rows == 0 writes nothing; cols == 0 writes the
 * epsilon scale for each (row) group.
 */
FP8SM_API size_t fp8_quantize_workspace_bytes(fp8_quant_recipe recipe, int64_t rows,
                                    int64_t cols);

FP8SM_API fp8_status fp8_quantize(const void* x_bf16, int64_t rows, int64_t cols,
                        int64_t ld_x, fp8_quant_recipe recipe, void* out_fp8,
                        float* out_scales, void* workspace, size_t ws_bytes,
                        fp8_stream_t stream);

/*
 * Dynamic quantization exactly as fp8_quantize (same recipes, layouts,
 * results and errors), but without a workspace argument, for callers that
 * cannot allocate device memory: for example a plugin running inside a host
 * application that owns every device allocation and hands its plugins no
 * scratch, or a service that fixes its memory plan at start-up and may not
 * call cudaMalloc afterwards (it synchronizes the device and can fail under
 * memory pressure).  The caller still passes x, out_fp8 and out_scales.
 *
 * This entry point allocates nothing and calls no allocating routine.  The
 * scratch it needs (the tensorwise recipe's amax word and grid-barrier
 * counter) lives in a fixed FP8_NOALLOC_SCRATCH_BYTES-byte array inside the
 * library's device code; every GPU that loads the library holds one copy
 * until the process exits.  The first call on each device looks up that
 * array's device address (cudaGetSymbolAddress) with the device current;
 * make that first call before any stream capture.  All calls share the
 * array and each call clears the part that must start at zero, so calls that
 * run at the same time on the GPU (for example on two streams) race with
 * each other: order them on one stream.  A call that would need more scratch
 * than the array holds returns FP8_ERR_VALUE.  No counterpart on the pages.
 */
#define FP8_NOALLOC_SCRATCH_BYTES 256

FP8SM_API fp8_status fp8_quantize_noalloc(const void* x_bf16, int64_t rows,
                                          int64_t cols, int64_t ld_x,
                                          fp8_quant_recipe recipe,
                                          void* out_fp8, float* out_scales,
                                          fp8_stream_t stream);

/*
 * Tensorwise quantization of a tensor split by rows across ranks (one process
 * per GPU, each holding a row shard), with the scale of the WHOLE tensor:
 * the "tensorwise" recipe of [P4]'s recipe table has one scale per tensor,
 * i.e. one amax over all of it (then [P3] Highlights' scale and cast steps),
 * so the ranks exchange their shard maxima once (an all-reduce(MAX) of one
 * fp32 value, done by the caller, e.g. over NCCL) between the two steps.
 *   fp8_tensor_amax               amax[0] = max |x| over the shard (0 for an
 *                                 empty shard); amax is device memory, which
 *                                 the call clears first.
 *   fp8_quantize_tensor_with_amax with a = max(amax[0], 1e-12): out_scale[0] =
 *                                 a / 448 and out_fp8 = e4m3_satfinite(x * (448
 *                                 / a)), the steps of fp8_quantize's tensorwise
 *                                 recipe; amax is read on the device.
 * With one shard the two steps give exactly fp8_quantize(FP8_SCALE_TENSOR).
 * Layouts as fp8_quantize: x bf16 (rows, cols) row stride ld_x, out_fp8
 * (rows, cols) row stride cols.  Requirements: cols % 8 == 0, ld_x % 8 == 0,
 * x and out_fp8 16-byte aligned, amax and out_scale 4-byte aligned.  Errors:
 * FP8_ERR_VALUE for sizes, null or misaligned pointers.
 */
FP8SM_API fp8_status fp8_tensor_amax(const void* x_bf16, int64_t rows, int64_t cols,
                                     int64_t ld_x, float* amax, fp8_stream_t stream);
FP8SM_API fp8_status fp8_quantize_tensor_with_amax(const void* x_bf16, int64_t rows,
                                                   int64_t cols, int64_t ld_x,
                                                   const float* amax, void* out_fp8,
                                                   float* out_scale, fp8_stream_t stream);

/*
 * Transposed dynamic quantization, for the training GEMMs of [P5] (the
 * 1x128_128x128 GEMM also serves grad_input = grad_output @ weight, the
 * 1x128_128x1 GEMM serves grad_weight = grad_output_t @ input) and [P1]'s
 * backward pass: both need an operand whose contraction runs along x's
 * rows.  The result is exactly what fp8_quantize() gives for the transpose
 * of x, without materializing the bf16 transpose:
 *
 *   x_bf16     (rows, cols) bf16, row stride ld_x elements; 16-byte aligned,
 *              ld_x % 8 == 0, cols % 8 == 0, rows % 128 == 0.
 *   out_fp8    (cols, rows) e4m3 = quantized x^T, row stride rows;
 *              16-byte aligned.
 *   out_scales the recipe's layout for a (cols, rows) matrix, 4-byte aligned:
 *                1x128:    (rows/128) * cols values, scale[kb*cols + c]
 *                          (group: rows 128 kb .. 128 kb + 127 of column c)
 *                128x128:  (rows/128) * ceil(cols/128) values,
 *                          scale[kb*ceil(cols/128) + c/128]
 *   recipe     FP8_SCALE_BLOCK_1x128 or FP8_SCALE_BLOCK_128x128; the
 *              tensorwise and rowwise recipes return FP8_ERR_UNSUPPORTED.
 * rows == 0 or cols == 0 writes nothing.  No workspace is needed.
 */
FP8SM_API fp8_status fp8_quantize_transposed(const void* x_bf16, int64_t rows,
                                             int64_t cols, int64_t ld_x,
                                             fp8_quant_recipe recipe, void* out_fp8,
                                             float* out_scales, fp8_stream_t stream);

/*
 * Batched quantization of `batch` equal matrices stored one after the other
 * (matrix e = rows x cols at x_bf16 + e * rows * ld_x, e.g. the (E, N, K)
 * expert weights of [P2]), each quantized on its own, in one launch: the
 * same codes and scales as `batch` separate calls.
 *
 * fp8_quantize_batched: 128x128 only.  out_fp8 (batch, rows, cols);
 *   out_scales (batch, cols/128, ceil(rows/128)) -- each matrix's fp8_quantize
 *   layout, matrices in order (the per-expert layout
 *   fp8_grouped_scaled_mm_blockwise reads).  cols % 128 == 0.
 * fp8_quantize_transposed_batched: 1x128 or 128x128 of each matrix's
 *   transpose.  out_fp8 (batch, cols, rows); out_scales: each matrix's
 *   fp8_quantize_transposed layout, matrices in order.  rows % 128 == 0.
 * 1 <= batch <= 65535 (batch == 0 is a no-op); other requirements and
 * errors as the single-matrix calls.
 */
FP8SM_API fp8_status fp8_quantize_batched(const void* x_bf16, int32_t batch, int64_t rows,
                                int64_t cols, int64_t ld_x, fp8_quant_recipe recipe,
                                void* out_fp8, float* out_scales, fp8_stream_t stream);

FP8SM_API fp8_status fp8_quantize_transposed_batched(const void* x_bf16, int32_t batch,
                                           int64_t rows, int64_t cols, int64_t ld_x,
                                           fp8_quant_recipe recipe, void* out_fp8,
                                           float* out_scales, fp8_stream_t stream);

/*
 * Scaled GEMM ([P1] forward; [P4] recipes; [P5] blockwise recipes):
 *   out[m, n] = sum_k (a[m,k] * sA) * (b[n,k] * sB)  (+ bias[n])
 * with the scales picked per recipe (see fp8_mm_recipe).  Products are
 * accumulated in fp32 on the tensor cores; the blockwise recipes accumulate
 * each 128-wide K block separately and apply its scales on the CUDA cores
 * before summing in fp32.
 *
 *   a        (M, K) e4m3, K contiguous, 16-byte aligned.
 *   b        (N, K) e4m3, K contiguous, 16-byte aligned.
 *   scale_a, scale_b  fp32 scale arrays in the recipe's layout; 16-byte aligned.
 *   bias_bf16 (N) bf16 or NULL; 16-byte aligned.
 *   out      (M, N) row-major, bf16 or fp32 per `out_dtype`; 16-byte aligned.
 * Requirements: K % 16 == 0 (K % 128 == 0 for the blockwise recipes),
 * N % 16 == 0.  M is arbitrary.  M == 0 or N == 0 is a no-op; K == 0 writes
 * bias (or zeros).
 */
FP8SM_API fp8_status fp8_scaled_mm(const void* a, const void* b, int64_t M, int64_t N,
                         int64_t K, const float* scale_a, const float* scale_b,
                         fp8_mm_recipe recipe, const void* bias_bf16,
                         fp8_out_dtype out_dtype, void* out,
                         fp8_stream_t stream);

/*
 * Scaled GEMM whose output leaves already quantized for the next layer's
 * GEMM: the fp32 result of fp8_scaled_mm (same operands, recipes, bias and
 * K-order of accumulation) is grouped 1x128 along n and each group is cast
 * to e4m3 with its own scale, exactly as fp8_quantize's 1x128 recipe would
 * cast those fp32 values:
 *   y[m, n]       = fp8_scaled_mm(...)[m, n] in fp32
 *   s[j, m]       = max(amax_{n in group j} |y[m, n]|, 1e-12) / 448
 *   out[m, n]     = e4m3_satfinite_rn(y[m, n] * (1 / s[n / 128, m]))
 * This is the chained FP8 linear of [P1] Solution (forward: x_fp8 @ w_fp8^T;
 * its output is the next layer's x) with the activation quantize of [P3]
 * and [P5] moved into the producing GEMM's epilogue, so the fp32/bf16 result
 * never goes to HBM and no separate quantize pass reads it back.
 *
 *   a, b, scale_a, scale_b, recipe, bias_bf16: as fp8_scaled_mm.
 *   out_fp8    (M, N) e4m3 row-major, 16-byte aligned.
 *   out_scales (N / 128, M) fp32, K-block-major like fp8_quantize's 1x128
 *              scales (entry [j * M + m]); 4-byte aligned.
 * Requirements: K > 0, K % 16 == 0 (K % 128 == 0 for the blockwise recipes),
 * N % 128 == 0.  M is arbitrary; M == 0 or N == 0 is a no-op.
 */
FP8SM_API fp8_status fp8_scaled_mm_quantized(const void* a, const void* b, int64_t M,
                                   int64_t N, int64_t K, const float* scale_a,
                                   const float* scale_b, fp8_mm_recipe recipe,
                                   const void* bias_bf16, void* out_fp8,
                                   float* out_scales, fp8_stream_t stream);

/*
 * Scaled GEMM that writes both e4m3 forms of its result, for the backward of
 * a chain of FP8 linears ([P1] Solution, backward pass; [P5]: grad_input
 * with 1x128_128x128, grad_weight with 1x128_128x1): with y the fp32 result
 * of fp8_scaled_mm (bias added),
 *   out_fp8, out_scales     = fp8_scaled_mm_quantized's output: y in 1x128
 *                             groups along n (the next grad_input's operand)
 *   out_t_fp8 (N, M), out_t_scales (M/128, N)
 *                           = y^T quantized with 1x128 groups along m, i.e.
 *                             fp8_quantize_transposed(y, 1x128) of the fp32
 *                             values (the next grad_weight's operand):
 *                             scale[(m/128) * N + n], codes row n = tokens.
 * a (M, K) and b (N, K) e4m3 codes with the recipe's scales as for
 * fp8_scaled_mm; all buffers are caller-owned device memory; the call is
 * asynchronous on `stream`.
 * Recipe FP8_MM_1x128_128x128 only (others: FP8_ERR_UNSUPPORTED).
 * Requirements: M % 128 == 0, N % 128 == 0, K > 0, K % 128 == 0; code
 * buffers 16-byte aligned, scales 4-byte aligned.  Errors: FP8_ERR_VALUE
 * (sizes, null or misaligned pointers; nothing is launched), FP8_ERR_CUDA
 * (launch); M == 0 or N == 0 returns FP8_OK without a launch.
 */
FP8SM_API fp8_status fp8_scaled_mm_quantized_dual(const void* a, const void* b, int64_t M,
                                        int64_t N, int64_t K, const float* scale_a,
                                        const float* scale_b, fp8_mm_recipe recipe,
                                        const void* bias_bf16, void* out_fp8,
                                        float* out_scales, void* out_t_fp8,
                                        float* out_t_scales, fp8_stream_t stream);

/*
 * MXFP8 ("mxfp8" in the recipe table of [P4]; the pages name the recipe but
 * do not define it, so the OCP Microscaling (MX) specification's definition
 * is used): one power-of-two E8M0 scale per block of 32 consecutive elements
 * along K, E4M3 elements.  Per block:
 *   e     = floor(log2(max |x|)) - 8, clamped to [-127, 127]; -127 for an
 *           all-zero block (8: 2^8 = 256 is the largest power of two in E4M3)
 *   byte  = e + 127                       (the block's scale is 2^e)
 *   q     = e4m3_satfinite_rn(x * 2^-e)   (exact scaling; amax/2^e < 512)
 *
 * Scale bytes are stored in the tensor core's scale-factor tiles: for a
 * (rows, cols) matrix, tiles of 128 rows x 4 blocks (128 elements of K),
 * 512 bytes each, ordered tile (i, j) at byte offset (i * ceil(cols/128) + j)
 * * 512; inside a tile the byte of row r (< 128) and block k (< 4) sits at
 *   (r % 32) * 16 + (r / 32) * 4 + k.
 * fp8_mx_scale_bytes(rows, cols) = ceil(rows/128) * ceil(cols/128) * 512.
 * Bytes for rows past `rows` and blocks past cols/32 are padding;
 * fp8_quantize_mx writes them as zero.
 */
FP8SM_API size_t fp8_mx_scale_bytes(int64_t rows, int64_t cols);

/*
 *   x_bf16          (rows, cols) bf16, row stride ld_x (elements, a multiple
 *                   of 8), 16-byte aligned; finite values.
 *   out_fp8         (rows, cols) e4m3 codes, row stride cols, 16-byte aligned.
 *   out_scales_e8m0 fp8_mx_scale_bytes(rows, cols) bytes, 16-byte aligned.
 * Requirements: cols % 32 == 0.  rows == 0 or cols == 0 is a no-op.
 */
FP8SM_API fp8_status fp8_quantize_mx(const void* x_bf16, int64_t rows, int64_t cols,
                           int64_t ld_x, void* out_fp8, void* out_scales_e8m0,
                           fp8_stream_t stream);

/*
 * MXFP8 GEMM:
 *   out[m, n] = sum_k (a[m,k] 2^(sa[m, k/32] - 127)) (b[n,k] 2^(sb[n, k/32] - 127))
 *               (+ bias[n])
 * with sa, sb the E8M0 scale bytes of a (M, K) and b (N, K) in the
 * scale-factor tile layout above (fp8_mx_scale_bytes(M, K) and
 * fp8_mx_scale_bytes(N, K) bytes, 16-byte aligned; padding bytes must not be
 * 0xFF).  The tensor core applies the scales (tcgen05.mma block_scale); fp32
 * accumulation.  out (M, N) bf16 or fp32, 16-byte aligned.
 * Requirements: K > 0, K % 32 == 0, N % 16 == 0.  M == 0 or N == 0 is a no-op.
 */
FP8SM_API fp8_status fp8_scaled_mm_mx(const void* a, const void* b, int64_t M, int64_t N,
                            int64_t K, const void* scale_a_e8m0,
                            const void* scale_b_e8m0, const void* bias_bf16,
                            fp8_out_dtype out_dtype, void* out, fp8_stream_t stream);

/*
 * MXFP8 GEMM whose output leaves MXFP8-quantized, ready to be the A operand
 * of the next MXFP8 GEMM (the chained linear of [P1] Solution, forward pass,
 * with the next layer's activation quantize moved into this GEMM's
 * epilogue).  With y the fp32 result of fp8_scaled_mm_mx (same operands, bias
 * and accumulation order), each block of 32 consecutive columns of a row is
 * quantized exactly as fp8_quantize_mx quantizes a block (e from the fp32
 * amax of y, codes e4m3_satfinite_rn(y * 2^-e)).
 *   out_fp8          (M, N) e4m3 codes, 16-byte aligned.
 *   out_scales_e8m0  fp8_mx_scale_bytes(M, N) bytes in the scale-factor tile
 *                    layout, 16-byte aligned; padding rows are written zero.
 * Requirements: K > 0, K % 32 == 0, N % 128 == 0.
 */
FP8SM_API fp8_status fp8_scaled_mm_mx_quantized(const void* a, const void* b, int64_t M,
                                      int64_t N, int64_t K, const void* scale_a_e8m0,
                                      const void* scale_b_e8m0, const void* bias_bf16,
                                      void* out_fp8, void* out_scales_e8m0,
                                      fp8_stream_t stream);

/*
 * Grouped (MoE) scaled GEMM, rowwise recipe only ([P2] Design, RowWise path;
 * other weight granularities return FP8_ERR_UNSUPPORTED as [P2]'s review
 * requires):
 *   for g in 0..E-1, rows m in [offs[g-1], offs[g])  (offs[-1] = 0):
 *     out[m, n] = sum_k (a[m,k] * scale_a[m]) * (b_experts[g,n,k] * scale_b[g*N + n])
 *
 *   a          (M_total, K) e4m3, 16-byte aligned.
 *   b_experts  (E, N, K) e4m3, 16-byte aligned (the experts' weights as
 *              stored, used as weight.transpose(-2, -1)).
 *   scale_a    (M_total) fp32 per-token scales.
 *   scale_b    (E, N) fp32 per-expert per-output-channel scales.
 *   offs       DEVICE (E) int32 cumulative END offsets: non-decreasing,
 *              offs[E-1] == M_total; empty groups allowed.  It is read on the
 *              device; if it is malformed nothing is written and the device
 *              status becomes FP8_ERR_VALUE.
 *   out        (M_total, N) row-major, bf16 or fp32.
 * Requirements: K % 16 == 0, N % 16 == 0, 1 <= E <= 65535.
 */
FP8SM_API fp8_status fp8_grouped_scaled_mm(const void* a, const void* b_experts,
                                 int64_t M_total, int64_t N, int64_t K,
                                 int32_t E, const float* scale_a,
                                 const float* scale_b, const int32_t* offs,
                                 fp8_out_dtype out_dtype, void* out,
                                 fp8_stream_t stream);

/*
 * Grouped (MoE) scaled GEMM with blockwise scales, the 1x128_128x128 recipe
 * of [P4]/[P5] applied per expert (the blockwise-scaled expert weights that
 * [P2]'s handler leaves for later):
 *   for g in 0..E-1, rows m in [offs[g-1], offs[g]):
 *     out[m, n] = sum_kb scale_a[kb*M_total + m] * scale_b[(g*(K/128) + kb)*ceil(N/128) + n/128]
 *                        * sum_{k in block kb} a[m,k] * b_experts[g,n,k]
 *
 *   a          (M_total, K) e4m3; scale_a (K/128, M_total) fp32 (1x128 groups,
 *              K-block-major as fp8_quantize writes them).
 *   b_experts  (E, N, K) e4m3; scale_b (E, K/128, ceil(N/128)) fp32 (each
 *              expert's 128x128 scales, as fp8_quantize of that expert writes
 *              them).
 *   offs, out, out_dtype, alignment and the device-side offs check as for
 *   fp8_grouped_scaled_mm.
 * Requirements: K % 128 == 0, N % 16 == 0, 1 <= E <= 65535.
 */
FP8SM_API fp8_status fp8_grouped_scaled_mm_blockwise(const void* a, const void* b_experts,
                                                     int64_t M_total, int64_t N, int64_t K,
                                                     int32_t E, const float* scale_a,
                                                     const float* scale_b, const int32_t* offs,
                                                     fp8_out_dtype out_dtype, void* out,
                                                     fp8_stream_t stream);

/*
 * Grouped (MoE) MXFP8 GEMM: for g in 0..E-1, rows m in [offs[g-1], offs[g]):
 *   out[m, n] = sum_k (a[m,k] 2^(sa[m, k/32] - 127)) (b_experts[g,n,k] 2^(sb_g[n, k/32] - 127))
 * (the MoE form of [P2] with the MXFP8 recipe of fp8_scaled_mm_mx).
 *   scale_a_e8m0  A's scale-factor tiles, fp8_mx_scale_bytes(M_total, K)
 *                 bytes (fp8_quantize_mx of a); groups may start anywhere.
 *   scale_b_e8m0  E consecutive per-expert tile sets of fp8_mx_scale_bytes(N, K)
 *                 bytes each (fp8_quantize_mx of each expert's (N, K) weight;
 *                 when N % 128 == 0, also one fp8_quantize_mx of the (E*N, K)
 *                 view).
 *   offs, out, out_dtype as fp8_grouped_scaled_mm.
 * Requirements: K > 0, K % 32 == 0, N % 16 == 0, 1 <= E <= 65535.
 */
FP8SM_API fp8_status fp8_grouped_scaled_mm_mx(const void* a, const void* b_experts,
                                    int64_t M_total, int64_t N, int64_t K, int32_t E,
                                    const void* scale_a_e8m0, const void* scale_b_e8m0,
                                    const int32_t* offs, fp8_out_dtype out_dtype, void* out,
                                    fp8_stream_t stream);

/*
 * MoE weight gradient ([P2]'s grouped layer, backward; the grad_weight GEMM
 * of [P5] with the 1x128_128x1 recipe): for every expert g,
 *   out[g] (M, N) = dY_g^T @ X_g = sum over the tokens t of group g of
 *                   (a_t[m, t] * sa) (b_t[n, t] * sb)
 * where group g's tokens are [offs[g-1], offs[g]).  The contraction runs
 * over each group's own tokens, so 128-token quantization blocks must not
 * mix groups: the operands are quantized per group with
 * fp8_quantize_transposed_grouped, which lays every group's tokens out
 * padded to a multiple of 128 (zero codes in the padding).
 *
 * fp8_grouped_padded_tokens(T, E) = (ceil(T/128) + E) * 128 = P, the padded
 * width (an upper bound of sum_g ceil(size_g/128) * 128, known on the host).
 *
 * fp8_quantize_transposed_grouped: x_bf16 (T, cols) bf16 (row stride ld_x,
 *   a multiple of 8; cols % 8 == 0), offs DEVICE (E) int32 cumulative token
 *   ends (non-decreasing, offs[E-1] == T), 1 <= E <= 2048.  Writes
 *   out_fp8 (cols, P) e4m3 (row stride P; group g's tokens at columns
 *   128 * pb0[g] .., pb0[g] = sum_{h<g} ceil(size_h/128)) and out_scales
 *   (P/128, cols) fp32 (scale[(pb) * cols + c] for padded block pb), each
 *   block's scale from its own group's tokens only.  Columns of the padded
 *   width past the last group are not written.  A malformed offs writes
 *   nothing and sets the device status to FP8_ERR_VALUE.
 * fp8_grouped_scaled_mm_wgrad: a_t (M, P), b_t (N, P) from the quantizer
 *   above (a_t = dY^T with M = the layer's outputs, b_t = X^T with N = its
 *   inputs), scale_a (P/128, M), scale_b (P/128, N), offs as above with
 *   tokens = T; out (E, M, N) bf16 or fp32 (an empty group's gradient is
 *   zero).  Requirements: M % 128 == 0, N % 16 == 0, 1 <= E <= 65535.
 */
FP8SM_API int64_t fp8_grouped_padded_tokens(int64_t tokens, int32_t E);

FP8SM_API fp8_status fp8_quantize_transposed_grouped(const void* x_bf16, int64_t tokens,
                                           int64_t cols, int64_t ld_x, const int32_t* offs,
                                           int32_t E, void* out_fp8, float* out_scales,
                                           fp8_stream_t stream);

FP8SM_API fp8_status fp8_grouped_scaled_mm_wgrad(const void* a_t, const void* b_t, int64_t M,
                                       int64_t N, int64_t tokens, int32_t E,
                                       const float* scale_a, const float* scale_b,
                                       const int32_t* offs, fp8_out_dtype out_dtype,
                                       void* out, fp8_stream_t stream);

/*
 * Synchronizes `stream`, then returns and clears the current device's status
 * word: FP8_OK, FP8_ERR_VALUE (malformed offs), FP8_ERR_TIMEOUT (a pipeline
 * wait gave up; the kernel released its resources and returned), or
 * FP8_ERR_CUDA if the synchronization itself failed.
 */
FP8SM_API fp8_status fp8_get_device_status(fp8_stream_t stream);

/* Message for the last error returned on this host thread ("" if none). */
FP8SM_API const char* fp8_last_error(void);

/*
 * Test hook for the failure-detection path: launches one CTA that waits on a
 * pipeline barrier nothing will ever complete, with a wait limit of
 * `limit_us` microseconds (1..2000000).  The wait gives up, the kernel
 * records FP8_ERR_TIMEOUT in the status word and returns normally, so the
 * CUDA context stays usable.  No counterpart on the pages.
 */
FP8SM_API fp8_status fp8_debug_timeout_probe(uint32_t limit_us, fp8_stream_t stream);

/* Library version (major*10000 + minor*100 + patch). */
FP8SM_API int fp8_version(void);

#ifdef __cplusplus
}
#endif
#endif /* FP8SM_H */
