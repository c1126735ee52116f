/*
 * CPU oracle for the FP8 scaled matrix multiply and its dynamic quantizer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library in
 * fp8_scaled_matrix_b200/) may include, link or call this code; only tests/,
 * the smoke check in __graft_entry__.py and bench.py's CPU-baseline leg do.
 * It shares no source, header, table or constant with the CUDA path.
 *
 * What it computes (plain, slow, obviously correct):
 *   - e4m3 decode from the bit fields (1 sign, 4 exponent bits with bias 7,
 *     3 mantissa bits; subnormals m*2^-9; 0x7F/0xFF NaN; max 448).
 *   - fp32 -> e4m3 round-to-nearest-even with saturation to +-448, by integer
 *     manipulation of the fp32 bit pattern.
 *   - the quantizer: amax over a group -> scale = max(amax, eps)/448 ->
 *     y = x * (448/max(amax, eps)) -> e4m3 code ("per-token scaling for fp8
 *     linear", Highlights: dynamic per-token scale, pre-scaled input, cast).
 *   - MXFP8 (the "mxfp8" recipe of "Add _scaled_mm_v2 API", defined by the
 *     OCP Microscaling specification): power-of-two E8M0 scale per 32
 *     elements, E4M3 elements, and its GEMM.
 *   - the scaled GEMM as the plain definition "dequantize, then matmul"
 *     ("Fix: Handle LowLevelZeroPlugin with use_fp8=True", Solution, forward
 *     pass): products of exactly decoded values, accumulated exactly in int64
 *     per 128-wide K block, then scaled and summed in fp64, plus bias.
 *
 * Parity pins live in tests/test_oracle_*.py (closed forms, torch's own fp8
 * cast, brute force with Python integers/Fractions, hand-worked fixtures under
 * tests/golden/).  Every function here is pinned; none is "parity unpinned".
 */
#ifndef FP8SM_ORACLE_H
#define FP8SM_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Granularity of one quantization group. */
enum {
  OR_GROUP_TENSOR = 0,      /* whole tensor, one scale                       */
  OR_GROUP_ROW = 1,         /* one row (all columns), scales[r]              */
  OR_GROUP_1x128 = 2,       /* 1 row x 128 cols, scales[(c/128)*rows + r]    */
  OR_GROUP_128x128 = 3      /* 128 rows x 128 cols, scales[(c/128)*RB + r/128]
                               with RB = ceil(rows/128)                      */
};

/* GEMM scaling recipes: A scale granularity x B scale granularity. */
enum {
  OR_MM_TENSOR_TENSOR = 0,  /* sA[0], sB[0]                                   */
  OR_MM_ROW_ROW = 1,        /* sA[m], sB[n]                                   */
  OR_MM_1x128_128x128 = 2,  /* sA[kb*M + m], sB[kb*ceil(N/128) + n/128]       */
  OR_MM_1x128_128x1 = 3     /* sA[kb*M + m], sB[kb*N + n]                     */
};

#define OR_EPS 1e-12f

/* Exact value of one e4m3 code (NaN for 0x7F / 0xFF). */
double or_e4m3_decode(uint8_t code);

/* fp32 -> e4m3 code, round to nearest even, saturating at +-448, NaN -> 0x7F,
 * sign of zero kept (negative values that round to zero give 0x80). */
uint8_t or_e4m3_encode(float y);

/* Encode n floats given as raw fp32 bit patterns (used for exhaustive sweeps). */
void or_e4m3_encode_bits(const uint32_t* bits, int64_t n, uint8_t* out);

/* bf16 bit pattern -> float (exact). */
float or_bf16_to_float(uint16_t h);

/* Dynamic quantization of a bf16 matrix x (rows x cols, row stride ld, in
 * elements) into e4m3 codes q (rows x cols, row stride cols) and fp32 scales
 * (layout per group kind, see the enum).  Returns 0, or -1 on bad arguments.
 * Blockwise kinds need cols % 128 == 0. */
int or_quantize(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                int group, uint8_t* q, float* scales);

/* or_quantize on fp32 input x (row stride ld): the same steps; used to check
 * a GEMM whose epilogue quantizes its fp32 result. */
int or_quantize_f32(const float* x, int64_t rows, int64_t cols, int64_t ld,
                    int group, uint8_t* q, float* scales);

/* Cast step alone with a caller-supplied inverse scale: q = e4m3(x * inv).
 * Used to pin saturation, which the amax-derived scale never reaches. */
int or_cast_with_inverse(const uint16_t* x, int64_t rows, int64_t cols,
                         int64_t ld, float inv, uint8_t* q);

/* Scaled GEMM reference for the listed output rows.
 *   a: (M,K) e4m3 codes row-major; b: (N,K) e4m3 codes row-major.
 *   bias: N bf16 bit patterns or NULL.
 *   rows: n_rows row indices (or NULL = all M rows, n_rows ignored).
 *   ref, mag: (n_rows, N) fp64 outputs: the exact-products reference value
 *   and the magnitude sum  sum_kb |sA||sB| sum_k |a_k b_k|  used by the
 *   tolerance |out - ref| <= 1e-2 |ref| + 1e-3 mag.
 * Returns 0, or -1 on bad arguments. */
int or_scaled_mm(const uint8_t* a, const uint8_t* b, int64_t M, int64_t N,
                 int64_t K, const float* sA, const float* sB, int recipe,
                 const uint16_t* bias, const int64_t* rows, int64_t n_rows,
                 double* ref, double* mag);

/* Same definition written the other way round ("dequantize then matmul"):
 * decode each operand to fp64, multiply by its scale, then a plain
 * triple-loop matmul in fp64, plus bias.  All M rows. */
int or_dequant_then_matmul(const uint8_t* a, const uint8_t* b, int64_t M,
                           int64_t N, int64_t K, const float* sA,
                           const float* sB, int recipe, const uint16_t* bias,
                           double* ref);

/* Grouped (MoE) GEMM: rows [offs[g-1], offs[g]) of a (offs[-1] = 0) times
 * expert g of b_experts (E,N,K), rowwise scales sA (M_total) and sB (E,N).
 * offs: E cumulative end offsets, non-decreasing, offs[E-1] == M_total.
 * rows/n_rows as in or_scaled_mm.  Returns 0, or -1 on bad arguments
 * (including a malformed offs array). */
int or_grouped_scaled_mm(const uint8_t* a, const uint8_t* b_experts,
                         int64_t M_total, int64_t N, int64_t K, int32_t E,
                         const float* sA, const float* sB, const int32_t* offs,
                         const int64_t* rows, int64_t n_rows, double* ref,
                         double* mag);

/* MXFP8 (OCP Microscaling, E4M3 elements, one E8M0 scale per 32 elements
 * along each row).  x: (rows, cols) bf16 bit patterns, row stride ld,
 * cols % 32 == 0.  q: (rows, cols) codes; e8: (rows, cols/32) scale bytes
 * (2^(byte-127)).  Returns 0, or -1 on bad arguments. */
int or_mx_quantize(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                   uint8_t* q, uint8_t* e8);

/* or_mx_quantize on fp32 input x (row stride ld): the same steps. */
int or_mx_quantize_f32(const float* x, int64_t rows, int64_t cols, int64_t ld,
                       uint8_t* q, uint8_t* e8);

/* e8 (rows, kblocks) rearranged into 512-byte scale-factor tiles (128 rows x
 * 4 blocks each, row-tile-major; byte (r%32)*16 + (r/32)*4 + k inside), zero
 * past the matrix.  tiles holds ceil(rows/128) * ceil(kblocks/4) * 512 bytes. */
int or_mx_scales_to_tiles(const uint8_t* e8, int64_t rows, int64_t kblocks,
                          uint8_t* tiles);

/* MXFP8 GEMM reference: a (M,K), b (N,K) codes; ea (M,K/32), eb (N,K/32)
 * plain scale bytes; bias, rows, ref, mag as in or_scaled_mm. */
int or_mx_scaled_mm(const uint8_t* a, const uint8_t* b, int64_t M, int64_t N,
                    int64_t K, const uint8_t* ea, const uint8_t* eb,
                    const uint16_t* bias, const int64_t* rows, int64_t n_rows,
                    double* ref, double* mag);

/* Threads the oracle's OpenMP loops use (1 when built without OpenMP). */
int or_num_threads(void);

#ifdef __cplusplus
}
#endif
#endif
