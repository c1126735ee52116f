/*
 * CPU oracle: TEST INFRASTRUCTURE ONLY (see oracle.h).  Plain C99, built with
 * -O2 -ffp-contract=off so every fp32 operation is a single IEEE operation
 * rounded to nearest even, exactly as written.
 *
 * Sources on the pages:
 *   - "per-token scaling for fp8 linear" (DiffSynth-Engine PR #160),
 *     Highlights: per-row amax -> scale, input divided by the scale (plus a
 *     small epsilon), cast to fp8.
 *   - "Fix: Handle LowLevelZeroPlugin with use_fp8=True" (ColossalAI PR
 *     #6419), Solution, forward pass: scaled-mm equals dequantize-then-matmul,
 *     bias added after the matmul.
 *   - "Add _scaled_mm_v2 API" (PyTorch PR #164141), Blas.cpp review threads:
 *     A, B fp8 with fp32 scales; Blockwise_1x128 for A, Blockwise_128x128 for B.
 *   - "improve fp8 blockwise gemm perf" (torchao PR #2784): the 1x128_128x128
 *     and 1x128_128x1 recipes and their GEMMs.
 *   - "Add _grouped_mm dispatch handler to Float8Tensor" (torchao PR #4390):
 *     (E, N, K) expert weights, rowwise scales of shape (E, N), offs.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int or_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ------------------------------------------------------------------ e4m3 */

/* Bit fields: s eeee mmm, exponent bias 7.  E == 0 is subnormal (m * 2^-9);
 * E == 15 with m == 7 is NaN; everything else (1 + m/8) * 2^(E-7). */
double or_e4m3_decode(uint8_t code) {
  int s = code >> 7;
  int E = (code >> 3) & 0xF;
  int m = code & 0x7;
  double v;
  if (E == 15 && m == 7) return NAN;
  if (E == 0)
    v = ldexp((double)m, -9);
  else
    v = ldexp(1.0 + m / 8.0, E - 7);
  return s ? -v : v;
}

/* Right-shift an unsigned significand by sh bits, rounding to nearest even. */
static uint64_t rne_shift(uint64_t sig, int sh) {
  if (sh <= 0) return sig << (-sh);
  if (sh >= 63) return 0; /* far below half of the quantum */
  uint64_t q = sig >> sh;
  uint64_t rem = sig & ((1ull << sh) - 1);
  uint64_t half = 1ull << (sh - 1);
  if (rem > half || (rem == half && (q & 1))) q += 1;
  return q;
}

uint8_t or_e4m3_encode(float y) {
  uint32_t u;
  memcpy(&u, &y, 4);
  uint8_t sign = (u >> 31) ? 0x80 : 0x00;
  uint32_t au = u & 0x7FFFFFFFu;
  if (au > 0x7F800000u) return 0x7F; /* NaN */
  if (au == 0) return sign;
  if (au == 0x7F800000u) return sign | 0x7E; /* +-inf saturates */

  /* |y| = sig * 2^ex exactly, sig an integer below 2^24. */
  int bexp = (int)(au >> 23);
  uint64_t sig;
  int ex;
  if (bexp == 0) {
    sig = au & 0x7FFFFF;
    ex = -149;
  } else {
    sig = (au & 0x7FFFFF) | 0x800000;
    ex = bexp - 150;
  }
  /* Unbiased exponent of the leading bit of |y|. */
  int lead = 63 - __builtin_clzll(sig) + ex;

  /* Quantum of e4m3 around |y|: 2^(lead-3) in the normal range (lead >= -6),
   * 2^-9 in the subnormal range. */
  int qexp = lead >= -6 ? lead - 3 : -9;
  /* n = |y| / 2^qexp rounded to nearest even. */
  uint64_t n = rne_shift(sig, qexp - ex);
  /* Rebuild the value n * 2^qexp as a code.  n may have carried to 16 (next
   * binade) in the normal range, or to 8 (the smallest normal) from below. */
  int E, m;
  if (lead < -6) {
    if (n >= 8) { /* rounded up into the normal range: 2^-6 */
      E = 1;
      m = (int)(n - 8);
    } else {
      E = 0;
      m = (int)n;
    }
  } else {
    int e = lead;
    if (n >= 16) { /* carry into the next binade */
      n >>= 1;
      e += 1;
    }
    E = e + 7;
    m = (int)(n - 8);
  }
  /* Saturate: anything past 448 (E=15, m=6) becomes 448. */
  if (E > 15 || (E == 15 && m > 6)) {
    E = 15;
    m = 6;
  }
  return (uint8_t)(sign | (E << 3) | m);
}

void or_e4m3_encode_bits(const uint32_t* bits, int64_t n, uint8_t* out) {
  int64_t i;
#pragma omp parallel for schedule(static)
  for (i = 0; i < n; i++) {
    float f;
    memcpy(&f, &bits[i], 4);
    out[i] = or_e4m3_encode(f);
  }
}

float or_bf16_to_float(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* ------------------------------------------------------------- quantizer */

/* One group: steps of the dynamic quantizer in order.
 *   1. amax = max |x| over the group
 *   2. a = max(amax, eps)               (epsilon guard)
 *   3. scale = a / 448 (stored), inv = 448 / a
 *   4. y = x * inv                       (one fp32 multiply)
 *   5. q = e4m3(y), RNE, saturating */
typedef struct {
  const uint16_t* x;   /* bf16 input, or */
  const float* xf;     /* fp32 input (when not NULL) */
  int64_t ld;
  uint8_t* q;
  int64_t ldq;
} mat_view;

static float mv_get(const mat_view* v, int64_t i) {
  return v->xf ? v->xf[i] : or_bf16_to_float(v->x[i]);
}

static float group_scale(const mat_view* v, int64_t r0, int64_t r1, int64_t c0,
                         int64_t c1, float* inv_out) {
  float amax = 0.0f;
  for (int64_t r = r0; r < r1; r++)
    for (int64_t c = c0; c < c1; c++) {
      float f = fabsf(mv_get(v, r * v->ld + c));
      if (f > amax) amax = f;
    }
  float a = amax > OR_EPS ? amax : OR_EPS;
  volatile float s = a / 448.0f;
  volatile float inv = 448.0f / a;
  *inv_out = inv;
  return s;
}

static void group_cast(const mat_view* v, int64_t r0, int64_t r1, int64_t c0,
                       int64_t c1, float inv) {
  for (int64_t r = r0; r < r1; r++)
    for (int64_t c = c0; c < c1; c++) {
      volatile float y = mv_get(v, r * v->ld + c) * inv;
      v->q[r * v->ldq + c] = or_e4m3_encode(y);
    }
}

static int quantize_view(const mat_view* vp, int64_t rows, int64_t cols, int group,
                         float* scales) {
  const mat_view v = *vp;
  if (group == OR_GROUP_TENSOR) {
    float inv;
    scales[0] = group_scale(&v, 0, rows, 0, cols, &inv);
    group_cast(&v, 0, rows, 0, cols, inv);
    return 0;
  }
  if (group == OR_GROUP_ROW) {
    int64_t r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < rows; r++) {
      float inv;
      scales[r] = group_scale(&v, r, r + 1, 0, cols, &inv);
      group_cast(&v, r, r + 1, 0, cols, inv);
    }
    return 0;
  }
  if (cols % 128 != 0) return -1;
  int64_t KB = cols / 128;
  if (group == OR_GROUP_1x128) {
    int64_t r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < rows; r++)
      for (int64_t kb = 0; kb < KB; kb++) {
        float inv;
        scales[kb * rows + r] =
            group_scale(&v, r, r + 1, kb * 128, kb * 128 + 128, &inv);
        group_cast(&v, r, r + 1, kb * 128, kb * 128 + 128, inv);
      }
    return 0;
  }
  if (group == OR_GROUP_128x128) {
    int64_t RB = (rows + 127) / 128;
    int64_t rb;
#pragma omp parallel for schedule(static)
    for (rb = 0; rb < RB; rb++)
      for (int64_t kb = 0; kb < KB; kb++) {
        int64_t r0 = rb * 128, r1 = r0 + 128 < rows ? r0 + 128 : rows;
        float inv;
        scales[kb * RB + rb] =
            group_scale(&v, r0, r1, kb * 128, kb * 128 + 128, &inv);
        group_cast(&v, r0, r1, kb * 128, kb * 128 + 128, inv);
      }
    return 0;
  }
  return -1;
}

int or_quantize(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                int group, uint8_t* q, float* scales) {
  if (rows < 0 || cols < 0 || ld < cols || !x || !q || !scales) return -1;
  mat_view v = {x, NULL, ld, q, cols};
  return quantize_view(&v, rows, cols, group, scales);
}

/* The same steps on fp32 input (a GEMM result quantized for the next FP8
 * operation). */
int or_quantize_f32(const float* x, int64_t rows, int64_t cols, int64_t ld,
                    int group, uint8_t* q, float* scales) {
  if (rows < 0 || cols < 0 || ld < cols || !x || !q || !scales) return -1;
  mat_view v = {NULL, x, ld, q, cols};
  return quantize_view(&v, rows, cols, group, scales);
}

int or_cast_with_inverse(const uint16_t* x, int64_t rows, int64_t cols,
                         int64_t ld, float inv, uint8_t* q) {
  if (rows < 0 || cols < 0 || ld < cols || !x || !q) return -1;
  mat_view v = {x, NULL, ld, q, cols};
  group_cast(&v, 0, rows, 0, cols, inv);
  return 0;
}

/* ------------------------------------------------------------------ GEMM */

/* Every finite e4m3 value times 2^9 is an integer (smallest step 2^-9), at
 * most 448 * 512 = 229376 in magnitude.  A product of two is below 2^36 and a
 * sum of up to 2^26 of them stays far below 2^63, so int64 sums are exact. */
static int32_t lut_int[256];
static int lut_nan[256];
static int lut_ready = 0;

static void build_lut(void) {
  if (lut_ready) return;
  for (int c = 0; c < 256; c++) {
    double v = or_e4m3_decode((uint8_t)c);
    lut_nan[c] = isnan(v);
    lut_int[c] = lut_nan[c] ? 0 : (int32_t)ldexp(v, 9);
  }
  lut_ready = 1;
}

static double bias_at(const uint16_t* bias, int64_t n) {
  return bias ? (double)or_bf16_to_float(bias[n]) : 0.0;
}

static int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

/* Scale pair for output (m, n) and K block kb, per recipe. */
static void scale_pair(int recipe, const float* sA, const float* sB, int64_t M,
                       int64_t N, int64_t m, int64_t n, int64_t kb, double* sa,
                       double* sb) {
  switch (recipe) {
    case OR_MM_TENSOR_TENSOR:
      *sa = sA[0];
      *sb = sB[0];
      break;
    case OR_MM_ROW_ROW:
      *sa = sA[m];
      *sb = sB[n];
      break;
    case OR_MM_1x128_128x128:
      *sa = sA[kb * M + m];
      *sb = sB[kb * ceil_div(N, 128) + n / 128];
      break;
    default: /* OR_MM_1x128_128x1 */
      *sa = sA[kb * M + m];
      *sb = sB[kb * N + n];
      break;
  }
}

/* One output element: exact per-block integer dot products, then
 *   ref = 2^-18 * sum_kb sA*sB*D_kb (+ bias),  mag = 2^-18 * sum_kb |sA sB| |D|_kb */
static void dot_one(const uint8_t* arow, const uint8_t* brow, int64_t K,
                    int recipe, const float* sA, const float* sB, int64_t M,
                    int64_t N, int64_t m, int64_t n, double bias, double* ref,
                    double* mag) {
  double acc = 0.0, accm = 0.0;
  int any_nan = 0;
  int64_t KB = ceil_div(K, 128);
  for (int64_t kb = 0; kb < KB; kb++) {
    int64_t k0 = kb * 128, k1 = k0 + 128 < K ? k0 + 128 : K;
    int64_t d = 0, dabs = 0;
    for (int64_t k = k0; k < k1; k++) {
      int64_t p = (int64_t)lut_int[arow[k]] * (int64_t)lut_int[brow[k]];
      d += p;
      dabs += p < 0 ? -p : p;
      any_nan |= lut_nan[arow[k]] | lut_nan[brow[k]];
    }
    double sa, sb;
    scale_pair(recipe, sA, sB, M, N, m, n, kb, &sa, &sb);
    acc += sa * sb * (double)d;
    accm += fabs(sa * sb) * (double)dabs;
  }
  *ref = any_nan ? NAN : ldexp(acc, -18) + bias;
  *mag = ldexp(accm, -18);
}

static int recipe_ok(int recipe, int64_t K) {
  if (recipe == OR_MM_TENSOR_TENSOR || recipe == OR_MM_ROW_ROW) return 1;
  if (recipe == OR_MM_1x128_128x128 || recipe == OR_MM_1x128_128x1)
    return K % 128 == 0;
  return 0;
}

int or_scaled_mm(const uint8_t* a, const uint8_t* b, int64_t M, int64_t N,
                 int64_t K, const float* sA, const float* sB, int recipe,
                 const uint16_t* bias, const int64_t* rows, int64_t n_rows,
                 double* ref, double* mag) {
  if (M < 0 || N < 0 || K < 0 || !recipe_ok(recipe, K)) return -1;
  build_lut();
  int64_t R = rows ? n_rows : M;
  for (int64_t i = 0; i < R; i++)
    if (rows && (rows[i] < 0 || rows[i] >= M)) return -1;
  int64_t i;
#pragma omp parallel for schedule(dynamic, 1)
  for (i = 0; i < R; i++) {
    int64_t m = rows ? rows[i] : i;
    for (int64_t n = 0; n < N; n++)
      dot_one(a + m * K, b + n * K, K, recipe, sA, sB, M, N, m, n,
              bias_at(bias, n), &ref[i * N + n], &mag[i * N + n]);
  }
  return 0;
}

int or_dequant_then_matmul(const uint8_t* a, const uint8_t* b, int64_t M,
                           int64_t N, int64_t K, const float* sA,
                           const float* sB, int recipe, const uint16_t* bias,
                           double* ref) {
  if (M < 0 || N < 0 || K < 0 || !recipe_ok(recipe, K)) return -1;
  /* Dequantize both operands to fp64 with their scales ... */
  double* ad = (double*)malloc(sizeof(double) * (size_t)(M * K + 1));
  double* bd = (double*)malloc(sizeof(double) * (size_t)(N * K + 1));
  if (!ad || !bd) {
    free(ad);
    free(bd);
    return -1;
  }
  for (int64_t m = 0; m < M; m++)
    for (int64_t k = 0; k < K; k++) {
      double sa, sb;
      scale_pair(recipe, sA, sB, M, N, m, 0, k / 128, &sa, &sb);
      ad[m * K + k] = or_e4m3_decode(a[m * K + k]) * sa;
    }
  for (int64_t n = 0; n < N; n++)
    for (int64_t k = 0; k < K; k++) {
      double sa, sb;
      scale_pair(recipe, sA, sB, M, N, 0, n, k / 128, &sa, &sb);
      bd[n * K + k] = or_e4m3_decode(b[n * K + k]) * sb;
    }
  /* ... then a plain matmul, then the bias. */
  for (int64_t m = 0; m < M; m++)
    for (int64_t n = 0; n < N; n++) {
      double s = 0.0;
      for (int64_t k = 0; k < K; k++) s += ad[m * K + k] * bd[n * K + k];
      ref[m * N + n] = s + bias_at(bias, n);
    }
  free(ad);
  free(bd);
  return 0;
}

int or_grouped_scaled_mm(const uint8_t* a, const uint8_t* b_experts,
                         int64_t M_total, int64_t N, int64_t K, int32_t E,
                         const float* sA, const float* sB, const int32_t* offs,
                         const int64_t* rows, int64_t n_rows, double* ref,
                         double* mag) {
  if (M_total < 0 || N < 0 || K < 0 || E <= 0 || !offs) return -1;
  int32_t prev = 0;
  for (int32_t g = 0; g < E; g++) {
    if (offs[g] < prev) return -1;
    prev = offs[g];
  }
  if ((int64_t)offs[E - 1] != M_total) return -1;
  build_lut();
  int64_t R = rows ? n_rows : M_total;
  for (int64_t i = 0; i < R; i++)
    if (rows && (rows[i] < 0 || rows[i] >= M_total)) return -1;
  int64_t i;
#pragma omp parallel for schedule(dynamic, 1)
  for (i = 0; i < R; i++) {
    int64_t m = rows ? rows[i] : i;
    /* group of row m: the first g with m < offs[g] */
    int32_t g = 0;
    while (m >= (int64_t)offs[g]) g++;
    const uint8_t* bg = b_experts + (int64_t)g * N * K;
    const float* sBg = sB + (int64_t)g * N;
    for (int64_t n = 0; n < N; n++)
      dot_one(a + m * K, bg + n * K, K, OR_MM_ROW_ROW, sA, sBg, M_total, N, m,
              n, 0.0, &ref[i * N + n], &mag[i * N + n]);
  }
  return 0;
}

/* ----------------------------------------------------------------- MXFP8 */

/* "Add _scaled_mm_v2 API" (Blas.cpp review, recipe table) names an "mxfp8"
 * recipe (MXFP8_MXFP8) without defining it; the name is the OCP Microscaling
 * (MX) format, whose published definition (OCP MX v1.0) is followed here:
 * each block of 32 consecutive elements along the contraction dimension has
 * one E8M0 scale X = 2^e (stored as the byte e + 127), and elements are E4M3.
 * Converting one block, in the specification's order:
 *   1. amax = max |v_i| over the block
 *   2. e = floor(log2(amax)) - 8   (8 = exponent of 256, the largest power of
 *      two E4M3 represents); an all-zero block takes e = -127; e is clamped
 *      to the E8M0 range [-127, 127]
 *   3. q_i = E4M3(v_i / 2^e), round to nearest even, saturating at +-448
 *      (the specification leaves overflow to the implementation; values of a
 *      block with amax in [448, 512) * 2^e saturate). */
static int mx_block_exponent(float amax) {
  if (amax == 0.0f) return -127;
  int fe;
  (void)frexp((double)amax, &fe); /* amax = f * 2^fe, 0.5 <= f < 1 */
  int e = (fe - 1) - 8;
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return e;
}

/* One row of blocks; x values read through mv_get (bf16 or fp32 input). */
static void mx_quantize_row(const mat_view* v, int64_t r, int64_t cols, uint8_t* e8) {
  int64_t KB = cols / 32;
  for (int64_t kb = 0; kb < KB; kb++) {
    float amax = 0.0f;
    for (int i = 0; i < 32; i++) {
      float f = fabsf(mv_get(v, r * v->ld + kb * 32 + i));
      if (f > amax) amax = f;
    }
    int e = mx_block_exponent(amax);
    e8[r * KB + kb] = (uint8_t)(e + 127);
    for (int i = 0; i < 32; i++) {
      /* v / 2^e is exact in fp64; below 2^-126 it rounds to zero in E4M3
       * whatever the fp32 rounding, so the float conversion loses nothing */
      double y = ldexp((double)mv_get(v, r * v->ld + kb * 32 + i), -e);
      v->q[r * v->ldq + kb * 32 + i] = or_e4m3_encode((float)y);
    }
  }
}

int or_mx_quantize(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                   uint8_t* q, uint8_t* e8) {
  if (rows < 0 || cols < 0 || cols % 32 != 0 || ld < cols || !x || !q || !e8)
    return -1;
  mat_view v = {x, NULL, ld, q, cols};
  int64_t r;
#pragma omp parallel for schedule(static)
  for (r = 0; r < rows; r++) mx_quantize_row(&v, r, cols, e8);
  return 0;
}

/* The same conversion of an fp32 matrix (a GEMM result quantized for the
 * next MXFP8 GEMM). */
int or_mx_quantize_f32(const float* x, int64_t rows, int64_t cols, int64_t ld,
                       uint8_t* q, uint8_t* e8) {
  if (rows < 0 || cols < 0 || cols % 32 != 0 || ld < cols || !x || !q || !e8)
    return -1;
  mat_view v = {NULL, x, ld, q, cols};
  int64_t r;
#pragma omp parallel for schedule(static)
  for (r = 0; r < rows; r++) mx_quantize_row(&v, r, cols, e8);
  return 0;
}

/* Scale bytes rearranged into the tensor core's scale-factor tiles: one
 * 512-byte tile per 128 rows x 4 blocks (128 elements of K), tiles ordered
 * row-tile-major, and inside a tile the byte of (row r, block k) at
 *   (r % 32) * 16 + (r / 32) * 4 + k        (r < 128, k < 4).
 * Positions past the matrix (rows beyond `rows`, blocks beyond `kblocks`)
 * are zero. */
int or_mx_scales_to_tiles(const uint8_t* e8, int64_t rows, int64_t kblocks,
                          uint8_t* tiles) {
  if (rows < 0 || kblocks < 0 || !e8 || !tiles) return -1;
  int64_t RT = ceil_div(rows, 128), KT = ceil_div(kblocks, 4);
  memset(tiles, 0, (size_t)(RT * KT * 512));
  for (int64_t r = 0; r < rows; r++)
    for (int64_t kb = 0; kb < kblocks; kb++) {
      int64_t tile = (r / 128) * KT + kb / 4;
      int64_t rr = r % 128, k = kb % 4;
      tiles[tile * 512 + (rr % 32) * 16 + (rr / 32) * 4 + k] = e8[r * kblocks + kb];
    }
  return 0;
}

/* MXFP8 GEMM: out[m, n] = sum_k (a[m,k] 2^(ea[m,k/32]-127)) (b[n,k]
 * 2^(eb[n,k/32]-127)) (+ bias[n]).  Exact integer dot product per 32-block,
 * scaled by the power of two and summed in fp64; mag as in or_scaled_mm.
 * ea (M, K/32), eb (N, K/32): plain row-major E8M0 bytes. */
int or_mx_scaled_mm(const uint8_t* a, const uint8_t* b, int64_t M, int64_t N,
                    int64_t K, const uint8_t* ea, const uint8_t* eb,
                    const uint16_t* bias, const int64_t* rows, int64_t n_rows,
                    double* ref, double* mag) {
  if (M < 0 || N < 0 || K < 0 || K % 32 != 0 || !ref || !mag) return -1;
  build_lut();
  int64_t R = rows ? n_rows : M;
  for (int64_t i = 0; i < R; i++)
    if (rows && (rows[i] < 0 || rows[i] >= M)) return -1;
  int64_t KB = K / 32;
  int64_t i;
#pragma omp parallel for schedule(dynamic, 1)
  for (i = 0; i < R; i++) {
    int64_t m = rows ? rows[i] : i;
    const uint8_t* arow = a + m * K;
    for (int64_t n = 0; n < N; n++) {
      const uint8_t* brow = b + n * K;
      double acc = 0.0, accm = 0.0;
      int any_nan = 0;
      for (int64_t kb = 0; kb < KB; kb++) {
        int64_t d = 0, dabs = 0;
        for (int64_t k = kb * 32; k < kb * 32 + 32; k++) {
          int64_t p = (int64_t)lut_int[arow[k]] * (int64_t)lut_int[brow[k]];
          d += p;
          dabs += p < 0 ? -p : p;
          any_nan |= lut_nan[arow[k]] | lut_nan[brow[k]];
        }
        int ex = (int)ea[m * KB + kb] - 127 + (int)eb[n * KB + kb] - 127;
        any_nan |= ea[m * KB + kb] == 0xFF || eb[n * KB + kb] == 0xFF;
        acc += ldexp((double)d, ex - 18);
        accm += ldexp((double)dabs, ex - 18);
      }
      ref[i * N + n] = any_nan ? NAN : acc + bias_at(bias, n);
      mag[i * N + n] = accm;
    }
  }
  return 0;
}
