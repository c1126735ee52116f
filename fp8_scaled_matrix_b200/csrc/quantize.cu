// Dynamic e4m3 quantizers ("per-token scaling for fp8 linear", Highlights:
// per-row amax -> scale, input pre-scaled, fp8 cast; the 1x128 / 128x128
// groups of "Add _scaled_mm_v2 API" and "improve fp8 blockwise gemm perf").
//
// Per group G:  a = max(max|x|, 1e-12);  scale = a / 448;  inv = 448 / a;
//               q = cvt.rn.satfinite.e4m3(x * inv)
// Every step is one IEEE fp32 operation (no FMA contraction, no fast math),
// so the codes and scales are bit-identical to any other implementation of
// the same steps.
//
// HBM-bound: 2 bytes read + 1 byte written per element.  All kernels move
// 16-byte vectors (8 bf16 in, 8 e4m3 out or 16 in / 16 out), reduce the
// amax with warp shuffles, and keep the group in registers between the amax
// and the cast so x is read from HBM once (the tensorwise recipe re-reads x
// when it does not fit on chip).
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "fp8cast.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace fp8sm {
namespace {

__device__ __forceinline__ float bf16_lo(uint32_t w) {
  return __uint_as_float(w << 16);
}
__device__ __forceinline__ float bf16_hi(uint32_t w) {
  return __uint_as_float(w & 0xFFFF0000u);
}

__device__ __forceinline__ float amax8(const uint4& v, float m) {
  m = fmaxf(m, fabsf(bf16_lo(v.x)));
  m = fmaxf(m, fabsf(bf16_hi(v.x)));
  m = fmaxf(m, fabsf(bf16_lo(v.y)));
  m = fmaxf(m, fabsf(bf16_hi(v.y)));
  m = fmaxf(m, fabsf(bf16_lo(v.z)));
  m = fmaxf(m, fabsf(bf16_hi(v.z)));
  m = fmaxf(m, fabsf(bf16_lo(v.w)));
  m = fmaxf(m, fabsf(bf16_hi(v.w)));
  return m;
}

__device__ __forceinline__ uint32_t cast2(uint32_t w, float inv) {
  return cast_f32x2(bf16_lo(w), bf16_hi(w), inv);
}

// 8 bf16 -> 8 e4m3 bytes (little-endian order preserved).
__device__ __forceinline__ uint2 cast8(const uint4& v, float inv) {
  return make_uint2(cast2(v.x, inv) | (cast2(v.y, inv) << 16),
                    cast2(v.z, inv) | (cast2(v.w, inv) << 16));
}

__device__ __forceinline__ float warp_max(float m) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  return m;
}

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  return __ldcs(p);
}

// ------------------------------------------------------------ rowwise
// One warp per row; lane l holds vectors l, l+32, ... (VPT of them) in
// registers, so each row is read once.  cols <= 256 * VPT.
template <int VPT>
__global__ void __launch_bounds__(256) quant_row_kernel(
    const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
    uint8_t* __restrict__ q, float* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int nvec = static_cast<int>(cols >> 3);
  const uint4* xr = reinterpret_cast<const uint4*>(x + row * ld);
  uint4 v[VPT];
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int idx = i * 32 + lane;
    if (idx < nvec) {
      v[i] = ld_stream(xr + idx);
      m = amax8(v[i], m);
    }
  }
  m = warp_max(m);
  const ScalePair sp = scales_from_amax(m);
  if (lane == 0) scales[row] = sp.s;
  uint2* qr = reinterpret_cast<uint2*>(q + row * cols);
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int idx = i * 32 + lane;
    if (idx < nvec) qr[idx] = cast8(v[i], sp.inv);
  }
}

// One CTA per row (rows up to 16384 columns): thread t holds 16 consecutive
// elements (two 16-byte loads, one 16-byte store); warp amax -> shared
// memory -> block amax.  Many small CTAs keep enough loads in flight and let
// the stores of finishing CTAs overlap the loads of new ones.
__global__ void __launch_bounds__(1024) quant_row_cta_kernel(
    const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
    uint8_t* __restrict__ q, float* __restrict__ scales) {
  __shared__ float warp_amax[32];
  const int64_t row = blockIdx.x;
  const int t = threadIdx.x;
  const int nvec = static_cast<int>(cols >> 3);
  const uint4* xr = reinterpret_cast<const uint4*>(x + row * ld);
  const int i0 = 2 * t;
  const bool v0 = i0 < nvec, v1 = i0 + 1 < nvec;
  uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
  if (v0) a = ld_stream(xr + i0);
  if (v1) b = ld_stream(xr + i0 + 1);
  float m = amax8(b, amax8(a, 0.0f));  // zero padding does not change the max
  m = warp_max(m);
  if ((t & 31) == 0) warp_amax[t >> 5] = m;
  __syncthreads();
  const int nw = static_cast<int>(blockDim.x >> 5);
  float bm = warp_amax[0];
  for (int i = 1; i < nw; ++i) bm = fmaxf(bm, warp_amax[i]);
  const ScalePair sp = scales_from_amax(bm);
  if (t == 0) scales[row] = sp.s;
  uint8_t* qr = q + row * cols + static_cast<int64_t>(i0) * 8;
  // 16-byte stores need cols % 16 == 0 (row starts 16-byte aligned);
  // otherwise two 8-byte stores.
  if (v1 && (cols & 15) == 0) {
    const uint2 lo = cast8(a, sp.inv), hi = cast8(b, sp.inv);
    *reinterpret_cast<uint4*>(qr) = make_uint4(lo.x, lo.y, hi.x, hi.y);
  } else {
    if (v0) *reinterpret_cast<uint2*>(qr) = cast8(a, sp.inv);
    if (v1) *reinterpret_cast<uint2*>(qr + 8) = cast8(b, sp.inv);
  }
}

// Rows longer than 256*16 elements: amax pass, then a second read (served
// from L2 for the row just read) for the cast.
__global__ void __launch_bounds__(256) quant_row_long_kernel(
    const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
    uint8_t* __restrict__ q, float* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int64_t nvec = cols >> 3;
  const uint4* xr = reinterpret_cast<const uint4*>(x + row * ld);
  float m = 0.0f;
  for (int64_t base = 0; base < nvec; base += 128) {
    uint4 v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t idx = base + i * 32 + lane;
      if (idx < nvec) v[i] = __ldg(xr + idx);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t idx = base + i * 32 + lane;
      if (idx < nvec) m = amax8(v[i], m);
    }
  }
  m = warp_max(m);
  const ScalePair sp = scales_from_amax(m);
  if (lane == 0) scales[row] = sp.s;
  uint2* qr = reinterpret_cast<uint2*>(q + row * cols);
  for (int64_t idx = lane; idx < nvec; idx += 32)
    qr[idx] = cast8(ld_stream(xr + idx), sp.inv);
}

// -------------------------------------------------------------- 1x128
// A warp handles 4 rows x one 128-column block per task: lane = 8*g + j
// covers row r0+g, columns kb*128 + 16j .. +16 (two 16-byte loads, one
// 16-byte store).  Scales K-block-major: scales[kb*rows + r], so one warp
// writes 4 consecutive floats.  Each warp runs kTasks tasks (the next K
// blocks of the same rows) with all loads issued first.
constexpr int k1x128Tasks = 4;

__global__ void __launch_bounds__(256) quant_1x128_kernel(
    const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
    uint8_t* __restrict__ q, float* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int g = lane >> 3;
  const int j = lane & 7;
  const int64_t KB = cols >> 7;
  const int64_t kb_groups = (KB + k1x128Tasks - 1) / k1x128Tasks;
  const int64_t warp = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int64_t quad = warp / kb_groups;
  const int64_t kb0 = (warp % kb_groups) * k1x128Tasks;
  const int64_t row = quad * 4 + g;
  const bool row_ok = row < rows;
  if (quad * 4 >= rows) return;
  uint4 v[k1x128Tasks][2];
#pragma unroll
  for (int t = 0; t < k1x128Tasks; ++t) {
    const int64_t kb = kb0 + t;
    if (row_ok && kb < KB) {
      const uint4* p = reinterpret_cast<const uint4*>(x + row * ld + kb * 128 + j * 16);
      v[t][0] = ld_stream(p);
      v[t][1] = ld_stream(p + 1);
    }
  }
#pragma unroll
  for (int t = 0; t < k1x128Tasks; ++t) {
    const int64_t kb = kb0 + t;
    if (kb >= KB) break;  // uniform across the warp
    float m = 0.0f;
    if (row_ok) m = amax8(v[t][1], amax8(v[t][0], 0.0f));
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
    if (!row_ok) continue;
    const ScalePair sp = scales_from_amax(m);
    if (j == 0) scales[kb * rows + row] = sp.s;
    const uint2 lo = cast8(v[t][0], sp.inv);
    const uint2 hi = cast8(v[t][1], sp.inv);
    *reinterpret_cast<uint4*>(q + row * cols + kb * 128 + j * 16) =
        make_uint4(lo.x, lo.y, hi.x, hi.y);
  }
}

// ------------------------------------------------------------ MXFP8
// OCP Microscaling (the "mxfp8" recipe of "Add _scaled_mm_v2 API"): per block
// of 32 elements along a row, e = floor(log2(amax)) - 8 clamped to
// [-127, 127] (an all-zero block: -127), scale byte e + 127 (E8M0), codes
// e4m3_satfinite(x * 2^-e).  Both the exponent (from the bits of amax) and
// the scaling (by a power of two) are exact.
// One warp per 2048-element span of a row: lane l holds the 32-byte
// (16-element) pieces l + 32 i (i < 4), so two consecutive lanes hold one
// block (amax over one shuffle) and each lane writes 16 codes at once.
// Scale bytes go straight into the GEMM's scale-factor tiles: tile (row / 128,
// block / 4), byte (row % 32) * 16 + ((row % 128) / 32) * 4 + block % 4.
// Warps past the last row (up to the next multiple of 128) and the blocks
// past the last one of a row (up to the next multiple of 4) write zero scale
// bytes, so the tiles hold no stale bytes.
constexpr int kMxItems = 4;                  // 16-element pieces per lane
constexpr int kMxSpan = 32 * kMxItems * 16;  // elements per warp

// Block maximum of |x| as bf16 magnitude bits: for finite values the order of
// |x| is the unsigned order of (bits & 0x7FFF), so two bf16 per word are
// compared at once; the exponent of the maximum is then bits >> 7.
__device__ __forceinline__ uint32_t absmax_bits16(const uint4& a, const uint4& b) {
  const uint32_t m0 = __vmaxu2(__vmaxu2(a.x & 0x7FFF7FFFu, a.y & 0x7FFF7FFFu),
                               __vmaxu2(a.z & 0x7FFF7FFFu, a.w & 0x7FFF7FFFu));
  const uint32_t m1 = __vmaxu2(__vmaxu2(b.x & 0x7FFF7FFFu, b.y & 0x7FFF7FFFu),
                               __vmaxu2(b.z & 0x7FFF7FFFu, b.w & 0x7FFF7FFFu));
  const uint32_t m = __vmaxu2(m0, m1);
  return max(m & 0xFFFFu, m >> 16);
}

__global__ void __launch_bounds__(256) quant_mx_kernel(
    const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
    uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
  const int lane = threadIdx.x & 31;
  const int64_t spans = (cols + kMxSpan - 1) / kMxSpan;
  const int64_t warp = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int64_t row = warp / spans;
  const int64_t p0 = (warp % spans) * (kMxSpan / 16);  // first 16-element piece of the span
  const int64_t P = cols >> 4;                          // pieces per row (even)
  const int64_t KB = cols >> 5;
  const int64_t KT = (KB + 3) >> 2;
  const int64_t rows_pad = (rows + 127) & ~int64_t(127);
  if (row >= rows_pad) return;
  const int64_t r7 = row & 127;
  // this row's scale bytes: tile row (row / 128), byte (row % 32) * 16 + (row % 128 / 32) * 4
  uint8_t* sfr = sf + (row >> 7) * KT * 512 + (r7 & 31) * 16 + (r7 >> 5) * 4;
  if (row >= rows) {
    // padding rows of the last row tile: zero scale bytes
    for (int64_t kb = (p0 >> 1) + lane; kb < KT * 4 && kb < (p0 >> 1) + kMxSpan / 32; kb += 32)
      sfr[(kb >> 2) * 512 + (kb & 3)] = 0;
    return;
  }
  // pieces of this span inside the row (even, as P is)
  const int np = static_cast<int>(P - p0 < kMxSpan / 16 ? P - p0 : kMxSpan / 16);
  const uint4* xs = reinterpret_cast<const uint4*>(x + row * ld) + 2 * p0;
  uint4* qs = reinterpret_cast<uint4*>(q + row * cols) + p0;
  uint4 v[kMxItems][2];
#pragma unroll
  for (int i = 0; i < kMxItems; ++i)
    if (lane + 32 * i < np) {
      v[i][0] = ld_stream(xs + 2 * (lane + 32 * i));
      v[i][1] = ld_stream(xs + 2 * (lane + 32 * i) + 1);
    }
#pragma unroll
  for (int i = 0; i < kMxItems; ++i) {
    const int pl = lane + 32 * i;
    // a block's two lanes agree on pl < np
    uint32_t m = pl < np ? absmax_bits16(v[i][0], v[i][1]) : 0u;
    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
    if (pl >= np) continue;
    // floor(log2(amax)) = biased exponent - 127 for normal amax; zero and
    // subnormal amax clamp to -127 like every exponent below it
    const int e = max(static_cast<int>(m >> 7) - 127 - 8, -127);   // <= 119 for finite amax
    const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);  // 2^-e
    const uint2 lo = cast8(v[i][0], inv);
    const uint2 hi = cast8(v[i][1], inv);
    qs[pl] = make_uint4(lo.x, lo.y, hi.x, hi.y);
    if ((lane & 1) == 0) {
      const int64_t kb = (p0 + pl) >> 1;
      sfr[(kb >> 2) * 512 + (kb & 3)] = static_cast<uint8_t>(e + 127);
      if (kb == KB - 1)
        for (int64_t k = KB; k < KT * 4; ++k) sfr[(k >> 2) * 512 + (k & 3)] = 0;
    }
  }
}

// ------------------------------------------------------------ 128x128
// One CTA (512 threads) per 128x128 tile: thread t covers the 16-byte chunk
// t%16 of rows t/16 + 32 i (i < 4), so each warp-wide load reads two whole
// 256-byte row segments (coalesced); the 4 chunks stay in registers.
// Ragged last row block: rows past the end take no part in the amax and are
// not written.
constexpr int k128Threads = 512;
// Batched (blockIdx.y = matrix e of a stack of equal matrices, e.g. the
// experts' weights): matrix e at x + e * rows * ld, its codes at
// q + e * rows * cols, its scales at scales + e * (cols / 128) * ceil(rows / 128).
__global__ void __launch_bounds__(k128Threads) quant_128x128_kernel(
    const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
    uint8_t* __restrict__ q, float* __restrict__ scales) {
  constexpr int kWarps = k128Threads / 32;
  constexpr int kRowStep = k128Threads / 16;       // rows covered per load round
  constexpr int kRounds = 128 / kRowStep;
  __shared__ float warp_amax[kWarps];
  const int64_t RB = (rows + 127) >> 7;
  {
    const int64_t e = blockIdx.y;
    x += e * rows * ld;
    q += e * rows * cols;
    scales += e * (cols >> 7) * RB;
  }
  const int64_t rb = blockIdx.x % RB;
  const int64_t kb = blockIdx.x / RB;
  const int t = threadIdx.x;
  const int64_t row0 = rb * 128 + (t >> 4);
  const int64_t col = kb * 128 + (t & 15) * 8;
  const uint16_t* xp = x + row0 * ld + col;
  uint4 v[kRounds];
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < kRounds; ++i)
    v[i] = row0 + kRowStep * i < rows
               ? ld_stream(reinterpret_cast<const uint4*>(xp + kRowStep * i * ld))
               : make_uint4(0, 0, 0, 0);  // zero padding does not change the max
#pragma unroll
  for (int i = 0; i < kRounds; ++i) m = amax8(v[i], m);
  m = warp_max(m);
  if ((t & 31) == 0) warp_amax[t >> 5] = m;
  __syncthreads();
  float tm = warp_amax[0];
#pragma unroll
  for (int i = 1; i < kWarps; ++i) tm = fmaxf(tm, warp_amax[i]);
  const ScalePair sp = scales_from_amax(tm);
  if (t == 0) scales[kb * RB + rb] = sp.s;
  uint8_t* qp = q + row0 * cols + col;
#pragma unroll
  for (int i = 0; i < kRounds; ++i)
    if (row0 + kRowStep * i < rows)
      *reinterpret_cast<uint2*>(qp + kRowStep * i * cols) = cast8(v[i], sp.inv);
}

// ------------------------------------------------------- transposed
// Quantizes x^T ((cols, rows)) for the training GEMMs ("improve fp8
// blockwise gemm perf": grad_input = grad_output @ weight and grad_weight =
// grad_output_t @ input both need an operand whose contraction runs along
// x's rows).  The result equals the 1x128 / 128x128 quantization of the
// transposed matrix: a group is 128 consecutive rows of x within one column
// (1x128) or a 128 x 128 tile (128x128).
// Persistent CTAs (512 threads) walk the 128-row x 128-column tiles of x
// with a two-buffer cp.async pipeline: the next tile's 16-byte chunks
// (coalesced rows of x) stream into shared memory while this tile is
// processed.  Thread t takes column t % 128 and rows 32 (t / 128) .. +31 of
// the tile: it reads them from shared memory (a warp reads 32 consecutive
// columns of one row), the four quarter-columns' amax meet in shared memory,
// and the thread stages its 32 codes in shared memory; the tile's 128 output
// rows (x's columns) then leave as whole 128-byte lines.
constexpr int kTrRows = 128;
constexpr int kTrCols = 128;
constexpr int kTrThreads = 512;
constexpr int kTrPitch = kTrCols + 8;  // bf16 elements per shared row (16-byte pad)
constexpr int kTrTileElems = kTrRows * kTrPitch;
constexpr int kTrOutPitch = kTrRows + 16;  // bytes per staged output row (conflict-free 16-byte stores)
constexpr size_t kTrSmemBytes =
    2 * kTrTileElems * sizeof(uint16_t) + static_cast<size_t>(kTrCols) * kTrOutPitch;
constexpr int kTrCtasPerSm = 2;

// Grouped (per-expert) variant, 1x128 only: rows are tokens split into
// groups by cumulative offsets; each group's tokens are laid out in the
// output padded to a multiple of 128 (group g starts at output column
// 128 * pb0[g], pb0 = exclusive prefix of ceil(size / 128)), so no 128-token
// block mixes two groups; the padding is zero.  ldq = the output row stride.
constexpr int kTrMaxGroups = 2048;

// Batched (`batch` equal matrices, not grouped): matrix e at x + e * rows *
// ld, its transposed codes at q + e * cols * ldq, its scales after the e
// earlier matrices' scales; tiles are numbered matrix-major.
template <bool k128x128, bool kGroupedT>
__global__ void __launch_bounds__(kTrThreads) quant_transposed_kernel(
    const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
    uint8_t* __restrict__ q, float* __restrict__ scales, const int32_t* __restrict__ offs,
    int32_t E, int64_t ldq, int64_t n_kb, uint32_t* status, int32_t batch) {
  extern __shared__ __align__(16) uint16_t tiles_smem[];
  __shared__ float part[4][kTrCols];
  __shared__ float warp_amax[kTrThreads / 32];
  const int64_t n_cb = (cols + kTrCols - 1) / kTrCols;
  const int64_t per_matrix = n_kb * n_cb;
  const int64_t n_tiles = per_matrix * batch;
  const int64_t scales_per_matrix = k128x128 ? n_kb * n_cb : n_kb * cols;
  const int t = threadIdx.x;
  int32_t* pb0 = nullptr;  // grouped: pb0[g] = padded blocks before group g; pb0[E] = total
  if constexpr (kGroupedT) {
    __shared__ int32_t table[kTrMaxGroups + 1];
    __shared__ int32_t bad;
    pb0 = table;
    if (t < 32) {
      // lane l: groups [l * per, (l + 1) * per); block counts, then a scan
      const int32_t per = (E + 31) / 32;
      const int32_t g0 = t * per, g1 = min(E, g0 + per);
      int32_t sum = 0, bad_l = 0;
      for (int32_t g = g0; g < g1; ++g) {
        const int32_t prev = g ? offs[g - 1] : 0;
        const int32_t e = offs[g];
        if (e < prev || prev < 0) bad_l = 1;
        sum += (max(e - prev, 0) + kTrRows - 1) / kTrRows;
      }
      int32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (t >= o) incl += v;
      }
      int32_t run = incl - sum;
      for (int32_t g = g0; g < g1; ++g) {
        table[g] = run;
        const int32_t prev = g ? offs[g - 1] : 0;
        run += (max(offs[g] - prev, 0) + kTrRows - 1) / kTrRows;
      }
      if (t == 31) table[E] = incl;
      bad_l = __any_sync(0xFFFFFFFFu, bad_l);
      if (t == 0) bad = bad_l || offs[E - 1] != rows;
    }
    __syncthreads();
    if (bad || pb0[E] > n_kb) {
      if (t == 0 && blockIdx.x == 0) record_status(status, FP8_DEV_VALUE, SITE_OFFS);
      return;
    }
  }
  // padded block kb -> first input row and the rows it holds (grouped: the
  // block's group by binary search over pb0)
  auto block_rows = [&](int64_t kb, int64_t& row0, int32_t& nrows) {
    if constexpr (kGroupedT) {
      int32_t lo = 0, hi = E - 1;
      while (lo < hi) {  // last g with pb0[g] <= kb
        const int32_t mid = (lo + hi + 1) >> 1;
        if (pb0[mid] <= kb) lo = mid;
        else hi = mid - 1;
      }
      const int64_t start = lo ? offs[lo - 1] : 0;
      row0 = start + (kb - pb0[lo]) * kTrRows;
      const int64_t left = static_cast<int64_t>(offs[lo]) - row0;
      nrows = static_cast<int32_t>(left < kTrRows ? left : kTrRows);
    } else {
      row0 = kb * kTrRows;
      nrows = kTrRows;
    }
  };
  const int64_t n_kb_used = kGroupedT ? pb0[E] : n_kb;
  // copy tile `tile` into buffer `buf`: chunk t % 16 (8 columns) of rows
  // t / 16 + 32 i; columns past the end (and grouped: rows past the group)
  // are zero-filled (no effect on the max, zero codes)
  auto issue = [&](int64_t tile, int buf) {
    const int64_t e = tile / per_matrix;
    tile -= e * per_matrix;
    const int64_t kb = tile % n_kb, cb = tile / n_kb;
    if (kb >= n_kb_used) {
      cp_async_commit();
      return;
    }
    int64_t row0;
    int32_t nrows;
    block_rows(kb, row0, nrows);
    const int ch = t & 15;
    const int64_t col = cb * kTrCols + ch * 8;
    uint16_t* dst = tiles_smem + buf * kTrTileElems;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = (t >> 4) + 32 * i;
      const bool in = col < cols && r < nrows;
      cp_async_16(dst + r * kTrPitch + ch * 8, in ? x + e * rows * ld + (row0 + r) * ld + col : x,
                  in ? 16u : 0u);
    }
    cp_async_commit();
  };
  int64_t tile = blockIdx.x;
  if (tile < n_tiles) issue(tile, 0);
  const int c = t & (kTrCols - 1);   // column within the tile = output row
  const int qr = t >> 7;             // rows 32 qr .. 32 qr + 31
  for (int it = 0; tile < n_tiles; tile += gridDim.x, ++it) {
    const int buf = it & 1;
    if (tile + gridDim.x < n_tiles) issue(tile + gridDim.x, buf ^ 1);
    else cp_async_commit();          // empty group: the wait below counts groups
    cp_async_wait<1>();              // this tile's copies have landed
    __syncthreads();
    const uint16_t* tl = tiles_smem + buf * kTrTileElems;
    const int64_t e = tile / per_matrix;
    const int64_t kb = (tile - e * per_matrix) % n_kb, cb = (tile - e * per_matrix) / n_kb;
    float* const sc = scales + e * scales_per_matrix;
    uint8_t* const qm = q + e * cols * ldq;
    if (kb >= n_kb_used) continue;   // grouped: past the last group's blocks (uniform)
    uint32_t w[16];                  // the 32 values, packed bf16 pairs
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t lo = tl[(32 * qr + 2 * j) * kTrPitch + c];
      const uint32_t hi = tl[(32 * qr + 2 * j + 1) * kTrPitch + c];
      w[j] = lo | (hi << 16);
      m = fmaxf(m, fmaxf(fabsf(bf16_lo(w[j])), fabsf(bf16_hi(w[j]))));
    }
    float gm;
    if constexpr (k128x128) {
      m = warp_max(m);
      if ((t & 31) == 0) warp_amax[t >> 5] = m;
      __syncthreads();
      gm = warp_amax[0];
#pragma unroll
      for (int i = 1; i < kTrThreads / 32; ++i) gm = fmaxf(gm, warp_amax[i]);
    } else {
      part[qr][c] = m;
      __syncthreads();
      gm = fmaxf(fmaxf(part[0][c], part[1][c]), fmaxf(part[2][c], part[3][c]));
    }
    const ScalePair sp = scales_from_amax(gm);
    const int64_t col = cb * kTrCols + c;
    if constexpr (k128x128) {
      if (t == 0) sc[kb * n_cb + cb] = sp.s;
    } else {
      if (qr == 0 && col < cols) sc[kb * cols + col] = sp.s;
    }
    uint8_t* stage = reinterpret_cast<uint8_t*>(tiles_smem + 2 * kTrTileElems);
    {
      uint4 out[2];
      uint32_t* o = reinterpret_cast<uint32_t*>(out);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        o[j] = cast2(w[2 * j], sp.inv) | (cast2(w[2 * j + 1], sp.inv) << 16);
      uint4* sd = reinterpret_cast<uint4*>(stage + c * kTrOutPitch + 32 * qr);
      sd[0] = out[0];
      sd[1] = out[1];
    }
    __syncthreads();
    {
      // thread t: 32 bytes (chunk t % 4) of output row t / 4 of the tile
      const int orow = t >> 2, chunk = t & 3;
      const int64_t ocol = cb * kTrCols + orow;
      if (ocol < cols) {
        const uint4* ss = reinterpret_cast<const uint4*>(stage + orow * kTrOutPitch + 32 * chunk);
        uint4* dst = reinterpret_cast<uint4*>(qm + ocol * ldq + kb * kTrRows + 32 * chunk);
        dst[0] = ss[0];
        dst[1] = ss[1];
      }
    }
    // every thread is done with this buffer, the staging rows and part /
    // warp_amax before the next iteration refills them
    __syncthreads();
  }
  cp_async_wait_all();
}

// ------------------------------------------------------------- tensor
// One amax for the whole matrix.  Cooperative launch (all CTAs resident):
// phase 1 reduces each CTA's amax and folds it into ws[0] with an atomic
// max on the fp32 bit pattern (non-negative floats order like unsigned
// integers); a bounded grid barrier on ws[1]; phase 2 casts.  When every
// thread holds at most one vector (small tensors) phase 2 reuses the
// registers, otherwise it re-reads x (from L2 when it fits there).
// ws[0..1] must be zero on entry (the launcher clears them).
__global__ void __launch_bounds__(256) quant_tensor_kernel(
    const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
    uint8_t* __restrict__ q, float* __restrict__ scale, uint32_t* ws,
    uint32_t* status) {
  __shared__ float warp_amax[8];
  __shared__ uint32_t ok_flag;
  const int64_t nvec = cols >> 3;
  const bool single = (rows <= gridDim.x) && (nvec <= blockDim.x);
  uint4 keep = make_uint4(0, 0, 0, 0);
  float m = 0.0f;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + r * ld);
    for (int64_t c = threadIdx.x; c < nvec; c += blockDim.x) {
      const uint4 v = __ldg(xr + c);
      keep = v;
      m = amax8(v, m);
    }
  }
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) warp_amax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float bm = warp_amax[0];
    for (int i = 1; i < (int)(blockDim.x >> 5); ++i) bm = fmaxf(bm, warp_amax[i]);
    atomicMax(ws, __float_as_uint(bm));
    __threadfence();
    atomicAdd(ws + 1, 1u);
    // bounded grid barrier
    uint32_t ok = 1;
    const uint64_t t0 = globaltimer_ns();
    while (*reinterpret_cast<volatile uint32_t*>(ws + 1) < gridDim.x) {
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        record_status(status, FP8_DEV_TIMEOUT, SITE_GRID_BARRIER);
        ok = 0;
        break;
      }
    }
    __threadfence();
    ok_flag = ok;
  }
  __syncthreads();
  if (!ok_flag) return;
  const float amax = __uint_as_float(*reinterpret_cast<volatile uint32_t*>(ws));
  const ScalePair sp = scales_from_amax(amax);
  if (blockIdx.x == 0 && threadIdx.x == 0) scale[0] = sp.s;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + r * ld);
    uint2* qr = reinterpret_cast<uint2*>(q + r * cols);
    for (int64_t c = threadIdx.x; c < nvec; c += blockDim.x)
      qr[c] = cast8(single ? keep : __ldg(xr + c), sp.inv);
  }
}

// Resident quant_tensor_kernel CTAs per SM (the cooperative grid's bound),
// queried once per device.
int g_tensor_blocks_per_sm[kMaxDevices];
std::atomic<bool> g_tensor_occupancy_done[kMaxDevices];
std::mutex g_tensor_occupancy_mu;

// Sharded tensorwise quantization, step 1: max|x| of this shard folded into
// amax[0] (fp32 bits, atomic max; amax[0] must be zero on entry).
__global__ void __launch_bounds__(256) tensor_amax_kernel(
    const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
    uint32_t* amax) {
  __shared__ float warp_amax[8];
  const int64_t nvec = cols >> 3;
  float m = 0.0f;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + r * ld);
    for (int64_t c = threadIdx.x; c < nvec; c += blockDim.x) m = amax8(__ldg(xr + c), m);
  }
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) warp_amax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float bm = warp_amax[0];
    for (int i = 1; i < (int)(blockDim.x >> 5); ++i) bm = fmaxf(bm, warp_amax[i]);
    atomicMax(amax, __float_as_uint(bm));
  }
}

// Step 2 (after the caller's all-reduce(MAX) of amax over the shards): the
// tensorwise scale of the whole tensor and the cast of this shard.
__global__ void __launch_bounds__(256) tensor_cast_kernel(
    const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
    const float* amax, uint8_t* __restrict__ q, float* __restrict__ scale) {
  const ScalePair sp = scales_from_amax(*amax);
  if (blockIdx.x == 0 && threadIdx.x == 0) scale[0] = sp.s;
  const int64_t nvec = cols >> 3;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + r * ld);
    uint2* qr = reinterpret_cast<uint2*>(q + r * cols);
    for (int64_t c = threadIdx.x; c < nvec; c += blockDim.x) qr[c] = cast8(__ldg(xr + c), sp.inv);
  }
}

// Scratch for fp8_quantize_noalloc: a fixed array in device memory that the
// library owns.  Every GPU that loads the library holds one copy until the
// process exits.  All calls share it; a call leaves its contents behind, so
// the launcher clears what must start at zero before each use, and two
// calls that run at the same time on the GPU (different streams) race on it.
constexpr size_t kNoAllocScratchBytes = 256;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch for each device, taken once with that
// device current (in host code the array's name is only a stand-in).
void* g_noalloc_ptr[64] = {nullptr};
std::mutex g_noalloc_mu;

}  // namespace

size_t noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

cudaError_t noalloc_scratch_ptr(int device, void** out) {
  if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_ptr[device] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[device] = p;
  }
  *out = g_noalloc_ptr[device];
  return cudaSuccess;
}

size_t mx_scale_tile_bytes(int64_t rows, int64_t cols) {
  const int64_t KT = (cols / 32 + 3) / 4;
  return static_cast<size_t>(((rows + 127) / 128) * KT * 512);
}

cudaError_t launch_quantize_mx(const void* xv, int64_t rows, int64_t cols, int64_t ld,
                               void* qv, void* sfv, const LaunchCtx& ctx) {
  if (rows == 0 || cols == 0) return cudaSuccess;
  const int64_t spans = (cols + kMxSpan - 1) / kMxSpan;
  const int64_t warps = ((rows + 127) / 128) * 128 * spans;
  const unsigned grid = static_cast<unsigned>((warps + 7) / 8);
  quant_mx_kernel<<<grid, 256, 0, ctx.stream>>>(static_cast<const uint16_t*>(xv), rows, cols,
                                                ld, static_cast<uint8_t*>(qv),
                                                static_cast<uint8_t*>(sfv));
  return cudaGetLastError();
}

// The transposed kernels' dynamic shared-memory opt-in, once per device.
static cudaError_t configure_transposed(const LaunchCtx& ctx) {
  static std::atomic<bool> done[kMaxDevices];
  static std::mutex mu;
  return once_per_device(done, mu, ctx.device, [] {
    const void* fns[] = {(const void*)quant_transposed_kernel<true, false>,
                         (const void*)quant_transposed_kernel<false, false>,
                         (const void*)quant_transposed_kernel<false, true>};
    for (const void* f : fns) {
      cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(kTrSmemBytes));
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  });
}

cudaError_t launch_quantize_transposed(const void* xv, int64_t rows, int64_t cols,
                                       int64_t ld, int recipe, void* qv, float* scales,
                                       const LaunchCtx& ctx) {
  if (rows == 0 || cols == 0) return cudaSuccess;
  const uint16_t* x = static_cast<const uint16_t*>(xv);
  uint8_t* q = static_cast<uint8_t*>(qv);
  cudaError_t e = configure_transposed(ctx);
  if (e != cudaSuccess) return e;
  const int64_t n_kb = rows / kTrRows;
  const int64_t tiles = n_kb * ((cols + kTrCols - 1) / kTrCols);
  const int64_t max_grid = static_cast<int64_t>(ctx.num_sms) * kTrCtasPerSm;
  const unsigned grid = static_cast<unsigned>(tiles < max_grid ? tiles : max_grid);
  if (recipe == 3)
    quant_transposed_kernel<true, false><<<grid, kTrThreads, kTrSmemBytes, ctx.stream>>>(
        x, rows, cols, ld, q, scales, nullptr, 0, rows, n_kb, ctx.status, 1);
  else
    quant_transposed_kernel<false, false><<<grid, kTrThreads, kTrSmemBytes, ctx.stream>>>(
        x, rows, cols, ld, q, scales, nullptr, 0, rows, n_kb, ctx.status, 1);
  return cudaGetLastError();
}

cudaError_t launch_quantize_transposed_batched(const void* xv, int32_t batch, int64_t rows,
                                               int64_t cols, int64_t ld, int recipe, void* qv,
                                               float* scales, const LaunchCtx& ctx) {
  if (batch == 0 || rows == 0 || cols == 0) return cudaSuccess;
  cudaError_t e = configure_transposed(ctx);
  if (e != cudaSuccess) return e;
  const int64_t n_kb = rows / kTrRows;
  const int64_t tiles = n_kb * ((cols + kTrCols - 1) / kTrCols) * batch;
  const int64_t max_grid = static_cast<int64_t>(ctx.num_sms) * kTrCtasPerSm;
  const unsigned grid = static_cast<unsigned>(tiles < max_grid ? tiles : max_grid);
  const uint16_t* x = static_cast<const uint16_t*>(xv);
  uint8_t* q = static_cast<uint8_t*>(qv);
  if (recipe == 3)
    quant_transposed_kernel<true, false><<<grid, kTrThreads, kTrSmemBytes, ctx.stream>>>(
        x, rows, cols, ld, q, scales, nullptr, 0, rows, n_kb, ctx.status, batch);
  else
    quant_transposed_kernel<false, false><<<grid, kTrThreads, kTrSmemBytes, ctx.stream>>>(
        x, rows, cols, ld, q, scales, nullptr, 0, rows, n_kb, ctx.status, batch);
  return cudaGetLastError();
}

cudaError_t launch_quantize_128x128_batched(const void* xv, int32_t batch, int64_t rows,
                                            int64_t cols, int64_t ld, void* qv, float* scales,
                                            const LaunchCtx& ctx) {
  if (batch == 0 || rows == 0 || cols == 0) return cudaSuccess;
  const int64_t tiles = ((rows + 127) / 128) * (cols / 128);
  quant_128x128_kernel<<<dim3(static_cast<unsigned>(tiles), static_cast<unsigned>(batch)),
                         k128Threads, 0, ctx.stream>>>(static_cast<const uint16_t*>(xv), rows,
                                                       cols, ld, static_cast<uint8_t*>(qv),
                                                       scales);
  return cudaGetLastError();
}

int64_t grouped_padded_tokens(int64_t tokens, int32_t E) {
  return ((tokens + kTrRows - 1) / kTrRows + E) * kTrRows;
}

cudaError_t launch_quantize_transposed_grouped(const void* xv, int64_t rows, int64_t cols,
                                               int64_t ld, const int32_t* offs, int32_t E,
                                               void* qv, float* scales, const LaunchCtx& ctx) {
  if (cols == 0) return cudaSuccess;
  cudaError_t e = configure_transposed(ctx);
  if (e != cudaSuccess) return e;
  const int64_t P = grouped_padded_tokens(rows, E);
  const int64_t n_kb = P / kTrRows;
  const int64_t tiles = n_kb * ((cols + kTrCols - 1) / kTrCols);
  const int64_t max_grid = static_cast<int64_t>(ctx.num_sms) * kTrCtasPerSm;
  const unsigned grid = static_cast<unsigned>(tiles < max_grid ? tiles : max_grid);
  quant_transposed_kernel<false, true><<<grid, kTrThreads, kTrSmemBytes, ctx.stream>>>(
      static_cast<const uint16_t*>(xv), rows, cols, ld, static_cast<uint8_t*>(qv), scales,
      offs, E, P, n_kb, ctx.status, 1);
  return cudaGetLastError();
}

cudaError_t launch_quantize(const void* xv, int64_t rows, int64_t cols,
                            int64_t ld, int recipe, void* qv, float* scales,
                            void* workspace, const LaunchCtx& ctx) {
  const uint16_t* x = static_cast<const uint16_t*>(xv);
  uint8_t* q = static_cast<uint8_t*>(qv);
  cudaStream_t st = ctx.stream;
  if (recipe == 1) {  // rowwise
    if (rows == 0) return cudaSuccess;
    const unsigned grid = static_cast<unsigned>((rows + 7) / 8);
    const int64_t nvec = cols / 8;
    if (nvec >= 64 && nvec <= 2048) {
      // one CTA per row, 16 elements per thread
      const int64_t threads = ((nvec + 1) / 2 + 31) / 32 * 32;
      quant_row_cta_kernel<<<static_cast<unsigned>(rows), static_cast<unsigned>(threads), 0,
                             st>>>(x, rows, cols, ld, q, scales);
    } else if (nvec <= 32)
      quant_row_kernel<1><<<grid, 256, 0, st>>>(x, rows, cols, ld, q, scales);
    else if (nvec <= 64)
      quant_row_kernel<2><<<grid, 256, 0, st>>>(x, rows, cols, ld, q, scales);
    else if (nvec <= 128)
      quant_row_kernel<4><<<grid, 256, 0, st>>>(x, rows, cols, ld, q, scales);
    else if (nvec <= 256)
      quant_row_kernel<8><<<grid, 256, 0, st>>>(x, rows, cols, ld, q, scales);
    else if (nvec <= 512)
      quant_row_kernel<16><<<grid, 256, 0, st>>>(x, rows, cols, ld, q, scales);
    else
      quant_row_long_kernel<<<grid, 256, 0, st>>>(x, rows, cols, ld, q, scales);
    return cudaGetLastError();
  }
  if (recipe == 2) {  // 1x128
    if (rows == 0 || cols == 0) return cudaSuccess;
    const int64_t KB = cols / 128;
    const int64_t kb_groups = (KB + k1x128Tasks - 1) / k1x128Tasks;
    const int64_t warps = ((rows + 3) / 4) * kb_groups;
    const unsigned grid = static_cast<unsigned>((warps + 7) / 8);
    quant_1x128_kernel<<<grid, 256, 0, st>>>(x, rows, cols, ld, q, scales);
    return cudaGetLastError();
  }
  if (recipe == 3) {  // 128x128
    if (rows == 0 || cols == 0) return cudaSuccess;
    const int64_t tiles = ((rows + 127) / 128) * (cols / 128);
    quant_128x128_kernel<<<static_cast<unsigned>(tiles), k128Threads, 0, st>>>(
        x, rows, cols, ld, q, scales);
    return cudaGetLastError();
  }
  // tensorwise
  uint32_t* ws = static_cast<uint32_t*>(workspace);
  cudaError_t e = cudaMemsetAsync(ws, 0, 2 * sizeof(uint32_t), st);
  if (e != cudaSuccess) return e;
  e = once_per_device(g_tensor_occupancy_done, g_tensor_occupancy_mu, ctx.device, [&] {
    int n = 0;
    const cudaError_t r =
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, quant_tensor_kernel, 256, 0);
    g_tensor_blocks_per_sm[ctx.device] = n;
    return r;
  });
  if (e != cudaSuccess) return e;
  const int per_sm = g_tensor_blocks_per_sm[ctx.device];
  int64_t max_grid = static_cast<int64_t>(ctx.num_sms) * (per_sm > 0 ? per_sm : 1);
  int64_t grid = rows < max_grid ? rows : max_grid;
  if (grid < 1) grid = 1;
  unsigned g = static_cast<unsigned>(grid);
  uint32_t* status = ctx.status;
  void* args[] = {(void*)&x, (void*)&rows, (void*)&cols, (void*)&ld,
                  (void*)&q, (void*)&scales, (void*)&ws, (void*)&status};
  return cudaLaunchCooperativeKernel((const void*)quant_tensor_kernel, dim3(g),
                                     dim3(256), args, 0, st);
}

static unsigned tensor_grid(int64_t rows, const LaunchCtx& ctx) {
  const int64_t g = rows < 8 * static_cast<int64_t>(ctx.num_sms) ? rows : 8 * ctx.num_sms;
  return static_cast<unsigned>(g < 1 ? 1 : g);
}

cudaError_t launch_tensor_amax(const void* x, int64_t rows, int64_t cols, int64_t ld,
                               float* amax, const LaunchCtx& ctx) {
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float), ctx.stream);
  if (e != cudaSuccess || rows == 0 || cols == 0) return e;
  tensor_amax_kernel<<<tensor_grid(rows, ctx), 256, 0, ctx.stream>>>(
      static_cast<const uint16_t*>(x), rows, cols, ld, reinterpret_cast<uint32_t*>(amax));
  return cudaGetLastError();
}

cudaError_t launch_tensor_cast(const void* x, int64_t rows, int64_t cols, int64_t ld,
                               const float* amax, void* q, float* scale,
                               const LaunchCtx& ctx) {
  tensor_cast_kernel<<<tensor_grid(rows, ctx), 256, 0, ctx.stream>>>(
      static_cast<const uint16_t*>(x), rows, cols, ld, amax, static_cast<uint8_t*>(q), scale);
  return cudaGetLastError();
}

}  // namespace fp8sm
