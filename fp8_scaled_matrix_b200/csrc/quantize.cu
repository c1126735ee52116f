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

// A packed bf16 pair -> two e4m3 codes: one packed multiply (each lane an
// IEEE fp32 multiply, bit-identical to two scalar ones), one pair convert.
__device__ __forceinline__ uint32_t cast2(uint32_t w, float inv) {
  const float2 y = mul2(make_float2(bf16_lo(w), bf16_hi(w)), make_float2(inv, inv));
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(y, __NV_SATFINITE, __NV_E4M3));
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
// One CTA (256 threads) per 128 x 128 tile, blockIdx.y = the matrix of a
// stack of equal matrices (the experts' weights).  The tile arrives in
// shared memory by one TMA load (a 3-D map (cols, rows, matrix): a ragged
// last row block reads zeros past the matrix's last row, which leave the
// amax unchanged) and stays there: a first pass reads it for the amax, a
// second pass reads it again for the cast, so a thread holds one 16-byte
// chunk at a time.  Few registers and 32 KB of shared memory per CTA let up
// to seven tiles per SM be in flight, and the short-lived CTAs interleave
// with those of a concurrent quantization of the other GEMM operand.
// Thread t takes the chunks t + 256 i (row (t + 256 i) / 16, conflict-free);
// codes leave as 8-byte stores (16 threads write one row's 128 bytes); rows
// past the end are not written.  Tile (rb, kb) of matrix e has its scale at
// scales[e * (cols / 128) * RB + kb * RB + rb].
constexpr int k128Threads = 256;
constexpr uint32_t kQTileBytes = 128 * 128 * 2;
constexpr size_t kQSmemBytes = kQTileBytes + 128;  // + 128-byte alignment slack

__global__ void __launch_bounds__(k128Threads) quant_128x128_kernel(
    const __grid_constant__ CUtensorMap tm_x, int64_t rows, int64_t cols,
    uint8_t* __restrict__ q, float* __restrict__ scales, uint32_t* status) {
  extern __shared__ uint8_t qsmem_raw[];
  __shared__ uint64_t full;
  __shared__ float warp_amax[k128Threads / 32];
  __shared__ uint32_t abort_flag;
  const uint32_t raw = smem_u32(qsmem_raw);
  const uint4* tile = reinterpret_cast<const uint4*>(qsmem_raw + (((raw + 127u) & ~127u) - raw));
  const int t = threadIdx.x;
  const int64_t RB = (rows + 127) >> 7;
  const int64_t e = blockIdx.y;
  const int64_t rb = blockIdx.x % RB, kb = blockIdx.x / RB;
  if (t == 0) {
    mbar_init(&full, 1);
    abort_flag = 0u;
    fence_barrier_init();
    mbar_arrive_expect_tx(&full, kQTileBytes);
    tma_load_3d(const_cast<uint4*>(tile), &tm_x, &full, static_cast<int32_t>(kb * 128),
                static_cast<int32_t>(rb * 128), static_cast<int32_t>(e));
  }
  __syncthreads();
  const bool got = mbar_wait(&full, 0, &abort_flag, status, SITE_QUANT_TMA, kWaitLimitNs);
  if (!__syncthreads_and(got)) {
    // let the load land before the CTA exits
    if (t == 0) {
      uint32_t dummy = 0;
      mbar_wait(&full, 0, &dummy, nullptr, SITE_TEARDOWN, 10000000ull);
    }
    return;
  }
  float m = 0.0f;
#pragma unroll
  for (int k = 0; k < 8; ++k) m = amax8(tile[t + 256 * k], m);
  m = warp_max(m);
  if ((t & 31) == 0) warp_amax[t >> 5] = m;
  __syncthreads();
  float tm = warp_amax[0];
#pragma unroll
  for (int w = 1; w < k128Threads / 32; ++w) tm = fmaxf(tm, warp_amax[w]);
  const ScalePair sp = scales_from_amax(tm);
  if (t == 0) scales[e * RB * (cols >> 7) + kb * RB + rb] = sp.s;
  const int64_t nrows = rows - rb * 128 < 128 ? rows - rb * 128 : 128;
  uint8_t* qt = q + (e * rows + rb * 128) * cols + kb * 128 + (t & 15) * 8;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int row = (t >> 4) + 16 * k;
    const uint2 c = cast8(tile[t + 256 * k], sp.inv);
    if (row < nrows) *reinterpret_cast<uint2*>(qt + static_cast<int64_t>(row) * cols) = c;
  }
}

// ------------------------------------------------------- transposed
// Quantizes x^T ((cols, rows)) for the training GEMMs ("improve fp8
// blockwise gemm perf": grad_input = grad_output @ weight and grad_weight =
// grad_output_t @ input both need an operand whose contraction runs along
// x's rows).  The result equals the 1x128 / 128x128 quantization of the
// transposed matrix: a group is 128 consecutive rows of x within one column
// (1x128) or a 128 x 128 tile (128x128).
// Persistent CTAs (256 threads, two per SM) walk the 128-row x 128-column
// tiles of x; each tile arrives in shared memory by TMA (3-D map (cols,
// rows, matrix); columns past the end read as zero) through a two-buffer
// ring per CTA.  Thread t reads the 16-byte chunk t % 16 (8 columns) of the
// 8 consecutive rows 8 (t / 16) .. + 7 (whole 256-byte rows per warp access),
// so after the cast it holds 8 consecutive codes of each of its 8 columns:
// one 8-byte word per output row.  The words go to a 16 KB staging area laid
// out as the tile's 128 output rows of 128 bytes, with the 8-byte slot of a
// word XOR-swizzled by its column group (conflict-free stores), and leave as
// 16-byte stores, eight threads per 128-byte output row.  1x128: column
// maxima over 16 rows per warp (one shuffle), then over the 8 warps through
// shared memory, where one thread per column forms its scale.
constexpr int kTrRows = 128;
constexpr int kTrCols = 128;
constexpr int kTrThreads = 256;
constexpr int kTrStages = 2;
constexpr uint32_t kTrTileBytes = kTrRows * kTrCols * 2;
constexpr uint32_t kTrOutBytes = kTrCols * kTrRows;
constexpr size_t kTrSmemBytes = kTrStages * kTrTileBytes + kTrOutBytes + 1024;  // + alignment
constexpr int kTrCtasPerSm = 2;

// Grouped (per-expert) variant, 1x128 only: rows are tokens split into
// groups by cumulative offsets; each group's tokens are laid out in the
// output padded to a multiple of 128 (group g starts at output column
// 128 * pb0[g], pb0 = exclusive prefix of ceil(size / 128)), so no 128-token
// block mixes two groups; the padding is zero (rows of the next group that
// the block's tile load brings in are taken as zero).  ldq = the output row
// stride.
constexpr int kTrMaxGroups = 2048;

// Batched (`batch` equal matrices, not grouped): matrix e's transposed codes
// at q + e * cols * ldq, its scales after the e earlier matrices' scales;
// tiles are numbered matrix-major.
template <bool k128x128, bool kGroupedT>
__global__ void __launch_bounds__(kTrThreads) quant_transposed_kernel(
    const __grid_constant__ CUtensorMap tm_x, int64_t rows, int64_t cols,
    uint8_t* __restrict__ q, float* __restrict__ scales, const int32_t* __restrict__ offs,
    int32_t E, int64_t ldq, int64_t n_kb, uint32_t* status, int32_t batch) {
  extern __shared__ uint8_t tr_smem_raw[];
  __shared__ uint64_t full[kTrStages];
  __shared__ __align__(16) float part[kTrThreads / 32][kTrCols];
  __shared__ __align__(16) float inv_s[kTrCols];  // 1x128: the tile's column inverses
  __shared__ float warp_amax[kTrThreads / 32];
  __shared__ uint32_t abort_flag;
  // each buffer's first input row and row count, set by the thread that
  // issues its load (before its arrive, so the buffer's waiters see them)
  __shared__ int64_t buf_row0[kTrStages];
  __shared__ int32_t buf_nrows[kTrStages];
  const uint32_t raw = smem_u32(tr_smem_raw);
  uint8_t* const tiles = tr_smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* const stage_out = tiles + kTrStages * kTrTileBytes;
  const int64_t n_cb = (cols + kTrCols - 1) / kTrCols;
  const int64_t per_matrix = n_kb * n_cb;
  const int64_t n_tiles = per_matrix * batch;
  const int64_t scales_per_matrix = k128x128 ? n_kb * n_cb : n_kb * cols;
  const int t = threadIdx.x;
  const int w = t >> 5;
  int32_t* pb0 = nullptr;  // grouped: pb0[g] = padded blocks before group g; pb0[E] = total
  int32_t* gend = nullptr;  // grouped: gend[g] = offs[g], kept on chip for the tile loads
  if constexpr (kGroupedT) {
    __shared__ int32_t table[kTrMaxGroups + 1];
    __shared__ int32_t ends[kTrMaxGroups];
    __shared__ int32_t bad;
    pb0 = table;
    gend = ends;
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
        ends[g] = offs[g];
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
      const int64_t start = lo ? gend[lo - 1] : 0;
      row0 = start + (kb - pb0[lo]) * kTrRows;
      const int64_t left = static_cast<int64_t>(gend[lo]) - row0;
      nrows = static_cast<int32_t>(left < kTrRows ? left : kTrRows);
    } else {
      row0 = kb * kTrRows;
      nrows = kTrRows;
    }
  };
  const int64_t n_kb_used = kGroupedT ? pb0[E] : n_kb;
  // the load of tile `tile` into buffer s (grouped: blocks past the last
  // group's complete the buffer's phase without a copy)
  auto issue = [&](int64_t tile, int s) {
    const int64_t e = tile / per_matrix;
    const int64_t r = tile - e * per_matrix;
    // grouped: column blocks fastest (measured 2 % faster there; the dense
    // forms keep row blocks fastest, 4 % faster on 16640 x 5120)
    const int64_t kb = kGroupedT ? r / n_cb : r % n_kb;
    const int64_t cb = kGroupedT ? r % n_cb : r / n_kb;
    if (kb >= n_kb_used) {
      mbar_arrive(&full[s]);
      return;
    }
    int64_t row0;
    int32_t nrows;
    block_rows(kb, row0, nrows);
    buf_row0[s] = row0;
    buf_nrows[s] = nrows;
    mbar_arrive_expect_tx(&full[s], kTrTileBytes);
    tma_load_3d(tiles + s * kTrTileBytes, &tm_x, &full[s], static_cast<int32_t>(cb * kTrCols),
                static_cast<int32_t>(row0), static_cast<int32_t>(e));
  };
  if (t == 0) {
    for (int s = 0; s < kTrStages; ++s) mbar_init(&full[s], 1);
    abort_flag = 0u;
    fence_barrier_init();
    prefetch_tmap(&tm_x);
  }
  __syncthreads();
  if (t == 0) {
    int64_t tile = blockIdx.x;
    for (int s = 0; s < kTrStages && tile < n_tiles; ++s, tile += gridDim.x) issue(tile, s);
  }
  int64_t issued_to = blockIdx.x + static_cast<int64_t>(kTrStages) * gridDim.x;
  const int ch = t & 15;         // 16-byte chunk: columns 8 ch .. 8 ch + 7 of the tile
  const int rg = t >> 4;         // rows 8 rg .. 8 rg + 7 of the tile
  int i = 0;
  for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++i) {
    const int s = i % kTrStages;
    const uint32_t parity = static_cast<uint32_t>((i / kTrStages) & 1);
    const bool got = mbar_wait(&full[s], parity, &abort_flag, status, SITE_QUANT_TMA,
                               kWaitLimitNs);
    if (!__syncthreads_and(got)) break;
    const int64_t e = tile / per_matrix;
    const int64_t rr = tile - e * per_matrix;
    const int64_t kb = kGroupedT ? rr / n_cb : rr % n_kb;
    const int64_t cb = kGroupedT ? rr % n_cb : rr / n_kb;
    if (kb >= n_kb_used) {  // grouped: past the last group's blocks (uniform)
      if (t == 0 && issued_to < n_tiles) {
        issue(issued_to, s);
        issued_to += gridDim.x;
      }
      continue;
    }
    const int32_t nrows = buf_nrows[s];
    // this thread's 8 rows x 8 columns (rows past the block's end: zero)
    const uint8_t* tl = tiles + s * kTrTileBytes;
    uint4 v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int r = 8 * rg + k;
      v[k] = r < nrows ? *reinterpret_cast<const uint4*>(tl + r * 256 + ch * 16)
                       : make_uint4(0, 0, 0, 0);
    }
    float cm[8];  // column maxima over this thread's 8 rows
#pragma unroll
    for (int j = 0; j < 8; ++j) cm[j] = 0.0f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t wd[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        cm[2 * j] = fmaxf(cm[2 * j], fabsf(bf16_lo(wd[j])));
        cm[2 * j + 1] = fmaxf(cm[2 * j + 1], fabsf(bf16_hi(wd[j])));
      }
    }
    if constexpr (k128x128) {
      float m = cm[0];
#pragma unroll
      for (int j = 1; j < 8; ++j) m = fmaxf(m, cm[j]);
      m = warp_max(m);
      if ((t & 31) == 0) warp_amax[w] = m;
    } else {
      // lanes l and l + 16 hold rows 16 w .. 16 w + 7 and + 8 .. + 15
#pragma unroll
      for (int j = 0; j < 8; ++j) cm[j] = fmaxf(cm[j], __shfl_xor_sync(0xFFFFFFFFu, cm[j], 16));
      if ((t & 16) == 0) {
        float4* pw = reinterpret_cast<float4*>(&part[w][8 * ch]);
        pw[0] = make_float4(cm[0], cm[1], cm[2], cm[3]);
        pw[1] = make_float4(cm[4], cm[5], cm[6], cm[7]);
      }
    }
    __syncthreads();  // every thread holds its rows: the buffer may be refilled
    if (t == 0 && issued_to < n_tiles) {
      fence_proxy_async_smem();
      issue(issued_to, s);
      issued_to += gridDim.x;
    }
    float* const sc = scales + e * scales_per_matrix;
    float inv[8];
    if constexpr (k128x128) {
      float gm = warp_amax[0];
#pragma unroll
      for (int k = 1; k < kTrThreads / 32; ++k) gm = fmaxf(gm, warp_amax[k]);
      const ScalePair sp = scales_from_amax(gm);
#pragma unroll
      for (int j = 0; j < 8; ++j) inv[j] = sp.inv;
      if (t == 0) sc[kb * n_cb + cb] = sp.s;
    } else {
      // thread c < 128: column c's scale from the 8 warps' maxima, once
      if (t < kTrCols) {
        float gm = part[0][t];
#pragma unroll
        for (int k = 1; k < kTrThreads / 32; ++k) gm = fmaxf(gm, part[k][t]);
        const ScalePair sp = scales_from_amax(gm);
        inv_s[t] = sp.inv;
        const int64_t col = cb * kTrCols + t;
        if (col < cols) sc[kb * cols + col] = sp.s;
      }
      __syncthreads();
      const float4 a = reinterpret_cast<const float4*>(inv_s)[2 * ch];
      const float4 b = reinterpret_cast<const float4*>(inv_s)[2 * ch + 1];
      inv[0] = a.x; inv[1] = a.y; inv[2] = a.z; inv[3] = a.w;
      inv[4] = b.x; inv[5] = b.y; inv[6] = b.z; inv[7] = b.w;
    }
    // the 8 codes of column 8 ch + j (rows 8 rg .. + 7) -> one word of
    // output row 8 ch + j, at slot rg ^ ch (8-byte slots of a 128-byte row);
    // two rows per packed multiply (each lane one IEEE fp32 multiply)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float2 inv2 = make_float2(inv[j], inv[j]);
      uint32_t c16[4];
#pragma unroll
      for (int pr = 0; pr < 4; ++pr) {
        const uint32_t w0 = j < 2 ? v[2 * pr].x : j < 4 ? v[2 * pr].y : j < 6 ? v[2 * pr].z
                                                                              : v[2 * pr].w;
        const uint32_t w1 = j < 2 ? v[2 * pr + 1].x : j < 4 ? v[2 * pr + 1].y
                          : j < 6 ? v[2 * pr + 1].z : v[2 * pr + 1].w;
        const float2 xy = (j & 1) ? make_float2(bf16_hi(w0), bf16_hi(w1))
                                  : make_float2(bf16_lo(w0), bf16_lo(w1));
        c16[pr] = static_cast<uint32_t>(
            __nv_cvt_float2_to_fp8x2(mul2(xy, inv2), __NV_SATFINITE, __NV_E4M3));
      }
      const uint2 codes = make_uint2(c16[0] | (c16[1] << 16), c16[2] | (c16[3] << 16));
      *reinterpret_cast<uint2*>(stage_out + (8 * ch + j) * 128 + 8 * (rg ^ ch)) = codes;
    }
    __syncthreads();
    {
      uint8_t* const qm = q + e * cols * ldq;
      const int seg = t & 7;  // 16-byte segment of an output row
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = (t >> 3) + 32 * u;  // output row within the tile
        const int64_t ocol = cb * kTrCols + c;
        const int sw = (c >> 3) & 15;
        const uint2 lo = *reinterpret_cast<const uint2*>(stage_out + c * 128 + 8 * ((2 * seg) ^ sw));
        const uint2 hi =
            *reinterpret_cast<const uint2*>(stage_out + c * 128 + 8 * ((2 * seg + 1) ^ sw));
        if (ocol < cols)
          *reinterpret_cast<uint4*>(qm + ocol * ldq + kb * kTrRows + 16 * seg) =
              make_uint4(lo.x, lo.y, hi.x, hi.y);
      }
    }
    // every thread is done with the staging rows and part / warp_amax
    __syncthreads();
  }
  // a CTA that stopped early lets the loads it issued land before it exits
  if (t == 0) {
    for (int k = 0; k < kTrStages; ++k) {
      uint32_t dummy = 0;
      const int64_t jj = static_cast<int64_t>(i) + k;
      const int64_t tile_j = blockIdx.x + jj * gridDim.x;
      if (tile_j < n_tiles && tile_j < issued_to)
        mbar_wait(&full[jj % kTrStages], static_cast<uint32_t>((jj / kTrStages) & 1), &dummy,
                  nullptr, SITE_TEARDOWN, 10000000ull);
    }
  }
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

// Builds x's tile map ((cols, rows, batch) bf16, 128 x 128 boxes) and
// launches the persistent transposed kernel on up to kTrCtasPerSm CTAs per SM.
static cudaError_t launch_transposed(const void* xv, int64_t rows, int64_t cols, int64_t ld,
                                     bool k128, bool grouped, void* qv, float* scales,
                                     const int32_t* offs, int32_t E, int64_t ldq, int64_t n_kb,
                                     int32_t batch, const LaunchCtx& ctx) {
  cudaError_t e = configure_transposed(ctx);
  if (e != cudaSuccess) return e;
  CUtensorMap tm;
  // (an expert split with no tokens: the map is never read, but must be valid)
  const uint64_t map_rows = rows > 0 ? static_cast<uint64_t>(rows) : 1;
  const uint64_t dims[3] = {static_cast<uint64_t>(cols), map_rows, static_cast<uint64_t>(batch)};
  const uint64_t strides[2] = {static_cast<uint64_t>(ld) * 2, map_rows * ld * 2};
  const uint32_t box[3] = {kTrCols, kTrRows, 1};
  if (!make_tmap(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, xv != nullptr ? xv : qv, dims, strides,
                 box, CU_TENSOR_MAP_SWIZZLE_NONE, ctx.err))
    return cudaErrorInvalidValue;
  const int64_t tiles = n_kb * ((cols + kTrCols - 1) / kTrCols) * batch;
  const int64_t max_grid = static_cast<int64_t>(ctx.num_sms) * kTrCtasPerSm;
  const unsigned grid = static_cast<unsigned>(tiles < max_grid ? tiles : max_grid);
  uint8_t* q = static_cast<uint8_t*>(qv);
  if (grouped)
    quant_transposed_kernel<false, true><<<grid, kTrThreads, kTrSmemBytes, ctx.stream>>>(
        tm, rows, cols, q, scales, offs, E, ldq, n_kb, ctx.status, batch);
  else if (k128)
    quant_transposed_kernel<true, false><<<grid, kTrThreads, kTrSmemBytes, ctx.stream>>>(
        tm, rows, cols, q, scales, nullptr, 0, ldq, n_kb, ctx.status, batch);
  else
    quant_transposed_kernel<false, false><<<grid, kTrThreads, kTrSmemBytes, ctx.stream>>>(
        tm, rows, cols, q, scales, nullptr, 0, ldq, n_kb, ctx.status, batch);
  return cudaGetLastError();
}

cudaError_t launch_quantize_transposed(const void* xv, int64_t rows, int64_t cols,
                                       int64_t ld, int recipe, void* qv, float* scales,
                                       const LaunchCtx& ctx) {
  if (rows == 0 || cols == 0) return cudaSuccess;
  return launch_transposed(xv, rows, cols, ld, recipe == 3, false, qv, scales, nullptr, 0, rows,
                           rows / kTrRows, 1, ctx);
}

cudaError_t launch_quantize_transposed_batched(const void* xv, int32_t batch, int64_t rows,
                                               int64_t cols, int64_t ld, int recipe, void* qv,
                                               float* scales, const LaunchCtx& ctx) {
  if (batch == 0 || rows == 0 || cols == 0) return cudaSuccess;
  return launch_transposed(xv, rows, cols, ld, recipe == 3, false, qv, scales, nullptr, 0, rows,
                           rows / kTrRows, batch, ctx);
}

// The 128x128 quantizer over `batch` equal (rows, cols) matrices stored one
// after the other (row stride ld, matrix stride rows * ld).
static cudaError_t launch_128x128(const void* xv, int32_t batch, int64_t rows, int64_t cols,
                                  int64_t ld, void* qv, float* scales, const LaunchCtx& ctx) {
  if (batch == 0 || rows == 0 || cols == 0) return cudaSuccess;
  CUtensorMap tm;
  const uint64_t dims[3] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(rows),
                            static_cast<uint64_t>(batch)};
  const uint64_t strides[2] = {static_cast<uint64_t>(ld) * 2,
                               static_cast<uint64_t>(rows) * static_cast<uint64_t>(ld) * 2};
  const uint32_t box[3] = {128, 128, 1};
  if (!make_tmap(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, xv, dims, strides, box,
                 CU_TENSOR_MAP_SWIZZLE_NONE, ctx.err))
    return cudaErrorInvalidValue;
  const int64_t tiles = ((rows + 127) / 128) * (cols / 128);
  quant_128x128_kernel<<<dim3(static_cast<unsigned>(tiles), static_cast<unsigned>(batch)),
                         k128Threads, kQSmemBytes, ctx.stream>>>(
      tm, rows, cols, static_cast<uint8_t*>(qv), scales, ctx.status);
  return cudaGetLastError();
}

cudaError_t launch_quantize_128x128_batched(const void* xv, int32_t batch, int64_t rows,
                                            int64_t cols, int64_t ld, void* qv, float* scales,
                                            const LaunchCtx& ctx) {
  return launch_128x128(xv, batch, rows, cols, ld, qv, scales, ctx);
}

int64_t grouped_padded_tokens(int64_t tokens, int32_t E) {
  return ((tokens + kTrRows - 1) / kTrRows + E) * kTrRows;
}

cudaError_t launch_quantize_transposed_grouped(const void* xv, int64_t rows, int64_t cols,
                                               int64_t ld, const int32_t* offs, int32_t E,
                                               void* qv, float* scales, const LaunchCtx& ctx) {
  if (cols == 0) return cudaSuccess;
  const int64_t P = grouped_padded_tokens(rows, E);
  return launch_transposed(xv, rows, cols, ld, false, true, qv, scales, offs, E, P, P / kTrRows,
                           1, ctx);
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
  if (recipe == 3)  // 128x128
    return launch_128x128(x, 1, rows, cols, ld, q, scales, ctx);
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
