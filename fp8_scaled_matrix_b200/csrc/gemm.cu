// FP8 (e4m3) scaled GEMM on the 5th-generation tensor cores (sm_100a).
//
//   out[m, n] = sum_k (A[m,k] sA) (B[n,k] sB) (+ bias[n])
//
// "Fix: Handle LowLevelZeroPlugin with use_fp8=True" (Solution, forward pass)
// fixes what is computed: the scaled matmul equals dequantize-then-matmul plus
// bias.  Recipes: tensorwise and rowwise ("Add _scaled_mm_v2 API"),
// blockwise 1x128_128x128 and 1x128_128x1 ("improve fp8 blockwise gemm
// perf"), the grouped rowwise MoE form over (E, N, K) experts with
// cumulative offs ("Add _grouped_mm dispatch handler to Float8Tensor"), and
// MXFP8 (the "mxfp8" recipe of "Add _scaled_mm_v2 API": one E8M0 scale per
// 32 elements of K, applied by the tensor core itself through
// tcgen05.mma.kind::mxf8f6f4.block_scale with the scales staged in TMEM).
//
// One persistent kernel, one CTA per SM, 12 warps with fixed roles:
//   warp 0      TMA producer: A (128 x 128 B) and B (256 x 128 B) tiles into
//               a 4-stage shared-memory ring (128-byte swizzle)
//   warp 1      TMEM owner + MMA issuer: one thread issues
//               tcgen05.mma.kind::f8f6f4 into fp32 TMEM accumulators;
//               tcgen05.commit frees stages and hands accumulators over
//   warp 2      blockwise: scale producer (cp.async ring of per-K-block row
//               and column scales, kSclSlots K blocks ahead); grouped:
//               validates offs in the prologue
//   warp 3      idle after the prologue
//   warps 4-11  epilogue: warp w reads TMEM lanes 32*(w%4).. (the hardware's
//               lane quarter) and columns 128*((w-4)/4).. of each tile
// The blockwise kernels move registers from warpgroup 0 to the epilogue
// warpgroups (setmaxnreg) so each epilogue thread can hold its 128 fp32
// accumulators plus 64 freshly loaded TMEM values.
// TMEM holds two 256-column fp32 buffers.  Tensorwise / rowwise: each buffer
// is one whole tile's accumulator (M=128, N=256, K=32 MMAs), so the epilogue
// of tile i overlaps the MMAs of tile i+1.  Blockwise: each 128-wide K block
// is accumulated into a buffer on its own (no carry-in), and the epilogue
// warps promote it -- acc += partial * sA[m,kb] * sB[.,kb] -- into fp32
// registers while the tensor core fills the other buffer.  Results are scaled,
// biased, rounded to bf16 (or kept fp32), staged in shared memory and written
// by TMA stores (the grouped kernel masks rows past its group with plain
// 16-byte stores).
//
// Every wait is bounded (one second); a wait that gives up records
// FP8_ERR_TIMEOUT in the device status word, the CTA drains its in-flight
// copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <cstdlib>

#include "fp8cast.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace fp8sm {
namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;  // bytes == e4m3 elements per stage along K
constexpr int UMMA_K = 32;
constexpr int kEpiWarps = 8;
constexpr int kFirstEpiWarp = 4;  // warps 0-3 = warpgroup 0 (producer, MMA, 2 idle)
constexpr int kThreads = 32 * kFirstEpiWarp + 32 * kEpiWarps;
// Register split (blockwise kernels): warpgroup 0 gives registers up, the two
// epilogue warpgroups take them.  Launch: 384 threads x 168 registers =
// 64512 = 128 x kRegsLow + 256 x kRegsHigh.  The host refuses to launch a
// kernel that was compiled with fewer than kRegsAtLaunch registers.
constexpr uint32_t kRegsLow = 56;
constexpr uint32_t kRegsHigh = 224;
constexpr uint32_t kRegsAtLaunch = 168;
static_assert(128 * kRegsLow + 256 * kRegsHigh <= kThreads * kRegsAtLaunch,
              "register split exceeds the launch allocation");
constexpr uint32_t kTmemCols = 512;  // two 256-column fp32 buffers
constexpr uint32_t kEpiBuf = 32 * 64;  // 32 rows x 64 bytes, 64-byte swizzle
// dual e4m3 output: per epilogue warp, 16 columns x 32 rows of transposed
// codes (also the column maxima the half's warps exchange)
constexpr uint32_t kTposBuf = 512;
// Blockwise scale ring: one slot per K block, filled ahead by warp 2 with
// cp.async: [128 row scales sA[kb, m0..] | column scales: sB[kb, nb0],
// sB[kb, nb0 + 1] (1x128_128x128) or sB[kb, n0 .. n0 + 255] (1x128_128x1)].
constexpr int kSclSlots = 8;
constexpr int kSclSlotFloats = 128 + 256;
constexpr uint32_t kSclBytes = kSclSlots * kSclSlotFloats * 4;
// MXFP8: per stage, three 512-byte scale-factor tiles (A's 128 rows, B's two
// 128-row halves) land next to the operands, in the scale-ring region (which
// the MXFP8 kernel does not otherwise use); in TMEM each stage has a
// 16-column slot after the accumulator (A: 4 columns, B: 8).
constexpr uint32_t kMxSfTile = 512;
constexpr uint32_t kMxSfStage = 3 * kMxSfTile;
constexpr uint32_t kMxSfCols = 16;

// Shared-memory layout.  Tiles are 128 x 256: each stage holds A (128 rows)
// and B (256 rows) of a 128-byte K slice.  kStaged: one stage traded for
// four output staging buffers per epilogue warp (staged_epilogue below).
template <bool kStaged>
struct CfgT {
  static constexpr int kStages = kStaged ? 3 : 4;
  static constexpr int kEpiBufs = kStaged ? 4 : 1;  // staging buffers per epilogue warp
  static constexpr int kTileM = BM;   // output rows per work item
  static constexpr uint32_t kBRows = BN;  // B rows held per stage
  static constexpr uint32_t kAStage = BM * BK;
  static constexpr uint32_t kBStage = kBRows * BK;
  static constexpr uint32_t kOffA = 0;
  static constexpr uint32_t kOffB = kOffA + kStages * kAStage;
  static constexpr uint32_t kOffEpi = kOffB + kStages * kBStage;
  static constexpr uint32_t kOffScl = kOffEpi + kEpiWarps * kEpiBufs * kEpiBuf;
  static constexpr uint32_t kOffTpos = kOffScl + kSclBytes;
  static constexpr uint32_t kOffBar = kOffTpos + kEpiWarps * kTposBuf;
  // barriers: full[kStages], empty[kStages], acc_full[2], acc_empty[2], drain,
  // scale ring sfull[kSclSlots], sempty[kSclSlots], epilogue half sync hsync[2]
  static constexpr uint32_t kNumBars = 2 * kStages + 5 + 2 * kSclSlots + 2;
  static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
  static constexpr uint32_t kSmemUsed = kOffMisc + 16;
  static constexpr uint32_t kSmemBytes = kSmemUsed + 1024;  // + alignment slack
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kStages * kMxSfStage <= kSclBytes, "MXFP8 scale tiles fit the ring region");
  static_assert(BN + kStages * kMxSfCols <= kTmemCols, "MXFP8 TMEM slots");
};
using Cfg = CfgT<false>;

enum Recipe : int { kTensor = 0, kRow = 1, kBlock128 = 2, kBlock1 = 3, kMxfp8 = 4 };
// Output: bf16, fp32, e4m3 quantized in 1x128 groups along n (+ fp32
// scales), or MXFP8 (e4m3 + one E8M0 scale per 32 columns, in scale-factor
// tiles: the A operand of the next MXFP8 GEMM), or both e4m3 forms of the
// result (1x128 along n, and transposed with 1x128 groups along m: the two
// operands the next layer's backward GEMMs read)
enum OutKind : int { kOutBf16 = 0, kOutFp32 = 1, kOutE4M3 = 2, kOutMx = 3, kOutE4M3Dual = 4 };

// A blockwise epilogue writes its tile only after the last K block, while the
// MMA can run at most two K blocks ahead; with four staging buffers per warp
// the tile's boxes leave back to back instead of each waiting for the
// previous box's TMA store to read the one buffer.  Measured worth the stage
// it costs for 1x128_128x1 (844 against 867 us on 16640 x 5120 x 8192); the
// 1x128_128x128 kernels (every output kind) gain nothing from it and keep
// four stages.
__host__ __device__ constexpr bool staged_epilogue(int recipe, int /*out_kind*/) {
  return recipe == kBlock1;
}

struct GemmParams {
  int64_t M, N, K;
  const float* sa;
  const float* sb;
  const uint8_t* sfa;  // MXFP8: scale-factor tiles of A and B (E8M0 bytes)
  const uint8_t* sfb;
  int64_t sfa_bytes, sfb_bytes;  // their sizes: every copy is checked against them
  const uint16_t* bias;
  void* out;
  float* out_scales;  // e4m3 output: scale[(n/128) * M + m]; MXFP8 output: tiles
  uint8_t* out_t;      // dual e4m3 output: the result transposed, (N, M) codes
  float* out_t_scales; //   and its scales, 1x128 along m: scale[(m/128) * N + n]
  const int32_t* offs;
  int32_t E;
  int64_t tokens;    // K-grouped (weight gradient): offs[E-1] must equal this
  int32_t n_tiles;   // tiles along N
  int32_t m_tiles;   // tiles along M (dense)
  int32_t k_blocks;
  int32_t raster_m;  // dense: 0 = M-major tile order, else bands of this many M tiles
  uint32_t* status;
  // Dense kernels: work items [0, split_start) are whole 128 x 256 tiles in
  // M-major order; when the last wave would leave more than half of the SMs
  // idle, each of its tiles becomes two 128 x 128 items (split_start ..
  // total_items), so twice as many SMs finish it in half the time.
  int64_t split_start;
  int64_t total_items;
};

// Walks the concatenated per-group M tiles in increasing order.
struct GroupCursor {
  int32_t g;
  int64_t tiles_before;  // M tiles of groups < g
  int64_t row_start;
  int64_t row_end;
  int64_t m_tiles;  // M tiles of group g
  __device__ void init(const int32_t* offs, int64_t tm) {
    g = 0;
    tiles_before = 0;
    row_start = 0;
    row_end = offs[0];
    m_tiles = (row_end + tm - 1) / tm;
  }
  __device__ void seek(int64_t mt, const int32_t* offs, int32_t E, int64_t tm) {
    while (mt >= tiles_before + m_tiles && g + 1 < E) {
      tiles_before += m_tiles;
      ++g;
      row_start = row_end;
      row_end = offs[g];
      m_tiles = (row_end - row_start + tm - 1) / tm;
    }
  }
};

struct TileCoord {
  int32_t m0, n0, g;
  int64_t row_end;
  bool half_n;  // 128-wide item (columns n0 .. n0+127 only)
  int32_t out_m0;  // first output row (differs from m0 for the K-grouped GEMM)
  int64_t kb0;     // K-grouped: first (padded) K block of the item's group
  int32_t nkb;     // K-grouped: K blocks of the group
};

// K-grouped GEMM (per-expert weight gradient): walks the groups' padded K
// block ranges in increasing group order.
struct KGroupCursor {
  int32_t g;
  int64_t kb0;  // padded 128-blocks of groups < g
  int32_t nkb;  // padded 128-blocks of group g
  __device__ static int32_t blocks(const int32_t* offs, int32_t g) {
    const int32_t prev = g ? offs[g - 1] : 0;
    return (offs[g] - prev + BK - 1) / BK;
  }
  __device__ void init(const int32_t* offs) {
    g = 0;
    kb0 = 0;
    nkb = blocks(offs, 0);
  }
  __device__ void seek(int32_t target, const int32_t* offs) {
    while (g < target) {
      kb0 += nkb;
      ++g;
      nkb = blocks(offs, g);
    }
  }
};

// Work item t -> output tile (rows m0 .. m0 + kTM - 1).
template <bool kGrouped, int kTM, bool kRaster>
__device__ __forceinline__ TileCoord tile_coord(int64_t t, const GemmParams& p,
                                                GroupCursor& cur) {
  TileCoord c;
  c.half_n = false;
  int32_t sub = 0;
  if constexpr (!kGrouped) {
    if (t >= p.split_start) {
      const int64_t h = t - p.split_start;
      t = p.split_start + (h >> 1);
      sub = static_cast<int32_t>(h & 1);
      c.half_n = true;
    }
  }
  c.kb0 = 0;
  c.nkb = 0;
  int64_t mt = t / p.n_tiles;
  int64_t nt = t % p.n_tiles;
  if constexpr (!kGrouped && kRaster) {
    if (p.raster_m > 0) {
      // grouped raster: bands of raster_m M tiles, N-major inside a band,
      // so that a wave touches a band of A and a slice of B that fit in L2
      const int64_t per = static_cast<int64_t>(p.raster_m) * p.n_tiles;
      const int64_t band = t / per;
      const int64_t local = t - band * per;
      const int64_t left = p.m_tiles - band * p.raster_m;
      const int64_t gm = left < p.raster_m ? left : p.raster_m;
      mt = band * p.raster_m + local % gm;
      nt = local / gm;
    }
  }
  c.n0 = static_cast<int32_t>(nt * BN) + sub * (BN / 2);
  if constexpr (kGrouped) {
    cur.seek(mt, p.offs, p.E, kTM);
    c.g = cur.g;
    c.m0 = static_cast<int32_t>(cur.row_start + (mt - cur.tiles_before) * kTM);
    c.row_end = cur.row_end;
  } else {
    c.g = 0;
    c.m0 = static_cast<int32_t>(mt * kTM);
    c.row_end = p.M;
  }
  c.out_m0 = c.m0;
  return c;
}

// K-grouped work item t -> (group g, A rows m0.., B rows n0..) with the
// group's K blocks; output rows g * M + m0 ...
__device__ __forceinline__ TileCoord kgroup_coord(int64_t t, const GemmParams& p,
                                                  KGroupCursor& kc) {
  TileCoord c;
  c.half_n = false;
  const int64_t per_group = static_cast<int64_t>(p.m_tiles) * p.n_tiles;
  const int32_t g = static_cast<int32_t>(t / per_group);
  const int64_t r = t % per_group;
  kc.seek(g, p.offs);
  c.g = g;
  c.m0 = static_cast<int32_t>((r / p.n_tiles) * BM);
  c.n0 = static_cast<int32_t>((r % p.n_tiles) * BN);
  c.out_m0 = static_cast<int32_t>(static_cast<int64_t>(g) * p.M + c.m0);
  c.row_end = static_cast<int64_t>(g + 1) * p.M;
  c.kb0 = kc.kb0;
  c.nkb = kc.nkb;
  return c;
}

// 32 consecutive fp32 column values of `src` starting at column n (n a
// multiple of 32); columns >= N read as 0.  N is a multiple of 16, so each
// 16-column half is either wholly inside or wholly outside.
__device__ __forceinline__ void load_cols32_f32(const float* src, int64_t n,
                                                int64_t N, float (&v)[32]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (n + 16 * h < N) {
      const float4* p = reinterpret_cast<const float4*>(src + n + 16 * h);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 f = __ldg(p + i);
        v[16 * h + 4 * i + 0] = f.x;
        v[16 * h + 4 * i + 1] = f.y;
        v[16 * h + 4 * i + 2] = f.z;
        v[16 * h + 4 * i + 3] = f.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) v[16 * h + i] = 0.0f;
    }
  }
}

__device__ __forceinline__ void load_bias32(const uint16_t* bias, int64_t n,
                                            int64_t N, float (&v)[32]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (bias != nullptr && n + 16 * h < N) {
      const uint4* p = reinterpret_cast<const uint4*>(bias + n + 16 * h);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint4 u = __ldg(p + i);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          v[16 * h + 8 * i + 2 * j] = __uint_as_float(w[j] << 16);
          v[16 * h + 8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) v[16 * h + i] = 0.0f;
    }
  }
}

// Stage 4 x 16-byte chunks of this lane's row in the warp's 32 x 64-byte
// buffer (64-byte swizzle: chunk j of row r lives at slot j ^ ((r >> 1) & 3)),
// then write the 32 x 64-byte box to global memory.  kStore:
//   kStoreTma     TMA store (boxes wholly past the last row or column are
//                 skipped, partial ones clipped at the matrix's edges);
//   kStoreMixed   (row-grouped kernels, whose tiles may end inside a group)
//                 TMA store for a box whose 32 rows all lie before row_end,
//                 masked 16-byte stores for one that crosses row_end;
//   kStoreMasked  masked 16-byte stores always (the grouped blockwise
//                 kernel: its epilogue holds 128 accumulators per thread, and
//                 the second store path's registers cost it more than TMA
//                 stores save, measured).
enum StoreMode : int { kStoreTma = 0, kStoreMixed = 1, kStoreMasked = 2 };
// The warp's kBufs staging buffers (ebase, kEpiBuf bytes each) take the boxes
// in turn (nbox counts them); before the first buffer is reused, every
// earlier TMA store of the warp must have read its buffer.
template <int kStore, int kBufs>
__device__ __forceinline__ void store_box64(
    uint8_t* ebase, uint32_t& nbox, const uint4 (&chunk)[4], const CUtensorMap* tm_out,
    int32_t col0 /*elements*/, int32_t row0, int64_t row_end, uint8_t* out,
    int64_t N, uint32_t elem_bytes, uint32_t lane) {
  const uint32_t b = kBufs > 1 ? nbox % kBufs : 0u;
  uint8_t* buf = ebase + b * kEpiBuf;
  ++nbox;
  if constexpr (kStore != kStoreMasked) {
    if (b == 0) {
      if (lane == 0) bulk_wait_group_read0();
      __syncwarp();
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t slot = static_cast<uint32_t>(j) ^ ((lane >> 1) & 3u);
    *reinterpret_cast<uint4*>(buf + lane * 64 + slot * 16) = chunk[j];
  }
  // warp-uniform
  const bool whole = kStore == kStoreTma ||
                     (kStore == kStoreMixed && static_cast<int64_t>(row0) + 32 <= row_end);
  if (whole) {
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && row0 < row_end && col0 < N) {
      tma_store_2d(tm_out, buf, col0, row0);
      bulk_commit_group();
    }
  } else {
    __syncwarp();
    const uint32_t elems_per_chunk = 16u / elem_bytes;
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const uint32_t idx = it * 32 + lane;
      const uint32_t r = idx >> 2;
      const uint32_t j = idx & 3u;
      const uint32_t slot = j ^ ((r >> 1) & 3u);
      const uint4 v = *reinterpret_cast<const uint4*>(buf + r * 64 + slot * 16);
      const int64_t row = static_cast<int64_t>(row0) + r;
      const int64_t col = static_cast<int64_t>(col0) + j * elems_per_chunk;
      if (row < row_end && col < N)
        *reinterpret_cast<uint4*>(out + (row * N + col) * elem_bytes) = v;
    }
    __syncwarp();
  }
}

// Write 32 fp32 results of this lane's row (columns col0 .. col0+31).
template <bool kOutF32, int kStore, int kBufs>
__device__ __forceinline__ void store_cols32(
    uint8_t* ebase, uint32_t& nbox, const float (&v)[32], const CUtensorMap* tm_out,
    int32_t col0, int32_t row0, int64_t row_end, void* out, int64_t N, uint32_t lane) {
  if constexpr (!kOutF32) {
    uint4 c[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      c[j] = make_uint4(pack_bf16x2(v[8 * j + 0], v[8 * j + 1]),
                        pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                        pack_bf16x2(v[8 * j + 4], v[8 * j + 5]),
                        pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
    store_box64<kStore, kBufs>(ebase, nbox, c, tm_out, col0, row0, row_end,
                               static_cast<uint8_t*>(out), N, 2, lane);
  } else {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint4 c[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        c[j] = make_uint4(__float_as_uint(v[16 * h + 4 * j + 0]),
                          __float_as_uint(v[16 * h + 4 * j + 1]),
                          __float_as_uint(v[16 * h + 4 * j + 2]),
                          __float_as_uint(v[16 * h + 4 * j + 3]));
      store_box64<kStore, kBufs>(ebase, nbox, c, tm_out, col0 + 16 * h, row0, row_end,
                                 static_cast<uint8_t*>(out), N, 4, lane);
    }
  }
}

template <int kRecipe, int kOut, bool kGrouped>
__global__ void __launch_bounds__(kThreads, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                    const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ CUtensorMap tm_b_half,
                    const __grid_constant__ CUtensorMap tm_out,
                    const GemmParams p) {
  constexpr bool kBlockwise = (kRecipe == kBlock128 || kRecipe == kBlock1);
  constexpr bool kIsMx = kRecipe == kMxfp8;
  // grouped MXFP8: a group's 128-row tile rarely starts on a 128-row
  // boundary, so warp 2 gathers A's scale words into each stage
  constexpr bool kMxGather = kIsMx && kGrouped;
  // grouped 1x128_128x1 = the per-expert weight gradient: groups split K
  // (tokens), every group has its own (M, N) output
  constexpr bool kKGroups = kGrouped && kRecipe == kBlock1;
  // stores: TMA stores; the row-grouped kernels' tiles may end inside a
  // group, so there a 32-row box that crosses the group's end goes out by
  // masked plain stores instead (the K-grouped output's tiles are whole:
  // M % 128 == 0)
  constexpr bool kMasked = kGrouped && !kKGroups;
  constexpr int kStore = !kMasked ? kStoreTma : kBlockwise ? kStoreMasked : kStoreMixed;
  // epilogue threads that hold a whole 128-column row slice across K blocks
  // (blockwise promotion) get registers moved from warpgroup 0.  The MXFP8
  // epilogue reads its accumulators once per tile and runs without the split.
  constexpr bool kBigEpi = kBlockwise;
  constexpr bool kOutF32 = kOut == kOutFp32;
  constexpr bool kOutQT = kOut == kOutE4M3Dual;
  constexpr bool kOutQ = kOut == kOutE4M3 || kOutQT;
  constexpr bool kOutMxq = kOut == kOutMx;
  // the banded tile order (large B operands); the dual-output kernel, whose
  // epilogue is at the edge of its register budget, keeps the M-major order
  // (its B is a layer's weight, which fits in L2)
  constexpr bool kRaster = !kOutQT;
  using C = CfgT<staged_epilogue(kRecipe, kOut)>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::kStages;
  uint64_t* acc_full = bars + 2 * C::kStages;
  uint64_t* acc_empty = bars + 2 * C::kStages + 2;
  uint64_t* drain = bars + 2 * C::kStages + 4;
  uint64_t* sfull = bars + 2 * C::kStages + 5;
  uint64_t* sempty = sfull + kSclSlots;
  uint64_t* hsync = sempty + kSclSlots;  // the four epilogue warps of each half
  float* scl = reinterpret_cast<float*>(smem + C::kOffScl);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  uint32_t* tmem_slot = misc + 0;
  volatile uint32_t* abort_flag = misc + 1;
  int64_t* total_tiles_slot = reinterpret_cast<int64_t*>(misc + 2);

  const uint32_t warp = warp_id_in_cta();
  const uint32_t lane = lane_id();

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      // grouped MXFP8: each lane of warp 2 also arrives once its copies of
      // the stage's A scale words have landed
      mbar_init(&full[s], kMxGather ? 1 + 32 : 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) mbar_init(&acc_full[i], 1);
    // every epilogue warp hands a buffer back
    for (int i = 0; i < 2; ++i) mbar_init(&acc_empty[i], kEpiWarps);
    mbar_init(drain, 1);
    for (int i = 0; i < kSclSlots; ++i) {
      // one cp.async arrival per lane of warp 2, plus lane 0's (with the bulk
      // copies' byte count)
      mbar_init(&sfull[i], 33);
      mbar_init(&sempty[i], kEpiWarps);
    }
    for (int i = 0; i < 2; ++i) mbar_init(&hsync[i], kEpiWarps / 2);
    *abort_flag = 0u;
    fence_barrier_init();
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    if constexpr (!kGrouped) prefetch_tmap(&tm_b_half);
    prefetch_tmap(&tm_out);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 2) {
    int64_t total;
    if constexpr (kGrouped) {
      // Validate offs (non-decreasing, ends at M) and count M tiles.
      bool bad = false;
      int64_t mt = 0;
      for (int32_t i = static_cast<int32_t>(lane); i < p.E; i += 32) {
        const int32_t e = p.offs[i];
        const int32_t prev = i ? p.offs[i - 1] : 0;
        if (e < prev || prev < 0) bad = true;
        else mt += (static_cast<int64_t>(e) - prev + C::kTileM - 1) / C::kTileM;
      }
      if (lane == 0 && static_cast<int64_t>(p.offs[p.E - 1]) != (kKGroups ? p.tokens : p.M))
        bad = true;
      int64_t kblocks = 0;  // K-grouped: the groups' padded K blocks must fit in K
      if constexpr (kKGroups) {
        for (int32_t i = static_cast<int32_t>(lane); i < p.E; i += 32) {
          const int32_t prev = i ? p.offs[i - 1] : 0;
          kblocks += (static_cast<int64_t>(p.offs[i]) - prev + BK - 1) / BK;
        }
      }
      bad = __any_sync(0xFFFFFFFFu, bad);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        mt += __shfl_xor_sync(0xFFFFFFFFu, mt, o);
        kblocks += __shfl_xor_sync(0xFFFFFFFFu, kblocks, o);
      }
      if constexpr (kKGroups) {
        if (kblocks > p.k_blocks) bad = true;
        total = bad ? 0 : static_cast<int64_t>(p.E) * p.m_tiles * p.n_tiles;
      } else {
        total = bad ? 0 : mt * p.n_tiles;
      }
      if (bad && lane == 0 && blockIdx.x == 0)
        record_status(p.status, FP8_DEV_VALUE, SITE_OFFS);
    } else {
      total = p.total_items;
    }
    if (lane == 0) *total_tiles_slot = total;
  }
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const int64_t total_tiles = *total_tiles_slot;
  const int32_t KB = p.k_blocks;
  const int64_t item0 = blockIdx.x;
  const int64_t item_stride = gridDim.x;
  constexpr int kTM = C::kTileM;

  if (warp < kFirstEpiWarp) {
   // warpgroup 0: all four warps execute the same setmaxnreg
   if constexpr (kBigEpi) warpgroup_reg_dealloc<kRegsLow>();
   if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      GroupCursor cur;
      KGroupCursor kc;
      if constexpr (kKGroups) kc.init(p.offs);
      else if constexpr (kGrouped) cur.init(p.offs, kTM);
      uint32_t stage = 0, phase = 0;
      uint64_t issued = 0;
      bool ok = true;
      for (int64_t t = item0; t < total_tiles && ok; t += item_stride) {
        const TileCoord c =
            kKGroups ? kgroup_coord(t, p, kc) : tile_coord<kGrouped, kTM, kRaster>(t, p, cur);
        const int32_t nkb = kKGroups ? c.nkb : KB;
        for (int32_t kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status,
                         SITE_PRODUCER_EMPTY, kWaitLimitNs)) {
            ok = false;
            break;
          }
          const uint32_t b_bytes = c.half_n ? C::kBStage / 2 : C::kBStage;
          uint8_t* a_dst = smem + C::kOffA + stage * C::kAStage;
          uint8_t* b_dst = smem + C::kOffB + stage * C::kBStage;
          if constexpr (kIsMx) {
            // operands plus their scale-factor tiles (tile (i, kb) of a
            // matrix's scales is its 128 rows 128 i .. and K elements
            // 128 kb ..); B's second half-tile exists only below N
            // (grouped: expert g's tile set follows the g earlier ones; A's
            // scale tile is gathered by warp 2)
            // (the second half of a split last-wave tile can start at or past
            // N; its columns are never stored, so it takes B's last tile)
            const int64_t NB = (p.N + 127) / 128;
            const int64_t nb0 = c.n0 / 128 < NB ? c.n0 / 128 : NB - 1;
            const bool two = !c.half_n && nb0 + 1 < NB;
            mbar_arrive_expect_tx(&full[stage], C::kAStage + b_bytes +
                                                    ((two ? 2u : 1u) + (kGrouped ? 0u : 1u)) *
                                                        kMxSfTile);
            tma_load_2d(a_dst, &tm_a, &full[stage], kb * BK, c.m0);
            if constexpr (kGrouped)
              tma_load_3d(b_dst, &tm_b, &full[stage], kb * BK, c.n0, c.g);
            else
              tma_load_2d(b_dst, c.half_n ? &tm_b_half : &tm_b, &full[stage], kb * BK, c.n0);
            uint8_t* sf_dst = smem + C::kOffScl + stage * kMxSfStage;
            const int64_t kbb =
                ((kGrouped ? static_cast<int64_t>(c.g) * NB * KB : 0) + nb0 * KB + kb) * kMxSfTile;
            const int64_t ka = (static_cast<int64_t>(c.m0 / 128) * KB + kb) * kMxSfTile;
            const int64_t kb2 = kbb + static_cast<int64_t>(KB) * kMxSfTile;
            if ((!kGrouped && (ka < 0 || ka + kMxSfTile > p.sfa_bytes)) || kbb < 0 ||
                kbb + kMxSfTile > p.sfb_bytes || (two && kb2 + kMxSfTile > p.sfb_bytes)) {
              // a scale-tile copy outside the buffers: stop instead of faulting
              // (the stage's expected bytes never arrive; every waiter gives up)
              record_status(p.status, FP8_DEV_VALUE, SITE_BOUNDS);
              *abort_flag = 1u;
              ok = false;
              break;
            }
            if constexpr (!kGrouped) bulk_load_g2s(sf_dst, p.sfa + ka, kMxSfTile, &full[stage]);
            bulk_load_g2s(sf_dst + kMxSfTile, p.sfb + kbb, kMxSfTile, &full[stage]);
            if (two) bulk_load_g2s(sf_dst + 2 * kMxSfTile, p.sfb + kb2, kMxSfTile, &full[stage]);
          } else if constexpr (kKGroups) {
            // the group's padded K range; A and B are (rows, padded tokens)
            const int32_t kx = static_cast<int32_t>((c.kb0 + kb) * BK);
            mbar_arrive_expect_tx(&full[stage], C::kAStage + b_bytes);
            tma_load_2d(a_dst, &tm_a, &full[stage], kx, c.m0);
            tma_load_2d(b_dst, &tm_b, &full[stage], kx, c.n0);
          } else {
            mbar_arrive_expect_tx(&full[stage], C::kAStage + b_bytes);
            tma_load_2d(a_dst, &tm_a, &full[stage], kb * BK, c.m0);
            if constexpr (kGrouped)
              tma_load_3d(b_dst, &tm_b, &full[stage], kb * BK, c.n0, c.g);
            else if (p.raster_m > 0)
              // banded order: B is streamed once per band, A's band is reused
              // by every wave of the band; B's lines go first
              tma_load_2d_hint(b_dst, c.half_n ? &tm_b_half : &tm_b, &full[stage], kb * BK,
                               c.n0, l2_policy_evict_first());
            else
              tma_load_2d(b_dst, c.half_n ? &tm_b_half : &tm_b, &full[stage], kb * BK, c.n0);
          }
          ++issued;
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // Let the copies already in flight land before the CTA exits.
        const uint64_t first = issued > C::kStages ? issued - C::kStages : 0;
        for (uint64_t i = first; i < issued; ++i) {
          uint32_t dummy_abort = 0;
          mbar_wait(&full[i % C::kStages], static_cast<uint32_t>((i / C::kStages) & 1u),
                    &dummy_abort, nullptr, SITE_TEARDOWN, 10000000ull);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_full = idesc_e4m3_f32(kTM, BN);
      const uint32_t idesc_half = idesc_e4m3_f32(kTM, BN / 2);
      uint32_t stage = 0, phase = 0;
      uint32_t acc = 0, acc_phase = 0;
      bool ok = true;
      // The issue loop is kept lean (the single issuing thread, not the
      // tensor core, is the limit at 4 MMAs per stage): no fence after a
      // stage wait (TMA writes and MMA reads are both async-proxy, ordered by
      // the barrier), and the next stage's barrier is peeked while this
      // stage's MMAs go out.
      bool ready = mbar_test_wait(&full[stage], phase);
      if constexpr (kIsMx) {
        // MXFP8: per stage, the scale-factor tiles go from shared memory to
        // the stage's TMEM slot (tcgen05.cp: 32 rows x 16 bytes copied to
        // all four lane quarters; ordered before this thread's later MMAs),
        // then four block-scaled MMAs, MMA k reading byte k (its 32-wide K
        // block) of each scale word.  One accumulator buffer: the scale
        // slots take the other half of TMEM, and the epilogue hands the
        // buffer back as soon as it has read it into registers.
        uint32_t idesc_f[4], idesc_h[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          idesc_f[k] = idesc_mx_e4m3(kTM, BN, k, k);
          idesc_h[k] = idesc_mx_e4m3(kTM, BN / 2, k, k);
        }
        for (int64_t t = item0; t < total_tiles && ok; t += item_stride) {
          const bool hn = t >= p.split_start;
          if (!mbar_wait(&acc_empty[0], acc_phase ^ 1u, abort_flag, p.status,
                         SITE_MMA_ACC_EMPTY, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          for (int32_t kb = 0; kb < KB; ++kb) {
            if (!ready && !mbar_wait(&full[stage], phase, abort_flag, p.status, SITE_MMA_FULL,
                                     kWaitLimitNs)) {
              ok = false;
              break;
            }
            const uint32_t cur = stage;
            if (++stage == C::kStages) {
              stage = 0;
              phase ^= 1u;
            }
            ready = mbar_test_wait(&full[stage], phase);
            const uint32_t sf_t = tmem_base + BN + cur * kMxSfCols;
            const uint32_t sf_s = smem_u32(smem + C::kOffScl + cur * kMxSfStage);
            // grouped: warp 2's cp.async wrote A's scale words (generic
            // proxy); order them before tcgen05.cp reads them (async proxy)
            if constexpr (kMxGather) fence_proxy_async_smem();
            tmem_cp_32x128b_warpx4(sf_t, smem_desc_rows16(sf_s));
            tmem_cp_32x128b_warpx4(sf_t + 4, smem_desc_rows16(sf_s + kMxSfTile));
            if (!hn) tmem_cp_32x128b_warpx4(sf_t + 8, smem_desc_rows16(sf_s + 2 * kMxSfTile));
            const uint64_t da = smem_desc_k_sw128(smem_u32(smem + C::kOffA + cur * C::kAStage));
            const uint64_t db = smem_desc_k_sw128(smem_u32(smem + C::kOffB + cur * C::kBStage));
#pragma unroll
            for (int k = 0; k < BK / UMMA_K; ++k)
              mma_mx_e4m3(tmem_base, da + (k * UMMA_K) / 16, db + (k * UMMA_K) / 16,
                          hn ? idesc_h[k] : idesc_f[k], sf_t, sf_t + 4, (kb > 0) || (k > 0));
            mma_commit(&empty[cur]);
          }
          if (ok) {
            mma_commit(&acc_full[0]);
            acc_phase ^= 1u;
          }
        }
      } else if constexpr (!kBlockwise) {
        for (int64_t t = item0; t < total_tiles && ok; t += item_stride) {
          const uint32_t idesc = (!kGrouped && t >= p.split_start) ? idesc_half : idesc_full;
          if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort_flag, p.status,
                                SITE_MMA_ACC_EMPTY, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          for (int32_t kb = 0; kb < KB; ++kb) {
            if (!ready && !mbar_wait(&full[stage], phase, abort_flag, p.status,
                                            SITE_MMA_FULL, kWaitLimitNs)) {
              ok = false;
              break;
            }
            const uint32_t cur = stage;
            if (++stage == C::kStages) {
              stage = 0;
              phase ^= 1u;
            }
            ready = mbar_test_wait(&full[stage], phase);  // peek at the next stage
            const uint32_t d = tmem_base + acc * BN;
            const uint64_t da = smem_desc_k_sw128(smem_u32(smem + C::kOffA + cur * C::kAStage));
            const uint64_t db = smem_desc_k_sw128(smem_u32(smem + C::kOffB + cur * C::kBStage));
#pragma unroll
            for (int k = 0; k < BK / UMMA_K; ++k)
              mma_e4m3(d, da + (k * UMMA_K) / 16, db + (k * UMMA_K) / 16, idesc,
                       (kb > 0) || (k > 0));
            mma_commit(&empty[cur]);
          }
          if (ok) {
            mma_commit(&acc_full[acc]);
            acc ^= 1u;
            if (acc == 0) acc_phase ^= 1u;
          }
        }
      } else {
        // Blockwise: each K block goes into a TMEM buffer on its own (no
        // carry-in).  The stage's release commit also tells the epilogue that
        // the K block's partial product is complete.  (Splitting a K block
        // into two N = 128 halves with their own hand-back costs twice the
        // MMA instructions and commits, and the single issuing thread, not
        // the tensor core, then sets the pace.)
        KGroupCursor kc;
        if constexpr (kKGroups) kc.init(p.offs);
        for (int64_t t = item0; t < total_tiles && ok; t += item_stride) {
          const int32_t nkb = kKGroups ? kgroup_coord(t, p, kc).nkb : KB;
          for (int32_t kb = 0; kb < nkb; ++kb) {
            if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort_flag, p.status,
                                  SITE_MMA_ACC_EMPTY, kWaitLimitNs)) {
              ok = false;
              break;
            }
            tc_fence_after_sync();
            if (!ready && !mbar_wait(&full[stage], phase, abort_flag, p.status,
                                            SITE_MMA_FULL, kWaitLimitNs)) {
              ok = false;
              break;
            }
            const uint32_t cur = stage;
            if (++stage == C::kStages) {
              stage = 0;
              phase ^= 1u;
            }
            ready = mbar_test_wait(&full[stage], phase);
            const uint32_t d = tmem_base + acc * BN;
            const uint64_t da = smem_desc_k_sw128(smem_u32(smem + C::kOffA + cur * C::kAStage));
            const uint64_t db = smem_desc_k_sw128(smem_u32(smem + C::kOffB + cur * C::kBStage));
#pragma unroll
            for (int k = 0; k < BK / UMMA_K; ++k)
              mma_e4m3(d, da + (k * UMMA_K) / 16, db + (k * UMMA_K) / 16, idesc_full, k > 0);
            mma_commit(&empty[cur]);
            acc ^= 1u;
            if (acc == 0) acc_phase ^= 1u;
          }
        }
      }
      // All MMAs issued by this thread complete before TMEM is released.
      mma_commit(drain);
    }
    if (lane == 0) {
      uint32_t dummy_abort = 0;
      mbar_wait(drain, 0, &dummy_abort, p.status, SITE_TEARDOWN, kWaitLimitNs);
    }
   } else if (warp == 2) {
    // ----------------------------------------------- blockwise scale producer
    // Fills the scale ring kSclSlots K blocks ahead of the epilogue, so the
    // epilogue never waits on a global load.  A K block's 128 row scales (and
    // 1x128_128x1's 256 column scales) are contiguous in global memory: one
    // bulk copy each (lane 0, counted in bytes on the slot's sfull barrier)
    // when they are 16-byte aligned and wholly inside the matrix (measured:
    // 1x128_128x128 1.5 % faster than 4-byte copies); otherwise, and for
    // 1x128_128x128's two column scales, cp.async with zero fill past the
    // matrix (lane l: rows l, l+32, l+64, l+96), each lane's copies arriving
    // on the slot's sfull barrier.
    if constexpr (kBlockwise) {
      const int64_t NB = (p.N + 127) / 128;
      uint32_t slot = 0, sphase = 0;
      bool ok = true;
      uint64_t issued = 0;
      GroupCursor cur;
      KGroupCursor kc;
      if constexpr (kKGroups) kc.init(p.offs);
      else if constexpr (kGrouped) cur.init(p.offs, kTM);
      const bool rows_aligned = (reinterpret_cast<uintptr_t>(p.sa) & 15u) == 0 && (p.M & 3) == 0;
      const bool cols_aligned = (reinterpret_cast<uintptr_t>(p.sb) & 15u) == 0 && (p.N & 3) == 0;
      for (int64_t t = item0; t < total_tiles && ok; t += item_stride) {
        const TileCoord c =
            kKGroups ? kgroup_coord(t, p, kc) : tile_coord<kGrouped, kTM, kRaster>(t, p, cur);
        const int32_t nkb = kKGroups ? c.nkb : KB;
        for (int32_t kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&sempty[slot], sphase ^ 1u, abort_flag, p.status, SITE_SCALE_EMPTY,
                         kWaitLimitNs)) {
            ok = false;
            break;
          }
          float* dst = scl + slot * kSclSlotFloats;
          // K-grouped: the group's padded K blocks index the scale rows
          const int64_t kbs = kKGroups ? c.kb0 + kb : kb;
          const float* sa_k = p.sa + kbs * p.M;
          const bool rows_bulk =
              rows_aligned && (c.m0 & 3) == 0 && static_cast<int64_t>(c.m0) + 128 <= p.M;
          const bool cols_bulk = kRecipe == kBlock1 && cols_aligned &&
                                 static_cast<int64_t>(c.n0) + 256 <= p.N;
          if (lane == 0) {
            const uint32_t bytes = (rows_bulk ? 512u : 0u) + (cols_bulk ? 1024u : 0u);
            mbar_arrive_expect_tx(&sfull[slot], bytes);
            if (rows_bulk) bulk_load_g2s(dst, sa_k + c.m0, 512, &sfull[slot]);
            if (cols_bulk) bulk_load_g2s(dst + 128, p.sb + kbs * p.N + c.n0, 1024, &sfull[slot]);
          }
          if (!rows_bulk) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int64_t r = static_cast<int64_t>(c.m0) + lane + 32 * i;
              cp_async_4(dst + lane + 32 * i, r < p.M ? sa_k + r : p.sa, r < p.M ? 4u : 0u);
            }
          }
          if constexpr (kRecipe == kBlock128) {
            if (lane < 2) {
              // grouped: expert g's scales, layout (E, K/128, ceil(N/128))
              const int64_t kbg = (kGrouped ? static_cast<int64_t>(c.g) * KB : 0) + kb;
              const bool v = static_cast<int64_t>(c.n0) + 128 * lane < p.N;
              cp_async_4(dst + 128 + lane,
                         v ? p.sb + kbg * NB + c.n0 / 128 + lane : p.sb,
                         v ? 4u : 0u);
            }
          } else if (!cols_bulk) {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const int64_t n = static_cast<int64_t>(c.n0) + 8 * lane + 4 * i;
              cp_async_16(dst + 128 + 8 * lane + 4 * i,
                          n < p.N ? p.sb + kbs * p.N + n : p.sb,
                          n < p.N ? 16u : 0u);
            }
          }
          cp_async_mbar_arrive_noinc(&sfull[slot]);
          ++issued;
          if (++slot == kSclSlots) {
            slot = 0;
            sphase ^= 1u;
          }
        }
      }
      cp_async_wait_all();  // nothing lands in shared memory after the CTA exits
      // nor do the bulk copies: wait (bounded) for the last slots' copies,
      // which the epilogue may not have consumed if it stopped early
      // (otherwise these phases are complete and the waits return at once)
      const uint64_t first = issued > kSclSlots ? issued - kSclSlots : 0;
      for (uint64_t i = first; i < issued; ++i) {
        uint32_t dummy_abort = 0;
        mbar_wait(&sfull[i % kSclSlots], static_cast<uint32_t>((i / kSclSlots) & 1u),
                  &dummy_abort, nullptr, SITE_TEARDOWN, 10000000ull);
      }
    } else if constexpr (kMxGather) {
      // ------------------------------------- grouped MXFP8: A scale gather
      // For each stage, in the producer's order: the tile's 128 rows' four
      // scale bytes of this K tile (one word per row, read from A's
      // scale-factor tiles at the row's own position) are copied into the
      // stage's A slot at row r's position ((r % 32) * 16 + (r / 32) * 4) by
      // 4-byte cp.async (zero fill past the matrix); each lane's copies then
      // arrive on the stage's full barrier when they land
      // (cp.async.mbarrier.arrive.noinc), so the warp never waits for them.
      // The MMA thread fences them into the async proxy before tcgen05.cp.
      GroupCursor cur;
      cur.init(p.offs, kTM);
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      for (int64_t t = item0; t < total_tiles && ok; t += item_stride) {
        const TileCoord c = tile_coord<kGrouped, kTM, kRaster>(t, p, cur);
        for (int32_t kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status, SITE_SCALE_EMPTY,
                         kWaitLimitNs)) {
            ok = false;
            break;
          }
          uint8_t* slot = smem + C::kOffScl + stage * kMxSfStage;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t r = lane + 32u * j;
            const int64_t row = static_cast<int64_t>(c.m0) + r;
            const int64_t r7 = row & 127;
            const int64_t off = ((row >> 7) * KB + kb) * kMxSfTile + (r7 & 31) * 16 + (r7 >> 5) * 4;
            const bool in = row < p.M && off >= 0 && off + 4 <= p.sfa_bytes;
            cp_async_4(slot + (r & 31u) * 16 + (r >> 5) * 4, in ? p.sfa + off : p.sfa, in ? 4u : 0u);
          }
          cp_async_mbar_arrive_noinc(&full[stage]);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      cp_async_wait_all();  // nothing lands in shared memory after the CTA exits
    }
   }
  } else {
    // --------------------------------------------------------- epilogue
    if constexpr (kBigEpi) warpgroup_reg_alloc<kRegsHigh>();
    const uint32_t ew = warp - kFirstEpiWarp;  // 0..7
    const uint32_t q = warp & 3u;          // TMEM lane quarter of this warp
    const uint32_t half = ew >> 2;         // which 128 columns of the tile
    uint8_t* ebuf = smem + C::kOffEpi + ew * C::kEpiBufs * kEpiBuf;
    uint32_t nbox = 0;  // boxes this warp has staged
    const uint32_t lane_base = (q * 32u) << 16;
    GroupCursor cur;
    KGroupCursor kc;
    if constexpr (kKGroups) kc.init(p.offs);
    else if constexpr (kGrouped) cur.init(p.offs, kTM);
    uint32_t acc = 0, acc_phase = 0;
    uint32_t ep_stage = 0, ep_phase = 0;  // blockwise: mirrors the MMA's stage sequence
    uint32_t sslot = 0, sphase = 0;       // blockwise: scale ring position
    // blockwise: wait until the scale ring holds this K block's scales
    auto wait_scales = [&]() -> const float* {
      if (!mbar_wait(&sfull[sslot], sphase, abort_flag, p.status, SITE_EPI_SCALE_FULL,
                     kWaitLimitNs))
        return nullptr;
      return scl + sslot * kSclSlotFloats;
    };
    // ... and hand the slot back once every lane has read it
    auto release_scales = [&]() {
      __syncwarp();
      if (lane == 0) mbar_arrive(&sempty[sslot]);
      if (++sslot == kSclSlots) {
        sslot = 0;
        sphase ^= 1u;
      }
    };
    bool ok = true;
    auto release_acc = [&](uint32_t a) { mbar_arrive(&acc_empty[a]); };
    for (int64_t t = item0; t < total_tiles && ok; t += item_stride) {
      const TileCoord c =
          kKGroups ? kgroup_coord(t, p, kc) : tile_coord<kGrouped, kTM, kRaster>(t, p, cur);
      // the tile's output rows (K-grouped: group g's block of the output)
      const int32_t cta_m0 = c.out_m0;
      const int64_t row = static_cast<int64_t>(cta_m0) + q * 32 + lane;
      const bool row_ok = row < c.row_end;
      const int64_t ncol0 = static_cast<int64_t>(c.n0) + half * 128;
      const int32_t row0 = cta_m0 + static_cast<int32_t>(q * 32);
      const int32_t nkb = kKGroups ? c.nkb : KB;

      // next accumulator buffer (MXFP8: the one buffer, next phase)
      auto next_acc = [&]() {
        if constexpr (kIsMx) {
          acc_phase ^= 1u;
        } else {
          acc ^= 1u;
          if (acc == 0) acc_phase ^= 1u;
        }
      };
      if constexpr (!kBlockwise) {
        if (!mbar_wait(&acc_full[acc], acc_phase, abort_flag, p.status,
                       SITE_EPI_ACC_FULL, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        if (c.half_n && half == 1) {
          // 128-wide item: this warp's columns are not part of it
          __syncwarp();
          if (lane == 0) release_acc(acc);
          next_acc();
          continue;
        }
        if constexpr (kIsMx) {
          // scales were applied by the MMA: read the whole row slice, hand
          // the buffer back, then add bias and store
          const uint32_t tcol = tmem_base + lane_base + half * 128;
          uint32_t r[4][32];
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) tmem_ld_32x32b_x32(tcol + cc * 32, r[cc]);
          tmem_ld_wait();
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) release_acc(0);
          if constexpr (!kOutMxq) {
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              const int64_t n = ncol0 + cc * 32;
              float v[32];
              load_bias32(p.bias, n, p.N, v);
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = __fadd_rn(__uint_as_float(r[cc][i]), v[i]);
              store_cols32<kOutF32, kStore, C::kEpiBufs>(ebuf, nbox, v, &tm_out, static_cast<int32_t>(n), row0,
                                              c.row_end, p.out, p.N, lane);
            }
          } else {
            // MXFP8 output: the thread's 128 columns are four 32-wide blocks
            // of its row.  Per block: e = floor(log2(amax)) - 8 clamped to
            // [-127, 127] (from the bits of the fp32 amax), codes
            // e4m3_satfinite(v * 2^-e).  The four scale bytes leave as one
            // word of the output's scale-factor tiles (rows past M: zero).
            uint32_t sc = 0;
#pragma unroll
            for (int bx = 0; bx < 2; ++bx) {
              uint4 chunk[4];
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int cc = 2 * bx + h;
                float v[32];
                load_bias32(p.bias, ncol0 + cc * 32, p.N, v);
                float am = 0.0f;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                  v[i] = __fadd_rn(__uint_as_float(r[cc][i]), v[i]);
                  am = fmaxf(am, fabsf(v[i]));
                }
                const int e = max(static_cast<int>(__float_as_uint(am) >> 23) - 127 - 8, -127);
                const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
                sc |= static_cast<uint32_t>(e + 127) << (8 * cc);
                uint32_t* w = reinterpret_cast<uint32_t*>(&chunk[2 * h]);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                  w[j] = cast_f32x2(v[4 * j], v[4 * j + 1], inv) |
                         (cast_f32x2(v[4 * j + 2], v[4 * j + 3], inv) << 16);
              }
              store_box64<kStore, C::kEpiBufs>(ebuf, nbox, chunk, &tm_out, static_cast<int32_t>(ncol0 + 64 * bx),
                                    row0, c.row_end, static_cast<uint8_t*>(p.out), p.N, 1, lane);
            }
            if (ncol0 < p.N) {
              const int64_t r7 = row & 127;
              uint8_t* tiles = reinterpret_cast<uint8_t*>(p.out_scales);
              const int64_t off = ((row >> 7) * (p.N / 128) + ncol0 / 128) * kMxSfTile +
                                  (r7 & 31) * 16 + (r7 >> 5) * 4;
              *reinterpret_cast<uint32_t*>(tiles + off) = row_ok ? sc : 0u;
            }
          }
          next_acc();
          continue;
        }
        float sa;
        if constexpr (kRecipe == kTensor) sa = __ldg(p.sa) * __ldg(p.sb);
        else sa = row_ok ? __ldg(p.sa + row) : 0.0f;
        const float* sbg = p.sb + (kGrouped ? static_cast<int64_t>(c.g) * p.N : 0);
        const uint32_t tcol = tmem_base + lane_base + acc * BN + half * 128;
        // the fp32 results of 32-column chunk cc of this thread's row
        auto values32 = [&](int cc, float (&v)[32]) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tcol + cc * 32, r);
          tmem_ld_wait();
          const int64_t n = ncol0 + cc * 32;
          float bias[32];
          load_bias32(p.bias, n, p.N, bias);
          if constexpr (kRecipe == kTensor) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              v[i] = fmaf(__uint_as_float(r[i]), sa, bias[i]);
          } else {
            float sb[32];
            load_cols32_f32(sbg, n, p.N, sb);
#pragma unroll
            for (int i = 0; i < 32; ++i)
              v[i] = fmaf(__uint_as_float(r[i]), sa * sb[i], bias[i]);
          }
        };
        auto release_buf = [&]() {
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) release_acc(acc);
        };
        if constexpr (!kOutQ) {
#pragma unroll 1
          for (int cc = 0; cc < 4; ++cc) {
            float v[32];
            values32(cc, v);
            if (cc == 3) release_buf();
            store_cols32<kOutF32, kStore, C::kEpiBufs>(ebuf, nbox, v, &tm_out,
                                            static_cast<int32_t>(ncol0 + cc * 32), row0,
                                            c.row_end, p.out, p.N, lane);
          }
        } else {
          // e4m3 output in 1x128 groups along n: the group is this thread's
          // 128 columns of its row.  Pass 1 finds its amax; pass 2 reads the
          // accumulators again (TMEM reads are cheap next to the MMAs),
          // recomputes the same fp32 values, casts and stores them.
          float am = 0.0f;
#pragma unroll 1
          for (int cc = 0; cc < 4; ++cc) {
            float v[32];
            values32(cc, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) am = fmaxf(am, fabsf(v[i]));
          }
          const ScalePair sp = scales_from_amax(am);
          if (row_ok && ncol0 < p.N) p.out_scales[(ncol0 / 128) * p.M + row] = sp.s;
#pragma unroll 1
          for (int bx = 0; bx < 2; ++bx) {
            uint4 chunk[4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              float v[32];
              values32(2 * bx + h, v);
              if (bx == 1 && h == 1) release_buf();
              uint32_t* w = reinterpret_cast<uint32_t*>(&chunk[2 * h]);
#pragma unroll
              for (int j = 0; j < 8; ++j)
                w[j] = cast_f32x2(v[4 * j], v[4 * j + 1], sp.inv) |
                       (cast_f32x2(v[4 * j + 2], v[4 * j + 3], sp.inv) << 16);
            }
            store_box64<kStore, C::kEpiBufs>(ebuf, nbox, chunk, &tm_out, static_cast<int32_t>(ncol0 + 64 * bx),
                                  row0, c.row_end, static_cast<uint8_t*>(p.out), p.N, 1, lane);
          }
        }
        next_acc();
      } else {
        // Blockwise: promote each K block's partial product into registers.
        // Warp (q, half) reads TMEM lanes 32q.. and the 128 columns of its
        // half of the tile, in the 32x32b shape (thread = one row, 32
        // consecutive columns per load; the 16x256b shape reads TMEM at about
        // a third of the rate).  The four 32-column loads are pipelined
        // against the FMAs: the next chunk is in flight while this one is
        // promoted.
        //   1x128_128x128: the half is one 128-column block of B, so the
        //     scale product sA[m,kb] * sB[nb,kb] is one value per thread.
        //   1x128_128x1: acc += (P * sB[n,kb]) * sA[m,kb] per column, the
        //     column scales read from the scale ring (the same address in
        //     every lane: a broadcast).
        float2 accr[64];  // accr[16 c + i]: columns 32c + 2i, 32c + 2i + 1 of the warp's 128
#pragma unroll
        for (int i = 0; i < 64; ++i) accr[i] = make_float2(0.0f, 0.0f);
        for (int32_t kb = 0; kb < nkb && ok; ++kb) {
          const float* sl = wait_scales();
          if (sl == nullptr) {
            ok = false;
            break;
          }
          const float sa = sl[q * 32 + lane];
          float f = sa;
          if constexpr (kRecipe == kBlock128) {
            f = sa * sl[128 + half];
            release_scales();
          }
          const float2 f2 = make_float2(f, f);
          const float* sbl = sl + 128 + half * 128;  // 1x128_128x1: this warp's column scales
          // the K block's MMAs are done when its stage is released
          if (!mbar_wait(&empty[ep_stage], ep_phase, abort_flag, p.status, SITE_EPI_ACC_FULL,
                         kWaitLimitNs)) {
            ok = false;
            break;
          }
          if (++ep_stage == C::kStages) {
            ep_stage = 0;
            ep_phase ^= 1u;
          }
          tc_fence_after_sync();
          const uint32_t tcol = tmem_base + lane_base + acc * BN + half * 128;
          uint32_t r[2][32];
          tmem_ld_32x32b_x32(tcol, r[0]);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            if (c < 3) tmem_ld_32x32b_x32(tcol + 32 * (c + 1), r[(c + 1) & 1]);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float2 pv = make_float2(__uint_as_float(r[c & 1][2 * i]),
                                      __uint_as_float(r[c & 1][2 * i + 1]));
              if constexpr (kRecipe == kBlock1)
                pv = mul2(pv, *reinterpret_cast<const float2*>(sbl + 32 * c + 2 * i));
              accr[16 * c + i] = fma2(pv, f2, accr[16 * c + i]);
            }
            if (c < 3) tmem_ld_wait();
            if (c == 2) {
              // every TMEM read of this buffer is done: hand it back
              tc_fence_before_sync();
              __syncwarp();
              if (lane == 0) mbar_arrive(&acc_empty[acc]);
            }
          }
          if constexpr (kRecipe == kBlock1) release_scales();
          acc ^= 1u;
          if (acc == 0) acc_phase ^= 1u;
        }
        if (!ok) break;
        // the bias joins the accumulators once (one fp32 add per element),
        // so the output passes below read registers only
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          float bv[32];
          load_bias32(p.bias, ncol0 + cc * 32, p.N, bv);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            accr[cc * 16 + i].x += bv[2 * i];
            accr[cc * 16 + i].y += bv[2 * i + 1];
          }
        }
        // the tile's fp32 results for chunk cc (bias added)
        auto result32 = [&](int cc, float (&v)[32]) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            v[2 * i] = accr[cc * 16 + i].x;
            v[2 * i + 1] = accr[cc * 16 + i].y;
          }
        };
        if constexpr (!kOutQ) {
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            float v[32];
            result32(cc, v);
            store_cols32<kOutF32, kStore, C::kEpiBufs>(ebuf, nbox, v, &tm_out,
                                            static_cast<int32_t>(ncol0 + cc * 32), row0,
                                            c.row_end, p.out, p.N, lane);
          }
        } else {
          // e4m3 output in 1x128 groups along n (this thread's 128 columns).
          // The dual kind also writes the result transposed, where the
          // tile's 128 rows of each column form one 1x128 group along m:
          // the column maxima of the half's four warps meet in shared memory
          // (two bounded mbarrier meetings per tile), and each warp's codes
          // for 16 columns x 32 rows pass through its own 512-byte buffer.
          float am = 0.0f;
          [[maybe_unused]] uint32_t cmax[4];  // lane L: column 32 cc + L, max over the warp's rows
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            float v[32];
            result32(cc, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) am = fmaxf(am, fabsf(v[i]));
            if constexpr (kOutQT) {
              // |v| as bits orders like the values
              uint32_t mine = 0u;
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(fabsf(v[i])));
                mine = lane == static_cast<uint32_t>(i) ? m : mine;
              }
              cmax[cc] = mine;
            }
          }
          const ScalePair sp = scales_from_amax(am);
          if (row_ok && ncol0 < p.N) p.out_scales[(ncol0 / 128) * p.M + row] = sp.s;
          [[maybe_unused]] float tinv[4];  // lane L: 1 / scale of column 32 cc + L
          uint8_t* const tbuf = smem + C::kOffTpos + ew * kTposBuf;
          if constexpr (kOutQT) {
            // A tile makes two meetings on hsync[half], so the phase is 0 at
            // the start of every tile.
            uint32_t hphase = 0;
            auto half_sync = [&]() -> bool {
              __syncwarp();
              uint64_t* const hb = &hsync[half];
              if (lane == 0) mbar_arrive(hb);
              const bool done = mbar_wait(hb, hphase, abort_flag, p.status, SITE_EPI_ACC_FULL,
                                          kWaitLimitNs);
              hphase ^= 1u;
              return done;
            };
#pragma unroll
            for (int cc = 0; cc < 4; ++cc)
              reinterpret_cast<uint32_t*>(tbuf)[cc * 32 + lane] = cmax[cc];
            if (!half_sync()) {
              ok = false;
              break;
            }
            const uint8_t* const half_t = smem + C::kOffTpos + half * 4 * kTposBuf;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              uint32_t mx = 0u;
#pragma unroll
              for (int w = 0; w < 4; ++w)
                mx = max(mx, reinterpret_cast<const uint32_t*>(half_t + w * kTposBuf)[cc * 32 + lane]);
              const ScalePair tp = scales_from_amax(__uint_as_float(mx));
              tinv[cc] = tp.inv;
              const int64_t n = ncol0 + 32 * cc + lane;
              if (q == 0 && n < p.N) p.out_t_scales[(cta_m0 / 128) * p.N + n] = tp.s;
            }
            if (!half_sync()) {  // every warp has read the maxima
              ok = false;
              break;
            }
          }
#pragma unroll
          for (int bx = 0; bx < 2; ++bx) {
            uint4 chunk[4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int cc = 2 * bx + h;
              float v[32];
              result32(cc, v);
              uint32_t* w = reinterpret_cast<uint32_t*>(&chunk[2 * h]);
#pragma unroll
              for (int j = 0; j < 8; ++j)
                w[j] = cast_f32x2(v[4 * j], v[4 * j + 1], sp.inv) |
                       (cast_f32x2(v[4 * j + 2], v[4 * j + 3], sp.inv) << 16);
              if constexpr (kOutQT) {
#pragma unroll
                for (int rd = 0; rd < 2; ++rd) {
                  // columns 32 cc + 16 rd + i: byte (i, lane) of the buffer
#pragma unroll
                  for (int i = 0; i < 16; i += 2) {
                    const int col = 16 * rd + i;
                    const float i0 = __shfl_sync(0xFFFFFFFFu, tinv[cc], col);
                    const float i1 = __shfl_sync(0xFFFFFFFFu, tinv[cc], col + 1);
                    const uint32_t two = static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(
                        make_float2(__fmul_rn(v[col], i0), __fmul_rn(v[col + 1], i1)),
                        __NV_SATFINITE, __NV_E4M3));
                    tbuf[i * 32 + lane] = static_cast<uint8_t>(two & 0xFFu);
                    tbuf[(i + 1) * 32 + lane] = static_cast<uint8_t>(two >> 8);
                  }
                  __syncwarp();
                  // lane L: 16 of the 32 rows of column L / 2
                  const uint4 u =
                      *reinterpret_cast<const uint4*>(tbuf + (lane >> 1) * 32 + 16 * (lane & 1));
                  const int64_t n = ncol0 + 32 * cc + 16 * rd + (lane >> 1);
                  if (n < p.N)
                    *reinterpret_cast<uint4*>(p.out_t + n * p.M + row0 + 16 * (lane & 1)) = u;
                  __syncwarp();
                }
              }
            }
            store_box64<kStore, C::kEpiBufs>(ebuf, nbox, chunk, &tm_out, static_cast<int32_t>(ncol0 + 64 * bx),
                                  row0, c.row_end, static_cast<uint8_t*>(p.out), p.N, 1, lane);
          }
        }
      }
    }
    if (lane == 0) bulk_wait_group0();
    __syncwarp();
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// out[m, n] = bias[n] (or 0) for K == 0.
template <bool kOutF32>
__global__ void fill_bias_kernel(const uint16_t* bias, int64_t M, int64_t N,
                                 void* out) {
  const int64_t total = M * N;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
       i < total; i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float v = bias ? __uint_as_float(static_cast<uint32_t>(bias[i % N]) << 16) : 0.0f;
    if constexpr (kOutF32) static_cast<float*>(out)[i] = v;
    else static_cast<uint16_t*>(out)[i] = static_cast<uint16_t>(pack_bf16x2(v, 0.0f) & 0xFFFFu);
  }
}

// One CTA waits on a barrier nothing completes: exercises the bounded wait.
__global__ void timeout_probe_kernel(uint64_t limit_ns, uint32_t* status) {
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0)
    mbar_wait(&bar, 0, &abort_flag, status, SITE_PROBE, limit_ns);
  __syncthreads();
}

// ------------------------------------------------------------ host side

template <int kRecipe, int kOut, bool kGrouped>
cudaError_t launch_kernel(const CUtensorMap& ta, const CUtensorMap& tb,
                          const CUtensorMap& tbh, const CUtensorMap& to,
                          const GemmParams& p, unsigned grid, const LaunchCtx& ctx) {
  constexpr bool kBlockwise = kRecipe == kBlock128 || kRecipe == kBlock1;
  constexpr bool kBigEpi = kBlockwise;
  if constexpr (kRecipe == kMxfp8 && (kOut == kOutE4M3 || (kGrouped && kOut == kOutMx))) {
    return cudaErrorInvalidValue;  // MXFP8: bf16/fp32 out (dense: also MXFP8)
  } else if constexpr (kOut == kOutMx && kRecipe != kMxfp8) {
    return cudaErrorInvalidValue;  // MXFP8 output from the MXFP8 GEMM only
  } else if constexpr (kOut == kOutE4M3Dual && (kRecipe != kBlock128 || kGrouped)) {
    return cudaErrorInvalidValue;  // dual e4m3 output: dense 1x128_128x128 only
  } else if constexpr (kOut == kOutE4M3 && kGrouped) {
    return cudaErrorInvalidValue;  // quantized output: dense GEMM only
  } else {
    auto kern = fp8_gemm_kernel<kRecipe, kOut, kGrouped>;
    using Cfg = CfgT<staged_epilogue(kRecipe, kOut)>;
    // the dynamic shared-memory opt-in, once per device
    static std::atomic<bool> done[kMaxDevices];
    static std::mutex mu;
    cudaError_t e = once_per_device(done, mu, ctx.device, [&] {
      cudaError_t r = cudaFuncSetAttribute(
          kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
      if (r != cudaSuccess) return r;
      if (kBigEpi) {
        // setmaxnreg.inc would wait forever if the launch allocation were
        // smaller than the split assumes: check before the first launch.
        cudaFuncAttributes attr;
        r = cudaFuncGetAttributes(&attr, kern);
        if (r != cudaSuccess) return r;
        if (attr.numRegs < static_cast<int>(kRegsAtLaunch)) return cudaErrorInvalidConfiguration;
      }
      return cudaSuccess;
    });
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, Cfg::kSmemBytes, ctx.stream>>>(ta, tb, tbh, to, p);
    return cudaGetLastError();
  }
}

template <bool kGrouped>
cudaError_t dispatch(int recipe, int out_kind, const CUtensorMap& ta, const CUtensorMap& tb,
                     const CUtensorMap& tbh, const CUtensorMap& to, const GemmParams& p,
                     unsigned grid, const LaunchCtx& ctx) {
#define FP8SM_CASE(R)                                                              \
  if (recipe == R) {                                                               \
    switch (out_kind) {                                                            \
      case kOutBf16: return launch_kernel<R, kOutBf16, kGrouped>(ta, tb, tbh, to, p, grid, ctx); \
      case kOutFp32: return launch_kernel<R, kOutFp32, kGrouped>(ta, tb, tbh, to, p, grid, ctx); \
      case kOutE4M3: return launch_kernel<R, kOutE4M3, kGrouped>(ta, tb, tbh, to, p, grid, ctx); \
      case kOutMx: return launch_kernel<R, kOutMx, kGrouped>(ta, tb, tbh, to, p, grid, ctx);     \
      case kOutE4M3Dual:                                                           \
        return launch_kernel<R, kOutE4M3Dual, kGrouped>(ta, tb, tbh, to, p, grid, ctx);          \
      default: return cudaErrorInvalidValue;                                       \
    }                                                                              \
  }
  if constexpr (kGrouped) {
    FP8SM_CASE(kRow)
    FP8SM_CASE(kBlock128)
    FP8SM_CASE(kBlock1)  // K-grouped: the per-expert weight gradient
    FP8SM_CASE(kMxfp8)
  } else {
    FP8SM_CASE(kTensor)
    FP8SM_CASE(kRow)
    FP8SM_CASE(kBlock128)
    FP8SM_CASE(kBlock1)
    FP8SM_CASE(kMxfp8)
  }
#undef FP8SM_CASE
  return cudaErrorInvalidValue;
}

// Output map: 32-row x 64-byte boxes, 64-byte swizzle (the epilogue's
// staging layout) for bf16, fp32 or e4m3 output.
bool out_map(CUtensorMap* m, void* out, int64_t rows, int64_t N, int out_kind,
             std::string* err) {
  const bool q8 = out_kind == kOutE4M3 || out_kind == kOutMx || out_kind == kOutE4M3Dual;
  const uint64_t eb = out_kind == kOutFp32 ? 4 : q8 ? 1 : 2;
  uint64_t dims[2] = {static_cast<uint64_t>(N), static_cast<uint64_t>(rows)};
  uint64_t strides[1] = {static_cast<uint64_t>(N) * eb};
  uint32_t box[2] = {static_cast<uint32_t>(64 / eb), 32};
  const CUtensorMapDataType dt = out_kind == kOutFp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                 : q8                 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                                      : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  return make_tmap(m, dt, 2, out, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_64B, err);
}

// A operand map: 128-row boxes (one CTA's rows) in both modes.
bool a_map(CUtensorMap* m, const void* a, int64_t rows, int64_t K, std::string* err) {
  uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(rows)};
  uint64_t strides[1] = {static_cast<uint64_t>(K)};
  uint32_t box[2] = {BK, BM};
  return make_tmap(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a, dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B, err);
}

}  // namespace

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr,
                                cudaEnableDefault, &qres) == cudaSuccess &&
        qres == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// Tiled tensor map (no interleave, 256-byte L2 promotion, zero fill out of
// bounds); false with *err set when the driver refuses it.
bool make_tmap(CUtensorMap* m, CUtensorMapDataType dt, uint32_t rank,
               const void* base, const uint64_t* dims, const uint64_t* strides,
               const uint32_t* box, CUtensorMapSwizzle sw, std::string* err) {
  auto fn = encode_fn();
  if (!fn) {
    if (err) *err = "cuTensorMapEncodeTiled is not available from the driver";
    return false;
  }
  uint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, dt, rank, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    if (err) *err = "cuTensorMapEncodeTiled failed (code " + std::to_string((int)r) + ")";
    return false;
  }
  return true;
}

cudaError_t launch_scaled_mm(const void* a, const void* b, int64_t M,
                             int64_t N, int64_t K, const float* sa,
                             const float* sb, int recipe, const void* bias,
                             int out_kind, void* out, float* out_scales,
                             const LaunchCtx& ctx, void* out_t, float* out_t_scales) {
  if (M == 0 || N == 0) return cudaSuccess;
  if (K == 0 && (out_kind == kOutE4M3 || out_kind == kOutMx || out_kind == kOutE4M3Dual))
    return cudaErrorInvalidValue;
  const int out_f32 = out_kind == kOutFp32;
  if (K == 0) {
    const int64_t total = M * N;
    int64_t blocks = (total + 255) / 256;
    if (blocks > 65535) blocks = 65535;
    if (out_f32)
      fill_bias_kernel<true><<<(unsigned)blocks, 256, 0, ctx.stream>>>(
          static_cast<const uint16_t*>(bias), M, N, out);
    else
      fill_bias_kernel<false><<<(unsigned)blocks, 256, 0, ctx.stream>>>(
          static_cast<const uint16_t*>(bias), M, N, out);
    return cudaGetLastError();
  }
  const uint32_t b_rows = Cfg::kBRows;
  CUtensorMap ta, tb, tbh, to;
  if (!a_map(&ta, a, M, K, ctx.err)) return cudaErrorInvalidValue;
  {
    uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N)};
    uint64_t strides[1] = {static_cast<uint64_t>(K)};
    uint32_t box[2] = {BK, b_rows};
    if (!make_tmap(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, b, dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B, ctx.err))
      return cudaErrorInvalidValue;
    uint32_t box_half[2] = {BK, b_rows / 2};
    if (!make_tmap(&tbh, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, b, dims, strides, box_half,
                   CU_TENSOR_MAP_SWIZZLE_128B, ctx.err))
      return cudaErrorInvalidValue;
  }
  if (!out_map(&to, out, M, N, out_kind, ctx.err)) return cudaErrorInvalidValue;
  GemmParams p{};
  p.out_scales = out_scales;
  p.out_t = static_cast<uint8_t*>(out_t);
  p.out_t_scales = out_t_scales;
  p.M = M;
  p.N = N;
  p.K = K;
  if (recipe == kMxfp8) {
    // MXFP8: sa, sb carry the E8M0 scale-factor tiles
    p.sfa = reinterpret_cast<const uint8_t*>(sa);
    p.sfb = reinterpret_cast<const uint8_t*>(sb);
    p.sfa_bytes = static_cast<int64_t>(mx_scale_tile_bytes(M, K));
    p.sfb_bytes = static_cast<int64_t>(mx_scale_tile_bytes(N, K));
  } else {
    p.sa = sa;
    p.sb = sb;
  }
  p.bias = static_cast<const uint16_t*>(bias);
  p.out = out;
  p.offs = nullptr;
  p.E = 0;
  const int64_t tile_m = BM;
  p.n_tiles = static_cast<int32_t>((N + BN - 1) / BN);
  p.m_tiles = static_cast<int32_t>((M + tile_m - 1) / tile_m);
  p.k_blocks = static_cast<int32_t>((K + BK - 1) / BK);
  // Tile order: M-major keeps a band of A and all of B in L2 while B's codes
  // fit there comfortably; a larger B (the grad_weight shapes, K = tokens)
  // would be streamed from HBM once per wave, so the tiles go in bands of 16
  // M tiles instead, N-major inside a band: a wave then reads a band of A
  // and a slice of B, both L2-resident.
  p.raster_m = (N * K > (int64_t(64) << 20)) ? 16 : 0;
  p.status = ctx.status;
  const int64_t tiles = static_cast<int64_t>(p.n_tiles) * p.m_tiles;
  const int64_t G = ctx.num_sms;  // resident CTAs (one per SM)
  p.split_start = tiles;
  p.total_items = tiles;
  const bool blockwise = recipe == kBlock128 || recipe == kBlock1;
  if (!blockwise) {
    const int64_t waves = (tiles + G - 1) / G;
    const int64_t last = tiles - (waves - 1) * G;  // tiles in the last wave
    if (2 * last <= G) {
      p.split_start = (waves - 1) * G;
      p.total_items = p.split_start + 2 * last;
    }
  }
  const int64_t units = p.total_items < G ? p.total_items : G;
  const unsigned grid = static_cast<unsigned>(units);
  return dispatch<false>(recipe, out_kind, ta, tb, tbh, to, p, grid, ctx);
}

cudaError_t launch_grouped_scaled_mm(const void* a, const void* b,
                                     int64_t M_total, int64_t N, int64_t K,
                                     int32_t E, const float* sa,
                                     const float* sb, const int32_t* offs,
                                     int recipe, int out_f32, void* out,
                                     const LaunchCtx& ctx) {
  if (M_total == 0 || N == 0) return cudaSuccess;
  if (K == 0)
    return launch_scaled_mm(nullptr, nullptr, M_total, N, 0, nullptr, nullptr,
                            1, nullptr, out_f32 ? kOutFp32 : kOutBf16, out, nullptr, ctx);
  const uint32_t b_rows = Cfg::kBRows;
  CUtensorMap ta, tb, to;
  if (!a_map(&ta, a, M_total, K, ctx.err)) return cudaErrorInvalidValue;
  {
    uint64_t dims[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N),
                        static_cast<uint64_t>(E)};
    uint64_t strides[2] = {static_cast<uint64_t>(K),
                           static_cast<uint64_t>(N) * static_cast<uint64_t>(K)};
    uint32_t box[3] = {BK, b_rows, 1};
    if (!make_tmap(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, b, dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B, ctx.err))
      return cudaErrorInvalidValue;
  }
  // Output map over all M_total rows: boxes wholly inside a group leave by
  // TMA store, the box that crosses a group's end by masked stores.
  if (!out_map(&to, out, M_total, N, out_f32 ? kOutFp32 : kOutBf16, ctx.err))
    return cudaErrorInvalidValue;
  GemmParams p{};
  p.M = M_total;
  p.N = N;
  p.K = K;
  if (recipe == kMxfp8) {
    p.sfa = reinterpret_cast<const uint8_t*>(sa);
    p.sfb = reinterpret_cast<const uint8_t*>(sb);
    p.sfa_bytes = static_cast<int64_t>(mx_scale_tile_bytes(M_total, K));
    p.sfb_bytes = static_cast<int64_t>(E) * static_cast<int64_t>(mx_scale_tile_bytes(N, K));
  } else {
    p.sa = sa;
    p.sb = sb;
  }
  p.bias = nullptr;
  p.out = out;
  p.offs = offs;
  p.E = E;
  p.n_tiles = static_cast<int32_t>((N + BN - 1) / BN);
  p.m_tiles = 0;
  p.k_blocks = static_cast<int32_t>((K + BK - 1) / BK);
  p.status = ctx.status;
  p.split_start = INT64_MAX;
  p.total_items = 0;
  const unsigned grid = static_cast<unsigned>(ctx.num_sms);
  return dispatch<true>(recipe, out_f32, ta, tb, tb, to, p, grid, ctx);
}

cudaError_t launch_grouped_wgrad(const void* a_t, const void* b_t, int64_t M, int64_t N,
                                 int64_t P, int64_t tokens, int32_t E, const float* sa,
                                 const float* sb, const int32_t* offs, int out_f32, void* out,
                                 const LaunchCtx& ctx) {
  if (M == 0 || N == 0) return cudaSuccess;
  CUtensorMap ta, tb, to;
  if (!a_map(&ta, a_t, M, P, ctx.err)) return cudaErrorInvalidValue;
  {
    uint64_t dims[2] = {static_cast<uint64_t>(P), static_cast<uint64_t>(N)};
    uint64_t strides[1] = {static_cast<uint64_t>(P)};
    uint32_t box[2] = {BK, Cfg::kBRows};
    if (!make_tmap(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, b_t, dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B, ctx.err))
      return cudaErrorInvalidValue;
  }
  // output (E * M, N): every tile is whole and leaves by TMA store
  if (!out_map(&to, out, static_cast<int64_t>(E) * M, N, out_f32 ? kOutFp32 : kOutBf16, ctx.err))
    return cudaErrorInvalidValue;
  GemmParams p{};
  p.M = M;
  p.N = N;
  p.K = P;
  p.sa = sa;
  p.sb = sb;
  p.bias = nullptr;
  p.out = out;
  p.offs = offs;
  p.E = E;
  p.tokens = tokens;
  p.n_tiles = static_cast<int32_t>((N + BN - 1) / BN);
  p.m_tiles = static_cast<int32_t>(M / BM);
  p.k_blocks = static_cast<int32_t>(P / BK);
  p.status = ctx.status;
  p.split_start = INT64_MAX;
  p.total_items = 0;
  const int64_t items = static_cast<int64_t>(E) * p.m_tiles * p.n_tiles;
  const unsigned grid = static_cast<unsigned>(items < ctx.num_sms ? items : ctx.num_sms);
  return dispatch<true>(kBlock1, out_f32, ta, tb, tb, to, p, grid, ctx);
}

cudaError_t launch_timeout_probe(uint32_t limit_us, const LaunchCtx& ctx) {
  timeout_probe_kernel<<<1, 32, 0, ctx.stream>>>(
      static_cast<uint64_t>(limit_us) * 1000ull, ctx.status);
  return cudaGetLastError();
}

}  // namespace fp8sm
