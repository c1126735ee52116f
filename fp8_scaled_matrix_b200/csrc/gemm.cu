// FP8 (e4m3) scaled GEMM on the 5th-generation tensor cores (sm_100a).
//
//   out[m, n] = sum_k (A[m,k] sA) (B[n,k] sB) (+ bias[n])
//
// "Fix: Handle LowLevelZeroPlugin with use_fp8=True" (Solution, forward pass)
// fixes what is computed: the scaled matmul equals dequantize-then-matmul plus
// bias.  Recipes: tensorwise and rowwise ("Add _scaled_mm_v2 API"),
// blockwise 1x128_128x128 and 1x128_128x1 ("improve fp8 blockwise gemm
// perf"), and the grouped rowwise MoE form over (E, N, K) experts with
// cumulative offs ("Add _grouped_mm dispatch handler to Float8Tensor").
//
// One persistent kernel, one CTA per SM, 10 warps with fixed roles:
//   warp 0      TMA producer: A (128 x 128 B) and B (256 x 128 B) tiles into
//               a 4-stage shared-memory ring (128-byte swizzle)
//   warp 1      TMEM owner + MMA issuer: one thread issues
//               tcgen05.mma.kind::f8f6f4 (M=128, N=256, K=32) x 4 per stage
//               into fp32 TMEM accumulators; tcgen05.commit frees stages
//   warps 2-9   epilogue: warp w reads TMEM lanes 32*(w%4).. (the hardware's
//               lane quarter) and columns 128*((w-2)/4).. of each tile
// TMEM holds two 256-column fp32 buffers.  Tensorwise / rowwise: each buffer
// is one whole tile's accumulator, so the epilogue of tile i overlaps the
// MMAs of tile i+1.  Blockwise: each 128-wide K block is accumulated into a
// buffer on its own (no carry-in), and the epilogue warps promote it --
// acc += partial * sA[m,kb] * sB[.,kb] -- into fp32 registers while the tensor
// core fills the other buffer.  Results are scaled, biased, rounded to bf16
// (or kept fp32), staged in shared memory and written by TMA stores (the
// grouped kernel masks rows past its group with plain 16-byte stores).
//
// Every wait is bounded (one second); a wait that gives up records
// FP8_ERR_TIMEOUT in the device status word, the CTA drains its in-flight
// copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include "internal.h"
#include "sm100.cuh"

namespace fp8sm {
namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;  // bytes == e4m3 elements per stage along K
constexpr int UMMA_K = 32;
constexpr int STAGES = 4;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kTmemCols = 512;  // two 256-column fp32 buffers
constexpr uint32_t kAStage = BM * BK;
constexpr uint32_t kBStage = BN * BK;
constexpr uint32_t kEpiBuf = 32 * 64;  // 32 rows x 64 bytes, 64-byte swizzle
constexpr uint32_t kSbBuf = 128 * 4;   // 128 fp32 column scales per warp

constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffB = kOffA + STAGES * kAStage;
constexpr uint32_t kOffEpi = kOffB + STAGES * kBStage;
constexpr uint32_t kOffSb = kOffEpi + kEpiWarps * kEpiBuf;
constexpr uint32_t kOffBar = kOffSb + kEpiWarps * kSbBuf;
// barriers: full[STAGES], empty[STAGES], acc_full[2], acc_empty[2], drain
constexpr uint32_t kNumBars = 2 * STAGES + 5;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kSmemUsed = kOffMisc + 16;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;  // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget");

enum Recipe : int { kTensor = 0, kRow = 1, kBlock128 = 2, kBlock1 = 3 };

struct GemmParams {
  int64_t M, N, K;
  const float* sa;
  const float* sb;
  const uint16_t* bias;
  void* out;
  const int32_t* offs;
  int32_t E;
  int32_t n_tiles;   // tiles along N
  int32_t m_tiles;   // tiles along M (dense)
  int32_t k_blocks;
  uint32_t* status;
};

// Walks the concatenated per-group M tiles in increasing order.
struct GroupCursor {
  int32_t g;
  int64_t tiles_before;  // M tiles of groups < g
  int64_t row_start;
  int64_t row_end;
  int64_t m_tiles;  // M tiles of group g
  __device__ void init(const int32_t* offs) {
    g = 0;
    tiles_before = 0;
    row_start = 0;
    row_end = offs[0];
    m_tiles = (row_end + BM - 1) / BM;
  }
  __device__ void seek(int64_t mt, const int32_t* offs, int32_t E) {
    while (mt >= tiles_before + m_tiles && g + 1 < E) {
      tiles_before += m_tiles;
      ++g;
      row_start = row_end;
      row_end = offs[g];
      m_tiles = (row_end - row_start + BM - 1) / BM;
    }
  }
};

struct TileCoord {
  int32_t m0, n0, g;
  int64_t row_end;
};

template <bool kGrouped>
__device__ __forceinline__ TileCoord tile_coord(int64_t t, const GemmParams& p,
                                                GroupCursor& cur) {
  TileCoord c;
  const int64_t mt = t / p.n_tiles;
  c.n0 = static_cast<int32_t>((t % p.n_tiles) * BN);
  if constexpr (kGrouped) {
    cur.seek(mt, p.offs, p.E);
    c.g = cur.g;
    c.m0 = static_cast<int32_t>(cur.row_start + (mt - cur.tiles_before) * BM);
    c.row_end = cur.row_end;
  } else {
    c.g = 0;
    c.m0 = static_cast<int32_t>(mt * BM);
    c.row_end = p.M;
  }
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
// then write the 32 x 64-byte box to global memory: by TMA store for the
// dense kernel, by masked 16-byte stores for the grouped kernel.
template <bool kGrouped>
__device__ __forceinline__ void store_box64(
    uint8_t* buf, const uint4 (&chunk)[4], const CUtensorMap* tm_out,
    int32_t col0 /*elements*/, int32_t row0, int64_t row_end, uint8_t* out,
    int64_t N, uint32_t elem_bytes, uint32_t lane) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t slot = static_cast<uint32_t>(j) ^ ((lane >> 1) & 3u);
    *reinterpret_cast<uint4*>(buf + lane * 64 + slot * 16) = chunk[j];
  }
  if constexpr (!kGrouped) {
    fence_proxy_async_smem();
    __syncwarp();
    // Boxes wholly past the last row or column are skipped; partial boxes are
    // clipped by the TMA unit.
    if (lane == 0 && row0 < row_end && col0 < N) {
      tma_store_2d(tm_out, buf, col0, row0);
      bulk_commit_group();
      bulk_wait_group_read0();
    }
    __syncwarp();
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
template <bool kOutF32, bool kGrouped>
__device__ __forceinline__ void store_cols32(
    uint8_t* buf, const float (&v)[32], const CUtensorMap* tm_out, int32_t col0,
    int32_t row0, int64_t row_end, void* out, int64_t N, uint32_t lane) {
  if constexpr (!kOutF32) {
    uint4 c[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      c[j] = make_uint4(pack_bf16x2(v[8 * j + 0], v[8 * j + 1]),
                        pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                        pack_bf16x2(v[8 * j + 4], v[8 * j + 5]),
                        pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
    store_box64<kGrouped>(buf, c, tm_out, col0, row0, row_end,
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
      store_box64<kGrouped>(buf, c, tm_out, col0 + 16 * h, row0, row_end,
                            static_cast<uint8_t*>(out), N, 4, lane);
    }
  }
}

template <int kRecipe, bool kOutF32, bool kGrouped>
__global__ void __launch_bounds__(kThreads, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                    const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ CUtensorMap tm_out,
                    const GemmParams p) {
  constexpr bool kBlockwise = (kRecipe == kBlock128 || kRecipe == kBlock1);
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* acc_full = bars + 2 * STAGES;
  uint64_t* acc_empty = bars + 2 * STAGES + 2;
  uint64_t* drain = bars + 2 * STAGES + 4;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  uint32_t* tmem_slot = misc + 0;
  volatile uint32_t* abort_flag = misc + 1;
  int64_t* total_tiles_slot = reinterpret_cast<int64_t*>(misc + 2);

  const uint32_t warp = warp_id_in_cta();
  const uint32_t lane = lane_id();

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0u;
    fence_barrier_init();
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    if constexpr (!kGrouped) prefetch_tmap(&tm_out);
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
        else mt += (static_cast<int64_t>(e) - prev + BM - 1) / BM;
      }
      if (lane == 0 && static_cast<int64_t>(p.offs[p.E - 1]) != p.M) bad = true;
      bad = __any_sync(0xFFFFFFFFu, bad);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
        mt += __shfl_xor_sync(0xFFFFFFFFu, mt, o);
      total = bad ? 0 : mt * p.n_tiles;
      if (bad && lane == 0 && blockIdx.x == 0)
        record_status(p.status, FP8_DEV_VALUE, SITE_OFFS);
    } else {
      total = static_cast<int64_t>(p.m_tiles) * p.n_tiles;
    }
    if (lane == 0) *total_tiles_slot = total;
  }
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const int64_t total_tiles = *total_tiles_slot;
  const int32_t KB = p.k_blocks;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      GroupCursor cur;
      if constexpr (kGrouped) cur.init(p.offs);
      uint32_t stage = 0, phase = 0;
      uint64_t issued = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        const TileCoord c = tile_coord<kGrouped>(t, p, cur);
        for (int32_t kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.status,
                         SITE_PRODUCER_EMPTY, kWaitLimitNs)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], kAStage + kBStage);
          tma_load_2d(smem + kOffA + stage * kAStage, &tm_a, &full[stage],
                      kb * BK, c.m0);
          if constexpr (kGrouped)
            tma_load_3d(smem + kOffB + stage * kBStage, &tm_b, &full[stage],
                        kb * BK, c.n0, c.g);
          else
            tma_load_2d(smem + kOffB + stage * kBStage, &tm_b, &full[stage],
                        kb * BK, c.n0);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        // Let the copies already in flight land before the CTA exits.
        const uint64_t first = issued > STAGES ? issued - STAGES : 0;
        for (uint64_t i = first; i < issued; ++i) {
          uint32_t dummy_abort = 0;
          mbar_wait(&full[i % STAGES], static_cast<uint32_t>((i / STAGES) & 1u),
                    &dummy_abort, nullptr, SITE_TEARDOWN, 10000000ull);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_e4m3_f32(BM, BN);
      uint32_t stage = 0, phase = 0;
      uint32_t acc = 0, acc_phase = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        if constexpr (!kBlockwise) {
          if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort_flag, p.status,
                         SITE_MMA_ACC_EMPTY, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
        }
        for (int32_t kb = 0; kb < KB; ++kb) {
          if constexpr (kBlockwise) {
            if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1u, abort_flag,
                           p.status, SITE_MMA_ACC_EMPTY, kWaitLimitNs)) {
              ok = false;
              break;
            }
            tc_fence_after_sync();
          }
          if (!mbar_wait(&full[stage], phase, abort_flag, p.status,
                         SITE_MMA_FULL, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t d = tmem_base + acc * BN;
          const uint64_t da =
              smem_desc_k_sw128(smem_u32(smem + kOffA + stage * kAStage));
          const uint64_t db =
              smem_desc_k_sw128(smem_u32(smem + kOffB + stage * kBStage));
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k) {
            const uint32_t accumulate =
                kBlockwise ? (k > 0) : ((kb > 0) || (k > 0));
            mma_e4m3(d, da + (k * UMMA_K) / 16, db + (k * UMMA_K) / 16, idesc,
                     accumulate);
          }
          mma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
          if constexpr (kBlockwise) {
            mma_commit(&acc_full[acc]);
            acc ^= 1u;
            if (acc == 0) acc_phase ^= 1u;
          }
        }
        if constexpr (!kBlockwise) {
          if (ok) {
            mma_commit(&acc_full[acc]);
            acc ^= 1u;
            if (acc == 0) acc_phase ^= 1u;
          }
        }
      }
      // All MMAs issued by this thread complete before TMEM is released.
      mma_commit(drain);
      uint32_t dummy_abort = 0;
      mbar_wait(drain, 0, &dummy_abort, p.status, SITE_TEARDOWN, kWaitLimitNs);
    }
  } else {
    // --------------------------------------------------------- epilogue
    const uint32_t ew = warp - 2;          // 0..7
    const uint32_t q = warp & 3u;          // TMEM lane quarter of this warp
    const uint32_t half = ew >> 2;         // which 128 columns of the tile
    uint8_t* ebuf = smem + kOffEpi + ew * kEpiBuf;
    float* sbbuf = reinterpret_cast<float*>(smem + kOffSb + ew * kSbBuf);
    const uint32_t lane_base = (q * 32u) << 16;
    GroupCursor cur;
    if constexpr (kGrouped) cur.init(p.offs);
    uint32_t acc = 0, acc_phase = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
      const TileCoord c = tile_coord<kGrouped>(t, p, cur);
      const int64_t row = static_cast<int64_t>(c.m0) + q * 32 + lane;
      const bool row_ok = row < c.row_end;
      const int64_t ncol0 = static_cast<int64_t>(c.n0) + half * 128;
      const int32_t row0 = c.m0 + static_cast<int32_t>(q * 32);

      if constexpr (!kBlockwise) {
        if (!mbar_wait(&acc_full[acc], acc_phase, abort_flag, p.status,
                       SITE_EPI_ACC_FULL, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        float sa;
        if constexpr (kRecipe == kTensor) sa = __ldg(p.sa) * __ldg(p.sb);
        else sa = row_ok ? __ldg(p.sa + row) : 0.0f;
        const float* sbg = p.sb + (kGrouped ? static_cast<int64_t>(c.g) * p.N : 0);
        const uint32_t tcol = tmem_base + lane_base + acc * BN + half * 128;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tcol + cc * 32, r);
          tmem_ld_wait();
          if (cc == 3) {
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
          }
          const int64_t n = ncol0 + cc * 32;
          float bias[32];
          load_bias32(p.bias, n, p.N, bias);
          float v[32];
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
          store_cols32<kOutF32, kGrouped>(ebuf, v, &tm_out,
                                          static_cast<int32_t>(n), row0,
                                          c.row_end, p.out, p.N, lane);
        }
        acc ^= 1u;
        if (acc == 0) acc_phase ^= 1u;
      } else {
        // Blockwise: promote each K block's partial product into registers.
        float2 accr[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) accr[i] = make_float2(0.0f, 0.0f);
        const int64_t NB = (p.N + 127) / 128;
        const int64_t nb = ncol0 / 128;  // 128-column block of this warp
        const bool nb_ok = ncol0 < p.N;
        // first K block's scales
        float sa_next = row_ok ? __ldg(p.sa + row) : 0.0f;
        float sb_next = 0.0f;
        float4 sb4_next = make_float4(0.f, 0.f, 0.f, 0.f);
        if constexpr (kRecipe == kBlock128) {
          sb_next = nb_ok ? __ldg(p.sb + nb) : 0.0f;
        } else {
          const int64_t n = ncol0 + 4 * lane;
          if (n < p.N) sb4_next = __ldg(reinterpret_cast<const float4*>(p.sb + n));
        }
        for (int32_t kb = 0; kb < KB; ++kb) {
          const float sa_kb = sa_next;
          const float sb_kb = sb_next;
          if constexpr (kRecipe == kBlock1) {
            __syncwarp();
            reinterpret_cast<float4*>(sbbuf)[lane] = sb4_next;
            __syncwarp();
          }
          // prefetch the next K block's scales
          if (kb + 1 < KB) {
            sa_next = row_ok ? __ldg(p.sa + static_cast<int64_t>(kb + 1) * p.M + row) : 0.0f;
            if constexpr (kRecipe == kBlock128) {
              sb_next = nb_ok ? __ldg(p.sb + static_cast<int64_t>(kb + 1) * NB + nb) : 0.0f;
            } else {
              const int64_t n = ncol0 + 4 * lane;
              if (n < p.N)
                sb4_next = __ldg(reinterpret_cast<const float4*>(
                    p.sb + static_cast<int64_t>(kb + 1) * p.N + n));
            }
          }
          if (!mbar_wait(&acc_full[acc], acc_phase, abort_flag, p.status,
                         SITE_EPI_ACC_FULL, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t tcol = tmem_base + lane_base + acc * BN + half * 128;
          const float f = sa_kb * sb_kb;
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            uint32_t r[16];
            tmem_ld_32x32b_x16(tcol + cc * 16, r);
            tmem_ld_wait();
            if constexpr (kRecipe == kBlock128) {
              const float2 f2 = make_float2(f, f);
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float2 pv = make_float2(__uint_as_float(r[2 * i]),
                                              __uint_as_float(r[2 * i + 1]));
                accr[cc * 8 + i] = fma2(pv, f2, accr[cc * 8 + i]);
              }
            } else {
              const float2 sa2 = make_float2(sa_kb, sa_kb);
              const float4* sbv = reinterpret_cast<const float4*>(sbbuf) + cc * 4;
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float4 s4 = sbv[i];
                const float2 p0 = make_float2(__uint_as_float(r[4 * i]),
                                              __uint_as_float(r[4 * i + 1]));
                const float2 p1 = make_float2(__uint_as_float(r[4 * i + 2]),
                                              __uint_as_float(r[4 * i + 3]));
                const float2 t0 = mul2(p0, make_float2(s4.x, s4.y));
                const float2 t1 = mul2(p1, make_float2(s4.z, s4.w));
                accr[cc * 8 + 2 * i] = fma2(t0, sa2, accr[cc * 8 + 2 * i]);
                accr[cc * 8 + 2 * i + 1] = fma2(t1, sa2, accr[cc * 8 + 2 * i + 1]);
              }
            }
          }
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[acc]);
          acc ^= 1u;
          if (acc == 0) acc_phase ^= 1u;
        }
        if (!ok) break;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int64_t n = ncol0 + cc * 32;
          float v[32];
          load_bias32(p.bias, n, p.N, v);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            v[2 * i] += accr[cc * 16 + i].x;
            v[2 * i + 1] += accr[cc * 16 + i].y;
          }
          store_cols32<kOutF32, kGrouped>(ebuf, v, &tm_out,
                                          static_cast<int32_t>(n), row0,
                                          c.row_end, p.out, p.N, lane);
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

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

template <int kRecipe, bool kOutF32, bool kGrouped>
cudaError_t launch_kernel(const CUtensorMap& ta, const CUtensorMap& tb,
                          const CUtensorMap& to, const GemmParams& p,
                          unsigned grid, cudaStream_t st) {
  static bool configured = false;
  auto kern = fp8_gemm_kernel<kRecipe, kOutF32, kGrouped>;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(
        kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  kern<<<grid, kThreads, kSmemBytes, st>>>(ta, tb, to, p);
  return cudaGetLastError();
}

template <bool kGrouped>
cudaError_t dispatch(int recipe, int out_f32, const CUtensorMap& ta,
                     const CUtensorMap& tb, const CUtensorMap& to,
                     const GemmParams& p, unsigned grid, cudaStream_t st) {
#define FP8SM_CASE(R)                                                        \
  if (recipe == R)                                                           \
    return out_f32 ? launch_kernel<R, true, kGrouped>(ta, tb, to, p, grid, st) \
                   : launch_kernel<R, false, kGrouped>(ta, tb, to, p, grid, st);
  if constexpr (kGrouped) {
    FP8SM_CASE(kRow)
  } else {
    FP8SM_CASE(kTensor)
    FP8SM_CASE(kRow)
    FP8SM_CASE(kBlock128)
    FP8SM_CASE(kBlock1)
  }
#undef FP8SM_CASE
  return cudaErrorInvalidValue;
}

bool out_map(CUtensorMap* m, void* out, int64_t rows, int64_t N, int out_f32,
             std::string* err) {
  const uint64_t eb = out_f32 ? 4 : 2;
  uint64_t dims[2] = {static_cast<uint64_t>(N), static_cast<uint64_t>(rows)};
  uint64_t strides[1] = {static_cast<uint64_t>(N) * eb};
  uint32_t box[2] = {static_cast<uint32_t>(64 / eb), 32};
  return make_tmap(m, out_f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                              : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                   2, out, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_64B, err);
}

}  // namespace

cudaError_t launch_scaled_mm(const void* a, const void* b, int64_t M,
                             int64_t N, int64_t K, const float* sa,
                             const float* sb, int recipe, const void* bias,
                             int out_f32, void* out, const LaunchCtx& ctx) {
  if (M == 0 || N == 0) return cudaSuccess;
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
  CUtensorMap ta, tb, to;
  {
    uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M)};
    uint64_t strides[1] = {static_cast<uint64_t>(K)};
    uint32_t box[2] = {BK, BM};
    if (!make_tmap(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a, dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B, ctx.err))
      return cudaErrorInvalidValue;
  }
  {
    uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N)};
    uint64_t strides[1] = {static_cast<uint64_t>(K)};
    uint32_t box[2] = {BK, BN};
    if (!make_tmap(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, b, dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B, ctx.err))
      return cudaErrorInvalidValue;
  }
  if (!out_map(&to, out, M, N, out_f32, ctx.err)) return cudaErrorInvalidValue;
  GemmParams p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.sa = sa;
  p.sb = sb;
  p.bias = static_cast<const uint16_t*>(bias);
  p.out = out;
  p.offs = nullptr;
  p.E = 0;
  p.n_tiles = static_cast<int32_t>((N + BN - 1) / BN);
  p.m_tiles = static_cast<int32_t>((M + BM - 1) / BM);
  p.k_blocks = static_cast<int32_t>((K + BK - 1) / BK);
  p.status = ctx.status;
  const int64_t tiles = static_cast<int64_t>(p.n_tiles) * p.m_tiles;
  const unsigned grid = static_cast<unsigned>(tiles < ctx.num_sms ? tiles : ctx.num_sms);
  return dispatch<false>(recipe, out_f32, ta, tb, to, p, grid, ctx.stream);
}

cudaError_t launch_grouped_scaled_mm(const void* a, const void* b,
                                     int64_t M_total, int64_t N, int64_t K,
                                     int32_t E, const float* sa,
                                     const float* sb, const int32_t* offs,
                                     int out_f32, void* out,
                                     const LaunchCtx& ctx) {
  if (M_total == 0 || N == 0) {
    // Nothing to write; offs still has to end at 0, which the caller's
    // host-side checks cannot see.  A one-CTA launch would only validate.
    if (M_total == 0 && N == 0) return cudaSuccess;
  }
  if (K == 0 || M_total == 0 || N == 0) {
    if (M_total == 0 || N == 0) return cudaSuccess;
    return launch_scaled_mm(nullptr, nullptr, M_total, N, 0, nullptr, nullptr,
                            1, nullptr, out_f32, out, ctx);
  }
  CUtensorMap ta, tb, to;
  {
    uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M_total)};
    uint64_t strides[1] = {static_cast<uint64_t>(K)};
    uint32_t box[2] = {BK, BM};
    if (!make_tmap(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a, dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B, ctx.err))
      return cudaErrorInvalidValue;
  }
  {
    uint64_t dims[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N),
                        static_cast<uint64_t>(E)};
    uint64_t strides[2] = {static_cast<uint64_t>(K),
                           static_cast<uint64_t>(N) * static_cast<uint64_t>(K)};
    uint32_t box[3] = {BK, BN, 1};
    if (!make_tmap(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, b, dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B, ctx.err))
      return cudaErrorInvalidValue;
  }
  // The grouped kernel stores with plain masked stores; the map is unused
  // but must be a valid object.
  if (!out_map(&to, out, M_total, N, out_f32, ctx.err)) return cudaErrorInvalidValue;
  GemmParams p{};
  p.M = M_total;
  p.N = N;
  p.K = K;
  p.sa = sa;
  p.sb = sb;
  p.bias = nullptr;
  p.out = out;
  p.offs = offs;
  p.E = E;
  p.n_tiles = static_cast<int32_t>((N + BN - 1) / BN);
  p.m_tiles = 0;
  p.k_blocks = static_cast<int32_t>((K + BK - 1) / BK);
  p.status = ctx.status;
  return dispatch<true>(1, out_f32, ta, tb, to, p,
                        static_cast<unsigned>(ctx.num_sms), ctx.stream);
}

cudaError_t launch_timeout_probe(uint32_t limit_us, const LaunchCtx& ctx) {
  timeout_probe_kernel<<<1, 32, 0, ctx.stream>>>(
      static_cast<uint64_t>(limit_us) * 1000ull, ctx.status);
  return cudaGetLastError();
}

}  // namespace fp8sm
