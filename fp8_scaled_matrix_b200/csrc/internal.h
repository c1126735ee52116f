// Internal launcher interface between the C-ABI layer (capi.cu) and the
// kernel translation units.  Launchers assume arguments were validated.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <string>

namespace fp8sm {

// Devices the library keeps per-device state for (indices 0 .. 63).
constexpr int kMaxDevices = 64;

struct LaunchCtx {
  cudaStream_t stream;
  uint32_t* status;   // device status word of the current device
  int num_sms;
  int device;         // the current device (set-up below is per device)
  std::string* err;   // filled on failure
};

// One-time set-up that belongs to a device: kernel attributes (the dynamic
// shared-memory opt-in) and occupancy queries are per device, so a process
// that drives several GPUs needs them on each.  `done` holds one flag per
// device; the first caller on `device` runs `setup` under `mu`, and the
// flag is set only when it succeeds.  Safe to call from several threads.
template <class Setup>
cudaError_t once_per_device(std::atomic<bool> (&done)[kMaxDevices], std::mutex& mu,
                            int device, Setup&& setup) {
  if (device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
  if (done[device].load(std::memory_order_acquire)) return cudaSuccess;
  std::lock_guard<std::mutex> lk(mu);
  if (done[device].load(std::memory_order_relaxed)) return cudaSuccess;
  const cudaError_t e = setup();
  if (e == cudaSuccess) done[device].store(true, std::memory_order_release);
  return e;
}

// Tiled TMA tensor map over `base` (gemm.cu): rank 2 or 3, dims/strides in
// elements/bytes (innermost first, strides of dims 1..rank-1), box in
// elements; no interleave, 256-byte L2 promotion, zero fill out of bounds.
// Returns false with *err set when the driver refuses the map.
bool make_tmap(CUtensorMap* m, CUtensorMapDataType dt, uint32_t rank, const void* base,
               const uint64_t* dims, const uint64_t* strides, const uint32_t* box,
               CUtensorMapSwizzle sw, std::string* err);

// Quantizers (quantize.cu).  recipe: 0 tensor, 1 row, 2 1x128, 3 128x128.
cudaError_t launch_quantize(const void* x, int64_t rows, int64_t cols,
                            int64_t ld, int recipe, void* q, float* scales,
                            void* workspace, const LaunchCtx& ctx);

// Sharded tensorwise quantization (quantize.cu): max|x| of a shard into
// amax[0] (device; cleared first), then the cast of a shard with the scale
// of a given amax (written to scale[0]).  cols % 8 == 0.
cudaError_t launch_tensor_amax(const void* x, int64_t rows, int64_t cols, int64_t ld,
                               float* amax, const LaunchCtx& ctx);
cudaError_t launch_tensor_cast(const void* x, int64_t rows, int64_t cols, int64_t ld,
                               const float* amax, void* q, float* scale,
                               const LaunchCtx& ctx);

// Quantization of x^T (quantize.cu), recipe 2 (1x128) or 3 (128x128);
// rows % 128 == 0.  q is (cols, rows) with row stride rows.
cudaError_t launch_quantize_transposed(const void* x, int64_t rows, int64_t cols,
                                       int64_t ld, int recipe, void* q, float* scales,
                                       const LaunchCtx& ctx);

// MXFP8 quantization (quantize.cu): q (rows, cols) e4m3, scale bytes in the
// GEMM's scale-factor tiles (mx_scale_tile_bytes(rows, cols) bytes).
// cols % 32 == 0.
size_t mx_scale_tile_bytes(int64_t rows, int64_t cols);
cudaError_t launch_quantize_mx(const void* x, int64_t rows, int64_t cols, int64_t ld,
                               void* q, void* sf, const LaunchCtx& ctx);

// Batched quantization of `batch` equal (rows, cols) matrices stored one after
// the other (row stride ld; matrix e at x + e * rows * ld), each quantized on
// its own: 128x128 (codes (batch, rows, cols), scales (batch, cols/128,
// ceil(rows/128))), and transposed 1x128 / 128x128 (recipe 2 / 3; codes
// (batch, cols, rows), scales per matrix in the transposed layout; rows %
// 128 == 0) (quantize.cu).
cudaError_t launch_quantize_128x128_batched(const void* x, int32_t batch, int64_t rows,
                                            int64_t cols, int64_t ld, void* q, float* scales,
                                            const LaunchCtx& ctx);
cudaError_t launch_quantize_transposed_batched(const void* x, int32_t batch, int64_t rows,
                                               int64_t cols, int64_t ld, int recipe, void* q,
                                               float* scales, const LaunchCtx& ctx);

// Per-expert transposed 1x128 quantization (quantize.cu): x (rows = tokens,
// cols) with groups of tokens by cumulative offs (device, E entries); the
// output (cols, P) codes with P = grouped_padded_tokens(rows, E) hold each
// group's tokens padded to a multiple of 128 (zero codes in the padding);
// scales (P/128, cols).  E <= 2048.
int64_t grouped_padded_tokens(int64_t tokens, int32_t E);
cudaError_t launch_quantize_transposed_grouped(const void* x, int64_t rows, int64_t cols,
                                               int64_t ld, const int32_t* offs, int32_t E,
                                               void* q, float* scales, const LaunchCtx& ctx);

// Library-owned scratch for the no-allocation quantize entry point
// (quantize.cu): its size, and its device address on `device` (looked up
// once per device; the device must be current).
size_t noalloc_scratch_bytes();
cudaError_t noalloc_scratch_ptr(int device, void** out);

// Dense scaled GEMM (gemm.cu).  recipe: 0 tensor, 1 row, 2 1x128_128x128,
// 3 1x128_128x1, 4 MXFP8 (sa, sb then point to E8M0 scale-factor tiles).
// out_kind: 0 bf16, 1 fp32, 2 e4m3 quantized in 1x128 groups along n with
// fp32 scales written to out_scales[(n/128) * M + m], 3 MXFP8 (recipe 4
// only; E8M0 scale-factor tiles written to out_scales as bytes), 4 both
// e4m3 forms (recipe 2 only, M % 128 == 0): out / out_scales as for 2, and
// the result transposed in out_t (N, M) with 1x128-along-m scales
// out_t_scales[(m/128) * N + n].
cudaError_t launch_scaled_mm(const void* a, const void* b, int64_t M,
                             int64_t N, int64_t K, const float* sa,
                             const float* sb, int recipe, const void* bias,
                             int out_kind, void* out, float* out_scales,
                             const LaunchCtx& ctx, void* out_t = nullptr,
                             float* out_t_scales = nullptr);

// Grouped scaled GEMM (gemm.cu).  recipe: 1 rowwise, 2 1x128_128x128.
cudaError_t launch_grouped_scaled_mm(const void* a, const void* b,
                                     int64_t M_total, int64_t N, int64_t K,
                                     int32_t E, const float* sa,
                                     const float* sb, const int32_t* offs,
                                     int recipe, int out_f32, void* out,
                                     const LaunchCtx& ctx);

// Per-expert weight gradient (gemm.cu): for g < E, out[g] (M, N) =
// sum over group g's padded K blocks of (a_t * sa)(b_t * sb)^T with the
// 1x128_128x1 recipe.  a_t (M, P), b_t (N, P): per-expert padded transposed
// codes (launch_quantize_transposed_grouped); sa (P/128, M), sb (P/128, N);
// offs (device, E) token offsets ending at `tokens`.  M % 128 == 0.
cudaError_t launch_grouped_wgrad(const void* a_t, const void* b_t, int64_t M, int64_t N,
                                 int64_t P, int64_t tokens, int32_t E, const float* sa,
                                 const float* sb, const int32_t* offs, int out_f32, void* out,
                                 const LaunchCtx& ctx);

// Failure-detection probe (gemm.cu): one CTA waits on a barrier nothing
// completes, with the given limit.
cudaError_t launch_timeout_probe(uint32_t limit_us, const LaunchCtx& ctx);

}  // namespace fp8sm
