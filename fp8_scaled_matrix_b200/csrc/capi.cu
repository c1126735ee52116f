// C ABI of the library (declared in include/fp8sm.h): argument validation,
// recipe -> kernel selection (one kernel per recipe, no fallback), the
// per-device status word and per-thread error messages.
//
// Error classes follow "Add _scaled_mm_v2 API" (Blas.cpp review): invalid
// arguments are a user error (FP8_ERR_VALUE), combinations that could exist
// but are not implemented are FP8_ERR_UNSUPPORTED, everything else
// (CUDA failures) FP8_ERR_CUDA.  "Add _grouped_mm dispatch handler to
// Float8Tensor" requires that an unsupported granularity raises instead of
// silently running something else; nothing here ever falls back.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <string>

#include "../../include/fp8sm.h"
#include "internal.h"

namespace fp8sm {
// Device status words (one per device, since __device__ variables are
// instantiated per device): [0] first error code, [1] site.
__device__ uint32_t g_status_word[2];
}  // namespace fp8sm

namespace {

thread_local std::string t_last_error;

using fp8sm::kMaxDevices;
struct DeviceInfo {
  bool ready = false;
  int device = 0;
  uint32_t* status = nullptr;
  int num_sms = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

fp8_status fail(fp8_status s, const std::string& msg) {
  t_last_error = msg;
  return s;
}

fp8_status cuda_fail(cudaError_t e, const char* what) {
  return fail(FP8_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

// Per-device set-up on first use: the status word's device address (taken
// with the device current) and the SM count.
fp8_status device_info(DeviceInfo** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(FP8_ERR_CUDA, "device index out of range");
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, fp8sm::g_status_word);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status)");
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0)
      return fail(FP8_ERR_UNSUPPORTED,
                  "this library is built for sm_100a (B200); device has compute capability " +
                      std::to_string(major) + "." + std::to_string(minor));
    d.device = dev;
    d.status = static_cast<uint32_t*>(p);
    d.num_sms = sms;
    d.ready = true;
  }
  *out = &d;
  return FP8_OK;
}

fp8sm::LaunchCtx make_ctx(const DeviceInfo* d, fp8_stream_t stream, std::string* err) {
  return fp8sm::LaunchCtx{reinterpret_cast<cudaStream_t>(stream), d->status, d->num_sms,
                          d->device, err};
}

bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

fp8_status finish_launch(cudaError_t e, const std::string& err, const char* what) {
  if (e == cudaSuccess) {
    t_last_error.clear();
    return FP8_OK;
  }
  if (!err.empty()) return fail(FP8_ERR_VALUE, std::string(what) + ": " + err);
  return cuda_fail(e, what);
}

}  // namespace

extern "C" {

int fp8_version(void) { return 100; }

const char* fp8_last_error(void) { return t_last_error.c_str(); }

size_t fp8_quantize_workspace_bytes(fp8_quant_recipe recipe, int64_t rows,
                                    int64_t cols) {
  (void)rows;
  (void)cols;
  return recipe == FP8_SCALE_TENSOR ? 16 : 0;
}

fp8_status fp8_quantize(const void* x_bf16, int64_t rows, int64_t cols,
                        int64_t ld_x, fp8_quant_recipe recipe, void* out_fp8,
                        float* out_scales, void* workspace, size_t ws_bytes,
                        fp8_stream_t stream) {
  if (recipe < FP8_SCALE_TENSOR || recipe > FP8_SCALE_BLOCK_128x128)
    return fail(FP8_ERR_VALUE, "fp8_quantize: unknown recipe");
  if (rows < 0 || cols < 0) return fail(FP8_ERR_VALUE, "fp8_quantize: negative size");
  if (rows >= (int64_t(1) << 31) || cols >= (int64_t(1) << 31))
    return fail(FP8_ERR_VALUE, "fp8_quantize: size too large");
  if (ld_x < cols) return fail(FP8_ERR_VALUE, "fp8_quantize: ld_x < cols");
  if (cols % 8 != 0 || ld_x % 8 != 0)
    return fail(FP8_ERR_VALUE, "fp8_quantize: cols and ld_x must be multiples of 8");
  if ((recipe == FP8_SCALE_BLOCK_1x128 || recipe == FP8_SCALE_BLOCK_128x128) &&
      cols % 128 != 0)
    return fail(FP8_ERR_VALUE, "fp8_quantize: blockwise recipes need cols % 128 == 0");
  const bool empty = rows == 0 || cols == 0;
  const bool writes_scales = !(rows == 0 && recipe != FP8_SCALE_TENSOR) &&
                             !(cols == 0 && (recipe == FP8_SCALE_BLOCK_1x128 ||
                                             recipe == FP8_SCALE_BLOCK_128x128));
  if (!empty && (x_bf16 == nullptr || out_fp8 == nullptr))
    return fail(FP8_ERR_VALUE, "fp8_quantize: null tensor pointer");
  if (writes_scales && out_scales == nullptr)
    return fail(FP8_ERR_VALUE, "fp8_quantize: null scale pointer");
  if (!empty && (!aligned(x_bf16, 16) || !aligned(out_fp8, 16)))
    return fail(FP8_ERR_VALUE, "fp8_quantize: x and out_fp8 must be 16-byte aligned");
  if (out_scales && !aligned(out_scales, 4))
    return fail(FP8_ERR_VALUE, "fp8_quantize: out_scales must be 4-byte aligned");
  const size_t need = fp8_quantize_workspace_bytes(recipe, rows, cols);
  if (need > 0 && (workspace == nullptr || ws_bytes < need || !aligned(workspace, 16)))
    return fail(FP8_ERR_VALUE, "fp8_quantize: tensorwise recipe needs a 16-byte aligned "
                               "workspace of fp8_quantize_workspace_bytes() bytes");
  if (!writes_scales) {
    t_last_error.clear();
    return FP8_OK;
  }
  DeviceInfo* d = nullptr;
  fp8_status s = device_info(&d);
  if (s != FP8_OK) return s;
  std::string err;
  fp8sm::LaunchCtx ctx = make_ctx(d, stream, &err);
  cudaError_t e = fp8sm::launch_quantize(x_bf16, rows, cols, ld_x, (int)recipe,
                                         out_fp8, out_scales, workspace, ctx);
  return finish_launch(e, err, "fp8_quantize");
}

fp8_status fp8_quantize_transposed(const void* x_bf16, int64_t rows, int64_t cols,
                                   int64_t ld_x, fp8_quant_recipe recipe, void* out_fp8,
                                   float* out_scales, fp8_stream_t stream) {
  if (recipe < FP8_SCALE_TENSOR || recipe > FP8_SCALE_BLOCK_128x128)
    return fail(FP8_ERR_VALUE, "fp8_quantize_transposed: unknown recipe");
  if (recipe != FP8_SCALE_BLOCK_1x128 && recipe != FP8_SCALE_BLOCK_128x128)
    return fail(FP8_ERR_UNSUPPORTED,
                "fp8_quantize_transposed: only the 1x128 and 128x128 recipes are implemented");
  if (rows < 0 || cols < 0) return fail(FP8_ERR_VALUE, "fp8_quantize_transposed: negative size");
  if (rows >= (int64_t(1) << 31) || cols >= (int64_t(1) << 31))
    return fail(FP8_ERR_VALUE, "fp8_quantize_transposed: size too large");
  if (ld_x < cols) return fail(FP8_ERR_VALUE, "fp8_quantize_transposed: ld_x < cols");
  if (cols % 8 != 0 || ld_x % 8 != 0)
    return fail(FP8_ERR_VALUE,
                "fp8_quantize_transposed: cols and ld_x must be multiples of 8");
  if (rows % 128 != 0)
    return fail(FP8_ERR_VALUE, "fp8_quantize_transposed: rows must be a multiple of 128");
  if (rows == 0 || cols == 0) {
    t_last_error.clear();
    return FP8_OK;
  }
  if (x_bf16 == nullptr || out_fp8 == nullptr || out_scales == nullptr)
    return fail(FP8_ERR_VALUE, "fp8_quantize_transposed: null pointer");
  if (!aligned(x_bf16, 16) || !aligned(out_fp8, 16) || !aligned(out_scales, 4))
    return fail(FP8_ERR_VALUE,
                "fp8_quantize_transposed: x and out_fp8 must be 16-byte aligned, "
                "out_scales 4-byte aligned");
  DeviceInfo* d = nullptr;
  fp8_status s = device_info(&d);
  if (s != FP8_OK) return s;
  std::string err;
  fp8sm::LaunchCtx ctx = make_ctx(d, stream, &err);
  cudaError_t e = fp8sm::launch_quantize_transposed(x_bf16, rows, cols, ld_x, (int)recipe,
                                                    out_fp8, out_scales, ctx);
  return finish_launch(e, err, "fp8_quantize_transposed");
}

fp8_status fp8_quantize_batched(const void* x_bf16, int32_t batch, int64_t rows, int64_t cols,
                                int64_t ld_x, fp8_quant_recipe recipe, void* out_fp8,
                                float* out_scales, fp8_stream_t stream) {
  const std::string n("fp8_quantize_batched");
  if (recipe < FP8_SCALE_TENSOR || recipe > FP8_SCALE_BLOCK_128x128)
    return fail(FP8_ERR_VALUE, n + ": unknown recipe");
  if (recipe != FP8_SCALE_BLOCK_128x128)
    return fail(FP8_ERR_UNSUPPORTED, n + ": only the 128x128 recipe is implemented");
  if (batch < 0 || batch > 65535 || rows < 0 || cols < 0)
    return fail(FP8_ERR_VALUE, n + ": bad batch or size");
  if (rows >= (int64_t(1) << 31) || cols >= (int64_t(1) << 31))
    return fail(FP8_ERR_VALUE, n + ": size too large");
  if (ld_x < cols) return fail(FP8_ERR_VALUE, n + ": ld_x < cols");
  if (cols % 128 != 0 || ld_x % 8 != 0)
    return fail(FP8_ERR_VALUE, n + ": cols % 128 == 0 and ld_x % 8 == 0 are required");
  if (batch == 0 || rows == 0 || cols == 0) {
    t_last_error.clear();
    return FP8_OK;
  }
  if (x_bf16 == nullptr || out_fp8 == nullptr || out_scales == nullptr)
    return fail(FP8_ERR_VALUE, n + ": null pointer");
  if (!aligned(x_bf16, 16) || !aligned(out_fp8, 16) || !aligned(out_scales, 4))
    return fail(FP8_ERR_VALUE, n + ": x and out_fp8 must be 16-byte aligned, out_scales 4");
  DeviceInfo* d = nullptr;
  fp8_status s = device_info(&d);
  if (s != FP8_OK) return s;
  std::string err;
  fp8sm::LaunchCtx ctx = make_ctx(d, stream, &err);
  cudaError_t e = fp8sm::launch_quantize_128x128_batched(x_bf16, batch, rows, cols, ld_x,
                                                         out_fp8, out_scales, ctx);
  return finish_launch(e, err, n.c_str());
}

fp8_status fp8_quantize_transposed_batched(const void* x_bf16, int32_t batch, int64_t rows,
                                           int64_t cols, int64_t ld_x, fp8_quant_recipe recipe,
                                           void* out_fp8, float* out_scales,
                                           fp8_stream_t stream) {
  const std::string n("fp8_quantize_transposed_batched");
  if (recipe < FP8_SCALE_TENSOR || recipe > FP8_SCALE_BLOCK_128x128)
    return fail(FP8_ERR_VALUE, n + ": unknown recipe");
  if (recipe != FP8_SCALE_BLOCK_1x128 && recipe != FP8_SCALE_BLOCK_128x128)
    return fail(FP8_ERR_UNSUPPORTED, n + ": only the 1x128 and 128x128 recipes are implemented");
  if (batch < 0 || batch > 65535 || rows < 0 || cols < 0)
    return fail(FP8_ERR_VALUE, n + ": bad batch or size");
  if (rows >= (int64_t(1) << 31) || cols >= (int64_t(1) << 31))
    return fail(FP8_ERR_VALUE, n + ": size too large");
  if (ld_x < cols) return fail(FP8_ERR_VALUE, n + ": ld_x < cols");
  if (cols % 8 != 0 || ld_x % 8 != 0)
    return fail(FP8_ERR_VALUE, n + ": cols and ld_x must be multiples of 8");
  if (rows % 128 != 0) return fail(FP8_ERR_VALUE, n + ": rows must be a multiple of 128");
  if (batch == 0 || rows == 0 || cols == 0) {
    t_last_error.clear();
    return FP8_OK;
  }
  if (x_bf16 == nullptr || out_fp8 == nullptr || out_scales == nullptr)
    return fail(FP8_ERR_VALUE, n + ": null pointer");
  if (!aligned(x_bf16, 16) || !aligned(out_fp8, 16) || !aligned(out_scales, 4))
    return fail(FP8_ERR_VALUE, n + ": x and out_fp8 must be 16-byte aligned, out_scales 4");
  DeviceInfo* d = nullptr;
  fp8_status s = device_info(&d);
  if (s != FP8_OK) return s;
  std::string err;
  fp8sm::LaunchCtx ctx = make_ctx(d, stream, &err);
  cudaError_t e = fp8sm::launch_quantize_transposed_batched(x_bf16, batch, rows, cols, ld_x,
                                                            (int)recipe, out_fp8, out_scales, ctx);
  return finish_launch(e, err, n.c_str());
}

// Shape and pointer checks shared by the two steps of the sharded tensorwise
// quantization.
static fp8_status check_tensor_shard(const char* name, const void* x, int64_t rows,
                                     int64_t cols, int64_t ld) {
  const std::string n(name);
  if (rows < 0 || cols < 0) return fail(FP8_ERR_VALUE, n + ": negative size");
  if (rows >= (int64_t(1) << 31) || cols >= (int64_t(1) << 31))
    return fail(FP8_ERR_VALUE, n + ": size too large");
  if (ld < cols) return fail(FP8_ERR_VALUE, n + ": ld_x < cols");
  if (cols % 8 != 0 || ld % 8 != 0)
    return fail(FP8_ERR_VALUE, n + ": cols and ld_x must be multiples of 8");
  if (rows > 0 && cols > 0 && (x == nullptr || !aligned(x, 16)))
    return fail(FP8_ERR_VALUE, n + ": x must be a 16-byte aligned device pointer");
  return FP8_OK;
}

fp8_status fp8_tensor_amax(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld_x,
                           float* amax, fp8_stream_t stream) {
  fp8_status s = check_tensor_shard("fp8_tensor_amax", x_bf16, rows, cols, ld_x);
  if (s != FP8_OK) return s;
  if (amax == nullptr || !aligned(amax, 4))
    return fail(FP8_ERR_VALUE, "fp8_tensor_amax: amax must be a 4-byte aligned device pointer");
  DeviceInfo* d = nullptr;
  s = device_info(&d);
  if (s != FP8_OK) return s;
  std::string err;
  fp8sm::LaunchCtx ctx = make_ctx(d, stream, &err);
  return finish_launch(fp8sm::launch_tensor_amax(x_bf16, rows, cols, ld_x, amax, ctx), err,
                       "fp8_tensor_amax");
}

fp8_status fp8_quantize_tensor_with_amax(const void* x_bf16, int64_t rows, int64_t cols,
                                         int64_t ld_x, const float* amax, void* out_fp8,
                                         float* out_scale, fp8_stream_t stream) {
  const char* n = "fp8_quantize_tensor_with_amax";
  fp8_status s = check_tensor_shard(n, x_bf16, rows, cols, ld_x);
  if (s != FP8_OK) return s;
  if (amax == nullptr || out_scale == nullptr || !aligned(amax, 4) || !aligned(out_scale, 4))
    return fail(FP8_ERR_VALUE, std::string(n) + ": amax and out_scale must be 4-byte aligned "
                                                "device pointers");
  if (rows > 0 && cols > 0 && (out_fp8 == nullptr || !aligned(out_fp8, 16)))
    return fail(FP8_ERR_VALUE, std::string(n) + ": out_fp8 must be 16-byte aligned");
  DeviceInfo* d = nullptr;
  s = device_info(&d);
  if (s != FP8_OK) return s;
  std::string err;
  fp8sm::LaunchCtx ctx = make_ctx(d, stream, &err);
  return finish_launch(
      fp8sm::launch_tensor_cast(x_bf16, rows, cols, ld_x, amax, out_fp8, out_scale, ctx), err, n);
}

fp8_status fp8_quantize_noalloc(const void* x_bf16, int64_t rows, int64_t cols,
                                int64_t ld_x, fp8_quant_recipe recipe,
                                void* out_fp8, float* out_scales,
                                fp8_stream_t stream) {
  if (recipe < FP8_SCALE_TENSOR || recipe > FP8_SCALE_BLOCK_128x128)
    return fail(FP8_ERR_VALUE, "fp8_quantize_noalloc: unknown recipe");
  const size_t need = fp8_quantize_workspace_bytes(recipe, rows, cols);
  const size_t have = fp8sm::noalloc_scratch_bytes();
  if (need > have)
    return fail(FP8_ERR_VALUE,
                "fp8_quantize_noalloc: this call needs " + std::to_string(need) +
                    " bytes of scratch, more than the library's fixed " +
                    std::to_string(have) + "-byte scratch");
  void* scratch = nullptr;
  if (need > 0) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "fp8_quantize_noalloc: cudaGetDevice");
    e = fp8sm::noalloc_scratch_ptr(dev, &scratch);
    if (e != cudaSuccess)
      return cuda_fail(e, "fp8_quantize_noalloc: cudaGetSymbolAddress(scratch)");
  }
  // Same validation and kernels as fp8_quantize, with the library's own
  // scratch standing in for the caller's workspace.
  return fp8_quantize(x_bf16, rows, cols, ld_x, recipe, out_fp8, out_scales,
                      scratch, need > 0 ? have : 0, stream);
}

fp8_status fp8_scaled_mm(const void* a, const void* b, int64_t M, int64_t N,
                         int64_t K, const float* scale_a, const float* scale_b,
                         fp8_mm_recipe recipe, const void* bias_bf16,
                         fp8_out_dtype out_dtype, void* out,
                         fp8_stream_t stream) {
  if (recipe < FP8_MM_TENSOR_TENSOR || recipe > FP8_MM_1x128_128x1)
    return fail(FP8_ERR_VALUE, "fp8_scaled_mm: unknown recipe");
  if (out_dtype != FP8_OUT_BF16 && out_dtype != FP8_OUT_F32)
    return fail(FP8_ERR_VALUE, "fp8_scaled_mm: unknown out_dtype");
  if (M < 0 || N < 0 || K < 0) return fail(FP8_ERR_VALUE, "fp8_scaled_mm: negative size");
  if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
    return fail(FP8_ERR_VALUE, "fp8_scaled_mm: size too large");
  if (K % 16 != 0) return fail(FP8_ERR_VALUE, "fp8_scaled_mm: K must be a multiple of 16");
  if (N % 16 != 0) return fail(FP8_ERR_VALUE, "fp8_scaled_mm: N must be a multiple of 16");
  const bool blockwise = recipe == FP8_MM_1x128_128x128 || recipe == FP8_MM_1x128_128x1;
  if (blockwise && K % 128 != 0)
    return fail(FP8_ERR_VALUE, "fp8_scaled_mm: blockwise recipes need K % 128 == 0");
  if (M == 0 || N == 0) {
    t_last_error.clear();
    return FP8_OK;
  }
  if (out == nullptr) return fail(FP8_ERR_VALUE, "fp8_scaled_mm: null out");
  if (K > 0 && (a == nullptr || b == nullptr || scale_a == nullptr || scale_b == nullptr))
    return fail(FP8_ERR_VALUE, "fp8_scaled_mm: null operand or scale pointer");
  if (!aligned(out, 16) || (a && !aligned(a, 16)) || (b && !aligned(b, 16)) ||
      (bias_bf16 && !aligned(bias_bf16, 16)) || (scale_a && !aligned(scale_a, 16)) ||
      (scale_b && !aligned(scale_b, 16)))
    return fail(FP8_ERR_VALUE, "fp8_scaled_mm: pointers must be 16-byte aligned");
  DeviceInfo* d = nullptr;
  fp8_status s = device_info(&d);
  if (s != FP8_OK) return s;
  std::string err;
  fp8sm::LaunchCtx ctx = make_ctx(d, stream, &err);
  cudaError_t e = fp8sm::launch_scaled_mm(a, b, M, N, K, scale_a, scale_b,
                                          (int)recipe, bias_bf16,
                                          out_dtype == FP8_OUT_F32 ? 1 : 0, out, nullptr, ctx);
  return finish_launch(e, err, "fp8_scaled_mm");
}

fp8_status fp8_scaled_mm_quantized(const void* a, const void* b, int64_t M, int64_t N,
                                   int64_t K, const float* scale_a, const float* scale_b,
                                   fp8_mm_recipe recipe, const void* bias_bf16,
                                   void* out_fp8, float* out_scales, fp8_stream_t stream) {
  if (recipe < FP8_MM_TENSOR_TENSOR || recipe > FP8_MM_1x128_128x1)
    return fail(FP8_ERR_VALUE, "fp8_scaled_mm_quantized: unknown recipe");
  if (M < 0 || N < 0 || K < 0)
    return fail(FP8_ERR_VALUE, "fp8_scaled_mm_quantized: negative size");
  if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
    return fail(FP8_ERR_VALUE, "fp8_scaled_mm_quantized: size too large");
  if (K == 0 || K % 16 != 0)
    return fail(FP8_ERR_VALUE, "fp8_scaled_mm_quantized: K must be a positive multiple of 16");
  if (N % 128 != 0)
    return fail(FP8_ERR_VALUE,
                "fp8_scaled_mm_quantized: N must be a multiple of 128 (1x128 output groups)");
  const bool blockwise = recipe == FP8_MM_1x128_128x128 || recipe == FP8_MM_1x128_128x1;
  if (blockwise && K % 128 != 0)
    return fail(FP8_ERR_VALUE, "fp8_scaled_mm_quantized: blockwise recipes need K % 128 == 0");
  if (M == 0 || N == 0) {
    t_last_error.clear();
    return FP8_OK;
  }
  if (a == nullptr || b == nullptr || scale_a == nullptr || scale_b == nullptr ||
      out_fp8 == nullptr || out_scales == nullptr)
    return fail(FP8_ERR_VALUE, "fp8_scaled_mm_quantized: null pointer");
  if (!aligned(out_fp8, 16) || !aligned(a, 16) || !aligned(b, 16) ||
      (bias_bf16 && !aligned(bias_bf16, 16)) || !aligned(scale_a, 16) ||
      !aligned(scale_b, 16) || !aligned(out_scales, 4))
    return fail(FP8_ERR_VALUE, "fp8_scaled_mm_quantized: misaligned pointer");
  DeviceInfo* d = nullptr;
  fp8_status s = device_info(&d);
  if (s != FP8_OK) return s;
  std::string err;
  fp8sm::LaunchCtx ctx = make_ctx(d, stream, &err);
  cudaError_t e = fp8sm::launch_scaled_mm(a, b, M, N, K, scale_a, scale_b, (int)recipe,
                                          bias_bf16, 2, out_fp8, out_scales, ctx);
  return finish_launch(e, err, "fp8_scaled_mm_quantized");
}

size_t fp8_mx_scale_bytes(int64_t rows, int64_t cols) {
  if (rows < 0 || cols < 0) return 0;
  return fp8sm::mx_scale_tile_bytes(rows, cols);
}

fp8_status fp8_quantize_mx(const void* x_bf16, int64_t rows, int64_t cols, int64_t ld_x,
                           void* out_fp8, void* out_scales_e8m0, fp8_stream_t stream) {
  if (rows < 0 || cols < 0) return fail(FP8_ERR_VALUE, "fp8_quantize_mx: negative size");
  if (rows >= (int64_t(1) << 31) || cols >= (int64_t(1) << 31))
    return fail(FP8_ERR_VALUE, "fp8_quantize_mx: size too large");
  if (cols % 32 != 0) return fail(FP8_ERR_VALUE, "fp8_quantize_mx: cols must be a multiple of 32");
  if (ld_x < cols || ld_x % 8 != 0)
    return fail(FP8_ERR_VALUE, "fp8_quantize_mx: ld_x must be >= cols and a multiple of 8");
  if (rows == 0 || cols == 0) {
    t_last_error.clear();
    return FP8_OK;
  }
  if (x_bf16 == nullptr || out_fp8 == nullptr || out_scales_e8m0 == nullptr)
    return fail(FP8_ERR_VALUE, "fp8_quantize_mx: null pointer");
  if (!aligned(x_bf16, 16) || !aligned(out_fp8, 16) || !aligned(out_scales_e8m0, 16))
    return fail(FP8_ERR_VALUE, "fp8_quantize_mx: pointers must be 16-byte aligned");
  DeviceInfo* d = nullptr;
  fp8_status s = device_info(&d);
  if (s != FP8_OK) return s;
  std::string err;
  fp8sm::LaunchCtx ctx = make_ctx(d, stream, &err);
  cudaError_t e = fp8sm::launch_quantize_mx(x_bf16, rows, cols, ld_x, out_fp8,
                                            out_scales_e8m0, ctx);
  return finish_launch(e, err, "fp8_quantize_mx");
}

fp8_status fp8_scaled_mm_mx(const void* a, const void* b, int64_t M, int64_t N, int64_t K,
                            const void* scale_a_e8m0, const void* scale_b_e8m0,
                            const void* bias_bf16, fp8_out_dtype out_dtype, void* out,
                            fp8_stream_t stream) {
  if (out_dtype != FP8_OUT_BF16 && out_dtype != FP8_OUT_F32)
    return fail(FP8_ERR_VALUE, "fp8_scaled_mm_mx: unknown out_dtype");
  if (M < 0 || N < 0 || K < 0) return fail(FP8_ERR_VALUE, "fp8_scaled_mm_mx: negative size");
  if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
    return fail(FP8_ERR_VALUE, "fp8_scaled_mm_mx: size too large");
  if (K == 0 || K % 32 != 0)
    return fail(FP8_ERR_VALUE, "fp8_scaled_mm_mx: K must be a positive multiple of 32");
  if (N % 16 != 0) return fail(FP8_ERR_VALUE, "fp8_scaled_mm_mx: N must be a multiple of 16");
  if (M == 0 || N == 0) {
    t_last_error.clear();
    return FP8_OK;
  }
  if (a == nullptr || b == nullptr || scale_a_e8m0 == nullptr || scale_b_e8m0 == nullptr ||
      out == nullptr)
    return fail(FP8_ERR_VALUE, "fp8_scaled_mm_mx: null pointer");
  if (!aligned(a, 16) || !aligned(b, 16) || !aligned(scale_a_e8m0, 16) ||
      !aligned(scale_b_e8m0, 16) || !aligned(out, 16) || (bias_bf16 && !aligned(bias_bf16, 16)))
    return fail(FP8_ERR_VALUE, "fp8_scaled_mm_mx: pointers must be 16-byte aligned");
  DeviceInfo* d = nullptr;
  fp8_status s = device_info(&d);
  if (s != FP8_OK) return s;
  std::string err;
  fp8sm::LaunchCtx ctx = make_ctx(d, stream, &err);
  cudaError_t e = fp8sm::launch_scaled_mm(
      a, b, M, N, K, static_cast<const float*>(scale_a_e8m0),
      static_cast<const float*>(scale_b_e8m0), 4, bias_bf16,
      out_dtype == FP8_OUT_F32 ? 1 : 0, out, nullptr, ctx);
  return finish_launch(e, err, "fp8_scaled_mm_mx");
}

fp8_status fp8_scaled_mm_quantized_dual(const void* a, const void* b, int64_t M, int64_t N,
                                        int64_t K, const float* scale_a, const float* scale_b,
                                        fp8_mm_recipe recipe, const void* bias_bf16,
                                        void* out_fp8, float* out_scales, void* out_t_fp8,
                                        float* out_t_scales, fp8_stream_t stream) {
  const std::string n("fp8_scaled_mm_quantized_dual");
  if (recipe < FP8_MM_TENSOR_TENSOR || recipe > FP8_MM_1x128_128x1)
    return fail(FP8_ERR_VALUE, n + ": unknown recipe");
  if (recipe != FP8_MM_1x128_128x128)
    return fail(FP8_ERR_UNSUPPORTED, n + ": only the 1x128_128x128 recipe is implemented");
  if (M < 0 || N < 0 || K < 0) return fail(FP8_ERR_VALUE, n + ": negative size");
  if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
    return fail(FP8_ERR_VALUE, n + ": size too large");
  if (K == 0 || K % 128 != 0)
    return fail(FP8_ERR_VALUE, n + ": K must be a positive multiple of 128");
  if (M % 128 != 0 || N % 128 != 0)
    return fail(FP8_ERR_VALUE, n + ": M and N must be multiples of 128");
  if (M == 0 || N == 0) {
    t_last_error.clear();
    return FP8_OK;
  }
  if (a == nullptr || b == nullptr || scale_a == nullptr || scale_b == nullptr ||
      out_fp8 == nullptr || out_scales == nullptr || out_t_fp8 == nullptr ||
      out_t_scales == nullptr)
    return fail(FP8_ERR_VALUE, n + ": null pointer");
  if (!aligned(out_fp8, 16) || !aligned(out_t_fp8, 16) || !aligned(a, 16) || !aligned(b, 16) ||
      (bias_bf16 && !aligned(bias_bf16, 16)) || !aligned(scale_a, 16) || !aligned(scale_b, 16) ||
      !aligned(out_scales, 4) || !aligned(out_t_scales, 4))
    return fail(FP8_ERR_VALUE, n + ": misaligned pointer");
  DeviceInfo* d = nullptr;
  fp8_status s = device_info(&d);
  if (s != FP8_OK) return s;
  std::string err;
  fp8sm::LaunchCtx ctx = make_ctx(d, stream, &err);
  cudaError_t e = fp8sm::launch_scaled_mm(a, b, M, N, K, scale_a, scale_b, (int)recipe, bias_bf16,
                                          4, out_fp8, out_scales, ctx, out_t_fp8, out_t_scales);
  return finish_launch(e, err, n.c_str());
}

fp8_status fp8_scaled_mm_mx_quantized(const void* a, const void* b, int64_t M, int64_t N,
                                      int64_t K, const void* scale_a_e8m0,
                                      const void* scale_b_e8m0, const void* bias_bf16,
                                      void* out_fp8, void* out_scales_e8m0,
                                      fp8_stream_t stream) {
  if (M < 0 || N < 0 || K < 0)
    return fail(FP8_ERR_VALUE, "fp8_scaled_mm_mx_quantized: negative size");
  if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
    return fail(FP8_ERR_VALUE, "fp8_scaled_mm_mx_quantized: size too large");
  if (K == 0 || K % 32 != 0)
    return fail(FP8_ERR_VALUE,
                "fp8_scaled_mm_mx_quantized: K must be a positive multiple of 32");
  if (N % 128 != 0)
    return fail(FP8_ERR_VALUE, "fp8_scaled_mm_mx_quantized: N must be a multiple of 128");
  if (M == 0 || N == 0) {
    t_last_error.clear();
    return FP8_OK;
  }
  if (a == nullptr || b == nullptr || scale_a_e8m0 == nullptr || scale_b_e8m0 == nullptr ||
      out_fp8 == nullptr || out_scales_e8m0 == nullptr)
    return fail(FP8_ERR_VALUE, "fp8_scaled_mm_mx_quantized: null pointer");
  if (!aligned(a, 16) || !aligned(b, 16) || !aligned(scale_a_e8m0, 16) ||
      !aligned(scale_b_e8m0, 16) || !aligned(out_fp8, 16) || !aligned(out_scales_e8m0, 16) ||
      (bias_bf16 && !aligned(bias_bf16, 16)))
    return fail(FP8_ERR_VALUE, "fp8_scaled_mm_mx_quantized: pointers must be 16-byte aligned");
  DeviceInfo* d = nullptr;
  fp8_status s = device_info(&d);
  if (s != FP8_OK) return s;
  std::string err;
  fp8sm::LaunchCtx ctx = make_ctx(d, stream, &err);
  cudaError_t e = fp8sm::launch_scaled_mm(
      a, b, M, N, K, static_cast<const float*>(scale_a_e8m0),
      static_cast<const float*>(scale_b_e8m0), 4, bias_bf16, 3, out_fp8,
      static_cast<float*>(out_scales_e8m0), ctx);
  return finish_launch(e, err, "fp8_scaled_mm_mx_quantized");
}

namespace {

// Shared by both grouped entry points; recipe 1 (rowwise) or 2 (1x128_128x128).
fp8_status grouped_common(const char* name, int recipe, const void* a, const void* b_experts,
                          int64_t M_total, int64_t N, int64_t K, int32_t E,
                          const float* scale_a, const float* scale_b, const int32_t* offs,
                          fp8_out_dtype out_dtype, void* out, fp8_stream_t stream) {
  const std::string n(name);
  if (out_dtype != FP8_OUT_BF16 && out_dtype != FP8_OUT_F32)
    return fail(FP8_ERR_VALUE, n + ": unknown out_dtype");
  if (offs == nullptr) return fail(FP8_ERR_VALUE, n + ": offs is required");
  if (M_total < 0 || N < 0 || K < 0 || E < 1 || E > 65535)
    return fail(FP8_ERR_VALUE, n + ": bad size or expert count");
  if (M_total >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
    return fail(FP8_ERR_VALUE, n + ": size too large");
  if (K % 16 != 0 || N % 16 != 0)
    return fail(FP8_ERR_VALUE, n + ": K and N must be multiples of 16");
  if (recipe == 2 && K % 128 != 0)
    return fail(FP8_ERR_VALUE, n + ": the blockwise recipe needs K % 128 == 0");
  if (recipe == 4 && (K == 0 || K % 32 != 0))
    return fail(FP8_ERR_VALUE, n + ": MXFP8 needs K to be a positive multiple of 32");
  if (M_total == 0 || N == 0) {
    t_last_error.clear();
    return FP8_OK;
  }
  if (out == nullptr || (K > 0 && (a == nullptr || b_experts == nullptr ||
                                   scale_a == nullptr || scale_b == nullptr)))
    return fail(FP8_ERR_VALUE, n + ": null pointer");
  if (!aligned(out, 16) || (a && !aligned(a, 16)) || (b_experts && !aligned(b_experts, 16)) ||
      (scale_a && !aligned(scale_a, 16)) || (scale_b && !aligned(scale_b, 16)) ||
      !aligned(offs, 4))
    return fail(FP8_ERR_VALUE, n + ": pointers must be 16-byte aligned");
  DeviceInfo* d = nullptr;
  fp8_status s = device_info(&d);
  if (s != FP8_OK) return s;
  std::string err;
  fp8sm::LaunchCtx ctx = make_ctx(d, stream, &err);
  cudaError_t e = fp8sm::launch_grouped_scaled_mm(a, b_experts, M_total, N, K, E,
                                                  scale_a, scale_b, offs, recipe,
                                                  out_dtype == FP8_OUT_F32, out, ctx);
  return finish_launch(e, err, name);
}

}  // namespace

fp8_status fp8_grouped_scaled_mm(const void* a, const void* b_experts,
                                 int64_t M_total, int64_t N, int64_t K,
                                 int32_t E, const float* scale_a,
                                 const float* scale_b, const int32_t* offs,
                                 fp8_out_dtype out_dtype, void* out,
                                 fp8_stream_t stream) {
  return grouped_common("fp8_grouped_scaled_mm", 1, a, b_experts, M_total, N, K, E, scale_a,
                        scale_b, offs, out_dtype, out, stream);
}

fp8_status fp8_grouped_scaled_mm_blockwise(const void* a, const void* b_experts,
                                           int64_t M_total, int64_t N, int64_t K,
                                           int32_t E, const float* scale_a,
                                           const float* scale_b, const int32_t* offs,
                                           fp8_out_dtype out_dtype, void* out,
                                           fp8_stream_t stream) {
  return grouped_common("fp8_grouped_scaled_mm_blockwise", 2, a, b_experts, M_total, N, K, E,
                        scale_a, scale_b, offs, out_dtype, out, stream);
}

fp8_status fp8_grouped_scaled_mm_mx(const void* a, const void* b_experts, int64_t M_total,
                                    int64_t N, int64_t K, int32_t E,
                                    const void* scale_a_e8m0, const void* scale_b_e8m0,
                                    const int32_t* offs, fp8_out_dtype out_dtype, void* out,
                                    fp8_stream_t stream) {
  return grouped_common("fp8_grouped_scaled_mm_mx", 4, a, b_experts, M_total, N, K, E,
                        static_cast<const float*>(scale_a_e8m0),
                        static_cast<const float*>(scale_b_e8m0), offs, out_dtype, out, stream);
}

int64_t fp8_grouped_padded_tokens(int64_t tokens, int32_t E) {
  if (tokens < 0 || E < 1) return 0;
  return fp8sm::grouped_padded_tokens(tokens, E);
}

fp8_status fp8_quantize_transposed_grouped(const void* x_bf16, int64_t tokens, int64_t cols,
                                           int64_t ld_x, const int32_t* offs, int32_t E,
                                           void* out_fp8, float* out_scales,
                                           fp8_stream_t stream) {
  const char* n = "fp8_quantize_transposed_grouped";
  if (tokens < 0 || cols < 0) return fail(FP8_ERR_VALUE, std::string(n) + ": negative size");
  if (tokens >= (int64_t(1) << 31) || cols >= (int64_t(1) << 31))
    return fail(FP8_ERR_VALUE, std::string(n) + ": size too large");
  if (E < 1 || E > 2048)
    return fail(FP8_ERR_VALUE, std::string(n) + ": expert count must be in [1, 2048]");
  if (cols % 8 != 0 || ld_x % 8 != 0 || ld_x < cols)
    return fail(FP8_ERR_VALUE,
                std::string(n) + ": cols and ld_x must be multiples of 8, ld_x >= cols");
  if (offs == nullptr) return fail(FP8_ERR_VALUE, std::string(n) + ": offs is required");
  if (tokens == 0 || cols == 0) {
    t_last_error.clear();
    return FP8_OK;
  }
  if (x_bf16 == nullptr || out_fp8 == nullptr || out_scales == nullptr)
    return fail(FP8_ERR_VALUE, std::string(n) + ": null pointer");
  if (!aligned(x_bf16, 16) || !aligned(out_fp8, 16) || !aligned(out_scales, 4) ||
      !aligned(offs, 4))
    return fail(FP8_ERR_VALUE, std::string(n) + ": misaligned pointer");
  DeviceInfo* d = nullptr;
  fp8_status s = device_info(&d);
  if (s != FP8_OK) return s;
  std::string err;
  fp8sm::LaunchCtx ctx = make_ctx(d, stream, &err);
  cudaError_t e = fp8sm::launch_quantize_transposed_grouped(x_bf16, tokens, cols, ld_x, offs, E,
                                                            out_fp8, out_scales, ctx);
  return finish_launch(e, err, n);
}

fp8_status fp8_grouped_scaled_mm_wgrad(const void* a_t, const void* b_t, int64_t M, int64_t N,
                                       int64_t tokens, int32_t E, const float* scale_a,
                                       const float* scale_b, const int32_t* offs,
                                       fp8_out_dtype out_dtype, void* out, fp8_stream_t stream) {
  const std::string n("fp8_grouped_scaled_mm_wgrad");
  if (out_dtype != FP8_OUT_BF16 && out_dtype != FP8_OUT_F32)
    return fail(FP8_ERR_VALUE, n + ": unknown out_dtype");
  if (offs == nullptr) return fail(FP8_ERR_VALUE, n + ": offs is required");
  if (M < 0 || N < 0 || tokens < 0 || E < 1 || E > 65535)
    return fail(FP8_ERR_VALUE, n + ": bad size or expert count");
  if (M >= (int64_t(1) << 31) || N >= (int64_t(1) << 31) || tokens >= (int64_t(1) << 31))
    return fail(FP8_ERR_VALUE, n + ": size too large");
  if (M % 128 != 0) return fail(FP8_ERR_VALUE, n + ": M must be a multiple of 128");
  if (N % 16 != 0) return fail(FP8_ERR_VALUE, n + ": N must be a multiple of 16");
  if (M == 0 || N == 0) {
    t_last_error.clear();
    return FP8_OK;
  }
  if (a_t == nullptr || b_t == nullptr || scale_a == nullptr || scale_b == nullptr ||
      out == nullptr)
    return fail(FP8_ERR_VALUE, n + ": null pointer");
  if (!aligned(a_t, 16) || !aligned(b_t, 16) || !aligned(scale_a, 16) || !aligned(scale_b, 16) ||
      !aligned(out, 16) || !aligned(offs, 4))
    return fail(FP8_ERR_VALUE, n + ": pointers must be 16-byte aligned");
  DeviceInfo* d = nullptr;
  fp8_status s = device_info(&d);
  if (s != FP8_OK) return s;
  std::string err;
  fp8sm::LaunchCtx ctx = make_ctx(d, stream, &err);
  const int64_t P = fp8sm::grouped_padded_tokens(tokens, E);
  cudaError_t e = fp8sm::launch_grouped_wgrad(a_t, b_t, M, N, P, tokens, E, scale_a, scale_b,
                                              offs, out_dtype == FP8_OUT_F32, out, ctx);
  return finish_launch(e, err, n.c_str());
}

fp8_status fp8_get_device_status(fp8_stream_t stream) {
  DeviceInfo* d = nullptr;
  fp8_status s = device_info(&d);
  if (s != FP8_OK) return s;
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "fp8_get_device_status: sync");
  uint32_t w[2] = {0, 0};
  e = cudaMemcpy(w, d->status, sizeof(w), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "fp8_get_device_status: read");
  const uint32_t zero[2] = {0, 0};
  e = cudaMemcpy(d->status, zero, sizeof(zero), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "fp8_get_device_status: clear");
  if (w[0] == 0) {
    t_last_error.clear();
    return FP8_OK;
  }
  return fail(static_cast<fp8_status>(w[0]),
              "device status " + std::to_string(w[0]) + " recorded at site " +
                  std::to_string(w[1]));
}

fp8_status fp8_debug_timeout_probe(uint32_t limit_us, fp8_stream_t stream) {
  if (limit_us < 1 || limit_us > 2000000)
    return fail(FP8_ERR_VALUE, "fp8_debug_timeout_probe: limit_us out of range");
  DeviceInfo* d = nullptr;
  fp8_status s = device_info(&d);
  if (s != FP8_OK) return s;
  std::string err;
  fp8sm::LaunchCtx ctx = make_ctx(d, stream, &err);
  return finish_launch(fp8sm::launch_timeout_probe(limit_us, ctx), err,
                       "fp8_debug_timeout_probe");
}

}  // extern "C"
