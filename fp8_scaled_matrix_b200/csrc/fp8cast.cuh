// The dynamic quantizer's per-group arithmetic, shared by the quantize
// kernels and the GEMM epilogue that quantizes its result ("per-token
// scaling for fp8 linear", Highlights: amax -> scale -> pre-scaled input ->
// e4m3 cast):
//   a = max(amax, 1e-12);  scale = a / 448;  inv = 448 / a
//   q = cvt.rn.satfinite.e4m3(x * inv)
// Every step is one IEEE fp32 operation (no FMA contraction, no fast math).
#pragma once

#include <cuda_fp8.h>
#include <stdint.h>

namespace fp8sm {

constexpr float kE4M3Max = 448.0f;
constexpr float kEps = 1e-12f;

struct ScalePair {
  float s;    // dequantization multiplier, stored
  float inv;  // quantization multiplier
};

__device__ __forceinline__ ScalePair scales_from_amax(float amax) {
  const float a = fmaxf(amax, kEps);
  return {__fdiv_rn(a, kE4M3Max), __fdiv_rn(kE4M3Max, a)};
}

// Two fp32 values -> two e4m3 codes (low byte = first value).
__device__ __forceinline__ uint32_t cast_f32x2(float a, float b, float inv) {
  const float2 y = make_float2(__fmul_rn(a, inv), __fmul_rn(b, inv));
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(y, __NV_SATFINITE, __NV_E4M3));
}

}  // namespace fp8sm
