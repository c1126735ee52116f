// Per-device status word written by kernels when they detect a problem they
// cannot report through a return value (a malformed offs array read on the
// device, a pipeline wait that ran past its limit).  Word 0 holds the first
// error code recorded since the last read, word 1 the site that recorded it.
#pragma once

#include <stdint.h>

namespace fp8sm {

// Values match fp8_status in include/fp8sm.h.
enum : uint32_t {
  FP8_DEV_OK = 0,
  FP8_DEV_VALUE = 1,
  FP8_DEV_TIMEOUT = 4,
};

// Sites (which wait or check gave up), for diagnostics.
enum : uint32_t {
  SITE_PRODUCER_EMPTY = 1,
  SITE_MMA_FULL = 2,
  SITE_MMA_ACC_EMPTY = 3,
  SITE_EPI_ACC_FULL = 4,
  SITE_TEARDOWN = 5,
  SITE_GRID_BARRIER = 6,
  SITE_OFFS = 7,
  SITE_PROBE = 8,
  SITE_SCALE_EMPTY = 9,
  SITE_EPI_SCALE_FULL = 10,
  SITE_BOUNDS = 11,  // a copy index outside its buffer (checked before the copy)
  SITE_QUANT_TMA = 12,  // a quantizer waiting for a tile its TMA load brings
};

// Wait limit for every pipeline wait inside the GEMM / quantize kernels.
// A healthy wait is microseconds; one second means something is wrong.
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

#if defined(__CUDACC__)
__device__ __forceinline__ void record_status(uint32_t* status, uint32_t code,
                                              uint32_t site) {
  if (status == nullptr) return;
  if (atomicCAS(status, 0u, code) == 0u) atomicExch(status + 1, site);
}
#endif

}  // namespace fp8sm
