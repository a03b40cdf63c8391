// Definitions shared by every kernel of the library (one translation unit).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "dora.h"

namespace dora {

// First error recorded by any kernel on this device (0 = none); read and
// cleared by dora_get_device_status().
__device__ int g_device_status;

__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_device_status, 0, code); }

// DORA_DEBUG builds check the index of every computed-address global store:
// an out-of-range one is skipped and recorded as DORA_ERR_BOUNDS (never a
// trap or an assert).  Other builds compile the check away.
#ifdef DORA_DEBUG
__device__ __forceinline__ bool bounds_ok(bool ok) {
  if (!ok) record_error(DORA_ERR_BOUNDS);
  return ok;
}
#define DORA_BOUNDS_OK(cond) (::dora::bounds_ok(cond))
#else
#define DORA_BOUNDS_OK(cond) true
#endif

// A bound on waits that must end (draining copies or MMAs already issued),
// independent of the configurable timeout.
constexpr unsigned long long kDrainTimeoutNs = 200000000ull;  // 0.2 s

__host__ __device__ __forceinline__ long long ceil_div_ll(long long a, long long b) {
  return (a + b - 1) / b;
}
__host__ __device__ __forceinline__ int round_up_int(int a, int b) { return (a + b - 1) / b * b; }

// bf16 <-> fp32 on raw 16-bit patterns.
__device__ __forceinline__ float bf16lo_to_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint16_t f32_to_bf16_rn(float x) {
  __nv_bfloat16 v = __float2bfloat16_rn(x);
  return *reinterpret_cast<uint16_t*>(&v);
}

}  // namespace dora
