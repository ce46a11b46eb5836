// Device helpers shared by the kernels: status word, bounded waits, loads.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace tsa {

// First error wins; later errors leave the recorded code unchanged.
__device__ __forceinline__ void record_status(uint32_t* status, uint32_t code) {
  atomicCAS(status, 0u, code);
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Sortable key for a float: larger float -> larger unsigned key, and -0.0 is
// folded onto +0.0 so that the two compare equal.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Spin on a global flag with a poll budget.  Returns true if the flag became
// non-zero, false if the budget ran out (the caller records TSA_ERR_TIMEOUT).
__device__ __forceinline__ bool bounded_wait_flag(const volatile uint32_t* flag, uint64_t limit) {
  for (uint64_t i = 0; i < limit; ++i) {
    if (*flag != 0u) return true;
    __nanosleep(64);
  }
  return *flag != 0u;
}

}  // namespace tsa
