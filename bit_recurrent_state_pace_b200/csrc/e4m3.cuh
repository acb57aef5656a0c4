// FP8 E4M3 values of the buffered k, v rows of a pure-write-window pool:
// CUDA's conversions, round to nearest even, saturating at +-448.
#pragma once

#include <cuda_fp8.h>

#include "pace_internal.cuh"

namespace pace {

__device__ __forceinline__ uint8_t e4m3_code(float x) {
  return (uint8_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ float e4m3_value(uint32_t code) {
  return __half2float(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)(code & 0xffu), __NV_E4M3)));
}

__device__ __forceinline__ float e4m3_round(float x) { return e4m3_value(e4m3_code(x)); }

// Element idx of a buffered row: io dtype, or E4M3 bytes (R8).
template <bool R8>
__device__ __forceinline__ float row_at(const uint8_t* base, int idx, bool bf16) {
  if (R8) return e4m3_value(base[idx]);
  if (bf16) return __uint_as_float(((uint32_t)reinterpret_cast<const uint16_t*>(base)[idx]) << 16);
  return reinterpret_cast<const float*>(base)[idx];
}

}  // namespace pace
