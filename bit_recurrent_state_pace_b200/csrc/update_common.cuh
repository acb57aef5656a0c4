// Small helpers shared by the kernels that update and re-encode a state on
// the tensor cores (period commit, chunked prefill).
#pragma once

#include "encode.cuh"
#include "frag.cuh"

namespace pace {

// floor(log2(m)) for a positive normal float, from its exponent bits
__device__ __forceinline__ int exp2_floor(float m) { return (int)((__float_as_uint(m) >> 23) & 0xffu) - 127; }
// 2^e for e in [-126, 127], exact
__device__ __forceinline__ float pow2i(int e) { return __uint_as_float((uint32_t)(127 + e) << 23); }

// max that returns NaN if either input is NaN
__device__ __forceinline__ float max_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// element idx of an io-dtype array in shared or global memory, as float
__device__ __forceinline__ float io_at(const uint8_t* base, int idx, bool bf16) {
  if (bf16) return __uint_as_float(((uint32_t)reinterpret_cast<const uint16_t*>(base)[idx]) << 16);
  return reinterpret_cast<const float*>(base)[idx];
}

// Offset codes of two values, one per f16 half, in that half's low byte:
// fast path x * (1/s) + (1032 | 1152) rounded to f16 (round half to even).
template <int BITS>
__device__ __forceinline__ uint32_t magic_fast(float a, float b, float qa, float qb) {
  const float M = BITS == 4 ? 1032.f : 1152.f;
  const float2 r = __ffma2_rn(make_float2(a, b), make_float2(qa, qb), make_float2(M, M));
  return h2u(__floats2half2_rn(r.x, r.y));
}

// Same layout with the exact fp32 divide of the encoder (non-finite or
// clamped groups).
template <int BITS>
__device__ __forceinline__ uint32_t magic_exact(float a, float b, float sa, float sb) {
  const int qmax = BITS == 4 ? 7 : 127, off = BITS == 4 ? 8 : 128;
  const uint32_t ca = (uint32_t)(encode_value(a, sa, qmax) + off);
  const uint32_t cb = (uint32_t)(encode_value(b, sb, qmax) + off);
  return (0x6400u | ca) | ((0x6400u | cb) << 16);
}

}  // namespace pace
