// Channel-aligned absmax encoder shared by the quantize, pool-load and commit
// kernels ("PACE: A New 4-Bit Recurrent State Quantization Method ...",
// section "Channel-Aligned Encoding: Exploiting State Column Structure";
// "PACE: four-bit recurrent state by rounding less often", TL;DR (2)-(3)).
//
// Reading of the encoding (the pages give no formula): per group, amax =
// max|x|; s32 = amax / qmax in fp32 (IEEE divide, round to nearest); the FP16
// scale s16 = round-to-nearest-even(s32), raised to the smallest subnormal
// 2^-24 when a nonzero amax would round to 0 and clamped to 65504 on
// overflow; codes = clamp(rint_half_even(x / s16), -qmax, qmax) with an IEEE
// fp32 divide.  A group holding NaN/Inf gets scale NaN and codes 0.
#pragma once

#include "pace_internal.cuh"

namespace pace {

struct GroupScale {
  uint16_t bits;  // fp16 bit pattern stored in the record
  float sf;       // float(s16), or 0 for an all-zero / non-finite group
};

__device__ __forceinline__ GroupScale group_scale(float amax, bool finite, int qmax,
                                                  uint32_t* flags) {
  GroupScale r;
  if (!finite) {
    r.bits = 0x7E00;
    r.sf = 0.f;
    if (flags) atomicOr(flags, PACE_FLAG_NONFINITE);
    return r;
  }
  const float s32 = __fdiv_rn(amax, (float)qmax);
  uint16_t hb = __half_as_ushort(__float2half_rn(s32));
  if (amax > 0.f && hb == 0) hb = 1;
  if (hb == 0x7C00) {
    hb = 0x7BFF;
    if (flags) atomicOr(flags, PACE_FLAG_SCALE_OVERFLOW);
  }
  r.bits = hb;
  r.sf = __half2float(__ushort_as_half(hb));
  return r;
}

// The fast encode of the update kernels (x * (1 / s16) rounded by a
// magic-number add, no clamp) gives the exact encoder's codes, up to exact
// ties, when every |x| <= amax has |x / s16| < qmax + 1/2.  That holds when
// s16 rounds amax / qmax to a normal fp16 (relative error <= 2^-11) but can
// fail for a scale in the fp16 subnormal range or raised to 2^-24 (amax far
// below 1e-4); such groups, and non-finite ones, take the exact encoder.
__device__ __forceinline__ bool fast_encode_ok(float amax, const GroupScale& gs, int qmax) {
  if (!isfinite(amax)) return false;
  if (gs.sf == 0.f) return true;   // all-zero group: every code is 0
  return amax * __frcp_rn(gs.sf) < (float)qmax + 0.25f;
}

__device__ __forceinline__ int encode_value(float x, float sf, int qmax) {
  if (sf == 0.f) return 0;
  float c = rintf(__fdiv_rn(x, sf));
  c = fminf(fmaxf(c, (float)-qmax), (float)qmax);
  return (int)c;
}

__device__ __forceinline__ int decode_code(const uint8_t* codes, int row_bytes, int i, int j,
                                           int bits) {
  if (bits == 8) return (int)(int8_t)codes[(size_t)i * row_bytes + j];
  const uint8_t b = codes[(size_t)i * row_bytes + (j >> 1)];
  const int nib = (j & 1) ? (b >> 4) : (b & 0xF);
  return nib >= 8 ? nib - 16 : nib;
}

// Encode one d_v x d_k matrix reachable through get(i, j).  All threads of the
// block take part; sf_sm is shared scratch of max(d_k, d_v) floats.
template <class Get>
__device__ void encode_matrix(Get get, int d_k, int d_v, int bits, int axis, uint8_t* codes,
                              uint16_t* scales, uint32_t* flags, float* sf_sm) {
  const int qmax = bits == 4 ? 7 : 127;
  const int tid = threadIdx.x, nt = blockDim.x;
  if (axis == PACE_SCALE_COL) {
    for (int j = tid; j < d_k; j += nt) {
      float amax = 0.f;
      bool fin = true;
      for (int i = 0; i < d_v; ++i) {
        const float x = get(i, j);
        if (isfinite(x)) amax = fmaxf(amax, fabsf(x)); else fin = false;
      }
      const GroupScale gs = group_scale(amax, fin, qmax, flags);
      scales[j] = gs.bits;
      sf_sm[j] = gs.sf;
    }
  } else {
    const int lane = tid & 31, warp = tid >> 5, nw = nt >> 5;
    for (int i = warp; i < d_v; i += nw) {
      float amax = 0.f;
      bool fin = true;
      for (int j = lane; j < d_k; j += 32) {
        const float x = get(i, j);
        if (isfinite(x)) amax = fmaxf(amax, fabsf(x)); else fin = false;
      }
      for (int off = 16; off; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      fin = __all_sync(0xffffffffu, fin);
      if (lane == 0) {
        const GroupScale gs = group_scale(amax, fin, qmax, flags);
        scales[i] = gs.bits;
        sf_sm[i] = gs.sf;
      }
    }
  }
  __syncthreads();
  const int row_bytes = d_k * bits / 8;
  const int total = d_v * row_bytes;
  for (int idx = tid; idx < total; idx += nt) {
    const int i = idx / row_bytes, m = idx - i * row_bytes;
    if (bits == 8) {
      const float sf = axis == PACE_SCALE_COL ? sf_sm[m] : sf_sm[i];
      codes[idx] = (uint8_t)(int8_t)encode_value(get(i, m), sf, qmax);
    } else {
      const int j0 = 2 * m, j1 = 2 * m + 1;
      const float s0 = axis == PACE_SCALE_COL ? sf_sm[j0] : sf_sm[i];
      const float s1 = axis == PACE_SCALE_COL ? sf_sm[j1] : sf_sm[i];
      const int c0 = encode_value(get(i, j0), s0, qmax);
      const int c1 = encode_value(get(i, j1), s1, qmax);
      codes[idx] = (uint8_t)((c0 & 0xF) | ((c1 & 0xF) << 4));
    }
  }
}

}  // namespace pace
