// Tensor-core fragment helpers shared by the readout and commit kernels.
//
// The stored state is contracted on the tensor cores with mma.sync m16n8k16
// (f16 operands, fp32 accumulation).  Codes are small integers, exact in
// f16; the fp32 right-hand vectors are split into hi + lo f16 parts after a
// power-of-two normalisation, so products are exact and the only rounding is
// the fp32 accumulation.
//
// Code -> fragment mapping (one warp, rows 16r..16r+15 of a d_v x D state,
// lane = 4g + t): the lane reads the codes of rows 16r+g and 16r+g+8 that
// cover key channels J_t (INT4: the contiguous range [D/4 t, D/4 (t+1));
// INT8: two ranges of D/8 starting at D/8 t and D/2 + D/8 t).  Since the
// contraction index may be permuted freely (the right-hand side is permuted
// the same way), each lane's codes go straight into its A fragment registers;
// kslot_of() gives, for every key channel j, the k-step and the position
// inside the lane's 4 f16 B values of that step.
#pragma once

#include "pace_internal.cuh"

namespace pace {

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Integer tensor-core products (exact int32 accumulation).
__device__ __forceinline__ void mma_s8s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_u8s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lop3_6a(uint32_t a, uint32_t b, uint32_t c) {
  // out = b ? (a ^ c) : c  (bitwise)
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// 8 INT4 codes (two's complement nibbles, nibble e = code 8m+e) -> 4 f16x2:
// p[0] = (c0, c4), p[1] = (c1, c5), p[2] = (c2, c6), p[3] = (c3, c7).
// Each nibble is flipped to offset binary and placed in the mantissa of
// 1024.0 (or 16x that for the odd nibbles), then the bias is removed exactly.
__device__ __forceinline__ void dequant_int4(uint32_t w, uint32_t (&p)[4]) {
  const uint32_t w8 = w >> 8;
  const __half2 bias = __half2half2(__ushort_as_half((unsigned short)0x6408));   // 1032
  const __half2 s16 = __half2half2(__ushort_as_half((unsigned short)0x2C00));    // 1/16
  const __half2 b72 = __half2half2(__ushort_as_half((unsigned short)0xD480));    // -72
  p[0] = h2u(__hsub2(u2h(lop3_6a(w, 0x000F000Fu, 0x64086408u)), bias));
  p[1] = h2u(__hfma2(u2h(lop3_6a(w, 0x00F000F0u, 0x64806480u)), s16, b72));
  p[2] = h2u(__hsub2(u2h(lop3_6a(w8, 0x000F000Fu, 0x64086408u)), bias));
  p[3] = h2u(__hfma2(u2h(lop3_6a(w8, 0x00F000F0u, 0x64806480u)), s16, b72));
}

// 4 INT8 codes (two's complement bytes) -> 2 f16x2: (c0, c1), (c2, c3).
__device__ __forceinline__ void dequant_int8(uint32_t w, uint32_t (&p)[2]) {
  const uint32_t x = w ^ 0x80808080u;
  const __half2 bias = __half2half2(__ushort_as_half((unsigned short)0x6480));   // 1152
  p[0] = h2u(__hsub2(u2h(prmt(x, 0x64646464u, 0x4140u)), bias));
  p[1] = h2u(__hsub2(u2h(prmt(x, 0x64646464u, 0x4342u)), bias));
}

// Fragment position of key channel j: k-step s and position pos in the
// lane-group's 4 B values of that step (order b0, b1, b2, b3 of the m16n8k16
// B fragment: k slots 2t, 2t+1, 2t+8, 2t+9).  t is the lane group holding j.
template <int D, int BITS>
__device__ __forceinline__ void kslot_of(int j, int& t, int& s, int& pos) {
  if (BITS == 4) {
    constexpr int CPL = D / 4;              // codes per lane per row
    t = j / CPL;
    const int w = j - t * CPL;              // offset inside the lane's range
    const int m = w >> 3, e = w & 7;        // word m, nibble e
    const int odd = (e >> 1) & 1;           // nibbles 2,3,6,7 -> second step of the word
    s = 2 * m + odd;
    const int d = e - 2 * odd;              // 0, 1, 4 or 5
    pos = d == 0 ? 0 : d == 4 ? 1 : d == 1 ? 2 : 3;
  } else {
    constexpr int H = D / 2, C = D / 8;     // two halves, chunks of D/8 codes
    const int half = j >= H ? 1 : 0;
    const int jj = j - half * H;
    t = jj / C;
    const int w = jj - t * C;
    s = (w >> 2) + half * (C / 4);
    pos = w & 3;
  }
}

// Inverse of kslot_of: the key channel at (lane group t, k-step s, pos).
template <int D, int BITS>
__device__ __forceinline__ int jof(int t, int s, int pos) {
  if (BITS == 4) {
    const int base = (D / 4) * t + 8 * (s >> 1) + 2 * (s & 1);
    return base + (pos == 0 ? 0 : pos == 1 ? 4 : pos == 2 ? 1 : 5);
  }
  constexpr int WPC = D / 32;               // words per chunk
  const int base = s < WPC ? (D / 8) * t + 4 * s : D / 2 + (D / 8) * t + 4 * (s - WPC);
  return base + pos;
}

// Byte offsets (inside one code row) of the lane-group-t chunks.
template <int D, int BITS>
__device__ __forceinline__ int chunk_offset(int t, int c) {
  if (BITS == 4) return t * (D / 8);                 // one chunk of D/8 bytes
  return c * (D / 2) + t * (D / 8);                  // two chunks of D/8 bytes
}

// ---- small vector I/O: EPL consecutive elements per lane -------------------

template <int EPL, bool BF16>
struct Raw {
  static constexpr int BYTES = EPL * (BF16 ? 2 : 4);
  static constexpr int WORDS = BYTES < 4 ? 1 : BYTES / 4;
  uint32_t w[WORDS];

  __device__ __forceinline__ void load(const void* base, size_t elem) {
    const uint8_t* p = reinterpret_cast<const uint8_t*>(base) + elem * (BF16 ? 2 : 4);
    if (BYTES == 16) {
      uint4 v = *reinterpret_cast<const uint4*>(p);
      w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
    } else if (BYTES == 8) {
      uint2 v = *reinterpret_cast<const uint2*>(p);
      w[0] = v.x; w[1] = v.y;
    } else if (BYTES == 4) {
      w[0] = *reinterpret_cast<const uint32_t*>(p);
    } else {
      w[0] = *reinterpret_cast<const uint16_t*>(p);
    }
  }
  __device__ __forceinline__ void store(void* base, size_t elem) const {
    uint8_t* p = reinterpret_cast<uint8_t*>(base) + elem * (BF16 ? 2 : 4);
    if (BYTES == 16) {
      *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    } else if (BYTES == 8) {
      *reinterpret_cast<uint2*>(p) = make_uint2(w[0], w[1]);
    } else if (BYTES == 4) {
      *reinterpret_cast<uint32_t*>(p) = w[0];
    } else {
      *reinterpret_cast<uint16_t*>(p) = (uint16_t)w[0];
    }
  }
  // element e read as fp16 (the 16-bit layout shared with bf16)
  __device__ __forceinline__ float get_half(int e) const {
    const uint32_t x = w[e >> 1];
    return __half2float(__ushort_as_half((unsigned short)((e & 1) ? (x >> 16) : (x & 0xffffu))));
  }
  __device__ __forceinline__ float get(int e) const {
    if (BF16) {
      const uint32_t x = w[e >> 1];
      return __uint_as_float((e & 1) ? (x & 0xffff0000u) : (x << 16));
    }
    return __uint_as_float(w[e]);
  }
};

template <int EPL, bool BF16>
__device__ __forceinline__ void load_f(const void* base, size_t elem, float (&out)[EPL]) {
  Raw<EPL, BF16> r;
  r.load(base, elem);
#pragma unroll
  for (int e = 0; e < EPL; ++e) out[e] = r.get(e);
}

// ---- code chunks: lane-group slices of 16 rows -----------------------------

template <int BYTES>
__device__ __forceinline__ void ldg_stream(const uint8_t* p, uint32_t* w) {
  if (BYTES == 16) {
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "l"(p));
  } else if (BYTES == 8) {
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                 : "=r"(w[0]), "=r"(w[1]) : "l"(p));
  } else {
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(w[0]) : "l"(p));
  }
}

// Codes of rows 16r+g and 16r+g+8 held by lane (g, t).
template <int D, int BITS>
struct RowBlock {
  static constexpr int CHUNK = D / 8;                 // bytes per chunk
  static constexpr int CW = CHUNK / 4;                // words per chunk
  static constexpr int NCH = BITS == 4 ? 1 : 2;       // chunks per row
  static constexpr int ROWB = D * BITS / 8;           // bytes per code row
  uint32_t w[2][NCH * CW];                            // [row g | row g+8][words]

  __device__ __forceinline__ void load(const uint8_t* rec, int r, int g, int t) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint8_t* row = rec + (size_t)(16 * r + g + 8 * h) * ROWB;
#pragma unroll
      for (int c = 0; c < NCH; ++c) ldg_stream<CHUNK>(row + chunk_offset<D, BITS>(t, c), &w[h][c * CW]);
    }
  }
};

// A fragment of k-step s (16 key channels) from a row block.
template <int D, int BITS>
__device__ __forceinline__ void a_frag(const RowBlock<D, BITS>& rb, int s, uint32_t (&a)[4]) {
  if (BITS == 4) {
    uint32_t pg[4], ph[4];
    dequant_int4(rb.w[0][s >> 1], pg);
    dequant_int4(rb.w[1][s >> 1], ph);
    const int o = 2 * (s & 1);
    a[0] = pg[o]; a[1] = ph[o]; a[2] = pg[o + 1]; a[3] = ph[o + 1];
  } else {
    uint32_t pg[2], ph[2];
    dequant_int8(rb.w[0][s], pg);
    dequant_int8(rb.w[1][s], ph);
    a[0] = pg[0]; a[1] = ph[0]; a[2] = pg[1]; a[3] = ph[1];
  }
}

}  // namespace pace
