// Per-token readout: one decode token for every (slot, head) of a pool.
//
// "PACE: A New 4-Bit Recurrent State Quantization Method ...", section
// "Periodic Rounding: Reducing Error Accumulation": decoded tokens wait in a
// small buffer and the stored state is rounded only once per period; "PACE:
// four-bit recurrent state by rounding less often", flowchart "New tokens ->
// Small buffer".  The output of the n-th buffered token is exact in chunk
// form from the stored state S~0 (the working state is never materialised):
//
//   o_n = S_n q_n = S~0 q^ + sum_s z_s v_s,   q^ = gamma_n q_n - sum_s z_s gamma_s k_s,
//   z = diag(beta) (I + A)^{-T} w,  w_s = gamma_{n/s} (k_s . q_n),
//   A[t][s] = beta_t gamma_{t/s} (k_t . k_s) for s < t,
//
// which follows from the UT/WY chunk form S_n = gamma_n S~0 + sum_s
// gamma_{n/s} u_s k_s^T, U = (I + A)^{-1} diag(beta) (V - diag(gamma) X^T),
// X = S~0 K^T, by moving (I + A)^{-1} to the readout side: one state-sized
// product (S~0 q^) per token.
//
// Design (B200): one warp owns one head at a time (no block barriers); heads
// are strided over a persistent grid in work order (4-bit heads first).
//  * Staging: everything of a head except its codes -- q, k, v of the token,
//    the fp16 scales, the n-1 buffered (k, v) rows, their gates and Gram
//    block -- is brought into the warp's shared-memory stage by 1-D bulk
//    copies (TMA, no multicast) one head ahead, completing on a per-stage
//    mbarrier; the chunk algebra then reads on-chip data only.
//  * State stream: the codes go from HBM (L2-prefetched one head ahead) with
//    coalesced 128-bit non-allocating loads straight into the A fragments of
//    the int8 tensor cores (mma.sync m16n8k32, s8 x s8 for INT8 codes; INT4
//    nibbles widened to offset bytes, u8 x s8), two 16-row blocks ahead; the
//    right-hand side q^ (times the column scales) enters as 22-bit fixed
//    point split into three base-256 digits, so the products are exact int32.
//  * The small n x n chunk algebra runs lane-parallel over tokens with warp
//    shuffles; k.k dot products of earlier buffered tokens are cached in the
//    buffer's Gram block, so each step computes only the 2n-1 new ones.
#include "e4m3.cuh"
#include "frag.cuh"
#include "tma.cuh"

namespace pace {

namespace {

constexpr int kWarpsPerBlock = 8;
constexpr int kThreads = kWarpsPerBlock * 32;
constexpr unsigned FULL = 0xffffffffu;

// ADAPT (commit threshold set): two more right-hand sides, a^ and b^, as two
// digits each (rows 3..4 and 5..6; row 7 zeros), for the accumulated-update
// norm: all three fit one n8 product.
template <int D, bool ADAPT>
struct alignas(16) WarpScratch {
  static constexpr int NDIG = ADAPT ? 8 : 4;
  uint8_t dig[NDIG][D];            // digits 0..2 of q^, then (ADAPT) 0..1 of a^ and b^; last row zeros
  float y[D];                      // S~0 q^ by row, before the row scale
  float ya[ADAPT ? D : 1];         // S~0 a^
  float yb[ADAPT ? D : 1];         // S~0 b^
  float A[PACE_MAX_PERIOD * PACE_MAX_PERIOD];   // period end: A[t][s]
  float gsb[3][PACE_MAX_PERIOD];                // period end: gamma_s, gamma_{P/s}, beta_s
};

// Right-hand side x (the lane's EPL key channels, times the column scales)
// as 22-bit fixed point, split into three balanced base-256 digits:
// x 2^e = d0 + 256 d1 + 65536 d2.  Writes digit rows dig[0..2] in the
// order the code fragments expect and returns 2^-e; dsum: the lane's digit
// sums (for the offset-byte correction of INT4 codes).
template <int D, int EPL, int BITS>
__device__ __forceinline__ float rhs_digits(const float (&x)[EPL], uint8_t (*dig)[D], int lane,
                                            int (&dsum)[3]) {
  float m = 0.f;
#pragma unroll
  for (int e = 0; e < EPL; ++e) m = fmaxf(m, fabsf(x[e]));
#pragma unroll
  for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, off));
  int ex = 0;
  if (m > 0.f && m < INFINITY) ex = max(-120, min(120, 21 - ilogbf(m)));
  const float up = ldexpf(1.f, ex);
  dsum[0] = dsum[1] = dsum[2] = 0;
  uint32_t dw[3] = {0u, 0u, 0u};    // digit bytes of this lane's EPL elements
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    const int Q = __float2int_rn(x[e] * up);
    const int d0 = (int)(int8_t)(Q & 0xff);
    const int r1 = (Q - d0) >> 8;
    const int d1 = (int)(int8_t)(r1 & 0xff);
    const int d2 = (r1 - d1) >> 8;
    dsum[0] += d0; dsum[1] += d1; dsum[2] += d2;
    dw[0] |= (uint32_t)(d0 & 0xff) << (8 * e);
    dw[1] |= (uint32_t)(d1 & 0xff) << (8 * e);
    dw[2] |= (uint32_t)(d2 & 0xff) << (8 * e);
  }
  if (BITS == 8) {
    // natural key-channel order
#pragma unroll
    for (int d = 0; d < 3; ++d) {
      uint8_t* dst = &dig[d][EPL * lane];
      if (EPL == 4) *reinterpret_cast<uint32_t*>(dst) = dw[d];
      else if (EPL == 2) *reinterpret_cast<uint16_t*>(dst) = (uint16_t)dw[d];
      else *dst = (uint8_t)dw[d];
    }
  } else {
    // within each group of 8 key channels: even offsets first, then odd
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const int j = EPL * lane + e, o = j & 7;
      const int at = (j & ~7) + ((o & 1) ? 4 + (o >> 1) : (o >> 1));
#pragma unroll
      for (int d = 0; d < 3; ++d) dig[d][at] = (uint8_t)(dw[d] >> (8 * e));
    }
  }
  return ldexpf(1.f, -ex);
}

// INT4 codes enter the tensor cores as offset bytes c + 8: the correction
// 8 sum(digits) per digit column (zero for INT8).
template <int BITS>
__device__ __forceinline__ void offset_corr(const int (&dsum)[3], int (&corr)[3]) {
#pragma unroll
  for (int d = 0; d < 3; ++d) {
    int v2 = dsum[d];
    if (BITS == 4) {
#pragma unroll
      for (int off = 16; off; off >>= 1) v2 += __shfl_xor_sync(FULL, v2, off);
    }
    corr[d] = BITS == 4 ? 8 * v2 : 0;
  }
}

// The same split with two digits (14-bit fixed point: x 2^e = d0 + 256 d1,
// |x 2^e| < 2^14), for the norm-tracking right-hand sides, where 14 bits are
// ample: they only decide when to commit, not what is committed.
template <int D, int EPL, int BITS>
__device__ __forceinline__ float rhs_digits2(const float (&x)[EPL], uint8_t (*dig)[D], int lane,
                                             int (&dsum)[2]) {
  float m = 0.f;
#pragma unroll
  for (int e = 0; e < EPL; ++e) m = fmaxf(m, fabsf(x[e]));
#pragma unroll
  for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, off));
  int ex = 0;
  if (m > 0.f && m < INFINITY) ex = max(-120, min(120, 13 - ilogbf(m)));
  const float up = ldexpf(1.f, ex);
  dsum[0] = dsum[1] = 0;
  uint32_t dw[2] = {0u, 0u};
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    const int Q = __float2int_rn(x[e] * up);
    const int d0 = (int)(int8_t)(Q & 0xff);
    const int d1 = (Q - d0) >> 8;
    dsum[0] += d0; dsum[1] += d1;
    dw[0] |= (uint32_t)(d0 & 0xff) << (8 * e);
    dw[1] |= (uint32_t)(d1 & 0xff) << (8 * e);
  }
  if (BITS == 8) {
#pragma unroll
    for (int d = 0; d < 2; ++d) {
      uint8_t* dst = &dig[d][EPL * lane];
      if (EPL == 4) *reinterpret_cast<uint32_t*>(dst) = dw[d];
      else if (EPL == 2) *reinterpret_cast<uint16_t*>(dst) = (uint16_t)dw[d];
      else *dst = (uint8_t)dw[d];
    }
  } else {
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const int j = EPL * lane + e, o = j & 7;
      const int at = (j & ~7) + ((o & 1) ? 4 + (o >> 1) : (o >> 1));
#pragma unroll
      for (int d = 0; d < 2; ++d) dig[d][at] = (uint8_t)(dw[d] >> (8 * e));
    }
  }
  return ldexpf(1.f, -ex);
}

template <int BITS>
__device__ __forceinline__ void offset_corr2(const int (&dsum)[2], int (&corr)[2]) {
#pragma unroll
  for (int d = 0; d < 2; ++d) {
    int v2 = dsum[d];
    if (BITS == 4) {
#pragma unroll
      for (int off = 16; off; off >>= 1) v2 += __shfl_xor_sync(FULL, v2, off);
    }
    corr[d] = BITS == 4 ? 8 * v2 : 0;
  }
}

// B fragments (k32 x n8) of one right-hand-side set: column g of lane (g, t)
// is digit row row_of_g of `dig`.
template <int D, int BITS>
__device__ __forceinline__ void load_bfrag(const uint8_t* src, int t, uint32_t (&bfr)[D / 32][2]) {
  constexpr int NC = D / 32;
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    if (BITS == 4) {
      const int at = (D / 4) * t + 8 * c;
      bfr[c][0] = *reinterpret_cast<const uint32_t*>(src + at);
      bfr[c][1] = *reinterpret_cast<const uint32_t*>(src + at + 4);
    } else {
      const int m0 = 2 * c, m1 = 2 * c + 1;
      const int j0 = m0 < NC ? (D / 8) * t + 4 * m0 : D / 2 + (D / 8) * t + 4 * (m0 - NC);
      const int j1 = m1 < NC ? (D / 8) * t + 4 * m1 : D / 2 + (D / 8) * t + 4 * (m1 - NC);
      bfr[c][0] = *reinterpret_cast<const uint32_t*>(src + j0);
      bfr[c][1] = *reinterpret_cast<const uint32_t*>(src + j1);
    }
  }
}

// One warp's shared-memory stage for one head (byte offsets, all 16-aligned).
template <int D, bool BF16, int PMAX>
struct Stage {
  static constexpr int ESZ = BF16 ? 2 : 4;
  static constexpr int Q = 0, K = D * ESZ, V = 2 * D * ESZ;     // token inputs
  static constexpr int SC = 3 * D * ESZ;                          // fp16 scales [D]
  static constexpr int KV = SC + 2 * D;                           // rows [PMAX-1][k | v]
  static constexpr int AB = KV + (PMAX - 1) * 2 * D * ESZ;        // gates [PMAX][2]
  static constexpr int G = AB + (2 * PMAX * ESZ + 15) / 16 * 16;  // Gram block
  static constexpr int BYTES = G + (4 * (PMAX * (PMAX + 1) + 2) + 15) / 16 * 16;
  // two stages (copies one head ahead) while 8 warps fit twice per SM
  static constexpr int N = 2 * 8 * 2 * BYTES <= 160 * 1024 ? 2 : 1;
};

// EPL consecutive elements (from element index elem) of buffered rows: io
// dtype, or E4M3 bytes (R8).
template <int EPL, bool BF16, bool R8>
__device__ __forceinline__ void load_row(const uint8_t* base, size_t elem, float (&out)[EPL]) {
  if constexpr (R8) {
    const uint8_t* p = base + elem;
    const uint32_t w = EPL == 4 ? *reinterpret_cast<const uint32_t*>(p)
                     : EPL == 2 ? (uint32_t)*reinterpret_cast<const uint16_t*>(p) : (uint32_t)*p;
#pragma unroll
    for (int e = 0; e < EPL; ++e) out[e] = e4m3_value(w >> (8 * e));
  } else {
    load_f<EPL, BF16>(base, elem, out);
  }
}

// Lane L ends with the warp-wide sum of value index (L mod V).
template <int V>
__device__ __forceinline__ float transpose_reduce(float (&v)[V], int lane) {
#pragma unroll
  for (int c = V; c > 1; c >>= 1) {
    const int o = c >> 1;
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int k = 0; k < c / 2; ++k) {
      const float send = upper ? v[k] : v[k + c / 2];
      const float keep = upper ? v[k + c / 2] : v[k];
      v[k] = keep + __shfl_xor_sync(FULL, send, o);
    }
  }
  float r = v[0];
#pragma unroll
  for (int o = V; o < 32; o <<= 1) r += __shfl_xor_sync(FULL, r, o);
  return r;
}

// EXACT: the pool's period equals PMAX (compile-time loop bounds over tokens).
// ADAPT: a commit threshold is set: also track the accumulated update's norm
// and mark the head for an early commit when it reaches the threshold.
// R8: buffered k, v are E4M3 bytes; the token's k, v are rounded to E4M3 as
// they are buffered and used.
template <int D, bool BF16, int PMAX, int BITS, bool EXACT, bool ADAPT, bool R8>
__device__ __forceinline__ void decode_head(const PoolDev& p, int head, int n, const void* __restrict__ q,
                                            const void* __restrict__ k, const void* __restrict__ v,
                                            const void* __restrict__ alpha,
                                            const void* __restrict__ beta, float* __restrict__ o,
                                            WarpScratch<D, ADAPT>& scr, const uint8_t* stg, int lane) {
  using ST = Stage<D, BF16, PMAX>;
  constexpr int EPL = D / 32, RB = D / 16, PF = 2;
  constexpr int ESZ = BF16 ? 2 : 4;
  const int g = lane >> 2, t = lane & 3;
  const int h = head % p.H, b = head / p.H;
  const int P = EXACT ? PMAX : p.P;
  const uint8_t* rec = p.state + (size_t)b * p.slot_stride + p.rec_off[h];

  // 1. start streaming the first row blocks of codes
  RowBlock<D, BITS> rbuf[PF];
#pragma unroll
  for (int r = 0; r < PF; ++r) rbuf[r].load(rec, r, g, t);

  // 2. this token's inputs and the head's scales (lane holds elements EPL*lane..)
  const size_t e0 = (size_t)EPL * lane;
  Raw<EPL, BF16> k_raw, v_raw;
  k_raw.load(stg + ST::K, e0);
  v_raw.load(stg + ST::V, e0);
  float qf[EPL], kf[EPL], vf[EPL], sc[EPL];
  load_f<EPL, BF16>(stg + ST::Q, e0, qf);
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    kf[e] = R8 ? e4m3_round(k_raw.get(e)) : k_raw.get(e);
    vf[e] = R8 ? e4m3_round(v_raw.get(e)) : v_raw.get(e);
  }
  const float a_n = load_io(alpha, head, BF16 ? PACE_IO_BF16 : PACE_IO_F32);
  const float b_n = load_io(beta, head, BF16 ? PACE_IO_BF16 : PACE_IO_F32);
  {
    Raw<EPL, true> s_raw;   // fp16 scales share the bf16 byte layout
    s_raw.load(stg + ST::SC, (size_t)EPL * lane);
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const uint32_t x = s_raw.w[e >> 1];
      sc[e] = __half2float(__ushort_as_half((unsigned short)((e & 1) ? (x >> 16) : (x & 0xffff))));
    }
  }

  // 3. dot products with the buffered keys: k_n.k_s and q.k_s
  const size_t row_elems = 2 * (size_t)D;
  constexpr int RESZ = R8 ? 1 : ESZ;   // bytes per buffered element
  const uint8_t* kv_head = p.kv + (size_t)head * P * row_elems * RESZ;
  const uint8_t* kv_stg = stg + ST::KV;
  float part[2 * PMAX];
#pragma unroll
  for (int i = 0; i < 2 * PMAX; ++i) part[i] = 0.f;
#pragma unroll
  for (int s = 0; s < PMAX; ++s) {
    if (s < n - 1) {
      float ks[EPL];
      load_row<EPL, BF16, R8>(kv_stg, s * row_elems + (size_t)EPL * lane, ks);
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        part[s] = fmaf(kf[e], ks[e], part[s]);
        part[PMAX + s] = fmaf(qf[e], ks[e], part[PMAX + s]);
      }
    } else if (s == n - 1) {
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        part[PMAX + s] = fmaf(qf[e], kf[e], part[PMAX + s]);
        if (ADAPT) part[s] = fmaf(kf[e], kf[e], part[s]);
      }
    }
  }
  const float tot = transpose_reduce<2 * PMAX>(part, lane);
  // lane s < PMAX: gk = k_n . k_s (ADAPT: lane n-1 holds k_n . k_n); lane PMAX + s: q . k_s

  // 4. per-token decays / gates, lane s = token s (0-based); lanes >= n neutral
  float al = 1.f, be = 0.f;
  const uint8_t* ab_head = p.ab + (size_t)head * p.ab_stride;
  if (lane < n - 1) {
    Raw<2, BF16> ab;
    ab.load(stg + ST::AB, (size_t)lane * 2);
    al = ab.get(0);
    be = ab.get(1);
  } else if (lane == n - 1) {
    al = a_n;
    be = b_n;
  }
  float gcum = al;                                     // gamma through token s
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float x = __shfl_up_sync(FULL, gcum, off);
    if (lane >= off) gcum *= x;
  }
  float suf = __shfl_down_sync(FULL, al, 1);           // prod_{r > s} alpha_r
  if (lane == 31) suf = 1.f;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float x = __shfl_down_sync(FULL, suf, off);
    if (lane + off < 32) suf *= x;
  }
  const float gamma_n = __shfl_sync(FULL, gcum, n - 1);
  const float w_s = suf * __shfl_sync(FULL, tot, (lane + PMAX) & 31);

  // 5. column s of A: A[t][s] = beta_t gamma_{t/s} G[t][s], t > s
  const float* gram_head = reinterpret_cast<const float*>(p.gram + (size_t)head * p.gram_stride);
  float acol[PMAX];
  float run = 1.f;
#pragma unroll
  for (int tt = 0; tt < PMAX; ++tt) {
    const float at = __shfl_sync(FULL, al, tt);
    const float bt = __shfl_sync(FULL, be, tt);
    float G = 0.f;
    if (tt > lane) {
      run *= at;
      if (tt < n - 1) G = reinterpret_cast<const float*>(stg + ST::G)[tt * P + lane];
      else if (tt == n - 1) G = tot;
    }
    acol[tt] = (tt > lane && tt < n) ? bt * run * G : 0.f;
  }
  if ((ADAPT || n == P) && lane < PMAX) {   // kept for the period-end factors (step 12)
#pragma unroll
    for (int tt = 0; tt < PMAX; ++tt) scr.A[tt * PMAX + lane] = acol[tt];
    scr.gsb[0][lane] = gcum;
    scr.gsb[1][lane] = suf;
    scr.gsb[2][lane] = be;
  }
  // 6. backward substitution (I + A^T) y = w, lane-parallel over s.
  //    ADAPT: also the system of the first n-1 tokens for the query k_n with
  //    w'_s = gamma_{n/s} (k_s . k_n): then zeta = diag(beta) y' gives
  //    alpha_n S_{n-1} k_n = S~0 a^ + sum_s zeta_s v_s, a^ = gamma_n k_n - b^,
  //    b^ = sum_s zeta_s gamma_s k_s.
  float acc = w_s;
  float acc2 = ADAPT && lane < n - 1 ? suf * tot : 0.f;
#pragma unroll
  for (int tt = PMAX - 1; tt >= 0; --tt) {
    if (tt < n) {
      const float yt = __shfl_sync(FULL, acc, tt);
      if (lane < tt) acc = fmaf(-acol[tt], yt, acc);
    }
    if (ADAPT && tt < n - 1) {
      const float yt = __shfl_sync(FULL, acc2, tt);
      if (lane < tt) acc2 = fmaf(-acol[tt], yt, acc2);
    }
  }
  const float z = be * acc;              // z_s (0 on lanes >= n)
  const float zk = z * gcum;             // z_s gamma_s
  const float zeta = be * acc2;          // zeta_s (0 on lanes >= n - 1)
  const float zetak = zeta * gcum;

  // 7. q^ and the buffered-value term, lane-local over its EPL elements
  float qh[EPL], vt[EPL], bh[EPL], vt2[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    qh[e] = gamma_n * qf[e];
    vt[e] = 0.f;
    bh[e] = 0.f;
    vt2[e] = 0.f;
  }
#pragma unroll
  for (int s = 0; s < PMAX; ++s) {
    if (s < n) {
      const float zks = __shfl_sync(FULL, zk, s);
      const float zs = __shfl_sync(FULL, z, s);
      float ks[EPL], vs[EPL];
      if (s < n - 1) {
        load_row<EPL, BF16, R8>(kv_stg, s * row_elems + (size_t)EPL * lane, ks);
        load_row<EPL, BF16, R8>(kv_stg, s * row_elems + D + (size_t)EPL * lane, vs);
      } else {
#pragma unroll
        for (int e = 0; e < EPL; ++e) { ks[e] = kf[e]; vs[e] = vf[e]; }
      }
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        qh[e] = fmaf(-zks, ks[e], qh[e]);
        vt[e] = fmaf(zs, vs[e], vt[e]);
      }
      if (ADAPT && s < n - 1) {
        const float eks = __shfl_sync(FULL, zetak, s);
        const float es = __shfl_sync(FULL, zeta, s);
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          bh[e] = fmaf(eks, ks[e], bh[e]);
          vt2[e] = fmaf(es, vs[e], vt2[e]);
        }
      }
    }
  }

  // 8. right-hand sides (times the column scales) as digit rows
  const bool col = p.axis == PACE_SCALE_COL;
  float bv[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) bv[e] = col ? qh[e] * sc[e] : qh[e];
  int dsum[3], corr[3];
  const float down = rhs_digits<D, EPL, BITS>(bv, &scr.dig[0], lane, dsum);
  offset_corr<BITS>(dsum, corr);
  float down_a = 0.f, down_b = 0.f;
  int corr_a[2] = {0, 0}, corr_b[2] = {0, 0};
  if constexpr (ADAPT) {
    float av[EPL], bw[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const float ah = gamma_n * kf[e] - bh[e];
      av[e] = col ? ah * sc[e] : ah;
      bw[e] = col ? bh[e] * sc[e] : bh[e];
    }
    int ds2[2];
    down_a = rhs_digits2<D, EPL, BITS>(av, &scr.dig[3], lane, ds2);
    offset_corr2<BITS>(ds2, corr_a);
    down_b = rhs_digits2<D, EPL, BITS>(bw, &scr.dig[5], lane, ds2);
    offset_corr2<BITS>(ds2, corr_b);
  }
  __syncwarp();
  constexpr int NC = D / 32;           // k32 chunks
  // columns 0..2: q^ digits (3..7 zero); ADAPT: 3..4 a^ digits, 5..6 b^ digits, 7 zero
  uint32_t bfr[NC][2];
  if constexpr (ADAPT) load_bfrag<D, BITS>(&scr.dig[g][0], t, bfr);
  else load_bfrag<D, BITS>(&scr.dig[g < 3 ? g : 3][0], t, bfr);
  // accumulator columns 2t, 2t+1 of lane t: (d0, d1) for even t, (d2, -) for odd t
  const int cA = t == 0 ? corr[0] : t == 1 ? corr[2] : 0;
  const int cB = t == 0 ? corr[1] : 0;
  // ADAPT: the weight (256^digit) and offset correction of lane t's two
  // columns: t = 0: q^ d0, d1; t = 1: q^ d2, a^ d0; t = 2: a^ d1, b^ d0;
  // t = 3: b^ d1, zero.  Lane t then adds the first column of lane t + 1 to
  // its own and holds q^ (t = 0), a^ (t = 1) or b^ (t = 2).
  const float aw0 = t == 1 ? 65536.f : t == 0 ? 1.f : 256.f, aw1 = t == 0 ? 256.f : t == 3 ? 0.f : 1.f;
  const int ak0 = t == 0 ? corr[0] : t == 1 ? corr[2] : t == 2 ? corr_a[1] : corr_b[1];
  const int ak1 = t == 0 ? corr[1] : t == 1 ? corr_a[0] : t == 2 ? corr_b[0] : 0;

  // 9. y = S~0 (codes) x b on the int8 tensor cores (exact int32), 16 rows at a time
  // (unrolled by the prefetch depth only: a smaller loop body keeps the
  // instruction cache warm for the 16 warps of an SM)
#pragma unroll 1
  for (int r0 = 0; r0 < RB; r0 += PF)
#pragma unroll
  for (int rr = 0; rr < PF; ++rr) {
    const int r = r0 + rr;
    RowBlock<D, BITS> cur = rbuf[rr];
    if (r + PF < RB) rbuf[rr].load(rec, r + PF, g, t);
    int d[4] = {0, 0, 0, 0};
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      uint32_t a[4];
      if (BITS == 4) {
        const uint32_t w0 = cur.w[0][c], w1 = cur.w[1][c];
        a[0] = (w0 & 0x0F0F0F0Fu) ^ 0x08080808u;
        a[1] = (w1 & 0x0F0F0F0Fu) ^ 0x08080808u;
        a[2] = ((w0 >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
        a[3] = ((w1 >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
        mma_u8s8(d, a, bfr[c][0], bfr[c][1]);
      } else {
        a[0] = cur.w[0][2 * c];
        a[1] = cur.w[1][2 * c];
        a[2] = cur.w[0][2 * c + 1];
        a[3] = cur.w[1][2 * c + 1];
        mma_s8s8(d, a, bfr[c][0], bfr[c][1]);
      }
    }
    if constexpr (ADAPT) {
      const float v0 = aw0 * (float)(d[0] - ak0), v1 = aw1 * (float)(d[1] - ak1);
      const float u0 = aw0 * (float)(d[2] - ak0), u1 = aw1 * (float)(d[3] - ak1);
      const float pg = (t == 0 ? v0 + v1 : v1) + __shfl_down_sync(FULL, v0, 1);
      const float ph = (t == 0 ? u0 + u1 : u1) + __shfl_down_sync(FULL, u0, 1);
      if (t == 0) {
        scr.y[16 * r + g] = pg * down;
        scr.y[16 * r + g + 8] = ph * down;
      } else if (t == 1) {
        scr.ya[16 * r + g] = pg * down_a;
        scr.ya[16 * r + g + 8] = ph * down_a;
      } else if (t == 2) {
        scr.yb[16 * r + g] = pg * down_b;
        scr.yb[16 * r + g + 8] = ph * down_b;
      }
    } else {
      // digit columns: lane t = 0 holds d0, d1 and lane t = 1 holds d2 of q^
      const float wB = (t & 1) == 0 ? 256.f : 0.f, wA = (t & 1) == 0 ? 1.f : 65536.f;
      float pg = wA * (float)(d[0] - cA) + wB * (float)(d[1] - cB);
      float ph = wA * (float)(d[2] - cA) + wB * (float)(d[3] - cB);
      pg += __shfl_down_sync(FULL, pg, 1);
      ph += __shfl_down_sync(FULL, ph, 1);
      if (t == 0) {
        scr.y[16 * r + g] = pg * down;
        scr.y[16 * r + g + 8] = ph * down;
      }
    }
  }
  __syncwarp();

  // 10. o = (row scale) * y + sum_s z_s v_s
  {
    float out[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const float yv = scr.y[EPL * lane + e];
      out[e] = (col ? yv : yv * sc[e]) + vt[e];
    }
    float* op = o + (size_t)head * D + (size_t)EPL * lane;
    if (EPL == 4) *reinterpret_cast<float4*>(op) = make_float4(out[0], out[1], out[2], out[3]);
    else if (EPL == 2) *reinterpret_cast<float2*>(op) = make_float2(out[0], out[1]);
    else op[0] = out[0];
  }

  // 10a. ADAPT: the accumulated update Delta_n = S_n - gamma_n S~0 by
  //      |Delta_n|^2 = alpha_n^2 |Delta_{n-1}|^2 + 2 u_n . e^ + |u_n|^2 |k_n|^2,
  //      u_n = beta_n (v_n - alpha_n S_{n-1} k_n), e^ = alpha_n Delta_{n-1} k_n
  //      = sum_s zeta_s v_s - S~0 b^; the head is due when it reaches tau^2
  bool commit_now = n == P;
  float norm2 = 0.f;
  if constexpr (ADAPT) {
    float ue = 0.f, uu = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const float sa = col ? scr.ya[EPL * lane + e] : scr.ya[EPL * lane + e] * sc[e];
      const float sb = col ? scr.yb[EPL * lane + e] : scr.yb[EPL * lane + e] * sc[e];
      const float u = b_n * (vf[e] - (sa + vt2[e]));
      ue = fmaf(u, vt2[e] - sb, ue);
      uu = fmaf(u, u, uu);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) {
      ue += __shfl_xor_sync(FULL, ue, off);
      uu += __shfl_xor_sync(FULL, uu, off);
    }
    const float kk = __shfl_sync(FULL, tot, n - 1);
    const float prev = n > 1 ? reinterpret_cast<const float*>(stg + ST::G)[P * P + P] : 0.f;
    norm2 = fmaxf(a_n * a_n * prev + 2.f * ue + uu * kk, 0.f);
    commit_now = commit_now || norm2 >= p.tau2;
  }

  // 11. buffer the token: k, v, alpha, beta, its Gram row; then fill = n
  uint8_t* row = const_cast<uint8_t*>(kv_head) + (size_t)(n - 1) * row_elems * RESZ;
  if constexpr (R8) {
    uint32_t wk = 0u, wv = 0u;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      wk |= (uint32_t)e4m3_code(k_raw.get(e)) << (8 * e);
      wv |= (uint32_t)e4m3_code(v_raw.get(e)) << (8 * e);
    }
    uint8_t* pk = row + (size_t)EPL * lane;
    uint8_t* pv = row + D + (size_t)EPL * lane;
    if (EPL == 4) {
      *reinterpret_cast<uint32_t*>(pk) = wk;
      *reinterpret_cast<uint32_t*>(pv) = wv;
    } else if (EPL == 2) {
      *reinterpret_cast<uint16_t*>(pk) = (uint16_t)wk;
      *reinterpret_cast<uint16_t*>(pv) = (uint16_t)wv;
    } else {
      *pk = (uint8_t)wk;
      *pv = (uint8_t)wv;
    }
  } else {
    k_raw.store(row, (size_t)EPL * lane);
    v_raw.store(row, D + (size_t)EPL * lane);
  }
  if (lane == 0) {
    Raw<1, BF16> ra, rb2;
    ra.load(alpha, head);
    rb2.load(beta, head);
    uint8_t* abp = const_cast<uint8_t*>(ab_head) + (size_t)(n - 1) * 2 * ESZ;
    ra.store(abp, 0);
    rb2.store(abp, 1);
  }
  if (!commit_now && lane < n - 1) const_cast<float*>(gram_head)[(n - 1) * P + lane] = tot;
  if (ADAPT && !commit_now && lane == 0) const_cast<float*>(gram_head)[P * P + P] = norm2;

  // 12. period end (n == P, or marked early): replace the Gram block by the
  //     commit's chunk-form factors W[t][s] = gamma_{n/t} T[t][s] beta_s,
  //     T = (I + A)^{-1} (lane s solves column s by forward substitution;
  //     zero beyond n), followed by gamma_s (gamma_n beyond n), the largest
  //     |k| of the period and the largest stored scale
  if (commit_now) {
    float km = 0.f, sm = 0.f;
    {
      float x[EPL];
#pragma unroll
      for (int s = 0; s < PMAX; ++s) {
        if (s < n) {
          if constexpr (R8) {
            if (s < n - 1) {
              load_row<EPL, BF16, true>(stg + ST::KV, s * row_elems + (size_t)EPL * lane, x);
            } else {   // the token's own k, again from the stage, rounded as buffered
              load_f<EPL, BF16>(stg + ST::K, (size_t)EPL * lane, x);
#pragma unroll
              for (int e = 0; e < EPL; ++e) x[e] = e4m3_round(x[e]);
            }
          } else {
            load_f<EPL, BF16>(s < n - 1 ? stg + ST::KV : stg + ST::K,
                              s < n - 1 ? s * row_elems + (size_t)EPL * lane : (size_t)EPL * lane, x);
          }
#pragma unroll
          for (int e = 0; e < EPL; ++e) km = fmaxf(km, fabsf(x[e]));
        }
      }
      Raw<EPL, true> s_raw;
      s_raw.load(stg + ST::SC, (size_t)EPL * lane);
#pragma unroll
      for (int e = 0; e < EPL; ++e) sm = fmaxf(sm, fabsf(s_raw.get_half(e)));
#pragma unroll
      for (int off = 16; off; off >>= 1) {
        km = fmaxf(km, __shfl_xor_sync(FULL, km, off));
        sm = fmaxf(sm, __shfl_xor_sync(FULL, sm, off));
      }
    }
    __syncwarp();
    float Tc[PMAX];
#pragma unroll
    for (int tt = 0; tt < PMAX; ++tt) {
      float a2 = 0.f;
#pragma unroll
      for (int r = 0; r < tt; ++r)
        if (r >= lane) a2 = fmaf(scr.A[tt * PMAX + r], Tc[r], a2);
      Tc[tt] = tt == lane ? 1.f : (tt > lane ? -a2 : 0.f);
    }
    float* gw = const_cast<float*>(gram_head);
    if (lane < P) {
      const float bs = scr.gsb[2][lane];
#pragma unroll
      for (int tt = 0; tt < PMAX; ++tt)
        if (tt < P) gw[tt * P + lane] = scr.gsb[1][tt] * Tc[tt] * bs;
      gw[P * P + lane] = scr.gsb[0][lane];
    }
    if (lane == 0) {
      gw[P * P + P] = km;
      gw[P * P + P + 1] = sm;
    }
  }
  __syncwarp();
  if (lane == 0) p.fill[head] = commit_now && n < P ? (n | PACE_FILL_COMMIT) : n;
}

// Bulk-copy head `head`'s staged inputs into `stg` (lane 0 only): q, k, v, the
// scales, and -- when `fill` tokens (0 < fill < P) are buffered -- its rows,
// gates and Gram block.  Completes on `bar` with the exact byte count.
template <int D, bool BF16, int PMAX, bool R8>
__device__ __forceinline__ void issue_stage(const PoolDev& p, int head, int fill, const void* q,
                                            const void* k, const void* v, uint8_t* stg,
                                            uint64_t* bar) {
  using ST = Stage<D, BF16, PMAX>;
  constexpr uint32_t IO = D * ST::ESZ;
  const int h = head % p.H, b = head / p.H;
  const uint8_t* rec = p.state + (size_t)b * p.slot_stride + p.rec_off[h];
  const bool rows = fill > 0 && fill < p.P;
  constexpr uint32_t RB = D * (R8 ? 1u : (uint32_t)ST::ESZ);   // bytes of a buffered k or v
  const uint32_t kv_bytes = rows ? (uint32_t)fill * 2 * RB : 0u;
  const uint32_t bytes = 3 * IO + 2 * D + (rows ? kv_bytes + p.ab_stride + p.gram_stride : 0u);
  fence_proxy_async_smem();
  mbar_arrive_expect_tx(bar, bytes + p.dbg_extra_tx);
  tma_load_1d(stg + ST::Q, reinterpret_cast<const uint8_t*>(q) + (size_t)head * IO, IO, bar);
  tma_load_1d(stg + ST::K, reinterpret_cast<const uint8_t*>(k) + (size_t)head * IO, IO, bar);
  tma_load_1d(stg + ST::V, reinterpret_cast<const uint8_t*>(v) + (size_t)head * IO, IO, bar);
  tma_load_1d(stg + ST::SC, rec + code_bytes(D, D, p.bits[h]), 2 * D, bar);
  if (rows) {
    tma_load_1d(stg + ST::KV, p.kv + (size_t)head * p.P * 2 * RB, kv_bytes, bar);
    tma_load_1d(stg + ST::AB, p.ab + (size_t)head * p.ab_stride, p.ab_stride, bar);
    tma_load_1d(stg + ST::G, p.gram + (size_t)head * p.gram_stride, p.gram_stride, bar);
  }
}

template <int D, bool BF16, int PMAX, bool EXACT, bool ADAPT, bool R8>
__global__ void __launch_bounds__(kThreads, 2)
    decode_step_kernel(PoolDev p, const void* __restrict__ q, const void* __restrict__ k,
                       const void* __restrict__ v, const void* __restrict__ alpha,
                       const void* __restrict__ beta, float* __restrict__ o, Span sp) {
  using ST = Stage<D, BF16, PMAX>;
  constexpr int NS = ST::N;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  uint8_t* stages = smem_raw + (size_t)wib * NS * ST::BYTES;
  WarpScratch<D, ADAPT>& scr =
      reinterpret_cast<WarpScratch<D, ADAPT>*>(smem_raw + (size_t)kWarpsPerBlock * NS * ST::BYTES)[wib];
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem_raw + (size_t)kWarpsPerBlock * NS * ST::BYTES +
                                              kWarpsPerBlock * sizeof(WarpScratch<D, ADAPT>)) + NS * wib;
  for (int i = lane; i < D; i += 32) scr.dig[WarpScratch<D, ADAPT>::NDIG - 1][i] = 0;
  const int n_heads = sp.nb * p.H;   // work items of this launch
  const int warp0 = blockIdx.x * kWarpsPerBlock + wib;
  const int W = gridDim.x * kWarpsPerBlock;
  // lane 0 keeps the fill counts of the current head and the next one
  int f_cur = 0, f_nxt = 0;
  if (lane == 0) {
    for (int i = 0; i < NS; ++i) mbar_init(&bar[i], 1);
    fence_mbar_init();
    if (warp0 < n_heads) {
      const int h0 = head_in_order(p, warp0, sp.b0, sp.nb);
      f_cur = p.fill[h0];
      if (NS == 2) issue_stage<D, BF16, PMAX, R8>(p, h0, f_cur, q, k, v, stages, &bar[0]);
      f_nxt = warp0 + W < n_heads ? p.fill[head_in_order(p, warp0 + W, sp.b0, sp.nb)] : 0;
    }
  }
  __syncwarp();
  uint32_t parity = 0u;   // bit i: phase of stage i to wait for
  int s = 0;
  for (int it = warp0; it < n_heads; it += W) {
    const int head = head_in_order(p, it, sp.b0, sp.nb);
    const int nh = it + W < n_heads ? head_in_order(p, it + W, sp.b0, sp.nb) : -1;
    if (lane == 0) {
      if (NS == 2) {
        if (nh >= 0)
          issue_stage<D, BF16, PMAX, R8>(p, nh, f_nxt, q, k, v, stages + (s ^ 1) * ST::BYTES, &bar[s ^ 1]);
      } else {
        issue_stage<D, BF16, PMAX, R8>(p, head, f_cur, q, k, v, stages, &bar[0]);
      }
      if (nh >= 0) {   // the next head's codes on their way into L2
        const int hh = nh % p.H;
        prefetch_l2(p.state + (size_t)(nh / p.H) * p.slot_stride + p.rec_off[hh],
                    (uint32_t)record_bytes(D, D, p.bits[hh], D));
      }
    }
    const int nprev = __shfl_sync(FULL, f_cur, 0);
    if (lane == 0) {
      f_cur = f_nxt;
      f_nxt = it + 2 * W < n_heads ? p.fill[head_in_order(p, it + 2 * W, sp.b0, sp.nb)] : 0;
    }
    const bool ok =
        mbar_wait_bounded(&bar[s], (parity >> s) & 1u, lane == 0 ? p.flags : nullptr, p.wait_limit_ns);
    parity ^= 1u << s;
    if (!__all_sync(FULL, ok)) {
      // a copy did not land in time: this head's output row is NaN; let the
      // other stage's copy finish (bounded) before the warp stops using its
      // shared memory
      for (int i = lane; i < D; i += 32) o[(size_t)head * D + i] = __int_as_float(0x7fc00000);
      if (NS == 2 && nh >= 0) mbar_wait_bounded(&bar[s ^ 1], (parity >> (s ^ 1)) & 1u, nullptr, p.wait_limit_ns);
      return;
    }
    const uint8_t* stg = stages + s * ST::BYTES;
    if (NS == 2) s ^= 1;
    if (nprev < 0 || nprev >= p.P) {
      if (lane == 0) atomicOr(p.flags, PACE_FLAG_BUFFER_FULL);
      for (int i = lane; i < D; i += 32) o[(size_t)head * D + i] = __int_as_float(0x7fc00000);
      __syncwarp();
      continue;
    }
    const int n = nprev + 1;
    if (p.bits[head % p.H] == 4)
      decode_head<D, BF16, PMAX, 4, EXACT, ADAPT, R8>(p, head, n, q, k, v, alpha, beta, o, scr, stg, lane);
    else
      decode_head<D, BF16, PMAX, 8, EXACT, ADAPT, R8>(p, head, n, q, k, v, alpha, beta, o, scr, stg, lane);
  }
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = n > 0 ? n : 148;
  }
  return cached[dev];
}

template <int D, bool BF16, int PMAX, bool EXACT, bool ADAPT = false, bool R8 = false>
cudaError_t launch_t(const PoolDev& p, const Span& sp, const void* q, const void* k, const void* v,
                     const void* alpha, const void* beta, float* o, cudaStream_t st) {
  using ST = Stage<D, BF16, PMAX>;
  const size_t smem = (size_t)kWarpsPerBlock * (ST::N * ST::BYTES + sizeof(WarpScratch<D, ADAPT>) +
                                                ST::N * sizeof(uint64_t));
  cudaError_t e = cudaFuncSetAttribute(decode_step_kernel<D, BF16, PMAX, EXACT, ADAPT, R8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long heads = (long)sp.nb * p.H;
  if (heads == 0) return cudaSuccess;
  long blocks = (heads + kWarpsPerBlock - 1) / kWarpsPerBlock;
  const long cap = (long)(sp.blocks_per_sm > 0 ? sp.blocks_per_sm : 2) * sm_count();
  if (blocks > cap) blocks = cap;
  decode_step_kernel<D, BF16, PMAX, EXACT, ADAPT, R8><<<(unsigned)blocks, kThreads, smem, st>>>(
      p, q, k, v, alpha, beta, o, sp);
  return cudaGetLastError();
}

template <int D, bool BF16>
cudaError_t launch_p(const PoolDev& p, const Span& sp, const void* q, const void* k, const void* v,
                     const void* alpha, const void* beta, float* o, cudaStream_t st) {
  if (p.row8) {       // E4M3 buffered rows (no commit threshold on such pools)
    switch (p.P) {
      case 4: return launch_t<D, BF16, 4, true, false, true>(p, sp, q, k, v, alpha, beta, o, st);
      case 8: return launch_t<D, BF16, 8, true, false, true>(p, sp, q, k, v, alpha, beta, o, st);
      case 16: return launch_t<D, BF16, 16, true, false, true>(p, sp, q, k, v, alpha, beta, o, st);
    }
    if (p.P < 4) return launch_t<D, BF16, 4, false, false, true>(p, sp, q, k, v, alpha, beta, o, st);
    if (p.P < 8) return launch_t<D, BF16, 8, false, false, true>(p, sp, q, k, v, alpha, beta, o, st);
    return launch_t<D, BF16, 16, false, false, true>(p, sp, q, k, v, alpha, beta, o, st);
  }
  if (p.adaptive) {   // commit threshold set: the period is the buffer's capacity
    if (p.P <= 4) return launch_t<D, BF16, 4, false, true>(p, sp, q, k, v, alpha, beta, o, st);
    if (p.P <= 8) return launch_t<D, BF16, 8, false, true>(p, sp, q, k, v, alpha, beta, o, st);
    return launch_t<D, BF16, 16, false, true>(p, sp, q, k, v, alpha, beta, o, st);
  }
  switch (p.P) {
    case 4: return launch_t<D, BF16, 4, true>(p, sp, q, k, v, alpha, beta, o, st);
    case 8: return launch_t<D, BF16, 8, true>(p, sp, q, k, v, alpha, beta, o, st);
    case 16: return launch_t<D, BF16, 16, true>(p, sp, q, k, v, alpha, beta, o, st);
  }
  if (p.P < 4) return launch_t<D, BF16, 4, false>(p, sp, q, k, v, alpha, beta, o, st);
  if (p.P < 8) return launch_t<D, BF16, 8, false>(p, sp, q, k, v, alpha, beta, o, st);
  return launch_t<D, BF16, 16, false>(p, sp, q, k, v, alpha, beta, o, st);
}

}  // namespace

cudaError_t launch_decode_step(const PoolDev& p, const Span& sp, const void* q, const void* k,
                               const void* v, const void* alpha, const void* beta, float* o,
                               cudaStream_t st) {
  const bool bf = p.io == PACE_IO_BF16;
  switch (p.d_k) {
    case 32: return bf ? launch_p<32, true>(p, sp, q, k, v, alpha, beta, o, st)
                       : launch_p<32, false>(p, sp, q, k, v, alpha, beta, o, st);
    case 64: return bf ? launch_p<64, true>(p, sp, q, k, v, alpha, beta, o, st)
                       : launch_p<64, false>(p, sp, q, k, v, alpha, beta, o, st);
    case 128: return bf ? launch_p<128, true>(p, sp, q, k, v, alpha, beta, o, st)
                        : launch_p<128, false>(p, sp, q, k, v, alpha, beta, o, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace pace
