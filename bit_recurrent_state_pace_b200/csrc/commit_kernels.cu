// Period commit: apply the P buffered tokens to the stored state in one
// chunked fp32 update, then re-encode the state in place.
//
// "PACE: four-bit recurrent state by rounding less often", flowchart under
// "Fewer roundings, less compounded error": every k tokens the buffer feeds a
// "State update, chunked, high precision" followed by "4-bit encode,
// per-column scales", with long-memory heads kept at 8 bits; "PACE: A New
// 4-Bit Recurrent State Quantization Method ...", section "Periodic
// Rounding" (rounding per chunk, as chunked prefill kernels do).
//
// Chunk (UT/WY) form of the P tokens from the stored state S~0:
//   X = S~0 K^T;  U = (I + A)^{-1} diag(beta) (V - diag(gamma) X^T),
//   A[t][s] = beta_t gamma_{t/s} (k_t . k_s), s < t;
//   S_P = gamma_P S~0 + sum_s gamma_{P/s} u_s k_s^T = gamma_P S~0 + U^^T K,
// with U^ = W R, W[s][s'] = gamma_{P/s} T[s][s'] beta_s', T = (I + A)^{-1},
// R rows r_s = v_s - gamma_s x_s.
//
// Design (B200): one CTA per head, one warp per 16-row block; heads strided
// over a persistent grid, the next head's record, buffered rows, gates and
// Gram block brought into shared memory by 1-D TMA bulk copies while the
// current head computes (double buffer, mbarrier completion, bounded waits).
// Both contractions run on the tensor cores (mma.sync m16n8k16, f16
// operands, fp32 accumulation):
//   X:      A = codes (exact), B = K (times column scales) split hi + lo;
//   update: A = U^ split hi + lo, B = K, accumulator initialised with
//           gamma_P S~0 (the same fragments' codes times their scales),
// so the fp32 period-end state of a 16 x D row block lives in registers.
// Column absmax: per-lane pairs, a shuffle transpose over the 8 row lanes and
// a shared-memory max over the warps; the new codes are rounded with the
// f16 magic-number conversion (1032 + c, 1152 + c) and packed back in place.
#include "encode.cuh"
#include "frag.cuh"
#include "tma.cuh"

namespace pace {

namespace {

constexpr unsigned FULL = 0xffffffffu;

__device__ __forceinline__ float max_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

template <int D, bool BF16, int PMAX>
struct Cfg {
  static constexpr int RB = D / 16;                 // warps per CTA (16-row blocks)
  static constexpr int THREADS = 32 * RB;
  static constexpr int KS = D / 16;                 // k16 steps over key channels
  static constexpr int NT = D / 8;                  // n8 output tiles per row block
  static constexpr int NTX = (2 * PMAX + 7) / 8;    // X tiles: P vectors x (hi, lo)
  static constexpr int NSEG = BF16 ? 2 : 3;         // update K segments
  static constexpr int KU = (NSEG * PMAX + 15) / 16;  // update k16 steps
  static constexpr int NU = PMAX >= 16 ? 4 : 2;     // distinct U^ rows a lane needs
  static constexpr int ESZ = BF16 ? 2 : 4;
  static constexpr int REC = (D * D + 2 * D + 15) / 16 * 16;   // largest record (INT8)
  static constexpr int KVB = PMAX * 2 * D * ESZ;
  static constexpr int ABB = (2 * PMAX * ESZ + 15) / 16 * 16;
  static constexpr int GRB = (4 * PMAX * PMAX + 15) / 16 * 16;
  static constexpr int SLOT = REC + KVB + ABB + GRB;
};

template <int D, bool BF16, int PMAX>
struct alignas(16) Smem {
  using C = Cfg<D, BF16, PMAX>;
  uint8_t slot[2][C::SLOT];                     // staged record | kv rows | gates | Gram
  uint32_t bx[C::NTX][C::KS][8][4][2];          // X B fragments [tile][ks][g][t][b0,b1]
  __half bk[D][C::KU * 16 + 2];                 // update B: [key channel][slot] (+2: banks)
  float F[C::KS][4][4];                         // COL: gamma_P s_j, [ks][t][pos]
  float qfr[C::KS][4][4];                       // COL: new 1/s16, [ks][t][pos]
  float sfr[C::KS][4][4];                       // COL: new s16 as float, [ks][t][pos]
  float rowv[D];                                // ROW: gamma_P s_i
  float rowq[D], rows[D];                       // ROW: new 1/s16 and s16 per row
  float sc[D];                                  // old scales as float
  float vf[PMAX][D];                            // buffered values, fp32
  float A[PMAX][PMAX];
  float W[PMAX][PMAX];
  float gam[PMAX];
  float xinv[PMAX];
  float colmax[C::RB][D];
  uint64_t bar[2];
  float gP;
  int next_head;
  int slow;
  int abort_;
};

__device__ __forceinline__ int find_full(const PoolDev& p, int from, int step, int n_heads) {
  int hd = from;
  while (hd < n_heads && p.fill[hd] != p.P) hd += step;
  return hd;
}

template <int D, bool BF16, int PMAX>
__device__ __forceinline__ void issue_head(const PoolDev& p, int head, Smem<D, BF16, PMAX>& sm, int s) {
  using C = Cfg<D, BF16, PMAX>;
  const int h = head % p.H, b = head / p.H;
  const uint32_t rec_bytes = (uint32_t)record_bytes(D, D, p.bits[h], D);
  const uint32_t kv_bytes = (uint32_t)(p.P * 2 * D * C::ESZ);
  const uint8_t* rec = p.state + (size_t)b * p.slot_stride + p.rec_off[h];
  const uint8_t* kv = p.kv + (size_t)head * p.P * 2 * D * C::ESZ;
  const uint8_t* ab = p.ab + (size_t)head * p.ab_stride;
  const uint8_t* gr = p.gram + (size_t)head * p.gram_stride;
  uint8_t* dst = sm.slot[s];
  fence_proxy_async_smem();
  mbar_arrive_expect_tx(&sm.bar[s], rec_bytes + kv_bytes + p.ab_stride + p.gram_stride);
  tma_load_1d(dst, rec, rec_bytes, &sm.bar[s]);
  tma_load_1d(dst + C::REC, kv, kv_bytes, &sm.bar[s]);
  tma_load_1d(dst + C::REC + C::KVB, ab, p.ab_stride, &sm.bar[s]);
  tma_load_1d(dst + C::REC + C::KVB + C::ABB, gr, p.gram_stride, &sm.bar[s]);
}

__device__ __forceinline__ float io_at(const uint8_t* base, int idx, bool bf16) {
  if (bf16) return __uint_as_float(((uint32_t)reinterpret_cast<const uint16_t*>(base)[idx]) << 16);
  return reinterpret_cast<const float*>(base)[idx];
}

// Codes of rows 16r+g, 16r+g+8 for lane (g, t), read from shared memory.
template <int D, int BITS>
__device__ __forceinline__ void load_rows_smem(RowBlock<D, BITS>& rb, const uint8_t* rec, int r, int g,
                                               int t) {
  using RBk = RowBlock<D, BITS>;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint8_t* row = rec + (size_t)(16 * r + g + 8 * h) * RBk::ROWB;
#pragma unroll
    for (int c = 0; c < RBk::NCH; ++c) {
      const uint8_t* src = row + chunk_offset<D, BITS>(t, c);
      uint32_t* w = &rb.w[h][c * RBk::CW];
      if (RBk::CHUNK == 16) {
        const uint4 v = *reinterpret_cast<const uint4*>(src);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
      } else if (RBk::CHUNK == 8) {
        const uint2 v = *reinterpret_cast<const uint2*>(src);
        w[0] = v.x; w[1] = v.y;
      } else {
        w[0] = *reinterpret_cast<const uint32_t*>(src);
      }
    }
  }
}

// f16x2 "magic" values of two codes: the mantissa holds code + 8 (INT4) or
// code + 128 (INT8) on top of 1024.
template <int BITS>
__device__ __forceinline__ uint32_t magic_fast(float a, float b, float qa, float qb) {
  const float M = BITS == 4 ? 1032.f : 1152.f;
  return h2u(__floats2half2_rn(fmaf(a, qa, M), fmaf(b, qb, M)));
}

template <int BITS>
__device__ __forceinline__ uint32_t magic_exact(float a, float b, float sa, float sb) {
  const int qmax = BITS == 4 ? 7 : 127, off = BITS == 4 ? 8 : 128;
  const uint32_t ca = (uint32_t)(encode_value(a, sa, qmax) + off);
  const uint32_t cb = (uint32_t)(encode_value(b, sb, qmax) + off);
  return (0x6400u | ca) | ((0x6400u | cb) << 16);
}

// Four f16x2 magic values of code pairs (8m+0,8m+4), (8m+1,8m+5), (8m+2,8m+6),
// (8m+3,8m+7) -> one word of eight 4-bit two's complement codes.
__device__ __forceinline__ uint32_t pack_int4(uint32_t p0, uint32_t p1, uint32_t p2, uint32_t p3) {
  // low nibble of each f16 half = code + 8; flipping bit 3 gives the 4-bit two's complement
  const uint32_t m0 = (p0 & 0x000F000Fu) ^ 0x00080008u, m1 = (p1 & 0x000F000Fu) ^ 0x00080008u;
  const uint32_t m2 = (p2 & 0x000F000Fu) ^ 0x00080008u, m3 = (p3 & 0x000F000Fu) ^ 0x00080008u;
  return m0 | (m1 << 4) | (m2 << 8) | (m3 << 12);
}

// Two f16x2 magic values (codes j, j+1) and (j+2, j+3) -> four INT8 codes.
__device__ __forceinline__ uint32_t pack_int8(uint32_t lo, uint32_t hi) {
  return prmt(lo, hi, 0x6420u) ^ 0x80808080u;
}

template <int D, bool BF16, int PMAX, int BITS>
__device__ void commit_head(const PoolDev& p, int head, Smem<D, BF16, PMAX>& sm, const uint8_t* slot) {
  using C = Cfg<D, BF16, PMAX>;
  constexpr int KS = C::KS, NT = C::NT, NTX = C::NTX, KU = C::KU, NU = C::NU;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, g = lane >> 2, t = lane & 3;
  const int P = p.P, h = head % p.H, b = head / p.H;
  const bool col = p.axis == PACE_SCALE_COL;
  const int qmax = BITS == 4 ? 7 : 127;
  uint8_t* rec = p.state + (size_t)b * p.slot_stride + p.rec_off[h];
  uint16_t* rsc = reinterpret_cast<uint16_t*>(rec + code_bytes(D, D, BITS));
  const uint8_t* s_rec = slot;
  const uint8_t* s_kv = slot + C::REC;
  const uint8_t* s_ab = slot + C::REC + C::KVB;
  const float* s_gr = reinterpret_cast<const float*>(slot + C::REC + C::KVB + C::ABB);
  const uint16_t* s_sc = reinterpret_cast<const uint16_t*>(s_rec + code_bytes(D, D, BITS));

  // ---- phase 1: per-head operands ------------------------------------------
  float gP = 1.f;
  for (int s = 0; s < P; ++s) gP *= io_at(s_ab, 2 * s, BF16);
  for (int j = tid; j < D; j += C::THREADS) {
    const float s = __half2float(__ushort_as_half(s_sc[j]));
    sm.sc[j] = s;
    sm.rowv[j] = gP * s;
  }
  for (int idx = tid; idx < 4 * KS * 4; idx += C::THREADS) {
    const int tt = idx / (KS * 4), ks = (idx / 4) % KS, pos = idx & 3;
    const int j = jof<D, BITS>(tt, ks, pos);
    sm.F[ks][tt][pos] = gP * __half2float(__ushort_as_half(s_sc[j]));
  }
  for (int idx = tid; idx < P * D; idx += C::THREADS) {
    const int s = idx / D, i = idx - s * D;
    sm.vf[s][i] = io_at(s_kv, s * 2 * D + D + i, BF16);
  }
  for (int idx = tid; idx < D * P; idx += C::THREADS) {      // update B: K (hi, hi | lo)
    const int j = idx / P, s = idx - (idx / P) * P;
    const float kv = io_at(s_kv, s * 2 * D + j, BF16);
    const __half hi = __float2half_rn(kv);
    sm.bk[j][s] = hi;
    sm.bk[j][PMAX + s] = hi;
    if (C::NSEG == 3) sm.bk[j][2 * PMAX + s] = __float2half_rn(kv - __half2float(hi));
  }
  if (w == 0) {
    // gates, decay products, A, T = (I + A)^{-1} and W, lane s = token s
    const float al = lane < P ? io_at(s_ab, 2 * lane, BF16) : 1.f;
    const float be = lane < P ? io_at(s_ab, 2 * lane + 1, BF16) : 0.f;
    float gcum = al;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float x = __shfl_up_sync(FULL, gcum, off);
      if (lane >= off) gcum *= x;
    }
    float suf = __shfl_down_sync(FULL, al, 1);
    if (lane == 31) suf = 1.f;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float x = __shfl_down_sync(FULL, suf, off);
      if (lane + off < 32) suf *= x;
    }
    float run = 1.f;
#pragma unroll
    for (int tt = 0; tt < PMAX; ++tt) {
      const float at = __shfl_sync(FULL, al, tt), bt = __shfl_sync(FULL, be, tt);
      float a = 0.f;
      if (tt > lane) {
        run *= at;
        if (tt < P && lane < P) a = bt * run * s_gr[tt * P + lane];
      }
      if (lane < PMAX) sm.A[tt][lane] = a;
    }
    __syncwarp();
    float Tc[PMAX];
#pragma unroll
    for (int tt = 0; tt < PMAX; ++tt) {
      float acc = 0.f;
#pragma unroll
      for (int r = 0; r < tt; ++r)
        if (r >= lane) acc = fmaf(sm.A[tt][r], Tc[r], acc);
      Tc[tt] = tt == lane ? 1.f : (tt > lane ? -acc : 0.f);
    }
#pragma unroll
    for (int tt = 0; tt < PMAX; ++tt) {
      const float sf_t = __shfl_sync(FULL, suf, tt);
      if (lane < PMAX) sm.W[tt][lane] = (tt < P && lane < P) ? sf_t * Tc[tt] * be : 0.f;
    }
    if (lane < PMAX) sm.gam[lane] = gcum;
  } else {
    // X operand: vector s (scaled by column scales in COL mode), normalised, hi/lo
    for (int s = w - 1; s < P; s += C::RB - 1) {
      constexpr int E = D / 32;
      float val[E];
      float m = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int j = lane + 32 * e;
        const float kv = io_at(s_kv, s * 2 * D + j, BF16);
        val[e] = col ? kv * __half2float(__ushort_as_half(s_sc[j])) : kv;
        m = fmaxf(m, fabsf(val[e]));
      }
#pragma unroll
      for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, off));
      int ex = 0;
      if (m > 0.f && m < INFINITY) ex = max(-60, min(60, 14 - ilogbf(m)));
      const float up = ldexpf(1.f, ex);
      if (lane == 0) sm.xinv[s] = ldexpf(1.f, -ex);
      __half* bxh = reinterpret_cast<__half*>(&sm.bx[0][0][0][0][0]);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int j = lane + 32 * e;
        const float x = val[e] * up;
        const __half hi = __float2half_rn(x);
        const __half lo = __float2half_rn(x - __half2float(hi));
        int tt, ks, pos;
        kslot_of<D, BITS>(j, tt, ks, pos);
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const int c = 2 * s + part, tile = c >> 3, gc = c & 7;
          const size_t at = ((((size_t)tile * KS + ks) * 8 + gc) * 4 + tt) * 4 + pos;
          bxh[at] = part ? lo : hi;
        }
      }
    }
  }
  __syncthreads();

  // ---- phase 2: this warp's 16 rows ------------------------------------------
  const int i0 = 16 * w + g, i1 = i0 + 8;
  RowBlock<D, BITS> rbk;
  load_rows_smem<D, BITS>(rbk, s_rec, w, g, t);
  uint32_t Af[KS][4];
  float xacc[NTX][4];
#pragma unroll
  for (int x = 0; x < NTX; ++x) xacc[x][0] = xacc[x][1] = xacc[x][2] = xacc[x][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    a_frag<D, BITS>(rbk, ks, Af[ks]);
#pragma unroll
    for (int x = 0; x < NTX; ++x) {
      const uint2 bb = *reinterpret_cast<const uint2*>(&sm.bx[x][ks][g][t][0]);
      mma16816(xacc[x], Af[ks], bb.x, bb.y);
    }
  }
  // r_s = v_s - gamma_s x_s for this lane's vectors s = 4x + t, then all-gather in the quad
  float r[PMAX][2];
  {
    float ro[NTX][2];
    const float s0 = col ? 1.f : sm.sc[i0], s1 = col ? 1.f : sm.sc[i1];
#pragma unroll
    for (int x = 0; x < NTX; ++x) {
      const int s = 4 * x + t;
      ro[x][0] = ro[x][1] = 0.f;
      if (s < P) {
        const float xi = sm.xinv[s], gs = sm.gam[s];
        ro[x][0] = sm.vf[s][i0] - gs * ((xacc[x][0] + xacc[x][1]) * xi * s0);
        ro[x][1] = sm.vf[s][i1] - gs * ((xacc[x][2] + xacc[x][3]) * xi * s1);
      }
    }
#pragma unroll
    for (int x = 0; x < NTX; ++x)
#pragma unroll
      for (int src = 0; src < 4; ++src) {
        const int s = 4 * x + src;
        const float a = __shfl_sync(FULL, ro[x][0], (lane & ~3) | src);
        const float c = __shfl_sync(FULL, ro[x][1], (lane & ~3) | src);
        if (s < PMAX) {
          r[s][0] = a;
          r[s][1] = c;
        }
      }
  }
  // U^ rows this lane feeds into the update contraction
  float uh[NU][2];
  float um = 0.f;
#pragma unroll
  for (int q = 0; q < NU; ++q) {
    const int s = (2 * t + (q & 1) + 8 * (q >> 1)) % PMAX;
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int sp = 0; sp < PMAX; ++sp) {
      const float wv = sm.W[s][sp];
      a0 = fmaf(wv, r[sp][0], a0);
      a1 = fmaf(wv, r[sp][1], a1);
    }
    uh[q][0] = a0;
    uh[q][1] = a1;
    um = fmaxf(um, fmaxf(fabsf(a0), fabsf(a1)));
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) um = fmaxf(um, __shfl_xor_sync(FULL, um, off));
  int ex = 0;
  if (um > 0.f && um < INFINITY) ex = max(-60, min(60, 14 - ilogbf(um)));
  const float up = ldexpf(1.f, ex), down = ldexpf(1.f, -ex);
  uint32_t Au[KU][4];
  {
    __half hv[NU][2][2];   // [q][row][hi, lo]
#pragma unroll
    for (int q = 0; q < NU; ++q)
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const float x = uh[q][rr] * up;
        hv[q][rr][0] = __float2half_rn(x);
        hv[q][rr][1] = __float2half_rn(x - __half2float(hv[q][rr][0]));
      }
#pragma unroll
    for (int u = 0; u < KU; ++u) {
      __half v[4][2];   // [slot k][row]
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int sigma = 16 * u + 2 * t + (k & 1) + 8 * (k >> 1);
        const int seg = sigma / PMAX;
        const int q = NU == 4 ? k : (k & 1);
#pragma unroll
        for (int rr = 0; rr < 2; ++rr)
          v[k][rr] = seg >= C::NSEG ? __ushort_as_half((unsigned short)0)
                                    : hv[q][rr][seg == 1 ? 1 : 0];
      }
      Au[u][0] = h2u(__halves2half2(v[0][0], v[1][0]));
      Au[u][1] = h2u(__halves2half2(v[0][1], v[1][1]));
      Au[u][2] = h2u(__halves2half2(v[2][0], v[3][0]));
      Au[u][3] = h2u(__halves2half2(v[2][1], v[3][1]));
    }
  }
  // accumulator = up * gamma_P S~0 (codes of this lane's fragments times scales); += U^^T K
  float acc[NT][4];
  const float fr0 = sm.rowv[i0] * up, fr1 = sm.rowv[i1] * up;
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const float2 c0 = __half22float2(u2h(Af[ks][0])), c1 = __half22float2(u2h(Af[ks][1]));
    const float2 c2 = __half22float2(u2h(Af[ks][2])), c3 = __half22float2(u2h(Af[ks][3]));
    if (col) {
      const float4 f = *reinterpret_cast<const float4*>(&sm.F[ks][t][0]);
      const float f0 = f.x * up, f1 = f.y * up, f2 = f.z * up, f3 = f.w * up;
      acc[2 * ks][0] = c0.x * f0; acc[2 * ks][1] = c0.y * f1;
      acc[2 * ks][2] = c1.x * f0; acc[2 * ks][3] = c1.y * f1;
      acc[2 * ks + 1][0] = c2.x * f2; acc[2 * ks + 1][1] = c2.y * f3;
      acc[2 * ks + 1][2] = c3.x * f2; acc[2 * ks + 1][3] = c3.y * f3;
    } else {
      acc[2 * ks][0] = c0.x * fr0; acc[2 * ks][1] = c0.y * fr0;
      acc[2 * ks][2] = c1.x * fr1; acc[2 * ks][3] = c1.y * fr1;
      acc[2 * ks + 1][0] = c2.x * fr0; acc[2 * ks + 1][1] = c2.y * fr0;
      acc[2 * ks + 1][2] = c3.x * fr1; acc[2 * ks + 1][3] = c3.y * fr1;
    }
#pragma unroll
    for (int hs = 0; hs < 2; ++hs) {
      const int tile = 2 * ks + hs;
      const int j = jof<D, BITS>(g >> 1, ks, 2 * hs + (g & 1));
#pragma unroll
      for (int u = 0; u < KU; ++u) {
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(&sm.bk[j][16 * u + 2 * t]);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(&sm.bk[j][16 * u + 2 * t + 8]);
        mma16816(acc[tile], Au[u], b0, b1);
      }
    }
  }

  // ---- absmax ----------------------------------------------------------------
  if (col) {
    float v[2 * NT];
#pragma unroll
    for (int tile = 0; tile < NT; ++tile) {
      v[2 * tile] = max_nan(fabsf(acc[tile][0]), fabsf(acc[tile][2]));
      v[2 * tile + 1] = max_nan(fabsf(acc[tile][1]), fabsf(acc[tile][3]));
    }
    // transpose-reduce over the 8 row lanes (lane bits 4, 3, 2): 2*NT -> 2*NT/8 values
#pragma unroll
    for (int c = 2 * NT; c > 2 * NT / 8; c >>= 1) {
      const int o = c == 2 * NT ? 16 : (c == NT ? 8 : 4);
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int k = 0; k < c / 2; ++k) {
        const float send = upper ? v[k] : v[k + c / 2];
        const float keep = upper ? v[k + c / 2] : v[k];
        v[k] = max_nan(keep, __shfl_xor_sync(FULL, send, o));
      }
    }
    // lane keeps value indices 4g + k (k < 2NT/8 = D/32): tile 2g + (k >> 1), column 2t + (k & 1)
#pragma unroll
    for (int k = 0; k < 2 * NT / 8; ++k) {
      const int idx = (2 * NT / 8) * g + k;
      const int tile = idx >> 1, e = idx & 1;
      const int j = jof<D, BITS>(t, tile >> 1, 2 * (tile & 1) + e);
      sm.colmax[w][j] = v[k] * down;
    }
  } else {
    float m0 = 0.f, m1 = 0.f;
#pragma unroll
    for (int tile = 0; tile < NT; ++tile) {
      m0 = max_nan(m0, max_nan(fabsf(acc[tile][0]), fabsf(acc[tile][1])));
      m1 = max_nan(m1, max_nan(fabsf(acc[tile][2]), fabsf(acc[tile][3])));
    }
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
      m0 = max_nan(m0, __shfl_xor_sync(FULL, m0, off));
      m1 = max_nan(m1, __shfl_xor_sync(FULL, m1, off));
    }
    if (t == 0) {
      bool ovf = false;
      const float a0 = m0 * down, a1 = m1 * down;
      const GroupScale s0 = group_scale(a0, isfinite(a0), qmax, p.flags);
      const GroupScale s1 = group_scale(a1, isfinite(a1), qmax, p.flags);
      ovf = !isfinite(a0) || !isfinite(a1) ||
            (s0.bits == 0x7BFF && a0 / qmax > 65504.f) || (s1.bits == 0x7BFF && a1 / qmax > 65504.f);
      rsc[i0] = s0.bits;
      rsc[i1] = s1.bits;
      sm.rowq[i0] = s0.sf > 0.f ? 1.f / s0.sf : 0.f;
      sm.rowq[i1] = s1.sf > 0.f ? 1.f / s1.sf : 0.f;
      sm.rows[i0] = s0.sf;
      sm.rows[i1] = s1.sf;
      if (ovf) sm.slow = 1;
    }
  }
  __syncthreads();
  if (col) {
    for (int j = tid; j < D; j += C::THREADS) {
      float a = 0.f;
#pragma unroll
      for (int ww = 0; ww < C::RB; ++ww) a = max_nan(a, sm.colmax[ww][j]);
      const GroupScale s = group_scale(a, isfinite(a), qmax, p.flags);
      rsc[j] = s.bits;
      int tt, ks, pos;
      kslot_of<D, BITS>(j, tt, ks, pos);
      sm.qfr[ks][tt][pos] = s.sf > 0.f ? 1.f / s.sf : 0.f;
      sm.sfr[ks][tt][pos] = s.sf;
      if (!isfinite(a) || (s.bits == 0x7BFF && a / qmax > 65504.f)) sm.slow = 1;
    }
    __syncthreads();
  }

  // ---- encode and store this warp's rows ------------------------------------
  const bool slow = sm.slow != 0;
  uint32_t hm[KS][2][2];   // [ks][tile half][row] f16x2 magic pairs
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    float q0, q1, q2, q3, qa, qb;   // per column (COL) or per row (ROW)
    if (col) {
      const float4 qq = *reinterpret_cast<const float4*>(slow ? &sm.sfr[ks][t][0] : &sm.qfr[ks][t][0]);
      q0 = qq.x; q1 = qq.y; q2 = qq.z; q3 = qq.w;
      qa = qb = 0.f;
    } else {
      qa = slow ? sm.rows[i0] : sm.rowq[i0];
      qb = slow ? sm.rows[i1] : sm.rowq[i1];
      q0 = q1 = q2 = q3 = 0.f;
    }
#pragma unroll
    for (int hs = 0; hs < 2; ++hs) {
      const float* a = acc[2 * ks + hs];
      const float ca = col ? (hs ? q2 : q0) : qa, cb = col ? (hs ? q3 : q1) : qa;
      const float cc = col ? (hs ? q2 : q0) : qb, cd = col ? (hs ? q3 : q1) : qb;
      if (!slow) {
        hm[ks][hs][0] = magic_fast<BITS>(a[0], a[1], ca * down, cb * down);
        hm[ks][hs][1] = magic_fast<BITS>(a[2], a[3], cc * down, cd * down);
      } else {
        hm[ks][hs][0] = magic_exact<BITS>(a[0] * down, a[1] * down, ca, cb);
        hm[ks][hs][1] = magic_exact<BITS>(a[2] * down, a[3] * down, cc, cd);
      }
    }
  }
  constexpr int ROWB = D * BITS / 8;
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    uint8_t* row = rec + (size_t)(rr ? i1 : i0) * ROWB;
    if (BITS == 4) {
      constexpr int NW = D / 32;   // words per lane per row
      uint32_t wd[NW];
#pragma unroll
      for (int m = 0; m < NW; ++m)
        wd[m] = pack_int4(hm[2 * m][0][rr], hm[2 * m][1][rr], hm[2 * m + 1][0][rr], hm[2 * m + 1][1][rr]);
      uint8_t* dst = row + chunk_offset<D, 4>(t, 0);
      if (NW == 4) *reinterpret_cast<uint4*>(dst) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
      else if (NW == 2) *reinterpret_cast<uint2*>(dst) = make_uint2(wd[0], wd[1]);
      else *reinterpret_cast<uint32_t*>(dst) = wd[0];
    } else {
      constexpr int WPC = D / 32;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t wd[WPC];
#pragma unroll
        for (int m = 0; m < WPC; ++m) wd[m] = pack_int8(hm[c * WPC + m][0][rr], hm[c * WPC + m][1][rr]);
        uint8_t* dst = row + chunk_offset<D, 8>(t, c);
        if (WPC == 4) *reinterpret_cast<uint4*>(dst) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        else if (WPC == 2) *reinterpret_cast<uint2*>(dst) = make_uint2(wd[0], wd[1]);
        else *reinterpret_cast<uint32_t*>(dst) = wd[0];
      }
    }
  }
  if (tid == 0) p.fill[head] = 0;
}

template <int D, bool BF16, int PMAX>
__global__ void __launch_bounds__(Cfg<D, BF16, PMAX>::THREADS, 2)
    commit_kernel(PoolDev p) {
  using C = Cfg<D, BF16, PMAX>;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Smem<D, BF16, PMAX>& sm = *reinterpret_cast<Smem<D, BF16, PMAX>*>(smem_raw);
  const int tid = threadIdx.x;
  const int n_heads = p.B * p.H;
  // zero the operand slots that stay unused (tokens >= P, padding segments)
  {
    uint32_t* z = &sm.bx[0][0][0][0][0];
    for (int i = tid; i < (int)(sizeof(sm.bx) / 4); i += C::THREADS) z[i] = 0u;
    uint32_t* zb = reinterpret_cast<uint32_t*>(&sm.bk[0][0]);  // whole rows incl. padding
    for (int i = tid; i < (int)(sizeof(sm.bk) / 4); i += C::THREADS) zb[i] = 0u;
  }
  if (tid == 0) {
    mbar_init(&sm.bar[0], 1);
    mbar_init(&sm.bar[1], 1);
    fence_mbar_init();
    sm.slow = 0;
    sm.abort_ = 0;
    const int first = find_full(p, blockIdx.x, gridDim.x, n_heads);
    sm.next_head = first;
    if (first < n_heads) issue_head<D, BF16, PMAX>(p, first, sm, 0);
  }
  __syncthreads();
  uint32_t parity[2] = {0u, 0u};
  int s = 0;
  int head = sm.next_head;
  while (head < n_heads) {
    __syncthreads();                      // everyone has read next_head; slot s^1 is free
    if (tid == 0) {
      const int nxt = find_full(p, head + gridDim.x, gridDim.x, n_heads);
      sm.next_head = nxt;
      if (nxt < n_heads) issue_head<D, BF16, PMAX>(p, nxt, sm, s ^ 1);
    }
    const bool ok = mbar_wait_bounded(&sm.bar[s], parity[s], p.flags);
    parity[s] ^= 1u;
    if (__syncthreads_or(!ok)) {
      // a copy did not land in time: give the in-flight copies a bounded
      // second chance to finish before this block's shared memory goes away
      if (tid == 0) {
        mbar_wait_bounded(&sm.bar[s ^ 1], parity[s ^ 1], nullptr);
      }
      __syncthreads();
      return;
    }
    if (p.bits[head % p.H] == 4)
      commit_head<D, BF16, PMAX, 4>(p, head, sm, sm.slot[s]);
    else
      commit_head<D, BF16, PMAX, 8>(p, head, sm, sm.slot[s]);
    __syncthreads();
    if (tid == 0) sm.slow = 0;
    head = sm.next_head;
    s ^= 1;
  }
}

int sm_count_dev() {
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

template <int D, bool BF16, int PMAX>
cudaError_t launch_t(const PoolDev& p, cudaStream_t st) {
  using C = Cfg<D, BF16, PMAX>;
  const size_t smem = sizeof(Smem<D, BF16, PMAX>);
  cudaError_t e = cudaFuncSetAttribute(commit_kernel<D, BF16, PMAX>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long heads = (long)p.B * p.H;
  long blocks = 2L * sm_count_dev() * (D == 128 ? 1 : D == 64 ? 2 : 4);
  if (blocks > heads) blocks = heads;
  commit_kernel<D, BF16, PMAX><<<(unsigned)blocks, C::THREADS, smem, st>>>(p);
  return cudaGetLastError();
}

template <int D, bool BF16>
cudaError_t launch_p(const PoolDev& p, cudaStream_t st) {
  if (p.P <= 4) return launch_t<D, BF16, 4>(p, st);
  if (p.P <= 8) return launch_t<D, BF16, 8>(p, st);
  return launch_t<D, BF16, 16>(p, st);
}

}  // namespace

cudaError_t launch_commit(const PoolDev& p, cudaStream_t st) {
  const bool bf = p.io == PACE_IO_BF16;
  switch (p.d_k) {
    case 32: return bf ? launch_p<32, true>(p, st) : launch_p<32, false>(p, st);
    case 64: return bf ? launch_p<64, true>(p, st) : launch_p<64, false>(p, st);
    case 128: return bf ? launch_p<128, true>(p, st) : launch_p<128, false>(p, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace pace
