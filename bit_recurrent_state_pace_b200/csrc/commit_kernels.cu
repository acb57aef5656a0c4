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
// Gram block brought into shared memory by 1-D TMA bulk copies two heads
// ahead (three slots, mbarrier completion, bounded waits), issued by a thread
// that is otherwise idle during the scale pass.
// Both contractions run on the f16 tensor cores (mma.sync m16n8k16, fp32
// accumulation); the codes are exact in f16 and every fp32 operand is split
// hi + lo after a power-of-two normalisation:
//   X:      A = codes, B = the keys (times the column scales);
//   update: A = U^, B = K, accumulator initialised with gamma_P S~0 from the
//           same code fragments.
// The update's output columns follow the code fragments' key channels, so
// the initialisation, the column absmax and the re-encode stay lane-local.
// Column absmax: per-lane row pairs, a shuffle transpose over the 8 row lanes
// and a shared-memory max over the warps; the new codes are rounded with the
// f16 magic-number conversion (1032 + c, 1152 + c) and packed in place.
#include <type_traits>

#include "e4m3.cuh"
#include "tma.cuh"
#include "update_common.cuh"

namespace pace {

namespace {

constexpr unsigned FULL = 0xffffffffu;


template <int D, bool BF16, int PMAX>
struct Cfg {
  static constexpr int RB = D / 16;                 // warps per CTA (16-row blocks)
  static constexpr int THREADS = 32 * RB;
  static constexpr int KS = D / 16;                 // k16 steps over key channels
  static constexpr int NT = D / 8;                  // n8 output tiles per row block
  static constexpr int NTX = (2 * PMAX + 7) / 8;    // X tiles: P vectors x (hi, lo)
  static constexpr int NSEG = BF16 ? 2 : 3;         // update K segments: hi | lo (| hi x k_lo)
  static constexpr int KU = (NSEG * PMAX + 15) / 16;  // update k16 steps
  static constexpr int NU = PMAX >= 16 ? 4 : 2;     // distinct U^ rows a lane feeds
  static constexpr int ESZ = BF16 ? 2 : 4;
  static constexpr int REC = (D * D + 2 * D + 15) / 16 * 16;   // largest record (INT8)
  // buffered rows sit 16 bytes apart from a multiple of 128 so that the same
  // key channel of different tokens falls in different shared-memory banks
  static constexpr int ROWS = 2 * D * ESZ + 16;
  static constexpr int KVB = PMAX * ROWS;
  static constexpr int ABB = (2 * PMAX * ESZ + 15) / 16 * 16;
  static constexpr int GRB = (4 * (PMAX * (PMAX + 1) + 2) + 15) / 16 * 16;
  static constexpr int SLOT = REC + KVB + ABB + GRB;
};

template <int D>
struct alignas(16) WarpTab {
  float4 f[D / 16][4];            // [ks][t]: up * gamma_P * s_j at the lane's 4 fragment channels
  float4 q[D / 16][4];            // [ks][t]: this warp's quantisation factors, same order
};

template <int D, bool BF16, int PMAX>
struct alignas(16) Smem {
  using C = Cfg<D, BF16, PMAX>;
  uint8_t slot[3][C::SLOT];                       // staged record | kv rows | gates | Gram
  uint2 bx[C::NTX][C::KS][8][4];                  // X B fragments [tile][ks][g][t]
  uint2 bkf[C::NT][C::KU][8][4];                  // update B fragments [tile][u][g][t]
  float sc[D];                                    // old scales (float)
  float qf[D], sfv[D];                            // new 1/s16 and s16 (column or row)
  float colmax[C::RB][D];
  WarpTab<D> wt[C::RB];
  uint64_t bar[3];
  int hq[3];                                      // head staged in each slot
  int hn[3];                                      // its buffered tokens
  int next_head;
  int slow[2];                                    // by head parity: exact-encode fallback needed
};

// First head index >= from (stepping by step, below end) due for a commit,
// or end.  The 32 lanes of the calling warp test 32 candidates at a time.
__device__ __forceinline__ int find_full_warp(const PoolDev& p, int from, int step, int end, int lane) {
  for (int base = from; base < end; base += 32 * step) {
    const int hd = base + lane * step;
    const unsigned m = __ballot_sync(FULL, hd < end && commit_due(p.fill[hd], p.P));
    if (m) return base + (__ffs((int)m) - 1) * step;
  }
  return end;
}

template <int D, bool BF16, int PMAX, bool R8>
__device__ __forceinline__ void issue_head(const PoolDev& p, int head, Smem<D, BF16, PMAX>& sm, int s) {
  using C = Cfg<D, BF16, PMAX>;
  const int h = head % p.H, b = head / p.H;
  const uint32_t rec_bytes = (uint32_t)record_bytes(D, D, p.bits[h], D);
  constexpr uint32_t row = 2 * D * (R8 ? 1 : C::ESZ);   // bytes of a buffered row
  const uint32_t kv_bytes = (uint32_t)p.P * row;
  const uint8_t* rec = p.state + (size_t)b * p.slot_stride + p.rec_off[h];
  const uint8_t* kv = p.kv + (size_t)head * p.P * row;
  const uint8_t* ab = p.ab + (size_t)head * p.ab_stride;
  const uint8_t* gr = p.gram + (size_t)head * p.gram_stride;
  uint8_t* dst = sm.slot[s];
  fence_proxy_async_smem();
  mbar_arrive_expect_tx(&sm.bar[s], rec_bytes + kv_bytes + p.ab_stride + p.gram_stride);
  tma_load_1d(dst, rec, rec_bytes, &sm.bar[s]);
  for (int r = 0; r < p.P; ++r)
    tma_load_1d(dst + C::REC + r * C::ROWS, kv + (size_t)r * row, row, &sm.bar[s]);
  tma_load_1d(dst + C::REC + C::KVB, ab, p.ab_stride, &sm.bar[s]);
  tma_load_1d(dst + C::REC + C::KVB + C::ABB, gr, p.gram_stride, &sm.bar[s]);
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



// EXACT: the pool's period equals PMAX, so every loop bound over tokens is a
// compile-time constant.
// Returns false (every thread) when the staged copies of this head did not
// arrive in time (ok == false in some thread); nothing is written then.
// n_tok: the head's buffered tokens (P, or fewer for a head marked early).
// R8: the buffered rows are E4M3 bytes.
template <int D, bool BF16, int PMAX, int BITS, bool EXACT, bool R8, class Issue>
__device__ bool commit_head(const PoolDev& p, int head, Smem<D, BF16, PMAX>& sm, const uint8_t* slot,
                            int n_tok, bool ok, int parity_bit, Issue&& issue_next) {
  using C = Cfg<D, BF16, PMAX>;
  constexpr int KS = C::KS, NT = C::NT, NTX = C::NTX, KU = C::KU, NU = C::NU;
  constexpr int ROWB = D * BITS / 8;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, g = lane >> 2, t = lane & 3;
  // P: tokens to apply; PS: the pool's period, the stride of the factor block
  const int P = EXACT ? PMAX : n_tok, PS = EXACT ? PMAX : p.P, h = head % p.H, b = head / p.H;
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
  // W[s][s'] (P x P), gamma_s (P), max |k| and the largest stored scale were
  // left in the Gram block by the decode step that buffered the P-th token.
  const float* W = s_gr;
  const float* gam = s_gr + PS * PS;
  const float gP = gam[P - 1];
  // (the operands of the previous head were last read before its absmax
  // barrier, so these tables are rebuilt without a barrier of their own)
  for (int j = tid; j < D; j += C::THREADS) sm.sc[j] = __half2float(__ushort_as_half(s_sc[j]));
  // one power-of-two normalisation of the X operand for the whole head
  const float bmax = col ? s_gr[PS * PS + PS] * s_gr[PS * PS + PS + 1] : s_gr[PS * PS + PS];
  int exx = 0;
  if (bmax >= 1.17549435e-38f && bmax < INFINITY) exx = max(-120, min(120, 14 - exp2_floor(bmax)));
  const float upx = pow2i(exx);
  const float xinv = pow2i(-exx);
  {
    // X operand, built by fragment owner: entry (x, ks, g, t) holds rows
    // k = 2t, 2t+1 | 2t+8, 2t+9 (key channels jof(t, ks, 0..3)) of column
    // 8x + g = vector s = 4x + g/2, hi (g even) or lo (g odd) part.  One item
    // writes the hi and the lo entry of one (x, ks, g/2, t).
    for (int it = tid; it < NTX * KS * 16; it += C::THREADS) {
      const int tt = it & 3, ks = (it >> 2) % KS, rest = (it >> 2) / KS;
      const int gp = rest & 3, x = rest >> 2;
      const int s = 4 * x + gp;
      uint32_t hw[2] = {0u, 0u}, lw[2] = {0u, 0u};
      if (s < P) {
        __half hv[4], lv[4];
#pragma unroll
        for (int pos = 0; pos < 4; ++pos) {
          const int j = jof<D, BITS>(tt, ks, pos);
          const float kv = row_at<R8>(s_kv + s * C::ROWS, j, BF16);
          const float xv = (col ? kv * __half2float(__ushort_as_half(s_sc[j])) : kv) * upx;
          hv[pos] = __float2half_rn(xv);
          lv[pos] = __float2half_rn(xv - __half2float(hv[pos]));
        }
        hw[0] = h2u(__halves2half2(hv[0], hv[1]));
        hw[1] = h2u(__halves2half2(hv[2], hv[3]));
        lw[0] = h2u(__halves2half2(lv[0], lv[1]));
        lw[1] = h2u(__halves2half2(lv[2], lv[3]));
      }
      // stored at row slot g ^ (ks & 3): a permutation inside each 256-byte
      // [g][t] block that spreads these stores over the banks
      sm.bx[x][ks][(2 * gp) ^ (ks & 3)][tt] = make_uint2(hw[0], hw[1]);
      sm.bx[x][ks][(2 * gp + 1) ^ (ks & 3)][tt] = make_uint2(lw[0], lw[1]);
    }
    // update B, built by fragment owner: entry (tau, u, g, t): column n = g of
    // tile tau = 2ks + hs is key channel jof(g/2, ks, 2hs + g%2); rows are the
    // k-slots 16u + 2t + {0, 1} (b0) and + {8, 9} (b1); slot sigma is token
    // sigma % PMAX of segment sigma / PMAX (K, K, K_lo)
    for (int it = tid; it < NT * KU * 32; it += C::THREADS) {
      const int tt = it & 3, gg = (it >> 2) & 7, tu = it >> 5;   // tu = tau * KU + u
      const int u = tu % KU, tau = tu / KU;
      const int j = jof<D, BITS>(gg >> 1, tau >> 1, 2 * (tau & 1) + (gg & 1));
      uint32_t wv[2];
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        __half hv[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int sigma = 16 * u + 2 * tt + e + 8 * q2;
          const int seg = sigma / PMAX, s2 = sigma % PMAX;
          __half h = __ushort_as_half((unsigned short)0);
          if (seg < C::NSEG && s2 < P) {
            const float kv = row_at<R8>(s_kv + s2 * C::ROWS, j, BF16);
            h = __float2half_rn(kv);
            if (seg == 2) h = __float2half_rn(kv - __half2float(h));
          }
          hv[e] = h;
        }
        wv[q2] = h2u(__halves2half2(hv[0], hv[1]));
      }
      sm.bkf[tau][u][gg][tt] = make_uint2(wv[0], wv[1]);
    }
  }
  if (__syncthreads_or(!ok)) return false;
  // every thread is past the previous head's encode: its flag is free for the head after this one
  if (tid == 0) sm.slow[parity_bit ^ 1] = 0;
  int& slow_flag = sm.slow[parity_bit];

  // ---- phase 2: this warp's 16 rows ------------------------------------------
  const int i0 = 16 * w + g, i1 = i0 + 8;
  uint32_t Af[KS][4];
  {
    RowBlock<D, BITS> rbk;
    load_rows_smem<D, BITS>(rbk, s_rec, w, g, t);
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) a_frag<D, BITS>(rbk, ks, Af[ks]);
  }
  // X = S~0 K^T: column 2s = hi, 2s+1 = lo of vector s
  float xacc[NTX][4];
#pragma unroll
  for (int x = 0; x < NTX; ++x) xacc[x][0] = xacc[x][1] = xacc[x][2] = xacc[x][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < KS; ++ks)
#pragma unroll
    for (int x = 0; x < NTX; ++x) {
      const uint2 bb = sm.bx[x][ks][g ^ (ks & 3)][t];
      mma16816(xacc[x], Af[ks], bb.x, bb.y);
    }
  // r_s = v_s - gamma_s x_s for this lane's vectors s = 4x + t, then all-gather in the quad
  float r[PMAX][2];
  {
    float ro[NTX][2];
    const float s0 = (col ? 1.f : sm.sc[i0]) * xinv, s1 = (col ? 1.f : sm.sc[i1]) * xinv;
#pragma unroll
    for (int x = 0; x < NTX; ++x) {
      const int s = 4 * x + t;
      ro[x][0] = ro[x][1] = 0.f;
      if (s < P) {
        const float gs = gam[s];
        ro[x][0] = row_at<R8>(s_kv + s * C::ROWS, D + i0, BF16) - gs * ((xacc[x][0] + xacc[x][1]) * s0);
        ro[x][1] = row_at<R8>(s_kv + s * C::ROWS, D + i1, BF16) - gs * ((xacc[x][2] + xacc[x][3]) * s1);
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
    float wrow[PMAX];
    if ((PS & 3) == 0 && s < P) {         // row s of W in 16-byte pieces (zero beyond P)
#pragma unroll
      for (int c = 0; c < PMAX / 4; ++c) {
        const float4 w4 = 4 * c < P ? reinterpret_cast<const float4*>(W + s * PS)[c]
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
        wrow[4 * c] = w4.x; wrow[4 * c + 1] = w4.y; wrow[4 * c + 2] = w4.z; wrow[4 * c + 3] = w4.w;
      }
    } else {
#pragma unroll
      for (int sp = 0; sp < PMAX; ++sp) wrow[sp] = (s < P && sp < P) ? W[s * PS + sp] : 0.f;
    }
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int sp = 0; sp < PMAX; ++sp) {
      a0 = fmaf(wrow[sp], r[sp][0], a0);
      a1 = fmaf(wrow[sp], r[sp][1], a1);
    }
    uh[q][0] = a0;
    uh[q][1] = a1;
    um = fmaxf(um, fmaxf(fabsf(a0), fabsf(a1)));
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) um = fmaxf(um, __shfl_xor_sync(FULL, um, off));
  int ex = 0;
  if (um >= 1.17549435e-38f && um < INFINITY) ex = max(-60, min(60, 14 - exp2_floor(um)));
  const float up = pow2i(ex), down = pow2i(-ex);
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
  // this warp's initialisation factors in fragment order: up gamma_P s_j (COL)
  WarpTab<D>& wt = sm.wt[w];
  if (col) {
    const float gp = gP * up;
    for (int e = lane; e < KS * 4; e += 32) {
      const int ks = e >> 2, tt = e & 3;
      float f[4];
#pragma unroll
      for (int pos = 0; pos < 4; ++pos) f[pos] = gp * sm.sc[jof<D, BITS>(tt, ks, pos)];
      wt.f[ks][tt] = make_float4(f[0], f[1], f[2], f[3]);
    }
    __syncwarp();
  }
  const float fr0 = up * gP * sm.sc[i0], fr1 = up * gP * sm.sc[i1];
  // accumulator: up gamma_P S~0 (the lane's own code fragments), then += U^^T K.
  // Tile 2ks + hs, element e of lane (g, t) is key channel jof(t, ks, 2hs + e).
  float acc[NT][4];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const float2 c0 = __half22float2(u2h(Af[ks][0])), c1 = __half22float2(u2h(Af[ks][1]));
    const float2 c2 = __half22float2(u2h(Af[ks][2])), c3 = __half22float2(u2h(Af[ks][3]));
    float2 fa, fb, fc, fd;   // factors of c0 (row g, pos 0/1), c1 (row g+8), c2 (row g, pos 2/3), c3
    if (col) {
      const float4 f = wt.f[ks][t];
      fa = fb = make_float2(f.x, f.y);
      fc = fd = make_float2(f.z, f.w);
    } else {
      fa = fc = make_float2(fr0, fr0);
      fb = fd = make_float2(fr1, fr1);
    }
    const float2 v0 = __fmul2_rn(c0, fa), v1 = __fmul2_rn(c1, fb);
    const float2 v2 = __fmul2_rn(c2, fc), v3 = __fmul2_rn(c3, fd);
    acc[2 * ks][0] = v0.x; acc[2 * ks][1] = v0.y; acc[2 * ks][2] = v1.x; acc[2 * ks][3] = v1.y;
    acc[2 * ks + 1][0] = v2.x; acc[2 * ks + 1][1] = v2.y; acc[2 * ks + 1][2] = v3.x; acc[2 * ks + 1][3] = v3.y;
#pragma unroll
    for (int hs = 0; hs < 2; ++hs)
#pragma unroll
      for (int u = 0; u < KU; ++u) {
        const uint2 bb = sm.bkf[2 * ks + hs][u][g][t];
        mma16816(acc[2 * ks + hs], Au[u], bb.x, bb.y);
      }
  }

  // ---- absmax ----------------------------------------------------------------
  if (col) {
    float v[2 * NT];
#pragma unroll
    for (int tau = 0; tau < NT; ++tau) {
      v[2 * tau] = max_nan(fabsf(acc[tau][0]), fabsf(acc[tau][2]));
      v[2 * tau + 1] = max_nan(fabsf(acc[tau][1]), fabsf(acc[tau][3]));
    }
    // transpose-reduce over the 8 row lanes (lane bits 4, 3, 2)
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
    // the lane keeps value indices (2NT/8) g + k (tile idx >> 1, element idx & 1)
#pragma unroll
    for (int k = 0; k < 2 * NT / 8; ++k) {
      const int idx = (2 * NT / 8) * g + k;
      const int tau = idx >> 1;
      sm.colmax[w][jof<D, BITS>(t, tau >> 1, 2 * (tau & 1) + (idx & 1))] = v[k] * down;
    }
  } else {
    float m0 = 0.f, m1 = 0.f;
#pragma unroll
    for (int tau = 0; tau < NT; ++tau) {
      m0 = max_nan(m0, max_nan(fabsf(acc[tau][0]), fabsf(acc[tau][1])));
      m1 = max_nan(m1, max_nan(fabsf(acc[tau][2]), fabsf(acc[tau][3])));
    }
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
      m0 = max_nan(m0, __shfl_xor_sync(FULL, m0, off));
      m1 = max_nan(m1, __shfl_xor_sync(FULL, m1, off));
    }
    if (t == 0) {
      const float a0 = m0 * down, a1 = m1 * down;
      const GroupScale s0 = group_scale(a0, isfinite(a0), qmax, p.flags);
      const GroupScale s1 = group_scale(a1, isfinite(a1), qmax, p.flags);
      const bool bad = !fast_encode_ok(a0, s0, qmax) || !fast_encode_ok(a1, s1, qmax);
      rsc[i0] = s0.bits;
      rsc[i1] = s1.bits;
      sm.qf[i0] = s0.sf > 0.f ? __frcp_rn(s0.sf) : 0.f;
      sm.qf[i1] = s1.sf > 0.f ? __frcp_rn(s1.sf) : 0.f;
      sm.sfv[i0] = s0.sf;
      sm.sfv[i1] = s1.sf;
      if (bad) slow_flag = 1;
    }
  }
  __syncthreads();
  issue_next();   // the issuing thread is idle during the scale pass
  if (col) {
    for (int j = tid; j < D; j += C::THREADS) {
      float a = 0.f;
#pragma unroll
      for (int ww = 0; ww < C::RB; ++ww) a = max_nan(a, sm.colmax[ww][j]);
      const GroupScale s = group_scale(a, isfinite(a), qmax, p.flags);
      rsc[j] = s.bits;
      sm.qf[j] = s.sf > 0.f ? __frcp_rn(s.sf) : 0.f;
      sm.sfv[j] = s.sf;
      if (!fast_encode_ok(a, s, qmax)) slow_flag = 1;
    }
    __syncthreads();
  }

  // ---- encode and store this warp's rows ------------------------------------
  const bool slow = slow_flag != 0;
  if (col) {
    for (int e = lane; e < KS * 4; e += 32) {
      const int ks = e >> 2, tt = e & 3;
      float f[4];
#pragma unroll
      for (int pos = 0; pos < 4; ++pos) {
        const int j = jof<D, BITS>(tt, ks, pos);
        f[pos] = slow ? sm.sfv[j] : sm.qf[j] * down;
      }
      wt.q[ks][tt] = make_float4(f[0], f[1], f[2], f[3]);
    }
    __syncwarp();
  }
  const float qr0 = col ? 0.f : (slow ? sm.sfv[i0] : sm.qf[i0] * down);
  const float qr1 = col ? 0.f : (slow ? sm.sfv[i1] : sm.qf[i1] * down);
  auto encode_rows = [&](auto fast) {
    // magic f16 pair of tile tau, row half rr: elements (2rr, 2rr + 1) are the
    // key channels jof(t, tau / 2, 2 (tau % 2) + {0, 1}), adjacent registers
    auto hq = [&](int tau, int rr) -> uint32_t {
      const float a = acc[tau][2 * rr], bq = acc[tau][2 * rr + 1];
      float qa = rr ? qr1 : qr0, qb = qa;
      if (col) {
        const float4 q4 = wt.q[tau >> 1][t];
        qa = (tau & 1) ? q4.z : q4.x;
        qb = (tau & 1) ? q4.w : q4.y;
      }
      if (decltype(fast)::value) return magic_fast<BITS>(a, bq, qa, qb);
      return magic_exact<BITS>(a * down, bq * down, qa, qb);
    };
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      uint8_t* row = rec + (size_t)(rr ? i1 : i0) * ROWB;
      if (BITS == 4) {
        // word m holds channels 8m + k of the lane's range; tiles 4m .. 4m+3
        // hold k = (0, 4), (1, 5), (2, 6), (3, 7), each code in the low byte
        // of its f16 half
        constexpr int NW = D / 32;
        uint32_t wd[NW];
#pragma unroll
        for (int m = 0; m < NW; ++m) {
          const uint32_t h04 = hq(4 * m, rr), h15 = hq(4 * m + 1, rr);
          const uint32_t h26 = hq(4 * m + 2, rr), h37 = hq(4 * m + 3, rr);
          const uint32_t E = prmt(h04, h26, 0x6240u);   // k 0 2 4 6
          const uint32_t O = prmt(h15, h37, 0x6240u);   // k 1 3 5 7
          wd[m] = (E | (O << 4)) ^ 0x88888888u;
        }
        uint8_t* dst = row + chunk_offset<D, 4>(t, 0);
        if (NW == 4) *reinterpret_cast<uint4*>(dst) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        else if (NW == 2) *reinterpret_cast<uint2*>(dst) = make_uint2(wd[0], wd[1]);
        else *reinterpret_cast<uint32_t*>(dst) = wd[0];
      } else {
        // k-step ks covers channels base + pos of one code word: tiles 2ks, 2ks+1
        constexpr int WPC = D / 32;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t wd[WPC];
#pragma unroll
          for (int m = 0; m < WPC; ++m) {
            const int ks = c * WPC + m;
            wd[m] = prmt(hq(2 * ks, rr), hq(2 * ks + 1, rr), 0x6420u) ^ 0x80808080u;
          }
          uint8_t* dst = row + chunk_offset<D, 8>(t, c);
          if (WPC == 4) *reinterpret_cast<uint4*>(dst) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
          else if (WPC == 2) *reinterpret_cast<uint2*>(dst) = make_uint2(wd[0], wd[1]);
          else *reinterpret_cast<uint32_t*>(dst) = wd[0];
        }
      }
    }
  };
  if (!slow) encode_rows(std::true_type{});
  else encode_rows(std::false_type{});
  if (tid == 0) p.fill[head] = 0;
  return true;
}

template <int D, bool BF16, int PMAX, bool EXACT, bool R8>
__global__ void __launch_bounds__(Cfg<D, BF16, PMAX>::THREADS, 2)
    commit_kernel(PoolDev p, Span sp) {
  using C = Cfg<D, BF16, PMAX>;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Smem<D, BF16, PMAX>& sm = *reinterpret_cast<Smem<D, BF16, PMAX>*>(smem_raw);
  const int tid = threadIdx.x;
  // heads [b0 H, (b0 + nb) H) of this launch; n_heads is the end index
  const int first_head = sp.b0 * p.H;
  const int n_heads = (sp.b0 + sp.nb) * p.H;
  // thread ISS (idle during the scale pass) issues every bulk copy.  Its
  // warp finds the first due heads 32 at a time (a launch may have none);
  // afterwards ISS keeps the candidate after the staged heads and its fill
  // count, loaded one head ahead, so a due candidate costs no wait.
  constexpr int ISS = C::THREADS / 2;
  const bool iss_warp = (tid >> 5) == (ISS >> 5);
  const int lane = tid & 31;
  int cand = n_heads, cand_fill = 0;
  if (iss_warp) {
    if (tid == ISS) {
      for (int i = 0; i < 3; ++i) mbar_init(&sm.bar[i], 1);
      fence_mbar_init();
      for (int i = 0; i < 3; ++i) sm.hq[i] = n_heads;
    }
    int h = find_full_warp(p, first_head + blockIdx.x, gridDim.x, n_heads, lane);
    for (int i = 0; i < 2; ++i) {
      if (tid == ISS) {
        sm.hq[i] = h;
        if (h < n_heads) {
          sm.hn[i] = p.fill[h] & 0xff;
          issue_head<D, BF16, PMAX, R8>(p, h, sm, i);
        }
      }
      if (h < n_heads) h = find_full_warp(p, h + gridDim.x, gridDim.x, n_heads, lane);
    }
    cand = h;
    if (cand < n_heads) cand_fill = p.fill[cand];
  }
  if (tid == 0) sm.slow[0] = sm.slow[1] = 0;
  __syncthreads();
  uint32_t parity = 0u;
  int s = 0, iter = 0;
  while (true) {
    const int head = sm.hq[s];
    if (head >= n_heads) break;
    const bool ok = mbar_wait_bounded(&sm.bar[s], (parity >> s) & 1u, p.flags);
    parity ^= 1u << s;
    const int s2 = s == 0 ? 2 : s - 1;   // slot of the head two ahead (held the previous head)
    auto issue_next = [&]() {   // every thread of the block calls it
      if (tid == ISS) {
        int nxt = cand, nfill = cand_fill;
        while (nxt < n_heads && !commit_due(nfill, p.P)) {
          nxt += gridDim.x;
          nfill = nxt < n_heads ? p.fill[nxt] : 0;
        }
        sm.hq[s2] = nxt;
        if (nxt < n_heads) {
          sm.hn[s2] = nfill & 0xff;
          issue_head<D, BF16, PMAX, R8>(p, nxt, sm, s2);
        }
        cand = nxt < n_heads ? nxt + gridDim.x : n_heads;
        if (cand < n_heads) cand_fill = p.fill[cand];
      }
    };
    const bool done =
        p.bits[head % p.H] == 4
            ? commit_head<D, BF16, PMAX, 4, EXACT, R8>(p, head, sm, sm.slot[s], sm.hn[s], ok, iter & 1,
                                                   issue_next)
            : commit_head<D, BF16, PMAX, 8, EXACT, R8>(p, head, sm, sm.slot[s], sm.hn[s], ok, iter & 1,
                                                   issue_next);
    if (!done) {   // a bounded wait gave up: let the copies in flight land, then leave
      if (tid == ISS)
        for (int i = 0; i < 3; ++i)
          if (i != s && sm.hq[i] < n_heads) mbar_wait_bounded(&sm.bar[i], (parity >> i) & 1u, nullptr);
      __syncthreads();
      return;
    }
    ++iter;
    s = s == 2 ? 0 : s + 1;
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

template <int D, bool BF16, int PMAX, bool EXACT, bool R8 = false>
cudaError_t launch_t(const PoolDev& p, const Span& sp, cudaStream_t st) {
  using C = Cfg<D, BF16, PMAX>;
  const size_t smem = sizeof(Smem<D, BF16, PMAX>);
  cudaError_t e = cudaFuncSetAttribute(commit_kernel<D, BF16, PMAX, EXACT, R8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long heads = (long)sp.nb * p.H;
  if (heads == 0) return cudaSuccess;
  long blocks = (long)(sp.blocks_per_sm > 0 ? sp.blocks_per_sm : 2) * sm_count_dev() *
                (D == 128 ? 1 : D == 64 ? 2 : 4);
  if (blocks > heads) blocks = heads;
  commit_kernel<D, BF16, PMAX, EXACT, R8><<<(unsigned)blocks, C::THREADS, smem, st>>>(p, sp);
  return cudaGetLastError();
}

template <int D, bool BF16>
cudaError_t launch_p(const PoolDev& p, const Span& sp, cudaStream_t st) {
  if (p.row8) {   // E4M3 buffered rows
    if (!p.adaptive) switch (p.P) {
      case 4: return launch_t<D, BF16, 4, true, true>(p, sp, st);
      case 8: return launch_t<D, BF16, 8, true, true>(p, sp, st);
      case 16: return launch_t<D, BF16, 16, true, true>(p, sp, st);
    }
    if (p.P <= 4) return launch_t<D, BF16, 4, false, true>(p, sp, st);
    if (p.P <= 8) return launch_t<D, BF16, 8, false, true>(p, sp, st);
    return launch_t<D, BF16, 16, false, true>(p, sp, st);
  }
  // heads marked early hold fewer than P tokens: per-head token counts
  if (!p.adaptive) switch (p.P) {
    case 4: return launch_t<D, BF16, 4, true>(p, sp, st);
    case 8: return launch_t<D, BF16, 8, true>(p, sp, st);
    case 16: return launch_t<D, BF16, 16, true>(p, sp, st);
  }
  if (p.P <= 4) return launch_t<D, BF16, 4, false>(p, sp, st);
  if (p.P <= 8) return launch_t<D, BF16, 8, false>(p, sp, st);
  return launch_t<D, BF16, 16, false>(p, sp, st);
}

}  // namespace

cudaError_t launch_commit(const PoolDev& p, const Span& sp, cudaStream_t st) {
  const bool bf = p.io == PACE_IO_BF16;
  switch (p.d_k) {
    case 32: return bf ? launch_p<32, true>(p, sp, st) : launch_p<32, false>(p, sp, st);
    case 64: return bf ? launch_p<64, true>(p, sp, st) : launch_p<64, false>(p, sp, st);
    case 128: return bf ? launch_p<128, true>(p, sp, st) : launch_p<128, false>(p, sp, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace pace
