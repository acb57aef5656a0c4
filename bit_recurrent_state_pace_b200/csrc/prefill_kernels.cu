// Chunked fp32 prefill into the pool: T tokens for every (slot, head), with
// the state kept in fp32 from the stored (dequantised) state to the last
// token and rounded once, at the end.
//
// "PACE: A New 4-Bit Recurrent State Quantization Method ...", section
// "Periodic Rounding" (the chunked prefill kernels whose once-per-chunk
// rounding the method borrows), and "PACE: four-bit recurrent state by
// rounding less often", flowchart "State update, chunked, high precision".
// Chunks of CH = 8 tokens use the UT/WY form: for a chunk with decays
// gamma_s (products of alpha up to token s) and state S at its start,
//   X = S K^T, Y = S Q^T, U = T diag(beta) (V - diag(gamma) X^T),
//   T = (I + A)^{-1}, A[t][s] = beta_t gamma_{t/s} k_t.k_s (s < t),
//   o_t = gamma_t y_t + sum_{s <= t} gamma_{t/s} (q_t.k_s) u_s,
//   S' = gamma_n S + sum_s gamma_{n/s} u_s k_s^T.
//
// Design (B200): one CTA per head, one warp per 16 value rows; the state
// lives in the warps' MMA accumulators for the whole prompt.  The products
// with S use the accumulator tiles directly as A fragments (split hi + lo
// f16 under a per-warp power of two); K and Q enter as B-fragment tables
// built per chunk in shared memory; the chunk's 128 dot products run
// lane-parallel with a shuffle transpose-reduce; the T solve is
// column-per-lane.  The final state is encoded like a period commit
// (column or row absmax, FP16 scales, round half to even, packed in place).
#include "update_common.cuh"

namespace pace {

namespace {

constexpr unsigned FULL = 0xffffffffu;
constexpr int CH = 8;   // tokens per chunk

template <int D, bool BF16>
struct PCfg {
  static constexpr int RB = D / 16;                 // warps (16-row blocks)
  static constexpr int THREADS = 32 * RB;
  static constexpr int KS = D / 16;                 // k16 steps over key channels
  static constexpr int NT = D / 8;                  // n8 tiles over key channels
  static constexpr int NSEG = BF16 ? 2 : 3;         // update segments (K, K, K_lo)
  static constexpr int KU = (NSEG * CH + 15) / 16;  // update k16 steps
  static constexpr int NKX = BF16 ? 2 : 4;          // K, Q (+ K_lo, Q_lo) operand tiles
  static constexpr int MINB = D == 128 ? 2 : 1;     // CTAs (heads) in flight per SM
};

template <int D, bool BF16>
struct alignas(16) PSmem {
  using C = PCfg<D, BF16>;
  // chunk rows k [0], q [1], v [2] in the io dtype, double-buffered: chunk
  // c + 1 arrives by asynchronous copies while chunk c computes.  Rows sit
  // 16 bytes past a multiple of 128, so the same channel of different
  // tokens falls in different banks when the operand tables gather it.
  uint8_t raw[2][3][CH][D * (BF16 ? 2 : 4) + 16];
  float abuf[2][2][CH];               // [buffer][alpha, beta][token]
  uint2 bx[C::NKX][C::KS][8][4];      // K / Q B fragments [tile][ks][g][t]
  uint2 bkf[C::NT][C::KU][8][4];      // update B fragments [tile][u][g][t]
  float G[CH][CH], M[CH][CH];         // k_t.k_s and q_t.k_s
  float TB[CH][CH];                   // T[s][s'] beta_s'
  float MW[CH][CH];                   // gamma_{t/s} q_t.k_s for s <= t
  float gam[CH], suf[CH];
  float sc[D];                        // stored scales, then new 1/s16 and s16
  float qf[D], sfv[D];
  float colmax[C::RB][D];
  float4 wq[C::RB][C::KS][4];         // per-warp quantisation factors in fragment order
  int slow;
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Issue the asynchronous copies of chunk rows [c0, c0 + n) of k, q, v for
// `head` into staging buffer `buf` (16-byte pieces over the block's threads).
template <int D, bool BF16, class SM>
__device__ __forceinline__ void stage_chunk(SM& sm, int buf, int64_t c0, int n, int64_t BH, int head,
                                            const void* q, const void* k, const void* v, int nthreads) {
  constexpr int RBYTES = D * (BF16 ? 2 : 4);
  constexpr int PIECES = RBYTES / 16;
  for (int it = threadIdx.x; it < 3 * n * PIECES; it += nthreads) {
    const int which = it / (n * PIECES), rem = it - which * n * PIECES;
    const int s = rem / PIECES, pc = rem - s * PIECES;
    const uint8_t* src = reinterpret_cast<const uint8_t*>(which == 0 ? k : which == 1 ? q : v) +
                         (size_t)((c0 + s) * BH + head) * RBYTES + 16 * pc;
    cp_async16(&sm.raw[buf][which][s][16 * pc], src);
  }
  cp_async_commit();
}

// Four 8 x 8 b16 matrices from shared memory (lane l gives the address of
// row l % 8 of matrix l / 8), as the A fragment of m16n8k16.
__device__ __forceinline__ void ldsm_x4(const void* row, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"((uint32_t)__cvta_generic_to_shared(row)));
}
// Two 8 x 8 b16 matrices (lanes 0..15 give the row addresses), as the B
// fragment of m16n8k16 when the rows are B's columns.
__device__ __forceinline__ void ldsm_x2(const void* row, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"((uint32_t)__cvta_generic_to_shared(row)));
}
__device__ __forceinline__ void mma16816_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Lane L ends with the warp-wide sum of value index (L mod V).
template <int V>
__device__ __forceinline__ float transpose_sum(float (&v)[V], int lane) {
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

template <int D, bool BF16, int BITS>
__device__ void prefill_head(const PoolDev& p, int head, int64_t T, const void* q, const void* k,
                             const void* v, const void* alpha, const void* beta, float* o,
                             PSmem<D, BF16>& sm) {
  using C = PCfg<D, BF16>;
  constexpr int KS = C::KS, NT = C::NT, KU = C::KU, NKX = C::NKX;
  constexpr int ROWB = D * BITS / 8;
  constexpr int ESZ = BF16 ? 2 : 4;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, g = lane >> 2, t = lane & 3;
  const int h = head % p.H, b = head / p.H;
  const bool col = p.axis == PACE_SCALE_COL;
  const int qmax = BITS == 4 ? 7 : 127;
  const int64_t BH = (int64_t)p.B * p.H;
  uint8_t* rec = p.state + (size_t)b * p.slot_stride + p.rec_off[h];
  uint16_t* rsc = reinterpret_cast<uint16_t*>(rec + code_bytes(D, D, BITS));
  const int i0 = 16 * w + g, i1 = i0 + 8;

  // ---- stored state -> fp32 accumulators (rows i0, i1; fragment channels) ---
  for (int j = tid; j < D; j += C::THREADS) sm.sc[j] = __half2float(__ushort_as_half(rsc[j]));
  if (tid == 0) sm.slow = 0;
  __syncthreads();
  float acc[NT][4];
  {
    RowBlock<D, BITS> rbk;
    rbk.load(rec, w, g, t);
    const float fr0 = col ? 1.f : sm.sc[i0], fr1 = col ? 1.f : sm.sc[i1];
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      uint32_t af[4];
      a_frag<D, BITS>(rbk, ks, af);
#pragma unroll
      for (int hs = 0; hs < 2; ++hs) {
        const float2 c0 = __half22float2(u2h(af[2 * hs])), c1 = __half22float2(u2h(af[2 * hs + 1]));
        const float f0 = col ? sm.sc[jof<D, BITS>(t, ks, 2 * hs)] : fr0;
        const float f1 = col ? sm.sc[jof<D, BITS>(t, ks, 2 * hs + 1)] : fr0;
        const float f2 = col ? f0 : fr1, f3 = col ? f1 : fr1;
        acc[2 * ks + hs][0] = c0.x * f0;
        acc[2 * ks + hs][1] = c0.y * f1;
        acc[2 * ks + hs][2] = c1.x * f2;
        acc[2 * ks + hs][3] = c1.y * f3;
      }
    }
  }
  float F = 1.f;   // acc = F * S

  // ---- chunks ----------------------------------------------------------------
  const int io = BF16 ? PACE_IO_BF16 : PACE_IO_F32;
  auto kq = [&](int buf, int which, int s, int e) -> float { return io_at(sm.raw[buf][which][s], e, BF16); };
  // chunk 0: rows by asynchronous copy, gates directly
  if (T > 0) stage_chunk<D, BF16>(sm, 0, 0, T < CH ? (int)T : CH, BH, head, q, k, v, C::THREADS);
  if (tid < CH) {
    const bool in = tid < T;
    const size_t row = (size_t)(tid * BH + head);
    sm.abuf[0][0][tid] = in ? load_io(alpha, row, io) : 1.f;
    sm.abuf[0][1][tid] = in ? load_io(beta, row, io) : 0.f;
  }
  int buf = 0;
  for (int64_t c0 = 0; c0 < T; c0 += CH, buf ^= 1) {
    const int n = (int)((T - c0) < CH ? (T - c0) : CH);
    cp_async_wait_all();
    // rows past the last token read as zero
    for (int idx = tid; idx < 3 * (CH - n) * D; idx += C::THREADS) {
      const int which = idx / ((CH - n) * D), rem = idx - which * (CH - n) * D;
      const int s = n + rem / D, e = rem % D;
      if (BF16) reinterpret_cast<uint16_t*>(sm.raw[buf][which][s])[e] = 0;
      else reinterpret_cast<float*>(sm.raw[buf][which][s])[e] = 0.f;
    }
    __syncthreads();   // chunk c staged; the previous chunk's readers are done
    // chunk c + 1: rows now (asynchronous), gates into registers of the last
    // warp's first lanes, stored before the chunk ends
    const int64_t c1 = c0 + CH;
    const int n1 = c1 < T ? (int)((T - c1) < CH ? (T - c1) : CH) : 0;
    if (n1 > 0) stage_chunk<D, BF16>(sm, buf ^ 1, c1, n1, BH, head, q, k, v, C::THREADS);
    const int gl = tid - (C::THREADS - 32);   // lane of the last warp
    float a_nx = 1.f, b_nx = 0.f;
    if (gl >= 0 && gl < CH && gl < n1) {
      const size_t row = (size_t)((c1 + gl) * BH + head);
      a_nx = load_io(alpha, row, io);
      b_nx = load_io(beta, row, io);
    }

    // b. dot products k_t.k_s (G) and q_t.k_s (M).  bf16 rows: one warp on the
    //    tensor cores (exact products, fp32 sums), A = [k rows; q rows], B =
    //    the k rows as columns, while the other warps go on to the operand
    //    tables.  fp32 rows: lane-parallel sums in groups of 16 (G: 0..63,
    //    M: 64..127), groups strided over the warps.
    if constexpr (BF16) {
      if (w == 0) {
        float dg[4] = {0.f, 0.f, 0.f, 0.f};
        const int mq = lane >> 3, rr = lane & 7;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          uint32_t a[4], b0, b1;
          // matrices: (k rows, cols 16ks..), (q rows, 16ks..), (k rows, 16ks+8..), (q rows, 16ks+8..)
          ldsm_x4(&sm.raw[buf][mq & 1][rr][2 * (16 * ks + 8 * (mq >> 1))], a);
          ldsm_x2(&sm.raw[buf][0][rr][2 * (16 * ks + 8 * (mq & 1))], b0, b1);
          mma16816_bf16(dg, a, b0, b1);
        }
        sm.G[g][2 * t] = dg[0];
        sm.G[g][2 * t + 1] = dg[1];
        sm.M[g][2 * t] = dg[2];
        sm.M[g][2 * t + 1] = dg[3];
        __syncwarp();
      }
    } else {
    for (int base = 16 * w; base < 2 * CH * CH; base += 16 * C::RB) {
      float part[16];
#pragma unroll
      for (int d = 0; d < 16; ++d) {
        const int dd = base + d;
        const int which = dd / (CH * CH), tt = (dd / CH) % CH, ss = dd % CH;
        float a = 0.f;
#pragma unroll
        for (int e = lane; e < D; e += 32) a = fmaf(kq(buf, which, tt, e), kq(buf, 0, ss, e), a);
        part[d] = a;
      }
      const float r = transpose_sum<16>(part, lane);
      if (lane < 16) {
        const int dd = base + lane;
        const int which = dd / (CH * CH), tt = (dd / CH) % CH, ss = dd % CH;
        if (which == 0) sm.G[tt][ss] = r;
        else sm.M[tt][ss] = r;
      }
    }
    __syncthreads();   // dot products ready
    }
    // warps 1.. build the operand tables while warp 0 forms the chunk scalars
    const int tbl_tid = tid - 32, tbl_n = C::THREADS - 32;
    // K / Q B-fragment tables: entry (x, ks, g, t) of tile x (K, Q, K_lo, Q_lo)
    // holds channels jof(t, ks, 0..3) of token g
    for (int it = tbl_tid; tbl_tid >= 0 && it < NKX * KS * 32; it += tbl_n) {
      const int tt = it & 3, gg = (it >> 2) & 7, xk = it >> 5;
      const int ks = xk % KS, x = xk / KS;
      __half hv[4];
#pragma unroll
      for (int pos = 0; pos < 4; ++pos) {
        const float val = kq(buf, x & 1, gg, jof<D, BITS>(tt, ks, pos));
        const __half hi = __float2half_rn(val);
        hv[pos] = x < 2 ? hi : __float2half_rn(val - __half2float(hi));
      }
      sm.bx[x][ks][gg][tt] = make_uint2(h2u(__halves2half2(hv[0], hv[1])), h2u(__halves2half2(hv[2], hv[3])));
    }
    // update B table, as in the period commit (slots: token sigma % CH of segment sigma / CH)
    for (int it = tbl_tid; tbl_tid >= 0 && it < NT * KU * 32; it += tbl_n) {
      const int tt = it & 3, gg = (it >> 2) & 7, tu = it >> 5;
      const int u = tu % KU, tau = tu / KU;
      const int j = jof<D, BITS>(gg >> 1, tau >> 1, 2 * (tau & 1) + (gg & 1));
      uint32_t wv[2];
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        __half hv[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int sigma = 16 * u + 2 * tt + e + 8 * q2;
          const int seg = sigma / CH, s2 = sigma % CH;
          __half hh = __ushort_as_half((unsigned short)0);
          if (seg < C::NSEG) {
            const float kv = kq(buf, 0, s2, j);
            hh = __float2half_rn(kv);
            if (seg == 2) hh = __float2half_rn(kv - __half2float(hh));
          }
          hv[e] = hh;
        }
        wv[q2] = h2u(__halves2half2(hv[0], hv[1]));
      }
      sm.bkf[tau][u][gg][tt] = make_uint2(wv[0], wv[1]);
    }

    // c. chunk scalars, lane s = token s (warp 0)
    if (w == 0) {
      const bool in = lane < n;
      const float al = in ? sm.abuf[buf][0][lane] : 1.f, be = in ? sm.abuf[buf][1][lane] : 0.f;
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
      // column s of A: A[t][s] = beta_t gamma_{t/s} G[t][s], t > s; column s of
      // the decayed scores: gamma_{t/s} M[t][s], t >= s
      float acol[CH], mcol[CH];
      float run = 1.f;
#pragma unroll
      for (int tt = 0; tt < CH; ++tt) {
        const float at = __shfl_sync(FULL, al, tt), bt = __shfl_sync(FULL, be, tt);
        if (tt > lane) run *= at;
        const bool valid = lane < CH;
        acol[tt] = (valid && tt > lane && tt < n) ? bt * run * sm.G[tt][lane < CH ? lane : 0] : 0.f;
        mcol[tt] = (valid && tt >= lane && tt < n) ? run * sm.M[tt][lane < CH ? lane : 0] : 0.f;
      }
      // T = (I + A)^{-1}, column s by forward substitution
      float Tc[CH];
#pragma unroll
      for (int tt = 0; tt < CH; ++tt) {
        float a2 = 0.f;
#pragma unroll
        for (int r = 0; r < tt; ++r) {
          const float Atr = __shfl_sync(FULL, acol[tt], r);   // A[tt][r] from lane r
          if (r >= lane) a2 = fmaf(Atr, Tc[r], a2);
        }
        Tc[tt] = tt == lane ? 1.f : (tt > lane ? -a2 : 0.f);
      }
      if (lane < CH) {
#pragma unroll
        for (int tt = 0; tt < CH; ++tt) {
          sm.TB[tt][lane] = Tc[tt] * be;
          sm.MW[tt][lane] = mcol[tt];
        }
        sm.gam[lane] = gcum;
        sm.suf[lane] = suf;
      }
    }
    __syncthreads();

    // d. X = S K^T, Y = S Q^T from the accumulator tiles (hi + lo under 2^ex)
    float m = 0.f;
#pragma unroll
    for (int tau = 0; tau < NT; ++tau)
#pragma unroll
      for (int e = 0; e < 4; ++e) m = fmaxf(m, fabsf(acc[tau][e]));
#pragma unroll
    for (int off = 16; off; off >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, off));
    int ex = 0;
    if (m >= 1.17549435e-38f && m < INFINITY) ex = max(-120, min(120, 14 - exp2_floor(m)));
    const float ups = pow2i(ex);
    float xk[4] = {0.f, 0.f, 0.f, 0.f}, xq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      uint32_t ahi[4], alo[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        // a0: tile 2ks rows g; a1: tile 2ks rows g+8; a2, a3: tile 2ks+1
        const float x0 = acc[2 * ks + (r >> 1)][2 * (r & 1)] * ups;
        const float x1 = acc[2 * ks + (r >> 1)][2 * (r & 1) + 1] * ups;
        const __half2 hh = __floats2half2_rn(x0, x1);
        const float2 back = __half22float2(hh);
        ahi[r] = h2u(hh);
        alo[r] = h2u(__floats2half2_rn(x0 - back.x, x1 - back.y));
      }
      // a0 = rows g, k 2t..; a1 = rows g+8; a2 = rows g, k+8; a3 = rows g+8, k+8
      // the A fragment order is (tile 2ks rows g, rows g+8, tile 2ks+1 rows g, rows g+8)
      const uint32_t A_hi[4] = {ahi[0], ahi[1], ahi[2], ahi[3]};
      const uint32_t A_lo[4] = {alo[0], alo[1], alo[2], alo[3]};
      const uint2 bk = sm.bx[0][ks][g][t], bq = sm.bx[1][ks][g][t];
      mma16816(xk, A_hi, bk.x, bk.y);
      mma16816(xk, A_lo, bk.x, bk.y);
      mma16816(xq, A_hi, bq.x, bq.y);
      mma16816(xq, A_lo, bq.x, bq.y);
      if (!BF16) {
        const uint2 bkl = sm.bx[2][ks][g][t], bql = sm.bx[3][ks][g][t];
        mma16816(xk, A_hi, bkl.x, bkl.y);
        mma16816(xq, A_hi, bql.x, bql.y);
      }
    }
    const float inv = 1.f / (ups * F);   // both powers of two
    // e. r_s = v_s - gamma_s x_s for tokens 2t, 2t+1 (rows i0, i1), gathered over the quad
    float r[CH][2];
    {
      float ro[2][2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int s = 2 * t + e;
        const float gs = sm.gam[s];
        ro[e][0] = kq(buf, 2, s, i0) - gs * (xk[e] * inv);
        ro[e][1] = kq(buf, 2, s, i1) - gs * (xk[2 + e] * inv);
      }
#pragma unroll
      for (int src = 0; src < 4; ++src)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          r[2 * src + e][0] = __shfl_sync(FULL, ro[e][0], (lane & ~3) | src);
          r[2 * src + e][1] = __shfl_sync(FULL, ro[e][1], (lane & ~3) | src);
        }
    }
    // f. u_s = sum_s' T[s][s'] beta_s' r_s' for every token; outputs of tokens 2t, 2t+1
    float u[CH][2];
#pragma unroll
    for (int s = 0; s < CH; ++s) {
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int sp = 0; sp < CH; ++sp) {
        const float tb = sm.TB[s][sp];
        a0 = fmaf(tb, r[sp][0], a0);
        a1 = fmaf(tb, r[sp][1], a1);
      }
      u[s][0] = a0;
      u[s][1] = a1;
    }
    if (o) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int tt = 2 * t + e;
        if (tt < n) {
          float o0 = sm.gam[tt] * (xq[e] * inv), o1 = sm.gam[tt] * (xq[2 + e] * inv);
#pragma unroll
          for (int s = 0; s < CH; ++s) {
            const float mw = sm.MW[tt][s];
            o0 = fmaf(mw, u[s][0], o0);
            o1 = fmaf(mw, u[s][1], o1);
          }
          float* orow = o + (size_t)((c0 + tt) * BH + head) * D;
          orow[i0] = o0;
          orow[i1] = o1;
        }
      }
    }
    // g. S' = gamma_n S + U^^T K with U^_s = gamma_{n/s} u_s; acc keeps F' = 2^eu S'
    float uh[2][2];   // this lane's update slots: tokens 2t, 2t+1
    float um = 0.f;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float sf = sm.suf[2 * t + e];
      uh[e][0] = sf * u[2 * t + e][0];
      uh[e][1] = sf * u[2 * t + e][1];
      um = fmaxf(um, fmaxf(fabsf(uh[e][0]), fabsf(uh[e][1])));
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) um = fmaxf(um, __shfl_xor_sync(FULL, um, off));
    int eu = 0;
    if (um >= 1.17549435e-38f && um < INFINITY) eu = max(-60, min(60, 14 - exp2_floor(um)));
    const float upu = pow2i(eu);
    const float rescale = sm.gam[n - 1] * upu / F;
#pragma unroll
    for (int tau = 0; tau < NT; ++tau)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[tau][e] *= rescale;
    F = upu;
    uint32_t Au[KU][4];
    {
      __half hv[2][2][2];   // [token e][row][hi, lo]
#pragma unroll
      for (int e = 0; e < 2; ++e)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const float x = uh[e][rr] * upu;
          hv[e][rr][0] = __float2half_rn(x);
          hv[e][rr][1] = __float2half_rn(x - __half2float(hv[e][rr][0]));
        }
#pragma unroll
      for (int uu = 0; uu < KU; ++uu) {
        __half vk[4][2];   // [slot k][row]
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const int sigma = 16 * uu + 2 * t + (kk & 1) + 8 * (kk >> 1);
          const int seg = sigma / CH;
#pragma unroll
          for (int rr = 0; rr < 2; ++rr)
            vk[kk][rr] = seg >= C::NSEG ? __ushort_as_half((unsigned short)0)
                                        : hv[kk & 1][rr][seg == 1 ? 1 : 0];
        }
        Au[uu][0] = h2u(__halves2half2(vk[0][0], vk[1][0]));
        Au[uu][1] = h2u(__halves2half2(vk[0][1], vk[1][1]));
        Au[uu][2] = h2u(__halves2half2(vk[2][0], vk[3][0]));
        Au[uu][3] = h2u(__halves2half2(vk[2][1], vk[3][1]));
      }
    }
#pragma unroll
    for (int tau = 0; tau < NT; ++tau)
#pragma unroll
      for (int uu = 0; uu < KU; ++uu) {
        const uint2 bb = sm.bkf[tau][uu][g][t];
        mma16816(acc[tau], Au[uu], bb.x, bb.y);
      }
    if (gl >= 0 && gl < CH) {
      sm.abuf[buf ^ 1][0][gl] = a_nx;
      sm.abuf[buf ^ 1][1][gl] = b_nx;
    }
  }

  // ---- encode the final state (acc = F S) --------------------------------------
  const float down = 1.f / F;
  if (col) {
    float vcol[2 * NT];
#pragma unroll
    for (int tau = 0; tau < NT; ++tau) {
      vcol[2 * tau] = max_nan(fabsf(acc[tau][0]), fabsf(acc[tau][2]));
      vcol[2 * tau + 1] = max_nan(fabsf(acc[tau][1]), fabsf(acc[tau][3]));
    }
#pragma unroll
    for (int c = 2 * NT; c > 2 * NT / 8; c >>= 1) {
      const int ob = c == 2 * NT ? 16 : (c == NT ? 8 : 4);
      const bool upper = (lane & ob) != 0;
#pragma unroll
      for (int kk = 0; kk < c / 2; ++kk) {
        const float send = upper ? vcol[kk] : vcol[kk + c / 2];
        const float keep = upper ? vcol[kk + c / 2] : vcol[kk];
        vcol[kk] = max_nan(keep, __shfl_xor_sync(FULL, send, ob));
      }
    }
#pragma unroll
    for (int kk = 0; kk < 2 * NT / 8; ++kk) {
      const int idx = (2 * NT / 8) * g + kk;
      const int tau = idx >> 1;
      sm.colmax[w][jof<D, BITS>(t, tau >> 1, 2 * (tau & 1) + (idx & 1))] = vcol[kk] * down;
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
      rsc[i0] = s0.bits;
      rsc[i1] = s1.bits;
      sm.qf[i0] = s0.sf > 0.f ? __frcp_rn(s0.sf) : 0.f;
      sm.qf[i1] = s1.sf > 0.f ? __frcp_rn(s1.sf) : 0.f;
      sm.sfv[i0] = s0.sf;
      sm.sfv[i1] = s1.sf;
      if (!fast_encode_ok(a0, s0, qmax) || !fast_encode_ok(a1, s1, qmax)) sm.slow = 1;
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
      sm.qf[j] = s.sf > 0.f ? __frcp_rn(s.sf) : 0.f;
      sm.sfv[j] = s.sf;
      if (!fast_encode_ok(a, s, qmax)) sm.slow = 1;
    }
    __syncthreads();
  }
  const bool slow = sm.slow != 0;
  if (col) {
    for (int e = lane; e < KS * 4; e += 32) {
      const int ks = e >> 2, tt = e & 3;
      float f[4];
#pragma unroll
      for (int pos = 0; pos < 4; ++pos) {
        const int j = jof<D, BITS>(tt, ks, pos);
        f[pos] = slow ? sm.sfv[j] : sm.qf[j] * down;
      }
      sm.wq[w][ks][tt] = make_float4(f[0], f[1], f[2], f[3]);
    }
    __syncwarp();
  }
  const float qr0 = col ? 0.f : (slow ? sm.sfv[i0] : sm.qf[i0] * down);
  const float qr1 = col ? 0.f : (slow ? sm.sfv[i1] : sm.qf[i1] * down);
  auto hq = [&](int tau, int rr) -> uint32_t {
    const float a = acc[tau][2 * rr], bq = acc[tau][2 * rr + 1];
    float qa = rr ? qr1 : qr0, qb = qa;
    if (col) {
      const float4 q4 = sm.wq[w][tau >> 1][t];
      qa = (tau & 1) ? q4.z : q4.x;
      qb = (tau & 1) ? q4.w : q4.y;
    }
    if (!slow) return magic_fast<BITS>(a, bq, qa, qb);
    return magic_exact<BITS>(a * down, bq * down, qa, qb);
  };
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    uint8_t* row = rec + (size_t)(rr ? i1 : i0) * ROWB;
    if (BITS == 4) {
      constexpr int NW = D / 32;
      uint32_t wd[NW];
#pragma unroll
      for (int mm = 0; mm < NW; ++mm) {
        const uint32_t E = prmt(hq(4 * mm, rr), hq(4 * mm + 2, rr), 0x6240u);
        const uint32_t O = prmt(hq(4 * mm + 1, rr), hq(4 * mm + 3, rr), 0x6240u);
        wd[mm] = (E | (O << 4)) ^ 0x88888888u;
      }
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
        for (int mm = 0; mm < WPC; ++mm) {
          const int ks = c * WPC + mm;
          wd[mm] = prmt(hq(2 * ks, rr), hq(2 * ks + 1, rr), 0x6420u) ^ 0x80808080u;
        }
        uint8_t* dst = row + chunk_offset<D, 8>(t, c);
        if (WPC == 4) *reinterpret_cast<uint4*>(dst) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        else if (WPC == 2) *reinterpret_cast<uint2*>(dst) = make_uint2(wd[0], wd[1]);
        else *reinterpret_cast<uint32_t*>(dst) = wd[0];
      }
    }
  }
  (void)ESZ;
}

template <int D, bool BF16>
__global__ void __launch_bounds__(PCfg<D, BF16>::THREADS, PCfg<D, BF16>::MINB)
    prefill_kernel(PoolDev p, Span sp, int64_t T, const void* __restrict__ q,
                   const void* __restrict__ k, const void* __restrict__ v,
                   const void* __restrict__ alpha, const void* __restrict__ beta,
                   float* __restrict__ o) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  PSmem<D, BF16>& sm = *reinterpret_cast<PSmem<D, BF16>*>(smem_raw);
  const int first = sp.b0 * p.H, end = (sp.b0 + sp.nb) * p.H;
  for (int head = first + blockIdx.x; head < end; head += gridDim.x) {
    if (p.fill[head] != 0) {   // tokens already buffered: the state is not at a period start
      if (threadIdx.x == 0) atomicOr(p.flags, PACE_FLAG_BUFFER_FULL);
      continue;
    }
    if (p.bits[head % p.H] == 4)
      prefill_head<D, BF16, 4>(p, head, T, q, k, v, alpha, beta, o, sm);
    else
      prefill_head<D, BF16, 8>(p, head, T, q, k, v, alpha, beta, o, sm);
    __syncthreads();
  }
}

template <int D, bool BF16>
cudaError_t launch_t(const PoolDev& p, const Span& sp, int64_t T, const void* q, const void* k,
                     const void* v, const void* alpha, const void* beta, float* o, cudaStream_t st) {
  const size_t smem = sizeof(PSmem<D, BF16>);
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D, BF16>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long heads = (long)sp.nb * p.H;
  if (heads == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long blocks = (long)(sp.blocks_per_sm > 0 ? sp.blocks_per_sm : 1) * sms * (D == 128 ? PCfg<D, BF16>::MINB : D == 64 ? 2 : 4);
  if (blocks > heads) blocks = heads;
  prefill_kernel<D, BF16><<<(unsigned)blocks, PCfg<D, BF16>::THREADS, smem, st>>>(p, sp, T, q, k, v,
                                                                                 alpha, beta, o);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PoolDev& p, const Span& sp, int64_t T, const void* q,
                           const void* k, const void* v, const void* alpha, const void* beta,
                           float* o, cudaStream_t st) {
  const bool bf = p.io == PACE_IO_BF16;
  switch (p.d_k) {
    case 32: return bf ? launch_t<32, true>(p, sp, T, q, k, v, alpha, beta, o, st)
                       : launch_t<32, false>(p, sp, T, q, k, v, alpha, beta, o, st);
    case 64: return bf ? launch_t<64, true>(p, sp, T, q, k, v, alpha, beta, o, st)
                       : launch_t<64, false>(p, sp, T, q, k, v, alpha, beta, o, st);
    case 128: return bf ? launch_t<128, true>(p, sp, T, q, k, v, alpha, beta, o, st)
                        : launch_t<128, false>(p, sp, T, q, k, v, alpha, beta, o, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace pace
