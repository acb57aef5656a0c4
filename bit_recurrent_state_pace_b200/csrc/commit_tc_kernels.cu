// Period commit on the fifth-generation tensor cores (tcgen05, TMEM), for
// d_k = d_v = 128 and column scales.
//
// "PACE: four-bit recurrent state by rounding less often", flowchart under
// "Fewer roundings, less compounded error": every k tokens the buffer feeds a
// "State update, chunked, high precision" followed by "4-bit encode,
// per-column scales" (8 bits for long-memory heads, TL;DR (3)).  Chunk (UT/WY)
// form of the n buffered tokens from the stored state S~0 = C diag(s):
//   X = S~0 K^T,  r_s = v_s - gamma_s x_s,  U^ = W R,
//   S_n = gamma_n S~0 + U^^T K,
// with W[s][s'] = gamma_{n/s} T[s][s'] beta_s', T = (I + A)^{-1}, left in the
// head's factor block by the decode step that filled the buffer.
//
// Design (one CTA per SM, warp-specialised, two heads in flight):
//  * producer warp: finds the heads due for a commit and stages each one's
//    record, buffered rows and factor block in shared memory by 1-D bulk
//    copies (no multicast), several heads ahead;
//  * converter warps (4): turn the codes into one exact f16 tile, [i][j] with
//    128-byte swizzling, that serves two MMAs: read K-major it is the A of
//    X = C (diag(s) K^T) and read MN-major it is the A of C^T = C^T I, a
//    transpose by block-identity products (N = 16 per block).  They also
//    build the scaled keys of both products, and, once X is in TMEM, compute
//    R and U^ for their TMEM lane (value channel i) and write U^ as the B of
//    the update;
//  * MMA warp: issues X and the transpose into TMEM (f32), then the update
//    U^T = K^T U^ (key channels on TMEM lanes, value channels on columns),
//    hi/lo f16 splits, fp32 accumulation;
//  * epilogue warps (8, two per TMEM lane quadrant): S^T = gamma_n s_j C^T +
//    U^T with one fma per element, per-column absmax thread-local plus two
//    shuffles, FP16 scales, round-half-even codes by the f16 magic number,
//    bytes transposed into a swizzled staging area by stmatrix, and the
//    record written back by one tensor store (codes) and one bulk store
//    (scales).
// Every wait is bounded; a wait that gives up sets PACE_FLAG_TIMEOUT and the
// CTA drains its tensor work, frees TMEM and returns.
#include "commit_tc.cuh"
#include "e4m3.cuh"
#include "tc.cuh"
#include "update_common.cuh"

namespace pace {

namespace {

constexpr unsigned FULL = 0xffffffffu;
constexpr int kSmemLimit = 232448;     // opt-in dynamic shared memory per block on sm_100

template <bool BF16, bool R8, int PMAX>
struct TcCfg {
  static constexpr int D = 128;
  static constexpr int ESZ = R8 ? 1 : (BF16 ? 2 : 4);     // bytes per buffered k or v element
  static constexpr int ROWB = 2 * D * ESZ;                // one buffered row: k then v
  static constexpr int REC = 16640;                       // largest record (INT8)
  static constexpr int KVB = PMAX * ROWB;
  static constexpr int GRB = (4 * (PMAX * (PMAX + 1) + 2) + 15) / 16 * 16;
  static constexpr int STAGE = (REC + KVB + GRB + 127) / 128 * 128;
  static constexpr int NSEG = (BF16 || R8) ? 2 : 3;       // key segments of the update's K
  static constexpr int NX = 2 * PMAX;                     // X columns: hi | lo per token
  static constexpr int KU = (NSEG * PMAX + 15) / 16 * 16; // update K, padded
  static constexpr int TILE = 32768;                      // 128 x 128 f16
  static constexpr int STG = 16384 + 1024;                // codes (swizzled) | scales at +16384
  static constexpr int BXB = NX * 256;
  static constexpr int AUB = KU * 256;
  static constexpr int FIXED = 2 * (TILE + STG + BXB + 2 * AUB) + 4096;
  static constexpr int NST_FIT = (kSmemLimit - 1024 - FIXED) / STAGE;
  static constexpr int NST = NST_FIT > 4 ? 4 : NST_FIT;  // staged heads
  static constexpr int THREADS = 14 * 32;                 // producer, MMA, 4 converter, 8 epilogue warps
  static constexpr int CONV0 = 2, EPI0 = 6;               // first converter / epilogue warp
};

template <bool BF16, bool R8, int PMAX>
struct alignas(1024) TcSmem {
  using C = TcCfg<BF16, R8, PMAX>;
  uint8_t tile[2][C::TILE];            // f16 codes [jh][i][64 positions], 128B swizzle
  uint8_t stg[2][C::STG];              // record staging: codes (64B/128B swizzle) + scales
  uint8_t bx[2][C::BXB];               // X operand B: [kh][NX rows][64], 128B swizzle
  uint8_t au[2][C::AUB];               // update A (keys, MN-major): [mh][KU rows][64], 128B swizzle
  uint8_t bu[2][C::AUB];               // update B (U^, K-major): [KU/16][16][2][8][8], no swizzle
  uint8_t stage[C::NST][C::STAGE];     // record | rows | factor block
  __half ident[256];                   // 16 x 16 identity, K-major, no swizzle
  float fj[2][128];                    // epilogue factors gamma_n s_j 2^e, by tile position
  float amax_x[2][128];                // per-column partial maxima of the two column halves
  float red[2][4];                     // converter maxima of |U^| (two heads alternate)
  int meta_head[2], meta_n[2], meta_e[2];
  int stage_head[C::NST], stage_n[C::NST];
  uint64_t stage_full[C::NST], stage_empty[C::NST];
  uint64_t tile_full[2], x_full[2], bupd_full[2], acc_full[2], tmem_empty[2], drain;
  uint32_t taddr;
  int abort;
};

// Tile position p (0..127) of key channel order: INT8 identity; INT4 puts the
// even channels of each 16-channel group first, then the odd ones.
template <int BITS>
__device__ __forceinline__ int chan_of(int p) {
  if (BITS == 8) return p;
  const int r = p & 15;
  return (p & ~15) + (r < 8 ? 2 * r : 2 * (r - 8) + 1);
}

// byte offset of element c (0..63) of row r inside a [rows][64] f16 block with 128-byte swizzling
__device__ __forceinline__ uint32_t sw128(int r, int chunk) { return (uint32_t)(r * 128 + ((chunk ^ (r & 7)) << 4)); }

__device__ __forceinline__ bool bounded_wait(uint64_t* bar, uint32_t parity, const PoolDev& p, int* abort) {
  if (mbar_wait_bounded(bar, parity, p.flags)) return true;
  *reinterpret_cast<volatile int*>(abort) = 1;
  return false;
}

__device__ __forceinline__ bool aborted(const int* abort) { return *reinterpret_cast<const volatile int*>(abort) != 0; }

__device__ __forceinline__ int clampi(int x, int lo, int hi) { return x < lo ? lo : (x > hi ? hi : x); }

// power-of-two exponent that brings m into [2^14, 2^15) (0 for zero or non-finite m)
__device__ __forceinline__ int norm_exp(float m, int lim) {
  if (!(m >= 1.17549435e-38f) || !(m < INFINITY)) return 0;
  return clampi(14 - exp2_floor(m), -lim, lim);
}

// First head index >= from (stepping by step, below end) due for a commit, or
// end.  The 32 lanes of the calling warp test 32 candidates at a time.
__device__ __forceinline__ int next_due(const PoolDev& p, int from, int step, int end, int lane) {
  for (int base = from; base < end; base += 32 * step) {
    const int hd = base + lane * step;
    const unsigned m = __ballot_sync(FULL, hd < end && commit_due(p.fill[hd], p.P));
    if (m) return base + (__ffs((int)m) - 1) * step;
  }
  return end;
}

// ---- producer: stage the heads due for a commit ------------------------------
template <bool BF16, bool R8, int PMAX>
__device__ void producer_role(const PoolDev& p, TcSmem<BF16, R8, PMAX>& sm, int first, int end, int lane) {
  using C = TcCfg<BF16, R8, PMAX>;
  const uint32_t row = (uint32_t)C::ROWB;
  int h = next_due(p, first, gridDim.x, end, lane);
  for (int k = 0;; ++k) {
    const int s = k % C::NST, r = k / C::NST;
    if (r > 0 && !bounded_wait(&sm.stage_empty[s], (uint32_t)((r - 1) & 1), p, &sm.abort)) return;
    const bool have = __shfl_sync(FULL, (h < end && !aborted(&sm.abort)) ? 1 : 0, 0) != 0;
    if (lane == 0) {
      sm.stage_head[s] = have ? h : -1;
      if (have) {
        const int hh = h % p.H, b = h / p.H;
        sm.stage_n[s] = p.fill[h] & 0xff;
        const uint32_t rec_bytes = (uint32_t)record_bytes(C::D, C::D, p.bits[hh], C::D);
        const uint32_t kv_bytes = (uint32_t)p.P * row;
        const uint8_t* rec = p.state + (size_t)b * p.slot_stride + p.rec_off[hh];
        uint8_t* dst = sm.stage[s];
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&sm.stage_full[s], rec_bytes + kv_bytes + p.gram_stride);
        tma_load_1d(dst, rec, rec_bytes, &sm.stage_full[s]);
        tma_load_1d(dst + C::REC, p.kv + (size_t)h * kv_bytes, kv_bytes, &sm.stage_full[s]);
        tma_load_1d(dst + C::REC + C::KVB, p.gram + (size_t)h * p.gram_stride, p.gram_stride, &sm.stage_full[s]);
      } else {
        tc::mbar_arrive(&sm.stage_full[s]);
      }
    }
    __syncwarp();
    if (!have) return;
    h = next_due(p, h + gridDim.x, gridDim.x, end, lane);
  }
}

// ---- MMA issuer (one thread) ------------------------------------------------
// TMEM columns of buffer t: [256 t, 256 t + 128) the transposed codes C^T,
// [256 t + 128, 256 t + 256) X (first NX columns) and then U^T.
template <bool BF16, bool R8, int PMAX>
__device__ void mma_role(const PoolDev& p, TcSmem<BF16, R8, PMAX>& sm, uint32_t tm) {
  using C = TcCfg<BF16, R8, PMAX>;
  constexpr uint32_t id_x = tc::idesc_f16(128, C::NX, 0, 0);
  constexpr uint32_t id_i = tc::idesc_f16(128, 16, 1, 0);
  constexpr uint32_t id_u = tc::idesc_f16(128, 128, 1, 0);
  const uint64_t d_ident = tc::smem_desc(smem_addr(sm.ident), 128, 256, tc::kSwizzleNone);
  for (int k = 0;; ++k) {
    const int t = k & 1;
    if (!bounded_wait(&sm.tile_full[t], (uint32_t)((k >> 1) & 1), p, &sm.abort)) break;
    if (sm.meta_head[t] < 0) {
      tc::mbar_arrive(&sm.acc_full[t]);
      break;
    }
    if (k >= 2 && !bounded_wait(&sm.tmem_empty[t], (uint32_t)(((k - 2) >> 1) & 1), p, &sm.abort)) break;
    tc::fence_after_sync();
    const uint32_t tile = smem_addr(sm.tile[t]), bx = smem_addr(sm.bx[t]);
    const uint32_t dC = tm + 256u * t, dU = dC + 128u;
    // X = C (diag(s) K^T): A = tile K-major (rows i), B = scaled keys K-major
#pragma unroll
    for (int kb = 0; kb < 8; ++kb) {
      const uint32_t ka = (kb >> 2) * 16384u + (kb & 3) * 32u;
      const uint32_t kx = (kb >> 2) * (uint32_t)(C::NX * 128) + (kb & 3) * 32u;
      tc::mma_f16(dU, tc::smem_desc(tile + ka, 16, 1024, tc::kSwizzle128),
                  tc::smem_desc(bx + kx, 16, 1024, tc::kSwizzle128), id_x, kb > 0);
    }
    // C^T by 16 x 16 blocks: A = tile MN-major (rows are the K index i), B = I
#pragma unroll
    for (int b = 0; b < 8; ++b)
      tc::mma_f16(dC + 16u * b, tc::smem_desc(tile + 2048u * b, 16384, 1024, tc::kSwizzle128), d_ident, id_i, false);
    tc::commit(&sm.x_full[t]);
    if (!bounded_wait(&sm.bupd_full[t], (uint32_t)((k >> 1) & 1), p, &sm.abort)) break;
    tc::fence_after_sync();
    // U^T = K^T U^: A = keys MN-major (key channels on lanes), B = U^ K-major
    const uint32_t au = smem_addr(sm.au[t]), bu = smem_addr(sm.bu[t]);
#pragma unroll
    for (int kb = 0; kb < C::KU / 16; ++kb)
      tc::mma_f16(dU, tc::smem_desc(au + 2048u * kb, C::KU * 128, 1024, tc::kSwizzle128),
                  tc::smem_desc(bu + 4096u * kb, 128, 256, tc::kSwizzleNone), id_u, kb > 0);
    tc::commit(&sm.acc_full[t]);
  }
  // every product issued has completed before TMEM is released
  tc::commit(&sm.drain);
  mbar_wait_bounded(&sm.drain, 0, p.flags);
}

// ---- converters --------------------------------------------------------------
// Codes of one staged record -> the f16 tile (exact values), [jh][i][64
// positions] with 128-byte swizzling.  Each lane converts 16 channels of one
// row per step; a quarter-warp covers two rows whose halves are swapped, so
// its loads and its 16-byte stores each fall in distinct banks.
template <int BITS>
__device__ __forceinline__ void convert_codes(const uint8_t* rec, uint8_t* tile, int cw, int lane) {
  const uint32_t K64 = 0x64646464u;
  const __half2 off8 = __float2half2_rn(1032.f), off16 = __float2half2_rn(72.f);
  const __half2 sixteenth = __float2half2_rn(0.0625f), off128 = __float2half2_rn(1152.f);
  const int qq = lane >> 3, r = (lane >> 2) & 1, mm = lane & 3;
#pragma unroll 2
  for (int it = 0; it < 8; ++it) {
    const int i = 32 * cw + 8 * (it >> 1) + 2 * qq + r;
    const int m16 = 4 * ((it & 1) ^ r) + mm;          // 16-channel group
    uint32_t hv[8];                                    // positions 16 m16 + 0..15 as f16 pairs
    if (BITS == 4) {
      const uint2 w = *reinterpret_cast<const uint2*>(rec + 64 * i + 8 * m16);
      // offset codes u = c + 8: even channels in the low nibbles, odd ones (x16) in the high
      const uint32_t x0 = (w.x & 0x0F0F0F0Fu) ^ 0x08080808u, y0 = (w.x & 0xF0F0F0F0u) ^ 0x80808080u;
      const uint32_t x1 = (w.y & 0x0F0F0F0Fu) ^ 0x08080808u, y1 = (w.y & 0xF0F0F0F0u) ^ 0x80808080u;
      hv[0] = h2u(__hsub2(u2h(prmt(x0, K64, 0x4140u)), off8));    // channels 0, 2
      hv[1] = h2u(__hsub2(u2h(prmt(x0, K64, 0x4342u)), off8));    // 4, 6
      hv[2] = h2u(__hsub2(u2h(prmt(x1, K64, 0x4140u)), off8));    // 8, 10
      hv[3] = h2u(__hsub2(u2h(prmt(x1, K64, 0x4342u)), off8));    // 12, 14
      hv[4] = h2u(__hfma2(u2h(prmt(y0, K64, 0x4140u)), sixteenth, __hneg2(off16)));   // 1, 3
      hv[5] = h2u(__hfma2(u2h(prmt(y0, K64, 0x4342u)), sixteenth, __hneg2(off16)));   // 5, 7
      hv[6] = h2u(__hfma2(u2h(prmt(y1, K64, 0x4140u)), sixteenth, __hneg2(off16)));   // 9, 11
      hv[7] = h2u(__hfma2(u2h(prmt(y1, K64, 0x4342u)), sixteenth, __hneg2(off16)));   // 13, 15
    } else {
      const uint4 w = *reinterpret_cast<const uint4*>(rec + 128 * i + 16 * m16);
      const uint32_t ws[4] = {w.x ^ 0x80808080u, w.y ^ 0x80808080u, w.z ^ 0x80808080u, w.w ^ 0x80808080u};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        hv[2 * e] = h2u(__hsub2(u2h(prmt(ws[e], K64, 0x4140u)), off128));
        hv[2 * e + 1] = h2u(__hsub2(u2h(prmt(ws[e], K64, 0x4342u)), off128));
      }
    }
    uint8_t* base = tile + (m16 >> 2) * 16384;
    const int ch = 2 * (m16 & 3);
    *reinterpret_cast<uint4*>(base + sw128(i, ch)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
    *reinterpret_cast<uint4*>(base + sw128(i, ch + 1)) = make_uint4(hv[4], hv[5], hv[6], hv[7]);
  }
}

// Per-head exponents of the key operands: exx for s_j k_s[j] (the X product),
// exk for k_s[j] (the update), from the largest |k| and the largest stored
// scale that the decode left in the factor block.
struct KeyExp { int exx, exk; };
__device__ __forceinline__ KeyExp key_exponents(const float* G, int P) {
  const float kmax = G[P * P + P], smax = G[P * P + P + 1];
  return KeyExp{norm_exp(kmax * smax, 120), norm_exp(kmax, 40)};
}

// The scaled keys of one head: B of X (rows s: hi, PMAX + s: lo of
// s_j k_s[j] 2^exx) and A of the update (rows s and PMAX + s: k_s[j] 2^exk
// in f16, and rows 2 PMAX + s: its low part for fp32 rows), by tile
// position.  Tokens s >= n give zero rows.
template <bool BF16, bool R8, int PMAX, int BITS>
__device__ __forceinline__ void build_keys(const uint8_t* stage, uint8_t* bx, uint8_t* au, int n, KeyExp ex, int ct) {
  using C = TcCfg<BF16, R8, PMAX>;
  const uint16_t* sc = reinterpret_cast<const uint16_t*>(stage + code_bytes(C::D, C::D, BITS));
  const uint8_t* rows = stage + C::REC;
  const float upx = pow2i(ex.exx), upk = pow2i(ex.exk);
  for (int u = ct; u < PMAX * 16; u += 128) {
    const int s = u >> 4, c16 = u & 15;                // token, 8-position chunk
    uint32_t bh[4], bl[4], kh[4], kl[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float b2[2], k2[2];
#pragma unroll
      for (int z = 0; z < 2; ++z) {
        const int j = chan_of<BITS>(8 * c16 + 2 * e + z);
        const float kv = s < n ? row_at<R8>(rows + s * C::ROWB, j, BF16) : 0.f;
        b2[z] = s < n ? kv * __half2float(__ushort_as_half(sc[j])) * upx : 0.f;
        k2[z] = kv * upk;
      }
      const __half2 bhi = __floats2half2_rn(b2[0], b2[1]);
      const float2 bhf = __half22float2(bhi);
      bh[e] = h2u(bhi);
      bl[e] = h2u(__floats2half2_rn(b2[0] - bhf.x, b2[1] - bhf.y));
      const __half2 khi = __floats2half2_rn(k2[0], k2[1]);
      const float2 khf = __half22float2(khi);
      kh[e] = h2u(khi);
      kl[e] = h2u(__floats2half2_rn(k2[0] - khf.x, k2[1] - khf.y));
    }
    uint8_t* xb = bx + (c16 >> 3) * (C::NX * 128);
    const int ch = c16 & 7;
    *reinterpret_cast<uint4*>(xb + sw128(s, ch)) = make_uint4(bh[0], bh[1], bh[2], bh[3]);
    *reinterpret_cast<uint4*>(xb + sw128(PMAX + s, ch)) = make_uint4(bl[0], bl[1], bl[2], bl[3]);
    uint8_t* ab = au + (c16 >> 3) * (C::KU * 128);
    *reinterpret_cast<uint4*>(ab + sw128(s, ch)) = make_uint4(kh[0], kh[1], kh[2], kh[3]);
    *reinterpret_cast<uint4*>(ab + sw128(PMAX + s, ch)) = make_uint4(kh[0], kh[1], kh[2], kh[3]);
    if (C::NSEG == 3)
      *reinterpret_cast<uint4*>(ab + sw128(2 * PMAX + s, ch)) = make_uint4(kl[0], kl[1], kl[2], kl[3]);
  }
}

// R and U^ for one head, one TMEM lane (value channel i) per converter thread:
// x_s from TMEM, r_s = v_s[i] - gamma_s x_s, U^[s][i] = sum_s' W[s][s'] r_s',
// normalised by one power of two for the head, split hi + lo into row i of
// the update's B.  Also the epilogue's per-position factors.
template <bool BF16, bool R8, int PMAX, int BITS>
__device__ __forceinline__ void residual_update(const PoolDev& p, TcSmem<BF16, R8, PMAX>& sm, const uint8_t* stage,
                                                int t, int n, uint32_t tm, int k, int ct, int warp, int lane) {
  using C = TcCfg<BF16, R8, PMAX>;
  const int P = p.P;
  const int qd = warp & 3, i = 32 * qd + lane;
  uint32_t xr[2 * PMAX];
  {
    uint32_t tmp[16];
    tc::ld_32x32b_x16(tm + ((uint32_t)(32 * qd) << 16) + 256u * t + 128u, tmp);
#pragma unroll
    for (int c = 0; c < 16; ++c) xr[c] = tmp[c];
    if (PMAX == 16) {
      tc::ld_32x32b_x16(tm + ((uint32_t)(32 * qd) << 16) + 256u * t + 144u, tmp);
#pragma unroll
      for (int c = 0; c < 16; ++c) xr[(16 + c) % (2 * PMAX)] = tmp[c];
    }
    tc::wait_ld();
  }
  const float* G = reinterpret_cast<const float*>(stage + C::REC + C::KVB);
  const float* W = G;
  const float* gam = G + P * P;
  const KeyExp ex = key_exponents(G, P);
  const float xinv = pow2i(-ex.exx);
  const uint8_t* rows = stage + C::REC;
  float r[PMAX];
#pragma unroll
  for (int s = 0; s < PMAX; ++s) {
    const float x = (__uint_as_float(xr[s]) + __uint_as_float(xr[PMAX + s])) * xinv;
    r[s] = s < n ? row_at<R8>(rows + s * C::ROWB, C::D + i, BF16) - gam[s] * x : 0.f;
  }
  float u[PMAX];
  float um = 0.f;
#pragma unroll
  for (int s = 0; s < PMAX; ++s) {
    float a = 0.f;
    if (s < n) {
      if ((P & 3) == 0) {
#pragma unroll
        for (int c = 0; c < PMAX / 4; ++c) {
          if (4 * c < P) {
            const float4 w4 = *reinterpret_cast<const float4*>(W + s * P + 4 * c);
            a = fmaf(w4.x, r[4 * c], a);
            a = fmaf(w4.y, r[4 * c + 1], a);
            a = fmaf(w4.z, r[4 * c + 2], a);
            a = fmaf(w4.w, r[4 * c + 3], a);
          }
        }
      } else {
#pragma unroll
        for (int sp = 0; sp < PMAX; ++sp)
          if (sp < n) a = fmaf(W[s * P + sp], r[sp], a);
      }
    }
    u[s] = a;
    um = max_nan(um, fabsf(a));
  }
  // one exponent for the head's U^ (all 128 lanes feed one product)
#pragma unroll
  for (int off = 16; off; off >>= 1) um = max_nan(um, __shfl_xor_sync(FULL, um, off));
  if (lane == 0) sm.red[k & 1][warp - C::CONV0] = um;
  tc::named_sync(6, 128);
  um = max_nan(max_nan(sm.red[k & 1][0], sm.red[k & 1][1]), max_nan(sm.red[k & 1][2], sm.red[k & 1][3]));
  int e_tot = ex.exk + norm_exp(um, 40);
  const float smax = G[P * P + P + 1];
  if (smax >= 1.17549435e-38f && smax < INFINITY) e_tot = min(e_tot, 111 - exp2_floor(smax));
  const float up = pow2i(e_tot - ex.exk);
  // row i of B (K-major, no swizzle): K entries [U^_hi (PMAX) | U^_lo (PMAX) | U^_hi (PMAX, fp32 rows)]
  uint32_t hi[PMAX / 2], lo[PMAX / 2];
#pragma unroll
  for (int e = 0; e < PMAX / 2; ++e) {
    const float a = u[2 * e] * up, b = u[2 * e + 1] * up;
    const __half2 h = __floats2half2_rn(a, b);
    const float2 hf = __half22float2(h);
    hi[e] = h2u(h);
    lo[e] = h2u(__floats2half2_rn(a - hf.x, b - hf.y));
  }
  uint8_t* row = sm.bu[t] + (i >> 3) * 256 + (i & 7) * 16;
  auto put = [&](int kk0, const uint32_t* src) {   // 8 K entries starting at kk0 (a multiple of 8)
    *reinterpret_cast<uint4*>(row + (kk0 >> 4) * 4096 + ((kk0 >> 3) & 1) * 128) =
        make_uint4(src[0], src[1], src[2], src[3]);
  };
#pragma unroll
  for (int c = 0; c < PMAX / 8; ++c) {
    put(8 * c, hi + 4 * c);
    put(PMAX + 8 * c, lo + 4 * c);
    if (C::NSEG == 3) put(2 * PMAX + 8 * c, hi + 4 * c);
  }
  // epilogue factors, one tile position per thread
  const uint16_t* sc = reinterpret_cast<const uint16_t*>(stage + code_bytes(C::D, C::D, BITS));
  sm.fj[t][ct] = gam[n - 1] * __half2float(__ushort_as_half(sc[chan_of<BITS>(ct)])) * pow2i(e_tot);
  if (ct == 0) sm.meta_e[t] = e_tot;
}

template <bool BF16, bool R8, int PMAX>
__device__ void converter_role(const PoolDev& p, TcSmem<BF16, R8, PMAX>& sm, uint32_t tm, int warp, int lane) {
  using C = TcCfg<BF16, R8, PMAX>;
  const int cw = warp - C::CONV0, ct = 32 * cw + lane;
  // Every wait is followed by a vote at the converters' named barrier, so that
  // the four warps leave together and none is left waiting in a barrier.
  for (int k = 0;; ++k) {
    const int s = k % C::NST, t = k & 1;
    bool ok = bounded_wait(&sm.stage_full[s], (uint32_t)((k / C::NST) & 1), p, &sm.abort);
    const int head = ok ? sm.stage_head[s] : -1;
    // buffer t is free once the epilogue of the head two back has read its
    // metadata and factors and released its TMEM (its update, which read this
    // buffer's keys, is then done as well)
    if (ok && k >= 2) ok = bounded_wait(&sm.tmem_empty[t], (uint32_t)(((k - 2) >> 1) & 1), p, &sm.abort);
    if (tc::named_sync_any(6, 128, !ok)) return;
    if (head >= 0) {
      const uint8_t* st = sm.stage[s];
      const int n = sm.stage_n[s];
      const KeyExp ex = key_exponents(reinterpret_cast<const float*>(st + C::REC + C::KVB), p.P);
      if (p.bits[head % p.H] == 4) {
        convert_codes<4>(st, sm.tile[t], cw, lane);
        build_keys<BF16, R8, PMAX, 4>(st, sm.bx[t], sm.au[t], n, ex, ct);
      } else {
        convert_codes<8>(st, sm.tile[t], cw, lane);
        build_keys<BF16, R8, PMAX, 8>(st, sm.bx[t], sm.au[t], n, ex, ct);
      }
      if (ct == 0) {
        sm.meta_head[t] = head;
        sm.meta_n[t] = n;
      }
    } else if (ct == 0) {
      sm.meta_head[t] = -1;
    }
    fence_proxy_async_smem();
    tc::mbar_arrive(&sm.tile_full[t]);
    if (k >= 1) {   // R and U^ of the previous head, whose X has had this head's conversion to land
      const int sp = (k - 1) % C::NST, tp = t ^ 1;
      ok = bounded_wait(&sm.x_full[tp], (uint32_t)(((k - 1) >> 1) & 1), p, &sm.abort);
      if (tc::named_sync_any(6, 128, !ok)) return;
      tc::fence_after_sync();
      const int hp = sm.stage_head[sp];
      if (p.bits[hp % p.H] == 4)
        residual_update<BF16, R8, PMAX, 4>(p, sm, sm.stage[sp], tp, sm.stage_n[sp], tm, k - 1, ct, warp, lane);
      else
        residual_update<BF16, R8, PMAX, 8>(p, sm, sm.stage[sp], tp, sm.stage_n[sp], tm, k - 1, ct, warp, lane);
      fence_proxy_async_smem();
      tc::fence_before_sync();
      tc::mbar_arrive(&sm.bupd_full[tp]);
      tc::mbar_arrive(&sm.stage_empty[sp]);
    }
    if (head < 0) return;
  }
}

// ---- epilogue ----------------------------------------------------------------
// Thread (g = lane / 4, q = lane % 4) of warp we holds, for 16-lane blocks blk
// of its quadrant qd, tile positions p = 32 qd + 16 blk + g + 8 h (h = 0, 1)
// and value channels i = 64 hf + 8 c + 2 q + {0, 1} (c = 0..7): 64 elements
// of S'^T = S^T 2^e.  INT4 tile positions pair the key channels 2m (h = 0)
// and 2m + 1 (h = 1) in one thread, so a code byte is thread-local.
template <bool BF16, bool R8, int PMAX, int BITS>
__device__ __forceinline__ void epilogue_head(const PoolDev& p, const CommitMaps& maps, TcSmem<BF16, R8, PMAX>& sm,
                                              uint32_t tm, int t, int head, int we, int lane) {
  using C = TcCfg<BF16, R8, PMAX>;
  const int qd = we & 3, hf = (we - C::EPI0) >> 2, g = lane >> 2, q = lane & 3;
  const int e_tot = sm.meta_e[t];
  const float down = pow2i(-e_tot);
  float S[2][32];
  {
    float f[2][2];
#pragma unroll
    for (int blk = 0; blk < 2; ++blk)
#pragma unroll
      for (int h = 0; h < 2; ++h) f[blk][h] = sm.fj[t][32 * qd + 16 * blk + g + 8 * h];
#pragma unroll
    for (int blk = 0; blk < 2; ++blk) {
      uint32_t cr[32], ur[32];
      const uint32_t lb = (uint32_t)(32 * qd + 16 * blk) << 16;
      tc::ld_16x256b_x8(tm + lb + 256u * t + 64u * hf, cr);
      tc::ld_16x256b_x8(tm + lb + 256u * t + 128u + 64u * hf, ur);
      tc::wait_ld();
#pragma unroll
      for (int c = 0; c < 8; ++c)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          S[blk][4 * c + k] = fmaf(__uint_as_float(cr[4 * c + k]), f[blk][k >> 1], __uint_as_float(ur[4 * c + k]));
    }
  }
  tc::fence_before_sync();
  tc::mbar_arrive(&sm.tmem_empty[t]);

  // column maxima: 16 values per (blk, h) here, the other three lanes of the
  // quad, then the warp holding the other 64 value channels
  float m[2][2];
#pragma unroll
  for (int blk = 0; blk < 2; ++blk)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float a = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) a = max_nan(a, max_nan(fabsf(S[blk][4 * c + 2 * h]), fabsf(S[blk][4 * c + 2 * h + 1])));
      a = max_nan(a, __shfl_xor_sync(FULL, a, 1));
      a = max_nan(a, __shfl_xor_sync(FULL, a, 2));
      m[blk][h] = a;
    }
  if (q == 0)
#pragma unroll
    for (int blk = 0; blk < 2; ++blk)
#pragma unroll
      for (int h = 0; h < 2; ++h) sm.amax_x[hf][32 * qd + 16 * blk + g + 8 * h] = m[blk][h];
  tc::named_sync(1 + qd, 64);
#pragma unroll
  for (int blk = 0; blk < 2; ++blk)
#pragma unroll
    for (int h = 0; h < 2; ++h) m[blk][h] = max_nan(m[blk][h], sm.amax_x[hf ^ 1][32 * qd + 16 * blk + g + 8 * h]);

  // scale of the column (blk, h) = (q >> 1, q & 1), then shared across the quad
  const int qmax = BITS == 4 ? 7 : 127;
  uint8_t* stg = sm.stg[t];
  float qf, sf;
  bool bad;
  {
    const int pos = 32 * qd + 16 * (q >> 1) + g + 8 * (q & 1);
    const float amax = m[q >> 1][q & 1] * down;
    const GroupScale gs = group_scale(amax, isfinite(amax), qmax, hf == 0 ? p.flags : nullptr);
    sf = gs.sf;
    qf = gs.sf > 0.f ? __frcp_rn(gs.sf) * down : 0.f;
    bad = !isfinite(amax) || (gs.bits == 0x7BFF && amax / qmax > 65504.f) || !(qf < INFINITY);
    if (hf == 0) reinterpret_cast<uint16_t*>(stg + 16384)[chan_of<BITS>(pos)] = gs.bits;
  }
  float qv[2][2], sv[2][2];
#pragma unroll
  for (int z = 0; z < 4; ++z) {
    qv[z >> 1][z & 1] = __shfl_sync(FULL, qf, (lane & ~3) | z);
    sv[z >> 1][z & 1] = __shfl_sync(FULL, sf, (lane & ~3) | z);
  }
  const bool slow = __any_sync(FULL, bad);

  // codes: f16 magic pairs (rows 2q, 2q + 1 of one column), bytes gathered and
  // stored transposed into the swizzled staging rows
  auto pair = [&](int blk, int c, int h) -> uint32_t {
    const float a = S[blk][4 * c + 2 * h], b = S[blk][4 * c + 2 * h + 1];
    if (!slow) return magic_fast<BITS>(a, b, qv[blk][h], qv[blk][h]);
    return magic_exact<BITS>(a * down, b * down, sv[blk][h], sv[blk][h]);
  };
  const uint32_t stg_a = smem_addr(stg);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const int i = 64 * hf + 8 * c + (lane & 7);     // the staging row whose address this lane gives
    if (BITS == 4) {
      uint32_t rb[2];
#pragma unroll
      for (int blk = 0; blk < 2; ++blk) {
        const uint32_t ev = pair(blk, c, 0), od = pair(blk, c, 1);
        rb[blk] = ev | ((od << 4) & 0x00F000F0u);
      }
      const uint32_t v = prmt(rb[0], rb[1], 0x6420u) ^ 0x88888888u;
      tc::stsm_trans_b8(stg_a + 64 * i + ((qd ^ ((i >> 1) & 3)) << 4), v);
    } else {
#pragma unroll
      for (int blk = 0; blk < 2; ++blk) {
        const uint32_t v = prmt(pair(blk, c, 0), pair(blk, c, 1), 0x6420u) ^ 0x80808080u;
        tc::stsm_trans_b8(stg_a + 128 * i + (((2 * qd + blk) ^ (i & 7)) << 4), v);
      }
    }
  }
  fence_proxy_async_smem();
  tc::named_sync(5, 256);
  if (we == C::EPI0 && lane == 0) {
    const int hh = head % p.H, b = head / p.H;
    const size_t off = (size_t)b * p.slot_stride + p.rec_off[hh];
    if (BITS == 4) tc::tensor_store_2d(&maps.codes4, stg_a, 0, (int)(off / 64));
    else tc::tensor_store_2d(&maps.codes8, stg_a, 0, (int)(off / 128));
    tc::bulk_store(p.state + off + code_bytes(C::D, C::D, BITS), stg_a + 16384, 256);
    tc::bulk_commit_group();
    tc::bulk_wait_read_all();
    p.fill[head] = 0;
  }
}

template <bool BF16, bool R8, int PMAX>
__device__ void epilogue_role(const PoolDev& p, const CommitMaps& maps, TcSmem<BF16, R8, PMAX>& sm, uint32_t tm,
                              int warp, int lane) {
  for (int k = 0;; ++k) {
    const int t = k & 1;
    // the eight warps vote after the wait and leave together (named barriers follow)
    const bool ok = bounded_wait(&sm.acc_full[t], (uint32_t)((k >> 1) & 1), p, &sm.abort);
    if (tc::named_sync_any(5, 256, !ok)) break;
    tc::fence_after_sync();
    const int head = sm.meta_head[t];
    if (head < 0) break;
    if (p.bits[head % p.H] == 4) epilogue_head<BF16, R8, PMAX, 4>(p, maps, sm, tm, t, head, warp, lane);
    else epilogue_head<BF16, R8, PMAX, 8>(p, maps, sm, tm, t, head, warp, lane);
  }
  if (warp == TcCfg<BF16, R8, PMAX>::EPI0 && lane == 0) tc::bulk_wait_all();
}

// ---- kernel ------------------------------------------------------------------
template <bool BF16, bool R8, int PMAX>
__global__ void __launch_bounds__(TcCfg<BF16, R8, PMAX>::THREADS, 1)
    commit_tc_kernel(const __grid_constant__ PoolDev p, const __grid_constant__ CommitMaps maps, Span sp) {
  using C = TcCfg<BF16, R8, PMAX>;
  using SM = TcSmem<BF16, R8, PMAX>;
  extern __shared__ uint8_t smem_raw[];
  SM& sm = *reinterpret_cast<SM*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int first = sp.b0 * p.H + (int)blockIdx.x, end = (sp.b0 + sp.nb) * p.H;
  if (tid == 0) {
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(&sm.stage_full[s], 1);
      mbar_init(&sm.stage_empty[s], 128);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&sm.tile_full[t], 128);
      mbar_init(&sm.x_full[t], 1);
      mbar_init(&sm.bupd_full[t], 128);
      mbar_init(&sm.acc_full[t], 1);
      mbar_init(&sm.tmem_empty[t], 256);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  // the identity blocks and the update operands' padding are never rewritten
  for (int e = tid; e < 256; e += C::THREADS) {
    const int n = e >> 4, kk = e & 15;
    sm.ident[(n >> 3) * 128 + (kk >> 3) * 64 + (n & 7) * 8 + (kk & 7)] = __float2half(n == kk ? 1.f : 0.f);
  }
  for (int e = tid; e < 2 * C::AUB / 16; e += C::THREADS) {
    reinterpret_cast<uint4*>(&sm.au[0][0])[e] = make_uint4(0u, 0u, 0u, 0u);
    reinterpret_cast<uint4*>(&sm.bu[0][0])[e] = make_uint4(0u, 0u, 0u, 0u);
  }
  if (warp == 1) tc::tmem_alloc(&sm.taddr, 512);
  fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tm = sm.taddr;
  if (warp == 0) {
    producer_role<BF16, R8, PMAX>(p, sm, first, end, lane);
  } else if (warp == 1) {
    if (lane == 0) mma_role<BF16, R8, PMAX>(p, sm, tm);
    __syncwarp();
  } else if (warp < C::EPI0) {
    converter_role<BF16, R8, PMAX>(p, sm, tm, warp, lane);
  } else {
    epilogue_role<BF16, R8, PMAX>(p, maps, sm, tm, warp, lane);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 1) tc::tmem_free(tm, 512);
}

int sm_count_tc() {
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

template <bool BF16, bool R8, int PMAX>
cudaError_t launch_tc_t(const PoolDev& p, const Span& sp, const CommitMaps& maps, cudaStream_t st) {
  using C = TcCfg<BF16, R8, PMAX>;
  using SM = TcSmem<BF16, R8, PMAX>;
  static_assert(C::NST >= 2, "two staged heads at least");
  static_assert(sizeof(SM) + 1024 <= (size_t)kSmemLimit, "shared memory");
  const size_t smem = sizeof(SM) + 1024;
  cudaError_t e = cudaFuncSetAttribute(commit_tc_kernel<BF16, R8, PMAX>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long heads = (long)sp.nb * p.H;
  if (heads == 0) return cudaSuccess;
  long blocks = sm_count_tc();
  if (blocks > heads) blocks = heads;
  commit_tc_kernel<BF16, R8, PMAX><<<(unsigned)blocks, C::THREADS, smem, st>>>(p, maps, sp);
  return cudaGetLastError();
}

}  // namespace

bool commit_tc_supported(const PoolDev& p) {
  if (p.d_k != 128 || p.d_v != 128 || p.axis != PACE_SCALE_COL) return false;
  return p.row8 || p.io == PACE_IO_BF16 || p.P <= 8;
}

cudaError_t launch_commit_tc(const PoolDev& p, const Span& sp, const CommitMaps& maps, cudaStream_t st) {
  if (!commit_tc_supported(p)) return cudaErrorNotSupported;
  const bool bf = p.io == PACE_IO_BF16;
  if (p.row8) {
    if (bf) return p.P <= 8 ? launch_tc_t<true, true, 8>(p, sp, maps, st) : launch_tc_t<true, true, 16>(p, sp, maps, st);
    return p.P <= 8 ? launch_tc_t<false, true, 8>(p, sp, maps, st) : launch_tc_t<false, true, 16>(p, sp, maps, st);
  }
  if (bf) return p.P <= 8 ? launch_tc_t<true, false, 8>(p, sp, maps, st) : launch_tc_t<true, false, 16>(p, sp, maps, st);
  return launch_tc_t<false, false, 8>(p, sp, maps, st);
}

bool make_commit_maps(uint8_t* state, size_t state_bytes, CommitMaps* maps) {
  using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
  static EncodeFn encode = nullptr;
  if (!encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn) {
      (void)cudaGetLastError();
      return false;
    }
    encode = reinterpret_cast<EncodeFn>(fn);
  }
  if (state_bytes % 128 != 0 || state_bytes / 64 > 0xffffffffull) return false;
  struct View { cuuint64_t row; CUtensorMapSwizzle swz; CUtensorMap* map; };
  const View views[2] = {{64, CU_TENSOR_MAP_SWIZZLE_64B, &maps->codes4}, {128, CU_TENSOR_MAP_SWIZZLE_128B, &maps->codes8}};
  for (const View& v : views) {
    const cuuint64_t dims[2] = {v.row, (cuuint64_t)(state_bytes / v.row)};
    const cuuint64_t strides[1] = {v.row};
    const cuuint32_t box[2] = {(cuuint32_t)v.row, 128};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(v.map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, state, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               v.swz, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  return true;
}

}  // namespace pace
