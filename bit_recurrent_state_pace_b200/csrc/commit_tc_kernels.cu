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
// Design (one CTA of 18 warps per SM, warp-specialised, two heads in flight;
// each CTA takes its 4-bit heads before its 8-bit heads):
//  * producer warp: finds the heads due for a commit (one ballot over 32 fill
//    counters per global round trip) and stages each one's record, buffered
//    rows and factor block in shared memory by 1-D bulk copies (no
//    multicast), several heads ahead;
//  * converter warps (8, two per TMEM lane quadrant): turn the codes into one
//    exact f16 tile, [i][j] with 128-byte swizzling, that serves two MMAs:
//    read K-major it is the A of X = C (diag(s) K^T) and read MN-major it is
//    the A of C^T = C^T I, a transpose by block-identity products (N = 16 per
//    block).  They also build the scaled keys of both products, and, once X
//    is in TMEM, compute R and U^ for their TMEM lane (value channel i), the
//    two warps of a quadrant each for half of the tokens, and write U^ as the
//    B of the update;
//  * MMA warp: issues X and the transpose into TMEM (f32), then the update
//    U^T = K^T U^ (key channels on TMEM lanes, value channels on columns),
//    hi/lo f16 splits, fp32 accumulation;
//  * epilogue warps (8, two per TMEM lane quadrant, one per half of the value
//    channels): S^T = gamma_n s_j C^T + U^T with one fma per element,
//    per-column absmax thread-local plus two shuffles and one exchange
//    between the quadrant's two warps, FP16 scales, round-half-even codes by
//    the f16 magic number, bytes transposed into a swizzled staging area by
//    stmatrix, and the record written back by one tensor store (codes) and
//    one bulk store (scales).
// Every wait is bounded; a wait that gives up sets PACE_FLAG_TIMEOUT and the
// CTA drains its tensor work, frees TMEM and returns.
#include <type_traits>

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
  static constexpr int NCONV = 8, NEPI = 8;               // converter / epilogue warps (two per TMEM quadrant)
  static constexpr int THREADS = (2 + NCONV + NEPI) * 32; // producer, MMA, converters, epilogue
  static constexpr int CONV0 = 2, EPI0 = 2 + NCONV;       // first converter / epilogue warp
  static constexpr int NCT = 32 * NCONV, NET = 32 * NEPI; // converter / epilogue threads
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
  // per-head values handed from the converters to the MMA warp and the
  // epilogue, in a ring of four (the head k + 4 reuses the slot of head k)
  float fj[4][128];                    // epilogue factors gamma_n s_j 2^e, by tile position
  int meta_head[4], meta_e[4], meta_bits[4];
  float red[2][8];                     // converter maxima of |U^| (two heads alternate)
  float emax[2][128];                  // epilogue column maxima of the two value-channel halves
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
  if (tc::mbar_wait_sleep(bar, parity, p.flags)) return true;
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

// max of three that returns NaN if any input is NaN
__device__ __forceinline__ float max3_nan(float a, float b, float c) {
  float r;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// The producer's walk over its work items (work index i is head
// head_in_order(i): the 4-bit heads of the span first, so that a CTA runs one
// code path at a time).  The warp reads the fill counters of 32 items at a
// time and keeps the mask of the due ones, so each head costs one global
// round trip per 32 items, and the fill of the chosen one comes with it.
struct DueScan {
  int base;        // work index of lane 0's item in the current window
  unsigned mask;   // due items of the window not taken yet
  int fill;        // this lane's fill counter in the window
};
__device__ __forceinline__ void due_window(const PoolDev& p, DueScan& d, int step, int end, int b0, int nb, int lane) {
  const int it = d.base + lane * step;
  d.fill = it < end ? p.fill[head_in_order(p, it, b0, nb)] : 0;
  d.mask = __ballot_sync(FULL, it < end && commit_due(d.fill, p.P));
}
// Next due work index (and its fill), or end.
__device__ __forceinline__ int next_due(const PoolDev& p, DueScan& d, int step, int end, int b0, int nb, int lane,
                                        int* fill) {
  while (d.mask == 0) {
    d.base += 32 * step;
    if (d.base >= end) return end;
    due_window(p, d, step, end, b0, nb, lane);
  }
  const int l = __ffs((int)d.mask) - 1;
  d.mask &= d.mask - 1;
  *fill = __shfl_sync(FULL, d.fill, l);
  return d.base + l * step;
}

// ---- producer: stage the heads due for a commit ------------------------------
template <bool BF16, bool R8, int PMAX>
__device__ void producer_role(const PoolDev& p, TcSmem<BF16, R8, PMAX>& sm, const Span& sp, int lane) {
  using C = TcCfg<BF16, R8, PMAX>;
  const uint32_t row = (uint32_t)C::ROWB;
  const int end = sp.nb * p.H;
  DueScan due;
  due.base = (int)blockIdx.x;
  due_window(p, due, gridDim.x, end, sp.b0, sp.nb, lane);
  int fill = 0;
  int it = due.base < end ? next_due(p, due, gridDim.x, end, sp.b0, sp.nb, lane, &fill) : end;
  for (int k = 0;; ++k) {
    const int s = k % C::NST, r = k / C::NST;
    if (r > 0 && !bounded_wait(&sm.stage_empty[s], (uint32_t)((r - 1) & 1), p, &sm.abort)) return;
    const bool have = __shfl_sync(FULL, (it < end && !aborted(&sm.abort)) ? 1 : 0, 0) != 0;
    const int h = have ? head_in_order(p, it, sp.b0, sp.nb) : -1;
    if (lane == 0) {
      sm.stage_head[s] = have ? h : -1;
      if (have) {
        const int hh = h % p.H, b = h / p.H;
        sm.stage_n[s] = fill & 0xff;
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
    it = next_due(p, due, gridDim.x, end, sp.b0, sp.nb, lane, &fill);
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
    // the epilogue has taken the head two back out of buffer t; this also
    // keeps the end-of-work arrival below from running two phases ahead of it
    if (k >= 2 && !bounded_wait(&sm.tmem_empty[t], (uint32_t)(((k - 2) >> 1) & 1), p, &sm.abort)) break;
    if (sm.meta_head[k & 3] < 0) {
      tc::mbar_arrive(&sm.acc_full[t]);
      break;
    }
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
  tc::mbar_wait_sleep(&sm.drain, 0, p.flags);
}

// ---- converters --------------------------------------------------------------
// Codes of one staged record -> the f16 tile (exact values), [jh][i][64
// positions] with 128-byte swizzling.  Each lane converts 16 channels of one
// row per step; a quarter-warp covers two rows whose halves are swapped, so
// its loads and its 16-byte stores each fall in distinct banks.  A warp
// converts RPW rows in RPW / 4 steps, which differ by constant offsets (the
// swizzle term depends only on the row modulo 8, which is fixed per lane).
template <int BITS, int RPW>
__device__ __forceinline__ void convert_codes(const uint8_t* rec, uint8_t* tile, int cw, int lane) {
  const uint32_t K64 = 0x64646464u;
  const __half2 off8 = __float2half2_rn(1032.f), off16 = __float2half2_rn(-72.f);
  const __half2 sixteenth = __float2half2_rn(0.0625f), off128 = __float2half2_rn(1152.f);
  const int qq = lane >> 3, r = (lane >> 2) & 1, mm = lane & 3;
  const int i0 = RPW * cw + 2 * qq + r;              // row of step 0; step it adds 8 (it >> 1)
  const int r7 = i0 & 7;
  // group of the even steps (m16 = 4 r + mm) and of the odd ones (m16 = 4 (1 - r) + mm)
  const int mA = 4 * r + mm, mB = 4 * (1 - r) + mm;
  const uint8_t* srcA = rec + (BITS == 4 ? 64 * i0 + 8 * mA : 128 * i0 + 16 * mA);
  const uint8_t* srcB = rec + (BITS == 4 ? 64 * i0 + 8 * mB : 128 * i0 + 16 * mB);
  uint8_t* dstA = tile + (mA >> 2) * 16384 + 128 * i0;
  uint8_t* dstB = tile + (mB >> 2) * 16384 + 128 * i0;
  const int cA0 = ((2 * (mA & 3)) ^ r7) << 4, cA1 = ((2 * (mA & 3) + 1) ^ r7) << 4;
  const int cB0 = ((2 * (mB & 3)) ^ r7) << 4, cB1 = ((2 * (mB & 3) + 1) ^ r7) << 4;
  const int rstride = BITS == 4 ? 512 : 1024;         // 8 rows of codes
#pragma unroll
  for (int it = 0; it < RPW / 4; ++it) {
    const bool odd = it & 1;
    const uint8_t* src = (odd ? srcB : srcA) + rstride * (it >> 1);
    uint8_t* dst = (odd ? dstB : dstA) + 1024 * (it >> 1);
    uint32_t hv[8];                                    // positions 16 m16 + 0..15 as f16 pairs
    if (BITS == 4) {
      const uint2 w = *reinterpret_cast<const uint2*>(src);
      // offset codes u = c + 8: even channels in the low nibbles, odd ones (x16) in the high
      const uint32_t x0 = (w.x & 0x0F0F0F0Fu) ^ 0x08080808u, y0 = (w.x & 0xF0F0F0F0u) ^ 0x80808080u;
      const uint32_t x1 = (w.y & 0x0F0F0F0Fu) ^ 0x08080808u, y1 = (w.y & 0xF0F0F0F0u) ^ 0x80808080u;
      hv[0] = h2u(__hsub2(u2h(prmt(x0, K64, 0x4140u)), off8));    // channels 0, 2
      hv[1] = h2u(__hsub2(u2h(prmt(x0, K64, 0x4342u)), off8));    // 4, 6
      hv[2] = h2u(__hsub2(u2h(prmt(x1, K64, 0x4140u)), off8));    // 8, 10
      hv[3] = h2u(__hsub2(u2h(prmt(x1, K64, 0x4342u)), off8));    // 12, 14
      hv[4] = h2u(__hfma2(u2h(prmt(y0, K64, 0x4140u)), sixteenth, off16));   // 1, 3
      hv[5] = h2u(__hfma2(u2h(prmt(y0, K64, 0x4342u)), sixteenth, off16));   // 5, 7
      hv[6] = h2u(__hfma2(u2h(prmt(y1, K64, 0x4140u)), sixteenth, off16));   // 9, 11
      hv[7] = h2u(__hfma2(u2h(prmt(y1, K64, 0x4342u)), sixteenth, off16));   // 13, 15
    } else {
      const uint4 w = *reinterpret_cast<const uint4*>(src);
      const uint32_t ws[4] = {w.x ^ 0x80808080u, w.y ^ 0x80808080u, w.z ^ 0x80808080u, w.w ^ 0x80808080u};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        hv[2 * e] = h2u(__hsub2(u2h(prmt(ws[e], K64, 0x4140u)), off128));
        hv[2 * e + 1] = h2u(__hsub2(u2h(prmt(ws[e], K64, 0x4342u)), off128));
      }
    }
    *reinterpret_cast<uint4*>(dst + (odd ? cB0 : cA0)) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
    *reinterpret_cast<uint4*>(dst + (odd ? cB1 : cA1)) = make_uint4(hv[4], hv[5], hv[6], hv[7]);
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
// position.  Thread ct (of the NCT converter threads) owns the position
// pair 2 (ct % 64) + {0, 1} and a share NCT / 64 of the tokens.  Tokens
// s >= n give zero rows.
template <bool BF16, bool R8, int PMAX, int BITS>
__device__ __forceinline__ void build_keys(const uint8_t* stage, uint8_t* bx, uint8_t* au, int n, KeyExp ex, int ct) {
  using C = TcCfg<BF16, R8, PMAX>;
  const uint16_t* sc = reinterpret_cast<const uint16_t*>(stage + code_bytes(C::D, C::D, BITS));
  const uint8_t* rows = stage + C::REC;
  constexpr int SPT = PMAX / (C::NCT / 64);   // tokens per thread
  const int pp = ct & 63, s0 = (ct >> 6) * SPT;
  const int j0 = chan_of<BITS>(2 * pp), j1 = chan_of<BITS>(2 * pp + 1);
  const float upx = pow2i(ex.exx), upk = pow2i(ex.exk);
  const float2 sx = make_float2(__half2float(__ushort_as_half(sc[j0])) * upx,
                                __half2float(__ushort_as_half(sc[j1])) * upx);
  const float2 uk = make_float2(upk, upk);
  // byte offset of the pair inside a [rows][64] 128B-swizzled block: chunk (pp % 32) / 4, word pp % 4
  const int half = pp >> 5, chunk = (pp & 31) >> 2, word = (pp & 3) * 4;
  uint8_t* xb = bx + half * (C::NX * 128) + word;
  uint8_t* ab = au + half * (C::KU * 128) + word;
#pragma unroll
  for (int s = s0; s < s0 + SPT; ++s) {
    float2 kv = make_float2(0.f, 0.f);
    if (s < n) {
      kv.x = row_at<R8>(rows + s * C::ROWB, j0, BF16);
      kv.y = row_at<R8>(rows + s * C::ROWB, j1, BF16);
    }
    const float2 b = __fmul2_rn(kv, sx);
    const __half2 bh = __float22half2_rn(b);
    const float2 bhf = __half22float2(bh);
    const __half2 bl = __float22half2_rn(make_float2(b.x - bhf.x, b.y - bhf.y));
    const float2 k2 = __fmul2_rn(kv, uk);
    const __half2 kh = __float22half2_rn(k2);
    *reinterpret_cast<uint32_t*>(xb + sw128(s, chunk)) = h2u(bh);
    *reinterpret_cast<uint32_t*>(xb + sw128(PMAX + s, chunk)) = h2u(bl);
    *reinterpret_cast<uint32_t*>(ab + sw128(s, chunk)) = h2u(kh);
    *reinterpret_cast<uint32_t*>(ab + sw128(PMAX + s, chunk)) = h2u(kh);
    if (C::NSEG == 3) {
      const float2 khf = __half22float2(kh);
      *reinterpret_cast<uint32_t*>(ab + sw128(2 * PMAX + s, chunk)) =
          h2u(__float22half2_rn(make_float2(k2.x - khf.x, k2.y - khf.y)));
    }
  }
}

// R and U^ for one head, one TMEM lane (value channel i) per converter thread:
// x_s from TMEM, r_s = v_s[i] - gamma_s x_s, U^[s][i] = sum_s' W[s][s'] r_s',
// normalised by one power of two for the head, split hi + lo into row i of
// the update's B.  The two converter warps of a TMEM lane quadrant split the
// tokens s (each forms all of R).  Also the epilogue's per-position factors.
// A head with all PMAX tokens takes packed pair arithmetic over the factor
// rows; early commits (n < PMAX) take guarded scalar loops.
template <bool BF16, bool R8, int PMAX>
__device__ __forceinline__ void residual_update(const PoolDev& p, TcSmem<BF16, R8, PMAX>& sm, const uint8_t* stage,
                                                int bits, int t, int n, uint32_t tm, int k, int ct, int warp,
                                                int lane) {
  using C = TcCfg<BF16, R8, PMAX>;
  constexpr int H2 = PMAX / 2;                   // tokens per half
  const int m = k & 3;   // ring slot of this head
  const int P = p.P;
  const int qd = warp & 3, i = 32 * qd + lane;
  const int sb = ((warp - C::CONV0) >> 2) * H2;  // this warp's tokens [sb, sb + H2)
  const float* G = reinterpret_cast<const float*>(stage + C::REC + C::KVB);
  const float* W = G;
  const float* gam = G + P * P;
  const KeyExp ex = key_exponents(G, P);
  const float xinv = pow2i(-ex.exx);
  const uint8_t* vrow = stage + C::REC + C::D * C::ESZ + i * C::ESZ;   // v_0[i]
  float x[PMAX], r[PMAX], u[H2];
  {
    uint32_t xa[16], xb[16];
    tc::ld_32x32b_x16(tm + ((uint32_t)(32 * qd) << 16) + 256u * t + 128u, xa);
    if (PMAX == 16) tc::ld_32x32b_x16(tm + ((uint32_t)(32 * qd) << 16) + 256u * t + 144u, xb);
    tc::wait_ld();
#pragma unroll
    for (int s2 = 0; s2 < PMAX; s2 += 2) {
      const int h0 = s2, l0 = PMAX + s2;   // hi and lo columns of tokens s2, s2 + 1
      const float2 hi = make_float2(__uint_as_float(h0 < 16 ? xa[h0] : xb[h0 - 16]),
                                    __uint_as_float(h0 + 1 < 16 ? xa[h0 + 1] : xb[h0 - 15]));
      const float2 lo = make_float2(__uint_as_float(l0 < 16 ? xa[l0] : xb[l0 - 16]),
                                    __uint_as_float(l0 + 1 < 16 ? xa[l0 + 1] : xb[l0 - 15]));
      const float2 xs = __fadd2_rn(hi, lo);
      x[s2] = xs.x;
      x[s2 + 1] = xs.y;
    }
  }
  const bool full = n == PMAX && P == PMAX;
  float um = 0.f;
  if (full) {
#pragma unroll
    for (int s2 = 0; s2 < PMAX; s2 += 2) {
      const float2 g = __fmul2_rn(*reinterpret_cast<const float2*>(gam + s2), make_float2(-xinv, -xinv));
      const float2 v = make_float2(row_at<R8>(vrow + s2 * C::ROWB, 0, BF16), row_at<R8>(vrow + (s2 + 1) * C::ROWB, 0, BF16));
      const float2 rr = __ffma2_rn(g, make_float2(x[s2], x[s2 + 1]), v);
      r[s2] = rr.x;
      r[s2 + 1] = rr.y;
    }
#pragma unroll
    for (int s = 0; s < H2; ++s) {
      float2 acc = make_float2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < PMAX; c += 4) {
        const float4 w4 = *reinterpret_cast<const float4*>(W + (sb + s) * PMAX + c);
        acc = __ffma2_rn(make_float2(w4.x, w4.y), make_float2(r[c], r[c + 1]), acc);
        acc = __ffma2_rn(make_float2(w4.z, w4.w), make_float2(r[c + 2], r[c + 3]), acc);
      }
      u[s] = acc.x + acc.y;
    }
#pragma unroll
    for (int s = 0; s < H2; s += 2) um = max3_nan(um, fabsf(u[s]), fabsf(u[s + 1]));
  } else {
#pragma unroll
    for (int s = 0; s < PMAX; ++s)
      r[s] = s < n ? row_at<R8>(vrow + s * C::ROWB, 0, BF16) - gam[s] * (x[s] * xinv) : 0.f;
#pragma unroll
    for (int s = 0; s < H2; ++s) {
      const int ss = sb + s;
      float a = 0.f;
#pragma unroll
      for (int sp = 0; sp < PMAX; ++sp)
        if (ss < n && sp < n) a = fmaf(W[ss * P + sp], r[sp], a);
      u[s] = a;
      um = max_nan(um, fabsf(a));
    }
  }
  // one exponent for the head's U^ (all 128 lanes and both halves feed one product)
#pragma unroll
  for (int off = 16; off; off >>= 1) um = max_nan(um, __shfl_xor_sync(FULL, um, off));
  if (lane == 0) sm.red[k & 1][warp - C::CONV0] = um;
  tc::named_sync(6, C::NCT);
  um = 0.f;
#pragma unroll
  for (int w = 0; w < C::NCONV; ++w) um = max_nan(um, sm.red[k & 1][w]);
  int e_tot = ex.exk + norm_exp(um, 40);
  const float smax = G[P * P + P + 1];
  if (smax >= 1.17549435e-38f && smax < INFINITY) e_tot = min(e_tot, 111 - exp2_floor(smax));
  const float up = pow2i(e_tot - ex.exk);
  // row i of B (K-major, no swizzle): K entries [U^_hi (PMAX) | U^_lo (PMAX) | U^_hi (PMAX, fp32 rows)];
  // this thread writes entries sb .. sb + H2 - 1 of each segment
  uint32_t hi[H2 / 2], lo[H2 / 2];
#pragma unroll
  for (int e = 0; e < H2 / 2; ++e) {
    const float2 a = __fmul2_rn(make_float2(u[2 * e], u[2 * e + 1]), make_float2(up, up));
    const __half2 h = __float22half2_rn(a);
    const float2 hf = __half22float2(h);
    hi[e] = h2u(h);
    lo[e] = h2u(__float22half2_rn(make_float2(a.x - hf.x, a.y - hf.y)));
  }
  uint8_t* row = sm.bu[t] + (i >> 3) * 256 + (i & 7) * 16;
  auto put = [&](int kk, const uint32_t (&w)[H2 / 2]) {
    uint8_t* a = row + (kk >> 4) * 4096 + ((kk >> 3) & 1) * 128 + (kk & 7) * 2;
    if constexpr (H2 == 4) *reinterpret_cast<uint2*>(a) = make_uint2(w[0], w[1]);
    else *reinterpret_cast<uint4*>(a) = make_uint4(w[0], w[1], w[2], w[3]);
  };
  put(sb, hi);
  put(PMAX + sb, lo);
  if (C::NSEG == 3) put(2 * PMAX + sb, hi);
  // epilogue factors, one tile position per thread of the first 128
  if (ct < 128) {
    const uint16_t* sc = reinterpret_cast<const uint16_t*>(stage + code_bytes(C::D, C::D, bits));
    const int j = bits == 4 ? chan_of<4>(ct) : ct;
    sm.fj[m][ct] = gam[n - 1] * __half2float(__ushort_as_half(sc[j])) * pow2i(e_tot);
  }
  if (ct == 0) sm.meta_e[m] = e_tot;
}

template <bool BF16, bool R8, int PMAX>
__device__ void converter_role(const PoolDev& p, TcSmem<BF16, R8, PMAX>& sm, uint32_t tm, int warp, int lane) {
  using C = TcCfg<BF16, R8, PMAX>;
  const int cw = warp - C::CONV0, ct = 32 * cw + lane;   // ct < NCT
  // Every wait is followed by a vote at the converters' named barrier, so that
  // the four warps leave together and none is left waiting in a barrier.
  for (int k = 0;; ++k) {
    const int s = k % C::NST, t = k & 1, m = k & 3;
    bool ok = bounded_wait(&sm.stage_full[s], (uint32_t)((k / C::NST) & 1), p, &sm.abort);
    const int head = ok ? sm.stage_head[s] : -1;
    if (tc::named_sync_any(6, C::NCT, !ok)) return;
    const uint8_t* st = sm.stage[s];
    const int bits = head >= 0 ? p.bits[head % p.H] : 4;
    // the tile and X's keys of buffer t were last read by the products of the
    // head two back, whose completion the previous R step waited for
    if (head >= 0) {
      if (bits == 4) convert_codes<4, 128 / C::NCONV>(st, sm.tile[t], cw, lane);
      else convert_codes<8, 128 / C::NCONV>(st, sm.tile[t], cw, lane);
    }
    // the update of the head two back read this buffer's update keys; its
    // completion also means the epilogue of the head four back, which used
    // this ring slot, has read it
    if (k >= 2) ok = bounded_wait(&sm.acc_full[t], (uint32_t)(((k - 2) >> 1) & 1), p, &sm.abort);
    if (tc::named_sync_any(6, C::NCT, !ok)) return;
    if (head >= 0) {
      const int n = sm.stage_n[s];
      const KeyExp ex = key_exponents(reinterpret_cast<const float*>(st + C::REC + C::KVB), p.P);
      if (bits == 4) build_keys<BF16, R8, PMAX, 4>(st, sm.bx[t], sm.au[t], n, ex, ct);
      else build_keys<BF16, R8, PMAX, 8>(st, sm.bx[t], sm.au[t], n, ex, ct);
    }
    if (ct == 0) {
      sm.meta_head[m] = head;
      sm.meta_bits[m] = bits;
    }
    fence_proxy_async_smem();
    tc::mbar_arrive(&sm.tile_full[t]);
    if (k >= 1) {   // R and U^ of the previous head, whose X has had this head's conversion to land
      const int sp = (k - 1) % C::NST, tp = t ^ 1;
      ok = bounded_wait(&sm.x_full[tp], (uint32_t)(((k - 1) >> 1) & 1), p, &sm.abort);
      if (tc::named_sync_any(6, C::NCT, !ok)) return;
      tc::fence_after_sync();
      const int hp = sm.stage_head[sp];
      residual_update<BF16, R8, PMAX>(p, sm, sm.stage[sp], p.bits[hp % p.H], tp, sm.stage_n[sp], tm, k - 1, ct,
                                      warp, lane);
      fence_proxy_async_smem();
      tc::fence_before_sync();
      tc::mbar_arrive(&sm.bupd_full[tp]);
      tc::mbar_arrive(&sm.stage_empty[sp]);
    }
    if (head < 0) return;
  }
}

// ---- epilogue ----------------------------------------------------------------
// Four warps, one per TMEM lane quadrant qd.  Thread (g = lane / 4, q = lane % 4)
// holds, for 16-lane blocks blk of the quadrant, tile positions p = 32 qd +
// 16 blk + g + 8 h (h = 0, 1) and value channels i = 64 cb + 8 c + 2 q + {0, 1}
// (column half cb = 0, 1; c = 0..7): 128 elements of S'^T = S^T 2^e, four key
// channels of 32 values each.  INT4 tile positions pair the key channels 2m
// (h = 0) and 2m + 1 (h = 1) in one thread, so a code byte is thread-local.

// Codes of two values as the low byte (INT8) or low nibble (INT4) of each
// f16 half: x q + 1280 (resp. 1040) rounded to f16 is the integer 1280 + c
// (1040 + c) with c = rint_half_even(x q), whose mantissa's low byte is c
// modulo 256 (low nibble c modulo 16).
template <int BITS>
__device__ __forceinline__ uint32_t code_pair_fast(float a, float b, float q) {
  const float M = BITS == 4 ? 1040.f : 1280.f;
  return h2u(__float22half2_rn(__ffma2_rn(make_float2(a, b), make_float2(q, q), make_float2(M, M))));
}
// Same layout from the exact encoder (fp32 divide by the scale).
template <int BITS>
__device__ __forceinline__ uint32_t code_pair_exact(float a, float b, float sf) {
  const int qmax = BITS == 4 ? 7 : 127, off = BITS == 4 ? 16 : 256;
  const uint32_t ca = (uint32_t)(encode_value(a, sf, qmax) + off), cb = (uint32_t)(encode_value(b, sf, qmax) + off);
  return (0x6400u + ca) | ((0x6400u + cb) << 16);
}

template <bool BF16, bool R8, int PMAX, int BITS>
__device__ __forceinline__ void epilogue_head(const PoolDev& p, const CommitMaps& maps, TcSmem<BF16, R8, PMAX>& sm,
                                              uint32_t tm, int t, int m, int head, int we, int lane) {
  using C = TcCfg<BF16, R8, PMAX>;
  const int qd = we & 3, g = lane >> 2, q = lane & 3;
  const int cb = (we - C::EPI0) >> 2;   // value-channel half of this warp (two warps per quadrant)
  const int e_tot = sm.meta_e[m];
  const float down = pow2i(-e_tot);
  float f[2][2];
#pragma unroll
  for (int blk = 0; blk < 2; ++blk)
#pragma unroll
    for (int h = 0; h < 2; ++h) f[blk][h] = sm.fj[m][32 * qd + 16 * blk + g + 8 * h];
  // S'^T of block blk, column half cb: v[4 c + 2 h + z] = rows 64 cb + 8 c + 2 q + z of lane g + 8 h
  auto load = [&](int blk, float (&v)[32]) {
    uint32_t cr[32], ur[32];
    const uint32_t a = tm + ((uint32_t)(32 * qd + 16 * blk) << 16) + 256u * t + 64u * cb;
    tc::ld_16x256b_x8(a, cr);
    tc::ld_16x256b_x8(a + 128u, ur);
    tc::wait_ld();
#pragma unroll
    for (int c = 0; c < 8; ++c)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float2 r2 = __ffma2_rn(make_float2(__uint_as_float(cr[4 * c + 2 * h]), __uint_as_float(cr[4 * c + 2 * h + 1])),
                                     make_float2(f[blk][h], f[blk][h]),
                                     make_float2(__uint_as_float(ur[4 * c + 2 * h]), __uint_as_float(ur[4 * c + 2 * h + 1])));
        v[4 * c + 2 * h] = r2.x;
        v[4 * c + 2 * h + 1] = r2.y;
      }
  };

  // pass 1: column maxima, 16 values per key channel here, then the other
  // three lanes of the quad, then the other value-channel half
  float mx[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
  for (int blk = 0; blk < 2; ++blk) {
    float v[32];
    load(blk, v);
#pragma unroll
    for (int c = 0; c < 8; ++c)
#pragma unroll
      for (int h = 0; h < 2; ++h) mx[blk][h] = max3_nan(mx[blk][h], fabsf(v[4 * c + 2 * h]), fabsf(v[4 * c + 2 * h + 1]));
  }
#pragma unroll
  for (int blk = 0; blk < 2; ++blk)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      mx[blk][h] = max_nan(mx[blk][h], __shfl_xor_sync(FULL, mx[blk][h], 1));
      mx[blk][h] = max_nan(mx[blk][h], __shfl_xor_sync(FULL, mx[blk][h], 2));
    }
  if (q == 0) {
#pragma unroll
    for (int blk = 0; blk < 2; ++blk)
#pragma unroll
      for (int h = 0; h < 2; ++h) sm.emax[cb][32 * qd + 16 * blk + g + 8 * h] = mx[blk][h];
  }
  tc::named_sync(7 + qd, 64);   // the two warps of this quadrant
#pragma unroll
  for (int blk = 0; blk < 2; ++blk)
#pragma unroll
    for (int h = 0; h < 2; ++h) mx[blk][h] = max_nan(mx[blk][h], sm.emax[cb ^ 1][32 * qd + 16 * blk + g + 8 * h]);

  // scale of the column (blk, h) = (q >> 1, q & 1), then shared across the quad
  const int qmax = BITS == 4 ? 7 : 127;
  uint8_t* stg = sm.stg[t];
  float qf, sf;
  bool bad;
  {
    const int pos = 32 * qd + 16 * (q >> 1) + g + 8 * (q & 1);
    const float amax = mx[q >> 1][q & 1] * down;
    const GroupScale gs = group_scale(amax, isfinite(amax), qmax, p.flags);
    sf = gs.sf;
    qf = gs.sf > 0.f ? __frcp_rn(gs.sf) * down : 0.f;
    bad = !fast_encode_ok(amax, gs, qmax) || !(qf < INFINITY);
    if (cb == 0) reinterpret_cast<uint16_t*>(stg + 16384)[chan_of<BITS>(pos)] = gs.bits;
  }
  const bool slow = __any_sync(FULL, bad);
  float qv[2][2];
#pragma unroll
  for (int z = 0; z < 4; ++z) qv[z >> 1][z & 1] = __shfl_sync(FULL, slow ? sf : qf, (lane & ~3) | z);

  // pass 2: codes, gathered and stored transposed (four 8-row matrices per
  // stmatrix) into the swizzled staging rows; lane l gives the address of
  // row l % 8 of matrix l / 8
  const uint32_t stg_a = smem_addr(stg);
  const int r8 = lane & 7, mq = lane >> 3;
  auto encode = [&](auto fast) {
    auto pair = [&](const float (&v)[32], int blk, int c, int h) -> uint32_t {
      if (decltype(fast)::value) return code_pair_fast<BITS>(v[4 * c + 2 * h], v[4 * c + 2 * h + 1], qv[blk][h]);
      return code_pair_exact<BITS>(v[4 * c + 2 * h] * down, v[4 * c + 2 * h + 1] * down, qv[blk][h]);
    };
    if (BITS == 4) {
      const uint32_t base = stg_a + 64 * r8 + ((qd ^ ((r8 >> 1) & 3)) << 4) + 512 * mq;
      {
        uint32_t rb[2][8];   // [blk][c]: bytes 0 and 2 are the row pairs' code bytes
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
          float v[32];
          load(blk, v);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            rb[blk][c] = (pair(v, blk, c, 0) & 0x000F000Fu) | ((pair(v, blk, c, 1) << 4) & ~0x000F000Fu);
        }
#pragma unroll
        for (int c0 = 0; c0 < 8; c0 += 4)
          tc::stsm_trans_b8_x4(base + 512u * (8 * cb + c0), prmt(rb[0][c0], rb[1][c0], 0x6420u),
                               prmt(rb[0][c0 + 1], rb[1][c0 + 1], 0x6420u), prmt(rb[0][c0 + 2], rb[1][c0 + 2], 0x6420u),
                               prmt(rb[0][c0 + 3], rb[1][c0 + 3], 0x6420u));
      }
    } else {
#pragma unroll
      for (int blk = 0; blk < 2; ++blk) {
        const uint32_t base = stg_a + 128 * r8 + (((2 * qd + blk) ^ r8) << 4) + 1024 * mq;
        {
          float v[32];
          load(blk, v);
          uint32_t w[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) w[c] = prmt(pair(v, blk, c, 0), pair(v, blk, c, 1), 0x6420u);
#pragma unroll
          for (int c0 = 0; c0 < 8; c0 += 4)
            tc::stsm_trans_b8_x4(base + 1024u * (8 * cb + c0), w[c0], w[c0 + 1], w[c0 + 2], w[c0 + 3]);
        }
      }
    }
  };
  if (!slow) encode(std::true_type{});
  else encode(std::false_type{});
  tc::fence_before_sync();
  tc::mbar_arrive(&sm.tmem_empty[t]);
  fence_proxy_async_smem();
  tc::named_sync(5, C::NET);
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
    const int t = k & 1, m = k & 3;
    // the four warps vote after the wait and leave together (named barriers follow)
    bool ok = bounded_wait(&sm.acc_full[t], (uint32_t)((k >> 1) & 1), p, &sm.abort);
    // the converters' per-head values (factors, exponent) are read directly after their arrival
    if (ok && sm.meta_head[m] >= 0) ok = bounded_wait(&sm.bupd_full[t], (uint32_t)((k >> 1) & 1), p, &sm.abort);
    if (tc::named_sync_any(5, TcCfg<BF16, R8, PMAX>::NET, !ok)) break;
    tc::fence_after_sync();
    const int head = sm.meta_head[m];
    if (head < 0) break;
    if (sm.meta_bits[m] == 4) epilogue_head<BF16, R8, PMAX, 4>(p, maps, sm, tm, t, m, head, warp, lane);
    else epilogue_head<BF16, R8, PMAX, 8>(p, maps, sm, tm, t, m, head, warp, lane);
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
  if (tid == 0) {
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(&sm.stage_full[s], 1);
      mbar_init(&sm.stage_empty[s], C::NCT);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&sm.tile_full[t], C::NCT);
      mbar_init(&sm.x_full[t], 1);
      mbar_init(&sm.bupd_full[t], C::NCT);
      mbar_init(&sm.acc_full[t], 1);
      mbar_init(&sm.tmem_empty[t], C::NET);
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
    producer_role<BF16, R8, PMAX>(p, sm, sp, lane);
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
