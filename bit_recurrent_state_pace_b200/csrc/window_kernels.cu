// Pure-write window: the pool's buffer as a sliding window of FP8 writes.
//
// "低比特量化新突破：GGA+PW让线性注意力长文本生成更准更短", section
// "PW：让近期写入走“纯净通道”": the most recent writes are kept apart from the
// low-bit history as FP8 (k, v) pairs that take full part in the state
// transition, and a pair is merged into the history only when it leaves the
// window of S steps.
//
// With S = the pool's P, one window step is the pool's own path plus three
// small kernels:
//  * k and v are rounded to E4M3 (round to nearest even, saturating) and kept
//    in the io dtype, which holds every E4M3 value exactly;
//  * the decode step reads out o_t from the stored history and the window,
//    exactly in chunk form, and appends the pair;
//  * a head whose window now holds S pairs gets the one-token factors of its
//    oldest pair (W = beta_0, gamma = alpha_0, max |k_0|, largest stored
//    scale) in the entries of its factor block that the Gram cache does not
//    use, and the commit applies that pair alone (n = 1);
//  * the remaining S - 1 pairs move down one row, their Gram entries are
//    recomputed, and fill = S - 1.
#include "e4m3.cuh"
#include "window.cuh"

namespace pace {

namespace {

constexpr unsigned FULL = 0xffffffffu;

// dst[i] = E4M3(src[i]) in the io dtype, for n elements.
__global__ void e4m3_round_kernel(const void* __restrict__ src, void* __restrict__ dst, int64_t n, int io) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    if (io == PACE_IO_BF16) {
      const float x = bf16_bits_to_float(reinterpret_cast<const uint16_t*>(src)[i]);
      reinterpret_cast<uint16_t*>(dst)[i] = float_to_bf16_bits_rn(e4m3_round(x));   // exact
    } else {
      reinterpret_cast<float*>(dst)[i] = e4m3_round(reinterpret_cast<const float*>(src)[i]);
    }
  }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int off = 16; off; off >>= 1) v = fmaxf(v, __shfl_xor_sync(FULL, v, off));
  return v;
}

// One warp per head.  A head whose window holds P pairs: the commit factors
// of its oldest pair, and the mark that commits one token.
__global__ void window_prepare_kernel(PoolDev p, int n_heads) {
  const int lane = threadIdx.x & 31;
  const int head = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
  if (head >= n_heads || p.fill[head] != p.P) return;
  const int P = p.P, h = head % p.H, b = head / p.H;
  const uint8_t* k0 = p.kv + (size_t)head * P * (size_t)(p.d_k + p.d_v) * row_esz(p);
  float km = 0.f;
  for (int j = lane; j < p.d_k; j += 32)
    km = fmaxf(km, fabsf(p.row8 ? row_at<true>(k0, j, false) : load_io(k0, j, p.io)));
  km = warp_max(km);
  const uint8_t* rec = p.state + (size_t)b * p.slot_stride + p.rec_off[h];
  const uint16_t* sc = reinterpret_cast<const uint16_t*>(rec + code_bytes(p.d_k, p.d_v, p.bits[h]));
  float sm = 0.f;
  for (int j = lane; j < p.n_groups; j += 32) sm = fmaxf(sm, fabsf(__half2float(__ushort_as_half(sc[j]))));
  sm = warp_max(sm);
  if (lane == 0) {
    const uint8_t* ab = p.ab + (size_t)head * p.ab_stride;      // row 0: alpha_0, beta_0
    float* g = reinterpret_cast<float*>(p.gram + (size_t)head * p.gram_stride);
    g[0] = load_io(ab, 1, p.io);                                // W[0][0] = gamma_{1/1} T beta = beta_0
    g[P * P] = load_io(ab, 0, p.io);                            // gamma_0 = alpha_0
    g[P * P + P] = km;
    g[P * P + P + 1] = sm;
    p.fill[head] = PACE_FILL_COMMIT | 1;
  }
}

// One warp per head.  A head whose oldest pair was just merged (fill 0 after
// the commit): rows 1..P-1 and their gates move down one, the Gram entries of
// the remaining pairs are recomputed, fill = P - 1.  The moves go four rows
// at a time (loads in flight together, then the stores); the keys of the
// remaining pairs are read once into registers (EPL channels per lane) and
// every Gram entry is a register dot product and a warp sum.
template <int D, int PMAX>
__global__ void window_shift_kernel(PoolDev p, int n_heads) {
  constexpr int EPL = D / 32;
  const int lane = threadIdx.x & 31;
  const int head = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
  if (head >= n_heads || p.fill[head] != 0) return;
  const int P = p.P;
  const size_t row = (size_t)(p.d_k + p.d_v) * row_esz(p);      // bytes, a multiple of 64
  const int n16 = (int)(row / 16);                              // <= 64
  uint8_t* kv = p.kv + (size_t)head * P * row;
  for (int r0 = 0; r0 + 1 < P; r0 += 4) {
    uint4 tmp[4][2];
#pragma unroll
    for (int rr = 0; rr < 4; ++rr)
#pragma unroll
      for (int i = 0; i < 2; ++i)
        if (r0 + rr + 1 < P && lane + 32 * i < n16)
          tmp[rr][i] = reinterpret_cast<const uint4*>(kv + (r0 + rr + 1) * row)[lane + 32 * i];
    __syncwarp();
#pragma unroll
    for (int rr = 0; rr < 4; ++rr)
#pragma unroll
      for (int i = 0; i < 2; ++i)
        if (r0 + rr + 1 < P && lane + 32 * i < n16)
          reinterpret_cast<uint4*>(kv + (r0 + rr) * row)[lane + 32 * i] = tmp[rr][i];
    __syncwarp();
  }
  {
    uint8_t* ab = p.ab + (size_t)head * p.ab_stride;            // [P][2] io elements
    const bool mv = lane + 2 < 2 * P;
    float x = 0.f;
    if (mv) x = load_io(ab, lane + 2, p.io);
    __syncwarp();
    if (mv) {
      if (p.io == PACE_IO_BF16) reinterpret_cast<uint16_t*>(ab)[lane] = float_to_bf16_bits_rn(x);   // exact
      else reinterpret_cast<float*>(ab)[lane] = x;
    }
  }
  __syncwarp();
  // Gram entries G[t][s] = k_t . k_s of the remaining pairs, s < t < P - 1
  float kr[PMAX][EPL];
#pragma unroll
  for (int t = 0; t < PMAX; ++t)
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const int j = EPL * lane + e;
      kr[t][e] = t + 1 < P ? (p.row8 ? row_at<true>(kv + t * row, j, false) : load_io(kv + t * row, j, p.io))
                           : 0.f;
    }
  float* g = reinterpret_cast<float*>(p.gram + (size_t)head * p.gram_stride);
#pragma unroll
  for (int t = 1; t < PMAX; ++t)
#pragma unroll
    for (int s = 0; s < t; ++s) {
      if (t + 1 < P) {
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc = fmaf(kr[t][e], kr[s][e], acc);
#pragma unroll
        for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(FULL, acc, off);
        if (lane == 0) g[t * P + s] = acc;
      }
    }
  if (lane == 0) p.fill[head] = P - 1;
}

template <int D>
cudaError_t launch_shift_d(const PoolDev& p, cudaStream_t st) {
  const int n = p.B * p.H;
  const unsigned blocks = (unsigned)((n + 7) / 8);
  if (p.P <= 4) window_shift_kernel<D, 4><<<blocks, 256, 0, st>>>(p, n);
  else if (p.P <= 8) window_shift_kernel<D, 8><<<blocks, 256, 0, st>>>(p, n);
  else window_shift_kernel<D, 16><<<blocks, 256, 0, st>>>(p, n);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_e4m3_round(const void* src, void* dst, int64_t n, int io, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  e4m3_round_kernel<<<(unsigned)blocks, 256, 0, st>>>(src, dst, n, io);
  return cudaGetLastError();
}

cudaError_t launch_window_prepare(const PoolDev& p, cudaStream_t st) {
  const int n = p.B * p.H;
  window_prepare_kernel<<<(unsigned)((n + 7) / 8), 256, 0, st>>>(p, n);
  return cudaGetLastError();
}

cudaError_t launch_window_shift(const PoolDev& p, cudaStream_t st) {
  switch (p.d_k) {
    case 32: return launch_shift_d<32>(p, st);
    case 64: return launch_shift_d<64>(p, st);
    case 128: return launch_shift_d<128>(p, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace pace
