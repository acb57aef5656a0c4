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
//   A[t][s] = beta_t gamma_{t/s} (k_t . k_s), s < t  (forward substitution);
//   S_P = gamma_P S~0 + sum_s gamma_{P/s} u_s k_s^T.
#include "encode.cuh"

namespace pace {

namespace {

constexpr int kThreads = 128;

struct SmemGet {
  const float* S;
  int ld;
  __device__ __forceinline__ float operator()(int i, int j) const { return S[i * ld + j]; }
};

__global__ void __launch_bounds__(kThreads) commit_kernel(PoolDev p) {
  extern __shared__ float smem[];
  __shared__ float al[PACE_MAX_PERIOD], be[PACE_MAX_PERIOD], gam[PACE_MAX_PERIOD + 1];
  __shared__ float gram[PACE_MAX_PERIOD][PACE_MAX_PERIOD];
  __shared__ float A[PACE_MAX_PERIOD][PACE_MAX_PERIOD];
  __shared__ float glast[PACE_MAX_PERIOD];
  __shared__ float sf_sm[PACE_MAX_D];
  __shared__ int go;

  const int head = blockIdx.x;
  const int h = head % p.H, b = head / p.H;
  const int d_k = p.d_k, d_v = p.d_v, P = p.P, io = p.io, tid = threadIdx.x;
  const int esz = io_size(io);
  const int bits = p.bits[h];
  const int ld = d_k + 1;
  float* S = smem;                         // [d_v][d_k + 1]
  float* Ks = S + d_v * ld;                // [P][d_k]
  float* Vs = Ks + P * d_k;                // [P][d_v]

  if (tid == 0) go = (p.fill[head] == P);
  __syncthreads();
  if (!go) return;

  uint8_t* rec = p.state + (size_t)b * p.slot_stride + p.rec_off[h];
  uint16_t* rsc = reinterpret_cast<uint16_t*>(rec + code_bytes(d_k, d_v, bits));
  const int row_bytes = d_k * bits / 8;
  for (int idx = tid; idx < d_v * d_k; idx += kThreads) {
    const int i = idx / d_k, j = idx - i * d_k;
    const float sf = __half2float(__ushort_as_half(rsc[p.axis == PACE_SCALE_COL ? j : i]));
    S[i * ld + j] = (float)decode_code(rec, row_bytes, i, j, bits) * sf;
  }
  const size_t row_elems = (size_t)(d_k + d_v);
  const uint8_t* kv_head = p.kv + (size_t)head * P * row_elems * esz;
  const uint8_t* ab_head = p.ab + (size_t)head * P * 2 * esz;
  for (int idx = tid; idx < P * (int)row_elems; idx += kThreads) {
    const int s = idx / (int)row_elems, e = idx - s * (int)row_elems;
    const float x = load_io(kv_head, (size_t)s * row_elems + e, io);
    if (e < d_k) Ks[s * d_k + e] = x; else Vs[s * d_v + e - d_k] = x;
  }
  for (int s = tid; s < P; s += kThreads) {
    al[s] = load_io(ab_head, (size_t)s * 2 + 0, io);
    be[s] = load_io(ab_head, (size_t)s * 2 + 1, io);
  }
  __syncthreads();

  {  // gram[t][s] = k_t . k_s, s < t
    const int lane = tid & 31, warp = tid >> 5;
    const int npairs = P * (P - 1) / 2;
    for (int d = warp; d < npairs; d += kThreads / 32) {
      int t = 1;
      while (t * (t + 1) / 2 <= d) ++t;
      const int s = d - t * (t - 1) / 2;
      float acc = 0.f;
      for (int j = lane; j < d_k; j += 32) acc = fmaf(Ks[t * d_k + j], Ks[s * d_k + j], acc);
      for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (lane == 0) gram[t][s] = acc;
    }
  }
  __syncthreads();
  if (tid == 0) {
    gam[0] = 1.f;
    for (int t = 1; t <= P; ++t) gam[t] = gam[t - 1] * al[t - 1];
    for (int s = 1; s <= P; ++s) {
      float g = 1.f;                                  // gamma_{t/s}
      for (int t = s + 1; t <= P; ++t) {
        g *= al[t - 1];
        A[t - 1][s - 1] = be[t - 1] * g * gram[t - 1][s - 1];
      }
      glast[s - 1] = g;                               // gamma_{P/s}
    }
  }
  __syncthreads();

  // per row i: x_s = S~0[i,:] . k_s ; forward substitution for u_t ; row update
  for (int i = tid; i < d_v; i += kThreads) {
    float u[PACE_MAX_PERIOD];
    float* Si = S + i * ld;
#pragma unroll
    for (int t = 0; t < PACE_MAX_PERIOD; ++t) {
      if (t < P) {
        float x = 0.f;
        for (int j = 0; j < d_k; ++j) x = fmaf(Si[j], Ks[t * d_k + j], x);
        float acc = be[t] * (Vs[t * d_v + i] - gam[t + 1] * x);
#pragma unroll
        for (int s = 0; s < PACE_MAX_PERIOD; ++s)
          if (s < t) acc = fmaf(-A[t][s], u[s], acc);
        u[t] = acc;
      }
    }
#pragma unroll
    for (int s = 0; s < PACE_MAX_PERIOD; ++s)
      if (s < P) u[s] *= glast[s];
    const float gP = gam[P];
    for (int j = 0; j < d_k; ++j) {
      float acc = gP * Si[j];
#pragma unroll
      for (int s = 0; s < PACE_MAX_PERIOD; ++s)
        if (s < P) acc = fmaf(u[s], Ks[s * d_k + j], acc);
      Si[j] = acc;
    }
  }
  __syncthreads();

  encode_matrix(SmemGet{S, ld}, d_k, d_v, bits, p.axis, rec, rsc, p.flags, sf_sm);
  if (tid == 0) p.fill[head] = 0;
}

}  // namespace

static size_t commit_smem_bytes(const PoolDev& p) {
  return sizeof(float) * ((size_t)p.d_v * (p.d_k + 1) + (size_t)p.P * (p.d_k + p.d_v));
}

cudaError_t launch_commit(const PoolDev& p, cudaStream_t st) {
  const size_t smem = commit_smem_bytes(p);
  cudaError_t e = cudaFuncSetAttribute(commit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  commit_kernel<<<(unsigned)(p.B * p.H), kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace pace
