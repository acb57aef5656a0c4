// Per-token readout: one decode token for every (slot, head) of a pool.
//
// "PACE: A New 4-Bit Recurrent State Quantization Method ...", section
// "Periodic Rounding: Reducing Error Accumulation": decoded tokens wait in a
// small buffer and the stored state is rounded only once per period; "PACE:
// four-bit recurrent state by rounding less often", flowchart "New tokens ->
// Small buffer".  The output of the n-th buffered token is exact in chunk
// form from the stored state S~0 (the state is never materialised):
//
//   o_n = S_n q_n = S~0 q^ + sum_s z_s v_s,   q^ = gamma_n q_n - sum_s z_s gamma_s k_s,
//   z = diag(beta) (I + A)^{-T} w,  w_s = gamma_{n/s} (k_s . q_n),
//   A[t][s] = beta_t gamma_{t/s} (k_t . k_s) for s < t,
//
// which follows from the UT/WY chunk form S_n = gamma_n S~0 + sum_s
// gamma_{n/s} u_s k_s^T with U = (I + A)^{-1} diag(beta) (V - diag(gamma) X^T),
// X = S~0 K^T, by moving (I + A)^{-1} onto the readout side: only one
// state-sized product (S~0 q^) is needed per token.
#include "encode.cuh"

namespace pace {

namespace {

constexpr int kThreads = 128;

__global__ void __launch_bounds__(kThreads) decode_step_kernel(PoolDev p, const void* __restrict__ q,
                                                               const void* __restrict__ k,
                                                               const void* __restrict__ v,
                                                               const void* __restrict__ alpha,
                                                               const void* __restrict__ beta,
                                                               float* __restrict__ o) {
  __shared__ float Ks[PACE_MAX_PERIOD][PACE_MAX_D];
  __shared__ float Vs[PACE_MAX_PERIOD][PACE_MAX_D];
  __shared__ float qs[PACE_MAX_D], qhat[PACE_MAX_D], sc[PACE_MAX_D];
  __shared__ float al[PACE_MAX_PERIOD], be[PACE_MAX_PERIOD], kq[PACE_MAX_PERIOD];
  __shared__ float gram[PACE_MAX_PERIOD][PACE_MAX_PERIOD];
  __shared__ float zv[PACE_MAX_PERIOD], zk[PACE_MAX_PERIOD], gamma_n;
  __shared__ int n_sh;

  const int head = blockIdx.x;
  const int h = head % p.H, b = head / p.H;
  const int d_k = p.d_k, d_v = p.d_v, P = p.P, io = p.io, tid = threadIdx.x;
  const int esz = io_size(io);
  const int bits = p.bits[h];

  if (tid == 0) {
    const int n_prev = p.fill[head];
    n_sh = (n_prev >= 0 && n_prev < P) ? n_prev + 1 : -1;
    if (n_sh < 0) atomicOr(p.flags, PACE_FLAG_BUFFER_FULL);
  }
  __syncthreads();
  const int n = n_sh;
  if (n < 0) {
    for (int i = tid; i < d_v; i += kThreads) o[(size_t)head * d_v + i] = __int_as_float(0x7fc00000);
    return;
  }

  // current token -> shared memory and buffer row n-1 (raw io bits copied)
  const size_t row_elems = (size_t)(d_k + d_v);
  uint8_t* kv_head = p.kv + (size_t)head * P * row_elems * esz;
  uint8_t* ab_head = p.ab + (size_t)head * P * 2 * esz;
  for (int j = tid; j < d_k; j += kThreads) {
    Ks[n - 1][j] = load_io(k, (size_t)head * d_k + j, io);
    qs[j] = load_io(q, (size_t)head * d_k + j, io);
    if (esz == 2)
      reinterpret_cast<uint16_t*>(kv_head)[(n - 1) * row_elems + j] =
          reinterpret_cast<const uint16_t*>(k)[(size_t)head * d_k + j];
    else
      reinterpret_cast<float*>(kv_head)[(n - 1) * row_elems + j] =
          reinterpret_cast<const float*>(k)[(size_t)head * d_k + j];
  }
  for (int i = tid; i < d_v; i += kThreads) {
    Vs[n - 1][i] = load_io(v, (size_t)head * d_v + i, io);
    if (esz == 2)
      reinterpret_cast<uint16_t*>(kv_head)[(n - 1) * row_elems + d_k + i] =
          reinterpret_cast<const uint16_t*>(v)[(size_t)head * d_v + i];
    else
      reinterpret_cast<float*>(kv_head)[(n - 1) * row_elems + d_k + i] =
          reinterpret_cast<const float*>(v)[(size_t)head * d_v + i];
  }
  if (tid == 0) {
    al[n - 1] = load_io(alpha, head, io);
    be[n - 1] = load_io(beta, head, io);
    if (esz == 2) {
      reinterpret_cast<uint16_t*>(ab_head)[(n - 1) * 2 + 0] = reinterpret_cast<const uint16_t*>(alpha)[head];
      reinterpret_cast<uint16_t*>(ab_head)[(n - 1) * 2 + 1] = reinterpret_cast<const uint16_t*>(beta)[head];
    } else {
      reinterpret_cast<float*>(ab_head)[(n - 1) * 2 + 0] = reinterpret_cast<const float*>(alpha)[head];
      reinterpret_cast<float*>(ab_head)[(n - 1) * 2 + 1] = reinterpret_cast<const float*>(beta)[head];
    }
  }
  // earlier buffered tokens
  for (int idx = tid; idx < (n - 1) * (int)row_elems; idx += kThreads) {
    const int s = idx / (int)row_elems, e = idx - s * (int)row_elems;
    const float x = load_io(kv_head, (size_t)s * row_elems + e, io);
    if (e < d_k) Ks[s][e] = x; else Vs[s][e - d_k] = x;
  }
  for (int s = tid; s < n - 1; s += kThreads) {
    al[s] = load_io(ab_head, (size_t)s * 2 + 0, io);
    be[s] = load_io(ab_head, (size_t)s * 2 + 1, io);
  }
  // scales of the stored state
  const uint8_t* rec = p.state + (size_t)b * p.slot_stride + p.rec_off[h];
  const uint16_t* rsc = reinterpret_cast<const uint16_t*>(rec + code_bytes(d_k, d_v, bits));
  for (int g = tid; g < p.n_groups; g += kThreads) sc[g] = __half2float(__ushort_as_half(rsc[g]));
  __syncthreads();

  // dot products: gram[t][s] = k_t.k_s (s < t), kq[s] = k_s.q
  {
    const int lane = tid & 31, warp = tid >> 5;
    const int npairs = n * (n - 1) / 2;
    for (int d = warp; d < npairs + n; d += kThreads / 32) {
      int t, s;
      const float* a;
      const float* c;
      if (d < npairs) {
        t = 1;
        while (t * (t + 1) / 2 <= d) ++t;
        s = d - t * (t - 1) / 2;
        a = Ks[t];
        c = Ks[s];
      } else {
        t = -1;
        s = d - npairs;
        a = Ks[s];
        c = qs;
      }
      float acc = 0.f;
      for (int j = lane; j < d_k; j += 32) acc = fmaf(a[j], c[j], acc);
      for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (lane == 0) {
        if (t >= 0) gram[t][s] = acc; else kq[s] = acc;
      }
    }
  }
  __syncthreads();

  // small n x n solve: y = (I + A)^{-T} w by backward substitution; z = beta * y
  if (tid == 0) {
    float y[PACE_MAX_PERIOD];
    float gam[PACE_MAX_PERIOD + 1];
    gam[0] = 1.f;
    for (int t = 1; t <= n; ++t) gam[t] = gam[t - 1] * al[t - 1];       // gamma_t
    for (int s = n; s >= 1; --s) {
      float g_ns = 1.f;                                                   // gamma_{n/s}
      for (int r = s + 1; r <= n; ++r) g_ns *= al[r - 1];
      float acc = g_ns * kq[s - 1];
      float g_ts = 1.f;                                                   // gamma_{t/s}
      for (int t = s + 1; t <= n; ++t) {
        g_ts *= al[t - 1];
        const float a_ts = be[t - 1] * g_ts * gram[t - 1][s - 1];
        acc -= a_ts * y[t - 1];
      }
      y[s - 1] = acc;
    }
    for (int s = 1; s <= n; ++s) {
      const float z = be[s - 1] * y[s - 1];
      zv[s - 1] = z;
      zk[s - 1] = z * gam[s];
    }
    gamma_n = gam[n];
  }
  __syncthreads();

  // q^ = gamma_n q - sum_s z_s gamma_s k_s  (COL: folded with the column scales)
  for (int j = tid; j < d_k; j += kThreads) {
    float acc = gamma_n * qs[j];
    for (int s = 0; s < n; ++s) acc = fmaf(-zk[s], Ks[s][j], acc);
    qhat[j] = p.axis == PACE_SCALE_COL ? acc * sc[j] : acc;
  }
  __syncthreads();

  // o_i = (S~0 q^)_i + sum_s z_s v_s[i]
  const int row_bytes = d_k * bits / 8;
  for (int i = tid; i < d_v; i += kThreads) {
    float acc = 0.f;
    for (int j = 0; j < d_k; ++j) acc = fmaf((float)decode_code(rec, row_bytes, i, j, bits), qhat[j], acc);
    if (p.axis == PACE_SCALE_ROW) acc *= sc[i];
    for (int s = 0; s < n; ++s) acc = fmaf(zv[s], Vs[s][i], acc);
    o[(size_t)head * d_v + i] = acc;
  }
  if (tid == 0) p.fill[head] = n;
}

}  // namespace

cudaError_t launch_decode_step(const PoolDev& p, const void* q, const void* k, const void* v,
                               const void* alpha, const void* beta, float* o, cudaStream_t st) {
  decode_step_kernel<<<(unsigned)(p.B * p.H), kThreads, 0, st>>>(p, q, k, v, alpha, beta, o);
  return cudaGetLastError();
}

}  // namespace pace
