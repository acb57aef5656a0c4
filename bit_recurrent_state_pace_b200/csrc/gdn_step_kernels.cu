// Unquantised one-token update of the gated delta rule for n independent
// heads, state updated in place (fp32 or bf16 storage).  Not PACE: used for
// the fp32 warm-up prefill, the unquantised reference trajectory and the
// bf16-state throughput comparison.
//
// Rule (reading of the gate + delta rule of "低比特量化新突破：GGA+PW让线性注意力
// 长文本生成更准更短", section "为什么低比特状态量化会“越写越错”"):
//   S <- a S (I - b k k^T) + b v k^T = a (S - b (S k) k^T) + b v k^T,  o = S q.
// One warp per state row; each lane holds D/32 consecutive entries.
#include "pace_internal.cuh"

namespace pace {

namespace {

constexpr int kThreads = 256;

template <int D, bool BF16>
__global__ void __launch_bounds__(kThreads) gdn_step_kernel(void* __restrict__ Sv,
                                                            const void* __restrict__ q,
                                                            const void* __restrict__ k,
                                                            const void* __restrict__ v,
                                                            const void* __restrict__ alpha,
                                                            const void* __restrict__ beta, int io,
                                                            float* __restrict__ o) {
  constexpr int EPL = D / 32;
  __shared__ float ks[D], qs[D];
  const size_t head = blockIdx.x;
  for (int j = threadIdx.x; j < D; j += kThreads) {
    ks[j] = load_io(k, head * D + j, io);
    qs[j] = load_io(q, head * D + j, io);
  }
  const float a = load_io(alpha, head, io), bt = load_io(beta, head, io);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float kr[EPL], qr[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    kr[e] = ks[lane * EPL + e];
    qr[e] = qs[lane * EPL + e];
  }
  for (int i = warp; i < D; i += kThreads / 32) {
    float x[EPL];
    if (BF16) {
      const uint16_t* row = reinterpret_cast<const uint16_t*>(Sv) + (head * D + i) * D + lane * EPL;
#pragma unroll
      for (int e = 0; e < EPL; ++e) x[e] = bf16_bits_to_float(row[e]);
    } else {
      const float* row = reinterpret_cast<const float*>(Sv) + (head * D + i) * D + lane * EPL;
#pragma unroll
      for (int e = 0; e < EPL; ++e) x[e] = row[e];
    }
    float sk = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) sk = fmaf(x[e], kr[e], sk);
    for (int off = 16; off; off >>= 1) sk += __shfl_xor_sync(0xffffffffu, sk, off);
    const float vi = load_io(v, head * D + i, io);
    const float c = bt * vi - a * bt * sk;   // coefficient of k^T in the new row
    float so = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      x[e] = fmaf(a, x[e], c * kr[e]);
      if (BF16) x[e] = bf16_bits_to_float(float_to_bf16_bits_rn(x[e]));
      so = fmaf(x[e], qr[e], so);
    }
    if (BF16) {
      uint16_t* row = reinterpret_cast<uint16_t*>(Sv) + (head * D + i) * D + lane * EPL;
#pragma unroll
      for (int e = 0; e < EPL; ++e) row[e] = float_to_bf16_bits_rn(x[e]);
    } else {
      float* row = reinterpret_cast<float*>(Sv) + (head * D + i) * D + lane * EPL;
#pragma unroll
      for (int e = 0; e < EPL; ++e) row[e] = x[e];
    }
    if (o) {
      for (int off = 16; off; off >>= 1) so += __shfl_xor_sync(0xffffffffu, so, off);
      if (lane == 0) o[head * D + i] = so;
    }
  }
}

template <bool BF16>
cudaError_t launch(void* S, const void* q, const void* k, const void* v, const void* alpha,
                   const void* beta, int io, float* o, int64_t n, int d, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  switch (d) {
    case 32: gdn_step_kernel<32, BF16><<<(unsigned)n, kThreads, 0, st>>>(S, q, k, v, alpha, beta, io, o); break;
    case 64: gdn_step_kernel<64, BF16><<<(unsigned)n, kThreads, 0, st>>>(S, q, k, v, alpha, beta, io, o); break;
    case 128: gdn_step_kernel<128, BF16><<<(unsigned)n, kThreads, 0, st>>>(S, q, k, v, alpha, beta, io, o); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gdn_step_f32(float* S, const void* q, const void* k, const void* v,
                                const void* alpha, const void* beta, int io, float* o, int64_t n,
                                int d_k, int d_v, cudaStream_t st) {
  (void)d_v;
  return launch<false>(S, q, k, v, alpha, beta, io, o, n, d_k, st);
}

cudaError_t launch_gdn_step_bf16(uint16_t* S, const void* q, const void* k, const void* v,
                                 const void* alpha, const void* beta, int io, float* o, int64_t n,
                                 int d_k, int d_v, cudaStream_t st) {
  (void)d_v;
  return launch<true>(S, q, k, v, alpha, beta, io, o, n, d_k, st);
}

}  // namespace pace
