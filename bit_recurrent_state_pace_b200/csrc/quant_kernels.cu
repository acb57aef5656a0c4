// Encode / decode kernels: pace_quantize, pace_dequantize, pool load/export.
#include "encode.cuh"

namespace pace {

namespace {

constexpr int kEncThreads = 128;

struct GlobalGet {
  const float* S;
  int d_k;
  __device__ __forceinline__ float operator()(int i, int j) const { return S[(size_t)i * d_k + j]; }
};

__global__ void __launch_bounds__(kEncThreads) quantize_kernel(const float* __restrict__ S,
                                                               int d_k, int d_v, int bits, int axis,
                                                               uint8_t* __restrict__ codes,
                                                               uint16_t* __restrict__ scales,
                                                               uint32_t* flags) {
  __shared__ float sf_sm[256];
  const size_t m = blockIdx.x;
  const int ng = axis == PACE_SCALE_COL ? d_k : d_v;
  GlobalGet get{S + m * (size_t)d_v * d_k, d_k};
  encode_matrix(get, d_k, d_v, bits, axis, codes + m * code_bytes(d_k, d_v, bits),
                scales + m * (size_t)ng, flags, sf_sm);
}

__global__ void dequantize_kernel(const uint8_t* __restrict__ codes,
                                  const uint16_t* __restrict__ scales, int d_k, int d_v, int bits,
                                  int axis, float* __restrict__ S) {
  const size_t m = blockIdx.x;
  const int ng = axis == PACE_SCALE_COL ? d_k : d_v;
  const uint8_t* c = codes + m * code_bytes(d_k, d_v, bits);
  const uint16_t* s = scales + m * (size_t)ng;
  float* out = S + m * (size_t)d_v * d_k;
  const int row_bytes = d_k * bits / 8;
  for (int idx = threadIdx.x; idx < d_v * d_k; idx += blockDim.x) {
    const int i = idx / d_k, j = idx - i * d_k;
    const float sf = __half2float(__ushort_as_half(s[axis == PACE_SCALE_COL ? j : i]));
    out[idx] = (float)decode_code(c, row_bytes, i, j, bits) * sf;
  }
}

__global__ void __launch_bounds__(kEncThreads) pool_load_kernel(PoolDev p, const float* __restrict__ S) {
  __shared__ float sf_sm[256];
  const int b = blockIdx.x / p.H, h = blockIdx.x - (blockIdx.x / p.H) * p.H;
  const int bits = p.bits[h];
  uint8_t* rec = p.state + (size_t)b * p.slot_stride + p.rec_off[h];
  uint16_t* sc = reinterpret_cast<uint16_t*>(rec + code_bytes(p.d_k, p.d_v, bits));
  GlobalGet get{S + (size_t)blockIdx.x * p.d_v * p.d_k, p.d_k};
  encode_matrix(get, p.d_k, p.d_v, bits, p.axis, rec, sc, p.flags, sf_sm);
  if (threadIdx.x == 0) p.fill[blockIdx.x] = 0;
}

__global__ void pool_export_kernel(PoolDev p, float* __restrict__ S) {
  const int b = blockIdx.x / p.H, h = blockIdx.x - (blockIdx.x / p.H) * p.H;
  const int bits = p.bits[h];
  const uint8_t* rec = p.state + (size_t)b * p.slot_stride + p.rec_off[h];
  const uint16_t* sc = reinterpret_cast<const uint16_t*>(rec + code_bytes(p.d_k, p.d_v, bits));
  float* out = S + (size_t)blockIdx.x * p.d_v * p.d_k;
  const int row_bytes = p.d_k * bits / 8;
  for (int idx = threadIdx.x; idx < p.d_v * p.d_k; idx += blockDim.x) {
    const int i = idx / p.d_k, j = idx - i * p.d_k;
    const float sf = __half2float(__ushort_as_half(sc[p.axis == PACE_SCALE_COL ? j : i]));
    out[idx] = (float)decode_code(rec, row_bytes, i, j, bits) * sf;
  }
}

}  // namespace

cudaError_t launch_quantize(const float* S, int64_t n, int d_k, int d_v, int bits, int axis,
                            uint8_t* codes, uint16_t* scales, uint32_t* flags, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  quantize_kernel<<<(unsigned)n, kEncThreads, 0, st>>>(S, d_k, d_v, bits, axis, codes, scales, flags);
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t* codes, const uint16_t* scales, int64_t n, int d_k,
                              int d_v, int bits, int axis, float* S, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  dequantize_kernel<<<(unsigned)n, 256, 0, st>>>(codes, scales, d_k, d_v, bits, axis, S);
  return cudaGetLastError();
}

cudaError_t launch_pool_load(const PoolDev& p, const float* S, cudaStream_t st) {
  pool_load_kernel<<<(unsigned)(p.B * p.H), kEncThreads, 0, st>>>(p, S);
  return cudaGetLastError();
}

cudaError_t launch_pool_export(const PoolDev& p, float* S, cudaStream_t st) {
  pool_export_kernel<<<(unsigned)(p.B * p.H), 256, 0, st>>>(p, S);
  return cudaGetLastError();
}

}  // namespace pace
