// Per-head decay statistics for choosing the 8-bit heads.
//
// "PACE: A New 4-Bit Recurrent State Quantization Method ...", paragraph on
// 8-bit precision for selected heads, and "PACE: four-bit recurrent state by
// rounding less often", TL;DR (3): heads whose errors persist -- long-memory
// heads -- are kept at 8 bits.  A head's memory length is set by its gate
// alpha (a write survives k tokens with weight prod alpha), so the statistic
// used here is the mean decay rate  r_h = mean over tokens and sequences of
// -ln(alpha): the smaller r_h, the longer the head remembers.
//
// The rates are accumulated in fp64: one thread per head reads a contiguous
// [rows][H] gate matrix row by row (coalesced across heads) and adds its
// partial sum with one fp64 atomic per block; a second launch divides by the
// number of rows.
#include "pace_internal.cuh"

namespace pace {

namespace {

__global__ void decay_rate_sum_kernel(const void* __restrict__ alpha, int64_t rows, int H, int io,
                                      double* __restrict__ sums) {
  const int h = threadIdx.x;
  if (h >= H) return;
  const int64_t per = (rows + gridDim.x - 1) / gridDim.x;
  const int64_t r0 = (int64_t)blockIdx.x * per;
  const int64_t r1 = r0 + per < rows ? r0 + per : rows;
  double acc = 0.0;
  for (int64_t r = r0; r < r1; ++r) acc += -log((double)load_io(alpha, r * H + h, io));
  if (r1 > r0) atomicAdd(&sums[h], acc);
}

__global__ void scale_kernel(double* __restrict__ v, int n, double f) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) v[i] *= f;
}

}  // namespace

cudaError_t launch_decay_rates(const void* alpha, int64_t rows, int H, int io, double* rates,
                               cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(rates, 0, sizeof(double) * (size_t)H, st);
  if (e != cudaSuccess || rows == 0) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (rows + 63) / 64;
  if (blocks > 4L * sms) blocks = 4L * sms;
  const int threads = (H + 31) / 32 * 32;
  decay_rate_sum_kernel<<<(unsigned)blocks, threads, 0, st>>>(alpha, rows, H, io, rates);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  scale_kernel<<<(H + 255) / 256, 256, 0, st>>>(rates, H, 1.0 / (double)rows);
  return cudaGetLastError();
}

}  // namespace pace
