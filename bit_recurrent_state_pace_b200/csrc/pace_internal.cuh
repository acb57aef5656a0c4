// Internal declarations shared by the libpace CUDA sources.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>
#include <stddef.h>

#include "../../include/pace.h"

#define PACE_MAX_HEADS 256
#define PACE_MAX_PERIOD 16
#define PACE_MAX_D 128

namespace pace {

// Everything a pool kernel needs, passed by value as a kernel parameter.
struct PoolDev {
  int32_t B, H, d_k, d_v, P, axis, io;
  int32_t n_groups;           // scale groups per head: d_k (COL) or d_v (ROW)
  uint64_t slot_stride;       // bytes per slot in the state region
  uint8_t* state;             // [B][slot_stride]
  uint8_t* kv;                // [B][H][P][d_k + d_v] io elements
  uint8_t* ab;                // [B][H] blocks of ab_stride bytes: [P][2] io elements
  uint8_t* gram;              // [B][H] blocks of gram_stride bytes: [P][P] + [P] + [2] fp32
  uint32_t ab_stride;         // round_up(2 P io bytes, 16)
  uint32_t gram_stride;       // round_up(4 (P (P + 1) + 2), 16)
  int32_t* fill;              // [B][H]
  uint32_t* flags;            // status word
  uint32_t rec_off[PACE_MAX_HEADS];   // record offset of head h inside a slot
  uint8_t bits[PACE_MAX_HEADS];       // 4 or 8
  uint8_t order[PACE_MAX_HEADS];      // head indices, the 4-bit heads first
  int32_t H4;                         // number of 4-bit heads
  float tau2;                         // commit threshold squared (+inf: fixed period)
  int32_t adaptive;                   // tau2 finite
  int32_t row8;                       // buffered k, v rows are E4M3 bytes
  uint32_t dbg_extra_tx;              // 0; > 0 only under pace_debug_wait_fault
  uint64_t wait_limit_ns;             // bound of the decode's mbarrier waits
};

// Bytes per buffered k or v element.
__host__ __device__ inline int row_esz(const PoolDev& p) { return p.row8 ? 1 : (p.io == PACE_IO_BF16 ? 2 : 4); }

// A head's buffer is due for a commit: full, or marked by the decode step
// (which marks only heads holding at least one token).
__host__ __device__ inline bool commit_due(int32_t fill, int32_t P) {
  return fill == P || ((fill & PACE_FILL_COMMIT) != 0 && (fill & 0xff) > 0);
}

// The slots a launch works on, and how many blocks per SM it may occupy
// (fewer than the default leaves room for a launch on another stream).
struct Span {
  int32_t b0, nb;            // slots [b0, b0 + nb)
  int32_t blocks_per_sm;     // 0: the kernel's default
};

// The i-th (slot, head) of span slots [b0, b0 + nb) in work order: all 4-bit
// heads of every slot, then all 8-bit ones, so that the warps of a launch run
// one code path at a time.
__device__ __forceinline__ int head_in_order(const PoolDev& p, int i, int b0, int nb) {
  const int n4 = nb * p.H4;
  if (i < n4) {
    const int b = i / p.H4;
    return (b0 + b) * p.H + p.order[i - b * p.H4];
  }
  const int h8 = p.H - p.H4, j = i - n4, b = j / h8;
  return (b0 + b) * p.H + p.order[p.H4 + j - b * h8];
}

__host__ __device__ inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline size_t code_bytes(int d_k, int d_v, int bits) {
  return (size_t)d_v * (size_t)d_k * (size_t)bits / 8;
}

__host__ __device__ inline size_t record_bytes(int d_k, int d_v, int bits, int n_groups) {
  return round_up(code_bytes(d_k, d_v, bits) + 2 * (size_t)n_groups, 16);
}

__host__ __device__ inline int io_size(int io) { return io == PACE_IO_BF16 ? 2 : 4; }

__host__ __device__ inline uint32_t ab_stride_bytes(int P, int io) {
  return (uint32_t)round_up((size_t)2 * P * io_size(io), 16);
}

__host__ __device__ inline uint32_t gram_stride_bytes(int P) {
  return (uint32_t)round_up((size_t)4 * (P * (P + 1) + 2), 16);
}

// Load element `idx` of an io-dtype array as fp32.
__device__ __forceinline__ float load_io(const void* p, size_t idx, int io) {
  if (io == PACE_IO_BF16) {
    uint16_t b = reinterpret_cast<const uint16_t*>(p)[idx];
    return __uint_as_float(((uint32_t)b) << 16);
  }
  return reinterpret_cast<const float*>(p)[idx];
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}

__device__ __forceinline__ uint16_t float_to_bf16_bits_rn(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// Host-side launchers (defined in the .cu files, called by pool.cu).
cudaError_t launch_quantize(const float* S, int64_t n, int d_k, int d_v, int bits, int axis,
                            uint8_t* codes, uint16_t* scales, uint32_t* flags, cudaStream_t st);
cudaError_t launch_dequantize(const uint8_t* codes, const uint16_t* scales, int64_t n, int d_k,
                              int d_v, int bits, int axis, float* S, cudaStream_t st);
cudaError_t launch_pool_load(const PoolDev& p, const float* S, cudaStream_t st);
cudaError_t launch_pool_export(const PoolDev& p, float* S, cudaStream_t st);
cudaError_t launch_decode_step(const PoolDev& p, const Span& sp, const void* q, const void* k,
                               const void* v, const void* alpha, const void* beta, float* o,
                               cudaStream_t st);
cudaError_t launch_commit(const PoolDev& p, const Span& sp, cudaStream_t st);
cudaError_t launch_prefill(const PoolDev& p, const Span& sp, int64_t T, const void* q,
                           const void* k, const void* v, const void* alpha, const void* beta,
                           float* o, cudaStream_t st);
cudaError_t launch_decay_rates(const void* alpha, int64_t rows, int H, int io, double* rates,
                               cudaStream_t st);
cudaError_t launch_gdn_step_f32(float* S, const void* q, const void* k, const void* v,
                                const void* alpha, const void* beta, int io, float* o, int64_t n,
                                int d_k, int d_v, cudaStream_t st);
cudaError_t launch_gdn_step_bf16(uint16_t* S, const void* q, const void* k, const void* v,
                                 const void* alpha, const void* beta, int io, float* o, int64_t n,
                                 int d_k, int d_v, cudaStream_t st);

}  // namespace pace
