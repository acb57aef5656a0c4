// Launchers of the pure-write window kernels (window_kernels.cu), used by the
// host ABI in pool.cu.
#pragma once

#include "pace_internal.cuh"

namespace pace {

// dst = E4M3(src) element-wise, n elements of the io dtype (stored back in it).
cudaError_t launch_e4m3_round(const void* src, void* dst, int64_t n, int io, cudaStream_t st);
// Heads whose window holds P pairs: one-token commit factors of the oldest pair, fill = 1 | commit mark.
cudaError_t launch_window_prepare(const PoolDev& p, cudaStream_t st);
// Heads merged by the commit (fill 0): drop the merged row, fill = P - 1.
cudaError_t launch_window_shift(const PoolDev& p, cudaStream_t st);

}  // namespace pace
