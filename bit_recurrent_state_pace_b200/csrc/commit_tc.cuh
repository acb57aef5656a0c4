// Launcher of the tensor-memory period commit (commit_tc_kernels.cu) and the
// TMA tensor maps it writes records through.
#pragma once

#include <cuda.h>

#include "pace_internal.cuh"

namespace pace {

// Two views of a pool's state region as rows of code bytes, for the commit's
// tensor stores: INT4 records (64-byte rows, 64-byte swizzle) and INT8
// records (128-byte rows, 128-byte swizzle).  Box: one record's 128 code rows.
struct alignas(64) CommitMaps {
  CUtensorMap codes4;
  CUtensorMap codes8;
};

// The pool shapes the tensor-memory commit is built for: d_k = d_v = 128,
// column scales, and (for fp32 buffered rows) P <= 8.
bool commit_tc_supported(const PoolDev& p);

// Encode the two maps over [state, state + state_bytes); false if the driver
// call is unavailable or refuses the layout.
bool make_commit_maps(uint8_t* state, size_t state_bytes, CommitMaps* maps);

cudaError_t launch_commit_tc(const PoolDev& p, const Span& sp, const CommitMaps& maps, cudaStream_t st);

}  // namespace pace
