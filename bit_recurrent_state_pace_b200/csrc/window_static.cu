// Allocation-free variant of the pure-write window step.
//
// pace_window_step needs device scratch for the E4M3-rounded k and v of one
// token, which the caller allocates.  Some callers cannot allocate device
// memory on their own: a plugin inside an inference engine whose memory
// manager owns the whole device budget and only hands out the tensors of a
// call's inputs and outputs, or a hot loop that must not call cudaMalloc
// (it can synchronise the device).  For them this file keeps the scratch in
// one file-scope device array that the module holds from load to exit, and
// pace_window_step_static passes that array to the same launches as
// pace_window_step.
//
// Host code cannot use the array's name as a device address (it is a
// host-side stand-in for the symbol): the address comes from
// cudaGetSymbolAddress, looked up once per device, with that device current,
// on the first call made on it.
#include <mutex>

#include "pace_internal.cuh"

// Every call on a device shares this array; it keeps the last call's
// contents.  Nothing in it has to start at zero: the rounding kernels
// overwrite the k and v halves completely before the decode reads them.
static __device__ __align__(256) uint8_t g_window_scratch[PACE_WINDOW_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

// Device address of g_window_scratch on the current device (looked up on the
// first call for that device), or an error.
cudaError_t scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_window_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" pace_status pace_window_step_static(pace_pool* pool, const void* q, const void* k,
                                               const void* v, const void* alpha, const void* beta,
                                               float* o, void* stream) {
  if (!pool) return PACE_ERR_INVALID_ARG;
  size_t need = 0;
  pace_status st = pace_window_scratch_bytes(pool, &need);
  if (st != PACE_OK) return st;
  if (need > (size_t)PACE_WINDOW_STATIC_SCRATCH_BYTES) return PACE_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return PACE_ERR_CUDA;
  }
  return pace_window_step(pool, q, k, v, alpha, beta, o, scratch, stream);
}
