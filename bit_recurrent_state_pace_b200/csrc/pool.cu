// Host side of the libpace C ABI: argument validation, pool layout, launches.
#include <new>
#include <string.h>

#include <cmath>

#include "commit_tc.cuh"
#include "pace_internal.cuh"
#include "tma.cuh"
#include "window.cuh"

struct pace_pool {
  pace::PoolDev dev;
  // tensor maps of the state region for the tensor-memory commit (d = 128)
  pace::CommitMaps maps;
  bool maps_ok = false;
  int32_t commit_engine = PACE_COMMIT_MMA;
  pace_pool_desc desc;
  size_t state_bytes, buffer_bytes, aux_bytes, kv_bytes;
  size_t rec_bytes[PACE_MAX_HEADS];
  // pace_decode_host: per staging slot, the event of its last output copy,
  // and the staging buffer they refer to
  cudaEvent_t host_done[2] = {nullptr, nullptr};
  const void* host_staging = nullptr;
};

namespace {

using pace::round_up;

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline pace_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return PACE_OK;
  (void)cudaGetLastError();  // clear a non-sticky error so later calls start clean
  return PACE_ERR_CUDA;
}

// Period commit of the heads due in a span, by the pool's commit engine.
inline cudaError_t commit_launch(const pace_pool* pool, const pace::PoolDev& dev, const pace::Span& sp,
                                 cudaStream_t st) {
  if (pool->commit_engine == PACE_COMMIT_TCGEN05 && pool->maps_ok && pace::commit_tc_supported(dev))
    return pace::launch_commit_tc(dev, sp, pool->maps, st);
  return pace::launch_commit(dev, sp, st);
}

inline bool mul_ok(size_t a, size_t b, size_t* out) {
  if (a != 0 && b > SIZE_MAX / a) return false;
  *out = a * b;
  return true;
}

struct Layout {
  size_t slot_stride;
  size_t rec_off[PACE_MAX_HEADS];
  size_t rec_bytes[PACE_MAX_HEADS];
  size_t state_bytes, kv_bytes, ab_bytes, buffer_bytes, aux_bytes;
  int n_groups;
};

pace_status check_desc(const pace_pool_desc* d) {
  if (!d) return PACE_ERR_INVALID_ARG;
  if (d->num_slots < 1 || d->num_heads < 1 || d->num_heads > PACE_MAX_HEADS) return PACE_ERR_INVALID_ARG;
  if (d->period < 1 || d->period > PACE_MAX_PERIOD) return PACE_ERR_INVALID_ARG;
  if (d->scale_axis != PACE_SCALE_COL && d->scale_axis != PACE_SCALE_ROW) return PACE_ERR_INVALID_ARG;
  if (d->io_dtype != PACE_IO_BF16 && d->io_dtype != PACE_IO_F32) return PACE_ERR_INVALID_ARG;
  if (!d->head_bits) return PACE_ERR_INVALID_ARG;
  for (int h = 0; h < d->num_heads; ++h)
    if (d->head_bits[h] != 4 && d->head_bits[h] != 8) return PACE_ERR_INVALID_ARG;
  if (d->d_k < 1 || d->d_v < 1) return PACE_ERR_INVALID_ARG;
  if (d->buffer_e4m3 != 0 && d->buffer_e4m3 != 1) return PACE_ERR_INVALID_ARG;
  if (d->d_k != d->d_v) return PACE_ERR_UNSUPPORTED;
  if (d->d_k != 32 && d->d_k != 64 && d->d_k != 128) return PACE_ERR_UNSUPPORTED;
  return PACE_OK;
}

pace_status compute_layout(const pace_pool_desc* d, Layout* L) {
  pace_status st = check_desc(d);
  if (st != PACE_OK) return st;
  L->n_groups = d->scale_axis == PACE_SCALE_COL ? d->d_k : d->d_v;
  size_t off = 0;
  for (int h = 0; h < d->num_heads; ++h) {
    L->rec_off[h] = off;
    L->rec_bytes[h] = pace::record_bytes(d->d_k, d->d_v, d->head_bits[h], L->n_groups);
    off += L->rec_bytes[h];
  }
  L->slot_stride = round_up(off, 16);
  if (!mul_ok(L->slot_stride, (size_t)d->num_slots, &L->state_bytes)) return PACE_ERR_INVALID_ARG;
  const size_t esz = d->buffer_e4m3 ? 1 : (size_t)pace::io_size(d->io_dtype);   // buffered k, v
  size_t heads = 0, rows = 0, kv = 0, ab = 0, gram = 0;
  if (!mul_ok((size_t)d->num_slots, (size_t)d->num_heads, &heads)) return PACE_ERR_INVALID_ARG;
  if (!mul_ok(heads, (size_t)d->period, &rows)) return PACE_ERR_INVALID_ARG;
  if (!mul_ok(rows, (size_t)(d->d_k + d->d_v) * esz, &kv)) return PACE_ERR_INVALID_ARG;
  if (!mul_ok(heads, pace::ab_stride_bytes(d->period, d->io_dtype), &ab)) return PACE_ERR_INVALID_ARG;
  if (!mul_ok(heads, pace::gram_stride_bytes(d->period), &gram)) return PACE_ERR_INVALID_ARG;
  L->kv_bytes = round_up(kv, 256);
  L->ab_bytes = round_up(ab, 256);
  L->buffer_bytes = L->kv_bytes + L->ab_bytes + round_up(gram, 256);
  L->aux_bytes = round_up(4 * heads, 256) + 256;
  if (heads > 0x7fffffffULL) return PACE_ERR_UNSUPPORTED;
  return PACE_OK;
}

}  // namespace

extern "C" {

const char* pace_status_string(pace_status s) {
  switch (s) {
    case PACE_OK: return "PACE_OK";
    case PACE_ERR_INVALID_ARG: return "PACE_ERR_INVALID_ARG";
    case PACE_ERR_UNSUPPORTED: return "PACE_ERR_UNSUPPORTED";
    case PACE_ERR_CUDA: return "PACE_ERR_CUDA";
    case PACE_ERR_DEVICE_FLAGS: return "PACE_ERR_DEVICE_FLAGS";
  }
  return "PACE_ERR_UNKNOWN";
}

const char* pace_version(void) { return "0.1.0"; }

pace_status pace_pool_bytes(const pace_pool_desc* desc, size_t* state_bytes, size_t* buffer_bytes,
                            size_t* aux_bytes) {
  if (!state_bytes || !buffer_bytes || !aux_bytes) return PACE_ERR_INVALID_ARG;
  Layout L;
  pace_status st = compute_layout(desc, &L);
  if (st != PACE_OK) return st;
  *state_bytes = L.state_bytes;
  *buffer_bytes = L.buffer_bytes;
  *aux_bytes = L.aux_bytes;
  return PACE_OK;
}

pace_status pace_init_pool(const pace_pool_desc* desc, void* d_state, void* d_buffer, void* d_aux,
                           void* stream, pace_pool** out) {
  if (!out) return PACE_ERR_INVALID_ARG;
  *out = nullptr;
  Layout L;
  pace_status st = compute_layout(desc, &L);
  if (st != PACE_OK) return st;
  if (!d_state || !d_buffer || !d_aux) return PACE_ERR_INVALID_ARG;
  if (!aligned(d_state, 256) || !aligned(d_buffer, 256) || !aligned(d_aux, 256)) return PACE_ERR_INVALID_ARG;
  pace_pool* p = new (std::nothrow) pace_pool;
  if (!p) return PACE_ERR_INVALID_ARG;
  memset(p, 0, sizeof(*p));
  p->desc = *desc;
  p->desc.head_bits = nullptr;
  p->state_bytes = L.state_bytes;
  p->buffer_bytes = L.buffer_bytes;
  p->aux_bytes = L.aux_bytes;
  p->kv_bytes = L.kv_bytes;
  pace::PoolDev& dv = p->dev;
  dv.B = desc->num_slots;
  dv.H = desc->num_heads;
  dv.d_k = desc->d_k;
  dv.d_v = desc->d_v;
  dv.P = desc->period;
  dv.axis = desc->scale_axis;
  dv.io = desc->io_dtype;
  dv.n_groups = L.n_groups;
  dv.slot_stride = L.slot_stride;
  dv.state = static_cast<uint8_t*>(d_state);
  dv.kv = static_cast<uint8_t*>(d_buffer);
  dv.ab = static_cast<uint8_t*>(d_buffer) + L.kv_bytes;
  dv.gram = static_cast<uint8_t*>(d_buffer) + L.kv_bytes + L.ab_bytes;
  dv.ab_stride = pace::ab_stride_bytes(desc->period, desc->io_dtype);
  dv.gram_stride = pace::gram_stride_bytes(desc->period);
  dv.fill = static_cast<int32_t*>(d_aux);
  dv.flags = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(d_aux) + L.aux_bytes - 256);
  {
    int n4 = 0;
    for (int h = 0; h < desc->num_heads; ++h)
      if (desc->head_bits[h] == 4) dv.order[n4++] = (uint8_t)h;
    dv.H4 = n4;
    for (int h = 0; h < desc->num_heads; ++h)
      if (desc->head_bits[h] != 4) dv.order[n4++] = (uint8_t)h;
  }
  dv.tau2 = INFINITY;
  dv.adaptive = 0;
  dv.row8 = desc->buffer_e4m3;
  dv.dbg_extra_tx = 0;
  dv.wait_limit_ns = pace::kWaitLimitNs;
  for (int h = 0; h < desc->num_heads; ++h) {
    dv.rec_off[h] = (uint32_t)L.rec_off[h];
    dv.bits[h] = desc->head_bits[h];
    p->rec_bytes[h] = L.rec_bytes[h];
  }
  // the tensor stores address a record by its first 64-byte row as a signed
  // 32-bit coordinate: a state region beyond 2^31 such rows (128 GiB) takes
  // the mma.sync commit
  if (desc->d_k == 128 && desc->d_v == 128 && L.state_bytes / 64 <= 0x7fffffffull)
    p->maps_ok = pace::make_commit_maps(dv.state, L.state_bytes, &p->maps);
  // the tensor-memory commit where it is built for the shape, else mma.sync
  p->commit_engine = p->maps_ok && pace::commit_tc_supported(dv) ? PACE_COMMIT_TCGEN05 : PACE_COMMIT_MMA;
  cudaError_t e = cudaMemsetAsync(d_aux, 0, L.aux_bytes, as_stream(stream));
  if (e != cudaSuccess) {
    delete p;
    return from_cuda(e);
  }
  *out = p;
  return PACE_OK;
}

void pace_destroy_pool(pace_pool* pool) {
  if (!pool) return;
  for (cudaEvent_t ev : pool->host_done)
    if (ev) cudaEventDestroy(ev);
  delete pool;
}

pace_status pace_pool_layout(const pace_pool* pool, int32_t head, size_t* record_offset,
                             size_t* record_bytes, size_t* slot_stride) {
  if (!pool || !record_offset || !record_bytes || !slot_stride) return PACE_ERR_INVALID_ARG;
  if (head < 0 || head >= pool->dev.H) return PACE_ERR_INVALID_ARG;
  *record_offset = pool->dev.rec_off[head];
  *record_bytes = pool->rec_bytes[head];
  *slot_stride = pool->dev.slot_stride;
  return PACE_OK;
}

pace_status pace_pool_load(pace_pool* pool, const float* S, void* stream) {
  if (!pool || !S || !aligned(S, 16)) return PACE_ERR_INVALID_ARG;
  return from_cuda(pace::launch_pool_load(pool->dev, S, as_stream(stream)));
}

pace_status pace_pool_export(pace_pool* pool, float* S, void* stream) {
  if (!pool || !S || !aligned(S, 16)) return PACE_ERR_INVALID_ARG;
  return from_cuda(pace::launch_pool_export(pool->dev, S, as_stream(stream)));
}

namespace {
bool span_ok(const pace_pool* pool, int32_t slot_begin, int32_t slot_count, int32_t blocks_per_sm) {
  return slot_begin >= 0 && slot_count >= 0 && (int64_t)slot_begin + slot_count <= pool->dev.B &&
         blocks_per_sm >= 0 && blocks_per_sm <= 8;
}
}  // namespace

pace_status pace_decode_step_range(pace_pool* pool, int32_t slot_begin, int32_t slot_count,
                                   int32_t blocks_per_sm, const void* q, const void* k,
                                   const void* v, const void* alpha, const void* beta, float* o,
                                   void* stream) {
  if (!pool || !q || !k || !v || !alpha || !beta || !o) return PACE_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16)) return PACE_ERR_INVALID_ARG;
  if (!aligned(alpha, 4) || !aligned(beta, 4)) return PACE_ERR_INVALID_ARG;
  if (!span_ok(pool, slot_begin, slot_count, blocks_per_sm)) return PACE_ERR_INVALID_ARG;
  const pace::Span sp{slot_begin, slot_count, blocks_per_sm};
  return from_cuda(pace::launch_decode_step(pool->dev, sp, q, k, v, alpha, beta, o, as_stream(stream)));
}

pace_status pace_decode_step(pace_pool* pool, const void* q, const void* k, const void* v,
                             const void* alpha, const void* beta, float* o, void* stream) {
  if (!pool) return PACE_ERR_INVALID_ARG;
  return pace_decode_step_range(pool, 0, pool->dev.B, 0, q, k, v, alpha, beta, o, stream);
}

pace_status pace_set_commit_threshold(pace_pool* pool, float tau) {
  if (!pool || !(tau >= 0.f)) return PACE_ERR_INVALID_ARG;   // NaN fails the comparison
  if (pool->dev.row8 && std::isfinite(tau)) return PACE_ERR_UNSUPPORTED;
  pool->dev.adaptive = std::isfinite(tau) ? 1 : 0;
  pool->dev.tau2 = pool->dev.adaptive ? tau * tau : INFINITY;
  return PACE_OK;
}

pace_status pace_set_commit_engine(pace_pool* pool, int32_t engine) {
  if (!pool || (engine != PACE_COMMIT_MMA && engine != PACE_COMMIT_TCGEN05)) return PACE_ERR_INVALID_ARG;
  if (engine == PACE_COMMIT_TCGEN05 && !(pool->maps_ok && pace::commit_tc_supported(pool->dev)))
    return PACE_ERR_UNSUPPORTED;
  pool->commit_engine = engine;
  return PACE_OK;
}

pace_status pace_debug_wait_fault(pace_pool* pool, uint64_t wait_limit_ns, uint32_t extra_tx_bytes) {
  if (!pool) return PACE_ERR_INVALID_ARG;
  if (extra_tx_bytes == 0 && wait_limit_ns == 0) {   // back to the defaults
    pool->dev.dbg_extra_tx = 0;
    pool->dev.wait_limit_ns = pace::kWaitLimitNs;
    return PACE_OK;
  }
  if (wait_limit_ns < 1000 || wait_limit_ns > pace::kWaitLimitNs || extra_tx_bytes > 16 ||
      (extra_tx_bytes & 15u) != 0)
    return PACE_ERR_INVALID_ARG;
  if (extra_tx_bytes > 0 && (wait_limit_ns > 10000000ull || pool->dev.B * pool->dev.H != 1))
    return PACE_ERR_INVALID_ARG;
  pool->dev.dbg_extra_tx = extra_tx_bytes;
  pool->dev.wait_limit_ns = wait_limit_ns;
  return PACE_OK;
}

pace_status pace_commit_period_range(pace_pool* pool, int32_t slot_begin, int32_t slot_count,
                                     int32_t blocks_per_sm, void* stream) {
  if (!pool || !span_ok(pool, slot_begin, slot_count, blocks_per_sm)) return PACE_ERR_INVALID_ARG;
  const pace::Span sp{slot_begin, slot_count, blocks_per_sm};
  return from_cuda(commit_launch(pool, pool->dev, sp, as_stream(stream)));
}

pace_status pace_prefill_range(pace_pool* pool, int32_t slot_begin, int32_t slot_count,
                               int64_t T, const void* q, const void* k, const void* v,
                               const void* alpha, const void* beta, float* o, void* stream) {
  if (!pool || T < 0 || (T > 0 && (!q || !k || !v || !alpha || !beta))) return PACE_ERR_INVALID_ARG;
  if (!span_ok(pool, slot_begin, slot_count, 0)) return PACE_ERR_INVALID_ARG;
  const size_t esz = pool->dev.io == PACE_IO_BF16 ? 2 : 4;
  if (!aligned(q, esz) || !aligned(k, esz) || !aligned(v, esz) || !aligned(alpha, esz) ||
      !aligned(beta, esz) || !aligned(o, 4))
    return PACE_ERR_INVALID_ARG;
  const pace::Span sp{slot_begin, slot_count, 0};
  return from_cuda(pace::launch_prefill(pool->dev, sp, T, q, k, v, alpha, beta, o, as_stream(stream)));
}

pace_status pace_prefill(pace_pool* pool, int64_t T, const void* q, const void* k, const void* v,
                         const void* alpha, const void* beta, float* o, void* stream) {
  if (!pool) return PACE_ERR_INVALID_ARG;
  return pace_prefill_range(pool, 0, pool->dev.B, T, q, k, v, alpha, beta, o, stream);
}

namespace {
struct HostSlot {   // byte offsets of one token's staging inside a slot
  size_t q, k, v, a, b, o, bytes;
};
HostSlot host_slot(const pace_pool* pool) {
  const size_t BH = (size_t)pool->dev.B * pool->dev.H;
  const size_t esz = pool->dev.io == PACE_IO_BF16 ? 2 : 4;
  HostSlot h;
  h.q = 0;
  h.k = round_up(BH * pool->dev.d_k * esz, 256);
  h.v = h.k + round_up(BH * pool->dev.d_k * esz, 256);
  h.a = h.v + round_up(BH * pool->dev.d_v * esz, 256);
  h.b = h.a + round_up(BH * esz, 256);
  h.o = h.b + round_up(BH * esz, 256);
  h.bytes = h.o + round_up(BH * pool->dev.d_v * 4, 256);
  return h;
}
}  // namespace

pace_status pace_host_staging_bytes(const pace_pool* pool, size_t* bytes) {
  if (!pool || !bytes) return PACE_ERR_INVALID_ARG;
  *bytes = 2 * host_slot(pool).bytes;
  return PACE_OK;
}

pace_status pace_decode_host(pace_pool* pool, int32_t n_tokens, const void* h_q, const void* h_k,
                             const void* h_v, const void* h_alpha, const void* h_beta, float* h_o,
                             void* d_staging, void* stream, void* h2d_stream, void* d2h_stream) {
  if (!pool || n_tokens < 0 || !d_staging || !aligned(d_staging, 256)) return PACE_ERR_INVALID_ARG;
  if (n_tokens > 0 && (!h_q || !h_k || !h_v || !h_alpha || !h_beta)) return PACE_ERR_INVALID_ARG;
  const HostSlot hs = host_slot(pool);
  const size_t BH = (size_t)pool->dev.B * pool->dev.H;
  const size_t esz = pool->dev.io == PACE_IO_BF16 ? 2 : 4;
  const size_t qb = BH * pool->dev.d_k * esz, vb = BH * pool->dev.d_v * esz, ab = BH * esz;
  const size_t ob = BH * pool->dev.d_v * 4;
  cudaStream_t cs = as_stream(stream), hs_in = as_stream(h2d_stream), hs_out = as_stream(d2h_stream);
  if (cs == hs_in || cs == hs_out || hs_in == hs_out) return PACE_ERR_INVALID_ARG;
  cudaError_t e = cudaSuccess;
  cudaEvent_t* done = pool->host_done;   // [slot]: its last output copy (persists across calls)
  for (int j = 0; j < 2 && e == cudaSuccess; ++j)
    if (!done[j]) e = cudaEventCreateWithFlags(&done[j], cudaEventDisableTiming);
  cudaEvent_t landed[2] = {nullptr, nullptr}, computed[2] = {nullptr, nullptr};
  for (int j = 0; j < 2 && e == cudaSuccess; ++j) {
    e = cudaEventCreateWithFlags(&landed[j], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&computed[j], cudaEventDisableTiming);
  }
  // The staging buffer of this pool's previous call is reused once each slot's
  // last output copy is done, so consecutive calls keep the copy engines busy.
  // A new buffer waits for all work already on `stream`.
  const bool reuse = pool->host_staging == d_staging;
  if (e == cudaSuccess && !reuse) {
    for (int j = 0; j < 2 && e == cudaSuccess; ++j) e = cudaEventRecord(done[j], cs);
    pool->host_staging = d_staging;
  }
  for (int t = 0; t < n_tokens && e == cudaSuccess; ++t) {
    const int sl = t & 1;
    uint8_t* base = static_cast<uint8_t*>(d_staging) + sl * hs.bytes;
    const uint8_t* hq = static_cast<const uint8_t*>(h_q) + (size_t)t * qb;
    const uint8_t* hk = static_cast<const uint8_t*>(h_k) + (size_t)t * qb;
    const uint8_t* hv = static_cast<const uint8_t*>(h_v) + (size_t)t * vb;
    const uint8_t* ha = static_cast<const uint8_t*>(h_alpha) + (size_t)t * ab;
    const uint8_t* hb = static_cast<const uint8_t*>(h_beta) + (size_t)t * ab;
    e = cudaStreamWaitEvent(hs_in, done[sl], 0);   // slot sl's previous token has been copied out
    if (e == cudaSuccess) e = cudaMemcpyAsync(base + hs.q, hq, qb, cudaMemcpyHostToDevice, hs_in);
    if (e == cudaSuccess) e = cudaMemcpyAsync(base + hs.k, hk, qb, cudaMemcpyHostToDevice, hs_in);
    if (e == cudaSuccess) e = cudaMemcpyAsync(base + hs.v, hv, vb, cudaMemcpyHostToDevice, hs_in);
    if (e == cudaSuccess) e = cudaMemcpyAsync(base + hs.a, ha, ab, cudaMemcpyHostToDevice, hs_in);
    if (e == cudaSuccess) e = cudaMemcpyAsync(base + hs.b, hb, ab, cudaMemcpyHostToDevice, hs_in);
    if (e == cudaSuccess) e = cudaEventRecord(landed[sl], hs_in);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, landed[sl], 0);
    if (e != cudaSuccess) break;
    const pace::Span all{0, pool->dev.B, 0};
    e = pace::launch_decode_step(pool->dev, all, base + hs.q, base + hs.k, base + hs.v, base + hs.a,
                                 base + hs.b, reinterpret_cast<float*>(base + hs.o), cs);
    if (e == cudaSuccess) e = commit_launch(pool, pool->dev, all, cs);   // heads whose buffer filled
    if (e == cudaSuccess) e = cudaEventRecord(computed[sl], cs);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(hs_out, computed[sl], 0);
    if (e == cudaSuccess && h_o)
      e = cudaMemcpyAsync(h_o + (size_t)t * BH * pool->dev.d_v, base + hs.o, ob, cudaMemcpyDeviceToHost, hs_out);
    if (e == cudaSuccess) e = cudaEventRecord(done[sl], hs_out);
  }
  // `stream` completes after the last output copy
  if (e == cudaSuccess && n_tokens > 0) e = cudaStreamWaitEvent(cs, done[(n_tokens - 1) & 1], 0);
  if (e != cudaSuccess) pool->host_staging = nullptr;   // next call orders on `stream` again
  for (int j = 0; j < 2; ++j) {
    if (landed[j]) cudaEventDestroy(landed[j]);
    if (computed[j]) cudaEventDestroy(computed[j]);
  }
  return from_cuda(e);
}

pace_status pace_window_scratch_bytes(const pace_pool* pool, size_t* bytes) {
  if (!pool || !bytes) return PACE_ERR_INVALID_ARG;
  const size_t BH = (size_t)pool->dev.B * pool->dev.H, esz = pool->dev.io == PACE_IO_BF16 ? 2 : 4;
  *bytes = round_up(BH * pool->dev.d_k * esz, 256) + round_up(BH * pool->dev.d_v * esz, 256);
  return PACE_OK;
}

pace_status pace_window_step(pace_pool* pool, const void* q, const void* k, const void* v,
                             const void* alpha, const void* beta, float* o, void* d_scratch,
                             void* stream) {
  if (!pool || !q || !k || !v || !alpha || !beta || !o || !d_scratch) return PACE_ERR_INVALID_ARG;
  if (!aligned(d_scratch, 256) || pool->dev.adaptive) return PACE_ERR_INVALID_ARG;
  const size_t BH = (size_t)pool->dev.B * pool->dev.H, esz = pool->dev.io == PACE_IO_BF16 ? 2 : 4;
  uint8_t* k8 = static_cast<uint8_t*>(d_scratch);
  uint8_t* v8 = k8 + round_up(BH * pool->dev.d_k * esz, 256);
  cudaStream_t st = as_stream(stream);
  const pace::Span all{0, pool->dev.B, 0};
  cudaError_t e = cudaSuccess;
  if (pool->dev.row8) {   // E4M3 rows: the decode rounds k and v as it buffers them
    e = pace::launch_decode_step(pool->dev, all, q, k, v, alpha, beta, o, st);
  } else {
    e = pace::launch_e4m3_round(k, k8, (int64_t)(BH * pool->dev.d_k), pool->dev.io, st);
    if (e == cudaSuccess) e = pace::launch_e4m3_round(v, v8, (int64_t)(BH * pool->dev.d_v), pool->dev.io, st);
    if (e == cudaSuccess) e = pace::launch_decode_step(pool->dev, all, q, k8, v8, alpha, beta, o, st);
  }
  if (e == cudaSuccess) e = pace::launch_window_prepare(pool->dev, st);
  if (e == cudaSuccess) {
    pace::PoolDev one = pool->dev;   // commits the marked heads with their own token count
    one.adaptive = 1;
    // one token per head: the mma.sync commit (measured 4.80 ms per window
    // step on the 4096 x 48 pool, against 4.95 ms with the tensor-memory one)
    e = pace::launch_commit(one, all, st);
  }
  if (e == cudaSuccess) e = pace::launch_window_shift(pool->dev, st);
  return from_cuda(e);
}

pace_status pace_commit_period(pace_pool* pool, void* stream) {
  if (!pool) return PACE_ERR_INVALID_ARG;
  return pace_commit_period_range(pool, 0, pool->dev.B, 0, stream);
}

pace_status pace_quantize(const float* S, int64_t n_mats, int32_t d_k, int32_t d_v, int32_t bits,
                          int32_t scale_axis, void* codes, uint16_t* scales, uint32_t* d_flags,
                          void* stream) {
  if (n_mats < 0 || n_mats > 0x7fffffffLL) return PACE_ERR_INVALID_ARG;
  if (d_k < 2 || d_v < 2 || d_k > 256 || d_v > 256 || (d_k & 1)) return PACE_ERR_INVALID_ARG;
  if (bits != 4 && bits != 8) return PACE_ERR_INVALID_ARG;
  if (scale_axis != PACE_SCALE_COL && scale_axis != PACE_SCALE_ROW) return PACE_ERR_INVALID_ARG;
  if (n_mats == 0) return PACE_OK;
  if (!S || !codes || !scales) return PACE_ERR_INVALID_ARG;
  return from_cuda(pace::launch_quantize(S, n_mats, d_k, d_v, bits, scale_axis,
                                         static_cast<uint8_t*>(codes), scales, d_flags,
                                         as_stream(stream)));
}

pace_status pace_dequantize(const void* codes, const uint16_t* scales, int64_t n_mats, int32_t d_k,
                            int32_t d_v, int32_t bits, int32_t scale_axis, float* S, void* stream) {
  if (n_mats < 0 || n_mats > 0x7fffffffLL) return PACE_ERR_INVALID_ARG;
  if (d_k < 2 || d_v < 2 || d_k > 256 || d_v > 256 || (d_k & 1)) return PACE_ERR_INVALID_ARG;
  if (bits != 4 && bits != 8) return PACE_ERR_INVALID_ARG;
  if (scale_axis != PACE_SCALE_COL && scale_axis != PACE_SCALE_ROW) return PACE_ERR_INVALID_ARG;
  if (n_mats == 0) return PACE_OK;
  if (!S || !codes || !scales) return PACE_ERR_INVALID_ARG;
  return from_cuda(pace::launch_dequantize(static_cast<const uint8_t*>(codes), scales, n_mats, d_k,
                                           d_v, bits, scale_axis, S, as_stream(stream)));
}

pace_status pace_pool_status(pace_pool* pool, void* stream, uint32_t* flags) {
  if (!pool || !flags) return PACE_ERR_INVALID_ARG;
  uint32_t host = 0;
  cudaError_t e = cudaMemcpyAsync(&host, pool->dev.flags, sizeof(host), cudaMemcpyDeviceToHost,
                                  as_stream(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return from_cuda(e);
  *flags = host;
  return host ? PACE_ERR_DEVICE_FLAGS : PACE_OK;
}

pace_status pace_pool_clear_status(pace_pool* pool, void* stream) {
  if (!pool) return PACE_ERR_INVALID_ARG;
  return from_cuda(cudaMemsetAsync(pool->dev.flags, 0, sizeof(uint32_t), as_stream(stream)));
}

static pace_status check_step_args(const void* S, const void* q, const void* k, const void* v,
                                   const void* alpha, const void* beta, int32_t io, int64_t n,
                                   int32_t d_k, int32_t d_v) {
  if (n < 0 || n > 0x7fffffffLL) return PACE_ERR_INVALID_ARG;
  if (io != PACE_IO_BF16 && io != PACE_IO_F32) return PACE_ERR_INVALID_ARG;
  if (d_k != d_v) return PACE_ERR_UNSUPPORTED;
  if (d_k != 32 && d_k != 64 && d_k != 128) return PACE_ERR_UNSUPPORTED;
  if (n > 0 && (!S || !q || !k || !v || !alpha || !beta)) return PACE_ERR_INVALID_ARG;
  return PACE_OK;
}

pace_status pace_gdn_step_f32(float* S, const void* q, const void* k, const void* v,
                              const void* alpha, const void* beta, int32_t io_dtype, float* o,
                              int64_t n, int32_t d_k, int32_t d_v, void* stream) {
  pace_status st = check_step_args(S, q, k, v, alpha, beta, io_dtype, n, d_k, d_v);
  if (st != PACE_OK) return st;
  return from_cuda(pace::launch_gdn_step_f32(S, q, k, v, alpha, beta, io_dtype, o, n, d_k, d_v,
                                             as_stream(stream)));
}

pace_status pace_gdn_step_bf16(uint16_t* S, const void* q, const void* k, const void* v,
                               const void* alpha, const void* beta, int32_t io_dtype, float* o,
                               int64_t n, int32_t d_k, int32_t d_v, void* stream) {
  pace_status st = check_step_args(S, q, k, v, alpha, beta, io_dtype, n, d_k, d_v);
  if (st != PACE_OK) return st;
  return from_cuda(pace::launch_gdn_step_bf16(S, q, k, v, alpha, beta, io_dtype, o, n, d_k, d_v,
                                              as_stream(stream)));
}

pace_status pace_decay_rates(const void* alpha, int64_t rows, int32_t num_heads, int32_t io_dtype,
                             double* rates, void* stream) {
  if (!alpha || !rates || rows < 0 || num_heads < 1 || num_heads > PACE_MAX_HEADS)
    return PACE_ERR_INVALID_ARG;
  if (io_dtype != PACE_IO_BF16 && io_dtype != PACE_IO_F32) return PACE_ERR_INVALID_ARG;
  if (!aligned(alpha, io_dtype == PACE_IO_BF16 ? 2 : 4) || !aligned(rates, 8)) return PACE_ERR_INVALID_ARG;
  return from_cuda(pace::launch_decay_rates(alpha, rows, num_heads, io_dtype, rates, as_stream(stream)));
}

pace_status pace_select_head_bits(const double* rates, int32_t num_heads, int32_t num_int8,
                                  uint8_t* head_bits) {
  if (!rates || !head_bits || num_heads < 1 || num_heads > PACE_MAX_HEADS || num_int8 < 0 ||
      num_int8 > num_heads)
    return PACE_ERR_INVALID_ARG;
  int order[PACE_MAX_HEADS];
  for (int h = 0; h < num_heads; ++h) order[h] = h;
  // slowest decay first; NaN rates last; ties by head index (stable)
  auto before = [&](int a, int b) {
    const double ra = rates[a], rb = rates[b];
    const bool na = ra != ra, nb = rb != rb;
    if (na != nb) return nb;
    if (!na && ra != rb) return ra < rb;
    return a < b;
  };
  for (int i = 1; i < num_heads; ++i) {   // insertion sort: H <= 256
    const int x = order[i];
    int j = i - 1;
    while (j >= 0 && before(x, order[j])) {
      order[j + 1] = order[j];
      --j;
    }
    order[j + 1] = x;
  }
  for (int h = 0; h < num_heads; ++h) head_bits[h] = 4;
  for (int i = 0; i < num_int8; ++i) head_bits[order[i]] = 8;
  return PACE_OK;
}

}  // extern "C"
