/*
 * pace.h -- C ABI of libpace: batched decode of a Gated DeltaNet linear-
 * attention layer whose per-sequence recurrent state is stored as INT4 (or
 * INT8 for chosen heads) with channel-aligned FP16 scales, rounded once per
 * period of P tokens (PACE).
 *
 * Sources (page title, section):
 *  [P2] "PACE: A New 4-Bit Recurrent State Quantization Method That Makes
 *       Linear Attention Models More Memory-Efficient"
 *  [P3] "低比特量化新突破：GGA+PW让线性注意力长文本生成更准更短"
 *  [P4] "PACE: four-bit recurrent state by rounding less often"
 *
 * Conventions for every call:
 *  - All tensors live in device memory allocated and owned by the caller
 *    (e.g. by PyTorch); the library keeps pointers only, never allocates
 *    device memory, and never frees caller memory.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Every call is asynchronous on that stream unless it says it
 *    synchronises.
 *  - Every call returns pace_status and never throws or aborts.  Argument
 *    errors are detected on the host before any launch.  Conditions seen
 *    on the device (non-finite values, a decode into a full buffer, a
 *    bounded wait that gave up) set bits of the pool's device status word,
 *    read with pace_pool_status().
 *  - State matrices are S in R^{d_v x d_k}, stored row-major (row i = value
 *    channel, column j = key channel), the state of the rule
 *      S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T,  o_t = S_t q_t
 *    (reading of the gate + delta rule described in [P3], section
 *    "为什么低比特状态量化会“越写越错”").
 */
#ifndef PACE_H_
#define PACE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PACE_OK = 0,
  PACE_ERR_INVALID_ARG = 1,  /* null pointer, bad size, bad enum, misaligned pointer */
  PACE_ERR_UNSUPPORTED = 2,  /* a shape the kernels are not built for */
  PACE_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
  PACE_ERR_DEVICE_FLAGS = 4  /* pace_pool_status found device status bits set */
} pace_status;

/* Device status bits (pace_pool_status, pace_quantize's d_flags). */
#define PACE_FLAG_NONFINITE      0x1u  /* a scale group held a NaN/Inf: scale NaN, codes 0 */
#define PACE_FLAG_SCALE_OVERFLOW 0x2u  /* amax/qmax exceeded fp16: scale clamped to 65504 */
#define PACE_FLAG_BUFFER_FULL    0x4u  /* decode into a head whose buffer held P tokens:
                                          that head's output row is NaN, nothing stored */
#define PACE_FLAG_TIMEOUT        0x8u  /* a bounded wait inside a kernel gave up */

/* Fill-counter bit: the head's accumulated update reached the pool's commit
 * threshold (pace_set_commit_threshold) before its buffer filled; the low
 * bits still count its buffered tokens. */
#define PACE_FILL_COMMIT 0x100

/* Scale axis ([P2] "Channel-Aligned Encoding"; [P4] TL;DR (2)).
 * COL: one scale per key channel j, shared by the d_v entries S[:, j].
 * ROW: one scale per value channel i, shared by the d_k entries S[i, :]. */
typedef enum { PACE_SCALE_COL = 0, PACE_SCALE_ROW = 1 } pace_scale_axis;

/* Element type of q, k, v, alpha, beta and of the token buffer. */
typedef enum { PACE_IO_BF16 = 0, PACE_IO_F32 = 1 } pace_io_dtype;

typedef struct pace_pool pace_pool;  /* opaque, host-side */

typedef struct {
  int32_t num_slots;          /* B: sequences decoded together (>= 1) */
  int32_t num_heads;          /* H: value heads (1..256) */
  int32_t d_k, d_v;           /* head dims; supported: d_k == d_v in {32, 64, 128} */
  int32_t period;             /* P: tokens per rounding period, 1..16 */
  int32_t scale_axis;         /* pace_scale_axis */
  int32_t io_dtype;           /* pace_io_dtype */
  const uint8_t* head_bits;   /* host array [num_heads], each 4 or 8 ([P4] TL;DR (3)) */
  int32_t buffer_e4m3;        /* 0: buffered k, v in io_dtype; 1: as FP8 E4M3 bytes (the
                                 pure-write window's pairs, see pace_window_step) */
} pace_pool_desc;

/*
 * Memory a pool needs, in bytes (host-only query, no CUDA call).
 *
 * state  : B slots of `slot_stride` bytes.  Slot b holds every head's record
 *          at the offset pace_pool_layout() reports.  A record is the codes,
 *          d_v rows of d_k*bits/8 bytes (INT8: two's complement bytes; INT4:
 *          two codes per byte, the even key index j in the low nibble, each
 *          nibble the 4-bit two's complement of a code in [-7, 7]), followed
 *          by the head's FP16 scales (d_k of them for COL, d_v for ROW), the
 *          record padded to 16 bytes.
 * buffer : the token buffer ([P2] "Periodic Rounding"; [P4] flowchart "Small
 *          buffer, last few tokens"): region KV = [B][H][P][d_k + d_v]
 *          io_dtype elements (row = k then v of one buffered token; one E4M3
 *          byte per element when buffer_e4m3 is set, the token's k and v then
 *          rounded to E4M3 as they are buffered and used), then at
 *          byte offset round_up(size(KV), 256) region AB: [B][H] blocks of
 *          round_up(2*P*io_size, 16) bytes, each [P][2] io_dtype elements
 *          (alpha, beta); then at the next 256-byte boundary region G: [B][H]
 *          blocks of round_up(4*(P*(P+1)+2), 16) bytes, each [P][P] + [P]
 *          + [2] fp32.  While a period fills, G[t][s] = k_t . k_s for s < t,
 *          the Gram entries of the buffered keys, written by the decode step
 *          that buffers token t (so each step computes only its own).  The
 *          step that buffers the P-th token replaces them with the period's
 *          chunk-form factors for the commit: W[s][s'] = gamma_{P/s}
 *          T[s][s'] beta_s' with T = (I + A)^{-1}, then the P decay products
 *          gamma_s, then max |k_s[j]| over the period's keys and the largest
 *          stored scale of the head.  q is not stored: no later step reads
 *          an old query.  With a commit threshold set, float P*P + P of the
 *          block holds, while the period fills, the squared norm of the
 *          accumulated update, and the factors above are written for the n
 *          buffered tokens by the step that marks the head (zero beyond n).
 * aux    : fill counters int32 [B][H] (tokens in each head's buffer, plus
 *          PACE_FILL_COMMIT when the head is due early), then at
 *          byte offset round_up(4*B*H, 256) the uint32 status word.
 * All three regions must be 256-byte aligned.
 */
pace_status pace_pool_bytes(const pace_pool_desc* desc, size_t* state_bytes,
                            size_t* buffer_bytes, size_t* aux_bytes);

/*
 * Bind caller-owned device regions to a new pool: the per-request state pool
 * whose size sets how many sequences can be served ([P4] TL;DR: 4-bit states
 * fit about four times the concurrency of FP16 ones; [P2] "Periodic
 * Rounding": the state, its small token buffer and the per-period factors).
 * Copies the descriptor
 * (head_bits included), computes the record layout, and zeroes aux (all
 * buffers empty, status clear) with cudaMemsetAsync on `stream`.  The state
 * contents are the caller's (fill them with pace_pool_load or by writing
 * records directly).  The regions must outlive the pool.
 */
pace_status pace_init_pool(const pace_pool_desc* desc, void* d_state, void* d_buffer,
                           void* d_aux, void* stream, pace_pool** out);

/* Release the host-side pool object (caller memory is untouched). NULL is a no-op. */
void pace_destroy_pool(pace_pool* pool);

/* Byte offset of head h's record inside a slot, its size, and the slot stride. */
pace_status pace_pool_layout(const pace_pool* pool, int32_t head, size_t* record_offset,
                             size_t* record_bytes, size_t* slot_stride);

/*
 * Encode S (device fp32 [B][H][d_v][d_k]) into every head's record with that
 * head's bit width, and empty every buffer (fill = 0).  Same encoding as
 * pace_quantize.
 */
pace_status pace_pool_load(pace_pool* pool, const float* S, void* stream);

/* Decode every stored state to S (device fp32 [B][H][d_v][d_k]); buffered
 * tokens are not applied. */
pace_status pace_pool_export(pace_pool* pool, float* S, void* stream);

/*
 * One decode token for every head of every slot ([P2] "Periodic Rounding":
 * tokens wait in a small buffer and the state is not rounded).
 * q, k: [B][H][d_k]; v: [B][H][d_v]; alpha, beta: [B][H]; all io_dtype.
 * o: fp32 [B][H][d_v].
 * For each head with n-1 buffered tokens (n <= P): appends the token as row
 * n-1 of the head's buffer and writes o_n = S_n q_n exactly in chunk form
 * from the stored state S~0 (the decayed stored state applied to q_n plus
 * the delta-rule correction of the n buffered tokens, fp32 accumulation),
 * then sets fill = n.  The stored state is not modified.  A head whose buffer
 * already holds P tokens is skipped (o row NaN, PACE_FLAG_BUFFER_FULL): call
 * pace_commit_period after the step that fills the buffer.
 */
pace_status pace_decode_step(pace_pool* pool, const void* q, const void* k, const void* v,
                             const void* alpha, const void* beta, float* o, void* stream);

/*
 * Adaptive period ([P4] "Research angle": round when the accumulated update
 * norm crosses a threshold rather than every k tokens).  With tau set, the
 * decode step also tracks, for each head, the Frobenius norm of the update
 * accumulated since the last rounding,
 *   Delta_n = S_n - gamma_n S~0 = sum_s gamma_{n/s} u_s k_s^T
 * (the writes; the decay alone needs no re-encoding), by the recursion
 *   |Delta_n|^2 = alpha_n^2 |Delta_{n-1}|^2 + 2 alpha_n u_n . (Delta_{n-1} k_n)
 *                 + |u_n|^2 |k_n|^2,   u_n = beta_n (v_n - alpha_n S_{n-1} k_n),
 * whose vectors come from the same pass over the stored codes as o_n
 * (fp32; decisions within rounding of the threshold may go either way).
 * When |Delta_n| >= tau and n < P the step marks the head (fill = n |
 * PACE_FILL_COMMIT); pace_commit_period then commits it with its n tokens,
 * and a decode step on a marked head is skipped like one on a full buffer.
 * tau = +inf (the default) is the fixed period P; tau = 0 commits after
 * every token.  A negative or NaN tau is PACE_ERR_INVALID_ARG; a finite tau
 * on a pool with buffer_e4m3 set is PACE_ERR_UNSUPPORTED.  Host-only:
 * applies to launches enqueued after the call.
 */
pace_status pace_set_commit_threshold(pace_pool* pool, float tau);

/*
 * Period end ([P4] flowchart "every k tokens -> State update, chunked, high
 * precision -> 4-bit encode, per-column scales"; 8-bit heads from TL;DR (3)).
 * For every head whose buffer holds P tokens (or is marked PACE_FILL_COMMIT
 * with n tokens): dequantise the stored state,
 * apply the P buffered tokens in one chunked (UT/WY) update in fp32, encode
 * the result with fresh absmax scales at the head's bit width, write it back
 * in place, and empty the buffer.  Heads with fewer than P tokens are left
 * untouched, so slots may run at different phases.
 */
pace_status pace_commit_period(pace_pool* pool, void* stream);

/*
 * Which kernel applies the period commit (same results: both encode the
 * fp32 update of the page's chunked, high-precision period end, see
 * pace_commit_period; codes may differ only at exact rounding ties).
 *  PACE_COMMIT_MMA: warp-level tensor-core products (mma.sync) with the
 *    update and the encode in registers; every pool shape.
 *  PACE_COMMIT_TCGEN05: fifth-generation tensor cores with the update in
 *    tensor memory and the records written back by TMA stores; pools with
 *    d_k = d_v = 128 and column scales (fp32 io only with P <= 8) whose
 *    state region is at most 128 GiB, else PACE_ERR_UNSUPPORTED.
 * A new pool starts with PACE_COMMIT_TCGEN05 where that engine is built for
 * its shape, else PACE_COMMIT_MMA.
 * Host-only; applies to launches enqueued after the call.  Any other value
 * is PACE_ERR_INVALID_ARG.
 */
typedef enum { PACE_COMMIT_MMA = 0, PACE_COMMIT_TCGEN05 = 1 } pace_commit_engine;
pace_status pace_set_commit_engine(pace_pool* pool, int32_t engine);

/*
 * The same two operations restricted to slots [slot_begin, slot_begin +
 * slot_count) (0 <= slot_begin, slot_begin + slot_count <= num_slots).  q, k,
 * v, alpha, beta and o keep the full-pool layout; only the rows of the range
 * are read or written.  blocks_per_sm bounds how many blocks of the launch
 * each SM may hold (0 = the kernel's default, at most 8): launches on two
 * streams that each take part of every SM run side by side, which is how
 * slots at different phases overlap one group's period commit (arithmetic-
 * bound) with the other slots' decode (memory-bound).  Launches on different
 * streams must cover disjoint slot ranges.  PACE_ERR_INVALID_ARG for a range
 * or blocks_per_sm out of bounds.  This scheduling hook has no counterpart on
 * the pages; it serves continuous batching, where requests start at
 * different steps.
 */
pace_status pace_decode_step_range(pace_pool* pool, int32_t slot_begin, int32_t slot_count,
                                   int32_t blocks_per_sm, const void* q, const void* k,
                                   const void* v, const void* alpha, const void* beta, float* o,
                                   void* stream);
pace_status pace_commit_period_range(pace_pool* pool, int32_t slot_begin, int32_t slot_count,
                                     int32_t blocks_per_sm, void* stream);

/*
 * Encode n_mats fp32 matrices S [n_mats][d_v][d_k] (device) with one FP16
 * scale per group ([P2] "Channel-Aligned Encoding"):
 *   amax = max|x| (group); s32 = amax/qmax (fp32 divide, round to nearest);
 *   s16 = fp16_rn(s32), raised to 2^-24 if amax > 0 and s16 == 0, clamped to
 *   65504 (+ PACE_FLAG_SCALE_OVERFLOW) if it overflows;
 *   code = clamp(rint_half_even(x / float(s16)), -qmax, qmax), fp32 divide;
 *   all codes 0 if s16 == 0; a group holding NaN/Inf gets scale NaN (0x7E00),
 *   codes 0 and PACE_FLAG_NONFINITE.
 * qmax = 7 (bits 4) or 127 (bits 8).
 * codes: [n_mats][d_v][d_k*bits/8] bytes, packed as in a pool record.
 * scales: fp16 bits [n_mats][d_k] (COL) or [n_mats][d_v] (ROW).
 * d_flags: optional device uint32 that receives the status bits (atomic OR).
 * d_k, d_v: even, 2..256.
 */
pace_status pace_quantize(const float* S, int64_t n_mats, int32_t d_k, int32_t d_v,
                          int32_t bits, int32_t scale_axis, void* codes, uint16_t* scales,
                          uint32_t* d_flags, void* stream);

/* Inverse of pace_quantize ([P2] "Channel-Aligned Encoding": each state entry
 * is its code times its channel's scale): S = float(code) * float(scale),
 * exact in fp32. */
pace_status pace_dequantize(const void* codes, const uint16_t* scales, int64_t n_mats,
                            int32_t d_k, int32_t d_v, int32_t bits, int32_t scale_axis,
                            float* S, void* stream);

/* The conditions the kernels detect on the device are kept as bits of one
 * status word (the encoder's non-finite and clamped groups of [P2]
 * "Channel-Aligned Encoding", a decode into a full buffer of [P2] "Periodic
 * Rounding", a bounded wait that gave up).
 * Synchronise `stream`, then read the pool's device status word into *flags.
 * Returns PACE_ERR_DEVICE_FLAGS if any bit is set, PACE_OK otherwise. */
pace_status pace_pool_status(pace_pool* pool, void* stream, uint32_t* flags);

/* Clear the device status word (async on `stream`). */
pace_status pace_pool_clear_status(pace_pool* pool, void* stream);

/*
 * Debug only: exercise the bounded waits of pace_decode_step.  No passage of
 * the pages corresponds; it tests the failure detection of the status word
 * (PACE_FLAG_TIMEOUT).  The decode stages each head's inputs with bulk
 * copies that complete on an mbarrier, and its warps wait for that barrier
 * for at most a fixed time (2 s by default) before giving up.
 *  wait_limit_ns:   that bound, 1000 .. 2e9 ns.
 *  extra_tx_bytes:  0 or 16.  With 16, every stage's barrier expects 16
 *    bytes more than its copies bring: every copy still lands (nothing is
 *    left in flight), the barrier never completes, each warp's wait runs
 *    out after wait_limit_ns, the head's output row is NaN, nothing is
 *    buffered, and PACE_FLAG_TIMEOUT is set.  Allowed only on a pool of
 *    one head (B = H = 1) with wait_limit_ns <= 1e7.
 * (0, 0) restores the defaults.  Out-of-range values are
 * PACE_ERR_INVALID_ARG and change nothing.  Host-only; applies to launches
 * enqueued after the call.
 */
pace_status pace_debug_wait_fault(pace_pool* pool, uint64_t wait_limit_ns, uint32_t extra_tx_bytes);

/*
 * Unquantised comparison paths (not PACE; used for the fp32 warm-up prefill,
 * the drift reference trajectory and the bf16-state throughput comparison).
 * One token of the rule above for n independent heads, state updated in
 * place: S [n][d_v][d_k] fp32 (pace_gdn_step_f32) or bf16 bits
 * (pace_gdn_step_bf16); q, k [n][d_k], v [n][d_v], alpha, beta [n] in
 * io_dtype; o: fp32 [n][d_v] or NULL.  d_k == d_v in {32, 64, 128}.
 */
pace_status pace_gdn_step_f32(float* S, const void* q, const void* k, const void* v,
                              const void* alpha, const void* beta, int32_t io_dtype,
                              float* o, int64_t n, int32_t d_k, int32_t d_v, void* stream);
pace_status pace_gdn_step_bf16(uint16_t* S, const void* q, const void* k, const void* v,
                               const void* alpha, const void* beta, int32_t io_dtype,
                               float* o, int64_t n, int32_t d_k, int32_t d_v, void* stream);

/*
 * Decode from host memory.  n_tokens decode steps for every head with inputs
 * and outputs in host memory (pinned for full copy speed):
 *   h_q, h_k: [n_tokens][num_slots][num_heads][d_k], h_v: [...][d_v],
 *   h_alpha, h_beta: [n_tokens][num_slots][num_heads] (io_dtype);
 *   h_o: fp32 [n_tokens][num_slots][num_heads][d_v], or NULL.
 * After every step each head whose buffer filled is committed (as
 * pace_commit_period).  Token t's inputs are copied in on h2d_stream while
 * token t-1 computes on `stream`, and its outputs are copied out on
 * d2h_stream while token t+1 computes, through d_staging: a device buffer
 * of pace_host_staging_bytes bytes (two token slots), 256-byte aligned,
 * owned by the caller and not used by anything else meanwhile.  The first
 * copies wait for the work already on `stream`, except when d_staging is the
 * buffer of this pool's previous call: then each slot is refilled as soon as
 * that call's last output copy from it is done, so consecutive calls keep
 * the copy engines busy.  That reuse is recognised by the pointer value
 * alone: a caller that frees the staging buffer and gets the same address
 * back for other work must order that work after this call (e.g. on
 * `stream`), since the next call's input copies start without waiting for
 * `stream`.  The three streams must be distinct
 * (PACE_ERR_INVALID_ARG otherwise, as for a NULL or unaligned d_staging or a
 * NULL input).  Enqueues only; `stream` completes after the last output
 * copy.  Not safe to call concurrently on one pool.  This host-buffer entry
 * point has no counterpart in the pages; it is the end-to-end path of a
 * serving loop.
 */
pace_status pace_host_staging_bytes(const pace_pool* pool, size_t* bytes);
pace_status pace_decode_host(pace_pool* pool, int32_t n_tokens, const void* h_q, const void* h_k,
                             const void* h_v, const void* h_alpha, const void* h_beta, float* h_o,
                             void* d_staging, void* stream, void* h2d_stream, void* d2h_stream);

/*
 * Pure-write window ("低比特量化新突破：GGA+PW让线性注意力长文本生成更准更短",
 * section "PW：让近期写入走“纯净通道”": the most recent writes stay apart from
 * the low-bit history as FP8 (k, v) pairs that take full part in the state
 * transition, and a pair is merged into the history when it leaves the
 * window).  The pool's buffer is the window and P its length S.  One step
 * for every head: k and v are rounded to FP8 E4M3 (nearest, ties to even,
 * saturating at +-448; kept in the io dtype, which holds every E4M3 value
 * exactly), o_t = S_t q_t is read out from the stored history and the
 * window as pace_decode_step does, and a head whose window then holds P
 * pairs applies its oldest pair alone to the history, re-encodes it, and
 * drops that pair (fill returns to P - 1).  Inputs and o as
 * pace_decode_step; d_scratch: device memory of pace_window_scratch_bytes
 * bytes, 256-byte aligned, for the rounded k and v.  A pool with a commit
 * threshold set is PACE_ERR_INVALID_ARG.  Enqueues only.
 */
pace_status pace_window_scratch_bytes(const pace_pool* pool, size_t* bytes);
pace_status pace_window_step(pace_pool* pool, const void* q, const void* k, const void* v,
                             const void* alpha, const void* beta, float* o, void* d_scratch,
                             void* stream);

/*
 * pace_window_step without caller scratch.  The paper has no counterpart:
 * this entry point exists for callers that cannot allocate device memory
 * themselves -- e.g. a plugin inside an inference engine whose allocator owns
 * the whole device budget and hands out only the tensors of a call's inputs
 * and outputs, or a hot loop that must not call cudaMalloc, which can
 * synchronise the device.  It allocates nothing: the scratch for the rounded
 * k and v is a device array of PACE_WINDOW_STATIC_SCRATCH_BYTES bytes inside
 * the library, which every GPU that loads the library holds until the
 * process exits.
 *  - Same arguments, results and errors as pace_window_step, minus
 *    d_scratch.
 *  - A pool whose pace_window_scratch_bytes exceeds
 *    PACE_WINDOW_STATIC_SCRATCH_BYTES is PACE_ERR_UNSUPPORTED (nothing is
 *    launched); use pace_window_step for it.
 *  - The first call on a device, with that device current, looks up the
 *    array's device address (cudaGetSymbolAddress; PACE_ERR_CUDA if that
 *    fails).  Make that first call before any stream capture.
 *  - Every call on a device shares the one array.  Calls whose work overlaps
 *    on the GPU (two streams, or two pools) race on it: order them, e.g. on
 *    one stream.  Nothing in the array needs clearing between calls: each
 *    call overwrites what it reads.
 */
#define PACE_WINDOW_STATIC_SCRATCH_BYTES 8388608u   /* 8 MiB */
pace_status pace_window_step_static(pace_pool* pool, const void* q, const void* k, const void* v,
                                    const void* alpha, const void* beta, float* o, void* stream);

/*
 * Chunked fp32 prefill (the chunked prefill kernels that [P2] "Periodic
 * Rounding" cites; [P4] flowchart "State update, chunked, high precision").
 * For every head of the slots (all of them, or [slot_begin, slot_begin +
 * slot_count)) whose buffer is empty: start from the stored state, apply T
 * tokens exactly in fp32 in chunks of 8 (UT/WY form), write every token's
 * output, and encode the final state into the pool once, at the end (fresh
 * absmax scales at the head's bit width); the buffer stays empty.
 *   q, k: [T][num_slots][num_heads][d_k], v: [T][num_slots][num_heads][d_v],
 *   alpha, beta: [T][num_slots][num_heads], all io_dtype, device, aligned
 *   to the element size; o: fp32 [T][num_slots][num_heads][d_v] or NULL.
 * A head with buffered tokens is skipped (PACE_FLAG_BUFFER_FULL).  A pool
 * that starts from zeros (all codes and scales 0) prefills from S = 0.
 */
pace_status pace_prefill(pace_pool* pool, int64_t T, const void* q, const void* k, const void* v,
                         const void* alpha, const void* beta, float* o, void* stream);
pace_status pace_prefill_range(pace_pool* pool, int32_t slot_begin, int32_t slot_count,
                               int64_t T, const void* q, const void* k, const void* v,
                               const void* alpha, const void* beta, float* o, void* stream);

/*
 * Choosing the 8-bit heads from their gates ([P2] paragraph on 8-bit
 * precision for selected heads; [P4] TL;DR (3): heads whose errors persist,
 * the long-memory heads, are kept at 8 bits).
 *
 * pace_decay_rates: alpha is a device matrix [rows][num_heads] in io_dtype
 * (e.g. the gates of a calibration prefill, rows = tokens x sequences);
 * rates (device, num_heads doubles, overwritten) receives each head's mean
 * decay rate  r_h = (1/rows) sum_rows -ln(alpha[row][h]), accumulated in
 * fp64.  A smaller rate is a longer memory.  Gates <= 0 or NaN give +inf or
 * NaN rates.  Asynchronous on `stream`.
 *
 * pace_select_head_bits (host only): head_bits[h] = 8 for the num_int8 heads
 * with the smallest rates (NaN rates last, ties to the lower head index),
 * 4 for the others -- ready for pace_pool_desc.head_bits.
 *
 * Neither call has a counterpart in the pages' text beyond the statement
 * that long-memory heads get 8 bits; the statistic is this library's
 * reading.
 */
pace_status pace_decay_rates(const void* alpha, int64_t rows, int32_t num_heads, int32_t io_dtype,
                             double* rates, void* stream);
pace_status pace_select_head_bits(const double* rates, int32_t num_heads, int32_t num_int8,
                                  uint8_t* head_bits);

/* Human-readable name of a status code (static string). */
const char* pace_status_string(pace_status s);

/* Library version, e.g. "0.1.0". */
const char* pace_version(void);

#ifdef __cplusplus
}
#endif
#endif /* PACE_H_ */
