// Blackwell (sm_100a) building blocks for the tensor-memory commit kernel:
// TMEM allocation, tcgen05.mma with shared-memory matrix descriptors,
// tcgen05.ld, commits to mbarriers, bulk and tensor stores, stmatrix of
// bytes, and named barriers.  Inline PTX only; the descriptor bit layout is
// the one the PTX ISA defines for tcgen05 shared-memory matrix descriptors
// and instruction descriptors (kind::f16, f32 accumulation).
#pragma once

#include <cuda.h>

#include "tma.cuh"

namespace pace {
namespace tc {

// ---- shared-memory matrix descriptors --------------------------------------
// Layout types (bits 61..63).
constexpr uint32_t kSwizzleNone = 0;
constexpr uint32_t kSwizzle128 = 2;

// addr: shared-space byte address of the first core matrix (16-byte aligned;
// 1024-byte aligned swizzle atoms for 128-byte swizzling); lbo / sbo: the
// leading- and stride-dimension byte offsets.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  uint64_t d = (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;          // descriptor version for sm_100
  d |= (uint64_t)layout << 61;
  return d;
}

// Instruction descriptor: f16 x f16 -> f32, M x N, each operand K-major (0)
// or MN-major (1).
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A * B, issued by one thread.
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"((uint32_t)accumulate)
      : "memory");
}

// Arrive on `bar` once every tcgen05.mma this thread issued so far has completed.
__device__ __forceinline__ void commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ---- TMEM allocation (one full warp) ----------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_free(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// ---- TMEM loads -------------------------------------------------------------
// 32x32b.x16: thread t of the warp gets lane (base + t), 16 consecutive columns.
__device__ __forceinline__ void ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// 16x256b.x8: lanes base..base+15, 64 columns.  Thread (g = t/4, q = t%4)
// gets, for column block c (8 columns): r[4c] = (lane g, col 8c + 2q),
// r[4c+1] = (g, 8c + 2q + 1), r[4c+2] = (g + 8, 8c + 2q), r[4c+3] = (g + 8, 8c + 2q + 1).
__device__ __forceinline__ void ld_16x256b_x8(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x8.b32 {"
      "%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// ---- bytes into shared memory, transposed -----------------------------------
// stmatrix.m16n8.x1.trans.b8: threads 0..7 give the addresses of 8 rows of 16
// bytes; byte b of thread t (g = t/4, q = t%4) lands in row 2q + (b & 1),
// column g + 8 (b >> 1).
__device__ __forceinline__ void stsm_trans_b8(uint32_t row_addr, uint32_t v) {
  asm volatile("stmatrix.sync.aligned.m16n8.x1.trans.shared.b8 [%0], {%1};" ::"r"(row_addr), "r"(v) : "memory");
}

// Four 8 x 16-byte matrices at once: threads 8m .. 8m + 7 give the row
// addresses of matrix m, register m holds that matrix's bytes as above.
__device__ __forceinline__ void stsm_trans_b8_x4(uint32_t row_addr, uint32_t v0, uint32_t v1, uint32_t v2, uint32_t v3) {
  asm volatile("stmatrix.sync.aligned.m16n8.x4.trans.shared.b8 [%0], {%1, %2, %3, %4};" ::"r"(row_addr), "r"(v0),
               "r"(v1), "r"(v2), "r"(v3)
               : "memory");
}

// ---- bulk and tensor stores (shared -> global) ------------------------------
__device__ __forceinline__ void bulk_store(void* gdst, uint32_t ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(ssrc), "r"(bytes)
               : "memory");
}
// 2-D tiled store of a box at coordinates (x, y); x * element size must be a
// multiple of 16 bytes (here x = 0).
__device__ __forceinline__ void tensor_store_2d(const CUtensorMap* map, uint32_t ssrc, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(map),
               "r"(ssrc), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until the shared-memory sources of every committed group have been read.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Wait until every committed group has completed (writes visible).
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// ---- waits --------------------------------------------------------------------
// Wait for phase `parity` of `bar`, letting the hardware suspend the thread
// between tests (up to 1 ms per test) instead of spinning; false and
// PACE_FLAG_TIMEOUT once kWaitLimitNs of global time have passed.
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t* flags) {
  const uint64_t t0 = global_ns();
  while (true) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(1000000u)
        : "memory");
    if (ok) return true;
    if (global_ns() - t0 > kWaitLimitNs) {
      if (flags) atomicOr(flags, PACE_FLAG_TIMEOUT);
      return false;
    }
  }
}

// ---- mbarrier arrive and named barriers --------------------------------------
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ void named_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Named barrier that also returns whether any participating thread passed
// pred = true: the threads of a group leave a loop together.
__device__ __forceinline__ bool named_sync_any(uint32_t id, uint32_t nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 q, %1, 0;\n bar.red.or.pred p, %2, %3, q;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

}  // namespace tc
}  // namespace pace
