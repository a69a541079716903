// Shared device/host helpers for libi8q: status plumbing, the device error word, bounded
// mbarrier waits, TMA and tcgen05 (5th-generation tensor core) PTX wrappers for sm_100a.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/i8q.h"

namespace i8q {

// ------------------------------------------------------------------ error word --------------
// Set by a kernel whose bounded wait expired; read and cleared by i8q_status_check().
// Bit layout: bit 0 = some wait expired; bits 8..15 = code of the first wait that expired.
__device__ unsigned int g_error_word;

enum WaitSite : unsigned {
  SITE_FULL = 1, SITE_EMPTY = 2, SITE_TMEM_FULL = 3, SITE_TMEM_EMPTY = 4, SITE_DRAIN = 5,
  SITE_CLUSTER = 6, SITE_CONVERT = 7,
};

// A wait gives up after this many nanoseconds of %globaltimer (no kernel here legitimately
// waits anywhere near this long on one barrier phase).  g_wait_limit_ns holds the limit of the
// pipeline waits and may be lowered for a test (i8q_test_set_wait_limit_ns); the drain waits,
// which let copies and MMAs already in flight finish before a CTA exits, always use the default.
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;  // 2 s
__device__ unsigned long long g_wait_limit_ns = kWaitTimeoutNs;

// Test aid, normally 0.  When set (i8q_test_skip_accumulator_signal), the first CTA of the
// decode-size channel-wise W8A8 GEMM that reads it clears it and withholds its accumulator-ready
// signal once, so that its epilogue's bounded wait expires: the kernel then returns early and
// i8q_status_check() reports I8Q_ERR_TIMEOUT.  Nothing else in flight depends on that signal.
__device__ unsigned int g_test_skip_acc_signal;

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void raise_error(unsigned site) {
  atomicOr(&g_error_word, 1u | (site << 8));
}

// ------------------------------------------------------------------ mbarrier ----------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits until the phase with the given parity has completed.  Returns false (and raises the
// device error word) if that does not happen within kWaitTimeoutNs; `abort_flag` (shared
// memory, may be null) is polled so that one expired wait makes every other role give up fast.
__device__ __noinline__ unsigned long long wait_limit_ns(unsigned site) {
  return site == SITE_DRAIN ? (unsigned long long)kWaitTimeoutNs
                            : *reinterpret_cast<volatile unsigned long long*>(&g_wait_limit_ns);
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned site,
                                          volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  unsigned long long t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (abort_flag && *abort_flag) return false;
      const unsigned long long dt = globaltimer_ns() - t0;
      // the limit (a global-memory read) is fetched only once a wait has lasted 100 us
      if (dt > 100000ull && dt > wait_limit_ns(site)) {
        raise_error(site);
        if (abort_flag) *abort_flag = 1;
        return false;
      }
    }
  }
}

// Warp-uniform wait: lane 0 polls, the verdict is broadcast.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, unsigned site, volatile int* abort_flag) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, site, abort_flag) ? 1 : 0;
  return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

// ------------------------------------------------------------------ TMA ---------------------
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// Pull a tile into L2 only (nothing reaches shared memory, no barrier).  L2 is the device's point
// of coherence, so this is harmless even when the data is still being written by an earlier kernel:
// such writes land in L2 and later loads see them.
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap* map, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y)
               : "memory");
}

// Programmatic dependent launch.  A kernel launched with programmatic stream serialization may
// start while the previous kernel on the stream is still running; grid_dependency_wait() blocks
// until that kernel has completed and its memory is visible (it returns at once when there is no
// such dependency).  grid_dependents_launch() lets the next kernel start early.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dependents_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }


// ------------------------------------------------------------------ tcgen05 -----------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive on `bar` once every tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, int8 x int8 -> int32, one instruction (K = 32).
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 columns of 32-bit TMEM -> 32 registers per thread (thread t gets lane base+t).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
// 32 lanes x 16 columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }


// Shared-memory matrix descriptor for a K-major operand stored with the 128-byte swizzle that
// TMA (CU_TENSOR_MAP_SWIZZLE_128B) writes: rows of 128 bytes, 8-row core groups 1024 bytes
// apart.  Field layout (sm_100 UMMA descriptor): [0,14) start >> 4, [16,30) leading byte
// offset >> 4 (unused for swizzled K-major, set to 1), [32,46) stride byte offset >> 4,
// [46,48) descriptor version = 1, [49,52) base offset = 0 (buffers are 1024-byte aligned),
// [61,64) layout = 2 (128-byte swizzle).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor: kind::i8, signed A and B, int32 D, both K-major.
__host__ __device__ constexpr uint32_t idesc_i8(int M, int N) {
  return (2u << 4)              // D format: s32
         | (1u << 7)            // A: signed 8-bit
         | (1u << 10)           // B: signed 8-bit
         | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// Instruction descriptor: kind::f16, f16 A and B, f32 D, both K-major.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N) {
  return (1u << 4)              // D format: f32
         | (0u << 7) | (0u << 10)  // A, B: f16
         | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ------------------------------------------------------------------ small utils -------------
__host__ __device__ constexpr int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace i8q
