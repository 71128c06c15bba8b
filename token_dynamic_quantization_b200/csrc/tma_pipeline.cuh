// Bulk-copy (TMA) row pipeline primitives for sm_100a.
//
// Each row group of a persistent CTA owns a ring of S shared-memory stages.
// One elected thread streams whole rows from HBM into the ring with
// cp.async.bulk (no tensor map: a row is one contiguous, 16-byte aligned run
// of bytes), and the transfer completes a transaction-count mbarrier per
// stage. Consumers wait on the stage's mbarrier phase, read the row from
// shared memory, and the next copy into that stage is issued only after the
// whole group has passed a barrier that follows those reads.
//
// Every wait is bounded in time: after kWaitLimitNs without completion the
// caller gets `false` and must take its error path (no GPU hang).
#pragma once

#include <stdint.h>

namespace dq {

// Every wait gives up after DQ_WAIT_LIMIT_NS nanoseconds of the global timer
// (one second: far above any legitimate wait for a copy or an MMA, short
// enough that a lost copy ends the kernel instead of hanging the GPU).
#ifndef DQ_WAIT_LIMIT_NS
#define DQ_WAIT_LIMIT_NS 1000000000ull
#endif
constexpr uint64_t kWaitLimitNs = DQ_WAIT_LIMIT_NS;

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Make mbarrier initialisation visible to the async (bulk copy) proxy.
__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Order this thread's earlier generic-proxy shared memory accesses before
// subsequent async-proxy (bulk copy) accesses.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

// L2 policy for data read exactly once: evict first.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t policy;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(policy));
  return policy;
}

// Global -> shared bulk copy of `bytes` (multiple of 16, both addresses
// 16-byte aligned) completing on `bar`.
__device__ __forceinline__ void bulk_copy_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_addr(dst_smem)),
      "l"(src_gmem), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t addr, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(addr), "r"(parity)
      : "memory");
  return done != 0;
}

// Bounded wait for phase `parity` of `bar` to complete. Returns false after
// kWaitLimitNs without completion.
__device__ __forceinline__ bool mbar_wait_parity(uint64_t* bar, uint32_t parity) {
  const uint32_t addr = smem_addr(bar);
  if (mbar_try_wait(addr, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    if (mbar_try_wait(addr, parity)) return true;
    if (global_ns() - t0 > kWaitLimitNs) return false;
  }
}

// Bounded wait with an explicit limit in nanoseconds.
__device__ __forceinline__ bool mbar_wait_parity_for(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint32_t addr = smem_addr(bar);
  if (mbar_try_wait(addr, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    if (mbar_try_wait(addr, parity)) return true;
    if (global_ns() - t0 > limit_ns) return false;
  }
}

// The same wait that also gives up as soon as *abort (shared memory) is
// non-zero: another warp of the CTA has met a failed wait.
__device__ __forceinline__ bool mbar_wait_parity_or_abort(uint64_t* bar, uint32_t parity,
                                                          const volatile uint32_t* abort) {
  const uint32_t addr = smem_addr(bar);
  if (mbar_try_wait(addr, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    if (mbar_try_wait(addr, parity)) return true;
    if (*abort != 0u || global_ns() - t0 > kWaitLimitNs) return false;
  }
}

// Bounded wait until *round (shared memory, written by another warp of the
// CTA) equals `want`; gives up on the abort flag or after kWaitLimitNs. The
// fence orders what the writer did before its write (it had observed the
// slot's previous phase complete) before anything this thread does next.
__device__ __forceinline__ bool wait_round(const volatile int32_t* round, int32_t want,
                                           const volatile uint32_t* abort) {
  if (*round != want) {
    const uint64_t t0 = global_ns();
    while (*round != want) {
      if (*abort != 0u || global_ns() - t0 > kWaitLimitNs) return false;
    }
  }
  __threadfence_block();
  return true;
}

// Plain arrival (count 1) on `bar`.
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Group barrier over `nthreads` (a multiple of 32) that also ORs a predicate
// across the group: every participant gets true if any passed true.
__device__ __forceinline__ bool group_barrier_or(int id, int nthreads, bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(out)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(nthreads)
      : "memory");
  return out != 0;
}

}  // namespace dq
