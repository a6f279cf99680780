// mbarrier and bulk-copy helpers shared by the kernels of libsbn (sm_100a).
#pragma once

#include "common.cuh"

namespace sbn {

constexpr unsigned long long kMbarWaitNs = 250000000ull;  // an mbarrier wait gives up after 0.25 s
constexpr uint32_t kMbarSuspendNs = 20000;                 // suspend-time hint of one try_wait

SBN_DEVFN uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

SBN_DEVFN void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
SBN_DEVFN void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}
SBN_DEVFN void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// Wait for the phase of the given parity, bounded in time (kMbarWaitNs); false
// (and SBN_ERR_TIMEOUT in the device error word) if it gave up. try_wait
// suspends the thread until the phase completes or the hinted time passes,
// so a waiting thread does not spin. Kernels let one thread (or one lane
// per warp) wait and the others meet it at a barrier: the phase completion
// it observes, followed by the barrier, orders the arrived data before the
// others' reads.
SBN_DEVFN bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned long long limit_ns = kMbarWaitNs) {
  const uint32_t a = smem_u32(bar);
  unsigned long long t0 = 0;
  for (uint32_t i = 0;; ++i) {
    uint32_t done;
    asm volatile(
        "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\nselp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(a), "r"(parity), "r"(kMbarSuspendNs)
        : "memory");
    if (done) return true;
    const unsigned long long t = global_ns();
    if (i == 0u) t0 = t;
    else if (t - t0 > limit_ns) break;
  }
  atomicOr(&g_dev_error, kDevErrTimeout);
  return false;
}

// One non-blocking probe of the phase of the given parity (no suspension,
// no time bound): true if it has completed. Callers fall back to mbar_wait.
SBN_DEVFN bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n.reg .pred p;\nmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\nselp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Bulk copy (no tensor map) of `bytes` (a multiple of 16, both addresses
// 16-byte aligned) from global to this CTA's shared memory, completing
// `bytes` transactions on `bar`.
SBN_DEVFN void bulk_g2s(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
          smem_u32(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

}  // namespace sbn
