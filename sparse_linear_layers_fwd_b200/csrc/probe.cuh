// Small kernels that serve measurement and testing, not the method:
//
// * i8_peak_kernel: the tensor pipe's INT8 rate on this part. Every CTA (one
//   per SM) issues a long run of `tcgen05.mma.cta_group::1.kind::i8` (M = 128,
//   N = 256, K = 32 bytes, int32 accumulate in tensor memory) from one thread
//   on shared-memory operands, the same instruction, descriptors and tile
//   shapes as the prefill contraction (bl_tc.cuh), with no loads in between.
//   The host times the launch; 2 * 128 * 256 * 32 operations per instruction.
// * wait_selftest_kernel: runs one of the library's bounded device waits on a
//   condition that never comes, with a short limit, so that the give-up path
//   (the device error word, then SBN_ERR_TIMEOUT from sbn_get_device_error)
//   can be exercised without a fault or a hang: no asynchronous copy or MMA is
//   outstanding when the wait gives up, and the kernel then returns normally.
#pragma once

#include "async.cuh"
#include "bl_tc.cuh"
#include "bl_tc2.cuh"
#include "common.cuh"
#include "qw_stream.cuh"

namespace sbn {

constexpr int kPkThreads = 128;
constexpr uint32_t kPkTmemCols = 256;
constexpr size_t kPkSmemBytes = 1024 + (size_t)kTcABytes + (size_t)kTcBBytes + 64;

__global__ void __launch_bounds__(kPkThreads, 1) i8_peak_kernel(int iters) {
  extern __shared__ uint8_t pk_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(pk_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kTcABytes + kTcBBytes);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bar + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // operands: zeros (the rate does not depend on the values)
  for (int i = tid; i < (kTcABytes + kTcBBytes) / 16; i += kPkThreads)
    reinterpret_cast<uint4*>(smem)[i] = make_uint4(0u, 0u, 0u, 0u);
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
  if (tid == 0) {
    mbar_init(bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(s_tmem)),
                 "r"(kPkTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  if (warp == 1 && lane == 0) {
    const uint64_t adesc = sw128_kmajor_desc(smem_u32(smem));
    const uint64_t bdesc = sw128_kmajor_desc(smem_u32(smem + kTcABytes));
    for (int i = 0; i < iters; ++i) {
      const uint64_t k = (uint64_t)(2 * (i & 3));   // 32-byte K steps inside the swizzled row
      tc_mma_i8(tmem, adesc + k, bdesc + k, i > 0 ? 1u : 0u);
    }
    tc_commit(bar);   // arrives once every MMA has completed
  }
  if (lane == 0) mbar_wait(bar, 0u);
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kPkTmemCols) : "memory");
  }
}

// The sparse INT8 rate on CTA pairs: clusters of two CTAs (one per SM: the
// shared memory asked for leaves no room for a second CTA, so no CTA waits
// for another's tensor memory), the leader issuing back-to-back
// `tcgen05.mma.sp.cta_group::2.kind::i8` of M = 256, N = 224, K = 64 logical
// positions (the prefill pair kernel's 2:4 instruction), with valid
// metadata (positions 0 and 1 of every group) copied into tensor memory once.
// 2 * 256 * 224 * 64 logical operations per instruction, half of them
// products of kept weights.
constexpr size_t kPsSmemBytes = 120 * 1024;
constexpr uint32_t kPsTmemCols = 256;
__global__ void __launch_bounds__(kPkThreads, 1) i8_sparse_peak_kernel(int iters) {
  extern __shared__ uint8_t ps_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ps_raw) + 1023) & ~uintptr_t(1023));
  // A 128 x 128 bytes | B 112 x 128 bytes | metadata 128 x 16 bytes | barrier, TMEM slot
  constexpr int kA = 128 * 128, kB = 112 * 128, kE = 128 * 16;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kA + kB + kE);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bar + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < (kA + kB + kE) / 4; i += kPkThreads) reinterpret_cast<uint32_t*>(smem)[i] = 0x44444444u;
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
  if (tid == 0) {
    mbar_init(bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(s_tmem)),
                 "r"(kPsTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  if (warp == 1 && lane == 0 && cluster_rank() == 0) {
    const uint64_t adesc = sw128_kmajor_desc(smem_u32(smem));
    const uint64_t bdesc = sw128_kmajor_desc(smem_u32(smem + kA));
    const uint32_t e = tmem + 224;
    tc_cp_meta_pair(e, meta_block_desc(smem_u32(smem + kA + kB)));
    for (int i = 0; i < iters; ++i) {
      // 32-byte steps of A and 64-byte steps of B inside the swizzled rows
      tc_mma_pair<true, T2Cfg<true>::IDESC>(tmem, adesc + (uint64_t)(2 * (i & 3)), bdesc + (uint64_t)(4 * (i & 1)),
                        e + 2u * (uint32_t)(i & 1), i > 0 ? 1u : 0u);
    }
    tc_commit_pair(bar);   // arrives in both CTAs once every MMA has completed
  }
  if (lane == 0) mbar_wait(bar, 0u);
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kPsTmemCols) : "memory");
  }
}

__device__ uint32_t g_selftest_counter;

// which 0: an mbarrier (one expected arrival) that nobody arrives on; which
// 1: the grid barrier of the weight quantizer with a target no launch reaches.
__global__ void wait_selftest_kernel(int which, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int s_abort;
  if (which == 0) {
    if (threadIdx.x == 0) {
      mbar_init(&bar, 1);
      asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0u, limit_ns);
  } else {
    if (threadIdx.x == 0) g_selftest_counter = 0u;   // one CTA: this launch's own counter
    __threadfence();
    __syncthreads();
    qs_grid_barrier(&g_selftest_counter, 2u, &s_abort, limit_ns);
  }
}

}  // namespace sbn
