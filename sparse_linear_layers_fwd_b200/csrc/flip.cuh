// Mask flip count between two versions of the packed weights.
//
// "Sparse-BitNet: 1.58-bit LLMs are Naturally Friendly to Semi-Structured
// Sparsity", Figure 3(b): the mask flip rate r_t tracks how stable the
// dynamic N:M pattern is from one training step to the next (its equation is
// not in the extracted page). Read plainly: the number of positions whose
// keep bit differs between the two masks, over N_out * K positions. This
// kernel produces the exact count; the rate is count / (N_out * K).
//
// HBM-bound: both keep bitmasks are read once with 16-byte loads
// (grid-stride, consecutive threads on consecutive 16 bytes); popcounts of
// the XOR are reduced per warp and added with one 64-bit atomic per warp.
#pragma once

#include "common.cuh"

namespace sbn {

constexpr int kFlipThreads = 256;

__global__ void __launch_bounds__(kFlipThreads)
flip_count_kernel(const uint4* __restrict__ a, const uint4* __restrict__ b, long long n16,
                  unsigned long long* __restrict__ out) {
  unsigned long long c = 0ull;
  for (long long i = (long long)blockIdx.x * kFlipThreads + threadIdx.x; i < n16;
       i += (long long)gridDim.x * kFlipThreads) {
    const uint4 x = __ldg(a + i), y = __ldg(b + i);
    c += __popc(x.x ^ y.x) + __popc(x.y ^ y.y) + __popc(x.z ^ y.z) + __popc(x.w ^ y.w);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if ((threadIdx.x & 31) == 0 && c) atomicAdd(out, c);
}

}  // namespace sbn
