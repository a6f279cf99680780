// Expansion of packed ternary weights into a dense int8 matrix [N_out, K]
// (pruned positions 0, kept ones -1/0/+1), for the prefill contraction.
//
// The contraction of many tokens reuses every weight tile once per token
// tile. Expanding the packed rows once per call into a caller workspace lets
// the tensor-core kernel load both operands with TMA, instead of expanding
// each weight tile again for every token tile.
//
// One thread expands one unit (16 positions of one row) into one 16-byte
// store; a warp takes 32 consecutive units (coalesced reads of codes and keep
// bits, coalesced 16-byte writes), the warps' chunks dealt out over all CTAs
// so that each CTA has a share even when the layer is small. CTAs of 512
// threads leave room on an SM for the contraction that follows (launched
// early, it sets up next to them).
#pragma once

#include "common.cuh"
#include "expand.cuh"

namespace sbn {

constexpr int kXdThreads = 512;

template <int MM, int CB, bool DENSE>
__global__ void __launch_bounds__(kXdThreads)
expand_dense_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ meta, int n_out,
                    int k, int cstride, int mstride, int8_t* __restrict__ wd) {
  __shared__ uint32_t s_sel[256];
  if (!DENSE) fill_selector_table(s_sel);
  __syncthreads();
  griddep_wait();
  griddep_launch_dependents();
  const int upr = k >> 4;
  const long long total = (long long)n_out * upr;
  // chunks of 32 consecutive units, one per warp, dealt out CTA-first so that
  // every CTA (every SM) has work even when the layer is small
  const long long nchunk = (total + 31) / 32;
  for (long long c = (long long)(threadIdx.x >> 5) * gridDim.x + blockIdx.x; c < nchunk;
       c += (long long)gridDim.x * (kXdThreads / 32)) {
    const long long g = c * 32 + (threadIdx.x & 31);
    if (g >= total) continue;
    const int row = (int)(g / upr);
    const int u = (int)(g - (long long)row * upr);
    const uint8_t* cp = codes + (size_t)row * cstride + (size_t)u * CB;
    uint32_t cw = 0u;
#pragma unroll
    for (int b = 0; b < CB; ++b) cw |= (uint32_t)cp[b] << (8 * b);
    uint32_t out[4];
    if (DENSE) {
      codes8_to_s8(cw & 0xFFFFu, out[0], out[1]);
      codes8_to_s8(cw >> 16, out[2], out[3]);
    } else {
      const uint32_t m16 = *reinterpret_cast<const uint16_t*>(meta + (size_t)row * mstride + 2 * u);
      const uint32_t m0 = m16 & 0xFFu, m1 = m16 >> 8;
      const int p0 = (MM == 16) ? __popc(m0) : 2 * CB;     // kept codes among the first 8
      const uint32_t v0 = cw & ((1u << (2 * p0)) - 1u);
      const uint32_t rest = cw >> (2 * p0);
      const int p1 = (MM == 16) ? __popc(m1) : 2 * CB;
      const uint32_t v1 = rest & ((1u << (2 * p1)) - 1u);
      expand8(m0, v0, s_sel, out[0], out[1]);
      expand8(m1, v1, s_sel, out[2], out[3]);
    }
    *reinterpret_cast<uint4*>(wd + (size_t)row * k + (size_t)u * 16) = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

}  // namespace sbn
