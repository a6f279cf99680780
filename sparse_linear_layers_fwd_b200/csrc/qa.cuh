// sbn_quantize_acts kernel: per-token absmax INT8 activations.
//
// "Microsoft BitNet 1.58: The Era of 1-Bit Large Language Models", section
// "The BitLinear Layer", second operation (bf16 -> INT8 with absmax scaling,
// scale preserved); per-token scale as on the promptingindex page, section
// "How ternary quantization works during training".
//
// One warp (K <= 2560) or one CTA of 128 threads (longer rows) per token
// row. The row is held in registers (MAXC 16-byte chunks per thread), so X
// is read from HBM exactly once: max |x| (integer max of the 15 magnitude
// bits), one IEEE division for the multiplier 127/s, then
// q = clamp(rint(x * mult), -127, 127).
// The grid is a full wave (as many CTAs as can be resident on every SM) and
// the rows are dealt out CTA-first: launched behind another kernel, CTAs are
// placed as that kernel's CTAs retire, and a full wave still ends up evenly
// spread, so every SM gets the same number of rows.
#pragma once

#include "common.cuh"

namespace sbn {

constexpr int kQaThreads = 128;

SBN_DEVFN uint32_t quant_pair(uint32_t wd, float mult) {
  int q0 = __float2int_rn(__fmul_rn(__uint_as_float(wd << 16), mult));
  int q1 = __float2int_rn(__fmul_rn(__uint_as_float(wd & 0xFFFF0000u), mult));
  q0 = min(max(q0, -127), 127);
  q1 = min(max(q1, -127), 127);
  return ((uint32_t)q0 & 0xFFu) | (((uint32_t)q1 & 0xFFu) << 8);
}

SBN_DEVFN uint32_t mag_max8(const uint4& v) {
  const uint32_t m0 = max(v.x & 0x7FFFu, (v.x >> 16) & 0x7FFFu);
  const uint32_t m1 = max(v.y & 0x7FFFu, (v.y >> 16) & 0x7FFFu);
  const uint32_t m2 = max(v.z & 0x7FFFu, (v.z >> 16) & 0x7FFFu);
  const uint32_t m3 = max(v.w & 0x7FFFu, (v.w >> 16) & 0x7FFFu);
  return max(max(m0, m1), max(m2, m3));
}

SBN_DEVFN uint2 quant8(const uint4& v, float mult) {
  const uint32_t p0 = quant_pair(v.x, mult), p1 = quant_pair(v.y, mult);
  const uint32_t p2 = quant_pair(v.z, mult), p3 = quant_pair(v.w, mult);
  return make_uint2(p0 | (p1 << 16), p2 | (p3 << 16));
}

// The same rounding as quant_pair without the float-to-integer conversion
// unit, for values with |x| <= s (x from the row whose maximum magnitude is
// s, mult = fl32(127 / s)): then |fl32(x * mult)| <= 127 * (1 + 2^-23), which
// rounds to at most 127, so the clamp of quant_pair never acts and is left
// out. fl32(p + 1.5 * 2^23) rounds p = fl32(x * mult) to the nearest integer
// with ties to even (the sum lies in [2^23, 2^24), where the spacing of fp32
// is 1, and 1.5 * 2^23 is even). The sum's bit pattern is
// 0x4B400000 + rint(p), so its low byte is the two's-complement INT8 value;
// four of them are gathered with byte permutes.
SBN_DEVFN uint32_t quant4_magic(uint32_t wa, uint32_t wb, float mult) {
  const float kMagic = 12582912.0f;
  const float r0 = __fadd_rn(__fmul_rn(__uint_as_float(wa << 16), mult), kMagic);
  const float r1 = __fadd_rn(__fmul_rn(__uint_as_float(wa & 0xFFFF0000u), mult), kMagic);
  const float r2 = __fadd_rn(__fmul_rn(__uint_as_float(wb << 16), mult), kMagic);
  const float r3 = __fadd_rn(__fmul_rn(__uint_as_float(wb & 0xFFFF0000u), mult), kMagic);
  const uint32_t lo = __byte_perm(__float_as_uint(r0), __float_as_uint(r1), 0x0040u);
  const uint32_t hi = __byte_perm(__float_as_uint(r2), __float_as_uint(r3), 0x0040u);
  return __byte_perm(lo, hi, 0x5410u);
}

// Eight values of a row (16 bytes of bf16) with |x| <= s -> eight INT8 bytes.
SBN_DEVFN uint2 quant8_magic(const uint4& v, float mult) {
  return make_uint2(quant4_magic(v.x, v.y, mult), quant4_magic(v.z, v.w, mult));
}

SBN_DEVFN float block_absmax_scale(uint32_t amax) {
  __shared__ uint32_t s_red[kQaThreads / 32];
  amax = __reduce_max_sync(0xffffffffu, amax);
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = amax;
  __syncthreads();
  uint32_t m = s_red[0];
#pragma unroll
  for (int i = 1; i < kQaThreads / 32; ++i) m = max(m, s_red[i]);
  return fmaxf(__uint_as_float(m << 16), 1e-5f);
}

// MAXC > 0: the row stays in registers. kc = K / 8 chunks of 16 bytes.
template <int MAXC>
__global__ void __launch_bounds__(kQaThreads)
qa_kernel(const uint4* __restrict__ x, int t, int kc, uint2* __restrict__ xq, float* __restrict__ scale) {
  griddep_wait();
  griddep_launch_dependents();
  for (size_t row = blockIdx.x; row < (size_t)t; row += gridDim.x) {
    const uint4* xr = x + row * kc;
    uint4 v[MAXC];
    uint32_t amax = 0u;
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
      const int idx = threadIdx.x + c * kQaThreads;
      v[c] = (idx < kc) ? __ldg(xr + idx) : make_uint4(0u, 0u, 0u, 0u);
      amax = max(amax, mag_max8(v[c]));
    }
    const float s = block_absmax_scale(amax);
    const float mult = __fdiv_rn(127.0f, s);
    if (threadIdx.x == 0) scale[row] = s;
    uint2* qr = xq + row * kc;
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
      const int idx = threadIdx.x + c * kQaThreads;
      if (idx < kc) qr[idx] = quant8(v[c], mult);
    }
    __syncthreads();   // the reduction's shared words are reused by the next row
  }
}

// One warp per token row (rows of kc <= 32 * MAXC chunks, K <= 2560): the
// row in registers, all its loads in flight at once, the maximum reduced in
// the warp (no block barrier); rows dealt out to warp w of CTA b in the order
// (w, b), so a full wave covers thousands of rows with each SM's share even.
constexpr int kQawThreads = 128;   // small CTAs: 7 per SM at K = 2560
template <int MAXC>
__global__ void __launch_bounds__(kQawThreads)
qa_warp_kernel(const uint4* __restrict__ x, int t, int kc, uint2* __restrict__ xq, float* __restrict__ scale) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  for (int row = (threadIdx.x >> 5) * gridDim.x + blockIdx.x; row < t; row += (kQawThreads / 32) * gridDim.x) {
    const uint4* xr = x + (size_t)row * kc;
    uint4 v[MAXC];
    uint32_t amax = 0u;
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
      const int idx = lane + 32 * c;
      v[c] = (idx < kc) ? __ldg(xr + idx) : make_uint4(0u, 0u, 0u, 0u);
      amax = max(amax, mag_max8(v[c]));
    }
    amax = __reduce_max_sync(0xffffffffu, amax);
    const float s = fmaxf(__uint_as_float(amax << 16), 1e-5f);
    const float mult = __fdiv_rn(127.0f, s);
    if (lane == 0) scale[row] = s;
    uint2* qr = xq + (size_t)row * kc;
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
      const int idx = lane + 32 * c;
      if (idx < kc) qr[idx] = quant8(v[c], mult);
    }
  }
}

// Rows too long for registers: two passes over the row (the second from L2).
__global__ void __launch_bounds__(kQaThreads)
qa_kernel_long(const uint4* __restrict__ x, int t, int kc, uint2* __restrict__ xq, float* __restrict__ scale) {
  griddep_wait();
  griddep_launch_dependents();
  for (size_t row = blockIdx.x; row < (size_t)t; row += gridDim.x) {
    const uint4* xr = x + row * kc;
    uint32_t amax = 0u;
    for (int idx = threadIdx.x; idx < kc; idx += kQaThreads) amax = max(amax, mag_max8(__ldg(xr + idx)));
    const float s = block_absmax_scale(amax);
    const float mult = __fdiv_rn(127.0f, s);
    if (threadIdx.x == 0) scale[row] = s;
    uint2* qr = xq + row * kc;
    for (int idx = threadIdx.x; idx < kc; idx += kQaThreads) qr[idx] = quant8(__ldg(xr + idx), mult);
    __syncthreads();   // the reduction's shared words are reused by the next row
  }
}

}  // namespace sbn
