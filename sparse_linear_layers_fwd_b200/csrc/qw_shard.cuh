// Weight quantization of one shard of a layer split along N_out
// (column-parallel): the absmean scale is a per-tensor quantity, so every
// shard contributes its exact gamma bins, the bins are summed over the
// shards (an integer all-reduce, exact and order-free), and every shard then
// quantizes its rows with the gamma of the whole tensor.
//
// Absmean quantizer: "BitNet b1.58: How Ternary Weights Cut LLM Memory by
// 82% Without Losing Accuracy", section "How ternary quantization works
// during training". Magnitude mask: "Sparse-BitNet: 1.58-bit LLMs are
// Naturally Friendly to Semi-Structured Sparsity", Abstract and Figure 6.
//
// Bins: 256 unsigned 64-bit integers B[e] whose weighted sum
// S = sum_e B[e] * 2^(e - 134) is the exact sum of |w| of the shard (a bf16
// magnitude with biased exponent e and fraction f is (128 + f) * 2^(e - 134),
// a subnormal f * 2^(1 - 134)). The split of S across e is not unique -- a
// thread files its windowed fixed-point sum under three exponents -- but any
// such vectors add up to the bins of the union of their shards.
#pragma once

#include "common.cuh"
#include "qw.cuh"
#include "qw_fused.cuh"

namespace sbn {

constexpr int kQbThreads = 512;

// Exact bins of |w| over the tensor (grid-stride over 16-byte chunks). The
// bins must be zero on entry (the host clears them on the same stream).
__global__ void __launch_bounds__(kQbThreads)
gamma_bins_kernel(const uint4* __restrict__ w, long long chunks, unsigned long long* __restrict__ bins) {
  __shared__ unsigned long long sbins[kQwBins];
  __shared__ unsigned long long swarp[kQbThreads / 32];
  for (int i = threadIdx.x; i < kQwBins; i += kQbThreads) sbins[i] = 0ull;
  __syncthreads();
  unsigned long long acc = 0ull;   // window sum in units of 2^(kWinLo - 134)
  for (long long c = (long long)blockIdx.x * kQbThreads + threadIdx.x; c < chunks;
       c += (long long)gridDim.x * kQbThreads) {
    const uint4 v = __ldg(w + c);
    const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      exact_accumulate(wd[i] & 0x7FFFu, acc, sbins);
      exact_accumulate((wd[i] >> 16) & 0x7FFFu, acc, sbins);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) swarp[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long a = 0ull;
    for (int i = 0; i < kQbThreads / 32; ++i) a += swarp[i];
    // a counts units of 2^(kWinLo - 134): file it under exponents kWinLo,
    // kWinLo + 21 and kWinLo + 42 in 21-bit pieces so every bin stays small
    const unsigned long long mask21 = (1ull << 21) - 1ull;
    const unsigned long long a0 = a & mask21, a1 = (a >> 21) & mask21, a2 = a >> 42;
    if (a0) atomicAdd(&bins[kWinLo], a0);
    if (a1) atomicAdd(&bins[kWinLo + 21], a1);
    if (a2) atomicAdd(&bins[kWinLo + 42], a2);
  }
  for (int i = threadIdx.x; i < kQwBins; i += kQbThreads)
    if (sbins[i]) atomicAdd(&bins[i], sbins[i]);
}

// Mask, codes and packing of the shard's rows with the gamma of the whole
// tensor, from the summed bins: gamma = max(fl32(fl64(S) / n_elems), 1e-5)
// and its code threshold tau, computed by every CTA; then one pass over the
// units (16 consecutive weights of a row), each thread taking whole units.
template <int M>
__global__ void __launch_bounds__(kQbThreads)
qw_from_bins_kernel(const uint16_t* __restrict__ w, int n_out, int k, int n,
                    const unsigned long long* __restrict__ bins, long long n_elems,
                    uint8_t* __restrict__ codes, int codes_stride, uint8_t* __restrict__ meta,
                    int meta_stride, float* __restrict__ gamma_out) {
  __shared__ uint32_t s_csel[256];
  __shared__ uint32_t s_tau;
  fill_compact_table(s_csel);
  if (threadIdx.x < 32) {
    float g;
    uint32_t tau;
    gamma_and_tau_from_bins(bins, n_elems, &g, &tau);
    if (threadIdx.x == 0) {
      s_tau = tau;
      if (blockIdx.x == 0) *gamma_out = g;
    }
  }
  __syncthreads();
  const uint32_t tau = s_tau;
  const uint32_t tau2 = tau | (tau << 16);
  const bool has_meta = (n != M);
  const int cb = 4 * n / M;   // code bytes per unit
  const int upr = k >> 4;     // units per row
  const long long units = (long long)n_out * upr;
  for (long long gu = (long long)blockIdx.x * kQbThreads + threadIdx.x; gu < units;
       gu += (long long)gridDim.x * kQbThreads) {
    const int row = (int)(gu / upr), u = (int)(gu - (long long)row * upr);
    const uint4* src = reinterpret_cast<const uint4*>(w + (size_t)row * k + (size_t)u * 16);
    const uint4 a = __ldg(src), b = __ldg(src + 1);
    const uint32_t wd[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t keep = 0xFFFFu;
    if (has_meta) {
      uint32_t mw[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mw[i] = wd[i] & 0x7FFF7FFFu;
      keep = unit_keep_fast<M>(mw, n);
      *reinterpret_cast<uint16_t*>(meta + (size_t)row * meta_stride + 2 * u) = (uint16_t)keep;
    }
    const uint32_t packed = unit_codes(wd, tau2, keep, s_csel);
    uint8_t* dst = codes + (size_t)row * codes_stride + (size_t)u * cb;
    if (cb == 4) {
      *reinterpret_cast<uint32_t*>(dst) = packed;
    } else if (cb == 2) {
      *reinterpret_cast<uint16_t*>(dst) = (uint16_t)packed;
    } else {
      for (int bb = 0; bb < cb; ++bb) dst[bb] = (uint8_t)(packed >> (8 * bb));
    }
    if (u == upr - 1) {
      // zero padding at the end of the row
      for (int i = upr * cb; i < codes_stride; ++i) codes[(size_t)row * codes_stride + i] = 0u;
    }
  }
}

}  // namespace sbn
