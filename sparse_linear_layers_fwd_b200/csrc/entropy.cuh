// Entropy-tight packed weights: one integer word per group of m positions,
//     word = rank(kept positions) * 3^n + sum_i (code_i + 1) * 3^i,
// with the keep pattern ranked in the combinatorial number system (colex:
// kept offsets c_1 < ... < c_n give rank = sum_i C(c_i, i)) and the kept
// ternary codes, in ascending position, as base-3 digits. A word takes
// ceil(log2(C(m, n) * 3^n)) bits; the words of a row are concatenated
// little-endian and rows are padded to 16 bytes.
//
// "From 2:4 to 8:16 sparsity patterns in LLMs for Outliers and Weights with
// Variance Correction", Abstract: the 2:4 and 8:16 masks cost 0.75 and 0.875
// bits per element -- ceil(log2 C(m, n)) / m, the size of such a rank. Joined
// with the kept values, 6:8 takes 15 bits per 8 weights (1.875 bits) instead
// of the 2.5 bits of codes + keep bits.
#pragma once

#include "common.cuh"

namespace sbn {

__host__ __device__ constexpr uint32_t binom_u32(int a, int b) {
  if (b < 0 || b > a) return 0u;
  uint32_t r = 1u;
  for (int i = 1; i <= b; ++i) r = r * (uint32_t)(a - b + i) / (uint32_t)i;
  return r;
}
__host__ __device__ constexpr uint32_t pow3_u32(int e) {
  uint32_t r = 1u;
  for (int i = 0; i < e; ++i) r *= 3u;
  return r;
}
// Bits of one group word.
__host__ __device__ constexpr int entropy_group_bits(int n, int m) {
  uint64_t v = (uint64_t)binom_u32(m, n) * pow3_u32(n) - 1u;
  int b = 0;
  while (v) {
    ++b;
    v >>= 1;
  }
  return b;
}
__host__ __device__ constexpr size_t entropy_row_bytes(int k, int n, int m) {
  return (((size_t)(k / m) * (size_t)entropy_group_bits(n, m) + 7u) / 8u + 15u) & ~(size_t)15;
}

constexpr int kEntRankSlots = 128;   // rank table entries (every word of M <= 8 has rank < 128)

// Shared-memory tables for decoding group words of an n:M pattern (M <= 8):
// keep mask of every colex rank, and the 2n-bit packed canonical codes of
// every base-3 value.
template <int M, int N>
SBN_DEVFN void fill_entropy_tables(uint16_t* s_rank_mask, uint16_t* s_val_codes) {
  constexpr int kRanks = (int)binom_u32(M, N);
  constexpr int kVals = (int)pow3_u32(N);
  // every one of the kEntRankSlots entries is written: words of rows past
  // the layer's end (never stored) can hold any rank, which must still map
  // to a mask of at most M bits
  for (int r = threadIdx.x; r < kEntRankSlots; r += blockDim.x) {
    uint32_t mask = 0u;
    if (r < kRanks) {
      // unrank: largest c with C(c, i) <= remaining, for i = N .. 1
      uint32_t rem = (uint32_t)r;
      for (int i = N; i >= 1; --i) {
        int c = i - 1;
        while (binom_u32(c + 1, i) <= rem) ++c;
        mask |= 1u << c;
        rem -= binom_u32(c, i);
      }
    }
    s_rank_mask[r] = (uint16_t)mask;
  }
  for (int v = threadIdx.x; v < kVals; v += blockDim.x) {
    uint32_t x = (uint32_t)v, out = 0u;
    for (int i = 0; i < N; ++i) {
      const uint32_t d = x % 3u;                 // digit = code + 1
      x /= 3u;
      const uint32_t c2 = d == 2u ? 1u : (d == 0u ? 3u : 0u);
      out |= c2 << (2 * i);
    }
    s_val_codes[v] = (uint16_t)out;
  }
}

}  // namespace sbn
