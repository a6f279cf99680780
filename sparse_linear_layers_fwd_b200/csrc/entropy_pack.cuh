// Canonical packed weights (2-bit kept codes + keep bits) -> entropy-tight
// group words (the format is described in entropy.cuh).
//
// A segment is 32 consecutive groups of one row; one warp packs up to four
// consecutive segments of a row at a time: lane l makes the word of group
// 32 s + l of each, the warp ORs the words into a shared-memory buffer at bit
// offsets (32 j + l) * bits, and writes the segments' output words with plain
// coalesced stores. 32 words of `bits` bits fill exactly `bits` 32-bit
// words, so segments never share an output word: every word of the stream,
// row padding included, is written once, with no atomics on global memory
// and no clearing pass before.
//
// The colex rank of a keep mask (m <= 8) and the base-3 value of four kept
// codes are read from tables built on the host for the call's pattern; for
// m = 16 the rank is summed over the kept positions from a binomial table.
#pragma once

#include "common.cuh"
#include "entropy.cuh"

namespace sbn {

constexpr int kEpThreads = 512;
constexpr int kEpWarps = kEpThreads / 32;
constexpr int kEpUnroll = 4;   // consecutive segments a warp packs at a time

// Per-pattern constants, passed by value.
struct EntPackParams {
  uint32_t binom[17 * 17];   // C(a, b) at [17 a + b], a, b <= 16
  uint16_t rank[256];        // colex rank of an m-bit keep mask (m <= 8)
  uint8_t val4[256];         // sum_j (code_j + 1) 3^j of four 2-bit codes (j = 0 in the low bits)
  uint32_t p3n;              // 3^n
  uint32_t voff;             // value of the padding codes of the last four-code chunk
  uint32_t pw81[4];          // 81^c
  int nch;                   // four-code chunks per group, ceil(n / 4)
  int bits;                  // bits of one group word
};

// Host side: the tables of pattern n:m.
inline void fill_ent_pack_params(EntPackParams& p, int n, int m) {
  for (int a = 0; a <= 16; ++a)
    for (int b = 0; b <= 16; ++b) p.binom[17 * a + b] = binom_u32(a, b);
  for (int mask = 0; mask < 256; ++mask) {
    uint32_t r = 0u;
    int i = 0;
    for (int pos = 0; pos < 8; ++pos)
      if ((mask >> pos) & 1) r += p.binom[17 * pos + (++i)];
    p.rank[mask] = (uint16_t)r;
  }
  for (int b = 0; b < 256; ++b) {
    uint32_t v = 0u, p3 = 1u;
    for (int j = 0; j < 4; ++j) {
      const int c2 = (b >> (2 * j)) & 3;   // 00 -> 0, 01 -> +1, 11 -> -1 (10 never written)
      v += (c2 == 1 ? 2u : (c2 == 3 ? 0u : 1u)) * p3;
      p3 *= 3u;
    }
    p.val4[b] = (uint8_t)v;
  }
  p.p3n = pow3_u32(n);
  p.nch = (n + 3) / 4;
  for (int c = 0; c < 4; ++c) p.pw81[c] = pow3_u32(4 * c);
  // the last chunk of n % 4 = r codes reads 4 - r zero codes beyond them,
  // each a digit 1 at positions r..3 of that chunk
  const int r = n % 4;
  p.voff = r ? (pow3_u32(4) - pow3_u32(r)) / 2u * p.pw81[p.nch - 1] : 0u;
  p.bits = entropy_group_bits(n, m);
}

// codes, meta and ent are addressed in 32-bit words; cws, mws and ews are the
// row strides in words (the byte strides are multiples of 16).
template <int M>
__global__ void __launch_bounds__(kEpThreads)
entropy_pack_kernel(const uint32_t* __restrict__ codes, const uint32_t* __restrict__ meta, int n_out,
                    int k, int n, int cws, int mws, uint32_t* __restrict__ ent, int ews,
                    const __grid_constant__ EntPackParams prm) {
  __shared__ uint32_t s_binom[17 * 17];
  __shared__ uint16_t s_rank[256];
  __shared__ uint8_t s_val4[256];
  __shared__ uint32_t s_buf[kEpWarps][32 * kEpUnroll];
  for (int i = threadIdx.x; i < 17 * 17; i += kEpThreads) s_binom[i] = prm.binom[i];
  for (int i = threadIdx.x; i < 256; i += kEpThreads) {
    s_rank[i] = prm.rank[i];
    s_val4[i] = prm.val4[i];
  }
  __syncthreads();

  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int groups = k / M;
  const int segs = (groups + 31) / 32;
  const int chunks = (segs + kEpUnroll - 1) / kEpUnroll;   // per row
  const int items = n_out * chunks;   // (row, kEpUnroll consecutive segments)
  const int bits = prm.bits;
  const int warps = gridDim.x * kEpWarps;
  const bool has_meta = (n != M);
  const uint64_t cmask = (n == 16) ? 0xFFFFFFFFull : ((1ull << (2 * n)) - 1ull);
  uint32_t* buf = s_buf[wib];

  for (int item = blockIdx.x * kEpWarps + wib; item < items; item += warps) {
    const int row = item / chunks;
    const int seg0 = (item - row * chunks) * kEpUnroll;
    const int nseg = min(kEpUnroll, segs - seg0);
    const uint32_t* cr = codes + (size_t)row * cws;
    const uint32_t* mr = meta + (size_t)row * mws;
    // the loads of all kEpUnroll segments first
    uint32_t lo[kEpUnroll], hi[kEpUnroll], mw[kEpUnroll];
#pragma unroll
    for (int j = 0; j < kEpUnroll; ++j) {
      lo[j] = hi[j] = mw[j] = 0u;
      const int g = (seg0 + j) * 32 + lane;
      if (j < nseg && g < groups) {
        const int wi = (2 * n * g) >> 5;
        lo[j] = __ldg(cr + wi);
        if (wi + 1 < cws) hi[j] = __ldg(cr + wi + 1);
        if (has_meta) mw[j] = __ldg(mr + ((g * M) >> 5));
      }
      buf[32 * j + lane] = 0u;
    }
    __syncwarp();
#pragma unroll
    for (int j = 0; j < kEpUnroll; ++j) {
      const int g = (seg0 + j) * 32 + lane;
      if (j < nseg && g < groups) {
        const uint32_t full = (1u << M) - 1u;
        const uint32_t keep = has_meta ? (mw[j] >> ((g * M) & 31)) & full : full;
        const uint64_t cw = ((((uint64_t)hi[j] << 32) | lo[j]) >> ((2 * n * g) & 31)) & cmask;
        uint32_t rank;
        if (M <= 8) {
          rank = s_rank[keep];
        } else {
          rank = 0u;
          uint32_t kb = keep;
          for (int i = 0; i < n; ++i) {
            const int pos = __ffs(kb | 0x10000u) - 1;   // <= 16 even if fewer than n bits are set
            kb &= kb - 1u;
            rank += s_binom[17 * pos + i + 1];
          }
        }
        uint32_t v = 0u;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (c < prm.nch) v += (uint32_t)s_val4[(uint32_t)(cw >> (8 * c)) & 0xFFu] * prm.pw81[c];
        // (a word of well-formed input is below 2^bits; the mask keeps any
        // other input inside its own group's bits)
        const uint32_t word = (rank * prm.p3n + (v - prm.voff)) & ((1u << bits) - 1u);
        const int bo = (32 * j + lane) * bits, sh = bo & 31;
        atomicOr(buf + (bo >> 5), word << sh);
        if (sh + bits > 32) atomicOr(buf + (bo >> 5) + 1, word >> (32 - sh));
      }
    }
    __syncwarp();
    // the segments fill output words [seg0 * bits, (seg0 + nseg) * bits);
    // the row's last segment also writes the zero padding up to its end
    const int first = seg0 * bits;
    const int count = (seg0 + nseg == segs) ? ews - first : nseg * bits;
    uint32_t* out = ent + (size_t)row * ews + first;
    for (int w = lane; w < count; w += 32) out[w] = (w < 32 * kEpUnroll) ? buf[w] : 0u;
    __syncwarp();
  }
}

}  // namespace sbn
