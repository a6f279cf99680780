// sbn_quantize_weights kernels: exact absmean gamma, N:M mask, ternary codes, packing.
//
// Absmean quantizer: "BitNet b1.58: How Ternary Weights Cut LLM Memory by 82%
// Without Losing Accuracy", section "How ternary quantization works during
// training" (divide by the mean |W|, round, clamp to [-1, 1]). Magnitude
// mask: "Sparse-BitNet: 1.58-bit LLMs are Naturally Friendly to
// Semi-Structured Sparsity", Abstract and Figure 6 (threshold t = |w|_(N+1)).
//
// Three launches on the caller's stream (after a memset of the bins):
//   qw_bins_kernel     streams W once and adds every |w| exactly into
//                      per-exponent integer bins (order-independent);
//   qw_finalize_kernel one warp: exact sum -> correctly rounded double ->
//                      gamma, and the magnitude threshold tau such that
//                      code != 0  <=>  |w| bits > tau;
//   qw_pack_kernel     re-reads W (L2-resident for the shapes served here),
//                      selects the kept positions, writes codes and meta.
#pragma once

#include "common.cuh"

namespace sbn {

// Workspace layout (bytes): [0, 2048) 256 x u64 exponent bins;
// [2048, 2052) u32 threshold tau. The rest is reserved.
constexpr int kQwBins = 256;
constexpr size_t kQwWorkspaceBytes = 4096;
constexpr size_t kQwTauOffset = kQwBins * sizeof(unsigned long long);

// In-register window of exponents [kWinLo, kWinLo + 31]: |w| in [2^-30, 4).
// Elements there are summed exactly into a per-thread u64 fixed-point
// accumulator (s << (e - kWinLo) < 2^39); all others go to shared bins.
constexpr uint32_t kWinLo = 97;

__global__ void __launch_bounds__(256)
qw_bins_kernel(const uint4* __restrict__ w, long long nchunks,
               unsigned long long* __restrict__ gbins) {
  __shared__ unsigned long long sbins[kQwBins];
  __shared__ unsigned long long swarp[8];
  for (int i = threadIdx.x; i < kQwBins; i += blockDim.x) sbins[i] = 0ull;
  __syncthreads();

  unsigned long long acc = 0ull;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long c = (long long)blockIdx.x * blockDim.x + threadIdx.x; c < nchunks; c += stride) {
    const uint4 v = __ldg(w + c);
    const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t mag = (wd[q] >> (16 * h)) & 0x7FFFu;
        const uint32_t e = mag >> 7;
        const uint32_t s = (mag & 0x7Fu) | (e ? 0x80u : 0u);
        const uint32_t eb = e ? e : 1u;
        const uint32_t sh = eb - kWinLo;
        if (sh < 32u) {
          acc += (unsigned long long)s << sh;
        } else if (s) {
          atomicAdd(&sbins[eb], (unsigned long long)s);
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) swarp[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long a = 0ull;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) a += swarp[i];
    // a is in units of 2^(kWinLo-134); file it as three 21-bit pieces under
    // exponents kWinLo, kWinLo+21 and kWinLo+42 so every bin stays small.
    const unsigned long long mask21 = (1ull << 21) - 1ull;
    const unsigned long long a0 = a & mask21, a1 = (a >> 21) & mask21, a2 = a >> 42;
    if (a0) atomicAdd(&gbins[kWinLo], a0);
    if (a1) atomicAdd(&gbins[kWinLo + 21], a1);
    if (a2) atomicAdd(&gbins[kWinLo + 42], a2);
  }
  for (int i = threadIdx.x; i < kQwBins; i += blockDim.x)
    if (sbins[i]) atomicAdd(&gbins[i], sbins[i]);
}

// Exact S = sum_e B[e] * 2^(e-134) (every B[e] < 2^40), rounded once to the
// nearest double (ties to even); returns 0.0 for S == 0. One thread.
SBN_DEVFN double exact_bins_to_double(const unsigned long long (&L)[16]) {
  // S_int = sum_l L[l] * 2^(16 l) with L[l] < 2^59; carry-propagate into
  // 16-bit words.
  uint32_t wd[20];
  unsigned long long carry = 0ull;
#pragma unroll
  for (int l = 0; l < 16; ++l) {
    const unsigned long long t = L[l] + carry;
    wd[l] = (uint32_t)(t & 0xFFFFull);
    carry = t >> 16;
  }
  wd[16] = (uint32_t)(carry & 0xFFFFull);
  wd[17] = (uint32_t)((carry >> 16) & 0xFFFFull);
  wd[18] = (uint32_t)((carry >> 32) & 0xFFFFull);
  wd[19] = (uint32_t)(carry >> 48);
  int P = -1;
  for (int p = 19; p >= 0; --p) {
    if (wd[p]) { P = p; break; }
  }
  if (P < 0) return 0.0;
  auto W = [&](int p) -> unsigned long long { return p >= 0 ? (unsigned long long)wd[p] : 0ull; };
  const unsigned long long hi = (W(P) << 48) | (W(P - 1) << 32) | (W(P - 2) << 16) | W(P - 3);
  const unsigned long long lo = W(P - 4);
  bool sticky = false;
  for (int p = P - 5; p >= 0; --p) sticky |= (wd[p] != 0u);
  const int lz = __clzll((long long)hi);  // 0..15: the top word is nonzero
  const unsigned long long T = lz ? ((hi << lz) | (lo >> (16 - lz))) : hi;
  const unsigned long long lorem = lz ? (lo & ((1ull << (16 - lz)) - 1ull)) : lo;
  sticky |= (lorem != 0ull) || ((T & 0x3FFull) != 0ull);
  unsigned long long mant = T >> 11;                // 53 bits, top bit set
  const unsigned long long rbit = (T >> 10) & 1ull;
  int ex = 16 * (P - 3) - lz + 11 - 133;            // S = mant * 2^ex
  if (rbit && (sticky || (mant & 1ull))) ++mant;
  if (mant == (1ull << 53)) { mant >>= 1; ++ex; }
  return ldexp((double)mant, ex);                    // exact scaling
}

// gamma = max(fl32(fl64(S) / n_elems), 1e-5); tau = the largest bf16
// magnitude b with fl32(b / gamma) <= 0.5 (rint then gives 0).
SBN_DEVFN void gamma_and_tau_from_bins(const unsigned long long* __restrict__ gbins,
                                       long long n_elems, float* g_out, uint32_t* tau_out) {
  // lanes 0..15 each fold 16 bins: L[l] = sum_i B[16 l + 1 + i] << i
  const int lane = threadIdx.x & 31;
  unsigned long long Ll = 0ull;
  if (lane < 16) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int e = 16 * lane + 1 + i;
      const unsigned long long b = (e <= 254) ? gbins[e] : 0ull;
      Ll += b << i;
    }
  }
  unsigned long long L[16];
#pragma unroll
  for (int l = 0; l < 16; ++l) L[l] = __shfl_sync(0xffffffffu, Ll, l);
  if (lane == 0) {
    const double d = exact_bins_to_double(L);
    const double q = __ddiv_rn(d, (double)n_elems);
    float g = __double2float_rn(q);
    g = fmaxf(g, 1e-5f);
    uint32_t lo_b = 0u, hi_b = 0x7F80u;  // pred(0) holds; pred(+inf) fails
    while (hi_b - lo_b > 1u) {
      const uint32_t mid = (lo_b + hi_b) >> 1;
      const float q32 = __fdiv_rn(__uint_as_float(mid << 16), g);
      if (q32 <= 0.5f) lo_b = mid; else hi_b = mid;
    }
    *g_out = g;
    *tau_out = lo_b;
  }
}

__global__ void __launch_bounds__(32)
qw_finalize_kernel(const unsigned long long* __restrict__ gbins, long long n_elems,
                   float* __restrict__ gamma_out, uint32_t* __restrict__ tau_out) {
  gamma_and_tau_from_bins(gbins, n_elems, gamma_out, tau_out);
}

// One warp per row; a row is processed in segments of 256 units (4096
// positions) staged in shared memory and flushed with 16-byte stores.
template <int M>
__global__ void __launch_bounds__(256)
qw_pack_kernel(const uint16_t* __restrict__ w, int n_out, int k, int n,
               const uint32_t* __restrict__ tau_ptr, uint8_t* __restrict__ codes,
               int codes_stride, uint8_t* __restrict__ meta, int meta_stride) {
  constexpr int kSeg = 256;
  __shared__ __align__(16) uint8_t s_codes[8][kSeg * 4];
  __shared__ __align__(16) uint8_t s_meta[8][kSeg * 2];
  const uint32_t tau = *tau_ptr;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cb = 4 * n / M;  // code bytes per unit of 16 positions
  const int units = k >> 4;
  const bool has_meta = (n != M);
  uint4* sc4 = reinterpret_cast<uint4*>(s_codes[warp]);
  const uint4* sm4 = reinterpret_cast<const uint4*>(s_meta[warp]);

  for (int row = blockIdx.x * 8 + warp; row < n_out; row += gridDim.x * 8) {
    const uint4* wrow = reinterpret_cast<const uint4*>(w + (size_t)row * k);
    for (int seg = 0; seg < units; seg += kSeg) {
      const int seg_units = min(kSeg, units - seg);
      for (int i = lane; i < kSeg * 4 / 16; i += 32) sc4[i] = make_uint4(0u, 0u, 0u, 0u);
      __syncwarp();
      for (int u = lane; u < seg_units; u += 32) {
        const uint4 a = __ldg(wrow + 2 * (seg + u));
        const uint4 b = __ldg(wrow + 2 * (seg + u) + 1);
        const uint32_t wd[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint32_t h[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          h[2 * i] = wd[i] & 0xFFFFu;
          h[2 * i + 1] = wd[i] >> 16;
        }
        uint32_t keep = 0u;
#pragma unroll
        for (int g = 0; g < 16 / M; ++g) {
          uint32_t mags[M];
#pragma unroll
          for (int i = 0; i < M; ++i) mags[i] = h[g * M + i] & 0x7FFFu;
          keep |= group_keep_bits<M>(mags, n) << (g * M);
        }
        uint32_t packed = 0u;
        int j = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          if ((keep >> i) & 1u) {
            const uint32_t c = ((h[i] & 0x7FFFu) > tau) ? ((h[i] & 0x8000u) ? 3u : 1u) : 0u;
            packed |= c << (2 * j);
            ++j;
          }
        }
        for (int bb = 0; bb < cb; ++bb) s_codes[warp][u * cb + bb] = (uint8_t)(packed >> (8 * bb));
        s_meta[warp][2 * u] = (uint8_t)(keep & 0xFFu);
        s_meta[warp][2 * u + 1] = (uint8_t)(keep >> 8);
      }
      __syncwarp();
      const int cstart = seg * cb;
      const int cend = min(cstart + kSeg * cb, codes_stride);
      uint4* cdst = reinterpret_cast<uint4*>(codes + (size_t)row * codes_stride + cstart);
      for (int i = lane; i < (cend - cstart) / 16; i += 32) cdst[i] = sc4[i];
      if (has_meta) {
        const int mstart = seg * 2;
        const int mend = min(mstart + kSeg * 2, meta_stride);
        uint4* mdst = reinterpret_cast<uint4*>(meta + (size_t)row * meta_stride + mstart);
        for (int i = lane; i < (mend - mstart) / 16; i += 32) mdst[i] = sm4[i];
      }
      __syncwarp();
    }
  }
}

}  // namespace sbn
