// sbn_quantize_weights kernels: exact absmean gamma, N:M mask, ternary codes, packing.
//
// Absmean quantizer: "BitNet b1.58: How Ternary Weights Cut LLM Memory by 82%
// Without Losing Accuracy", section "How ternary quantization works during
// training" (divide by the mean |W|, round, clamp to [-1, 1]). Magnitude
// mask: "Sparse-BitNet: 1.58-bit LLMs are Naturally Friendly to
// Semi-Structured Sparsity", Abstract and Figure 6 (threshold t = |w|_(N+1)).
//
// Exact helpers shared by the weight quantizer (qw_fused.cuh): the workspace
// layout, the exact conversion of per-exponent bins of |w| into a correctly
// rounded double, gamma, and the code threshold tau such that
// code != 0  <=>  |w| bits > tau.
#pragma once

#include "common.cuh"

namespace sbn {

// Workspace layout (bytes): [0, 2048) 256 x u64 exponent bins;
// [2048, 2052) u32 threshold tau. The rest is reserved.
constexpr int kQwBins = 256;
constexpr size_t kQwWorkspaceBytes = 4096;
constexpr size_t kQwTauOffset = kQwBins * sizeof(unsigned long long);

// Exact window of the rare exact pass: exponents [kWinLo, kWinLo + 31],
// |w| in [2^-30, 4), summed into a per-thread u64 fixed-point accumulator
// (s << (e - kWinLo) < 2^39); all other magnitudes go to shared bins.
constexpr uint32_t kWinLo = 97;

// One magnitude into the exact accumulators (u64 window or shared bins).
SBN_DEVFN void exact_accumulate(uint32_t mag, unsigned long long& acc, unsigned long long* sbins) {
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

// The largest bf16 magnitude b with fl32(b / g) <= 0.5 (rint then gives 0):
// start from the largest bf16 <= g/2 (fl32(b/g) <= 0.5 there since division
// rounds monotonically) and step up while the next one still rounds to <= 0.5
// (at most twice: two bf16 steps above g/2 the quotient exceeds 0.5 by more
// than an fp32 rounding).
SBN_DEVFN uint32_t code_threshold(float g) {
  uint32_t b = __float_as_uint(__fmul_rn(0.5f, g)) >> 16;
  if (b > 0x7F7Eu) b = 0x7F7Eu;
  while (b < 0x7F7Fu && __fdiv_rn(__uint_as_float((b + 1u) << 16), g) <= 0.5f) ++b;
  return b;
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
      const unsigned long long b = (e <= 254) ? __ldcg(gbins + e) : 0ull;
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
    const uint32_t lo_b = code_threshold(g);
    *g_out = g;
    *tau_out = lo_b;
  }
}

}  // namespace sbn
