// sbn_quantize_weights in one persistent kernel (cooperative launch).
//
// Absmean quantizer: "BitNet b1.58: How Ternary Weights Cut LLM Memory by
// 82% Without Losing Accuracy", section "How ternary quantization works
// during training". Magnitude mask: "Sparse-BitNet: 1.58-bit LLMs are
// Naturally Friendly to Semi-Structured Sparsity", Abstract and Figure 6.
//
// gamma depends on the whole tensor while the codes depend on gamma, so the
// kernel has two phases around one grid-wide barrier:
//   phase 1  every CTA streams its rows of W from HBM once, adds every |w|
//            exactly into per-exponent bins and computes the keep mask of
//            every group (independent of gamma), written to meta;
//   barrier  an arrival counter in the workspace; the spin is bounded and
//            gives up with SBN_ERR_TIMEOUT in the device error word;
//   phase 2  every CTA turns the bins into gamma and the code threshold tau
//            (qw.cuh, one warp), re-reads its rows (now L2-resident) with the
//            mask, and writes the kept codes.
// The launch is cooperative, so all CTAs are resident and the barrier ends.
//
// Exact sum in phase 1: a bf16 magnitude with biased exponent e in
// [97, 129] lies in [2^-30, 8) and is a multiple of 2^-37. A thread adds such
// values into an fp64 accumulator; after at most 2048 of them the partial sum
// is below 2^14 and still a multiple of 2^-37, i.e. an integer times 2^-37
// below 2^51, so every fp64 addition was exact. The accumulator is then
// moved (exactly) into a u64 count of 2^-37 units and restarted. All other
// nonzero magnitudes go to shared per-exponent bins.
#pragma once

#include "common.cuh"
#include "qw.cuh"

namespace sbn {

// Workspace offsets beyond the bins and tau of qw.cuh.
constexpr size_t kQwArriveOffset = kQwTauOffset + 16;   // u32 arrival counter
constexpr long long kQwSpinLimit = 1ll << 24;            // ~1-2 s of polling
constexpr uint32_t kQwF64Lo = 97u << 7;                  // smallest magnitude bits in the fp64 window
constexpr uint32_t kQwF64Hi = 130u << 7;                 // first magnitude bits above it
constexpr int kQwFlush = 2048;                           // fp64 window values per flush (at most)

SBN_DEVFN uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// fp64 value of a normal bf16 magnitude (bits m, exponent field >= 1).
SBN_DEVFN double bf16_mag_to_f64(uint32_t m) {
  return __hiloint2double((int)((m << 13) + (896u << 20)), 0);
}

// Exact accumulation of one magnitude: fp64 window or shared bins.
SBN_DEVFN void qw_accumulate(uint32_t mag, double& dacc, unsigned long long* sbins) {
  if (mag - kQwF64Lo < kQwF64Hi - kQwF64Lo) {
    dacc += bf16_mag_to_f64(mag);
  } else if (mag) {
    const uint32_t e = mag >> 7;
    const uint32_t s = (mag & 0x7Fu) | (e ? 0x80u : 0u);
    atomicAdd(&sbins[e ? e : 1u], (unsigned long long)s);
  }
}

// Keep bits of 8 positions for m = 8 with exactly two pruned (6:8): the two
// smallest of the keys (|w| << 3 | (7 - i)) are dropped -- equal magnitudes
// drop the higher index first, i.e. keep the lower index.
SBN_DEVFN uint32_t keep_6of8(const uint32_t (&h)[8]) {
  uint32_t key[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) key[i] = ((h[i] & 0x7FFFu) << 3) | (7u - i);
  uint32_t m1 = key[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) m1 = min(m1, key[i]);
  uint32_t m2 = 0xFFFFFFFFu;
#pragma unroll
  for (int i = 0; i < 8; ++i) m2 = min(m2, key[i] == m1 ? 0xFFFFFFFFu : key[i]);
  return 0xFFu ^ (1u << (7u - (m1 & 7u))) ^ (1u << (7u - (m2 & 7u)));
}

// Keep bits of 4 positions for m = 4 with two kept (2:4): the two largest keys.
SBN_DEVFN uint32_t keep_2of4(const uint32_t (&h)[4]) {
  uint32_t key[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) key[i] = ((h[i] & 0x7FFFu) << 2) | (3u - i);
  const uint32_t a = max(key[0], key[1]), b = min(key[0], key[1]);
  const uint32_t c = max(key[2], key[3]), d = min(key[2], key[3]);
  const uint32_t t1 = max(a, c);
  const uint32_t t2 = max(min(a, c), max(b, d));
  return (1u << (3u - (t1 & 3u))) | (1u << (3u - (t2 & 3u)));
}

// Keep bits of one unit of 16 positions (groups of M), from the 16 bf16s.
template <int M>
SBN_DEVFN uint32_t unit_keep_bits(const uint32_t (&h)[16], int n) {
  uint32_t keep = 0u;
  if (M == 8 && n == 6) {
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      uint32_t hh[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) hh[i] = h[8 * g + i];
      keep |= keep_6of8(hh) << (8 * g);
    }
  } else if (M == 4 && n == 2) {
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      uint32_t hh[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) hh[i] = h[4 * g + i];
      keep |= keep_2of4(hh) << (4 * g);
    }
  } else {
#pragma unroll
    for (int g = 0; g < 16 / M; ++g) {
      uint32_t mags[M];
#pragma unroll
      for (int i = 0; i < M; ++i) mags[i] = h[g * M + i] & 0x7FFFu;
      keep |= group_keep_bits<M>(mags, n) << (g * M);
    }
  }
  return keep;
}

// Dense 2-bit codes of 16 positions (code of position i in bits 2i..2i+1):
// 01 where |w| > tau and w > 0, 11 where |w| > tau and w < 0, else 00. The
// comparison is one bf16x2 compare per pair of magnitudes.
SBN_DEVFN uint32_t dense_codes16(const uint32_t (&wd)[8], uint32_t tau) {
  const __nv_bfloat162 t2 = __halves2bfloat162(__ushort_as_bfloat16((unsigned short)tau),
                                               __ushort_as_bfloat16((unsigned short)tau));
  uint32_t d = 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t mg = wd[i] & 0x7FFF7FFFu;
    const uint32_t gt = __hgt2_mask(*reinterpret_cast<const __nv_bfloat162*>(&mg), t2);
    // per half: bit 0 = nonzero, bit 1 = nonzero and negative
    const uint32_t c = (gt & 0x00010001u) | ((gt & wd[i] & 0x80008000u) >> 14);
    d |= ((c & 3u) | ((c >> 14) & 0xCu)) << (4 * i);
  }
  return d;
}

// Remove one 2-bit field of x: fields below low_mask stay, higher ones move down.
SBN_DEVFN uint32_t remove_field(uint32_t x, uint32_t low_mask) {
  return (x & low_mask) | ((x >> 2) & ~low_mask);
}

// Kept codes, in order, of 16 positions from their dense codes and keep bits.
template <int M>
SBN_DEVFN uint32_t compact_codes16(uint32_t d, uint32_t keep, int n, const uint32_t* s_rm) {
  if (n == M) return d;
  if (M == 8 && n == 6) {
    // per byte of keep bits, remove the two pruned fields (higher one first)
    uint32_t out = 0u;
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      const uint32_t r = s_rm[(keep >> (8 * g)) & 0xFFu];  // low masks: q in bits 0-15, p in 16-31
      uint32_t x = (d >> (16 * g)) & 0xFFFFu;
      x = remove_field(x, r & 0xFFFFu);
      x = remove_field(x, r >> 16);
      out |= (x & 0xFFFu) << (12 * g);
    }
    return out;
  }
  uint32_t out = 0u;
  int j = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    if ((keep >> i) & 1u) {
      out |= ((d >> (2 * i)) & 3u) << (2 * j);
      ++j;
    }
  }
  return out;
}

// Removal masks of 6:8 groups: for keep byte k with pruned positions p < q,
// entry = lowmask(q) | lowmask(p) << 16 where lowmask(j) = (1 << 2j) - 1.
SBN_DEVFN void fill_remove_table(uint32_t* s_rm) {
  for (int k = threadIdx.x; k < 256; k += blockDim.x) {
    uint32_t pr = (~(uint32_t)k) & 0xFFu, p = 0u, q = 0u;
    if (__popc(pr) == 2) {
      p = __ffs(pr) - 1;
      pr &= pr - 1u;
      q = __ffs(pr) - 1;
    }
    s_rm[k] = ((1u << (2 * q)) - 1u) | (((1u << (2 * p)) - 1u) << 16);
  }
}

template <int M>
__global__ void __launch_bounds__(512, 1)
qw_fused_kernel(const uint16_t* __restrict__ w, int n_out, int k, int n,
                uint8_t* __restrict__ codes, int codes_stride, uint8_t* __restrict__ meta,
                int meta_stride, float* __restrict__ gamma_out, unsigned char* __restrict__ ws) {
  constexpr int kSeg = 256;  // units per staged code segment
  constexpr int kWarps = 16;
  constexpr int kAhead = 4;  // units in flight per lane in phase 1
  __shared__ unsigned long long sbins[kQwBins];
  __shared__ unsigned long long swarp[kWarps];
  __shared__ __align__(16) uint8_t s_codes[kWarps][kSeg * 4];
  __shared__ uint32_t s_rm[256];
  __shared__ uint32_t s_tau;
  __shared__ int s_abort;

  unsigned long long* gbins = reinterpret_cast<unsigned long long*>(ws);
  uint32_t* arrive = reinterpret_cast<uint32_t*>(ws + kQwArriveOffset);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int units = k >> 4;
  const bool has_meta = (n != M);
  const int rows_per_cta = (n_out + gridDim.x - 1) / gridDim.x;
  const int r_begin = min(n_out, (int)blockIdx.x * rows_per_cta);
  const int r_end = min(n_out, r_begin + rows_per_cta);

  for (int i = threadIdx.x; i < kQwBins; i += blockDim.x) sbins[i] = 0ull;
  if (M == 8 && n == 6) fill_remove_table(s_rm);
  __syncthreads();

  // ---- phase 1: exact sum and keep masks ------------------------------------
  double dacc = 0.0;
  int dcount = 0;                  // window values since the last flush
  unsigned long long uacc = 0ull;  // flushed sum in units of 2^-37
  for (int row = r_begin + warp; row < r_end; row += kWarps) {
    const uint4* wrow = reinterpret_cast<const uint4*>(w + (size_t)row * k);
    for (int u0 = lane; u0 < units; u0 += 32 * kAhead) {
      uint4 va[kAhead], vb[kAhead];
#pragma unroll
      for (int j = 0; j < kAhead; ++j) {
        const int u = u0 + 32 * j;
        if (u < units) {
          va[j] = __ldg(wrow + 2 * u);
          vb[j] = __ldg(wrow + 2 * u + 1);
        }
      }
#pragma unroll
      for (int j = 0; j < kAhead; ++j) {
        const int u = u0 + 32 * j;
        if (u >= units) break;
        const uint32_t wd[8] = {va[j].x, va[j].y, va[j].z, va[j].w, vb[j].x, vb[j].y, vb[j].z, vb[j].w};
        uint32_t h[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          h[2 * i] = wd[i] & 0xFFFFu;
          h[2 * i + 1] = wd[i] >> 16;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) qw_accumulate(h[i] & 0x7FFFu, dacc, sbins);
        dcount += 16;
        if (dcount > kQwFlush - 16) {
          uacc += (unsigned long long)__double2ull_rz(dacc * 137438953472.0);  // * 2^37, exact
          dacc = 0.0;
          dcount = 0;
        }
        if (has_meta) {
          const uint32_t keep = unit_keep_bits<M>(h, n);
          *reinterpret_cast<uint16_t*>(meta + (size_t)row * meta_stride + 2 * u) = (uint16_t)keep;
        }
      }
    }
  }
  uacc += (unsigned long long)__double2ull_rz(dacc * 137438953472.0);
#pragma unroll
  for (int o = 16; o; o >>= 1) uacc += __shfl_xor_sync(0xffffffffu, uacc, o);
  if (lane == 0) swarp[warp] = uacc;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long a = 0ull;
    for (int i = 0; i < kWarps; ++i) a += swarp[i];
    // a counts units of 2^-37 = 2^(97-134): file it under exponents 97, 118
    // and 139 in 21-bit pieces so every bin stays small
    const unsigned long long mask21 = (1ull << 21) - 1ull;
    const unsigned long long a0 = a & mask21, a1 = (a >> 21) & mask21, a2 = a >> 42;
    if (a0) atomicAdd(&gbins[97], a0);
    if (a1) atomicAdd(&gbins[118], a1);
    if (a2) atomicAdd(&gbins[139], a2);
  }
  for (int i = threadIdx.x; i < kQwBins; i += blockDim.x)
    if (sbins[i]) atomicAdd(&gbins[i], sbins[i]);

  // ---- grid barrier (bounded) -----------------------------------------------
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    atomicAdd(arrive, 1u);
    long long spins = 0;
    int abort = 0;
    while (ld_acquire_u32(arrive) < gridDim.x) {
      if (++spins > kQwSpinLimit) {
        atomicOr(&g_dev_error, kDevErrTimeout);
        abort = 1;
        break;
      }
      __nanosleep(64);
    }
    s_abort = abort;
  }
  __syncthreads();
  if (s_abort) return;
  __threadfence();

  // ---- gamma and the code threshold (every CTA, one warp) -------------------
  if (warp == 0) {
    float g;
    uint32_t tau;
    gamma_and_tau_from_bins(gbins, (long long)n_out * k, &g, &tau);
    if (lane == 0) {
      s_tau = tau;
      if (blockIdx.x == 0) *gamma_out = g;
    }
  }
  __syncthreads();
  const uint32_t tau = s_tau;

  // ---- phase 2: codes of the kept positions ---------------------------------
  const int cb = 4 * n / M;
  uint4* sc4 = reinterpret_cast<uint4*>(s_codes[warp]);
  for (int row = r_begin + warp; row < r_end; row += kWarps) {
    const uint4* wrow = reinterpret_cast<const uint4*>(w + (size_t)row * k);
    const uint16_t* mrow = reinterpret_cast<const uint16_t*>(meta + (size_t)row * meta_stride);
    for (int seg = 0; seg < units; seg += kSeg) {
      const int seg_units = min(kSeg, units - seg);
      for (int i = lane; i < kSeg * 4 / 16; i += 32) sc4[i] = make_uint4(0u, 0u, 0u, 0u);
      __syncwarp();
      for (int u = lane; u < seg_units; u += 32) {
        const uint4 a = __ldg(wrow + 2 * (seg + u));
        const uint4 b = __ldg(wrow + 2 * (seg + u) + 1);
        const uint32_t wd[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        const uint32_t keep = has_meta ? (uint32_t)mrow[seg + u] : 0xFFFFu;
        const uint32_t packed = compact_codes16<M>(dense_codes16(wd, tau), keep, n, s_rm);
        for (int bb = 0; bb < cb; ++bb) s_codes[warp][u * cb + bb] = (uint8_t)(packed >> (8 * bb));
      }
      __syncwarp();
      const int cstart = seg * cb;
      const int cend = min(cstart + kSeg * cb, codes_stride);
      uint4* cdst = reinterpret_cast<uint4*>(codes + (size_t)row * codes_stride + cstart);
      for (int i = lane; i < (cend - cstart) / 16; i += 32) cdst[i] = sc4[i];
      __syncwarp();
    }
  }
}

}  // namespace sbn
