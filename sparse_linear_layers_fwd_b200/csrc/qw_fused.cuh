// sbn_quantize_weights in one persistent kernel (cooperative launch).
//
// Absmean quantizer: "BitNet b1.58: How Ternary Weights Cut LLM Memory by
// 82% Without Losing Accuracy", section "How ternary quantization works
// during training". Magnitude mask: "Sparse-BitNet: 1.58-bit LLMs are
// Naturally Friendly to Semi-Structured Sparsity", Abstract and Figure 6.
//
// gamma depends on the whole tensor while the codes depend on gamma, so the
// kernel has two phases around a grid-wide barrier:
//   phase 1  every CTA streams its rows of W from HBM once, sums |w| in fp64
//            and computes the keep mask of every group (independent of
//            gamma), written to meta;
//   barrier  an arrival counter in the workspace; the spin is bounded and
//            gives up with SBN_ERR_TIMEOUT in the device error word;
//   gamma    every CTA reads the fp64 total S'. Its rounding error has a
//            rigorous bound (positive terms: |S' - S| <= (additions on the
//            longest path) * 2^-53 * S', plus 2^-126 per zero or subnormal
//            |w|, which the fp64 construction below maps near 2^-127). If the
//            whole interval of possible exact means rounds to one fp32 value,
//            that value is gamma = max(fl32(fl64(S) / (N_out*K)), 1e-5). Else
//            (an exact mean within ~2^-40 of an fp32 rounding midpoint, rare)
//            every CTA re-reads its rows and adds every |w| exactly into
//            integer bins, a second barrier follows, and gamma comes from the
//            exact bins (qw.cuh);
//   phase 2  every CTA derives the code threshold tau, re-reads its rows
//            (now L2-resident) with the mask and writes the kept codes.
// The launch is cooperative, so all CTAs are resident and the barriers end.
#pragma once

#include "async.cuh"
#include "common.cuh"
#include "qw.cuh"

namespace sbn {

// Workspace offsets beyond the bins and tau of qw.cuh.
constexpr size_t kQwArriveOffset = kQwTauOffset + 16;   // u32 arrival counter
constexpr size_t kQwSumOffset = kQwArriveOffset + 16;   // f64 total of |w|
constexpr size_t kQwClearBytes = kQwSumOffset + 16;     // cleared before every launch
constexpr unsigned long long kQwWaitNs = 1000000000ull;  // the grid barrier gives up after 1 s

SBN_DEVFN uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// High word of the fp64 value of a bf16 magnitude given as bits 16-30 of a
// 32-bit word shifted down by 3 (exponent rebias 127 -> 1023); exact for
// normal magnitudes, near 2^-127 for zero and subnormals.
constexpr uint32_t kF64Rebias = 896u << 20;

// Bounded grid barrier: thread 0 of every CTA arrives and waits until the
// counter reaches target. Returns false (and records a timeout) on give-up.
SBN_DEVFN bool grid_barrier(uint32_t* arrive, uint32_t target, int* s_abort) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    atomicAdd(arrive, 1u);
    const unsigned long long t0 = global_ns();
    int abort = 0;
    while (ld_acquire_u32(arrive) < target) {
      if (global_ns() - t0 > kQwWaitNs) {
        atomicOr(&g_dev_error, kDevErrTimeout);
        abort = 1;
        break;
      }
      __nanosleep(64);
    }
    *s_abort = abort;
  }
  __syncthreads();
  const bool ok = !*s_abort;
  __threadfence();
  return ok;
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

// Launch shape and dynamic shared memory of qw_fused_kernel. Every CTA owns a
// contiguous range of units (16 consecutive weights of one row, 32 bytes),
// i.e. one contiguous byte range of W, and streams it through a ring of
// 16 KB stages filled by bulk copies: one stage is 512 units, one per thread.
constexpr int kQwThreads = 512;
constexpr int kQwWarps = kQwThreads / 32;
constexpr int kQwChunk = 16384;       // bytes per stage
constexpr int kQwStages = 8;          // 128 KB in flight per SM
constexpr int kQwKeepCap = 16384;     // units whose keep bits stay in shared memory
constexpr size_t kQwSmKeep = (size_t)kQwStages * kQwChunk;
constexpr size_t kQwSmRm = kQwSmKeep + (size_t)kQwKeepCap * 2;
constexpr size_t kQwSmBins = kQwSmRm + 256 * 4;
constexpr size_t kQwSmBars = kQwSmBins + (size_t)kQwBins * 8;
constexpr size_t kQwSmemBytes = kQwSmBars + (size_t)kQwStages * 8;

// Stream ring over one CTA's byte range of W.
struct QwRing {
  const uint8_t* src;   // first byte of the range
  long long bytes;      // length (a multiple of 32)
  int nch;              // chunks in the range
  uint8_t* buf;         // kQwStages x kQwChunk
  uint64_t* full;       // one mbarrier per stage
  uint32_t seq;         // chunks consumed so far, over all passes (uniform)
};

SBN_DEVFN void qw_issue(const QwRing& r, int c, uint32_t q) {
  const int st = (int)(q % kQwStages);
  const long long off = (long long)c * kQwChunk;
  const uint32_t nb = (uint32_t)min((long long)kQwChunk, r.bytes - off);
  mbar_arrive_expect_tx(&r.full[st], nb);
  bulk_g2s(r.buf + (size_t)st * kQwChunk, r.src + off, nb, &r.full[st]);
}

// Issues the first stages of the next pass (thread 0).
SBN_DEVFN void qw_prologue(const QwRing& r) {
  if (threadIdx.x == 0)
    for (int c = 0; c < min(r.nch, kQwStages); ++c) qw_issue(r, c, r.seq + (uint32_t)c);
}

// One pass over the range, whose prologue is already issued: f(c, stage,
// units_here) runs for every chunk on every thread, then the stage is
// refilled with chunk c + kQwStages. If a wait gives up, the copies still in
// flight are waited for (bounded) and false is returned on every thread.
template <class F>
SBN_DEVFN bool qw_pass(QwRing& r, F&& f) {
  for (int c = 0; c < r.nch; ++c) {
    const uint32_t q = r.seq + (uint32_t)c;
    const int st = (int)(q % kQwStages);
    const bool ok = mbar_wait(&r.full[st], (q / kQwStages) & 1u);
    const int units_here = (int)(min((long long)kQwChunk, r.bytes - (long long)c * kQwChunk) >> 5);
    if (ok) f(c, r.buf + (size_t)st * kQwChunk, units_here);
    if (__syncthreads_or(!ok)) {
      if (threadIdx.x == 0) {
        for (int d = c + 1; d < min(r.nch, c + kQwStages); ++d) {
          const uint32_t qd = r.seq + (uint32_t)d;
          if (!mbar_wait(&r.full[qd % kQwStages], (qd / kQwStages) & 1u)) break;
        }
      }
      __syncthreads();
      return false;
    }
    if (threadIdx.x == 0 && c + kQwStages < r.nch) qw_issue(r, c + kQwStages, q + kQwStages);
  }
  r.seq += (uint32_t)r.nch;
  return true;
}

// This thread's unit of a stage, read without bank conflicts: lanes 4-7 of
// every quarter-warp fetch their upper half first.
SBN_DEVFN void qw_load_unit(const uint8_t* stage, int t, uint32_t (&wd)[8]) {
  const uint4* p = reinterpret_cast<const uint4*>(stage) + 2 * t;
  const int sw = (t >> 2) & 1;
  const uint4 a = p[sw], b = p[sw ^ 1];
  const uint4 lo = sw ? b : a, hi = sw ? a : b;
  wd[0] = lo.x; wd[1] = lo.y; wd[2] = lo.z; wd[3] = lo.w;
  wd[4] = hi.x; wd[5] = hi.y; wd[6] = hi.z; wd[7] = hi.w;
}

template <int M>
__global__ void __launch_bounds__(kQwThreads, 1)
qw_fused_kernel(const uint16_t* __restrict__ w, int n_out, int k, int n,
                uint8_t* __restrict__ codes, int codes_stride, uint8_t* __restrict__ meta,
                int meta_stride, float* __restrict__ gamma_out, unsigned char* __restrict__ ws) {
  extern __shared__ __align__(128) uint8_t qw_smem[];
  uint16_t* s_keep = reinterpret_cast<uint16_t*>(qw_smem + kQwSmKeep);
  uint32_t* s_rm = reinterpret_cast<uint32_t*>(qw_smem + kQwSmRm);
  unsigned long long* sbins = reinterpret_cast<unsigned long long*>(qw_smem + kQwSmBins);
  uint64_t* full = reinterpret_cast<uint64_t*>(qw_smem + kQwSmBars);
  __shared__ double swarp_d[kQwWarps];
  __shared__ unsigned long long swarp[kQwWarps];
  __shared__ uint32_t s_tau;
  __shared__ int s_abort, s_exact;

  unsigned long long* gbins = reinterpret_cast<unsigned long long*>(ws);
  uint32_t* arrive = reinterpret_cast<uint32_t*>(ws + kQwArriveOffset);
  double* gsum = reinterpret_cast<double*>(ws + kQwSumOffset);

  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int upr = k >> 4;                       // units per row
  const long long total_units = (long long)n_out * upr;
  const long long u_begin = (long long)blockIdx.x * total_units / gridDim.x;
  const long long u_end = (long long)(blockIdx.x + 1) * total_units / gridDim.x;
  const bool has_meta = (n != M);
  const int cb = 4 * n / M;                     // code bytes per unit
  const int row_step = kQwThreads / upr, u_step = kQwThreads % upr;

  QwRing ring;
  ring.src = reinterpret_cast<const uint8_t*>(w) + u_begin * 32;
  ring.bytes = (u_end - u_begin) * 32;
  ring.nch = (int)((ring.bytes + kQwChunk - 1) / kQwChunk);
  ring.buf = qw_smem;
  ring.full = full;
  ring.seq = 0u;

  if (t == 0) {
    for (int s = 0; s < kQwStages; ++s) mbar_init(&full[s], 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (M == 8 && n == 6) fill_remove_table(s_rm);
  __syncthreads();
  qw_prologue(ring);

  // (row, u) of this thread's unit in chunk c, advanced chunk by chunk
  int row0, u0;
  {
    const long long g = u_begin + t;
    row0 = (int)(g / upr);
    u0 = (int)(g - (long long)row0 * upr);
  }
  auto advance = [&](int& row, int& u) {
    row += row_step;
    u += u_step;
    if (u >= upr) { u -= upr; ++row; }
  };

  // ---- phase 1: fp64 sum and keep masks -------------------------------------
  double d0 = 0.0, d1 = 0.0;
  {
    int row = row0, u = u0;
    const bool ok = qw_pass(ring, [&](int c, const uint8_t* stage, int units_here) {
      if (t < units_here) {
        uint32_t wd[8];
        qw_load_unit(stage, t, wd);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          d0 += __hiloint2double((int)(((wd[i] & 0x7FFFu) << 13) + kF64Rebias), 0);
          d1 += __hiloint2double((int)(((wd[i] >> 3) & 0x0FFFE000u) + kF64Rebias), 0);
        }
        if (has_meta) {
          uint32_t h[16];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            h[2 * i] = wd[i] & 0xFFFFu;
            h[2 * i + 1] = wd[i] >> 16;
          }
          const uint32_t keep = unit_keep_bits<M>(h, n);
          *reinterpret_cast<uint16_t*>(meta + (size_t)row * meta_stride + 2 * u) = (uint16_t)keep;
          const int li = c * kQwThreads + t;
          if (li < kQwKeepCap) s_keep[li] = (uint16_t)keep;
        }
      }
      advance(row, u);
    });
    if (!ok) return;
  }
  double dsum = d0 + d1;
#pragma unroll
  for (int o = 16; o; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
  if (lane == 0) swarp_d[warp] = dsum;
  __syncthreads();
  if (t == 0) {
    double a = 0.0;
    for (int i = 0; i < kQwWarps; ++i) a += swarp_d[i];
    atomicAdd(gsum, a);
  }
  // the second pass re-reads the same range (now mostly in L2): start it
  // before the grid barrier
  qw_prologue(ring);
  if (!grid_barrier(arrive, gridDim.x, &s_abort)) {
    qw_pass(ring, [](int, const uint8_t*, int) {});   // drain the prefetched stages
    return;
  }

  // ---- gamma: certified from the fp64 total, else exact ---------------------
  if (t == 0) {
    const double S = __ldcg(gsum);
    const double nk = (double)n_out * (double)k;
    // additions on the longest path: per-thread accumulator (8 per unit, one
    // unit per chunk), d0 + d1, warp tree, CTA sum, one global atomic per CTA
    const long long max_units = (total_units + gridDim.x - 1) / gridDim.x;
    const double per_thread = 8.0 * (double)((max_units + kQwThreads - 1) / kQwThreads);
    const double adds = per_thread + 1.0 + 5.0 + kQwWarps + (double)gridDim.x;
    const double err = S * adds * 0x1p-53 * 1.01 + nk * 0x1p-126 * 1.01;
    const double lo = (S - err) / nk * (1.0 - 0x1p-50);
    const double hi = (S + err) / nk * (1.0 + 0x1p-50);
    const float glo = fmaxf(__double2float_rn(lo), 1e-5f);
    const float ghi = fmaxf(__double2float_rn(hi), 1e-5f);
    s_exact = (glo == ghi) ? 0 : 1;
    if (!s_exact) {
      s_tau = code_threshold(glo);
      if (blockIdx.x == 0) *gamma_out = glo;
    }
  }
  __syncthreads();
  if (s_exact) {
    // rare: exact integer bins over the same range, second barrier
    for (int i = t; i < kQwBins; i += kQwThreads) sbins[i] = 0ull;
    __syncthreads();
    unsigned long long acc = 0ull;
    const bool ok = qw_pass(ring, [&](int, const uint8_t* stage, int units_here) {
      if (t < units_here) {
        uint32_t wd[8];
        qw_load_unit(stage, t, wd);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          exact_accumulate(wd[i] & 0x7FFFu, acc, sbins);
          exact_accumulate((wd[i] >> 16) & 0x7FFFu, acc, sbins);
        }
      }
    });
    if (!ok) return;
#pragma unroll
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) swarp[warp] = acc;
    __syncthreads();
    if (t == 0) {
      unsigned long long a = 0ull;
      for (int i = 0; i < kQwWarps; ++i) a += swarp[i];
      // a counts units of 2^(kWinLo-134): file it under exponents kWinLo,
      // kWinLo+21 and kWinLo+42 in 21-bit pieces so every bin stays small
      const unsigned long long mask21 = (1ull << 21) - 1ull;
      const unsigned long long a0 = a & mask21, a1 = (a >> 21) & mask21, a2 = a >> 42;
      if (a0) atomicAdd(&gbins[kWinLo], a0);
      if (a1) atomicAdd(&gbins[kWinLo + 21], a1);
      if (a2) atomicAdd(&gbins[kWinLo + 42], a2);
    }
    for (int i = t; i < kQwBins; i += kQwThreads)
      if (sbins[i]) atomicAdd(&gbins[i], sbins[i]);
    qw_prologue(ring);
    if (!grid_barrier(arrive, 2u * gridDim.x, &s_abort)) {
      qw_pass(ring, [](int, const uint8_t*, int) {});
      return;
    }
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
  }
  const uint32_t tau = s_tau;

  // ---- phase 2: codes of the kept positions ---------------------------------
  {
    int row = row0, u = u0;
    qw_pass(ring, [&](int c, const uint8_t* stage, int units_here) {
      if (t < units_here) {
        uint32_t wd[8];
        qw_load_unit(stage, t, wd);
        uint32_t keep = 0xFFFFu;
        if (has_meta) {
          const int li = c * kQwThreads + t;
          keep = (li < kQwKeepCap)
                     ? (uint32_t)s_keep[li]
                     : (uint32_t) * reinterpret_cast<const uint16_t*>(meta + (size_t)row * meta_stride + 2 * u);
        }
        const uint32_t packed = compact_codes16<M>(dense_codes16(wd, tau), keep, n, s_rm);
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
      advance(row, u);
    });
  }
}

}  // namespace sbn
