// sbn_quantize_weights in one persistent kernel (cooperative launch), the
// latent weights streamed straight into registers.
//
// Absmean quantizer: "BitNet b1.58: How Ternary Weights Cut LLM Memory by
// 82% Without Losing Accuracy", section "How ternary quantization works
// during training". Magnitude mask: "Sparse-BitNet: 1.58-bit LLMs are
// Naturally Friendly to Semi-Structured Sparsity", Abstract and Figure 6.
//
// gamma depends on the whole tensor while the codes depend on gamma, so the
// kernel has two passes around a grid-wide barrier (the steps are those of
// qw_fused.cuh, whose helpers it uses):
//   pass 1   every CTA reads its contiguous range of units (16 consecutive
//            weights of a row, 32 bytes) from HBM, sums |w| in fp64, and
//            computes and writes the keep mask of every group (independent
//            of gamma), keeping it in shared memory for pass 2;
//   barrier  an arrival counter in the workspace, bounded in time;
//   gamma    certified from the fp64 total when its rounding is fixed by the
//            error bound, else (an exact mean next to an fp32 midpoint) an
//            exact integer-bin pass over the range and a second barrier;
//   pass 2   every CTA re-reads its range (now in L2) and writes the codes.
// Every thread takes two units of each 1024-unit slice of the range and
// issues the next slice's 16-byte loads before it works on the current one,
// so four units per thread are in flight. Plain loads keep up with HBM
// where one thread's bulk copies into shared memory did not: on this part
// the copy engine paced both passes at well below the memory's rate.
#pragma once

#include "common.cuh"
#include "qw.cuh"
#include "qw_fused.cuh"

namespace sbn {

constexpr int kQsThreads = 512;
constexpr int kQsWarps = kQsThreads / 32;
constexpr int kQsSlice = 2 * kQsThreads;   // units per slice: two per thread
constexpr int kQsKeepCap = 16384;          // units whose keep bits stay in shared memory

// Bounded grid barrier: thread 0 of every CTA arrives and waits until the
// counter reaches target. Returns false on every thread (and records a
// timeout) if the wait gave up.
SBN_DEVFN bool qs_grid_barrier(uint32_t* arrive, uint32_t target, int* s_abort,
                               unsigned long long limit_ns = kQwWaitNs) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;\n" ::"l"(arrive) : "memory");
    const unsigned long long t0 = global_ns();
    int abort = 0;
    while (ld_acquire_u32(arrive) < target) {
      if (global_ns() - t0 > limit_ns) {
        atomicOr(&g_dev_error, kDevErrTimeout);
        abort = 1;
        break;
      }
      __nanosleep(32);
    }
    *s_abort = abort;
  }
  __syncthreads();
  const bool ok = !*s_abort;
  __threadfence();
  return ok;
}

// The two units (u0 = slice base + t, u1 = u0 + 512) of slice s of the range:
// four 16-byte loads, predicated on the range.
struct QsPair {
  uint4 a0, a1, b0, b1;
};

SBN_DEVFN void qs_load(const uint4* __restrict__ src, int nu, int s, int t, QsPair& p) {
  const int u0 = s * kQsSlice + t, u1 = u0 + kQsThreads;
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  p.a0 = u0 < nu ? __ldg(src + 2 * u0) : z;
  p.a1 = u0 < nu ? __ldg(src + 2 * u0 + 1) : z;
  p.b0 = u1 < nu ? __ldg(src + 2 * u1) : z;
  p.b1 = u1 < nu ? __ldg(src + 2 * u1 + 1) : z;
}

SBN_DEVFN void qs_words(const uint4& lo, const uint4& hi, uint32_t (&wd)[8]) {
  wd[0] = lo.x; wd[1] = lo.y; wd[2] = lo.z; wd[3] = lo.w;
  wd[4] = hi.x; wd[5] = hi.y; wd[6] = hi.z; wd[7] = hi.w;
}

template <int M>
__global__ void __launch_bounds__(kQsThreads, 1)
qw_stream_kernel(const uint16_t* __restrict__ w, int n_out, int k, int n,
                 uint8_t* __restrict__ codes, int codes_stride, uint8_t* __restrict__ meta,
                 int meta_stride, float* __restrict__ gamma_out, unsigned char* __restrict__ ws) {
  __shared__ uint16_t s_keep[kQsKeepCap];
  __shared__ uint32_t s_csel[256];
  __shared__ unsigned long long sbins[kQwBins];
  __shared__ double swarp_d[kQsWarps];
  __shared__ unsigned long long swarp[kQsWarps];
  __shared__ uint32_t s_tau;
  __shared__ int s_abort, s_exact;

  unsigned long long* gbins = reinterpret_cast<unsigned long long*>(ws);
  uint32_t* arrive = reinterpret_cast<uint32_t*>(ws + kQwArriveOffset);
  double* gpart = reinterpret_cast<double*>(ws + kQwPartOffset);

  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int upr = k >> 4;                        // units per row
  const long long total_units = (long long)n_out * upr;
  // CTA ranges start on 128-byte boundaries (4 units)
  auto range_start = [&](long long b) {
    return b >= (long long)gridDim.x ? total_units : (b * total_units / gridDim.x) & ~3LL;
  };
  const long long u_begin = range_start(blockIdx.x);
  const int nu = (int)(range_start(blockIdx.x + 1) - u_begin);   // < 2^27
  const int nslices = (nu + kQsSlice - 1) / kQsSlice;
  const uint4* src = reinterpret_cast<const uint4*>(w) + 2 * u_begin;
  const bool has_meta = (n != M);
  const int cb = 4 * n / M;                      // code bytes per unit
  const int row_step = kQsSlice / upr, u_step = kQsSlice % upr;

  fill_compact_table(s_csel);
  // (row, u) of this thread's two units in slice 0, advanced slice by slice
  int row0[2], u0[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const long long g = u_begin + t + (long long)kQsThreads * j;
    row0[j] = (int)(g / upr);
    u0[j] = (int)(g - (long long)row0[j] * upr);
  }
  auto advance = [&](int& row, int& u) {
    row += row_step;
    u += u_step;
    if (u >= upr) { u -= upr; ++row; }
  };

  // ---- pass 1: fp64 sum and keep masks -------------------------------------
  double dacc[2][4];
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int a = 0; a < 4; ++a) dacc[j][a] = 0.0;
  {
    int row[2] = {row0[0], row0[1]}, u[2] = {u0[0], u0[1]};
    QsPair cur, nxt;
    qs_load(src, nu, 0, t, cur);
    for (int s = 0; s < nslices; ++s) {
      if (s + 1 < nslices) qs_load(src, nu, s + 1, t, nxt);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int ui = s * kQsSlice + t + kQsThreads * j;
        if (ui < nu) {
          uint32_t wd[8], mw[8];
          if (j == 0) qs_words(cur.a0, cur.a1, wd); else qs_words(cur.b0, cur.b1, wd);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            mw[i] = wd[i] & 0x7FFF7FFFu;
            dacc[j][(2 * i) & 3] += __hiloint2double((int)(((mw[i] & 0xFFFFu) << 13) + kF64Rebias), 0);
            dacc[j][(2 * i + 1) & 3] += __hiloint2double((int)(((mw[i] >> 16) << 13) + kF64Rebias), 0);
          }
          if (has_meta) {
            const uint32_t keep = unit_keep_fast<M>(mw, n);
            *reinterpret_cast<uint16_t*>(meta + (size_t)row[j] * meta_stride + 2 * u[j]) = (uint16_t)keep;
            if (ui < kQsKeepCap) s_keep[ui] = (uint16_t)keep;
          }
        }
        advance(row[j], u[j]);
      }
      cur = nxt;
    }
  }
  double dsum = ((dacc[0][0] + dacc[0][1]) + (dacc[0][2] + dacc[0][3])) +
                ((dacc[1][0] + dacc[1][1]) + (dacc[1][2] + dacc[1][3]));
#pragma unroll
  for (int o = 16; o; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
  if (lane == 0) swarp_d[warp] = dsum;
  __syncthreads();
  if (t == 0) {
    double a = 0.0;
    for (int i = 0; i < kQsWarps; ++i) a += swarp_d[i];
    gpart[blockIdx.x] = a;
  }
  if (!qs_grid_barrier(arrive, gridDim.x, &s_abort)) return;

  // ---- gamma: certified from the fp64 total, else exact ---------------------
  // the CTA partials, summed in the same fixed order by every CTA
  {
    double v = (t < (int)gridDim.x) ? __ldcg(gpart + t) : 0.0;
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) swarp_d[warp] = v;
  }
  __syncthreads();
  if (t == 0) {
    double S = 0.0;
    for (int i = 0; i < kQsWarps; ++i) S += swarp_d[i];
    const double nk = (double)n_out * (double)k;
    // additions on the longest path: one accumulator chain (4 per unit, at
    // most one unit per slot and slice), the 3-level tree over the 8
    // chains, the warp tree, the warp sums of the CTA, then the same two
    // levels over the CTA partials (counted generously)
    const long long max_units = (total_units + gridDim.x - 1) / gridDim.x + 4;   // aligned ranges
    const double per_thread = 4.0 * (double)((max_units + kQsThreads - 1) / kQsThreads);
    const double adds = per_thread + 3.0 + 2.0 * (5.0 + kQsWarps) + (double)gridDim.x;
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
    for (int i = t; i < kQwBins; i += kQsThreads) sbins[i] = 0ull;
    __syncthreads();
    unsigned long long acc = 0ull;
    for (int s = 0; s < nslices; ++s) {
      QsPair cur;
      qs_load(src, nu, s, t, cur);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int ui = s * kQsSlice + t + kQsThreads * j;
        if (ui < nu) {
          uint32_t wd[8];
          if (j == 0) qs_words(cur.a0, cur.a1, wd); else qs_words(cur.b0, cur.b1, wd);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            exact_accumulate(wd[i] & 0x7FFFu, acc, sbins);
            exact_accumulate((wd[i] >> 16) & 0x7FFFu, acc, sbins);
          }
        }
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) swarp[warp] = acc;
    __syncthreads();
    if (t == 0) {
      unsigned long long a = 0ull;
      for (int i = 0; i < kQsWarps; ++i) a += swarp[i];
      // a counts units of 2^(kWinLo-134): file it under exponents kWinLo,
      // kWinLo+21 and kWinLo+42 in 21-bit pieces so every bin stays small
      const unsigned long long mask21 = (1ull << 21) - 1ull;
      const unsigned long long a0 = a & mask21, a1 = (a >> 21) & mask21, a2 = a >> 42;
      if (a0) atomicAdd(&gbins[kWinLo], a0);
      if (a1) atomicAdd(&gbins[kWinLo + 21], a1);
      if (a2) atomicAdd(&gbins[kWinLo + 42], a2);
    }
    for (int i = t; i < kQwBins; i += kQsThreads)
      if (sbins[i]) atomicAdd(&gbins[i], sbins[i]);
    if (!qs_grid_barrier(arrive, 2u * gridDim.x, &s_abort)) return;
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
  const uint32_t tau2 = s_tau | (s_tau << 16);

  // ---- pass 2: codes of the kept positions ---------------------------------
  {
    int row[2] = {row0[0], row0[1]}, u[2] = {u0[0], u0[1]};
    QsPair cur, nxt;
    qs_load(src, nu, 0, t, cur);
    for (int s = 0; s < nslices; ++s) {
      if (s + 1 < nslices) qs_load(src, nu, s + 1, t, nxt);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int ui = s * kQsSlice + t + kQsThreads * j;
        if (ui < nu) {
          uint32_t wd[8];
          if (j == 0) qs_words(cur.a0, cur.a1, wd); else qs_words(cur.b0, cur.b1, wd);
          uint32_t keep = 0xFFFFu;
          if (has_meta) {
            keep = (ui < kQsKeepCap)
                       ? (uint32_t)s_keep[ui]
                       : (uint32_t) * reinterpret_cast<const uint16_t*>(meta + (size_t)row[j] * meta_stride + 2 * u[j]);
          }
          const uint32_t packed = unit_codes(wd, tau2, keep, s_csel);
          uint8_t* dst = codes + (size_t)row[j] * codes_stride + (size_t)u[j] * cb;
          if (cb == 4) {
            *reinterpret_cast<uint32_t*>(dst) = packed;
          } else if (cb == 2) {
            *reinterpret_cast<uint16_t*>(dst) = (uint16_t)packed;
          } else {
            for (int bb = 0; bb < cb; ++bb) dst[bb] = (uint8_t)(packed >> (8 * bb));
          }
          if (u[j] == upr - 1) {
            // zero padding at the end of the row
            for (int i = upr * cb; i < codes_stride; ++i) codes[(size_t)row[j] * codes_stride + i] = 0u;
          }
        }
        advance(row[j], u[j]);
      }
      cur = nxt;
    }
  }
}

}  // namespace sbn
