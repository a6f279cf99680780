// Backward dX and dW of the BitLinear layer on the 5th-generation tensor cores
// (`tcgen05.mma.cta_group::1.kind::f16`, bf16 operands, fp32 accumulation
// in tensor memory).
//
// "Microsoft BitNet 1.58: The Era of 1-Bit Large Language Models", section
// "Training with the Straight-Through Estimator": the quantizer is the
// identity in the backward pass, so dX = dY Wd = gamma (dY C), contracted
// over the N_out output features. Every product dY[t, o] * C[o, k] is exact
// in fp32 (C is -1, 0 or +1); only the accumulation rounds.
//
// A persistent CTA per SM walks 128 (tokens) x 256 (input features) tiles:
//   warp 0      TMA of dY tiles (128 tokens x 64 features of N_out, 128-byte
//               swizzle, K-major: the contraction runs along dY's rows);
//   warp 1      TMEM (two 256-column fp32 accumulators) and the MMA thread:
//               4 MMAs (K = 16) per 64-feature stage;
//   warps 4-11  producers: C's rows are the packed weights, read in place.
//               A thread expands (output feature o, 16 positions) of a stage
//               to bf16 -1/0/+1 and stores the 32 bytes into the B tile,
//               which is MN-major (positions contiguous, as in C's rows):
//               1 KB swizzle atoms of 8 features x 64 positions, atoms 1 KB
//               apart along the positions and 4 KB apart along the features;
//   warps 12-15 epilogue: TMEM lane = token, 32 positions per load; dX =
//               bf16(gamma * acc) stored as 64 contiguous bytes per token.
// Features past N_out (the last stage) are zero in both operands (TMA fills
// dY's, the producers write C's); positions past K and tokens past T are not
// stored. Every mbarrier wait is bounded in time.
#pragma once

#include <cuda.h>

#include "async.cuh"
#include "bl_tc.cuh"
#include "common.cuh"
#include "expand.cuh"

namespace sbn {

constexpr int kBxBM = 128;                       // tokens per tile (MMA M)
constexpr int kBxBN = 256;                       // positions per tile (MMA N)
constexpr int kBxBK = 64;                        // output features per stage
constexpr int kBxStages = 4;
constexpr int kBxABytes = kBxBM * kBxBK * 2;     // 16 KB of dY
constexpr int kBxBBytes = kBxBK * kBxBN * 2;     // 32 KB of C
constexpr int kBxStageBytes = kBxABytes + kBxBBytes;
constexpr uint32_t kBxTmemCols = 512;
// instruction descriptor: f32 accumulate, bf16 A and B, A K-major, B
// MN-major (bit 16), N = 256, M = 128
constexpr uint32_t kBxIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(kBxBN >> 3) << 17) |
                              ((uint32_t)(kBxBM >> 4) << 24);
constexpr int kBxSelCopies = 8;
constexpr size_t kBxSmemBytes = 1024 + (size_t)kBxStages * kBxStageBytes + (2 * kBxStages + 4) * 8 + 16 +
                                 256 * 4 * kBxSelCopies;

struct BxParams {
  const uint8_t* codes;
  const uint8_t* meta;
  const float* gamma;
  uint16_t* dx;
  int T, K, N;
  int cstride, mstride;
};

// MN-major 128-byte-swizzled operand: 1 KB atoms of 8 rows (the contraction)
// x 128 bytes (64 bf16 along M or N); leading offset = distance between
// atoms along M/N, stride offset = distance between atoms along K.
SBN_DEVFN uint64_t sw128_mnmajor_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;                    // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                    // 128-byte swizzle
  return d;
}

SBN_DEVFN void tc_mma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(kBxIdesc), "r"(accumulate), "r"(0u)
      : "memory");
}

// Four int8 values (-1, 0, +1 in bytes of q) -> four bf16 (two per word).
SBN_DEVFN void s8x4_to_bf16x4(uint32_t q, uint32_t& lo, uint32_t& hi) {
  const uint32_t a = __byte_perm(q, 0u, 0x4140u);   // bytes 0, 1 -> 16-bit lanes
  const uint32_t b = __byte_perm(q, 0u, 0x4342u);   // bytes 2, 3
  // nonzero -> 0x3F80 (1.0); the byte's sign bit -> the lane's sign bit
  lo = (((a | (a >> 1)) & 0x00010001u) * 0x3F80u) | ((a >> 7) & 0x00010001u) << 15;
  hi = (((b | (b >> 1)) & 0x00010001u) * 0x3F80u) | ((b >> 7) & 0x00010001u) << 15;
}

template <int MM, int CB, bool DENSE>
__global__ void __launch_bounds__(kTcThreads, 1)
bwd_dx_tc_kernel(const __grid_constant__ CUtensorMap tmap_dy, const BxParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)kBxStages * kBxStageBytes);
  uint64_t* empty = full + kBxStages;
  uint64_t* acc_full = empty + kBxStages;   // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2]
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(acc_empty + 2);
  uint32_t* s_sel = s_tmem + 4;             // [256][kBxSelCopies]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nst = (p.N + kBxBK - 1) / kBxBK;
  const int col_tiles = (p.K + kBxBN - 1) / kBxBN;
  const int n_tiles = col_tiles * ((p.T + kBxBM - 1) / kBxBM);

  if (tid == 0) {
    for (int s = 0; s < kBxStages; ++s) {
      mbar_init(&full[s], kTcProducers / 32 + 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kTcEpilogue / 32);
    }
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(s_tmem)),
                 "r"(kBxTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  if (!DENSE) {
    for (int i = tid; i < 256 * kBxSelCopies; i += blockDim.x) s_sel[i] = expand_selector((uint32_t)(i / kBxSelCopies));
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 0) {
    // ---- TMA of the dY tiles ----
    if (lane == 0) {
      int it = 0;
      for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        const int t0 = (tile / col_tiles) * kBxBM;
        bool ok = true;
        for (int ks = 0; ks < nst; ++ks, ++it) {
          const int s = it % kBxStages;
          const uint32_t ph = (it / kBxStages) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[s], kBxABytes);
          tma_load_2d(smem + (size_t)s * kBxStageBytes, &tmap_dy, ks * kBxBK, t0, &full[s]);
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer ----
    if (lane == 0) {
      int it = 0, j = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++j) {
        const int b = j & 1;
        if (!mbar_wait(&acc_empty[b], ((j >> 1) & 1u) ^ 1u)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(b * kBxBN);
        for (int ks = 0; ks < nst; ++ks, ++it) {
          const int s = it % kBxStages;
          const uint32_t ph = (it / kBxStages) & 1u;
          if (!mbar_wait(&full[s], ph)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + (size_t)s * kBxStageBytes);
          const uint64_t adesc = sw128_kmajor_desc(a_addr);
          const uint64_t bdesc = sw128_mnmajor_desc(a_addr + kBxABytes, 1024u, 4096u);
#pragma unroll
          for (int k = 0; k < kBxBK / 16; ++k) {
            // 16 features per MMA: A advances 32 bytes inside its swizzled
            // rows, B two 4 KB atom rows
            tc_mma_f16(d_tmem, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(k * (8192 / 16)),
                       (ks > 0 || k > 0) ? 1u : 0u);
          }
          tc_commit(&empty[s]);
        }
        tc_commit(&acc_full[b]);
      }
    }
  } else if (warp >= 4 && warp < 12) {
    // ---- producers: item i of a stage = (feature i / 16, unit i % 16 of
    // the tile's 256 positions); a thread takes items pi, pi + 256, ... ----
    const int pi = tid - 128;
    const uint32_t* sel = s_sel + (lane & (kBxSelCopies - 1));
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
      const int k0 = (tile % col_tiles) * kBxBN;
      for (int ks = 0; ks < nst; ++ks, ++it) {
        const int s = it % kBxStages;
        const uint32_t ph = (it / kBxStages) & 1u;
        int got = 1;
        if (lane == 0) got = mbar_wait(&empty[s], ph ^ 1u) ? 1 : 0;
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) { ok = false; break; }
        uint8_t* bt = smem + (size_t)s * kBxStageBytes + kBxABytes;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int i = pi + 256 * q4;
          const int ol = i >> 4, u = i & 15;
          const int o = ks * kBxBK + ol;
          const int ku = (k0 >> 4) + u;   // unit index along the row
          uint32_t w8[4] = {0u, 0u, 0u, 0u};   // 16 int8 values
          if (o < p.N && ku < (p.K >> 4)) {
            const uint8_t* cp = p.codes + (size_t)o * p.cstride + (size_t)ku * CB;
            uint32_t cw = 0u;
#pragma unroll
            for (int bb = 0; bb < CB; ++bb) cw |= (uint32_t)__ldg(cp + bb) << (8 * bb);
            if (DENSE) {
              codes8_to_s8(cw & 0xFFFFu, w8[0], w8[1]);
              codes8_to_s8(cw >> 16, w8[2], w8[3]);
            } else {
              const uint32_t m16 = __ldg(reinterpret_cast<const uint16_t*>(p.meta + (size_t)o * p.mstride) + ku);
              const uint32_t m0 = m16 & 0xFFu, m1 = m16 >> 8;
              const int p0 = (MM == 16) ? __popc(m0) : 2 * CB;
              const uint32_t v0 = cw & ((1u << (2 * p0)) - 1u);
              const uint32_t rest = cw >> (2 * p0);
              const int p1 = (MM == 16) ? __popc(m1) : 2 * CB;
              const uint32_t v1 = rest & ((1u << (2 * p1)) - 1u);
              uint32_t q0, q1;
              codes8_to_s8(v0, q0, q1);
              const uint32_t s0 = sel[m0 * kBxSelCopies];
              w8[0] = __byte_perm(q0, q1, s0 & 0xFFFFu);
              w8[1] = __byte_perm(q0, q1, s0 >> 16);
              codes8_to_s8(v1, q0, q1);
              const uint32_t s1 = sel[m1 * kBxSelCopies];
              w8[2] = __byte_perm(q0, q1, s1 & 0xFFFFu);
              w8[3] = __byte_perm(q0, q1, s1 >> 16);
            }
          }
          uint32_t h[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) s8x4_to_bf16x4(w8[e], h[2 * e], h[2 * e + 1]);
          // positions 16u .. 16u + 15 of feature ol: atom (ol / 8, u / 4),
          // row ol % 8, 16-byte chunks 2 (u % 4) and 2 (u % 4) + 1, swizzled
          const int r = ol & 7;
          uint8_t* atom = bt + (size_t)(ol >> 3) * 4096 + (size_t)(u >> 2) * 1024 + (size_t)r * 128;
          const int c0 = 2 * (u & 3);
          *reinterpret_cast<uint4*>(atom + (((c0) ^ r) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
          *reinterpret_cast<uint4*>(atom + (((c0 + 1) ^ r) << 4)) = make_uint4(h[4], h[5], h[6], h[7]);
        }
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[s]);
      }
    }
  } else if (warp >= 12) {
    // ---- epilogue: lane = token, 32 positions per TMEM load ----
    const int q = warp & 3;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const float g = __ldg(p.gamma);
    int j = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++j) {
      const int b = j & 1;
      const int t = (tile / col_tiles) * kBxBM + 32 * q + lane;
      const int k0 = (tile % col_tiles) * kBxBN;
      int got = 1;
      if (lane == 0) got = mbar_wait(&acc_full[b], (j >> 1) & 1u) ? 1 : 0;
      got = __shfl_sync(0xffffffffu, got, 0);
      if (!got) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < kBxBN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + (uint32_t)(b * kBxBN + 32 * c), r);
        const int kc = k0 + 32 * c;
        if (t < p.T && kc < p.K) {
          uint32_t o16[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float v0 = __fmul_rn(g, __uint_as_float(r[2 * e]));
            const float v1 = __fmul_rn(g, __uint_as_float(r[2 * e + 1]));
            o16[e] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v0)) |
                     ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v1)) << 16);
          }
          uint4* dst = reinterpret_cast<uint4*>(p.dx + (size_t)t * p.K + kc);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(o16[4 * e], o16[4 * e + 1], o16[4 * e + 2], o16[4 * e + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) {
      const int my_tiles = n_tiles > (int)blockIdx.x ? (n_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
      for (int jj = my_tiles - 2; jj < my_tiles; ++jj)
        if (jj >= 0) mbar_wait(&acc_full[jj & 1], (jj >> 1) & 1u);
    }
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kBxTmemCols)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// dW = dY^T Xd on the tensor cores, contracted over the T tokens:
//     dW[o, k] = sum_t (dY[t, o] * s_t / 127) * Xq[t, k].
// Xq is exact in bf16 (|Xq| <= 127); a = fp32(dY * (s_t / 127)) is split
// into a_hi = bf16(a) and a_lo = bf16(a - a_hi), |a - a_hi - a_lo| <=
// 2^-18 |a|, and each token step runs two MMAs (a_hi Xq, a_lo Xq) whose
// products are exact in fp32. Both operands are MN-major (output features
// and positions are contiguous in dY's and Xq's rows), written by the
// producer warps, 64 tokens per stage:
//   A_hi, A_lo  128 features x 64 tokens each: 1 KB atoms (8 tokens x 64
//               features), 1 KB apart along the features, 2 KB along tokens;
//   B           256 positions x 64 tokens: atoms 1 KB apart along the
//               positions, 4 KB along tokens.
// Tile 128 features x 256 positions; warps 4-11 produce, warp 1 issues,
// warps 12-15 drain (lane = feature, 32 positions per load).
// ---------------------------------------------------------------------------
constexpr int kBwBM = 128;                       // output features per tile (MMA M)
constexpr int kBwBN = 256;                       // positions per tile (MMA N)
constexpr int kBwBK = 64;                        // tokens per stage
constexpr int kBwStages = 3;
constexpr int kBwAPlane = kBwBM * kBwBK * 2;     // 16 KB
constexpr int kBwBBytes = kBwBN * kBwBK * 2;     // 32 KB
constexpr int kBwStageBytes = 2 * kBwAPlane + kBwBBytes;
// instruction descriptor: f32 accumulate, bf16 A and B, both MN-major
// (bits 15 and 16), N = 256, M = 128
constexpr uint32_t kBwIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                              ((uint32_t)(kBwBN >> 3) << 17) | ((uint32_t)(kBwBM >> 4) << 24);
constexpr size_t kBwSmemBytes = 1024 + (size_t)kBwStages * kBwStageBytes + (2 * kBwStages + 4) * 8 + 16;

struct BwParams {
  const uint16_t* dy;
  const int8_t* xq;
  const float* xs;
  uint16_t* dw;
  int T, K, N;
};

SBN_DEVFN void tc_mma_f16_mn(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(kBwIdesc), "r"(accumulate), "r"(0u)
      : "memory");
}

// Eight bf16 (4 words) times one fp32 scale, split into hi and lo bf16 parts.
SBN_DEVFN void scale_split8(const uint4& v, float sc, uint4& hi, uint4& lo) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a0 = __fmul_rn(__uint_as_float(w[i] << 16), sc);
    const float a1 = __fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), sc);
    const __nv_bfloat16 h0 = __float2bfloat16_rn(a0), h1 = __float2bfloat16_rn(a1);
    const __nv_bfloat16 l0 = __float2bfloat16_rn(__fsub_rn(a0, __bfloat162float(h0)));
    const __nv_bfloat16 l1 = __float2bfloat16_rn(__fsub_rn(a1, __bfloat162float(h1)));
    h[i] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
    l[i] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// Four int8 (any values in -127..127) -> four bf16, exactly.
SBN_DEVFN void s8x4_to_bf16x4_any(uint32_t q, uint32_t& lo, uint32_t& hi) {
  const float f0 = (float)(int8_t)(q & 0xFFu), f1 = (float)(int8_t)((q >> 8) & 0xFFu);
  const float f2 = (float)(int8_t)((q >> 16) & 0xFFu), f3 = (float)(int8_t)(q >> 24);
  lo = (__float_as_uint(f0) >> 16) | (__float_as_uint(f1) & 0xFFFF0000u);
  hi = (__float_as_uint(f2) >> 16) | (__float_as_uint(f3) & 0xFFFF0000u);
}

__global__ void __launch_bounds__(kTcThreads, 1) bwd_dw_tc_kernel(const BwParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)kBwStages * kBwStageBytes);
  uint64_t* empty = full + kBwStages;
  uint64_t* acc_full = empty + kBwStages;   // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2]
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nst = (p.T + kBwBK - 1) / kBwBK;
  const int col_tiles = (p.K + kBwBN - 1) / kBwBN;
  const int n_tiles = col_tiles * ((p.N + kBwBM - 1) / kBwBM);

  if (tid == 0) {
    for (int s = 0; s < kBwStages; ++s) {
      mbar_init(&full[s], kTcProducers / 32);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kTcEpilogue / 32);
    }
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(s_tmem)),
                 "r"(kBxTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 1) {
    // ---- MMA issuer ----
    if (lane == 0) {
      int it = 0, j = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++j) {
        const int b = j & 1;
        if (!mbar_wait(&acc_empty[b], ((j >> 1) & 1u) ^ 1u)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(b * kBwBN);
        for (int ks = 0; ks < nst; ++ks, ++it) {
          const int s = it % kBwStages;
          const uint32_t ph = (it / kBwStages) & 1u;
          if (!mbar_wait(&full[s], ph)) { ok = false; break; }
          tc_fence_after();
          const uint32_t base = smem_u32(smem + (size_t)s * kBwStageBytes);
          const uint64_t ahi = sw128_mnmajor_desc(base, 1024u, 2048u);
          const uint64_t alo = sw128_mnmajor_desc(base + kBwAPlane, 1024u, 2048u);
          const uint64_t bd = sw128_mnmajor_desc(base + 2 * kBwAPlane, 1024u, 4096u);
#pragma unroll
          for (int k = 0; k < kBwBK / 16; ++k) {
            // 16 tokens per MMA: two atom rows of A (2 x 2 KB) and of B (2 x 4 KB)
            tc_mma_f16_mn(d_tmem, ahi + (uint64_t)(k * (4096 / 16)), bd + (uint64_t)(k * (8192 / 16)),
                          (ks > 0 || k > 0) ? 1u : 0u);
            tc_mma_f16_mn(d_tmem, alo + (uint64_t)(k * (4096 / 16)), bd + (uint64_t)(k * (8192 / 16)), 1u);
          }
          tc_commit(&empty[s]);
        }
        tc_commit(&acc_full[b]);
      }
    }
  } else if (warp >= 4 && warp < 12) {
    // ---- producers: A items (token, 8 features) and B items (token, 16
    // positions), four of each per thread and stage ----
    const int pi = tid - 128;
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
      const int o0 = (tile / col_tiles) * kBwBM;
      const int k0 = (tile % col_tiles) * kBwBN;
      for (int ks = 0; ks < nst; ++ks, ++it) {
        const int s = it % kBwStages;
        const uint32_t ph = (it / kBwStages) & 1u;
        int got = 1;
        if (lane == 0) got = mbar_wait(&empty[s], ph ^ 1u) ? 1 : 0;
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) { ok = false; break; }
        uint8_t* st = smem + (size_t)s * kBwStageBytes;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int i = pi + 256 * q4;
          // A: token tl = i / 16, features 8 (i % 16) .. +7
          {
            const int tl = i >> 4, f8 = i & 15;
            const int t = ks * kBwBK + tl, o = o0 + 8 * f8;
            uint4 hi = make_uint4(0u, 0u, 0u, 0u), lo = hi;
            if (t < p.T && o < p.N) {
              const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.dy + (size_t)t * p.N + o));
              scale_split8(v, __fdiv_rn(__ldg(p.xs + t), 127.0f), hi, lo);
            }
            const int r = tl & 7, c = f8 & 7;
            const size_t off = (size_t)(tl >> 3) * 2048 + (size_t)(f8 >> 3) * 1024 + (size_t)r * 128 + ((c ^ r) << 4);
            *reinterpret_cast<uint4*>(st + off) = hi;
            *reinterpret_cast<uint4*>(st + kBwAPlane + off) = lo;
          }
          // B: token tl = i / 16, positions 16 (i % 16) .. +15
          {
            const int tl = i >> 4, u = i & 15;
            const int t = ks * kBwBK + tl, kk = k0 + 16 * u;
            uint32_t h[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
            if (t < p.T && kk < p.K) {
              const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.xq + (size_t)t * p.K + kk));
              s8x4_to_bf16x4_any(v.x, h[0], h[1]);
              s8x4_to_bf16x4_any(v.y, h[2], h[3]);
              s8x4_to_bf16x4_any(v.z, h[4], h[5]);
              s8x4_to_bf16x4_any(v.w, h[6], h[7]);
            }
            const int r = tl & 7, c0 = 2 * (u & 3);
            uint8_t* atom = st + 2 * kBwAPlane + (size_t)(tl >> 3) * 4096 + (size_t)(u >> 2) * 1024 + (size_t)r * 128;
            *reinterpret_cast<uint4*>(atom + ((c0 ^ r) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
            *reinterpret_cast<uint4*>(atom + (((c0 + 1) ^ r) << 4)) = make_uint4(h[4], h[5], h[6], h[7]);
          }
        }
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[s]);
      }
    }
  } else if (warp >= 12) {
    // ---- epilogue: lane = output feature, 32 positions per TMEM load ----
    const int q = warp & 3;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    int j = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++j) {
      const int b = j & 1;
      const int o = (tile / col_tiles) * kBwBM + 32 * q + lane;
      const int k0 = (tile % col_tiles) * kBwBN;
      int got = 1;
      if (lane == 0) got = mbar_wait(&acc_full[b], (j >> 1) & 1u) ? 1 : 0;
      got = __shfl_sync(0xffffffffu, got, 0);
      if (!got) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < kBwBN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + (uint32_t)(b * kBwBN + 32 * c), r);
        const int kc = k0 + 32 * c;
        if (o < p.N && kc < p.K) {
          uint32_t o16[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            o16[e] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(r[2 * e]))) |
                     ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(r[2 * e + 1]))) << 16);
          uint4* dst = reinterpret_cast<uint4*>(p.dw + (size_t)o * p.K + kc);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(o16[4 * e], o16[4 * e + 1], o16[4 * e + 2], o16[4 * e + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) {
      const int my_tiles = n_tiles > (int)blockIdx.x ? (n_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
      for (int jj = my_tiles - 2; jj < my_tiles; ++jj)
        if (jj >= 0) mbar_wait(&acc_full[jj & 1], (jj >> 1) & 1u);
    }
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kBxTmemCols)
                 : "memory");
  }
}

}  // namespace sbn
