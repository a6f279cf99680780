// SIMT contraction of packed ternary weights with INT8 activations (dp4a).
//
// "Microsoft BitNet 1.58: The Era of 1-Bit Large Language Models", section
// "The BitLinear Layer", fourth and fifth operations (integer product of the
// quantized operands, then rescaling by the preserved scales); the W2A8
// scheme of the section "bitnet.cpp: Matrix-Free Inference" (unpack 2-bit
// weights on chip, integer dot products).
//
// Tile: 64 output features x 32 tokens per CTA, K blocks of 128. Each K
// block's packed weights are expanded to int8 in shared memory from the codes
// and the keep bitmask; each thread owns 2 x 4 outputs.
#pragma once

#include "common.cuh"

namespace sbn {

// Expand one unit (16 positions) of packed weights into 16 int8 values.
// cbits holds the unit's kept codes (value j in bits 2j..2j+1), keep its
// 16 keep bits.
SBN_DEVFN uint4 expand_unit(uint32_t cbits, uint32_t keep) {
  uint32_t bytes[4] = {0u, 0u, 0u, 0u};
  int j = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    if ((keep >> i) & 1u) {
      const uint32_t c = (cbits >> (2 * j)) & 3u;
      ++j;
      // 01 -> +1 (0x01), 11 -> -1 (0xFF), 00 -> 0
      const uint32_t b = (c == 1u) ? 0x01u : ((c == 3u) ? 0xFFu : 0u);
      bytes[i >> 2] |= b << (8 * (i & 3));
    }
  }
  return make_uint4(bytes[0], bytes[1], bytes[2], bytes[3]);
}

constexpr int kSimtO = 64, kSimtT = 32, kSimtK = 128;

template <int M, bool ACC_OUT>
__global__ void __launch_bounds__(256)
bl_simt_kernel(const int8_t* __restrict__ xq, const float* __restrict__ xs, int T, int K,
               int N, int n, const uint8_t* __restrict__ codes, int cstride,
               const uint8_t* __restrict__ meta, int mstride,
               const float* __restrict__ gamma_ptr, uint16_t* __restrict__ y,
               int32_t* __restrict__ acc_out) {
  __shared__ __align__(16) int8_t sW[kSimtO][kSimtK + 16];
  __shared__ __align__(16) int8_t sX[kSimtT][kSimtK + 16];
  const int o0 = blockIdx.x * kSimtO, t0 = blockIdx.y * kSimtT;
  const int cb = 4 * n / M;
  const int tid = threadIdx.x;
  const int ro = tid & 31, tg = tid >> 5;  // rows ro, ro+32; tokens 4*tg..4*tg+3
  int acc[2][4];
#pragma unroll
  for (int r = 0; r < 2; ++r)
#pragma unroll
    for (int t = 0; t < 4; ++t) acc[r][t] = 0;

  for (int kb = 0; kb < K; kb += kSimtK) {
    {
      const int tt = tid >> 3, c = tid & 7;
      const int t = t0 + tt;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (t < T) v = __ldg(reinterpret_cast<const uint4*>(xq + (size_t)t * K + kb + c * 16));
      *reinterpret_cast<uint4*>(&sX[tt][c * 16]) = v;
    }
#pragma unroll
    for (int r2 = 0; r2 < 2; ++r2) {
      const int idx = tid + r2 * 256;
      const int rr = idx >> 3, u = idx & 7;
      const int o = o0 + rr;
      uint4 out = make_uint4(0u, 0u, 0u, 0u);
      if (o < N) {
        const int unit = (kb >> 4) + u;
        const uint8_t* cp = codes + (size_t)o * cstride + (size_t)unit * cb;
        uint32_t cbits = 0u;
        for (int b = 0; b < cb; ++b) cbits |= (uint32_t)__ldg(cp + b) << (8 * b);
        uint32_t keep = 0xFFFFu;
        if (n != M) {
          const uint8_t* mp = meta + (size_t)o * mstride + 2 * unit;
          keep = (uint32_t)__ldg(mp) | ((uint32_t)__ldg(mp + 1) << 8);
        }
        out = expand_unit(cbits, keep);
      }
      *reinterpret_cast<uint4*>(&sW[rr][u * 16]) = out;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < kSimtK; kk += 16) {
      uint4 wv[2], xv[4];
#pragma unroll
      for (int r = 0; r < 2; ++r) wv[r] = *reinterpret_cast<const uint4*>(&sW[ro + 32 * r][kk]);
#pragma unroll
      for (int t = 0; t < 4; ++t) xv[t] = *reinterpret_cast<const uint4*>(&sX[4 * tg + t][kk]);
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          int a = acc[r][t];
          a = __dp4a((int)wv[r].x, (int)xv[t].x, a);
          a = __dp4a((int)wv[r].y, (int)xv[t].y, a);
          a = __dp4a((int)wv[r].z, (int)xv[t].z, a);
          a = __dp4a((int)wv[r].w, (int)xv[t].w, a);
          acc[r][t] = a;
        }
    }
    __syncthreads();
  }

  const float g = ACC_OUT ? 0.f : *gamma_ptr;
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int tok = t0 + 4 * tg + t;
    if (tok >= T) continue;
    const float sc = ACC_OUT ? 0.f : __fdiv_rn(__fmul_rn(g, __ldg(xs + tok)), 127.0f);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int o = o0 + ro + 32 * r;
      if (o >= N) continue;
      if (ACC_OUT) {
        acc_out[(size_t)tok * N + o] = acc[r][t];
      } else {
        const __nv_bfloat16 b = __float2bfloat16_rn(__fmul_rn((float)acc[r][t], sc));
        y[(size_t)tok * N + o] = __bfloat16_as_ushort(b);
      }
    }
  }
}

}  // namespace sbn
