// Backward of the BitLinear layer under the straight-through estimator
// ("Microsoft BitNet 1.58: The Era of 1-Bit Large Language Models", section
// "Training with the Straight-Through Estimator": the quantizer is the
// identity in the backward pass and the latent weights take the gradient).
// The forward multiplies Xd = Xq s_t / 127 by Wd = gamma C, so
//     dX = dY Wd = gamma (dY C)      [T, K]      contraction over N_out
//     dW = dY^T Xd                   [N_out, K]  contraction over T
// (dW reaches every latent weight, pruned positions included).
//
// Both kernels are tiled fp32 GEMMs on the CUDA cores: 64 x 64 output tiles,
// 256 threads with 4 x 4 outputs each, 32-deep slices of the contraction
// staged in shared memory. dX expands the packed weights of a slice (32 rows
// x 64 positions = 128 units) into +-1/0 as it stages them, so C is read in
// its packed form, transposed relative to the forward's use. Outputs are
// rounded once to bf16.
#pragma once

#include "common.cuh"

namespace sbn {

constexpr int kBwThreads = 256;
constexpr int kBwTile = 64;    // output tile edge
constexpr int kBwSlice = 32;   // contraction depth staged per step

SBN_DEVFN float bf16_to_f32(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

// 4 x 4 outputs of thread (ty, tx) from one staged slice: a[s][row], b[s][col].
SBN_DEVFN void bw_slice_fma(const float (*a)[kBwTile], const float (*b)[kBwTile], int ty, int tx,
                            float (&acc)[4][4]) {
#pragma unroll 8
  for (int s = 0; s < kBwSlice; ++s) {
    float av[4], bv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) av[i] = a[s][ty * 4 + i];
#pragma unroll
    for (int j = 0; j < 4; ++j) bv[j] = b[s][tx * 4 + j];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
  }
}

// dX = gamma (dY C). Grid (K / 64, ceil(T / 64)). MM: group size; CB: code
// bytes per 16-position unit; DENSE: n == m (no keep bits).
template <int MM, int CB, bool DENSE>
__global__ void __launch_bounds__(kBwThreads)
bwd_dx_kernel(const uint16_t* __restrict__ dy, int t_count, int k, int n_out, const uint8_t* __restrict__ codes,
              const uint8_t* __restrict__ meta, int cstride, int mstride, const float* __restrict__ gamma,
              uint16_t* __restrict__ dx) {
  __shared__ float s_a[kBwSlice][kBwTile];   // dY^T slice: [n][t]
  __shared__ float s_b[kBwSlice][kBwTile];   // C slice: [n][k]
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int k0 = blockIdx.x * kBwTile, t0 = blockIdx.y * kBwTile;
  float acc[4][4] = {};
  for (int n0 = 0; n0 < n_out; n0 += kBwSlice) {
    for (int i = tid; i < kBwSlice * kBwTile; i += kBwThreads) {
      const int tt = i / kBwSlice, nn = i - tt * kBwSlice;   // consecutive threads: consecutive n
      const int t = t0 + tt, n = n0 + nn;
      s_a[nn][tt] = (t < t_count && n < n_out) ? bf16_to_f32(dy[(size_t)t * n_out + n]) : 0.f;
    }
    if (tid < kBwSlice * (kBwTile / 16)) {
      // one 16-position unit of one weight row per thread
      const int nn = tid >> 2, uu = tid & 3;
      const int n = n0 + nn, u = (k0 >> 4) + uu;
      uint32_t cw = 0u, keep = 0xFFFFu;
      if (n < n_out) {
        const uint8_t* cp = codes + (size_t)n * cstride + (size_t)u * CB;
#pragma unroll
        for (int b = 0; b < CB; ++b) cw |= (uint32_t)cp[b] << (8 * b);
        if (!DENSE) keep = (uint32_t)meta[(size_t)n * mstride + 2 * u] | ((uint32_t)meta[(size_t)n * mstride + 2 * u + 1] << 8);
      } else {
        keep = 0u;
      }
      int ci = 0;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        float v = 0.f;
        if ((keep >> j) & 1u) {
          const uint32_t c2 = (cw >> (2 * ci)) & 3u;   // 00 -> 0, 01 -> +1, 11 -> -1
          v = (c2 == 1u) ? 1.f : ((c2 == 3u) ? -1.f : 0.f);
          ++ci;
        }
        s_b[nn][uu * 16 + j] = v;
      }
    }
    __syncthreads();
    bw_slice_fma(s_a, s_b, ty, tx, acc);
    __syncthreads();
  }
  const float g = __ldg(gamma);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= t_count) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      dx[(size_t)t * k + k0 + tx * 4 + j] = __bfloat16_as_ushort(__float2bfloat16_rn(g * acc[i][j]));
  }
}

// dW = dY^T (Xq s / 127). Grid (K / 64, ceil(N_out / 64)).
__global__ void __launch_bounds__(kBwThreads)
bwd_dw_kernel(const uint16_t* __restrict__ dy, const int8_t* __restrict__ xq, const float* __restrict__ xs,
              int t_count, int k, int n_out, uint16_t* __restrict__ dw) {
  __shared__ float s_a[kBwSlice][kBwTile];   // dY slice: [t][n]
  __shared__ float s_b[kBwSlice][kBwTile];   // Xd slice: [t][k]
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int k0 = blockIdx.x * kBwTile, n0 = blockIdx.y * kBwTile;
  float acc[4][4] = {};
  for (int t0 = 0; t0 < t_count; t0 += kBwSlice) {
    for (int i = tid; i < kBwSlice * kBwTile; i += kBwThreads) {
      const int tt = i / kBwTile, cc = i - tt * kBwTile;     // consecutive threads: consecutive n / k
      const int t = t0 + tt;
      const bool tok = t < t_count;
      s_a[tt][cc] = (tok && n0 + cc < n_out) ? bf16_to_f32(dy[(size_t)t * n_out + n0 + cc]) : 0.f;
      s_b[tt][cc] = tok ? (float)xq[(size_t)t * k + k0 + cc] * (__ldg(xs + t) / 127.0f) : 0.f;
    }
    __syncthreads();
    bw_slice_fma(s_a, s_b, ty, tx, acc);
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int n = n0 + ty * 4 + i;
    if (n >= n_out) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      dw[(size_t)n * k + k0 + tx * 4 + j] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[i][j]));
  }
}

}  // namespace sbn
