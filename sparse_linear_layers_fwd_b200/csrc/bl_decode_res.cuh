// Decode contraction (T <= 16 tokens), resident variant: every CTA copies
// the packed weights of its output rows and the INT8 activations into shared
// memory with per-thread 16-byte asynchronous copies (cp.async), then
// contracts them there.
//
// "Microsoft BitNet 1.58: The Era of 1-Bit Large Language Models", section
// "bitnet.cpp: Matrix-Free Inference": 2-bit weights are moved on chip,
// unpacked there and contracted with 8-bit activations, so HBM carries only
// the packed bytes. Decoding is bound by those bytes.
//
// A CTA owns a contiguous range of 16-row tiles. At entry all 1024 threads
// issue 16-byte asynchronous copies (cp.async) of the tiles' code rows and
// keep-bit rows and of the activations, about seven per thread, all in
// flight at once; one wait and one block barrier later everything is in
// shared memory. The 32 warps then walk the (tile, 128-position segment)
// items. Per item a thread
// expands 32 positions of two rows (expand.cuh) straight into the A fragment
// of `mma.sync.m16n8k32.s8` (weights as the 16-row operand, tokens as the 8
// columns, a K permutation shared with the activation fragment). A warp adds
// its partial sums into the tile's shared accumulator when it moves to
// another tile; the epilogue dequantizes y = acc * gamma * s_t / 127.
//
// XBF: the kernel takes the bf16 activations instead and quantizes them
// itself (the per-token absmax INT8 step fused into the contraction's
// prologue): every CTA copies X, one warp per token computes s_t and the
// INT8 row in shared memory with the arithmetic of sbn_quantize_acts
// (qa.cuh), and CTA 0 optionally writes Xq and s to global memory.
#pragma once

#include "bl_decode.cuh"
#include "common.cuh"
#include "expand.cuh"
#include "qa.cuh"

namespace sbn {

constexpr int kDresThreads = 1024;
constexpr int kDresWarps = kDresThreads / 32;
constexpr int kDresMaxTiles = 16;        // tiles per CTA at most
constexpr size_t kDresSmemMax = 227 * 1024;

struct DresLayout {
  size_t sel, acc, x, codes, meta, xbf, scale, bars, total;
  int xstride;
};

// Shared-memory layout of one CTA holding `tiles` tiles.
__host__ __device__ inline DresLayout dres_layout(int tiles, int nt, int k, int cstride, int mstride,
                                                  bool dense, bool xbf = false) {
  DresLayout L;
  L.xstride = k;
  L.sel = 0;
  L.acc = 1024;
  L.x = L.acc + (size_t)tiles * 16 * nt * 4;
  L.x = (L.x + 127) & ~(size_t)127;
  L.codes = L.x + (size_t)nt * L.xstride;
  L.codes = (L.codes + 127) & ~(size_t)127;
  L.meta = L.codes + (size_t)tiles * 16 * cstride;
  L.xbf = L.meta + (dense ? 0 : (size_t)tiles * 16 * mstride);
  L.xbf = (L.xbf + 127) & ~(size_t)127;
  L.scale = L.xbf + (xbf ? (size_t)nt * k * 2 : 0);
  L.bars = L.scale + (xbf ? 16 * 4 : 0);
  L.bars = (L.bars + 15) & ~(size_t)15;
  L.total = L.bars + (size_t)(tiles + 1) * 8;
  return L;
}

struct DresParams {
  const int8_t* xq;
  const float* xs;
  const uint16_t* xbf;   // XBF: bf16 activations [T, K]
  int8_t* xq_out;        // XBF: optional copies of Xq and s (written by CTA 0)
  float* xs_out;
  const uint8_t* codes;
  const uint8_t* meta;
  const float* gamma;
  uint16_t* y;
  int32_t* acc_out;
  int T, K, N;
  int cstride, mstride;
  int tiles_per_cta;  // tiles of the largest CTA range
};

// MM: group size m; CB: code bytes per 16 positions (= 4n/m); NT: token
// columns (8 or 16); DENSE: n == m (no keep bits); ACC: write int32 acc.
template <int MM, int CB, int NT, bool DENSE, bool ACC, bool XBF>
__global__ void __launch_bounds__(kDresThreads, 1)
bl_decode_res_kernel(const DresParams p) {
  extern __shared__ __align__(128) uint8_t dres_smem[];
  const int n_tiles = (p.N + 15) / 16;
  const int t_begin = (int)((long long)blockIdx.x * n_tiles / gridDim.x);
  const int t_end = (int)((long long)(blockIdx.x + 1) * n_tiles / gridDim.x);
  const int tiles = t_end - t_begin;
  const DresLayout L = dres_layout(p.tiles_per_cta, NT, p.K, p.cstride, p.mstride, DENSE, XBF);
  uint32_t* s_sel = reinterpret_cast<uint32_t*>(dres_smem + L.sel);
  int32_t* s_acc = reinterpret_cast<int32_t*>(dres_smem + L.acc);
  uint8_t* s_x = dres_smem + L.x;
  uint8_t* s_codes = dres_smem + L.codes;
  uint8_t* s_meta = dres_smem + L.meta;
  uint16_t* s_xbf = reinterpret_cast<uint16_t*>(dres_smem + L.xbf);
  float* s_scale = reinterpret_cast<float*>(dres_smem + L.scale);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int row0 = t_begin * 16;
  const int rows_valid = min(16 * tiles, p.N - row0);
  {
    // every thread issues its share of 16-byte asynchronous copies of this
    // CTA's code rows, keep-bit rows and activations: all of them are in
    // flight at once, with no per-copy cost of a bulk copy engine
    const int nx = XBF ? p.T * p.K * 2 / 16 : p.T * p.K / 16;
    const int nc = rows_valid * p.cstride / 16;
    const int nm = DENSE ? 0 : rows_valid * p.mstride / 16;
    const uint8_t* gx = XBF ? reinterpret_cast<const uint8_t*>(p.xbf) : reinterpret_cast<const uint8_t*>(p.xq);
    uint8_t* sx = XBF ? reinterpret_cast<uint8_t*>(s_xbf) : s_x;
    const uint8_t* gc = p.codes + (size_t)row0 * p.cstride;
    for (int i = tid; i < nx; i += kDresThreads) cp_async16(sx + 16 * (size_t)i, gx + 16 * (size_t)i, true);
    for (int i = tid; i < nc; i += kDresThreads) cp_async16(s_codes + 16 * (size_t)i, gc + 16 * (size_t)i, true);
    if (!DENSE) {
      const uint8_t* gm = p.meta + (size_t)row0 * p.mstride;
      for (int i = tid; i < nm; i += kDresThreads) cp_async16(s_meta + 16 * (size_t)i, gm + 16 * (size_t)i, true);
    }
    cp_async_commit();
  }
  if (!DENSE) fill_selector_table(s_sel);
  for (int i = tid; i < tiles * 16 * NT; i += kDresThreads) s_acc[i] = 0;
  cp_async_wait<0>();
  __syncthreads();
  if (XBF) {
    // warp `warp` quantizes token row `warp` (T <= 16 <= warps)
    if (warp < p.T) {
      const uint4* xr = reinterpret_cast<const uint4*>(s_xbf + (size_t)warp * p.K);
      const int kc = p.K / 8;
      uint32_t amax = 0u;
      for (int c = lane; c < kc; c += 32) amax = max(amax, mag_max8(xr[c]));
      amax = __reduce_max_sync(0xffffffffu, amax);
      const float sc = fmaxf(__uint_as_float(amax << 16), 1e-5f);
      const float mult = __fdiv_rn(127.0f, sc);
      uint2* qr = reinterpret_cast<uint2*>(s_x + (size_t)warp * L.xstride);
      const bool out = blockIdx.x == 0 && p.xq_out != nullptr;
      uint2* gq = out ? reinterpret_cast<uint2*>(p.xq_out + (size_t)warp * p.K) : nullptr;
      for (int c = lane; c < kc; c += 32) {
        const uint2 q = quant8(xr[c], mult);
        qr[c] = q;
        if (out) gq[c] = q;
      }
      if (lane == 0) {
        s_scale[warp] = sc;
        if (blockIdx.x == 0 && p.xs_out) p.xs_out[warp] = sc;
      }
    }
    __syncthreads();
  }
  const int ksegs = p.K / 128;
  const int items = tiles * ksegs;
  int cur_tile = -1;
  int acc0[4] = {0, 0, 0, 0};
  int acc1[4] = {0, 0, 0, 0};
  auto flush = [&](int tile) {
    int32_t* a = s_acc + (size_t)tile * 16 * NT;
    atomicAdd(&a[g * NT + 2 * t], acc0[0]);
    atomicAdd(&a[g * NT + 2 * t + 1], acc0[1]);
    atomicAdd(&a[(g + 8) * NT + 2 * t], acc0[2]);
    atomicAdd(&a[(g + 8) * NT + 2 * t + 1], acc0[3]);
    if (NT == 16) {
      atomicAdd(&a[g * NT + 8 + 2 * t], acc1[0]);
      atomicAdd(&a[g * NT + 8 + 2 * t + 1], acc1[1]);
      atomicAdd(&a[(g + 8) * NT + 8 + 2 * t], acc1[2]);
      atomicAdd(&a[(g + 8) * NT + 8 + 2 * t + 1], acc1[3]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) acc0[i] = acc1[i] = 0;
  };

  for (int it = warp; it < items; it += kDresWarps) {
    const int tile = it / ksegs, kseg = it - tile * ksegs;
    if (tile != cur_tile) {
      if (cur_tile >= 0) flush(cur_tile);
      cur_tile = tile;
    }
    const uint8_t* ct = s_codes + (size_t)tile * 16 * p.cstride;
    const uint8_t* mt = s_meta + (size_t)tile * 16 * p.mstride;
    const int ubase = kseg * 8 + 2 * t;   // first of this thread's two units
    const int coff = ubase * CB;          // even number of units: 2-byte aligned
    const int csh = (coff & 3) * 8;
    unsigned long long cbits[2];
    uint32_t mw[2];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int r = g + 8 * rr;
      const uint32_t* cw = reinterpret_cast<const uint32_t*>(ct + (size_t)r * p.cstride + (coff & ~3));
      const unsigned long long both = (unsigned long long)cw[0] | ((unsigned long long)cw[1] << 32);
      cbits[rr] = both >> csh;
      mw[rr] = DENSE ? 0xFFFFFFFFu : *reinterpret_cast<const uint32_t*>(mt + (size_t)r * p.mstride + ubase * 2);
    }
    int off[2] = {0, 0};
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      uint32_t w0[2], w1[2];
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const uint32_t m8 = (mw[rr] >> (8 * s)) & 0xFFu;
        const int pk = (MM == 16 && !DENSE) ? __popc(m8) : 2 * CB;   // kept in these 8
        const int o = (MM == 16 && !DENSE) ? off[rr] : s * 4 * CB;
        const uint32_t v = (uint32_t)(cbits[rr] >> o) & ((1u << (2 * pk)) - 1u);
        if (MM == 16 && !DENSE) off[rr] += 2 * pk;
        if (DENSE) {
          codes8_to_s8(v, w0[rr], w1[rr]);
        } else {
          expand8(m8, v, s_sel, w0[rr], w1[rr]);
        }
      }
      const int pos = ubase * 16 + 8 * s;
      const uint2 xa = *reinterpret_cast<const uint2*>(s_x + (size_t)g * L.xstride + pos);
      mma_s8_16x8x32(acc0, w0[0], w0[1], w1[0], w1[1], xa.x, xa.y);
      if (NT == 16) {
        const uint2 xb = *reinterpret_cast<const uint2*>(s_x + (size_t)(g + 8) * L.xstride + pos);
        mma_s8_16x8x32(acc1, w0[0], w0[1], w1[0], w1[1], xb.x, xb.y);
      }
    }
  }
  if (cur_tile >= 0) flush(cur_tile);
  __syncthreads();

  const float gm = ACC ? 0.f : __ldg(p.gamma);
  const int rows = min(16 * tiles, p.N - row0);
  for (int i = tid; i < rows * p.T; i += kDresThreads) {
    const int r = i % rows, tok = i / rows;
    const int a = s_acc[(size_t)(r >> 4) * 16 * NT + (r & 15) * NT + tok];
    const int grow = row0 + r;
    if (ACC) {
      p.acc_out[(size_t)tok * p.N + grow] = a;
    } else {
      const float st = XBF ? s_scale[tok] : __ldg(p.xs + tok);
      const float sc = __fdiv_rn(__fmul_rn(gm, st), 127.0f);
      p.y[(size_t)tok * p.N + grow] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn((float)a, sc)));
    }
  }
}

}  // namespace sbn
