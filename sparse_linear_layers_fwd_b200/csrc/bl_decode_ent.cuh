// Decode contraction (T <= 16 tokens) over entropy-tight packed weights
// (entropy.cuh; patterns with m = 4 or 8): the resident decode kernel of
// bl_decode_res.cuh with the weight rows holding one word per group. Two
// shared-memory tables turn a word into the group's keep bits (colex rank ->
// mask) and its packed kept codes (base-3 value -> 2-bit codes), which the
// expansion of expand.cuh takes as for the canonical format.
#pragma once

#include "bl_decode.cuh"
#include "bl_decode_res.cuh"
#include "common.cuh"
#include "entropy.cuh"
#include "expand.cuh"

namespace sbn {

// The decode tables follow the resident layout: rank -> keep mask
// (kEntRankSlots entries) and base-3 value -> codes (up to 729), u16 each.
__host__ __device__ inline size_t ent_tables_offset(const DresLayout& L) {
  return (L.total + 15) & ~(size_t)15;
}
__host__ __device__ inline size_t ent_smem_bytes(const DresLayout& L) {
  return ent_tables_offset(L) + (kEntRankSlots + 729) * 2;
}

// MM: group size m; CB: code bytes per 16 positions (= 4n/m); NT: token
// columns (8 or 16); ACC: write int32 acc; XBF: bf16 activations in, each
// token row quantized in the prologue (as in bl_decode_res.cuh).
template <int MM, int CB, int NT, bool ACC, bool XBF>
__global__ void __launch_bounds__(kDresThreads, 1)
bl_decode_ent_kernel(const DresParams p) {
  constexpr bool DENSE = false;
  constexpr int kEntN = CB * MM / 4;                  // kept per group
  constexpr int kEntBits = entropy_group_bits(kEntN, MM);
  constexpr uint32_t kEntP3 = pow3_u32(kEntN);
  extern __shared__ __align__(128) uint8_t dent_smem[];
  const int n_tiles = (p.N + 15) / 16;
  const int t_begin = (int)((long long)blockIdx.x * n_tiles / gridDim.x);
  const int t_end = (int)((long long)(blockIdx.x + 1) * n_tiles / gridDim.x);
  const int tiles = t_end - t_begin;
  // p.cstride is the entropy row stride; no keep-bit rows; the decode
  // tables follow the resident layout
  const DresLayout L = dres_layout(p.tiles_per_cta, NT, p.K, p.cstride, 0, true, XBF);
  uint16_t* s_rank_mask = reinterpret_cast<uint16_t*>(dent_smem + ent_tables_offset(L));
  uint16_t* s_val_codes = s_rank_mask + kEntRankSlots;
  uint32_t* s_sel = reinterpret_cast<uint32_t*>(dent_smem + L.sel);
  int32_t* s_acc = reinterpret_cast<int32_t*>(dent_smem + L.acc);
  uint8_t* s_x = dent_smem + L.x;
  uint8_t* s_codes = dent_smem + L.codes;
  uint16_t* s_xbf = reinterpret_cast<uint16_t*>(dent_smem + L.xbf);
  float* s_scale = reinterpret_cast<float*>(dent_smem + L.scale);

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
    const int nm = 0;
    const uint8_t* gx = XBF ? reinterpret_cast<const uint8_t*>(p.xbf) : reinterpret_cast<const uint8_t*>(p.xq);
    uint8_t* sx = XBF ? reinterpret_cast<uint8_t*>(s_xbf) : s_x;
    const uint8_t* gc = p.codes + (size_t)row0 * p.cstride;
    for (int i = tid; i < nx; i += kDresThreads) cp_async16(sx + 16 * (size_t)i, gx + 16 * (size_t)i, true);
    for (int i = tid; i < nc; i += kDresThreads) cp_async16(s_codes + 16 * (size_t)i, gc + 16 * (size_t)i, true);
    (void)nm;
    cp_async_commit();
  }
  fill_selector_table(s_sel);
  fill_entropy_tables<MM, kEntN>(s_rank_mask, s_val_codes);
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
    const int ubase = kseg * 8 + 2 * t;   // first of this thread's two units
    // one group word of row r (bit offset gi * kEntBits of the row stream)
    auto ent_word = [&](int r, int gi) -> uint32_t {
      const int bo = gi * kEntBits;
      const uint32_t* w = reinterpret_cast<const uint32_t*>(ct + (size_t)r * p.cstride) + (bo >> 5);
      const unsigned long long both = (unsigned long long)w[0] | ((unsigned long long)w[1] << 32);
      return (uint32_t)(both >> (bo & 31)) & ((1u << kEntBits) - 1u);
    };
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      uint32_t w0[2], w1[2];
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        // keep bits and kept codes of these 8 positions from 8 / MM words
        const int r = g + 8 * rr;
        const int gi = (ubase * 16 + 8 * s) / MM;
        uint32_t m8 = 0u, v = 0u;
#pragma unroll
        for (int h = 0; h < 8 / MM; ++h) {
          const uint32_t word = ent_word(r, gi + h);
          const uint32_t rank = min(word / kEntP3, (uint32_t)kEntRankSlots - 1u);
          // (a row past the layer's end holds arbitrary words: keep the mask
          // within M bits so the selector index stays below 256)
          m8 |= ((uint32_t)s_rank_mask[rank] & ((1u << MM) - 1u)) << (MM * h);
          v |= (uint32_t)s_val_codes[word - (word / kEntP3) * kEntP3] << (2 * kEntN * h);
        }
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
