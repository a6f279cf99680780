// Decode contraction (T <= 16 tokens) over the canonical packed weights.
//
// "Microsoft BitNet 1.58: The Era of 1-Bit Large Language Models", section
// "bitnet.cpp: Matrix-Free Inference": the 2-bit weights are moved on chip,
// unpacked there and contracted with 8-bit activations, so that HBM carries
// only the packed bytes; decoding is bound by those bytes.
//
// One CTA of 1024 threads per SM owns a contiguous range of 16-row tiles,
// with one producer warp and 31 consumer warps. The producer's lane 0 issues
// one bulk copy (cp.async.bulk) of each tile's code rows and one of its
// keep-bit rows, each tile completing its own mbarrier, so the consumers of
// the first tile start while the later tiles are still in flight; a bulk copy
// holds its issuing thread for a while on this part, so no consumer issues
// one. Meanwhile the consumers load the activations straight from global
// memory into registers, 16-byte chunks dealt out chunk-major over the 992
// consumer threads: in XBF mode the bf16 rows are quantized there (per-token
// absmax INT8 with the arithmetic of sbn_quantize_acts: chunk maxima,
// per-row maxima by shared atomics, the scales, then the rounding), otherwise
// the INT8 rows are copied. Either way the INT8 rows land in shared memory
// with a padded row stride and swizzled 16-byte chunks, so that the
// activation fragments of a warp are read without bank conflicts. The
// consumers synchronize among themselves on a named barrier; the producer
// never waits.
//
// Work item of a warp: 16 rows x 256 positions. Thread (g, t) of the warp
// expands rows g and g + 8 over its own 64 contiguous positions, eight at a
// time, straight into the A fragment of `mma.sync.m16n8k32.s8` (weights as
// the 16-row operand, tokens as the 8 columns; the K permutation maps
// logical k = 4t + j to position 8i + j and k = 16 + 4t + j to 8i + 4 + j of
// the thread's span, for both operands). The 8 positions of a group take a
// keep byte and the group's kept codes: the codes become bytes through a
// nibble spread and a byte permute of the table {0, +1, 0, -1}, and a second
// byte permute with the mask's selector puts them at their positions.
// A warp adds its partial sums into the tile's shared accumulator when it
// moves on; after one consumer barrier the epilogue writes
// y = bf16(acc * fl32(fl32(gamma * s_t) / 127)), the factor formed once per token.
#pragma once

#include "async.cuh"
#include "bl_decode.cuh"
#include "common.cuh"
#include "expand.cuh"
#include "qa.cuh"

namespace sbn {

constexpr int kGvThreads = 1024;
constexpr int kGvWarps = kGvThreads / 32;
constexpr int kGvConsumerWarps = kGvWarps - 1;   // the last warp issues the tile copies
constexpr int kGvConsumers = 32 * kGvConsumerWarps;
constexpr int kGvMaxTiles = 16;        // 16-row tiles per CTA at most
constexpr int kGvMaxChunks = 6;        // 16-byte activation chunks per consumer thread (registers)
constexpr size_t kGvSmemMax = 227 * 1024;

struct GvLayout {
  uint32_t sel, acc, rmax, scale, ysc, bars, x, codes, meta, total;
  int xstride;
};

__host__ __device__ inline uint32_t gv_align128(size_t x) { return (uint32_t)((x + 127) & ~(size_t)127); }

// Shared-memory layout of a CTA holding `tiles` tiles and `t` token rows.
__host__ __device__ inline GvLayout gv_layout(int tiles, int nt, int t, int k, int cstride, int mstride,
                                              bool dense) {
  GvLayout L;
  L.xstride = k + 16;
  L.sel = 0;                                                   // 256 selector pairs
  L.acc = 2048;                                                // [tiles][16][nt] int32
  L.rmax = gv_align128(L.acc + (size_t)tiles * 16 * nt * 4);   // [16] row maxima (bf16 magnitude bits)
  L.scale = L.rmax + 16 * 4;                                   // [16] token scales s_t
  L.ysc = L.scale + 16 * 4;                                    // [16] output factors
  L.bars = L.ysc + 16 * 4;                                     // [tiles] mbarriers
  L.x = gv_align128(L.bars + (size_t)tiles * 8);               // [t][xstride] INT8
  L.codes = gv_align128(L.x + (size_t)t * L.xstride);
  L.meta = gv_align128(L.codes + (size_t)tiles * 16 * cstride);
  L.total = L.meta + (dense ? 0u : (uint32_t)(tiles * 16 * mstride));
  return L;
}

struct GvParams {
  const int8_t* xq;       // INT8 activations [T, K] and scales [T] (not XBF)
  const float* xs;
  const uint16_t* xbf;    // XBF: bf16 activations [T, K]
  int8_t* xq_out;         // XBF: optional copies of Xq and s (written by CTA 0)
  float* xs_out;
  const uint8_t* codes;
  const uint8_t* meta;
  const float* gamma;
  uint16_t* y;
  int32_t* acc_out;
  int T, K, N;
  int cstride, mstride;
  int tiles_per_cta;      // tiles of the largest CTA range
  int tile_base, tile_rem;  // CTA b owns tile_base (+1 if b < tile_rem) tiles
  int kc;                 // 16-byte activation chunks per row (K/8 bf16 or K/16 INT8)
  uint32_t kc_magic;      // ceil(2^32 / kc): q / kc == umulhi(q, kc_magic) for q < 2^16
  int dr, drem;           // 992 = dr * kc + drem (the step of a thread's chunk index)
  GvLayout L;             // shared-memory layout (the host's gv_layout)
};

// Elementwise max(|a|, |b|) of two bf16 pairs (the sign of each result is
// the xor of the operands' signs; callers clear it).
SBN_DEVFN uint32_t gv_absmax2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Largest magnitude of a 16-byte chunk (8 bf16) folded into a running pair.
SBN_DEVFN uint32_t gv_chunk_absmax(const uint4& v, uint32_t run) {
  return gv_absmax2(gv_absmax2(gv_absmax2(v.x, v.y), gv_absmax2(v.z, v.w)), run);
}

// Named barriers: 1 among the consumer warps; 2 from the producer's set-up
// (it arrives) to the consumers (they wait).
SBN_DEVFN void gv_consumer_sync() { asm volatile("bar.sync 1, %0;\n" ::"n"(kGvConsumers) : "memory"); }
SBN_DEVFN void gv_setup_arrive() { asm volatile("bar.arrive 2, %0;\n" ::"n"(kGvThreads) : "memory"); }
SBN_DEVFN void gv_setup_wait() { asm volatile("bar.sync 2, %0;\n" ::"n"(kGvThreads) : "memory"); }

// Byte offset of 16-byte chunk c of an activation row: chunks are swizzled
// (bit 1 of the chunk index flipped by its bit 3) so that the four spans of
// a thread quad fall into distinct bank groups.
SBN_DEVFN int gv_xchunk(int c) { return 16 * (c ^ ((c >> 2) & 2)); }

// W bits of the word array starting at bit OFF (compile-time positions).
template <int OFF, int W, int NW>
SBN_DEVFN uint32_t gv_bits(const uint32_t (&w)[NW]) {
  constexpr int i = OFF / 32, s = OFF % 32;
  uint32_t v;
  if constexpr (s + W <= 32) {
    v = w[i] >> s;
    if constexpr (s + W < 32) v &= (1u << W) - 1u;
  } else {
    v = __funnelshift_r(w[i], w[i + 1], s);
    if constexpr (W < 32) v &= (1u << W) - 1u;
  }
  return v;
}

SBN_DEVFN uint32_t gv_prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;   // byte permute; only the low 16 bits of sel are read
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Up to eight codes (low 16 bits of v; codes past the group's count zero) ->
// int8 bytes of the even-indexed codes (ev: code 2k in byte k) and of the
// odd-indexed ones (od: code 2k+1 in byte k). Masking v with 0x3333 leaves
// code 2k alone in nibble k, which then selects its byte of the table
// {0, +1, 0, -1}; the odd codes are the same two bits higher.
SBN_DEVFN void gv_codes_eo(uint32_t v, uint32_t& ev, uint32_t& od) {
  ev = gv_prmt(kCodeByteTable, 0u, v & 0x3333u);
  od = gv_prmt(kCodeByteTable, 0u, (v >> 2) & 0x3333u);
}

// Selector pair of a keep mask over (ev, od): output byte i takes kept value
// j (the j-th set bit below i), found in ev byte j/2 (even j) or od byte
// (j-1)/2 (odd j); pruned positions take od byte 3 (code 7), which is zero
// because a group with a pruned position keeps fewer than 8 codes.
SBN_DEVFN uint2 gv_selector_pair(uint32_t mask8) {
  uint32_t sel = 0u, j = 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t bit = (mask8 >> i) & 1u;
    const uint32_t src = bit ? ((j & 1u) ? 4u + (j >> 1) : (j >> 1)) : 7u;
    sel |= src << (4 * i);
    j += bit;
  }
  return make_uint2(sel & 0xFFFFu, sel >> 16);
}

// The bits of the word array from bit OFF on, masked with MASK (compile-time
// positions; MASK's highest bit below 32 - OFF % 32 + 32).
template <int OFF, uint32_t MASK, int NW>
SBN_DEVFN uint32_t gv_field(const uint32_t (&w)[NW]) {
  constexpr int i = OFF / 32, s = OFF % 32;
  constexpr int width = 32 - __builtin_clz(MASK);
  if constexpr (s + width <= 32) {
    return (w[i] >> s) & MASK;
  } else {
    return __funnelshift_r(w[i], w[i + 1], s) & MASK;
  }
}

// Eight positions (group I of the thread's span) of one row -> int8 bytes
// 0-3 (w0) and 4-7 (w1). cw: the span's code words; mw: its 8 keep bytes;
// s_sel2: the selector pairs of the 256 keep masks.
template <int MM, int CB, bool DENSE, int I>
SBN_DEVFN void gv_expand(const uint32_t (&cw)[CB], const uint32_t (&mw)[2], const uint2* s_sel2, uint32_t& w0,
                         uint32_t& w1) {
  if constexpr (DENSE) {
    // n == m: 8 codes per group, no keep bits; interleave even and odd
    uint32_t ev, od;
    gv_codes_eo(gv_bits<16 * I, 16, CB>(cw), ev, od);
    w0 = gv_prmt(ev, od, 0x5140u);
    w1 = gv_prmt(ev, od, 0x7362u);
    return;
  } else if constexpr (MM != 16) {
    // m = 4 or 8: every 8 positions keep 2*CB codes; the even- and
    // odd-indexed codes are cut straight out of the code words
    constexpr int kOff = 4 * CB * I;
    constexpr uint32_t kMask = CB == 1 ? 0x3u : CB == 2 ? 0x33u : 0x333u;
    const uint32_t m8 = gv_prmt(mw[I / 4], 0u, 0x4440u | (I % 4));
    const uint32_t ev = gv_prmt(kCodeByteTable, 0u, gv_field<kOff, kMask, CB>(cw));
    const uint32_t od = gv_prmt(kCodeByteTable, 0u, gv_field<kOff + 2, kMask, CB>(cw));
    const uint2 sel = s_sel2[m8];
    w0 = gv_prmt(ev, od, sel.x);
    w1 = gv_prmt(ev, od, sel.y);
    return;
  } else {
    // m = 16: a 16-position group keeps 4*CB codes, split unevenly between
    // its halves; the second half's codes follow the first half's
    const uint32_t u = gv_bits<8 * CB * (I / 2), 8 * CB, CB>(cw);
    const uint32_t mlo = gv_prmt(mw[I / 4], 0u, 0x4440u | ((I & ~1) % 4));
    const int klo = __popc(mlo);
    uint32_t v;
    if constexpr (I % 2 == 0) {
      v = u & ((1u << (2 * klo)) - 1u);   // klo <= 8
    } else {
      v = u >> (2 * klo);
    }
    const uint32_t m8 = gv_prmt(mw[I / 4], 0u, 0x4440u | (I % 4));
    uint32_t ev, od;
    gv_codes_eo(v, ev, od);
    const uint2 sel = s_sel2[m8];
    w0 = gv_prmt(ev, od, sel.x);
    w1 = gv_prmt(ev, od, sel.y);
  }
}

// MM: group size m; CB: code bytes per 16 positions (= 4n/m); NT: token
// columns (8 or 16); DENSE: n == m (no keep bits); ACC: write int32 acc;
// XBF: quantize bf16 activations in the kernel.
template <int MM, int CB, int NT, bool DENSE, bool ACC, bool XBF>
__global__ void __launch_bounds__(kGvThreads, 1)
bl_gemv_kernel(const GvParams p) {
  extern __shared__ __align__(128) uint8_t gv_smem[];
  const GvLayout& L = p.L;
  const int bid = blockIdx.x;
  const int tiles = p.tile_base + (bid < p.tile_rem ? 1 : 0);
  const int t_begin = bid * p.tile_base + min(bid, p.tile_rem);
  const int row0 = t_begin * 16;
  uint2* s_sel2 = reinterpret_cast<uint2*>(gv_smem + L.sel);
  int32_t* s_acc = reinterpret_cast<int32_t*>(gv_smem + L.acc);
  uint32_t* s_rmax = reinterpret_cast<uint32_t*>(gv_smem + L.rmax);
  float* s_scale = reinterpret_cast<float*>(gv_smem + L.scale);
  float* s_ysc = reinterpret_cast<float*>(gv_smem + L.ysc);
  uint64_t* s_bar = reinterpret_cast<uint64_t*>(gv_smem + L.bars);
  uint8_t* s_x = gv_smem + L.x;
  uint8_t* s_codes = gv_smem + L.codes;
  uint8_t* s_meta = gv_smem + L.meta;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (warp == kGvConsumerWarps) {
    // ---- producer warp: barriers, then one bulk copy per tile and array ----
    if (lane < 16) s_rmax[lane] = 0u;
    if (lane == 0) {
      for (int i = 0; i < tiles; ++i) mbar_init(&s_bar[i], 1);
      asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    __syncwarp();
    gv_setup_arrive();
    griddep_wait();
    if (lane == 0) {
      for (int i = 0; i < tiles; ++i) {
        const int r = row0 + 16 * i;
        const uint32_t rows = (uint32_t)min(16, p.N - r);
        const uint32_t cbytes = rows * (uint32_t)p.cstride;
        const uint32_t mbytes = DENSE ? 0u : rows * (uint32_t)p.mstride;
        mbar_arrive_expect_tx(&s_bar[i], cbytes + mbytes);
        bulk_g2s(s_codes + (size_t)16 * i * p.cstride, p.codes + (size_t)r * p.cstride, cbytes, &s_bar[i]);
        if (!DENSE)
          bulk_g2s(s_meta + (size_t)16 * i * p.mstride, p.meta + (size_t)r * p.mstride, mbytes, &s_bar[i]);
      }
    }
    return;   // the consumers wait for every tile before they leave
  }

  // ---- consumers: activations global -> registers ----
  griddep_wait();
  const float gm = ACC ? 0.f : __ldg(p.gamma);
  // chunk q of the T x kc chunks (row q / kc): this thread takes
  // q = tid + 992 j; warps past the last chunk skip the phase
  const int kc = p.kc;
  const int nq = p.T * kc;
  const bool xwarp = warp * 32 < nq;
  const int q0r = (int)__umulhi((uint32_t)tid, p.kc_magic);
  const int q0c = tid - q0r * kc;
  const uint4* xsrc = reinterpret_cast<const uint4*>(XBF ? static_cast<const void*>(p.xbf)
                                                         : static_cast<const void*>(p.xq));
  uint4 v[kGvMaxChunks];
  if (xwarp) {
#pragma unroll
    for (int j = 0; j < kGvMaxChunks; ++j) {
      const int q = tid + j * kGvConsumers;
      if (q < nq) v[j] = __ldg(xsrc + q);
    }
  }
  float xs_t = 0.f;
  if (!XBF && !ACC && tid < p.T) xs_t = __ldg(p.xs + tid);

  // ---- tables (while the loads are in flight) ----
  if (!DENSE && tid < 256) s_sel2[tid] = gv_selector_pair((uint32_t)tid);
  for (int i = tid; i < tiles * 16 * NT; i += kGvConsumers) s_acc[i] = 0;
  gv_setup_wait();   // the producer's barriers and row maxima are initialized

  if (XBF) {
    if (xwarp) {
      // per-row maxima: chunk maxima, reduced per row within the warp, then
      // one shared atomic max per (warp, row)
      int r = q0r, c = q0c;
#pragma unroll
      for (int j = 0; j < kGvMaxChunks; ++j) {
        if (j * kGvConsumers + warp * 32 >= nq) break;   // the whole warp is done
        const bool ok = tid + j * kGvConsumers < nq;
        const uint32_t m2 = ok ? gv_chunk_absmax(v[j], 0u) : 0u;
        const uint32_t m = ok ? max(m2 & 0x7FFFu, (m2 >> 16) & 0x7FFFu) : 0u;
        const int row = ok ? r : -1;
        uint32_t todo = __ballot_sync(0xffffffffu, ok);
        while (todo) {
          const int lead = __ffs(todo) - 1;
          const int lr = __shfl_sync(0xffffffffu, row, lead);
          const bool mine = row == lr;
          const uint32_t rm = __reduce_max_sync(0xffffffffu, mine ? m : 0u);
          if (lane == lead) atomicMax(&s_rmax[lr], rm);
          todo &= ~__ballot_sync(0xffffffffu, mine);
        }
        r += p.dr;
        c += p.drem;
        if (c >= kc) { c -= kc; ++r; }
      }
    }
    gv_consumer_sync();
    if (tid < p.T) {
      const float sc = fmaxf(__uint_as_float(s_rmax[tid] << 16), 1e-5f);
      s_scale[tid] = __fdiv_rn(127.0f, sc);   // the rounding multiplier of the row
      s_ysc[tid] = __fdiv_rn(__fmul_rn(gm, sc), 127.0f);
      if (bid == 0 && p.xs_out) p.xs_out[tid] = sc;
    }
    gv_consumer_sync();
    if (xwarp) {
      const bool out = bid == 0 && p.xq_out != nullptr;
      int r = q0r, c = q0c;
#pragma unroll
      for (int j = 0; j < kGvMaxChunks; ++j) {
        if (j * kGvConsumers + warp * 32 >= nq) break;
        if (tid + j * kGvConsumers < nq) {
          const float mult = s_scale[r];
          // scalar multiply and add: each rounds on its own (a fused
          // multiply-add would round once and break ties of fl32(x * mult))
          const uint2 q = quant8_magic(v[j], mult);
          *reinterpret_cast<uint2*>(s_x + (size_t)r * L.xstride + gv_xchunk(c >> 1) + 8 * (c & 1)) = q;
          if (out) *reinterpret_cast<uint2*>(p.xq_out + (size_t)r * p.K + 8 * (size_t)c) = q;
        }
        r += p.dr;
        c += p.drem;
        if (c >= kc) { c -= kc; ++r; }
      }
    }
  } else {
    if (xwarp) {
      int r = q0r, c = q0c;
#pragma unroll
      for (int j = 0; j < kGvMaxChunks; ++j) {
        if (j * kGvConsumers + warp * 32 >= nq) break;
        if (tid + j * kGvConsumers < nq) *reinterpret_cast<uint4*>(s_x + (size_t)r * L.xstride + gv_xchunk(c)) = v[j];
        r += p.dr;
        c += p.drem;
        if (c >= kc) { c -= kc; ++r; }
      }
    }
    if (!ACC && tid < p.T) s_ysc[tid] = __fdiv_rn(__fmul_rn(gm, xs_t), 127.0f);
  }
  gv_consumer_sync();

  // ---- contraction: warp items of 16 rows x 256 positions ----
  const int g = lane >> 2, t = lane & 3;
  const int ipt = (p.K + 255) / 256;
  const int items = tiles * ipt;
  int cur_tile = -1;
  int acc0[4] = {0, 0, 0, 0};
  int acc1[4] = {0, 0, 0, 0};
  const bool tok0 = g < p.T;
  const bool tok1 = NT == 16 && g + 8 < p.T;
  auto flush = [&](int tile) {
    int32_t* a = s_acc + (size_t)tile * 16 * NT;
    if (2 * t < p.T) {
      atomicAdd(&a[g * NT + 2 * t], acc0[0]);
      atomicAdd(&a[(g + 8) * NT + 2 * t], acc0[2]);
    }
    if (2 * t + 1 < p.T) {
      atomicAdd(&a[g * NT + 2 * t + 1], acc0[1]);
      atomicAdd(&a[(g + 8) * NT + 2 * t + 1], acc0[3]);
    }
    if (NT == 16) {
      if (8 + 2 * t < p.T) {
        atomicAdd(&a[g * NT + 8 + 2 * t], acc1[0]);
        atomicAdd(&a[(g + 8) * NT + 8 + 2 * t], acc1[2]);
      }
      if (8 + 2 * t + 1 < p.T) {
        atomicAdd(&a[g * NT + 8 + 2 * t + 1], acc1[1]);
        atomicAdd(&a[(g + 8) * NT + 8 + 2 * t + 1], acc1[3]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) acc0[i] = acc1[i] = 0;
  };

  for (int it = warp; it < items; it += kGvConsumerWarps) {
    const int tile = it / ipt, kit = it - tile * ipt;
    if (tile != cur_tile) {
      if (cur_tile >= 0) flush(cur_tile);
      cur_tile = tile;
      mbar_wait(&s_bar[tile], 0u);
    }
    const int span = kit * 256 + 64 * t;   // first position of this thread's 64
    const bool valid = span < p.K;
    uint32_t cw[2][CB];
    uint32_t mw[2][2];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int r = tile * 16 + g + 8 * rr;
      const uint32_t* cp = reinterpret_cast<const uint32_t*>(s_codes + (size_t)r * p.cstride + span / 16 * CB);
#pragma unroll
      for (int j = 0; j < CB; ++j) cw[rr][j] = valid ? cp[j] : 0u;
      if (!DENSE) {
        const uint2 m = valid ? *reinterpret_cast<const uint2*>(s_meta + (size_t)r * p.mstride + span / 8)
                              : make_uint2(0u, 0u);
        mw[rr][0] = m.x;
        mw[rr][1] = m.y;
      } else {
        mw[rr][0] = mw[rr][1] = 0u;
      }
    }
    const uint8_t* xa = s_x + (size_t)g * L.xstride;
    const uint8_t* xb = s_x + (size_t)(g + 8) * L.xstride;
    const bool la = valid && tok0, lb = valid && tok1;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int xo = gv_xchunk(span / 16 + j);
      const uint4 fa = la ? *reinterpret_cast<const uint4*>(xa + xo) : make_uint4(0u, 0u, 0u, 0u);
      uint4 fb = make_uint4(0u, 0u, 0u, 0u);
      if (NT == 16) fb = lb ? *reinterpret_cast<const uint4*>(xb + xo) : fb;
      uint32_t a00, a01, a10, a11, b00, b01, b10, b11;
      // groups 2j and 2j+1 of both rows
#define SBN_GV_PAIR(IA, IB)                                             \
      gv_expand<MM, CB, DENSE, IA>(cw[0], mw[0], s_sel2, a00, a01); \
      gv_expand<MM, CB, DENSE, IA>(cw[1], mw[1], s_sel2, a10, a11); \
      gv_expand<MM, CB, DENSE, IB>(cw[0], mw[0], s_sel2, b00, b01); \
      gv_expand<MM, CB, DENSE, IB>(cw[1], mw[1], s_sel2, b10, b11);
      if (j == 0) {
        SBN_GV_PAIR(0, 1)
      } else if (j == 1) {
        SBN_GV_PAIR(2, 3)
      } else if (j == 2) {
        SBN_GV_PAIR(4, 5)
      } else {
        SBN_GV_PAIR(6, 7)
      }
#undef SBN_GV_PAIR
      mma_s8_16x8x32(acc0, a00, a10, a01, a11, fa.x, fa.y);
      mma_s8_16x8x32(acc0, b00, b10, b01, b11, fa.z, fa.w);
      if (NT == 16) {
        mma_s8_16x8x32(acc1, a00, a10, a01, a11, fb.x, fb.y);
        mma_s8_16x8x32(acc1, b00, b10, b01, b11, fb.z, fb.w);
      }
    }
  }
  if (cur_tile >= 0) flush(cur_tile);
  // every tile was waited for above (each has at least one item), so no copy
  // into this CTA's shared memory is still in flight past this barrier
  griddep_launch_dependents();
  gv_consumer_sync();

  const int rows = min(16 * tiles, p.N - row0);
  for (int tok = 0; tok < p.T; ++tok) {
    const float ysc = ACC ? 0.f : s_ysc[tok];
    for (int r = tid; r < rows; r += kGvConsumers) {
      const int a = s_acc[(size_t)(r >> 4) * 16 * NT + (r & 15) * NT + tok];
      if (ACC) {
        p.acc_out[(size_t)tok * p.N + row0 + r] = a;
      } else {
        p.y[(size_t)tok * p.N + row0 + r] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn((float)a, ysc)));
      }
    }
  }
}

}  // namespace sbn
