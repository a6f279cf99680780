// Prefill contraction of 2:4 weights on the sparse tensor-core path
// (`tcgen05.mma.sp.cta_group::1.kind::i8`, sm_100a).
//
// "Sparse-BitNet: 1.58-bit LLMs are Naturally Friendly to Semi-Structured
// Sparsity", Abstract and Table 3: the 2:4 pattern is the one the sparse
// tensor cores execute natively, so the weights stay compressed all the way
// into the MMA. The sparse MMA takes A (the weights, 128 rows) as the kept
// values only -- two int8 per group of four positions, in position order --
// plus 4 bits of metadata per group, the positions of the two kept values
// (i0 | i1 << 2, i0 < i1), read from tensor memory. One MMA covers 64 K
// positions: 32 bytes of A per row, 64 bytes of B per token, and two TMEM
// columns of metadata per row (lane = row, group g of the 64 positions at
// bits 4(g % 8) of column g / 8).
//
// The packed 2:4 format maps onto this directly: a unit of 16 positions has
// 8 kept 2-bit codes (in position order) and a 16-bit keep mask whose four
// nibbles are the groups' masks. The kept codes expand to the 8 bytes of A,
// and each group mask (exactly two bits set) maps to its metadata nibble.
//
// Tiles: 128 output features x 224 tokens per tile (two 224-column
// accumulators plus the metadata ring fit in the 512 TMEM columns), 128 K
// positions per pipeline stage:
//   A  128 rows x 64 bytes   (64-byte swizzle, K-major)
//   B  224 tokens x 128 bytes (128-byte swizzle, K-major)
//   E  128 rows x 16 bytes   (metadata, plain rows of 16 bytes)
// The MMA thread copies each stage's E into its TMEM slot (tcgen05.cp
// 128x128b) ahead of the stage's two MMAs; copies and MMAs of one thread run
// in issue order, and a slot is rewritten only after the stage's `empty`
// commit has come back through the load of the next round.
//
// This single-CTA kernel is the route without a workspace (the packed rows
// are expanded in shared memory); with a workspace, 2:4 runs on CTA pairs
// (bl_tc2.cuh). Warp roles as in the dense kernel: warp 0 TMA of the
// activations, warp 1 TMEM + MMA thread, warps 4-11 expanding the packed
// rows into A and E, warps 12-15 draining the accumulators.
#pragma once

#include <cuda.h>

#include "async.cuh"
#include "bl_tc.cuh"
#include "common.cuh"
#include "expand.cuh"

namespace sbn {

constexpr int kSpBM = 128;                      // output features per tile (MMA M)
constexpr int kSpBN = 224;                      // tokens per tile (MMA N)
constexpr int kSpBK = 128;                      // K positions per stage
constexpr int kSpStages = 5;
constexpr int kSpABytes = kSpBM * kSpBK / 2;    // 8 KB of kept values
constexpr int kSpBBytes = kSpBN * kSpBK;        // 28 KB of activations
constexpr int kSpEBytes = kSpBM * kSpBK / 8;    // 2 KB of metadata
constexpr int kSpStageBytes = kSpABytes + kSpBBytes + kSpEBytes;
static_assert(kSpStageBytes % 1024 == 0, "stages must stay 1024-byte aligned");
constexpr uint32_t kSpTmemCols = 512;
constexpr uint32_t kSpEcol = 2 * kSpBN;         // metadata slots start after the accumulators
static_assert(kSpEcol + 4 * kSpStages <= kSpTmemCols, "metadata ring must fit in TMEM");
// instruction descriptor: sparse (bit 2), s32 accumulate, signed 8-bit A and
// B, both K-major, N = 224, M = 128; metadata selector 0
constexpr uint32_t kSpIdesc = (1u << 2) | (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kSpBN >> 3) << 17) |
                              ((uint32_t)(kSpBM >> 4) << 24);
constexpr size_t kSpSmemBytes = 1024 + (size_t)kSpStages * kSpStageBytes + (2 * kSpStages + 4) * 8 + 16;

// Metadata nibble of one group mask: the positions of its two kept values
// (low one in bits 0-1). A mask without exactly two bits (never produced by
// the 2:4 mask) maps to positions (0, 1), so the MMA always sees valid
// metadata.
__host__ __device__ constexpr uint32_t sp_nibble(uint32_t m4) {
  uint32_t lo = 0, hi = 0, c = 0;
  for (uint32_t i = 0; i < 4; ++i)
    if ((m4 >> i) & 1u) {
      if (c == 0) lo = i;
      hi = i;
      ++c;
    }
  return c == 2 ? (lo | (hi << 2)) : 0x4u;
}
__host__ __device__ constexpr uint64_t sp_nibble_table() {
  uint64_t t = 0;
  for (uint32_t m = 0; m < 16; ++m) t |= (uint64_t)sp_nibble(m) << (4 * m);
  return t;
}
constexpr uint64_t kSpNibbles = sp_nibble_table();
static_assert(sp_nibble(0x3) == 0x4 && sp_nibble(0x5) == 0x8 && sp_nibble(0x9) == 0xC && sp_nibble(0x6) == 0x9 &&
                  sp_nibble(0xA) == 0xD && sp_nibble(0xC) == 0xE,
              "metadata nibbles of the six 2:4 group masks");

// 16-bit keep mask of a unit (four groups) -> its 16 metadata bits.
SBN_DEVFN uint32_t sp_meta16(uint32_t m16) {
  uint32_t r = 0;
#pragma unroll
  for (int g = 0; g < 4; ++g) r |= (uint32_t)((kSpNibbles >> (4 * ((m16 >> (4 * g)) & 0xFu))) & 0xFu) << (4 * g);
  return r;
}

SBN_DEVFN uint64_t sw64_kmajor_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);   // start address (16-byte units)
  d |= (uint64_t)1 << 16;                    // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(512 >> 4) << 32;           // stride byte offset: 8 rows x 64 bytes
  d |= (uint64_t)1 << 46;                    // descriptor version (sm_100)
  d |= (uint64_t)4 << 61;                    // 64-byte swizzle
  return d;
}

// Metadata block of a stage: 128 rows of 16 bytes, no swizzle. Core
// matrices of 8 rows x 16 bytes lie 128 bytes apart; there is a single one
// across the 16 bytes, so both offsets are given the same 128 bytes.
SBN_DEVFN uint64_t meta_block_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)(128 >> 4) << 16;
  d |= (uint64_t)(128 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  return d;
}

SBN_DEVFN void tc_cp_meta(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.128x128b [%0], %1;\n" ::"r"(taddr), "l"(sdesc) : "memory");
}

SBN_DEVFN void tc_mma_sp_i8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t tmem_e, uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.sp.cta_group::1.kind::i8 [%0], %1, %2, [%6], %3, {%5, %5, %5, %5}, p;\n}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(kSpIdesc), "r"(accumulate), "r"(0u), "r"(tmem_e)
      : "memory");
}

template <bool ACC>
__global__ void __launch_bounds__(kTcThreads, 1)
bl_tc_sp_kernel(const __grid_constant__ CUtensorMap tmap_x, const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)kSpStages * kSpStageBytes);
  uint64_t* empty = full + kSpStages;
  uint64_t* acc_full = empty + kSpStages;   // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2]
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nkb = p.K / kSpBK;
  const int row_tiles = (p.N + kSpBM - 1) / kSpBM;
  const int n_tiles = row_tiles * ((p.T + kSpBN - 1) / kSpBN);

  if (tid == 0) {
    for (int s = 0; s < kSpStages; ++s) {
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
                 "r"(kSpTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 0) {
    // ---- TMA producer of the activation tiles ----
    if (lane == 0) {
      int it = 0;
      for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        const int tok0 = (tile / row_tiles) * kSpBN;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kSpStages;
          const uint32_t ph = (it / kSpStages) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u)) { ok = false; break; }
          uint8_t* st = smem + (size_t)s * kSpStageBytes;
          mbar_arrive_expect_tx(&full[s], kSpBBytes);
          tma_load_2d(st + kSpABytes, &tmap_x, kb * kSpBK, tok0, &full[s]);
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
        const uint32_t d_tmem = tmem + (uint32_t)(b * kSpBN);
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kSpStages;
          const uint32_t ph = (it / kSpStages) & 1u;
          if (!mbar_wait(&full[s], ph)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + (size_t)s * kSpStageBytes);
          const uint64_t adesc = sw64_kmajor_desc(a_addr);
          const uint64_t bdesc = sw128_kmajor_desc(a_addr + kSpABytes);
          const uint32_t e_tmem = tmem + kSpEcol + 4u * (uint32_t)s;
          tc_cp_meta(e_tmem, meta_block_desc(a_addr + kSpABytes + kSpBBytes));
#pragma unroll
          for (int k = 0; k < kSpBK / 64; ++k) {
            // 64 K positions per MMA: A advances 32 bytes (2 units of 16
            // bytes), B 64 bytes (4 units), the metadata two columns
            tc_mma_sp_i8(d_tmem, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(4 * k), e_tmem + 2u * (uint32_t)k,
                         (kb > 0 || k > 0) ? 1u : 0u);
          }
          tc_commit(&empty[s]);
        }
        tc_commit(&acc_full[b]);
      }
    }
  } else if (warp >= 4 && warp < 12) {
    // ---- producers: thread (i, h) expands units 4h..4h+3 of row i ----
    const int pi = tid - 128;
    const int i = pi & (kSpBM - 1), h = pi >> 7;
    constexpr int kPre = 2;
    uint2 cq[kPre + 1], mq[kPre + 1];
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
      const int row = (tile % row_tiles) * kSpBM + i;
      const bool row_ok = row < p.N;
      // 2 code bytes and 2 keep-mask bytes per unit: 8 + 8 bytes per thread and stage
      const uint8_t* crow = p.codes + (size_t)(row_ok ? row : 0) * p.cstride + h * 8;
      const uint8_t* mrow = p.meta + (size_t)(row_ok ? row : 0) * p.mstride + h * 8;
      auto load_block = [&](int kb, uint2& cv, uint2& mv) {
        if (row_ok && kb < nkb) {
          cv = __ldg(reinterpret_cast<const uint2*>(crow + (size_t)kb * 16));
          mv = __ldg(reinterpret_cast<const uint2*>(mrow + (size_t)kb * 16));
        } else {
          cv = make_uint2(0u, 0u);
          mv = make_uint2(0x33333333u, 0x33333333u);   // zero values, valid metadata
        }
      };
#pragma unroll
      for (int jj = 0; jj < kPre; ++jj) load_block(jj, cq[jj], mq[jj]);
      for (int kb = 0; kb < nkb; ++kb, ++it) {
        const int s = it % kSpStages;
        const uint32_t ph = (it / kSpStages) & 1u;
        load_block(kb + kPre, cq[kPre], mq[kPre]);
        const uint2 cv = cq[0], mv = mq[0];
#pragma unroll
        for (int jj = 0; jj < kPre; ++jj) {
          cq[jj] = cq[jj + 1];
          mq[jj] = mq[jj + 1];
        }
        int got = 1;
        if (lane == 0) got = mbar_wait(&empty[s], ph ^ 1u) ? 1 : 0;
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) { ok = false; break; }
        uint8_t* st = smem + (size_t)s * kSpStageBytes;
        // A: row i holds 64 bytes (units 0-7, 8 bytes each); this thread
        // writes 16-byte chunks 2h and 2h+1, at their 64-byte-swizzle places
        uint32_t a[8];
        codes8_to_s8(cv.x & 0xFFFFu, a[0], a[1]);
        codes8_to_s8(cv.x >> 16, a[2], a[3]);
        codes8_to_s8(cv.y & 0xFFFFu, a[4], a[5]);
        codes8_to_s8(cv.y >> 16, a[6], a[7]);
        uint8_t* arow = st + (size_t)i * 64;
        const int sw = (i >> 1) & 3;
        *reinterpret_cast<uint4*>(arow + (((2 * h) ^ sw) << 4)) = make_uint4(a[0], a[1], a[2], a[3]);
        *reinterpret_cast<uint4*>(arow + (((2 * h + 1) ^ sw) << 4)) = make_uint4(a[4], a[5], a[6], a[7]);
        // E: row i holds 16 bytes, 2 per unit; this thread writes bytes 8h..8h+7
        const uint32_t e0 = sp_meta16(mv.x & 0xFFFFu) | (sp_meta16(mv.x >> 16) << 16);
        const uint32_t e1 = sp_meta16(mv.y & 0xFFFFu) | (sp_meta16(mv.y >> 16) << 16);
        *reinterpret_cast<uint2*>(st + kSpABytes + kSpBBytes + (size_t)i * 16 + 8 * h) = make_uint2(e0, e1);
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[s]);
      }
    }
  } else if (warp >= 12) {
    // ---- epilogue: TMEM -> registers -> y (or acc); warp w reads TMEM
    // lane quadrant w % 4 ----
    constexpr int kChunks = kSpBN / 32;
    const int q = warp & 3;
    const int c_first = 0;
    const int c_end = kChunks;
    const int row_in_tile = 32 * q + lane;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const float g = ACC ? 0.f : __ldg(p.gamma);
    int j = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++j) {
      const int b = j & 1;
      const int row = (tile % row_tiles) * kSpBM + row_in_tile;
      const int tok0 = (tile / row_tiles) * kSpBN;
      int got = 1;
      if (lane == 0) got = mbar_wait(&acc_full[b], (j >> 1) & 1u) ? 1 : 0;
      got = __shfl_sync(0xffffffffu, got, 0);
      if (!got) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = c_first; c < c_end; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + (uint32_t)(b * kSpBN + 32 * c), r);
        const int my_tok = tok0 + 32 * c + lane;
        const float my_sc = (ACC || my_tok >= p.T) ? 0.f : __fdiv_rn(__fmul_rn(g, __ldg(p.xs + my_tok)), 127.0f);
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          const int tok = tok0 + 32 * c + jj;
          const float sc = __shfl_sync(0xffffffffu, my_sc, jj);
          if (row < p.N && tok < p.T) {
            if (ACC) {
              p.acc_out[(size_t)tok * p.N + row] = (int32_t)r[jj];
            } else {
              const float yv = __fmul_rn((float)(int32_t)r[jj], sc);
              p.y[(size_t)tok * p.N + row] = __bfloat16_as_ushort(__float2bfloat16_rn(yv));
            }
          }
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
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kSpTmemCols)
                 : "memory");
  }
}

// Compressed 2:4 workspace (the operands of the CTA-pair kernel): kept
// values int8 [N_out, K/2] (a unit's 8 kept codes -> 8 bytes) and metadata
// [N_pad, K/8] (a unit's keep mask -> 16 metadata bits), N_pad = N_out
// rounded up to 256; pad rows get the metadata of positions (0, 1), so every
// row the MMA reads is valid. One thread takes 8 consecutive units of a row
// (K is a multiple of 128): 16-byte loads of their codes and keep masks,
// 16-byte stores of 64 value bytes and 16 metadata bytes; a warp takes 32
// consecutive groups, the chunks dealt out over all CTAs. One CTA of 1024
// threads per SM (the host requests more than half of an SM's shared memory,
// unused, to keep a second one off): launched behind the previous
// contraction, CTAs are placed as its CTAs retire, and several on the SMs
// freed first would leave the others idle. (The contraction that follows
// could not share the SM anyway: registers.)
constexpr int kSpXThreads = 1024;
constexpr int kSpXExclusiveSmem = 120 * 1024;
__global__ void __launch_bounds__(kSpXThreads)
expand_sparse24_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ meta, int n_out, int n_pad,
                       int k, int cstride, int mstride, int8_t* __restrict__ wsp, uint8_t* __restrict__ esp) {
  griddep_wait();
  griddep_launch_dependents();
  const int gpr = k >> 7;   // groups of 8 units per row
  const long long total = (long long)n_pad * gpr;
  // chunks of 32 consecutive groups, one per warp, dealt out CTA-first
  const long long nchunk = (total + 31) / 32;
  for (long long c = (long long)(threadIdx.x >> 5) * gridDim.x + blockIdx.x; c < nchunk;
       c += (long long)gridDim.x * (blockDim.x >> 5)) {
    const long long g = c * 32 + (threadIdx.x & 31);
    if (g >= total) continue;
    const int row = (int)(g / gpr);
    const int gu = (int)(g - (long long)row * gpr);
    uint4 e = make_uint4(0x44444444u, 0x44444444u, 0x44444444u, 0x44444444u);
    if (row < n_out) {
      const uint4 cw = __ldg(reinterpret_cast<const uint4*>(codes + (size_t)row * cstride + (size_t)gu * 16));
      const uint4 mw = __ldg(reinterpret_cast<const uint4*>(meta + (size_t)row * mstride + (size_t)gu * 16));
      const uint32_t c4[4] = {cw.x, cw.y, cw.z, cw.w};
      uint4* dst = reinterpret_cast<uint4*>(wsp + (size_t)row * (k / 2) + (size_t)gu * 64);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        // two units per 32-bit word of codes: 16 kept values -> 16 bytes
        uint32_t q0, q1, q2, q3;
        codes8_to_s8(c4[i] & 0xFFFFu, q0, q1);
        codes8_to_s8(c4[i] >> 16, q2, q3);
        dst[i] = make_uint4(q0, q1, q2, q3);
      }
      e.x = sp_meta16(mw.x & 0xFFFFu) | (sp_meta16(mw.x >> 16) << 16);
      e.y = sp_meta16(mw.y & 0xFFFFu) | (sp_meta16(mw.y >> 16) << 16);
      e.z = sp_meta16(mw.z & 0xFFFFu) | (sp_meta16(mw.z >> 16) << 16);
      e.w = sp_meta16(mw.w & 0xFFFFu) | (sp_meta16(mw.w >> 16) << 16);
    }
    *reinterpret_cast<uint4*>(esp + (size_t)row * (k / 8) + (size_t)gu * 16) = e;
  }
}

}  // namespace sbn
