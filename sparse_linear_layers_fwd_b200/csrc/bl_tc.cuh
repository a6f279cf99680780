// Prefill contraction on the 5th-generation tensor cores (tcgen05, sm_100a),
// without a workspace: the packed weights are expanded in shared memory by
// producer warps (with a workspace the contraction runs on CTA pairs,
// bl_tc2.cuh).
//
// "Microsoft BitNet 1.58: The Era of 1-Bit Large Language Models", section
// "The BitLinear Layer", fourth and fifth operations; the Sparse-BitNet page
// (Abstract, Table 3) runs the sparse BitLinear on tensor cores for prefill.
//
// A persistent CTA per SM walks over 128 (output features) x 256 (tokens)
// tiles of acc = Xq * W^T with `tcgen05.mma.cta_group::1.kind::i8` (int8 x
// int8 -> int32), accumulating in tensor memory:
//   warp 0      TMA loads of the activation tiles (256 x 128 bytes per K
//               block, 128-byte swizzle);
//   warp 1      TMEM allocation and the MMA thread: 4 MMAs (K = 32 each) per
//               K block, tcgen05.commit to free a stage and, after the last
//               K block of a tile, to hand the accumulator to the epilogue;
//   warps 4-11  producers: two threads per weight row read the packed codes +
//               keep bits of their row (prefetched two K blocks ahead),
//               expand them to int8 (expand.cuh) and store them in the K-major
//               128-byte-swizzled layout the MMA reads;
//   warps 12-15 epilogue: tcgen05.ld of the accumulator (each warp owns one
//               quadrant of the 128 TMEM lanes), y = acc * gamma * s_t / 127.
// Two accumulators (2 x 256 TMEM columns) let the epilogue of one tile run
// under the main loop of the next. Stage ring: `full` (256 producer arrivals
// + the TMA bytes) and `empty` (MMA commit) barriers; accumulator ring:
// `acc_full` (MMA commit) and `acc_empty` (one arrival per epilogue warp).
// Barriers are waited on and arrived at once per warp (lane 0, then
// __syncwarp), not per thread. Every mbarrier wait is bounded in time; a wait
// that gives up records SBN_ERR_TIMEOUT in the device error word and the CTA
// winds down.
#pragma once

#include <cuda.h>

#include "async.cuh"
#include "common.cuh"
#include "expand.cuh"

namespace sbn {

constexpr int kTcBM = 128;      // output features per tile (MMA M)
constexpr int kTcBN = 256;      // tokens per tile (MMA N)
constexpr int kTcBK = 128;      // K positions per stage (one 128-byte swizzle row)
constexpr int kTcStages = 4;
constexpr int kTcABytes = kTcBM * kTcBK;
constexpr int kTcBBytes = kTcBN * kTcBK;
constexpr int kTcStageBytes = kTcABytes + kTcBBytes;
constexpr int kTcThreads = 512;
constexpr int kTcProducers = 256;     // two threads per weight row
constexpr int kTcEpilogue = 128;
constexpr uint32_t kTcTmemCols = 512; // two 256-column accumulators
// instruction descriptor: s32 accumulate, signed 8-bit A and B, both K-major,
// N = 256 (bits 17-22 hold N >> 3), M = 128 (bits 24-28 hold M >> 4)
constexpr uint32_t kTcIdesc = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kTcBN >> 3) << 17) |
                              ((uint32_t)(kTcBM >> 4) << 24);

// dynamic shared memory: stages (1024-aligned), then barriers and tables
constexpr int kTcSelCopies = 8;       // selector table copies (fewer bank conflicts)
constexpr size_t kTcSmemBytes = 1024 /*alignment slack*/ + (size_t)kTcStages * kTcStageBytes +
                                 (2 * kTcStages + 4) * 8 + 16 + 256 * 4 * kTcSelCopies;

struct TcParams {
  const uint8_t* codes;
  const uint8_t* meta;
  const float* xs;
  const float* gamma;
  uint16_t* y;
  int32_t* acc_out;
  int T, K, N;
  int cstride, mstride;
};

SBN_DEVFN uint64_t sw128_kmajor_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);   // start address (16-byte units)
  d |= (uint64_t)1 << 16;                    // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;          // stride byte offset: 8 rows x 128 bytes
  d |= (uint64_t)1 << 46;                    // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                    // 128-byte swizzle
  return d;
}

SBN_DEVFN void tc_mma_i8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(kTcIdesc), "r"(accumulate), "r"(0u)
      : "memory");
}
SBN_DEVFN void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                   smem_u32(bar))
               : "memory");
}
SBN_DEVFN void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
SBN_DEVFN void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }

SBN_DEVFN void tma_load_2d(void* smem_dst, const CUtensorMap* tmap, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

SBN_DEVFN void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
}

// Code bits [bit, bit + nbits) (nbits <= 32) of a little-endian word array.
template <int NW>
SBN_DEVFN uint32_t code_bits(const uint32_t (&cw)[NW], int bit) {
  const int w = bit >> 5, s = bit & 31;
  const uint32_t lo = cw[w];
  const uint32_t hi = (w + 1 < NW) ? cw[w + 1] : 0u;
  return s ? ((lo >> s) | (hi << (32 - s))) : lo;
}

template <int MM, int CB, bool DENSE, bool ACC>
__global__ void __launch_bounds__(kTcThreads, 1)
bl_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)kTcStages * kTcStageBytes);
  uint64_t* empty = full + kTcStages;
  uint64_t* acc_full = empty + kTcStages;   // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2]
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(acc_empty + 2);
  uint32_t* s_sel = s_tmem + 4;             // [256][kTcSelCopies]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nkb = p.K / kTcBK;
  const int row_tiles = (p.N + kTcBM - 1) / kTcBM;
  const int n_tiles = row_tiles * ((p.T + kTcBN - 1) / kTcBN);

  if (tid == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      // one arrival per producer warp + the TMA thread's
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
                 "r"(kTcTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  if (!DENSE) {
    for (int i = tid; i < 256 * kTcSelCopies; i += blockDim.x) s_sel[i] = expand_selector((uint32_t)(i / kTcSelCopies));
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
        const int tok0 = (tile / row_tiles) * kTcBN;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kTcStages;
          const uint32_t ph = (it / kTcStages) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[s], kTcBBytes);
          tma_load_2d(smem + (size_t)s * kTcStageBytes + kTcABytes, &tmap_x, kb * kTcBK, tok0, &full[s]);
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
        const uint32_t d_tmem = tmem + (uint32_t)(b * kTcBN);
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kTcStages;
          const uint32_t ph = (it / kTcStages) & 1u;
          if (!mbar_wait(&full[s], ph)) { ok = false; break; }
          const uint32_t a_addr = smem_u32(smem + (size_t)s * kTcStageBytes);
          const uint64_t adesc = sw128_kmajor_desc(a_addr);
          const uint64_t bdesc = sw128_kmajor_desc(a_addr + kTcABytes);
#pragma unroll
          for (int k = 0; k < kTcBK / 32; ++k) {
            // K advances 32 bytes = 2 units of 16 bytes inside the swizzled row
            tc_mma_i8(d_tmem, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k), (kb > 0 || k > 0) ? 1u : 0u);
          }
          tc_commit(&empty[s]);
        }
        tc_commit(&acc_full[b]);  // arrives once every MMA of this tile has completed
      }
    }
  } else if (warp >= 4 && warp < 12) {
    // ---- producers: thread (i, h) expands units 4h..4h+3 of row i ----
    const int pi = tid - 128;
    const int i = pi & (kTcBM - 1), h = pi >> 7;
    constexpr int kPre = 2;
    constexpr int NW = CB;   // 32-bit words of codes for 4 units (4 * CB bytes)
    uint32_t cwq[kPre + 1][NW];
    uint2 mvq[kPre + 1];
    const uint32_t* sel = s_sel + (lane & (kTcSelCopies - 1));
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
      const int row = (tile % row_tiles) * kTcBM + i;
      const bool row_ok = row < p.N;
      const uint8_t* crow = p.codes + (size_t)(row_ok ? row : 0) * p.cstride + h * 4 * CB;
      const uint8_t* mrow = DENSE ? nullptr : p.meta + (size_t)(row_ok ? row : 0) * p.mstride + h * 8;
      auto load_block = [&](int kb, uint32_t (&cw)[NW], uint2& mv) {
        mv = make_uint2(0xFFFFFFFFu, 0xFFFFFFFFu);
        if (row_ok && kb < nkb) {
          const uint32_t* cp = reinterpret_cast<const uint32_t*>(crow + (size_t)kb * 8 * CB);
#pragma unroll
          for (int q = 0; q < NW; ++q) cw[q] = __ldg(cp + q);
          if (!DENSE) mv = __ldg(reinterpret_cast<const uint2*>(mrow + (size_t)kb * 16));
        } else {
#pragma unroll
          for (int q = 0; q < NW; ++q) cw[q] = 0u;
        }
      };
#pragma unroll
      for (int jj = 0; jj < kPre; ++jj) load_block(jj, cwq[jj], mvq[jj]);
      for (int kb = 0; kb < nkb; ++kb, ++it) {
        const int s = it % kTcStages;
        const uint32_t ph = (it / kTcStages) & 1u;
        load_block(kb + kPre, cwq[kPre], mvq[kPre]);
        uint32_t cw[NW];
#pragma unroll
        for (int q = 0; q < NW; ++q) cw[q] = cwq[0][q];
        const uint2 mv = mvq[0];
#pragma unroll
        for (int jj = 0; jj < kPre; ++jj) {
#pragma unroll
          for (int q = 0; q < NW; ++q) cwq[jj][q] = cwq[jj + 1][q];
          mvq[jj] = mvq[jj + 1];
        }
        // lane 0 waits for the stage, the warp follows
        int got = 1;
        if (lane == 0) got = mbar_wait(&empty[s], ph ^ 1u) ? 1 : 0;
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) { ok = false; break; }
        uint8_t* arow = smem + (size_t)s * kTcStageBytes + (size_t)i * 128;
        const uint32_t mw[2] = {mv.x, mv.y};
#pragma unroll
        for (int uu = 0; uu < 4; ++uu) {
          const int u = 4 * h + uu;
          const uint32_t m16 = (mw[uu >> 1] >> (16 * (uu & 1))) & 0xFFFFu;
          const uint32_t ucodes = code_bits<NW>(cw, uu * 8 * CB);  // this unit's 8*CB code bits
          uint32_t out[4];
          if (DENSE) {
            codes8_to_s8(ucodes & 0xFFFFu, out[0], out[1]);
            codes8_to_s8(ucodes >> 16, out[2], out[3]);
          } else {
            const uint32_t m0 = m16 & 0xFFu, m1 = m16 >> 8;
            const int p0 = (MM == 16) ? __popc(m0) : 2 * CB;
            const uint32_t v0 = ucodes & ((1u << (2 * p0)) - 1u);
            const uint32_t rest = ucodes >> (2 * p0);   // 2 * p0 <= 16
            const int p1 = (MM == 16) ? __popc(m1) : 2 * CB;
            const uint32_t v1 = rest & ((1u << (2 * p1)) - 1u);
            uint32_t q0, q1;
            codes8_to_s8(v0, q0, q1);
            const uint32_t s0 = sel[m0 * kTcSelCopies];
            out[0] = __byte_perm(q0, q1, s0 & 0xFFFFu);
            out[1] = __byte_perm(q0, q1, s0 >> 16);
            codes8_to_s8(v1, q0, q1);
            const uint32_t s1 = sel[m1 * kTcSelCopies];
            out[2] = __byte_perm(q0, q1, s1 & 0xFFFFu);
            out[3] = __byte_perm(q0, q1, s1 >> 16);
          }
          *reinterpret_cast<uint4*>(arow + ((u ^ (i & 7)) << 4)) = make_uint4(out[0], out[1], out[2], out[3]);
        }
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[s]);
      }
    }
  } else if (warp >= 12) {
    // ---- epilogue: TMEM -> registers -> y (or acc) ----
    // warp w reads TMEM lane quadrant w % 4
    const int q = warp & 3;
    const int c_first = 0;
    const int c_count = kTcBN / 32;
    const int row_in_tile = 32 * q + lane;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    const float g = ACC ? 0.f : __ldg(p.gamma);
    int j = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++j) {
      const int b = j & 1;
      const int row = (tile % row_tiles) * kTcBM + row_in_tile;
      const int tok0 = (tile / row_tiles) * kTcBN;
      int got = 1;
      if (lane == 0) got = mbar_wait(&acc_full[b], (j >> 1) & 1u) ? 1 : 0;
      got = __shfl_sync(0xffffffffu, got, 0);
      if (!got) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = c_first; c < c_first + c_count; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + (uint32_t)(b * kTcBN + 32 * c), r);
        // lane jj holds the scale gamma * s_t / 127 of token tok0 + 32c + jj
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
    // no MMA may still be writing an accumulator when TMEM is freed (this
    // matters only on the abort path): wait for the last commits
    if (lane == 0) {
      const int my_tiles = n_tiles > (int)blockIdx.x ? (n_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
      for (int jj = my_tiles - 2; jj < my_tiles; ++jj)
        if (jj >= 0) mbar_wait(&acc_full[jj & 1], (jj >> 1) & 1u);
    }
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTcTmemCols)
                 : "memory");
  }
}

}  // namespace sbn
