// Prefill contraction on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// "Microsoft BitNet 1.58: The Era of 1-Bit Large Language Models", section
// "The BitLinear Layer", fourth and fifth operations; the Sparse-BitNet page
// (Abstract, Table 3) runs the sparse BitLinear on tensor cores for prefill.
//
// One CTA computes a 128 (output features) x 256 (tokens) tile of
// acc = Xq * W^T with `tcgen05.mma.cta_group::1.kind::i8` (int8 x int8 ->
// int32), the accumulator in tensor memory:
//   A (weights, 128 x 128 per K block) -- four producer warps read the packed
//     codes + keep bits of their row from global memory, expand them to int8
//     (expand.cuh) and store them in shared memory in the K-major
//     128-byte-swizzled layout the MMA reads;
//   B (activations, 256 x 128 per K block) -- one TMA load per stage, same
//     swizzled layout;
//   a ring of kTcStages stages: `full` barriers (128 producer arrivals + the
//     TMA transaction bytes) and `empty` barriers (tcgen05.commit of the MMAs
//     that read the stage);
//   the MMA thread issues 4 MMAs (K = 32 each) per stage;
//   the epilogue (the producer warps, which own TMEM lanes 0-127) reads the
//     accumulator with tcgen05.ld and writes y = acc * gamma * s_t / 127.
// Every mbarrier wait is bounded; a wait that gives up records
// SBN_ERR_TIMEOUT in the device error word and the CTA winds down.
#pragma once

#include <cuda.h>

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
constexpr int kTcThreads = 256;
constexpr uint32_t kTcTmemCols = 256;
// instruction descriptor: s32 accumulate, signed 8-bit A and B, both K-major,
// N = 256 (bits 17-22 hold N >> 3), M = 128 (bits 24-28 hold M >> 4)
constexpr uint32_t kTcIdesc = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kTcBN >> 3) << 17) |
                              ((uint32_t)(kTcBM >> 4) << 24);
constexpr long long kTcSpinLimit = 1ll << 22;  // try_wait rounds before giving up (~seconds)

// dynamic shared memory: stages (1024-aligned), then barriers and tables
constexpr size_t kTcSmemBytes = 1024 /*alignment slack*/ + (size_t)kTcStages * kTcStageBytes +
                                 (2 * kTcStages + 2) * 8 + 16 + kTcBN * 4 + 256 * 4;

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

SBN_DEVFN uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

SBN_DEVFN void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
SBN_DEVFN void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}
SBN_DEVFN void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// Bounded wait for the phase of the given parity; false if it gave up.
SBN_DEVFN bool mbar_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  for (long long i = 0; i < kTcSpinLimit; ++i) {
    uint32_t done;
    asm volatile(
        "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\nselp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    if (done) return true;
  }
  atomicOr(&g_dev_error, kDevErrTimeout);
  return false;
}

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
  uint64_t* accf = empty + kTcStages;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(accf + 2);
  float* s_scale = reinterpret_cast<float*>(s_tmem + 4);
  uint32_t* s_sel = reinterpret_cast<uint32_t*>(s_scale + kTcBN);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row0 = blockIdx.x * kTcBM, tok0 = blockIdx.y * kTcBN;
  const int nkb = p.K / kTcBK;

  if (tid == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&full[s], kTcBM + 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accf, 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(s_tmem)),
                 "r"(kTcTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  if (!DENSE) fill_selector_table(s_sel);
  if (!ACC && (warp == 2 || warp == 3)) {
    const float g = __ldg(p.gamma);
    for (int j = tid - 64; j < kTcBN; j += 64) {
      const int tok = tok0 + j;
      s_scale[j] = tok < p.T ? __fdiv_rn(__fmul_rn(g, __ldg(p.xs + tok)), 127.0f) : 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 0) {
    // ---- TMA producer of the activation tiles ----
    if (lane == 0) {
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % kTcStages;
        const uint32_t ph = (kb / kTcStages) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u)) break;
        uint8_t* bdst = smem + (size_t)s * kTcStageBytes + kTcABytes;
        mbar_arrive_expect_tx(&full[s], kTcBBytes);
        tma_load_2d(bdst, &tmap_x, kb * kTcBK, tok0, &full[s]);
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer ----
    if (lane == 0) {
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % kTcStages;
        const uint32_t ph = (kb / kTcStages) & 1u;
        if (!mbar_wait(&full[s], ph)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + (size_t)s * kTcStageBytes);
        const uint32_t b_addr = a_addr + kTcABytes;
        const uint64_t adesc = sw128_kmajor_desc(a_addr);
        const uint64_t bdesc = sw128_kmajor_desc(b_addr);
#pragma unroll
        for (int k = 0; k < kTcBK / 32; ++k) {
          // advance K by 32 bytes = 2 units of 16 bytes inside the swizzled row
          tc_mma_i8(tmem, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k), (kb > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit(&empty[s]);
      }
      tc_commit(accf);  // arrives once every MMA issued above has completed
    }
  } else if (warp >= 4) {
    // ---- A producers: expand the packed weights of row i of the tile ----
    const int i = tid - 128;
    const int row = row0 + i;
    const bool row_ok = row < p.N;
    const uint8_t* crow = p.codes + (size_t)(row_ok ? row : 0) * p.cstride;
    const uint8_t* mrow = DENSE ? nullptr : p.meta + (size_t)(row_ok ? row : 0) * p.mstride;
    bool ok = true;
    for (int kb = 0; kb < nkb && ok; ++kb) {
      const int s = kb % kTcStages;
      const uint32_t ph = (kb / kTcStages) & 1u;
      // codes of this K block: 8 units x CB bytes; keep bits: 16 bytes
      uint32_t cw[2 * CB];
      uint4 mv = make_uint4(0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu, 0xFFFFFFFFu);
      if (row_ok) {
        const uint2* cp = reinterpret_cast<const uint2*>(crow + (size_t)kb * 8 * CB);
#pragma unroll
        for (int q = 0; q < CB; ++q) {
          const uint2 v = __ldg(cp + q);
          cw[2 * q] = v.x;
          cw[2 * q + 1] = v.y;
        }
        if (!DENSE) mv = __ldg(reinterpret_cast<const uint4*>(mrow + (size_t)kb * 16));
      } else {
#pragma unroll
        for (int q = 0; q < 2 * CB; ++q) cw[q] = 0u;
      }
      const uint32_t mw[4] = {mv.x, mv.y, mv.z, mv.w};
      if (!mbar_wait(&empty[s], ph ^ 1u)) {
        ok = false;
        break;
      }
      uint8_t* arow = smem + (size_t)s * kTcStageBytes + (size_t)i * 128;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t m16 = (mw[u >> 1] >> (16 * (u & 1))) & 0xFFFFu;
        const uint32_t ucodes = code_bits<2 * CB>(cw, u * 8 * CB);  // this unit's 8*CB code bits
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
          expand8(m0, v0, s_sel, out[0], out[1]);
          expand8(m1, v1, s_sel, out[2], out[3]);
        }
        *reinterpret_cast<uint4*>(arow + ((u ^ (i & 7)) << 4)) = make_uint4(out[0], out[1], out[2], out[3]);
      }
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      mbar_arrive(&full[s]);
    }

    // ---- epilogue: TMEM -> registers -> y (or acc) ----
    if (ok && mbar_wait(accf, 0u)) {
      tc_fence_after();
      const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
#pragma unroll 1
      for (int c = 0; c < kTcBN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + (uint32_t)(32 * c), r);
        if (row_ok) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int tok = tok0 + 32 * c + j;
            if (tok < p.T) {
              if (ACC) {
                p.acc_out[(size_t)tok * p.N + row] = (int32_t)r[j];
              } else {
                const float yv = __fmul_rn((float)(int32_t)r[j], s_scale[32 * c + j]);
                p.y[(size_t)tok * p.N + row] = __bfloat16_as_ushort(__float2bfloat16_rn(yv));
              }
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    // no MMA may still be writing the accumulator when it is freed (this
    // matters only on the abort path; otherwise the phase is long complete)
    if (lane == 0) mbar_wait(accf, 0u);
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kTcTmemCols)
                 : "memory");
  }
}

}  // namespace sbn
