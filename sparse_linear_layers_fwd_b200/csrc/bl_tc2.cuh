// Prefill contraction on CTA pairs: one `tcgen05.mma.cta_group::2` (M = 256)
// spans the tensor cores of two SMs of a cluster.
//
// "Microsoft BitNet 1.58: The Era of 1-Bit Large Language Models", section
// "The BitLinear Layer", fourth and fifth operations; "Sparse-BitNet:
// 1.58-bit LLMs are Naturally Friendly to Semi-Structured Sparsity",
// Abstract and Table 3 (2:4 on the sparse tensor cores).
//
// A CTA pair computes a 256 (weight rows) x BN (tokens) tile: each CTA loads
// its own 128 weight rows and half of the BN activation rows, and the pair's
// MMA reads both halves, so every activation byte serves 256 rows.
//
//   SPARSE (2:4): sparse MMA, BN = 224. Per CTA and 256-position stage: the
//                 kept values (128 rows x 128 bytes, 128-byte swizzle), two
//                 128-position blocks of 112 activation rows (128-byte
//                 swizzle) and two 128 x 16-byte metadata blocks, which one
//                 tcgen05.cp.cta_group::2 per stage moves into a TMEM ring
//                 (each CTA's own rows);
//   dense:        dense MMA on the expanded int8 weights, BN = 256. Per CTA
//                 and stage two 128 x 128-byte weight blocks and two
//                 128-row activation blocks;
//   dense NARROW: the same with BN = 128 (two 64-row activation blocks per
//                 CTA and stage, four stages), for layers whose 256-token
//                 tiles would leave CTA pairs idle: twice the tiles, each
//                 with half the MMA work per stage.
// A stage spans 256 positions because each stage costs the MMA thread one
// mbarrier wait and one commit, time in which it issues no MMA; at 128
// positions per stage that was as long as the stage's sparse MMAs. A K that
// is an odd multiple of 128 ends with a half stage (the second block is
// loaded as zeros by TMA and its MMAs are skipped).
//
// Both operands come by TMA from the caller's workspace. Roles (both CTAs
// run the same code):
//   warp 0   TMA into the CTA's own shared memory; the completions of both
//            CTAs count on the leader CTA's `full` barrier, for which the
//            leader's producer declares the pair's bytes;
//   warp 1   TMEM allocation for the pair; in the leader, the MMA thread.
//            Its commits arrive on the `empty` and `acc_full` barriers of
//            both CTAs (multicast commit);
//   warp 2   in the peer CTA, the relay: once its eight epilogue warps have
//            drained an accumulator (local `acc_empty`), one arrival on the
//            leader's `acc_peer` (a remote arrival costs a warp about a
//            microsecond, so the epilogue warps arrive locally);
//   warps 4-11 epilogue: each CTA drains its own 128 accumulator rows. A
//            warp reads the next 32 TMEM columns while it turns the current
//            32 rows x 32 tokens into bf16 in one of its two 2 KB tiles of
//            shared memory, and writes each tile with one TMA tile store
//            (clipped at the tensor's edges; plain 2-byte stores where the
//            output rows are not 16-byte aligned). Stores from registers
//            competed with the MMAs and cost a quarter of the kernel's time;
//            the tile stores cost a few percent. Then the warp arrives on
//            its CTA's `acc_empty`. The leader's MMA thread reuses an
//            accumulator once both `acc_empty` (its own CTA) and `acc_peer`
//            have completed.
// All waits are bounded; a wait that gives up records SBN_ERR_TIMEOUT and
// the CTA winds down to the closing cluster barrier.
#pragma once

#include <cuda.h>

#include "async.cuh"
#include "bl_tc.cuh"
#include "bl_tc_sp.cuh"
#include "common.cuh"

namespace sbn {

constexpr int kT2Threads = 384;         // warps 0-11
constexpr int kT2Epi = 256;             // warps 4-11
constexpr uint32_t kT2TmemCols = 512;

template <bool SPARSE, bool NARROW = false>
struct T2Cfg {
  static_assert(!(SPARSE && NARROW), "the narrow tile is a dense-MMA configuration");
  static constexpr int BN = SPARSE ? 224 : NARROW ? 128 : 256;   // tokens per pair tile (MMA N)
  static constexpr int HALF = BN / 2;                    // activation rows per CTA
  static constexpr int ABYTES = SPARSE ? 128 * 128 : 2 * 128 * 128;
  static constexpr int BSUB = HALF * 128;                // activations of one 128-position block
  static constexpr int BBYTES = 2 * BSUB;
  static constexpr int ESUB = 128 * 16;                  // metadata of one 128-position block
  static constexpr int EBYTES = SPARSE ? 2 * ESUB : 0;
  static constexpr int STAGE = ABYTES + BBYTES + EBYTES;
  static constexpr int STAGES = (SPARSE || NARROW) ? 4 : 3;
  static constexpr int YBUF = (kT2Epi / 32) * 4096;      // two 32 x 32 bf16 tiles per epilogue warp
  static constexpr int MMAS = SPARSE ? 2 : 4;            // MMAs per 128-position block
  static constexpr uint32_t ECOL = 2 * BN;               // metadata ring after the accumulators
  // instruction descriptor: (sparse), s32 accumulate, signed 8-bit A and B,
  // K-major, N = BN, M = 256
  static constexpr uint32_t IDESC = (SPARSE ? (1u << 2) : 0u) | (2u << 4) | (1u << 7) | (1u << 10) |
                                    ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(256 >> 4) << 24);
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE + YBUF + (2 * STAGES + 6) * 8 + 16;
  static_assert(STAGE % 1024 == 0, "stages must stay 1024-byte aligned");
  static_assert(!SPARSE || ECOL + 8 * STAGES <= kT2TmemCols, "metadata ring must fit in TMEM");
  static_assert(SPARSE || 2 * BN <= (int)kT2TmemCols, "accumulators must fit in TMEM");
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

SBN_DEVFN void tma_prefetch_map(const CUtensorMap* tmap) {
  asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}
SBN_DEVFN uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared-memory offset in CTA `rank`
SBN_DEVFN uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
SBN_DEVFN void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
SBN_DEVFN void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];\n" ::"r"(cluster_addr) : "memory");
}
// TMA tile load into this CTA's shared memory whose completion counts on an
// mbarrier of either CTA of the pair (cluster address)
SBN_DEVFN void tma_load_2d_pair(void* smem_dst, const CUtensorMap* tmap, int x, int y, uint32_t mbar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(mbar_cluster)
      : "memory");
}
// TMA tile store from this CTA's shared memory (elements outside the tensor
// are not written), and the waits on this thread's outstanding stores
SBN_DEVFN void tma_store_2d(const CUtensorMap* tmap, int x, int y, const void* smem_src) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];\n" ::"l"(
                   reinterpret_cast<uint64_t>(tmap)),
               "r"(x), "r"(y), "r"(smem_u32(smem_src))
               : "memory");
  asm volatile("cp.async.bulk.commit_group;\n" ::: "memory");
}
// at most one store group still reading its shared-memory source
SBN_DEVFN void tma_store_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;\n" ::: "memory"); }
SBN_DEVFN void tma_store_wait_all() { asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory"); }
// arrives once on the barrier at this offset in both CTAs when every prior
// tcgen05 operation of this thread has completed
SBN_DEVFN void tc_commit_pair(uint64_t* bar) {
  asm volatile(
      "{\n.reg .b16 msk;\nmov.b16 msk, 3;\n"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], msk;\n}\n" ::"r"(
          smem_u32(bar))
      : "memory");
}
// tcgen05.ld of 32 columns without the wait, and the wait that makes the
// registers valid (they are in/out operands of the wait, so no use of them
// can be scheduled before it)
SBN_DEVFN void tmem_ld32_issue(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
SBN_DEVFN void tmem_ld_wait(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;\n"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                 "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                 "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

template <bool SPARSE, uint32_t IDESC>
SBN_DEVFN void tc_mma_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t tmem_e, uint32_t accumulate) {
  if constexpr (SPARSE) {
    asm volatile(
        "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.sp.cta_group::2.kind::i8 [%0], %1, %2, [%6], %3, {%5, %5, %5, %5, %5, %5, %5, %5}, p;\n}\n" ::"r"(
            tmem_d),
        "l"(adesc), "l"(bdesc), "r"(IDESC), "r"(accumulate), "r"(0u), "r"(tmem_e)
        : "memory");
  } else {
    asm volatile(
        "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, {%5, %5, %5, %5, %5, %5, %5, %5}, p;\n}\n" ::"r"(
            tmem_d),
        "l"(adesc), "l"(bdesc), "r"(IDESC), "r"(accumulate), "r"(0u)
        : "memory");
  }
}
// Both metadata blocks of a stage in one copy: 128 rows x 32 bytes, the two
// 16-byte halves (block 0 and block 1, 2 KB apart) landing in columns 0-3
// and 4-7 of the ring slot. No swizzle: core matrices of 8 rows x 16 bytes,
// the next one along a row 2 KB further (leading offset), the next 8 rows
// 128 bytes further (stride offset).
SBN_DEVFN uint64_t meta_stage_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)(2048 >> 4) << 16;
  d |= (uint64_t)(128 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  return d;
}
SBN_DEVFN void tc_cp_meta_stage_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.128x256b [%0], %1;\n" ::"r"(taddr), "l"(sdesc) : "memory");
}
SBN_DEVFN void tc_cp_meta_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.128x128b [%0], %1;\n" ::"r"(taddr), "l"(sdesc) : "memory");
}

// tmap_w: kept values (SPARSE; boxes of 128 rows x 128 bytes) or dense int8
// weights (boxes of 128 rows x 128 bytes); tmap_e: metadata (SPARSE only),
// boxes of 128 rows x 16 bytes; tmap_x: activations, boxes of HALF rows x
// 128 bytes; tmap_y: the bf16 output, boxes of 32 tokens x 32 rows, used when
// y_tma != 0 (every output row starts on a 16-byte boundary). Launched in
// clusters of two CTAs; gridDim.x even.
template <bool SPARSE, bool ACC, bool NARROW>
__global__ void __launch_bounds__(kT2Threads, 1)
bl_tc2_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
              const __grid_constant__ CUtensorMap tmap_e, const __grid_constant__ CUtensorMap tmap_y,
              const TcParams p, const int y_tma) {
  using C = T2Cfg<SPARSE, NARROW>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ybuf = smem + (size_t)C::STAGES * C::STAGE;
  uint64_t* full = reinterpret_cast<uint64_t*>(ybuf + C::YBUF);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2] this CTA's epilogue warps
  uint64_t* acc_peer = acc_empty + 2;       // [2] leader only: the peer's epilogue is done
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(acc_peer + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);
  const int nkb = p.K / 128;                // 128-position blocks
  const int nst = (nkb + 1) / 2;            // 256-position stages
  const int row_pairs = (p.N + 255) / 256;
  const int n_tiles = row_pairs * ((p.T + C::BN - 1) / C::BN);

  if (tid == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kT2Epi / 32);
      mbar_init(&acc_peer[b], 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    // the tensor maps are kernel parameters: fetching them now takes their
    // first use off the first TMA's path
    tma_prefetch_map(&tmap_x);
    tma_prefetch_map(&tmap_w);
    if (SPARSE) tma_prefetch_map(&tmap_e);
    if (y_tma) tma_prefetch_map(&tmap_y);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(s_tmem)),
                 "r"(kT2TmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // the leader's barriers are initialized before any remote arrival
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  // the set-up above overlaps the previous grid on the stream; every role
  // below reads or writes global memory
  griddep_wait();
  if (pair >= n_tiles) griddep_launch_dependents();

  if (warp == 0) {
    // ---- TMA producer (both CTAs): every box of a stage is loaded, the
    // second block of a half stage as zeros, so each stage is STAGE bytes ----
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = pair; tile < n_tiles && ok; tile += npairs) {
        const int tok0 = (tile / row_pairs) * C::BN + (int)rank * C::HALF;
        const int row0 = (tile % row_pairs) * 256 + (int)rank * 128;
        for (int ks = 0; ks < nst; ++ks, ++it) {
          const int s = it % C::STAGES;
          const uint32_t ph = (it / C::STAGES) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(&full[s], 2u * (uint32_t)C::STAGE);
          const uint32_t fb = map_to_rank(smem_u32(&full[s]), 0);
          uint8_t* st = smem + (size_t)s * C::STAGE;
          if (SPARSE) {
            tma_load_2d_pair(st, &tmap_w, ks * 128, row0, fb);
          } else {
            tma_load_2d_pair(st, &tmap_w, ks * 256, row0, fb);
            tma_load_2d_pair(st + 128 * 128, &tmap_w, ks * 256 + 128, row0, fb);
          }
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            tma_load_2d_pair(st + C::ABYTES + j * C::BSUB, &tmap_x, ks * 256 + j * 128, tok0, fb);
            if (SPARSE) tma_load_2d_pair(st + C::ABYTES + C::BBYTES + j * C::ESUB, &tmap_e, ks * 32 + j * 16, row0, fb);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer (leader CTA) ----
    // The tensor core takes few MMAs ahead, so the thread spends most of a
    // stage blocked on issue, and what it does between two stages leaves the
    // pipe idle: there it only commits, probes the next `full` barrier (the
    // bounded wait runs only if the data is late) and picks the stage's
    // precomputed descriptors.
    if (leader && lane == 0) {
      // descriptors of stage 0; stage s adds s * STAGE bytes to the start
      // address field (16-byte units)
      const uint32_t a0 = smem_u32(smem);
      const uint64_t adesc0 = sw128_kmajor_desc(a0);
      const uint64_t bdesc0 = sw128_kmajor_desc(a0 + C::ABYTES);
      const uint64_t edesc0 = meta_stage_desc(a0 + C::ABYTES + C::BBYTES);
      static_assert(!SPARSE || C::ESUB == 2048, "the stage copy takes the two metadata blocks 2 KB apart");
      int it = 0, jt = 0;
      bool ok = true;
      for (int tile = pair; tile < n_tiles && ok; tile += npairs, ++jt) {
        const int b = jt & 1;
        const uint32_t pa = ((jt >> 1) & 1u) ^ 1u;
        if (!mbar_wait(&acc_empty[b], pa) || !mbar_wait(&acc_peer[b], pa)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(b * C::BN);
        int s = it % C::STAGES;
        uint32_t ph = (it / C::STAGES) & 1u;
        for (int ks = 0; ks < nst; ++ks, ++it) {
          if (!mbar_test(&full[s], ph) && !mbar_wait(&full[s], ph)) { ok = false; break; }
          const uint32_t e_tmem = tmem + C::ECOL + 8u * (uint32_t)s;
          const int nsub = (2 * ks + 1 < nkb) ? 2 : 1;
          // both blocks' metadata (a half stage's second block is zeros)
          if (SPARSE) tc_cp_meta_stage_pair(e_tmem, edesc0 + (uint64_t)(s * (C::STAGE / 16)));
          for (int j = 0; j < nsub; ++j) {
            // A: sparse, one 128-byte swizzled row of kept values per 256
            // positions (block j at +64 bytes, MMA k at +32 bytes); dense,
            // one swizzled tile per block (16 KB apart, MMA k at +32 bytes).
            // Descriptor addresses count 16-byte units.
            const uint64_t so = (uint64_t)(s * (C::STAGE / 16));
            const uint64_t adesc = adesc0 + so + (uint64_t)(SPARSE ? 4 * j : j * (128 * 128 / 16));
            const uint64_t bdesc = bdesc0 + so + (uint64_t)(j * (C::BSUB / 16));
#pragma unroll
            for (int k = 0; k < C::MMAS; ++k) {
              // B advances 64 bytes per sparse MMA (64 positions), 32 per
              // dense one; A 32 bytes either way; metadata two columns
              tc_mma_pair<SPARSE, C::IDESC>(d_tmem, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)((SPARSE ? 4 : 2) * k),
                                  e_tmem + 4u * (uint32_t)j + 2u * (uint32_t)k,
                                  (ks > 0 || j > 0 || k > 0) ? 1u : 0u);
            }
          }
          tc_commit_pair(&empty[s]);
          if (++s == C::STAGES) { s = 0; ph ^= 1u; }
        }
        tc_commit_pair(&acc_full[b]);
      }
      // the accumulators may be freed only after the last MMAs completed
      // (matters on the abort path only)
      const int my_tiles = n_tiles > pair ? (n_tiles - 1 - pair) / npairs + 1 : 0;
      for (int jj = my_tiles - 2; jj < my_tiles; ++jj)
        if (jj >= 0) mbar_wait(&acc_full[jj & 1], (jj >> 1) & 1u);
    }
  } else if (warp == 2) {
    // ---- peer CTA: one arrival on the leader's `acc_peer` per drained tile
    // (the eight epilogue warps arrive locally; one remote arrival is much
    // cheaper than eight) ----
    if (!leader && lane == 0) {
      const uint32_t ap0 = map_to_rank(smem_u32(&acc_peer[0]), 0);
      const uint32_t ap1 = map_to_rank(smem_u32(&acc_peer[1]), 0);
      int jt = 0;
      for (int tile = pair; tile < n_tiles; tile += npairs, ++jt) {
        const int b = jt & 1;
        if (!mbar_wait(&acc_empty[b], (jt >> 1) & 1u)) break;
        mbar_arrive_cluster(b ? ap1 : ap0);
      }
    }
  } else if (warp >= 4 && warp < 12) {
    // ---- epilogue: this CTA's 128 accumulator rows; two warps per TMEM
    // lane quadrant, the first taking the first half of the 32-column chunks
    constexpr int kChunks = C::BN / 32;
    const int q = warp & 3;
    const int second = (warp - 4) >> 2;
    const int c_first = second ? (kChunks + 1) / 2 : 0;
    const int c_end = second ? kChunks : (kChunks + 1) / 2;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    uint16_t* wbuf = reinterpret_cast<uint16_t*>(ybuf + (size_t)(warp - 4) * 4096);   // 2 x (32 tokens x 32 rows)
    int nstore = 0;
    constexpr int NCH = (kChunks + 1) / 2;
    const int nch = c_end - c_first;
    const float g = ACC ? 0.f : __ldg(p.gamma);
    int jt = 0;
    for (int tile = pair; tile < n_tiles; tile += npairs, ++jt) {
      const int b = jt & 1;
      const int row_w = (tile % row_pairs) * 256 + (int)rank * 128 + 32 * q;   // this warp's first row
      const int row = row_w + lane;
      const int tok0 = (tile / row_pairs) * C::BN;
      // scales of the warp's tokens (lane jj of chunk c: token tok0 + 32c + jj),
      // fetched before the accumulator is ready
      float scq[NCH];
#pragma unroll
      for (int cc = 0; cc < NCH; ++cc) {
        const int my_tok = tok0 + 32 * (c_first + cc) + lane;
        scq[cc] = (ACC || cc >= nch || my_tok >= p.T) ? 0.f : __fdiv_rn(__fmul_rn(g, __ldg(p.xs + my_tok)), 127.0f);
      }
      int got = 1;
      if (lane == 0) got = mbar_wait(&acc_full[b], (jt >> 1) & 1u) ? 1 : 0;
      got = __shfl_sync(0xffffffffu, got, 0);
      if (!got) break;
      if (tile + npairs >= n_tiles) griddep_launch_dependents();   // the last tile's MMAs are done
      tc_fence_after();
      // chunk cc + 1 is read from TMEM while chunk cc is converted and stored
      uint32_t ra[32], rb[32];
      tmem_ld32_issue(tmem + lane_base + (uint32_t)(b * C::BN + 32 * c_first), ra);
#pragma unroll
      for (int cc = 0; cc < NCH; ++cc) {
        if (cc >= nch) break;
        const int c = c_first + cc;
        uint32_t(&r)[32] = (cc & 1) ? rb : ra;
        uint32_t(&rn)[32] = (cc & 1) ? ra : rb;
        tmem_ld_wait(r);
        if (cc + 1 < nch) tmem_ld32_issue(tmem + lane_base + (uint32_t)(b * C::BN + 32 * (c + 1)), rn);
        if (!ACC && y_tma) {
          uint16_t* buf = wbuf + (nstore & 1) * 1024;
          if (lane == 0) tma_store_wait_read1();
          __syncwarp();
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            const float sc = __shfl_sync(0xffffffffu, scq[cc], jj);
            buf[jj * 32 + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn((float)(int32_t)r[jj], sc)));
          }
          asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
          __syncwarp();
          if (row_w < p.N && tok0 + 32 * c < p.T) {
            if (lane == 0) tma_store_2d(&tmap_y, row_w, tok0 + 32 * c, buf);
            ++nstore;
          }
        } else {
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            const int tok = tok0 + 32 * c + jj;
            const float sc = __shfl_sync(0xffffffffu, scq[cc], jj);
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
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
    }
    if (lane == 0) tma_store_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // no CTA leaves while its pair may still touch its memory
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(kT2TmemCols)
                 : "memory");
  }
}

}  // namespace sbn
