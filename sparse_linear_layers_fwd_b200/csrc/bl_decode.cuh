// Decode contraction (T <= 16 tokens): packed ternary weights streamed from
// HBM once, INT8 activations resident in shared memory.
//
// "Microsoft BitNet 1.58: The Era of 1-Bit Large Language Models", section
// "bitnet.cpp: Matrix-Free Inference": 2-bit weights are moved to on-chip
// memory, unpacked there and contracted with 8-bit activations, "minimizing
// HBM traffic". Decoding is bound by the weight bytes.
//
// CTA = RT tiles of 16 output rows; the K range is processed in chunks of
// 1024 positions. Each chunk's packed codes, keep bits and activations are
// copied into a ring of shared-memory stages with cp.async (two chunks ahead).
// Within a chunk, the KS = 8 warps of a row tile take 128 positions each;
// every thread expands its own 32 positions (expand.cuh), eight per step,
// straight into the A fragment of a warp-level INT8 MMA (m16n8k32, weights
// as the 16-row operand, tokens as the 8 columns). The positions a thread
// owns are contiguous in memory; the activation fragment follows the same
// permutation of K, so no data moves between lanes. Partial sums of the KS
// warps meet in shared memory; the epilogue dequantizes
// y = acc * gamma * s_t / 127 and writes bf16.
#pragma once

#include "common.cuh"
#include "expand.cuh"

namespace sbn {

constexpr int kDecKC = 1024;   // K positions per chunk
constexpr int kDecKS = 8;      // warps along K per row tile
constexpr int kDecStages = 3;  // shared-memory ring depth
constexpr int kDecMaxRT = 4;   // row tiles per CTA at most (1024 threads)
// Row strides of the staged arrays, padded by 16 bytes so that the eight
// row groups of a warp fall into different shared-memory banks.
constexpr int kDecMRow = kDecKC / 8 + 16;
constexpr int kDecXRow = kDecKC + 16;
__host__ __device__ constexpr int dec_crow(int cb) { return kDecKC / 16 * cb + 16; }

SBN_DEVFN void cp_async16(void* smem_dst, const void* gmem_src, bool valid) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
  const int src_bytes = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(gmem_src),
               "r"(src_bytes)
               : "memory");
}
SBN_DEVFN void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
SBN_DEVFN void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

SBN_DEVFN void mma_s8_16x8x32(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

struct DecodeParams {
  const int8_t* xq;
  const float* xs;
  const uint8_t* codes;
  const uint8_t* meta;
  const float* gamma;
  uint16_t* y;
  int32_t* acc_out;
  int T, K, N;
  int cstride, mstride;
  int rt;  // row tiles per CTA
};

// Shared-memory footprint of one CTA: selector table, partial sums of the
// K-split warps, and the stage ring (codes, keep bits and activations of
// one chunk each). Independent of K.
__host__ __device__ inline size_t decode_smem_bytes(int rt, int nt, int cb, bool dense) {
  const size_t rows = 16 * (size_t)rt;
  const size_t stage = rows * (dec_crow(cb) + (dense ? 0 : kDecMRow)) + (size_t)nt * kDecXRow;
  return 1024 + (size_t)rt * kDecKS * 16 * nt * 4 + kDecStages * stage;
}

// MM: group size m; CB: code bytes per 16 positions (= 4n/m); NT: token
// columns (8 or 16); DENSE: n == m (no keep bits); ACC: write int32 acc.
template <int MM, int CB, int NT, bool DENSE, bool ACC>
__global__ void __launch_bounds__(1024)
bl_decode_kernel(const DecodeParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int kCChunk = kDecKC / 16 * CB;   // code bytes per row per chunk (global)
  constexpr int kCRow = dec_crow(CB);         // staged row strides
  constexpr int kMRow = DENSE ? 0 : kDecMRow;
  constexpr int kCPieces = kCChunk / 16, kMPieces = DENSE ? 0 : kDecKC / 128;
  constexpr int kPerRow = kCPieces + kMPieces;
  constexpr int kXPieces = kDecKC / 16;
  const int rows = 16 * p.rt;
  const size_t stage_bytes = (size_t)rows * (kCRow + kMRow) + (size_t)NT * kDecXRow;

  uint32_t* s_sel = reinterpret_cast<uint32_t*>(smem);
  int32_t* s_red = reinterpret_cast<int32_t*>(smem + 1024);
  uint8_t* s_stage0 = smem + 1024 + (size_t)p.rt * kDecKS * 16 * NT * 4;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int rt = warp / kDecKS, ks = warp % kDecKS;
  const int row0 = blockIdx.x * rows;
  const int nchunks = (p.K + kDecKC - 1) / kDecKC;

  if (!DENSE) fill_selector_table(s_sel);
  // token rows >= T stay zero in every stage
  for (int s = 0; s < kDecStages; ++s) {
    uint8_t* xz = s_stage0 + s * stage_bytes + (size_t)rows * (kCRow + kMRow) + (size_t)p.T * kDecXRow;
    for (int i = tid; i < (NT - p.T) * kDecXRow / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(xz)[i] = make_uint4(0u, 0u, 0u, 0u);
  }

  auto load_chunk = [&](int c) {
    uint8_t* st = s_stage0 + (size_t)(c % kDecStages) * stage_bytes;
    const int kc_len = min(kDecKC, p.K - c * kDecKC);
    const int cpieces = ((kc_len / 16) * CB + 15) / 16;   // partial chunk: round up
    const int mpieces = kc_len / 128;
    for (int i = tid; i < rows * kPerRow; i += blockDim.x) {
      const int r = i / kPerRow, q = i % kPerRow;
      const int grow = row0 + r;
      const bool ok = grow < p.N;
      const size_t growc = ok ? (size_t)grow : 0;
      if (q < kCPieces) {
        if (q < cpieces)
          cp_async16(st + (size_t)r * kCRow + q * 16,
                     p.codes + growc * p.cstride + (size_t)c * kCChunk + q * 16, ok);
      } else if (!DENSE) {
        const int qm = q - kCPieces;
        if (qm < mpieces)
          cp_async16(st + (size_t)rows * kCRow + (size_t)r * kMRow + qm * 16,
                     p.meta + growc * p.mstride + (size_t)c * (kDecKC / 8) + qm * 16, ok);
      }
    }
    uint8_t* sx = st + (size_t)rows * (kCRow + kMRow);
    const int xp = kc_len / 16;
    for (int i = tid; i < p.T * kXPieces; i += blockDim.x) {
      const int tok = i / kXPieces, q = i % kXPieces;
      if (q < xp)
        cp_async16(sx + (size_t)tok * kDecXRow + q * 16,
                   p.xq + (size_t)tok * p.K + (size_t)c * kDecKC + q * 16, true);
    }
  };

  int acc0[4] = {0, 0, 0, 0};
  int acc1[4] = {0, 0, 0, 0};

#pragma unroll
  for (int s = 0; s < kDecStages - 1; ++s) {
    if (s < nchunks) load_chunk(s);
    cp_async_commit();
  }
  __syncthreads();  // selector table and zeroed token rows visible

  const int rA = rt * 16 + g, rB = rA + 8;
  const int ubase = ks * 8 + 2 * t;  // first of this thread's two units in a chunk
  const int coff = ubase * CB;       // its code bytes start here (2-byte aligned)
  const int csh = (coff & 3) * 8;
  for (int c = 0; c < nchunks; ++c) {
    if (c + kDecStages - 1 < nchunks) load_chunk(c + kDecStages - 1);
    cp_async_commit();
    cp_async_wait<kDecStages - 1>();
    __syncthreads();

    const int kc_units = min(kDecKC, p.K - c * kDecKC) / 16;
    if (ks * 8 < kc_units) {  // the whole warp's 8 units are present (kc_units % 8 == 0)
      const uint8_t* st = s_stage0 + (size_t)(c % kDecStages) * stage_bytes;
      const uint8_t* sx = st + (size_t)rows * (kCRow + kMRow);
      unsigned long long cbits[2];
      uint32_t mw[2];
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const int r = rr ? rB : rA;
        const uint32_t* cw = reinterpret_cast<const uint32_t*>(st + (size_t)r * kCRow + (coff & ~3));
        const unsigned long long both = (unsigned long long)cw[0] | ((unsigned long long)cw[1] << 32);
        cbits[rr] = both >> csh;
        mw[rr] = DENSE ? 0xFFFFFFFFu
                       : *reinterpret_cast<const uint32_t*>(st + (size_t)rows * kCRow +
                                                            (size_t)r * kMRow + ubase * 2);
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
        const uint2 xa = *reinterpret_cast<const uint2*>(sx + (size_t)g * kDecXRow + pos);
        mma_s8_16x8x32(acc0, w0[0], w0[1], w1[0], w1[1], xa.x, xa.y);
        if (NT == 16) {
          const uint2 xb = *reinterpret_cast<const uint2*>(sx + (size_t)(g + 8) * kDecXRow + pos);
          mma_s8_16x8x32(acc1, w0[0], w0[1], w1[0], w1[1], xb.x, xb.y);
        }
      }
    }
    __syncthreads();  // stage (c % kDecStages) is refilled in the next iteration
  }

  // partial sums of the KS warps of each row tile: s_red[rt][ks][row][tok]
  {
    int32_t* red = s_red + ((size_t)(rt * kDecKS + ks) * 16) * NT;
    red[g * NT + 2 * t] = acc0[0];
    red[g * NT + 2 * t + 1] = acc0[1];
    red[(g + 8) * NT + 2 * t] = acc0[2];
    red[(g + 8) * NT + 2 * t + 1] = acc0[3];
    if (NT == 16) {
      red[g * NT + 8 + 2 * t] = acc1[0];
      red[g * NT + 8 + 2 * t + 1] = acc1[1];
      red[(g + 8) * NT + 8 + 2 * t] = acc1[2];
      red[(g + 8) * NT + 8 + 2 * t + 1] = acc1[3];
    }
  }
  __syncthreads();
  const float gm = ACC ? 0.f : __ldg(p.gamma);
  for (int i = tid; i < rows * p.T; i += blockDim.x) {
    const int r = i % rows, tok = i / rows;
    const int grow = row0 + r;
    if (grow >= p.N) continue;
    const int trt = r / 16, tr = r % 16;
    int a = 0;
#pragma unroll
    for (int k2 = 0; k2 < kDecKS; ++k2) a += s_red[((size_t)(trt * kDecKS + k2) * 16 + tr) * NT + tok];
    if (ACC) {
      p.acc_out[(size_t)tok * p.N + grow] = a;
    } else {
      const float sc = __fdiv_rn(__fmul_rn(gm, __ldg(p.xs + tok)), 127.0f);
      p.y[(size_t)tok * p.N + grow] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn((float)a, sc)));
    }
  }
}

}  // namespace sbn
