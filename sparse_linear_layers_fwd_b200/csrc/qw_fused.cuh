// sbn_quantize_weights in one persistent kernel (cooperative launch).
//
// Absmean quantizer: "BitNet b1.58: How Ternary Weights Cut LLM Memory by
// 82% Without Losing Accuracy", section "How ternary quantization works
// during training". Magnitude mask: "Sparse-BitNet: 1.58-bit LLMs are
// Naturally Friendly to Semi-Structured Sparsity", Abstract and Figure 6.
//
// gamma depends on the whole tensor while the codes depend on gamma, so the
// kernel has two phases around a grid-wide barrier:
//   phase 1  every CTA streams its rows of W from HBM once, sums |w| in fp64
//            and computes the keep mask of every group (independent of
//            gamma), written to meta;
//   barrier  an arrival counter in the workspace; the spin is bounded and
//            gives up with SBN_ERR_TIMEOUT in the device error word;
//   gamma    every CTA reads the fp64 total S'. Its rounding error has a
//            rigorous bound (positive terms: |S' - S| <= (additions on the
//            longest path) * 2^-53 * S', plus 2^-126 per zero or subnormal
//            |w|, which the fp64 construction below maps near 2^-127). If the
//            whole interval of possible exact means rounds to one fp32 value,
//            that value is gamma = max(fl32(fl64(S) / (N_out*K)), 1e-5). Else
//            (an exact mean within ~2^-40 of an fp32 rounding midpoint, rare)
//            every CTA re-reads its rows and adds every |w| exactly into
//            integer bins, a second barrier follows, and gamma comes from the
//            exact bins (qw.cuh);
//   phase 2  every CTA derives the code threshold tau, re-reads its rows
//            (now L2-resident) with the mask and writes the kept codes.
// The launch is cooperative, so all CTAs are resident and the barriers end.
#pragma once

#include "async.cuh"
#include "common.cuh"
#include "qw.cuh"

namespace sbn {

// Workspace offsets beyond the bins and tau of qw.cuh.
constexpr size_t kQwArriveOffset = kQwTauOffset + 16;   // u32 arrival counter
constexpr size_t kQwClearBytes = kQwArriveOffset + 16;  // cleared before every launch
constexpr size_t kQwPartOffset = 2304;                  // f64 partial sum of |w| per CTA
constexpr int kQwMaxGrid = (int)((kQwWorkspaceBytes - kQwPartOffset) / 8);
constexpr unsigned long long kQwWaitNs = 1000000000ull;  // the grid barrier gives up after 1 s

SBN_DEVFN uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// High word of the fp64 value of a bf16 magnitude given as bits 16-30 of a
// 32-bit word shifted down by 3 (exponent rebias 127 -> 1023); exact for
// normal magnitudes, near 2^-127 for zero and subnormals.
constexpr uint32_t kF64Rebias = 896u << 20;

// Barrier of the 512 consumer threads of qw_fused_kernel (named barrier 1;
// the producer warp never takes part).
constexpr int kQwConsumerThreads = 512;
SBN_DEVFN void qw_cons_sync() {
  asm volatile("bar.sync 1, %0;\n" ::"n"(kQwConsumerThreads) : "memory");
}

// True on every consumer thread if v is true on any (barrier 1, with reduction).
SBN_DEVFN bool qw_cons_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n.reg .pred p, q;\nsetp.ne.u32 p, %1, 0;\nbar.red.or.pred q, 1, %2, p;\nselp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kQwConsumerThreads)
      : "memory");
  return r != 0u;
}

// Bounded grid barrier among the consumers: thread 0 of every CTA arrives and
// waits until the counter reaches target. Returns false (and records a
// timeout) on give-up.
SBN_DEVFN bool grid_barrier(uint32_t* arrive, uint32_t target, int* s_abort) {
  __threadfence();
  qw_cons_sync();
  if (threadIdx.x == 0) {
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;\n" ::"l"(arrive) : "memory");
    const unsigned long long t0 = global_ns();
    int abort = 0;
    while (ld_acquire_u32(arrive) < target) {
      if (global_ns() - t0 > kQwWaitNs) {
        atomicOr(&g_dev_error, kDevErrTimeout);
        abort = 1;
        break;
      }
      __nanosleep(64);
    }
    *s_abort = abort;
  }
  qw_cons_sync();
  const bool ok = !*s_abort;
  __threadfence();
  return ok;
}

// Keep bits of 8 positions for m = 8 with exactly two pruned (6:8): the two
// smallest of the keys (|w| << 3 | (7 - i)) are dropped -- equal magnitudes
// drop the higher index first, i.e. keep the lower index.
SBN_DEVFN uint32_t keep_6of8(const uint32_t (&h)[8]) {
  uint32_t key[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) key[i] = ((h[i] & 0x7FFFu) << 3) | (7u - i);
  uint32_t m1 = key[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) m1 = min(m1, key[i]);
  uint32_t m2 = 0xFFFFFFFFu;
#pragma unroll
  for (int i = 0; i < 8; ++i) m2 = min(m2, key[i] == m1 ? 0xFFFFFFFFu : key[i]);
  return 0xFFu ^ (1u << (7u - (m1 & 7u))) ^ (1u << (7u - (m2 & 7u)));
}

// Keep bits of 4 positions for m = 4 with two kept (2:4): the two largest keys.
SBN_DEVFN uint32_t keep_2of4(const uint32_t (&h)[4]) {
  uint32_t key[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) key[i] = ((h[i] & 0x7FFFu) << 2) | (3u - i);
  const uint32_t a = max(key[0], key[1]), b = min(key[0], key[1]);
  const uint32_t c = max(key[2], key[3]), d = min(key[2], key[3]);
  const uint32_t t1 = max(a, c);
  const uint32_t t2 = max(min(a, c), max(b, d));
  return (1u << (3u - (t1 & 3u))) | (1u << (3u - (t2 & 3u)));
}

// Keep bits of one unit of 16 positions (groups of M), from the 16 bf16s.
template <int M>
SBN_DEVFN uint32_t unit_keep_bits(const uint32_t (&h)[16], int n) {
  uint32_t keep = 0u;
  if (M == 8 && n == 6) {
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      uint32_t hh[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) hh[i] = h[8 * g + i];
      keep |= keep_6of8(hh) << (8 * g);
    }
  } else if (M == 4 && n == 2) {
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      uint32_t hh[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) hh[i] = h[4 * g + i];
      keep |= keep_2of4(hh) << (4 * g);
    }
  } else {
#pragma unroll
    for (int g = 0; g < 16 / M; ++g) {
      uint32_t mags[M];
#pragma unroll
      for (int i = 0; i < M; ++i) mags[i] = h[g * M + i] & 0x7FFFu;
      keep |= group_keep_bits<M>(mags, n) << (g * M);
    }
  }
  return keep;
}

// Packed pairs of bf16 magnitudes (sign bits clear) as raw 32-bit words.
// Their float order equals the order of their bit patterns.
SBN_DEVFN __nv_bfloat162 as_bf2(uint32_t x) {
  __nv_bfloat162 r;
  memcpy(&r, &x, 4);
  return r;
}
SBN_DEVFN uint32_t as_u32(__nv_bfloat162 x) {
  uint32_t r;
  memcpy(&r, &x, 4);
  return r;
}
SBN_DEVFN uint32_t bmin2(uint32_t a, uint32_t b) { return as_u32(__hmin2(as_bf2(a), as_bf2(b))); }
SBN_DEVFN uint32_t bmax2(uint32_t a, uint32_t b) { return as_u32(__hmax2(as_bf2(a), as_bf2(b))); }
SBN_DEVFN uint32_t ble2(uint32_t a, uint32_t b) { return __hle2_mask(as_bf2(a), as_bf2(b)); }
SBN_DEVFN uint32_t swap16(uint32_t a) { return __byte_perm(a, 0u, 0x1032u); }

SBN_DEVFN uint32_t blt2(uint32_t a, uint32_t b) { return __hlt2_mask(as_bf2(a), as_bf2(b)); }

// Bit j = element j of a group held as pairs (w0 = elements 0,1; ...), from
// per-pair compare masks (0xFFFF per true half).
SBN_DEVFN uint32_t pack_pair_masks(uint32_t m0, uint32_t m1, uint32_t m2, uint32_t m3) {
  const uint32_t P = (m0 & 0x00010001u) | ((m1 & 0x00010001u) << 2) | ((m2 & 0x00010001u) << 4) |
                     ((m3 & 0x00010001u) << 6);
  return (P | (P >> 15)) & 0xFFu;
}

// The `need` (1 or 2) highest set bits of e.
SBN_DEVFN uint32_t top_bits(uint32_t e, int need) {
  const uint32_t h1 = 0x80000000u >> __clz(e);
  return need == 1 ? h1 : h1 | (0x80000000u >> __clz(e ^ h1));
}

// Pruned positions (bit j = element j) of one group of 8 magnitudes held as
// four pairs (w0 = elements 0,1; ...): the two smallest, equal magnitudes
// pruning the higher index first. The second smallest a2 comes from a
// min/max network on the pairs; the elements with magnitude <= a2 are the
// answer unless more than two share that bound -- then the ones below a2 are
// pruned, and of those equal to a2 the highest-indexed fill up to two.
SBN_DEVFN uint32_t prune_2of8(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
  const uint32_t m01 = bmin2(w0, w1), M01 = bmax2(w0, w1);
  const uint32_t m23 = bmin2(w2, w3), M23 = bmax2(w2, w3);
  const uint32_t s1 = bmin2(m01, m23);                               // smallest per half
  const uint32_t s2 = bmin2(bmax2(m01, m23), bmin2(M01, M23));       // second per half
  const uint32_t a2 = bmin2(bmax2(s1, swap16(s1)), bmin2(s2, swap16(s2)));
  uint32_t le = pack_pair_masks(ble2(w0, a2), ble2(w1, a2), ble2(w2, a2), ble2(w3, a2));
  if (__popc(le) != 2) {
    const uint32_t lt = pack_pair_masks(blt2(w0, a2), blt2(w1, a2), blt2(w2, a2), blt2(w3, a2));
    le = lt | top_bits(le & ~lt, 2 - __popc(lt));
  }
  return le;
}

// The same for one group of 4 magnitudes held as two pairs.
SBN_DEVFN uint32_t prune_2of4(uint32_t w0, uint32_t w1) {
  const uint32_t m = bmin2(w0, w1), M = bmax2(w0, w1);
  const uint32_t a2 = bmin2(bmax2(m, swap16(m)), bmin2(M, swap16(M)));
  uint32_t le = pack_pair_masks(ble2(w0, a2), ble2(w1, a2), 0u, 0u) & 0xFu;
  if (__popc(le) != 2) {
    const uint32_t lt = pack_pair_masks(blt2(w0, a2), blt2(w1, a2), 0u, 0u) & 0xFu;
    le = lt | top_bits(le & ~lt, 2 - __popc(lt));
  }
  return le;
}

// Compare-exchange of two pairs, both lanes at once: a <- min, b <- max.
SBN_DEVFN void ce2(uint32_t& a, uint32_t& b) {
  const uint32_t lo = bmin2(a, b);
  b = bmax2(a, b);
  a = lo;
}

// Sorts the low halves of v[0..H) ascending and, independently, the high
// halves (sorting networks of 1, 5 and 19 compare-exchanges).
template <int H>
SBN_DEVFN void sort_lanes(uint32_t (&v)[H]) {
  if constexpr (H == 2) {
    ce2(v[0], v[1]);
  } else if constexpr (H == 4) {
    ce2(v[0], v[1]); ce2(v[2], v[3]); ce2(v[0], v[2]); ce2(v[1], v[3]); ce2(v[1], v[2]);
  } else if constexpr (H == 8) {
    ce2(v[0], v[1]); ce2(v[2], v[3]); ce2(v[4], v[5]); ce2(v[6], v[7]);
    ce2(v[0], v[2]); ce2(v[1], v[3]); ce2(v[4], v[6]); ce2(v[5], v[7]);
    ce2(v[1], v[2]); ce2(v[5], v[6]);
    ce2(v[0], v[4]); ce2(v[1], v[5]); ce2(v[2], v[6]); ce2(v[3], v[7]);
    ce2(v[2], v[4]); ce2(v[3], v[5]);
    ce2(v[1], v[2]); ce2(v[3], v[4]); ce2(v[5], v[6]);
  }
}

// Bit j = element j of a group of 2H elements held as H pairs, from per-pair
// compare masks (0xFFFF per true half).
template <int H>
SBN_DEVFN uint32_t pack_masks(const uint32_t (&m)[H]) {
  uint32_t P = 0u;
#pragma unroll
  for (int j = 0; j < H; ++j) P |= (m[j] & 0x00010001u) << (2 * j);
  return (P | (P >> 15)) & ((1u << (2 * H)) - 1u);
}

// Pruned positions (bit j = element j) of one group of M magnitudes held as
// M/2 pairs w[0..M/2): the P smallest, equal magnitudes pruning the higher
// index first. The even- and odd-indexed elements (low and high halves) are
// sorted separately; the P-th smallest of the group is then the least of
// max(A[i-1], B[P-1-i]) over the splits i of P between the two sorted lanes
// A and B. Elements below it are pruned, and of those equal to it the
// highest-indexed fill up to P.
template <int M, int P>
SBN_DEVFN uint32_t prune_group(const uint32_t* w) {
  constexpr int H = M / 2;
  constexpr int ilo = P > H ? P - H : 0, ihi = P < H ? P : H;
  uint32_t v[H];
#pragma unroll
  for (int j = 0; j < H; ++j) v[j] = w[j];
  sort_lanes<H>(v);
  uint32_t T = 0u;
#pragma unroll
  for (int i = ilo; i <= ihi; ++i) {
    uint32_t z;
    if (i == 0) {
      z = __byte_perm(v[P - 1], 0u, 0x3232u);            // B[P-1] in both halves
    } else if (i == P) {
      z = __byte_perm(v[P - 1], 0u, 0x1010u);            // A[P-1] in both halves
    } else {
      z = __byte_perm(v[i - 1], v[P - 1 - i], 0x7610u);  // (A[i-1], B[P-1-i])
      z = bmax2(z, swap16(z));
    }
    T = (i == ilo) ? z : bmin2(T, z);
  }
  uint32_t m[H];
#pragma unroll
  for (int j = 0; j < H; ++j) m[j] = ble2(w[j], T);
  uint32_t le = pack_masks<H>(m);
  if (__popc(le) != P) {
#pragma unroll
    for (int j = 0; j < H; ++j) m[j] = blt2(w[j], T);
    const uint32_t lt = pack_masks<H>(m);
    uint32_t e = le & ~lt;
    le = lt;
    for (int need = P - __popc(lt); need > 0; --need) {
      const uint32_t h = 0x80000000u >> __clz(e);
      le |= h;
      e ^= h;
    }
  }
  return le;
}

// Keep bits of one unit (16 magnitudes as 8 pairs): 6:8 and 2:4 through the
// specialized networks above, every other pattern through prune_group.
template <int M>
SBN_DEVFN uint32_t unit_keep_fast(const uint32_t (&mw)[8], int n) {
  if (M == 8 && n == 6) {
    const uint32_t p0 = prune_2of8(mw[0], mw[1], mw[2], mw[3]);
    const uint32_t p1 = prune_2of8(mw[4], mw[5], mw[6], mw[7]);
    return (~(p0 | (p1 << 8))) & 0xFFFFu;
  } else if (M == 4 && n == 2) {
    uint32_t keep = 0u;
#pragma unroll
    for (int g = 0; g < 4; ++g) keep |= ((~prune_2of4(mw[2 * g], mw[2 * g + 1])) & 0xFu) << (4 * g);
    return keep;
  }
  uint32_t prune = 0u;
#pragma unroll
  for (int g = 0; g < 16 / M; ++g) {
    const uint32_t* wg = mw + g * (M / 2);
    uint32_t pg = 0u;
    if (M == 4) {
      pg = n == 1 ? prune_group<4, 3>(wg) : n == 3 ? prune_group<4, 1>(wg) : 0u;
    } else if (M == 8) {
      pg = n == 2 ? prune_group<8, 6>(wg) : n == 4 ? prune_group<8, 4>(wg) : 0u;
    } else {
      pg = n == 4 ? prune_group<16, 12>(wg) : n == 8 ? prune_group<16, 8>(wg)
                  : n == 12 ? prune_group<16, 4>(wg) : 0u;
    }
    prune |= pg << (g * M);
  }
  return (~prune) & 0xFFFFu;
}

// Four bytes with values in {0, 1, 3} -> their low two bits packed into 8
// bits (byte i to bits 2i, 2i+1): one multiply collects the fields.
SBN_DEVFN uint32_t pack4_2bit(uint32_t x) { return (x * 0x01041040u) >> 24; }

// Kept codes of one unit, in order, from its 16 latent values (8 pairs), the
// threshold tau and the keep bits: per element a code byte (0 for |w| <=
// tau, else 1 or 3 by sign), then per 8 positions the kept bytes gathered
// by a byte permute (selectors from s_csel) and packed to 2 bits each.
SBN_DEVFN uint32_t unit_codes(const uint32_t (&wd)[8], uint32_t tau2, uint32_t keep,
                              const uint32_t* s_csel) {
  uint32_t B[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t wa = wd[2 * j], wb = wd[2 * j + 1];
    const uint32_t nza = __hgt2_mask(as_bf2(wa & 0x7FFF7FFFu), as_bf2(tau2));
    const uint32_t nzb = __hgt2_mask(as_bf2(wb & 0x7FFF7FFFu), as_bf2(tau2));
    const uint32_t nzB = __byte_perm(nza, nzb, 0x6420u);   // 0xFF per nonzero element
    const uint32_t sB = __byte_perm(wa, wb, 0x7531u);      // high byte (sign in bit 7)
    B[j] = nzB & (((sB >> 6) & 0x02020202u) | 0x01010101u);
  }
  uint32_t codes = 0u;
  int sh = 0;
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    const uint32_t kb = (keep >> (8 * b)) & 0xFFu;
    const uint32_t sel = s_csel[kb];
    const uint32_t r0 = __byte_perm(B[2 * b], B[2 * b + 1], sel & 0xFFFFu);
    const uint32_t r1 = __byte_perm(B[2 * b], B[2 * b + 1], sel >> 16);
    const int p = __popc(kb);
    const uint32_t v = (pack4_2bit(r0) | (pack4_2bit(r1) << 8)) & ((1u << (2 * p)) - 1u);
    codes |= v << sh;
    sh += 2 * p;
  }
  return codes;
}

// Byte-gather selectors: nibble i of entry k = position of the i-th set bit of k.
SBN_DEVFN void fill_compact_table(uint32_t* s_csel) {
  for (int k = threadIdx.x; k < 256; k += blockDim.x) {
    uint32_t s = 0u, i = 0u;
    for (uint32_t pos = 0; pos < 8; ++pos)
      if ((k >> pos) & 1) s |= pos << (4 * i++);
    s_csel[k] = s;
  }
}

// Launch shape and dynamic shared memory of qw_fused_kernel. Every CTA owns a
// contiguous range of units (16 consecutive weights of one row, 32 bytes),
// i.e. one contiguous byte range of W, and streams it through a ring of
// 32 KB stages filled by bulk copies: one stage is 1024 units, two per
// thread (units t and t + 512), whose instruction chains are independent.
constexpr int kQwThreads = kQwConsumerThreads;   // consumer threads; one producer warp more
constexpr int kQwWarps = kQwThreads / 32;
constexpr int kQwUpt = 2;             // units per thread per stage (two independent chains)
constexpr int kQwChunk = 32 * kQwThreads * kQwUpt;   // bytes per stage (32 KB)
constexpr int kQwStages = 4;          // 128 KB in flight per SM
constexpr int kQwKeepCap = 16384;     // units whose keep bits stay in shared memory
constexpr size_t kQwSmKeep = (size_t)kQwStages * kQwChunk;
constexpr size_t kQwSmCsel = kQwSmKeep + (size_t)kQwKeepCap * 2;
constexpr size_t kQwSmBins = kQwSmCsel + 256 * 4;
constexpr size_t kQwSmBars = kQwSmBins + (size_t)kQwBins * 8;
constexpr size_t kQwSmemBytes = kQwSmBars + (size_t)(2 * kQwStages + 1) * 8;

// Stream ring over one CTA's byte range of W. The producer warp copies the
// range once per pass into a ring of stages; the consumer warps take each
// stage when its `full` barrier completes (the copy's bytes) and release it
// with one arrival per warp on its `empty` barrier. Chunks are numbered
// across passes (q); chunk q uses stage q % kQwStages for the (q /
// kQwStages)-th time, so its phase parity is (q / kQwStages) & 1.
struct QwRing {
  const uint8_t* src;   // first byte of the range
  long long bytes;      // length (a multiple of 32)
  int nch;              // chunks in the range
  uint8_t* buf;         // kQwStages x kQwChunk
  uint64_t* full;       // per stage: the producer's arrival + the copied bytes
  uint64_t* empty;      // per stage: one arrival per consumer warp
};

// Producer (one thread): one pass over the range, chunk numbers q onwards.
SBN_DEVFN bool qw_produce_pass(const QwRing& r, uint32_t& q) {
  for (int c = 0; c < r.nch; ++c, ++q) {
    const int st = (int)(q % kQwStages);
    if (q >= (uint32_t)kQwStages && !mbar_wait(&r.empty[st], ((q / kQwStages) - 1u) & 1u)) return false;
    const long long off = (long long)c * kQwChunk;
    const uint32_t nb = (uint32_t)min((long long)kQwChunk, r.bytes - off);
    mbar_arrive_expect_tx(&r.full[st], nb);
    bulk_g2s(r.buf + (size_t)st * kQwChunk, r.src + off, nb, &r.full[st]);
  }
  return true;
}

// Consumer warp: one pass; f(c, stage, units_here) runs on every consumer
// thread for every chunk. Lane 0 waits, the warp follows; false if a wait
// gave up.
template <class F>
SBN_DEVFN bool qw_consume_pass(const QwRing& r, uint32_t& q, F&& f) {
  const int lane = threadIdx.x & 31;
  for (int c = 0; c < r.nch; ++c, ++q) {
    const int st = (int)(q % kQwStages);
    int got = 1;
    if (lane == 0) got = mbar_wait(&r.full[st], (q / kQwStages) & 1u) ? 1 : 0;
    if (!__shfl_sync(0xffffffffu, got, 0)) return false;
    const int units_here = (int)(min((long long)kQwChunk, r.bytes - (long long)c * kQwChunk) >> 5);
    f(c, r.buf + (size_t)st * kQwChunk, units_here);
    __syncwarp();
    if (lane == 0) mbar_arrive(&r.empty[st]);
  }
  return true;
}

// This thread's unit of a stage, read without bank conflicts: lanes 4-7 of
// every quarter-warp fetch their upper half first.
SBN_DEVFN void qw_load_unit(const uint8_t* stage, int t, uint32_t (&wd)[8]) {
  const uint4* p = reinterpret_cast<const uint4*>(stage) + 2 * t;
  const int sw = (t >> 2) & 1;
  const uint4 a = p[sw], b = p[sw ^ 1];
  const uint4 lo = sw ? b : a, hi = sw ? a : b;
  wd[0] = lo.x; wd[1] = lo.y; wd[2] = lo.z; wd[3] = lo.w;
  wd[4] = hi.x; wd[5] = hi.y; wd[6] = hi.z; wd[7] = hi.w;
}

template <int M>
__global__ void __launch_bounds__(kQwThreads + 32, 1)
qw_fused_kernel(const uint16_t* __restrict__ w, int n_out, int k, int n,
                uint8_t* __restrict__ codes, int codes_stride, uint8_t* __restrict__ meta,
                int meta_stride, float* __restrict__ gamma_out, unsigned char* __restrict__ ws) {
  extern __shared__ __align__(128) uint8_t qw_smem[];
  uint16_t* s_keep = reinterpret_cast<uint16_t*>(qw_smem + kQwSmKeep);
  uint32_t* s_csel = reinterpret_cast<uint32_t*>(qw_smem + kQwSmCsel);
  unsigned long long* sbins = reinterpret_cast<unsigned long long*>(qw_smem + kQwSmBins);
  uint64_t* full = reinterpret_cast<uint64_t*>(qw_smem + kQwSmBars);
  uint64_t* empty = full + kQwStages;
  uint64_t* decided = empty + kQwStages;     // thread 0: the pass count is known
  __shared__ double swarp_d[kQwWarps];
  __shared__ unsigned long long swarp[kQwWarps];
  __shared__ uint32_t s_tau;
  __shared__ int s_abort, s_exact;

  unsigned long long* gbins = reinterpret_cast<unsigned long long*>(ws);
  uint32_t* arrive = reinterpret_cast<uint32_t*>(ws + kQwArriveOffset);
  double* gpart = reinterpret_cast<double*>(ws + kQwPartOffset);

  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int upr = k >> 4;                       // units per row
  const long long total_units = (long long)n_out * upr;
  // CTA ranges start on 128-byte boundaries (4 units), so every bulk copy
  // reads whole 128-byte lines
  auto range_start = [&](long long b) {
    return b >= (long long)gridDim.x ? total_units : (b * total_units / gridDim.x) & ~3LL;
  };
  const long long u_begin = range_start(blockIdx.x);
  const long long u_end = range_start(blockIdx.x + 1);
  const bool has_meta = (n != M);
  const int cb = 4 * n / M;                     // code bytes per unit
  constexpr int kUnitsPerChunk = kQwThreads * kQwUpt;
  const int row_step = kUnitsPerChunk / upr, u_step = kUnitsPerChunk % upr;

  QwRing ring;
  ring.src = reinterpret_cast<const uint8_t*>(w) + u_begin * 32;
  ring.bytes = (u_end - u_begin) * 32;
  ring.nch = (int)((ring.bytes + kQwChunk - 1) / kQwChunk);
  ring.buf = qw_smem;
  ring.full = full;
  ring.empty = empty;

  if (t == 0) {
    for (int s = 0; s < kQwStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kQwWarps);
    }
    mbar_init(decided, 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  fill_compact_table(s_csel);
  __syncthreads();   // the only barrier of all 544 threads

  if (warp == kQwWarps) {
    // ---- producer warp: lane 0 streams the range for every pass ----------
    if (lane == 0) {
      uint32_t q = 0u;
      bool ok = qw_produce_pass(ring, q) && qw_produce_pass(ring, q);   // pass 1, then pass 2
      // a third pass when gamma needs the exact integer bins
      if (ok && mbar_wait(decided, 0u) && s_exact) ok = qw_produce_pass(ring, q);
      // no copy may still be in flight when the CTA exits
      for (uint32_t d = q > (uint32_t)kQwStages ? q - kQwStages : 0u; d < q; ++d)
        if (!mbar_wait(&full[d % kQwStages], (d / kQwStages) & 1u)) break;
    }
    return;
  }
  uint32_t cq = 0u;   // consumer chunk number (the same in every consumer warp)

  // (row, u) of this thread's units in chunk c (slots j: unit t + 512 j of
  // the chunk), advanced chunk by chunk
  int row0[kQwUpt], u0[kQwUpt];
#pragma unroll
  for (int j = 0; j < kQwUpt; ++j) {
    const long long g = u_begin + t + (long long)kQwThreads * j;
    row0[j] = (int)(g / upr);
    u0[j] = (int)(g - (long long)row0[j] * upr);
  }
  auto advance = [&](int& row, int& u) {
    row += row_step;
    u += u_step;
    if (u >= upr) { u -= upr; ++row; }
  };

  // ---- phase 1: fp64 sum and keep masks -------------------------------------
  // fp64 accumulators: four per unit slot (short dependency chains)
  double dacc[kQwUpt][4];
#pragma unroll
  for (int j = 0; j < kQwUpt; ++j)
#pragma unroll
    for (int a = 0; a < 4; ++a) dacc[j][a] = 0.0;
  {
    int row[kQwUpt], u[kQwUpt];
#pragma unroll
    for (int j = 0; j < kQwUpt; ++j) { row[j] = row0[j]; u[j] = u0[j]; }
    const bool ok = qw_consume_pass(ring, cq, [&](int c, const uint8_t* stage, int units_here) {
#pragma unroll
      for (int j = 0; j < kQwUpt; ++j) {
        const int ui = t + kQwThreads * j;
        if (ui < units_here) {
          uint32_t wd[8], mw[8];
          qw_load_unit(stage, ui, wd);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            mw[i] = wd[i] & 0x7FFF7FFFu;
            dacc[j][(2 * i) & 3] += __hiloint2double((int)(((mw[i] & 0xFFFFu) << 13) + kF64Rebias), 0);
            dacc[j][(2 * i + 1) & 3] += __hiloint2double((int)(((mw[i] >> 16) << 13) + kF64Rebias), 0);
          }
          if (has_meta) {
            const uint32_t keep = unit_keep_fast<M>(mw, n);
            *reinterpret_cast<uint16_t*>(meta + (size_t)row[j] * meta_stride + 2 * u[j]) = (uint16_t)keep;
            const int li = c * kUnitsPerChunk + ui;
            if (li < kQwKeepCap) s_keep[li] = (uint16_t)keep;
          }
        }
        advance(row[j], u[j]);
      }
    });
    // a warp whose wait gave up stops here; the others finish the pass (their
    // waits are bounded too), then all leave together
    if (qw_cons_any(!ok)) {
      if (t == 0) { s_exact = 0; mbar_arrive(decided); }
      return;
    }
  }
  double dsum = ((dacc[0][0] + dacc[0][1]) + (dacc[0][2] + dacc[0][3])) +
                ((dacc[1][0] + dacc[1][1]) + (dacc[1][2] + dacc[1][3]));
#pragma unroll
  for (int o = 16; o; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
  if (lane == 0) swarp_d[warp] = dsum;
  qw_cons_sync();
  if (t == 0) {
    double a = 0.0;
    for (int i = 0; i < kQwWarps; ++i) a += swarp_d[i];
    gpart[blockIdx.x] = a;
  }
  // meanwhile the producer already streams pass 2 (the same range, now
  // mostly in L2) into the stages pass 1 released
  if (!grid_barrier(arrive, gridDim.x, &s_abort)) {
    if (t == 0) { s_exact = 0; mbar_arrive(decided); }
    return;
  }

  // ---- gamma: certified from the fp64 total, else exact ---------------------
  // the CTA partials, summed in the same fixed order by every CTA (one per
  // thread, warp trees, then the warp sums in order), so all agree on S
  {
    double v = (t < (int)gridDim.x) ? __ldcg(gpart + t) : 0.0;
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) swarp_d[warp] = v;
  }
  qw_cons_sync();
  if (t == 0) {
    double S = 0.0;
    for (int i = 0; i < kQwWarps; ++i) S += swarp_d[i];
    const double nk = (double)n_out * (double)k;
    // additions on the longest path: one accumulator (4 per unit, one unit
    // per slot and chunk), the 3-level tree over the 8 accumulators, warp
    // tree, warp sums of the CTA, then the same two levels over the CTA
    // partials (counted generously)
    const long long max_units = (total_units + gridDim.x - 1) / gridDim.x + 4;  // aligned ranges
    const double per_thread = 4.0 * (double)((max_units + kQwThreads - 1) / kQwThreads);
    const double adds = per_thread + 3.0 + 2.0 * (5.0 + kQwWarps) + (double)gridDim.x;
    const double err = S * adds * 0x1p-53 * 1.01 + nk * 0x1p-126 * 1.01;
    const double lo = (S - err) / nk * (1.0 - 0x1p-50);
    const double hi = (S + err) / nk * (1.0 + 0x1p-50);
    const float glo = fmaxf(__double2float_rn(lo), 1e-5f);
    const float ghi = fmaxf(__double2float_rn(hi), 1e-5f);
    s_exact = (glo == ghi) ? 0 : 1;
    if (!s_exact) {
      s_tau = code_threshold(glo);
      if (blockIdx.x == 0) *gamma_out = glo;
    }
    mbar_arrive(decided);   // the producer learns whether a third pass follows
  }
  qw_cons_sync();
  if (s_exact) {
    // rare: exact integer bins over the same range, second barrier
    for (int i = t; i < kQwBins; i += kQwThreads) sbins[i] = 0ull;
    qw_cons_sync();
    unsigned long long acc = 0ull;
    const bool ok = qw_consume_pass(ring, cq, [&](int, const uint8_t* stage, int units_here) {
      for (int j = 0; j < kQwUpt; ++j) {
        const int ui = t + kQwThreads * j;
        if (ui < units_here) {
          uint32_t wd[8];
          qw_load_unit(stage, ui, wd);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            exact_accumulate(wd[i] & 0x7FFFu, acc, sbins);
            exact_accumulate((wd[i] >> 16) & 0x7FFFu, acc, sbins);
          }
        }
      }
    });
    if (qw_cons_any(!ok)) return;
#pragma unroll
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) swarp[warp] = acc;
    qw_cons_sync();
    if (t == 0) {
      unsigned long long a = 0ull;
      for (int i = 0; i < kQwWarps; ++i) a += swarp[i];
      // a counts units of 2^(kWinLo-134): file it under exponents kWinLo,
      // kWinLo+21 and kWinLo+42 in 21-bit pieces so every bin stays small
      const unsigned long long mask21 = (1ull << 21) - 1ull;
      const unsigned long long a0 = a & mask21, a1 = (a >> 21) & mask21, a2 = a >> 42;
      if (a0) atomicAdd(&gbins[kWinLo], a0);
      if (a1) atomicAdd(&gbins[kWinLo + 21], a1);
      if (a2) atomicAdd(&gbins[kWinLo + 42], a2);
    }
    for (int i = t; i < kQwBins; i += kQwThreads)
      if (sbins[i]) atomicAdd(&gbins[i], sbins[i]);
    if (!grid_barrier(arrive, 2u * gridDim.x, &s_abort)) return;
    if (warp == 0) {
      float g;
      uint32_t tau;
      gamma_and_tau_from_bins(gbins, (long long)n_out * k, &g, &tau);
      if (lane == 0) {
        s_tau = tau;
        if (blockIdx.x == 0) *gamma_out = g;
      }
    }
    qw_cons_sync();
  }
  const uint32_t tau = s_tau;

  // ---- phase 2: codes of the kept positions ---------------------------------
  {
    int row[kQwUpt], u[kQwUpt];
#pragma unroll
    for (int j = 0; j < kQwUpt; ++j) { row[j] = row0[j]; u[j] = u0[j]; }
    qw_consume_pass(ring, cq, [&](int c, const uint8_t* stage, int units_here) {
#pragma unroll
      for (int j = 0; j < kQwUpt; ++j) {
        const int ui = t + kQwThreads * j;
        if (ui < units_here) {
          uint32_t wd[8];
          qw_load_unit(stage, ui, wd);
          uint32_t keep = 0xFFFFu;
          if (has_meta) {
            const int li = c * kUnitsPerChunk + ui;
            keep = (li < kQwKeepCap)
                       ? (uint32_t)s_keep[li]
                       : (uint32_t) * reinterpret_cast<const uint16_t*>(meta + (size_t)row[j] * meta_stride +
                                                                         2 * u[j]);
          }
          const uint32_t packed = unit_codes(wd, tau | (tau << 16), keep, s_csel);
          uint8_t* dst = codes + (size_t)row[j] * codes_stride + (size_t)u[j] * cb;
          if (cb == 4) {
            *reinterpret_cast<uint32_t*>(dst) = packed;
          } else if (cb == 2) {
            *reinterpret_cast<uint16_t*>(dst) = (uint16_t)packed;
          } else {
            for (int bb = 0; bb < cb; ++bb) dst[bb] = (uint8_t)(packed >> (8 * bb));
          }
          if (u[j] == upr - 1) {
            // zero padding at the end of the row
            for (int i = upr * cb; i < codes_stride; ++i) codes[(size_t)row[j] * codes_stride + i] = 0u;
          }
        }
        advance(row[j], u[j]);
      }
    });
  }
}

}  // namespace sbn
