// Shared device helpers of libsbn (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#define SBN_DEVFN __device__ __forceinline__

namespace sbn {

// ---------------------------------------------------------------------------
// Error word: one per device, set by bounded waits that give up.
// ---------------------------------------------------------------------------
enum : unsigned { kDevErrNone = 0u, kDevErrTimeout = 1u };
// The library is one translation unit (sbn.cu includes every kernel header),
// so the word is defined here, once.
__device__ unsigned int g_dev_error;

// Nanoseconds of the GPU's global timer (for waits bounded in time).
SBN_DEVFN unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Programmatic dependent launch. A kernel launched with the programmatic
// stream-serialization attribute may start while the previous grid on the
// stream is still running: griddep_wait() blocks until that grid has
// completed and its writes are visible (a no-op for a launch without the
// attribute), so every such kernel calls it before its first access to
// global memory. griddep_launch_dependents() lets the next grid on the
// stream be scheduled once every CTA of this one has called it or exited;
// that grid's own griddep_wait() still waits for this grid to complete.
SBN_DEVFN void griddep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
SBN_DEVFN void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// Packed-format geometry. A "unit" is 16 consecutive positions along K; for
// every supported pattern a unit's kept codes fill a whole number of bytes
// (4*n/m) and its keep bits fill two bytes.
struct Pattern {
  int n, m;
};

SBN_DEVFN uint32_t bf16_mag(uint32_t h) { return h & 0x7FFFu; }
SBN_DEVFN float bf16_bits_to_float(uint32_t h) { return __uint_as_float(h << 16); }

// Rank-select of one group: bit i of the result is set iff element i is among
// the n largest magnitudes of mags[0..M) (ties keep the lower index).
template <int M>
SBN_DEVFN uint32_t group_keep_bits(const uint32_t (&mags)[M], int n) {
  uint32_t bits = 0;
#pragma unroll
  for (int i = 0; i < M; ++i) {
    int rank = 0;
#pragma unroll
    for (int j = 0; j < M; ++j) {
      if (j < i) rank += (mags[j] >= mags[i]) ? 1 : 0;
      if (j > i) rank += (mags[j] > mags[i]) ? 1 : 0;
    }
    bits |= (rank < n ? 1u : 0u) << i;
  }
  return bits;
}

}  // namespace sbn
