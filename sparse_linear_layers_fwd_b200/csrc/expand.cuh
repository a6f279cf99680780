// Expansion of packed ternary weights (2-bit codes of the kept positions +
// keep bitmask) into int8 values, eight positions at a time.
//
// For one meta byte M (eight consecutive positions, p = popcount(M) kept) and
// the next p codes of the row's code stream:
//   1. the p codes (low 2p bits; the rest masked to zero) become eight int8
//      bytes in stream order: 00 -> 0, 01 -> +1, 11 -> -1 (the codes are
//      spread to nibbles, which then select bytes of a constant table);
//   2. a byte permute places kept value j at the position of the j-th set bit
//      of M; pruned positions take byte 7, which is zero whenever p < 8.
// The permute selectors for all 256 masks live in a shared-memory table.
#pragma once

#include "common.cuh"

namespace sbn {

// Byte table of the code values, indexed by the 2-bit code: 00 -> 0x00,
// 01 -> 0x01, 10 -> 0x00 (never written), 11 -> 0xFF.
constexpr uint32_t kCodeByteTable = 0xFF000100u;

// Eight 2-bit codes (low 16 bits of v) -> one code per nibble (32 bits).
SBN_DEVFN uint32_t codes8_to_nibbles(uint32_t v) {
  uint32_t x = __byte_perm(v, 0u, 0x4140u);   // bytes: v.b0, 0, v.b1, 0
  x = (x | (x << 4)) & 0x0F0F0F0Fu;
  x = (x | (x << 2)) & 0x33333333u;
  return x;
}

// Eight 2-bit codes -> eight int8 bytes (code i in byte i): one byte
// permute per four codes, with the nibbles as selectors into the table.
SBN_DEVFN void codes8_to_s8(uint32_t v, uint32_t& q0, uint32_t& q1) {
  const uint32_t nib = codes8_to_nibbles(v);
  q0 = __byte_perm(kCodeByteTable, 0u, nib & 0xFFFFu);
  q1 = __byte_perm(kCodeByteTable, 0u, nib >> 16);
}

// Four 2-bit codes (b, 8 bits) -> four int8 bytes (code i in byte i).
SBN_DEVFN uint32_t codes4_to_s8(uint32_t b) {
  const uint32_t nib = codes8_to_nibbles(b & 0xFFu);
  return __byte_perm(kCodeByteTable, 0u, nib & 0xFFFFu);
}

// Selector of one mask: nibble i = source byte of output byte i.
SBN_DEVFN uint32_t expand_selector(uint32_t mask8) {
  uint32_t sel = 0u, j = 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t bit = (mask8 >> i) & 1u;
    sel |= (bit ? j : 7u) << (4 * i);
    j += bit;
  }
  return sel;
}

// Fill the 256-entry selector table (call with all threads, then sync).
SBN_DEVFN void fill_selector_table(uint32_t* s_sel) {
  for (int i = threadIdx.x; i < 256; i += blockDim.x) s_sel[i] = expand_selector((uint32_t)i);
}

// Expand eight positions: mask8 = keep bits, v = the kept codes (2*p bits,
// higher bits already zero). Returns bytes 0-3 in w0 and 4-7 in w1. For
// mask8 == 0xFF the selector is the identity.
SBN_DEVFN void expand8(uint32_t mask8, uint32_t v, const uint32_t* s_sel, uint32_t& w0,
                       uint32_t& w1) {
  uint32_t q0, q1;
  codes8_to_s8(v, q0, q1);
  const uint32_t sel = s_sel[mask8];
  w0 = __byte_perm(q0, q1, sel & 0xFFFFu);
  w1 = __byte_perm(q0, q1, sel >> 16);
}

}  // namespace sbn
