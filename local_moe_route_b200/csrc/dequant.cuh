// dequant.cuh -- int4 code -> fp16 weight conversion shared by the
// tensor-core expert GEMMs.
#pragma once

#include "common.cuh"

namespace strata {

// Packed int4 codes hold element i of a group of 8 in nibble i as a two's
// complement value q in [-8, 7].  XOR with 0x8 turns a nibble into q + 8, and
// placing q + 8 in the low mantissa bits of fp16 1024.0 gives 1032 + q
// exactly; subtracting 1032 leaves q and one fp16 multiply gives the weight
// RNE_fp16(q * s).

// 8 codes -> 4 fp16 pairs in natural K order: pair i = (element 2i, 2i+1).
__device__ __forceinline__ void dequant8(uint32_t w, uint32_t sc2, uint32_t* r) {
  const uint32_t wx = w ^ 0x88888888u;
  const uint32_t wx4 = wx >> 4;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // byte i of wx (element 2i in its low nibble) to the low half, byte i of
    // wx >> 4 (element 2i+1 in its low nibble) to the high half
    const uint32_t t = __byte_perm(wx, wx4, (uint32_t)i | ((uint32_t)(4 + i) << 8));
    const uint32_t v = (t & 0x000F000Fu) | 0x64006400u;        // 1032 + q, both halves
    uint32_t qv, o;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(qv) : "r"(v), "r"(0x3C003C00u), "r"(0xE408E408u));
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(o) : "r"(qv), "r"(sc2));
    r[i] = o;
  }
}

// 8 codes -> 4 fp16 pairs in the interleaved K order (0,4), (1,5), (2,6),
// (3,7): each pair comes out of one mask-and-or, with no byte permute.  The
// operand it is multiplied with must use the same order within each group
// of 8 (the grouped fp16 copy of x is written that way).
__device__ __forceinline__ void dequant8_interleaved(uint32_t w, uint32_t sc2, uint32_t* r) {
  const uint32_t wx = w ^ 0x88888888u;
  const uint32_t wx8 = wx >> 8;
  const uint32_t v0 = (wx & 0x000F000Fu) | 0x64006400u;   // 1024 + (q + 8):   elements 0, 4
  const uint32_t v1 = (wx & 0x00F000F0u) | 0x64006400u;   // 1024 + 16(q + 8): elements 1, 5
  const uint32_t v2 = (wx8 & 0x000F000Fu) | 0x64006400u;  // elements 2, 6
  const uint32_t v3 = (wx8 & 0x00F000F0u) | 0x64006400u;  // elements 3, 7
  uint32_t q0, q1, q2, q3;
  // 1024 + (q + 8) - 1032 = q;  (1024 + 16(q + 8)) / 16 - 72 = q  (all exact)
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(q0) : "r"(v0), "r"(0x3C003C00u), "r"(0xE408E408u));
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(q1) : "r"(v1), "r"(0x2C002C00u), "r"(0xD480D480u));
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(q2) : "r"(v2), "r"(0x3C003C00u), "r"(0xE408E408u));
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(q3) : "r"(v3), "r"(0x2C002C00u), "r"(0xD480D480u));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r[0]) : "r"(q0), "r"(sc2));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r[1]) : "r"(q1), "r"(sc2));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r[2]) : "r"(q2), "r"(sc2));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r[3]) : "r"(q3), "r"(sc2));
}

}  // namespace strata
