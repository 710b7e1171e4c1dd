// unpack.cuh -- integer codes to tensor-core operands, and the mma.sync
// steps shared by the small-batch kernels.
//
// bfloat16 operands: a 4-bit code u sits in the low mantissa bits of the
// bfloat16 128 (exponent 2^7, mantissa step 1), so one LOP3 turns two codes
// into the exact pair (128 + u_a, 128 + u_b); the 128 offset is removed in
// the binary32 epilogue with the group's activation sum.  8-bit codes go
// through the binary32 value 2^23 + u (exact) and a paired conversion to
// bfloat16 (exact for u < 256).
//
// binary16 operands: the binary16 1024 has mantissa step 1 and ten mantissa
// bits, so a code in bits 0-3 of a half reads 1024 + u and a code in bits
// 4-7 reads 1024 + 16 u (8-bit: a byte in bits 0-7 reads 1024 + u).  One
// shift by 8 brings the other nibble positions of a word down, so a word of
// eight codes costs one shift and four LOP3s; a packed subtraction (or FMA
// by 1/16) on the FMA pipe then leaves the exact small integers u - zc.
#pragma once

#include "common.cuh"

namespace wq {

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               const uint32_t (&b)[2]) {
  // not volatile: a pure function of its registers, free to be scheduled
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t mask, uint32_t bits) {
  uint32_t r;
  // (a & mask) | bits
  asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(r) : "r"(a), "r"(mask), "r"(bits));
  return r;
}

// Eight 4-bit codes of one 32-bit word -> four bfloat16 pairs (128 + u):
// r[i] = (u_i, u_{i+4}) for i = 0..3 (low half first).
__device__ __forceinline__ void unpack_u4(uint32_t w, uint32_t (&r)[4]) {
  constexpr uint32_t kMask = 0x000F000Fu, kMagic = 0x43004300u;  // bf16 128.0 pair
  r[0] = lop3_and_or(w, kMask, kMagic);
  r[1] = lop3_and_or(w >> 4, kMask, kMagic);
  r[2] = lop3_and_or(w >> 8, kMask, kMagic);
  r[3] = lop3_and_or(w >> 12, kMask, kMagic);
}

// Four 8-bit codes -> two bfloat16 pairs (u0, u1), (u2, u3), exact integers.
__device__ __forceinline__ void unpack_u8(uint32_t w, uint32_t (&r)[2]) {
  float f[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // 2^23 + u as binary32, minus 2^23: exact
    f[i] = __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7650 | i)) - 8388608.0f;
  }
  __nv_bfloat162 p0 = __floats2bfloat162_rn(f[0], f[1]);
  __nv_bfloat162 p1 = __floats2bfloat162_rn(f[2], f[3]);
  r[0] = *reinterpret_cast<uint32_t*>(&p0);
  r[1] = *reinterpret_cast<uint32_t*>(&p1);
}

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4],
                                              const uint32_t (&b)[2]) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ uint32_t hsub2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

// Eight 4-bit codes of one word -> four binary16 pairs (u_i - ZC, u_{i+4} -
// ZC), i = 0, 1, 2, 3 (low half first).  ZC is 0 (asymmetric: the zero is
// applied in the epilogue) or 8 (symmetric offset-binary codes).
template <int ZC>
__device__ __forceinline__ void unpack_u4_h(uint32_t w, uint32_t (&r)[4]) {
  static_assert(ZC == 0 || ZC == 8, "zero constant");
  constexpr uint32_t kMagic = 0x64006400u;                      // 1024, 1024
  constexpr uint32_t kLo = ZC == 0 ? 0x64006400u : 0x64086408u;  // 1024 + ZC
  constexpr uint32_t kHi = ZC == 0 ? 0xD400D400u : 0xD480D480u;  // -(64 + ZC)
  constexpr uint32_t kSixteenth = 0x2C002C00u;                   // 1/16
  const uint32_t w8 = w >> 8;
  r[0] = hsub2(lop3_and_or(w, 0x000F000Fu, kMagic), kLo);
  r[1] = hfma2(lop3_and_or(w, 0x00F000F0u, kMagic), kSixteenth, kHi);
  r[2] = hsub2(lop3_and_or(w8, 0x000F000Fu, kMagic), kLo);
  r[3] = hfma2(lop3_and_or(w8, 0x00F000F0u, kMagic), kSixteenth, kHi);
}

// Four 8-bit codes -> two binary16 pairs (u0 - ZC, u2 - ZC), (u1 - ZC, u3 -
// ZC); ZC is 0 or 128.
template <int ZC>
__device__ __forceinline__ void unpack_u8_h(uint32_t w, uint32_t (&r)[2]) {
  static_assert(ZC == 0 || ZC == 128, "zero constant");
  constexpr uint32_t kMagic = 0x64006400u;
  constexpr uint32_t kSub = ZC == 0 ? 0x64006400u : 0x64806480u;  // 1024 + ZC
  r[0] = hsub2(lop3_and_or(w, 0x00FF00FFu, kMagic), kSub);
  r[1] = hsub2(lop3_and_or(w >> 8, 0x00FF00FFu, kMagic), kSub);
}

}  // namespace wq
