// quantize2.cuh -- the groupwise affine quantizer of quantize.cuh with the
// same decisions, bit for bit, in fewer instructions and with the next
// chunk's weights in flight while the current one is computed.
//
// "vLLM 量化与推测解码" section 1 (asymmetric: q = clamp(round(w/s) + z, 0,
// 2^b - 1), s = (hi - lo)/(2^b - 1) over a range widened to contain 0,
// z = clamp(round(-lo/s)), s = 1 for a degenerate range) and "量化"
// (llminference s08) section 解法 (symmetric: z = 0, s = max|w|/(2^(b-1)-1),
// stored offset by 2^(b-1)).
//
// Each lane owns 32 consecutive weights (64 bytes); a group of G spans G/32
// lanes.  Per chunk of 1,024 weights a warp:
//   * takes the group's range with packed binary16 min/max (exact) and the
//     lanes' shuffles;
//   * forms the binary16 scale (binary64 quotient rounded up twice) and the
//     zero point exactly as quantize.cuh does;
//   * rounds t = w * inv, inv = 1/s rounded to nearest, with paired binary32
//     arithmetic: u = t + (C + zoff), C = 1.5 * 2^23, lands on the integer
//     grid, so the bits of u less those of C are rint(t) + zoff, the stored
//     code, whose low byte goes straight into the packed word.  |t - w/s| <=
//     qmax * 2^-23 < 2^-15 (two roundings of relative size 2^-24), so a t
//     farther than 2^-14 from every half-integer rounds as w/s does.  For
//     such a t neither clamp can bind either: asymmetric, w/s + z lies in
//     [-0.5 - 2^-16, qmax + 0.5 + 2^-16] (s >= (hi - lo)/qmax and z is
//     -lo/s rounded), so leaving [0, qmax] needs w/s + z within 2^-16 of
//     -0.5 or qmax + 0.5; symmetric, |w/s| <= qmax.  A mask records, per
//     weight, whether t is that far (e = t - rint(t) is exact, and the sign
//     of e^2 - (0.5 - 2^-14)^2 is taken in one fused rounding);
//   * recomputes, only where the mask says so (in practice where w/s is
//     exactly a half-integer, ~3e-4 of the weights of a normal layer), the
//     packed word holding the weight with the exact tie rule of quantize.cuh
//     (rint_quotient) and both clamps, from the weights in global memory.
#pragma once

#include "common.cuh"
#include "quantize.cuh"

namespace wq {

template <int BITS>
__device__ __forceinline__ uint32_t pack_codes_f(const float* q) {
  if constexpr (BITS == 4) {
    const float a = fmaf(q[3], 4096.f, fmaf(q[2], 256.f, fmaf(q[1], 16.f, q[0])));
    const float b = fmaf(q[7], 4096.f, fmaf(q[6], 256.f, fmaf(q[5], 16.f, q[4])));
    return __byte_perm(__float_as_uint(a + 8388608.f), __float_as_uint(b + 8388608.f), 0x5410);
  } else {
    const float a = fmaf(q[1], 256.f, q[0]);
    const float b = fmaf(q[3], 256.f, q[2]);
    return __byte_perm(__float_as_uint(a + 8388608.f), __float_as_uint(b + 8388608.f), 0x5410);
  }
}

// One pair of weights (a binary16 pair) through the fast path with paired
// binary32 arithmetic: t = w * inv; u = t + cz (cz = C + zoff, the code's
// integer lands in the low bits of u); r = u - cz = rint(t); e = t - r
// (exact); f = e^2 - thr2.  Returns the bits of u and of f for both weights.
__device__ __forceinline__ void quant_pair(uint32_t h2, uint64_t inv2, uint64_t cz2,
                                           uint64_t nthr2, uint32_t& u0, uint32_t& u1,
                                           uint32_t& f0, uint32_t& f1) {
  asm("{\n\t"
      ".reg .b16 a, b;\n\t"
      ".reg .f32 x, y;\n\t"
      ".reg .b64 w, t, u, r, e, f;\n\t"
      "mov.b32 {a, b}, %4;\n\t"
      "cvt.f32.f16 x, a;\n\t"
      "cvt.f32.f16 y, b;\n\t"
      "mov.b64 w, {x, y};\n\t"
      "mul.rn.f32x2 t, w, %5;\n\t"
      "add.rn.f32x2 u, t, %6;\n\t"
      "sub.rn.f32x2 r, u, %6;\n\t"
      "sub.rn.f32x2 e, t, r;\n\t"
      "fma.rn.f32x2 f, e, e, %7;\n\t"
      "mov.b64 {%0, %1}, u;\n\t"
      "mov.b64 {%2, %3}, f;\n\t"
      "}"
      : "=r"(u0), "=r"(u1), "=r"(f0), "=r"(f1)
      : "r"(h2), "l"(inv2), "l"(cz2), "l"(nthr2));
}

// The packed word of kPerWord codes at wp with the exact tie rule and both
// clamps; out of line (it runs only for flagged words), so that the main
// loop keeps its registers.
template <int BITS, bool SYM>
__device__ __noinline__ uint32_t exact_word(const __half* wp, float s, float inv, float z) {
  constexpr float kQmax = SYM ? float((1 << (BITS - 1)) - 1) : float((1 << BITS) - 1);
  constexpr float kQmin = SYM ? -float(1 << (BITS - 1)) : 0.f;
  constexpr float kOffset = SYM ? float(1 << (BITS - 1)) : 0.f;
  constexpr int kPerWord = 32 / BITS;
  float q[kPerWord];
#pragma unroll
  for (int e = 0; e < kPerWord; ++e) {
    const float r = rint_quotient(__half2float(wp[e]), s, inv);
    q[e] = SYM ? fminf(fmaxf(r, kQmin), kQmax) + kOffset : fminf(fmaxf(r + z, kQmin), kQmax);
  }
  return pack_codes_f<BITS>(q);
}

__device__ __forceinline__ uint64_t f32x2_splat(float v) {
  const uint32_t b = __float_as_uint(v);
  return (uint64_t(b) << 32) | b;
}

template <int BITS, bool SYM, int G>
__global__ void __launch_bounds__(256, 3) quantize2_kernel(const __half* __restrict__ W,
                                                          int64_t total,
                                                          uint8_t* __restrict__ codes,
                                                          __half* __restrict__ scales,
                                                          __half* __restrict__ zeros) {
  static_assert(G % 32 == 0 && G <= 1024, "group must be a multiple of 32");
  static_assert(BITS == 4 || BITS == 8, "4- or 8-bit codes");
  constexpr int kLanesPerGroup = G / 32;
  constexpr float kQmax = SYM ? float((1 << (BITS - 1)) - 1) : float((1 << BITS) - 1);
  constexpr float kQmin = SYM ? -float(1 << (BITS - 1)) : 0.f;
  constexpr float kOffset = SYM ? float(1 << (BITS - 1)) : 0.f;
  constexpr int kPerWord = 32 / BITS;  // codes per 32-bit word
  constexpr float kC = 12582912.f;     // 1.5 * 2^23
  // |t - w/s| <= qmax * 2^-23 < 2^-15; a t farther than 2^-14 from every
  // half-integer rounds as w/s does, and the clamps cannot bind on it
  constexpr float kNegThr2 = -0.24993896484375f;  // -(0.5 - 2^-14)^2, rounded
  const int lane = threadIdx.x & 31;
  const int64_t first_warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t warps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  const int64_t nchunks = (total + 1023) / 1024;

  // total is a multiple of 32: a lane's 32 weights are all in range or none
  auto load = [&](int64_t chunk, uint4 (&v)[4]) {
    const int64_t base = chunk * 1024 + int64_t(lane) * 32;
    if (chunk < nchunks && base < total) {
      const uint4* src = reinterpret_cast<const uint4*>(W + base);
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = ldg_stream128(src + j);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = make_uint4(0, 0, 0, 0);
    }
  };

  uint4 nxt[4];
  load(first_warp, nxt);
  for (int64_t chunk = first_warp; chunk < nchunks; chunk += warps) {
    uint4 cur[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) cur[j] = nxt[j];
    load(chunk + warps, nxt);  // the next chunk is in flight while this one is computed
    const int64_t base = chunk * 1024 + int64_t(lane) * 32;
    const bool valid = base < total;
    const uint32_t h[16] = {cur[0].x, cur[0].y, cur[0].z, cur[0].w, cur[1].x, cur[1].y,
                            cur[1].z, cur[1].w, cur[2].x, cur[2].y, cur[2].z, cur[2].w,
                            cur[3].x, cur[3].y, cur[3].z, cur[3].w};

    // Group range: [lo, hi] widened to contain 0 (asymmetric) or max|w|.
    float lo = 0.f, hi = 0.f;
    if (SYM) {
      __half2 m = *reinterpret_cast<const __half2*>(&h[0]);
      m = __habs2(m);
#pragma unroll
      for (int i = 1; i < 16; ++i) m = __hmax2(m, __habs2(*reinterpret_cast<const __half2*>(&h[i])));
      hi = fmaxf(__low2float(m), __high2float(m));
    } else {
      __half2 mn = *reinterpret_cast<const __half2*>(&h[0]), mx = mn;
#pragma unroll
      for (int i = 1; i < 16; ++i) {
        const __half2 v = *reinterpret_cast<const __half2*>(&h[i]);
        mn = __hmin2(mn, v);
        mx = __hmax2(mx, v);
      }
      lo = fminf(fminf(__low2float(mn), __high2float(mn)), 0.f);
      hi = fmaxf(fmaxf(__low2float(mx), __high2float(mx)), 0.f);
    }
#pragma unroll
    for (int off = 1; off < kLanesPerGroup; off <<= 1) {
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
      if (!SYM) lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
    }

    // Stored scale (binary16, rounded up) and zero point, as quantize.cuh.
    __half s16 = __float2half(1.0f);
    float s = 1.0f, inv = 1.0f, z = 0.f;
    if (hi != lo) {
      const double d = __ddiv_rn(double(hi) - double(lo), double(kQmax));
      s16 = __float2half_ru(__double2float_ru(d));
      s = __half2float(s16);
      inv = __frcp_rn(s);
      if (!SYM) z = fminf(fmaxf(rintf(__fdiv_rn(-lo, s)), 0.f), kQmax);
    }
    const float zoff = SYM ? kOffset : z;  // added to rint(w/s) in the stored code
    const uint64_t inv2 = f32x2_splat(inv), cz2 = f32x2_splat(kC + zoff);
    const uint64_t nthr2 = f32x2_splat(kNegThr2);

    // Fast path: the code is the low byte of u's bits (u - C = rint(t) +
    // zoff, an integer in [0, 2^b) unless t is near a half-integer); ok
    // collects, from bit 31 down, whether each weight is clear of the
    // half-integers (f < 0: sign bit set).
    uint32_t words[BITS];
    uint32_t ok = 0u;
#pragma unroll
    for (int wi = 0; wi < BITS; ++wi) {
      uint32_t u[kPerWord];
#pragma unroll
      for (int pp = 0; pp < kPerWord / 2; ++pp) {
        uint32_t f0, f1;
        quant_pair(h[wi * kPerWord / 2 + pp], inv2, cz2, nthr2, u[2 * pp], u[2 * pp + 1], f0, f1);
        ok = __funnelshift_l(f0, ok, 1);
        ok = __funnelshift_l(f1, ok, 1);
      }
      if constexpr (BITS == 4) {
        uint32_t b[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) b[j] = (u[2 * j + 1] << 4) + u[2 * j];
        words[wi] = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040),
                                0x5410);
      } else {
        words[wi] = __byte_perm(__byte_perm(u[0], u[1], 0x0040), __byte_perm(u[2], u[3], 0x0040),
                                0x5410);
      }
    }
    if (__any_sync(0xffffffffu, ok != 0xffffffffu)) {
      // some t within 2^-14 of a half-integer (in practice w/s exactly on
      // one): every word holding such a weight is recomputed with the exact
      // tie decision of quantize.cuh (rint_quotient), from the weights in
      // global memory
      constexpr uint32_t kWordBits = ~0u << (32 - kPerWord);
      uint32_t fl = ~ok;  // bit 31 - i: weight i flagged
      while (fl != 0u) {
        const int wi = __clz(fl) / kPerWord;
        fl &= ~(kWordBits >> (wi * kPerWord));
        const uint32_t word = exact_word<BITS, SYM>(W + base + wi * kPerWord, s, inv, z);
#pragma unroll
        for (int j = 0; j < BITS; ++j)
          if (j == wi) words[j] = word;
      }
    }
    if (valid) {
      uint4* dst = reinterpret_cast<uint4*>(codes + base * BITS / 8);
#pragma unroll
      for (int j = 0; j < BITS / 4; ++j)
        dst[j] = make_uint4(words[4 * j], words[4 * j + 1], words[4 * j + 2], words[4 * j + 3]);
      if (lane % kLanesPerGroup == 0) {
        const int64_t gi = base / G;
        scales[gi] = s16;
        if (!SYM) zeros[gi] = __float2half_rn(z);  // an integer 0..255: exact
      }
    }
  }
}

}  // namespace wq
