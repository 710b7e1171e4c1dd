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
//   * rounds t = w * inv, inv = 1/s rounded to nearest (|t - w/s| < 2^-15,
//     see quantize.cuh), by adding C + z with C = 1.5 * 2^23: the binary32
//     sum lands on the integer grid, so u - C = rint(t + z) = rint(t) + z for
//     every t that is not within 2^-12 of a half-integer.  Whether any lane
//     holds such a t is decided once per chunk (the largest |t - rint(t)|);
//     if one does, the chunk's codes are recomputed with the exact tie rule
//     of quantize.cuh (rint_quotient).  The lower clamp of the asymmetric
//     codes never binds (rint is monotone and rint(lo/s) = -z), the upper one
//     can (two half-way roundings up); symmetric codes never leave
//     [-2^(b-1)+1, 2^(b-1)-1] (|w| <= max|w| <= s (2^(b-1)-1));
//   * packs four codes at a time as the exact binary32 integer
//     q0 + 16 q1 + 256 q2 + 4096 q3 (or two 8-bit codes q0 + 256 q1), whose
//     low 16 bits are read off after adding 2^23.
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

template <int BITS>
struct CodeWords {
  uint32_t w[BITS];
};

// The exact path of a lane's 32 codes (rint_quotient's tie decision), out of
// line: it runs only for chunks where some t came within 2^-12 of a
// half-integer, and keeping it out of the main loop keeps that loop's
// registers free.
template <int BITS, bool SYM>
__device__ __noinline__ CodeWords<BITS> exact_codes(uint4 c0, uint4 c1, uint4 c2, uint4 c3,
                                                    float s, float inv, float z) {
  constexpr float kQmax = SYM ? float((1 << (BITS - 1)) - 1) : float((1 << BITS) - 1);
  constexpr float kQmin = SYM ? -float(1 << (BITS - 1)) : 0.f;
  constexpr float kOffset = SYM ? float(1 << (BITS - 1)) : 0.f;
  constexpr int kPerWord = 32 / BITS;
  const uint32_t h[16] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w,
                          c2.x, c2.y, c2.z, c2.w, c3.x, c3.y, c3.z, c3.w};
  CodeWords<BITS> out;
#pragma unroll
  for (int wi = 0; wi < BITS; ++wi) {
    float q[kPerWord];
#pragma unroll
    for (int e = 0; e < kPerWord; ++e) {
      const int i = wi * kPerWord + e;
      const __half2 pair = *reinterpret_cast<const __half2*>(&h[i >> 1]);
      const float w = (i & 1) ? __high2float(pair) : __low2float(pair);
      const float r = rint_quotient(w, s, inv);
      q[e] = SYM ? fminf(fmaxf(r, kQmin), kQmax) + kOffset : fminf(fmaxf(r + z, kQmin), kQmax);
    }
    out.w[wi] = pack_codes_f<BITS>(q);
  }
  return out;
}

template <int BITS, bool SYM, int G>
__global__ void __launch_bounds__(256, 4) quantize2_kernel(const __half* __restrict__ W,
                                                          int64_t total,
                                                          uint8_t* __restrict__ codes,
                                                          __half* __restrict__ scales,
                                                          __half* __restrict__ zeros) {
  static_assert(G % 32 == 0 && G <= 1024, "group must be a multiple of 32");
  constexpr int kLanesPerGroup = G / 32;
  constexpr float kQmax = SYM ? float((1 << (BITS - 1)) - 1) : float((1 << BITS) - 1);
  constexpr float kOffset = SYM ? float(1 << (BITS - 1)) : 0.f;
  constexpr int kPerWord = 32 / BITS;  // codes per 32-bit word
  constexpr float kC = 12582912.f;     // 1.5 * 2^23
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
    const float cz = kC + zoff;

    // Fast path: codes by the magic-number rounding; the largest distance
    // of t from its rounded value says whether any tie window was hit.
    uint32_t words[BITS];
    float far = 0.f;
#pragma unroll
    for (int wi = 0; wi < BITS; ++wi) {
      float q[kPerWord];
#pragma unroll
      for (int e = 0; e < kPerWord; ++e) {
        const int i = wi * kPerWord + e;
        const __half2 pair = *reinterpret_cast<const __half2*>(&h[i >> 1]);
        const float w = (i & 1) ? __high2float(pair) : __low2float(pair);
        const float t = w * inv;
        const float qq = (t + cz) - kC;  // rint(t) + zoff, exact integer
        far = fmaxf(far, fabsf(t - (qq - zoff)));
        q[e] = SYM ? qq : fminf(qq, kQmax);
      }
      words[wi] = pack_codes_f<BITS>(q);
    }
    if (__any_sync(0xffffffffu, far > 0.5f - 0x1p-12f)) {
      // a t within 2^-12 of a half-integer somewhere in the warp: redo this
      // lane's codes with the exact tie decision
      const CodeWords<BITS> ex = exact_codes<BITS, SYM>(cur[0], cur[1], cur[2], cur[3], s, inv, z);
#pragma unroll
      for (int wi = 0; wi < BITS; ++wi) words[wi] = ex.w[wi];
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
