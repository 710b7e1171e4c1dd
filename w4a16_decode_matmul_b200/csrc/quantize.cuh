// quantize.cuh -- groupwise affine quantize and the unfused dequantize.
//
// quantize: "vLLM 量化与推测解码" section 1 (asymmetric: q = clamp(round(w/s) + z,
// 0, 2^b - 1), s = (hi - lo)/(2^b - 1) over a range widened to contain 0,
// z = clamp(round(-lo/s)), s = 1 for a degenerate range) and "量化"
// (llminference s08) section 解法 (symmetric: z = 0, s = max|w|/(2^(b-1)-1),
// codes clipped to [-2^(b-1), 2^(b-1)-1], stored offset by 2^(b-1)).
//
// Exactness: the codes are round-half-to-even of the exact quotient w/s.
// The zero point rounds -lo/s through one IEEE division per group; the
// codes avoid a division per weight.  With inv = 1/s rounded to nearest,
// t = w * inv is within 2^-15 of w/s (|w/s| <= 255 because the range
// contains w and 0), so rintf(t) can differ from the exact rounding only
// when t lies within 2^-15 of a half-integer h.  In that window (taken as
// 2^-12) the side is decided exactly: fmaf(-h, s, w) rounds w - h*s once,
// so its sign is the sign of w/s - h, and it is zero exactly on a tie,
// which goes to the even neighbour.  The scale (hi - lo)/qmax is formed in
// binary64 (the difference of two binary16 values is exact there, and the
// quotient cannot cross a binary16 value), converted with round-up to
// binary32 and then to binary16; two round-ups compose to one.
#pragma once

#include "common.cuh"

namespace wq {

// rint(w / s), ties to even, for s > 0 and |w / s| <= 255 (see the
// exactness note above); inv is 1/s rounded to nearest.
__device__ __forceinline__ float rint_quotient(float w, float s, float inv) {
  const float t = w * inv;
  float q = rintf(t);
  const float f = t - q;
  if (fabsf(fabsf(f) - 0.5f) < 0x1p-12f) {
    const float h = q + copysignf(0.5f, f);  // the half-integer next to t
    const float e = fmaf(-h, s, w);          // sign(w/s - h), zero on a tie
    q = e > 0.f ? h + 0.5f : (e < 0.f ? h - 0.5f : rintf(h));
  }
  return q;
}

// Each lane owns 32 consecutive weights of the flattened [N*K] matrix, so a
// group of G weights spans G/32 lanes and a warp covers 1024 weights.
template <int BITS, bool SYM, int G>
__global__ void __launch_bounds__(256) quantize_kernel(const __half* __restrict__ W,
                                                      int64_t total,
                                                      uint8_t* __restrict__ codes,
                                                      __half* __restrict__ scales,
                                                      __half* __restrict__ zeros) {
  static_assert(G % 32 == 0 && G <= 1024, "group must be a multiple of 32");
  constexpr int kLanesPerGroup = G / 32;
  constexpr float kQmax = SYM ? float((1 << (BITS - 1)) - 1) : float((1 << BITS) - 1);
  constexpr float kQmin = SYM ? -float(1 << (BITS - 1)) : 0.f;
  constexpr float kOffset = SYM ? float(1 << (BITS - 1)) : 0.f;
  const int lane = threadIdx.x & 31;
  const int64_t first_warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t warps = (int64_t(gridDim.x) * blockDim.x) >> 5;

  for (int64_t chunk = first_warp; chunk * 1024 < total; chunk += warps) {
    const int64_t base = chunk * 1024 + int64_t(lane) * 32;
    const bool valid = base < total;
    float w[32];
    if (valid) {
      const uint4* src = reinterpret_cast<const uint4*>(W + base);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 v = ldg_stream128(src + j);
        const uint32_t r[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&r[i]));
          w[8 * j + 2 * i] = f.x;
          w[8 * j + 2 * i + 1] = f.y;
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) w[i] = 0.f;
    }

    // Group range: [lo, hi] widened to contain 0 (asymmetric) or max|w|.
    float lo = 0.f, hi = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if (SYM) {
        hi = fmaxf(hi, fabsf(w[i]));
      } else {
        lo = fminf(lo, w[i]);
        hi = fmaxf(hi, w[i]);
      }
    }
#pragma unroll
    for (int off = 1; off < kLanesPerGroup; off <<= 1) {
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
      if (!SYM) lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
    }

    // Stored scale (binary16, rounded up) and zero point.
    __half s16 = __float2half(1.0f);
    float s = 1.0f, inv = 1.0f, z = 0.f;
    if (hi != lo) {
      const double d = __ddiv_rn(double(hi) - double(lo), double(kQmax));
      s16 = __float2half_ru(__double2float_ru(d));
      s = __half2float(s16);
      inv = __frcp_rn(s);
      if (!SYM) z = fminf(fmaxf(rintf(__fdiv_rn(-lo, s)), 0.f), kQmax);
    }

    // Codes: round(w/s) first, then add the zero point, then clamp.
    uint32_t packed[BITS];
#pragma unroll
    for (int i = 0; i < BITS; ++i) packed[i] = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float r = rint_quotient(w[i], s, inv);
      const float q = SYM ? fminf(fmaxf(r, kQmin), kQmax) + kOffset
                          : fminf(fmaxf(r + z, kQmin), kQmax);
      const uint32_t u = static_cast<uint32_t>(static_cast<int>(q));
      packed[(i * BITS) / 32] |= u << ((i * BITS) % 32);
    }

    if (valid) {
      uint4* dst = reinterpret_cast<uint4*>(codes + base * BITS / 8);
#pragma unroll
      for (int j = 0; j < BITS / 4; ++j)
        dst[j] = make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2],
                            packed[4 * j + 3]);
      if (lane % kLanesPerGroup == 0) {
        const int64_t gi = base / G;
        scales[gi] = s16;
        if (!SYM) zeros[gi] = __float2half_rn(z);  // an integer 0..255: exact
      }
    }
  }
}

// Unfused baseline: What = s (q - z) rounded to bfloat16, written to memory.
template <int BITS, bool SYM, int G>
__global__ void __launch_bounds__(256) dequantize_kernel(const uint8_t* __restrict__ codes,
                                                        const __half* __restrict__ scales,
                                                        const __half* __restrict__ zeros,
                                                        int64_t total,
                                                        __nv_bfloat16* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t first_warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t warps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  for (int64_t chunk = first_warp; chunk * 1024 < total; chunk += warps) {
    const int64_t base = chunk * 1024 + int64_t(lane) * 32;
    if (base >= total) continue;
    const int64_t gi = base / G;
    const float s = __half2float(scales[gi]);
    const float z = SYM ? float(1 << (BITS - 1)) : __half2float(zeros[gi]);
    uint32_t packed[BITS];
    const uint4* src = reinterpret_cast<const uint4*>(codes + base * BITS / 8);
#pragma unroll
    for (int j = 0; j < BITS / 4; ++j) {
      const uint4 v = ldg_stream128(src + j);
      packed[4 * j] = v.x;
      packed[4 * j + 1] = v.y;
      packed[4 * j + 2] = v.z;
      packed[4 * j + 3] = v.w;
    }
    uint32_t outw[16];
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      float v[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int k = i + e;
        const uint32_t u = (packed[(k * BITS) / 32] >> ((k * BITS) % 32)) & ((1u << BITS) - 1);
        v[e] = s * (float(u) - z);  // exact in binary32
      }
      const __nv_bfloat162 b = __floats2bfloat162_rn(v[0], v[1]);
      outw[i / 2] = *reinterpret_cast<const uint32_t*>(&b);
    }
    uint4* dst = reinterpret_cast<uint4*>(out + base);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      dst[j] = make_uint4(outw[4 * j], outw[4 * j + 1], outw[4 * j + 2], outw[4 * j + 3]);
  }
}

}  // namespace wq
