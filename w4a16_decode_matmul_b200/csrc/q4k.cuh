// q4k.cuh -- nested superblocks (4.5 bits per weight): quantize and a fused
// small-batch matmul.  "量化" (llminference s08), the Q4_K superblock
// figure: 256 weights in 8 sub-blocks of 32; each sub-block has a 6-bit
// scale and a 6-bit minimum, quantized against a binary16 super-scale d and
// super-minimum dmin; 4-bit codes.  The page fixes the nesting and the bit
// counts; the arithmetic is this library's reading, stated with the format
// in include/wq.h:
//   sub-block j: lo = min(0, min w), hi = max(0, max w) ("vLLM 量化与推测解码"
//   section 1's range), s_j = (hi - lo)/15, m_j = -lo;
//   d = smallest binary16 >= max s_j / 63, dmin likewise for m_j (0 when
//   the maximum is 0); sc_j = clamp(round(s_j/d), 1, 63) (1 when d = 0),
//   mq_j = clamp(round(m_j/dmin), 0, 63) (0 when dmin = 0);
//   q = clamp(round((w + M_j)/S_j), 0, 15) with S_j = d sc_j, M_j = dmin mq_j
//   (0 when S_j = 0); w^ = S_j q - M_j.
// Every rounding is half-to-even of the exact value: the operands are
// binary16 values and their products with small integers, whose binary64
// sums and quotients decide each rounding exactly (ties stay exact), so
// the quantizer works in binary64.  Block (144 bytes): d, dmin (binary16,
// little-endian), twelve bytes of sixteen 6-bit fields (sc_0..7, mq_0..7,
// least significant bit first), 128 bytes of codes (low nibble = even k).
#pragma once

#include "common.cuh"

namespace wq {
namespace q4k {

constexpr int kBlockBytes = 144;
constexpr int kBlockWeights = 256;

// One warp per superblock: lane l holds weights 8l .. 8l+7 (sub-block l/4).
__global__ void __launch_bounds__(256) quantize_kernel(const __half* __restrict__ W,
                                                      int64_t blocks,
                                                      uint8_t* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t first = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t warps = (int64_t(gridDim.x) * blockDim.x) >> 5;
  for (int64_t b = first; b < blocks; b += warps) {
    const uint4 raw = ldg_stream128(W + b * kBlockWeights + 8 * lane);
    const uint32_t rw[4] = {raw.x, raw.y, raw.z, raw.w};
    double v[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2 h = *reinterpret_cast<const __half2*>(&rw[i]);
      v[2 * i] = double(__low2float(h));
      v[2 * i + 1] = double(__high2float(h));
    }
    double lo = 0.0, hi = 0.0;  // the range contains 0
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      lo = fmin(lo, v[i]);
      hi = fmax(hi, v[i]);
    }
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) {  // the sub-block's four lanes
      lo = fmin(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmax(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    const double s = __ddiv_rn(hi - lo, 15.0), m = -lo;
    double smax = s, mmax = m;
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      smax = fmax(smax, __shfl_xor_sync(0xffffffffu, smax, o));
      mmax = fmax(mmax, __shfl_xor_sync(0xffffffffu, mmax, o));
    }
    // smallest binary16 at or above: two round-ups compose to one
    const __half d16 = smax > 0.0 ? __float2half_ru(__double2float_ru(__ddiv_rn(smax, 63.0)))
                                  : __float2half(0.f);
    const __half dm16 = mmax > 0.0 ? __float2half_ru(__double2float_ru(__ddiv_rn(mmax, 63.0)))
                                   : __float2half(0.f);
    const double d = double(__half2float(d16)), dmin = double(__half2float(dm16));
    const int sc = d > 0.0 ? int(fmin(fmax(rint(__ddiv_rn(s, d)), 1.0), 63.0)) : 1;
    const int mq = dmin > 0.0 ? int(fmin(fmax(rint(__ddiv_rn(m, dmin)), 0.0), 63.0)) : 0;
    const double S = d * double(sc), M = dmin * double(mq);
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int q = S > 0.0 ? int(fmin(fmax(rint(__ddiv_rn(v[i] + M, S)), 0.0), 15.0)) : 0;
      packed |= uint32_t(q) << (4 * i);
    }
    uint8_t* blk = out + b * kBlockBytes;
    *reinterpret_cast<uint32_t*>(blk + 16 + 4 * lane) = packed;
    // the 96 field bits: sc_j from lane 4j, mq_j likewise
    uint64_t lo64 = 0, hi64 = 0;
#pragma unroll
    for (int f = 0; f < 16; ++f) {
      const uint64_t val = uint64_t(__shfl_sync(0xffffffffu, f < 8 ? sc : mq, 4 * (f & 7)));
      const int pos = 6 * f;
      if (pos + 6 <= 64) {
        lo64 |= val << pos;
      } else if (pos >= 64) {
        hi64 |= val << (pos - 64);
      } else {
        lo64 |= val << pos;
        hi64 |= val >> (64 - pos);
      }
    }
    if (lane == 0) {
      const uint32_t dd = uint32_t(__half_as_ushort(d16)) | (uint32_t(__half_as_ushort(dm16)) << 16);
      *reinterpret_cast<uint4*>(blk) =
          make_uint4(dd, uint32_t(lo64), uint32_t(lo64 >> 32), uint32_t(hi64));
    }
  }
}

__device__ __forceinline__ int field6(uint32_t w1, uint32_t w2, uint32_t w3, int f) {
  const uint64_t lo64 = uint64_t(w1) | (uint64_t(w2) << 32);
  const int pos = 6 * f;
  uint64_t v;
  if (pos + 6 <= 64)
    v = lo64 >> pos;
  else if (pos >= 64)
    v = uint64_t(w3) >> (pos - 64);
  else
    v = (lo64 >> pos) | (uint64_t(w3) << (64 - pos));
  return int(v & 63u);
}

// Fused small-batch matmul Y = X * What^T (M <= 8): one warp per output row;
// lane l takes sub-block l % 8 of superblock 4 i + l / 8 of the row, so a
// warp step covers four superblocks (576 contiguous bytes).  Per sub-block,
// in binary32: y += d sc (sum x q) - dmin mq (sum x).  The warp's partial
// sums are added by a fixed shuffle tree: deterministic.
template <int MT>
__global__ void __launch_bounds__(256) matmul_kernel(const __nv_bfloat16* __restrict__ X, int M,
                                                    const uint8_t* __restrict__ blocks, int N,
                                                    int K, void* Y, int y_bf16) {
  const int lane = threadIdx.x & 31;
  const int nb = K / kBlockWeights;
  const int warps = int((int64_t(gridDim.x) * blockDim.x) >> 5);
  const int j = lane & 7;
  for (int row = int((int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5); row < N;
       row += warps) {
    float acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0.f;
    const uint8_t* rowp = blocks + size_t(row) * nb * kBlockBytes;
    for (int sb = lane >> 3; sb < nb; sb += 4) {
      const uint8_t* blk = rowp + size_t(sb) * kBlockBytes;
      const uint4 hdr = *reinterpret_cast<const uint4*>(blk);
      const uint4 cw = ldg_stream128(blk + 16 + 16 * j);
      const float d = __half2float(__ushort_as_half(static_cast<unsigned short>(hdr.x & 0xFFFFu)));
      const float dmin = __half2float(__ushort_as_half(static_cast<unsigned short>(hdr.x >> 16)));
      const float S = d * float(field6(hdr.y, hdr.z, hdr.w, j));
      const float Mj = dmin * float(field6(hdr.y, hdr.z, hdr.w, 8 + j));
      const uint32_t c[4] = {cw.x, cw.y, cw.z, cw.w};
      const int k0 = sb * kBlockWeights + 32 * j;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m < M) {
          const uint4* xp = reinterpret_cast<const uint4*>(X + size_t(m) * K + k0);
          float sxq = 0.f, sx = 0.f;
#pragma unroll
          for (int w = 0; w < 4; ++w) {  // 8 codes and 8 activations per word
            const uint4 xv = xp[w];
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float x = e & 1 ? __uint_as_float(xw[e >> 1] & 0xFFFF0000u)
                                    : __uint_as_float(xw[e >> 1] << 16);
              const float q = float((c[w] >> (4 * e)) & 15u);
              sxq = fmaf(x, q, sxq);
              sx += x;
            }
          }
          acc[m] += fmaf(S, sxq, -Mj * sx);
        }
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], o);
    }
    if (lane == 0) {
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m < M) {
          if (y_bf16)
            static_cast<__nv_bfloat16*>(Y)[size_t(m) * N + row] = __float2bfloat16_rn(acc[m]);
          else
            static_cast<float*>(Y)[size_t(m) * N + row] = acc[m];
        }
      }
    }
  }
}

}  // namespace q4k
}  // namespace wq
