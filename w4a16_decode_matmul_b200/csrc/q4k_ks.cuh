// q4k_ks.cuh -- the small-batch matmul Y = X * What^T (M = 1) for nested
// superblock weights ("量化" (llminference s08), the Q4_K superblock figure:
// 256 weights in 8 sub-blocks of 32, each with a 6-bit scale and minimum
// under a binary16 super-scale d and super-minimum dmin; 4-bit codes) with
// K = 4096, on the tensor cores.  Per sub-block j of a row, in binary32:
// y += d sc_j (sum x q) - dmin mq_j (sum x), as the scalar kernel in q4k.cuh.
//
// Work split (the k-sliced structure of gemv_ks.cuh): K = 4096 is 16
// superblocks; warp w of a CTA's 16 owns superblock w of every 16-row tile
// of the CTA's range, so its activations stay in registers.  A unit is 16
// rows x one superblock (16 x 144 = 2,304 bytes), copied with 16-byte
// cp.async into the warp's ring (nine lanes per row, three rows per
// instruction; the rows stacked as in memory).
//
// Tensor-core mapping (mma.sync m16n8k16, bf16): A = the 16 rows' codes
// (the exact bfloat16 128 + u), B block-diagonal: the two k-steps of
// sub-block j carry that sub-block's activations in column j only, so the
// accumulator D[row][j] is the row's sum over sub-block j alone and every
// accumulator entry is used.  Lane (g, t) reads word t (codes 8t .. 8t+7)
// of sub-block j's 16 bytes of rows g and g + 8; one LOP3 per pair gives
// (128 + u_{8t+i}, 128 + u_{8t+i+4}), i = 0..3, the A registers of the
// sub-block's two k-steps.  B's k positions are permuted the same way, so
// the lane's B registers are its own eight activations of sub-block g
// (nonzero only in the two steps of sub-block g).
//
// Epilogue per unit: lane (g, t) holds D for rows g and g + 8 and
// sub-blocks 2t, 2t + 1; it decodes those rows' d, dmin and 6-bit fields from
// the 16-byte headers in the ring and forms, per row,
// S0 D0 + S1 D1 - (128 S0 + M0) Sx_{2t} - (128 S1 + M1) Sx_{2t+1}
// (S = d sc, M = dmin mq; the 128 removes the code bias); the four lanes of
// a row add theirs by two shuffles, and each tile's per-warp partial sums
// go through shared memory, added over the 16 warps in warp order at the
// end (deterministic).
#pragma once

#include "common.cuh"
#include "unpack.cuh"
#include "gemv_ld.cuh"

namespace wq {
namespace q4ks {

constexpr int kWarps = 16;                    // one superblock of the row per warp
constexpr int kThreads = kWarps * 32;
constexpr int kK = kWarps * 256;              // 4,096
constexpr int kTileRows = 16;
constexpr int kBlockBytes = 144;
constexpr int kUnitBytes = kTileRows * kBlockBytes;      // 2,304
constexpr int kRowBytes = (kK / 256) * kBlockBytes;      // 2,304 bytes of a row

struct Params {
  const __nv_bfloat16* X;  // [1][4096]
  void* Y;                 // [1][N]
  const uint8_t* blocks;   // [N][16][144]
  int N, tiles, y_bf16, pdl;
  uint32_t off_part;       // [tiles of the CTA][16 warps][16 rows] binary32
  uint32_t off_ring;       // [16 warps][DEPTH][2,304 bytes]
};

// small non-negative integer (< 2^22) -> binary32, exactly
__device__ __forceinline__ float small_u2f(uint32_t v) {
  return __uint_as_float(0x4B000000u | v) - 8388608.f;
}

// RAGGED: N is not a multiple of 16, so the last tile holds rows past N
// (their copies are zero-filled); without it every copy is unconditional.
template <int DEPTH, bool RAGGED = true>
__global__ void __launch_bounds__(kThreads, 2) gemv_q4k_kernel(const Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int tb0 = int(int64_t(blockIdx.x) * p.tiles / gridDim.x);
  const int tb1 = int(int64_t(blockIdx.x + 1) * p.tiles / gridDim.x);
  const int ntiles = tb1 - tb0;
  float* part = reinterpret_cast<float*>(smem + p.off_part);
  const uint32_t ring = smem_addr(smem) + p.off_ring + uint32_t(warp * DEPTH * kUnitBytes);

  // copy view: lanes 9r' + c (< 27) copy chunk c (16 bytes; chunk 0 is the
  // header) of rows r' + 3i, i = 0..5 (< 16): each instruction moves three
  // whole 144-byte rows, the rows stacked in the slot as in memory
  const bool copier = lane < 27;
  const int crow = lane / 9, cchunk = lane - 9 * (lane / 9);
  const uint32_t cdst = uint32_t(crow * kBlockBytes + cchunk * 16);
  const uint8_t* tbase = p.blocks + (size_t(tb0) * kTileRows + crow) * kRowBytes +
                         size_t(warp) * kBlockBytes + cchunk * 16;
  const int nfull = tb1 * kTileRows > p.N ? ntiles - 1 : ntiles;
  int fetched = 0;
  auto fetch = [&](int slot) {
    if (copier && fetched < ntiles) {
      const uint32_t dst = ring + uint32_t(slot) * kUnitBytes + cdst;
      const int row0 = (tb0 + fetched) * kTileRows + crow;
#pragma unroll
      for (int i = 0; i < 6; ++i) {
        if (crow + 3 * i < kTileRows) {
          const bool ok = !RAGGED || fetched < nfull || row0 + 3 * i < p.N;
          ld::cp_async16(dst + 3 * kBlockBytes * i, ok ? tbase + size_t(3 * i) * kRowBytes : p.blocks,
                         ok);
        }
      }
    }
    tbase += size_t(kTileRows) * kRowBytes;  // never dereferenced past the CTA's last tile
    ++fetched;
    ld::cp_async_commit();
  };
  // with static weights the first units stream before the wait on the
  // previous grid (the activations and outputs are touched only after it)
  if (p.pdl) {
#pragma unroll
    for (int j = 0; j < DEPTH; ++j) fetch(j);
  }
  grid_dependents_launch();
  grid_dependency_wait();
  if (!p.pdl) {
#pragma unroll
    for (int j = 0; j < DEPTH; ++j) fetch(j);
  }

  // B registers: this lane's activations of sub-block g, k = 256 w + 32 g +
  // 8 t .. + 7, paired (x0, x4), (x1, x5), (x2, x6), (x3, x7); and the
  // activation sums of the lane's two accumulator columns, sub-blocks 2t
  // and 2t + 1
  const uint4 xv = *reinterpret_cast<const uint4*>(p.X + 256 * warp + 32 * g + 8 * t);
  const uint32_t xb[4] = {__byte_perm(xv.x, xv.z, 0x5410), __byte_perm(xv.x, xv.z, 0x7632),
                          __byte_perm(xv.y, xv.w, 0x5410), __byte_perm(xv.y, xv.w, 0x7632)};
  float xs = 0.f;
  {
    const uint32_t w4[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      xs += __uint_as_float(w4[i] << 16) + __uint_as_float(w4[i] & 0xFFFF0000u);
  }
  xs += __shfl_xor_sync(0xffffffffu, xs, 1);
  xs += __shfl_xor_sync(0xffffffffu, xs, 2);  // lanes 4g .. 4g + 3: sum over sub-block g
  const float sx0 = __shfl_sync(0xffffffffu, xs, 8 * t);      // sub-block 2t
  const float sx1 = __shfl_sync(0xffffffffu, xs, 8 * t + 4);  // sub-block 2t + 1

  // one row's sum over the lane's two sub-blocks, from its header h and its
  // accumulators (columns 2t, 2t + 1)
  auto row_sum = [&](const uint4 h, float d0, float d1) {
    const float dsc = __half2float(__ushort_as_half(static_cast<unsigned short>(h.x & 0xFFFFu)));
    const float dmn = __half2float(__ushort_as_half(static_cast<unsigned short>(h.x >> 16)));
    // the 96 field bits (sc_0..7, mq_0..7, 6 bits each, least significant
    // first): sc_{2t}, sc_{2t+1} at bit 12t, mq_{2t}, mq_{2t+1} at bit 48 + 12t
    const uint64_t flo = (uint64_t(h.z) << 32) | h.y;
    const uint64_t fhi = (uint64_t(h.w) << 32) | h.z;
    const uint32_t sc = uint32_t(flo >> (12 * t)) & 0xFFFu;
    const uint32_t mq = uint32_t(fhi >> (16 + 12 * t)) & 0xFFFu;
    const float S0 = dsc * small_u2f(sc & 63u), S1 = dsc * small_u2f(sc >> 6);
    const float M0 = dmn * small_u2f(mq & 63u), M1 = dmn * small_u2f(mq >> 6);
    const float corr = fmaf(fmaf(128.f, S0, M0), sx0, fmaf(128.f, S1, M1) * sx1);
    return fmaf(S0, d0, fmaf(S1, d1, -corr));
  };

  const uint32_t lane_row = uint32_t(g * kBlockBytes);  // row g of a slot
  const uint32_t code_off = lane_row + 16u + 4u * uint32_t(t);
  uint32_t dst = smem_addr(part + warp * kTileRows + g);
  for (int it0 = 0; it0 < ntiles; it0 += DEPTH) {
#pragma unroll
    for (int slot = 0; slot < DEPTH; ++slot) {
      if (it0 + slot >= ntiles) break;
      ld::cp_async_wait<DEPTH - 1>();
      const uint32_t a = ring + uint32_t(slot) * kUnitBytes;
      float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
      for (int j = 0; j < 8; ++j) {
        const uint32_t w0 = lds32(a + code_off + 16u * j);
        const uint32_t w1 = lds32(a + code_off + 16u * j + 8u * kBlockBytes);
        uint32_t pa[4], pb[4];
        unpack_u4(w0, pa);
        unpack_u4(w1, pb);
        const bool mine = g == j;
        const uint32_t a_lo[4] = {pa[0], pb[0], pa[1], pb[1]};
        const uint32_t a_hi[4] = {pa[2], pb[2], pa[3], pb[3]};
        const uint32_t b_lo[2] = {mine ? xb[0] : 0u, mine ? xb[1] : 0u};
        const uint32_t b_hi[2] = {mine ? xb[2] : 0u, mine ? xb[3] : 0u};
        mma_bf16_16816(d, a_lo, b_lo);
        mma_bf16_16816(d, a_hi, b_hi);
      }
      // the headers of rows g and g + 8, then the slot is free
      const uint4 h0 = lds128(a + lane_row);
      const uint4 h1 = lds128(a + lane_row + 8u * kBlockBytes);
      fetch(slot);
      float v0 = row_sum(h0, d[0], d[1]);
      float v1 = row_sum(h1, d[2], d[3]);
      v0 += __shfl_xor_sync(0xffffffffu, v0, 1);
      v1 += __shfl_xor_sync(0xffffffffu, v1, 1);
      v0 += __shfl_xor_sync(0xffffffffu, v0, 2);
      v1 += __shfl_xor_sync(0xffffffffu, v1, 2);
      if (t == 0) {
        sts32(dst, v0);
        sts32(dst + 32, v1);
      }
      dst += kWarps * kTileRows * 4;
    }
  }
  ld::cp_async_wait<0>();
  __syncthreads();

  // Y[row] = the sum over the 16 warps in order
  const int outs = ntiles * kTileRows;
  for (int i = threadIdx.x; i < outs; i += kThreads) {
    const int tl = i / kTileRows, rr = i - tl * kTileRows;
    const float* s = part + tl * kWarps * kTileRows + rr;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) v += s[w * kTileRows];
    const int row = (tb0 + tl) * kTileRows + rr;
    if (row < p.N) {
      if (p.y_bf16)
        static_cast<__nv_bfloat16*>(p.Y)[row] = __float2bfloat16_rn(v);
      else
        static_cast<float*>(p.Y)[row] = v;
    }
  }
}

}  // namespace q4ks
}  // namespace wq
