// gemv_ks.cuh -- the k-sliced direct-load small-batch matmul Y = X * What^T
// for 4-bit codes in groups of 128 with K = 4096 (M <= 4): "vLLM 量化与推测
// 解码" section 2 (W4A16: packed INT4 weights and their group scales are
// unpacked and scaled on chip, multiplied with 16-bit activations and
// accumulated in higher precision) and "量化" (llminference s08) section 实现
// (each group's block is dequantized inside the accumulation).
//
// The loads and fragments are those of gemv_ld.cuh (a unit is 8 rows x one
// pair of groups = 1 KB of codes; lane L = 8 r + c copies bytes 16 c ..
// 16 c + 15 of rows r and r + 4 with cp.async into its own slots of a
// per-warp ring; one LOP3 per two codes gives the exact bfloat16 pair
// 128 + u; mma.sync m16n8k16 with A row g = (tile row g / 2, group g % 2)
// and B column n = 4 h + m).  What differs is the order of the work, chosen
// to take the bookkeeping out of the inner loop:
//
//   * K = 4096 is 16 pairs of groups, and warp w of the CTA's 16 owns pair w
//     of every 8-row tile of the CTA's range.  Its B fragments and group
//     sums never change: they are loaded from X once, after the wait on the
//     previous grid, and stay in registers.
//   * A warp's successive units are the same 128 bytes of the next tile:
//     the code pointer and the row of the {s, 128 + z} table advance by
//     constant strides; rows past N can only occur in the CTA's last tile,
//     which alone takes the bounds-checked path.
//   * A unit is one chain of eight MMAs; its two groups are added by a
//     shuffle and the tile's sum is left in shared memory at once (each unit
//     is a different tile); after one barrier each output is the sum over
//     the 16 warps in warp order (deterministic).
//   * The weight-side set-up (the first DEPTH units of every warp, the
//     {s, 128 + z} table, the cleared partial sums) happens before the wait
//     on the previous grid when the weights are static, and the CTA takes
//     at most half an SM, so the next launch's CTA streams its first units
//     while this one finishes.
#pragma once

#include "common.cuh"
#include "unpack.cuh"
#include "gemv_ld.cuh"

namespace wq {
namespace ks {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kPairs = 16;          // K = 4096: one pair of groups per warp
constexpr int kK = kPairs * 256;
constexpr int kTileRows = 8;
constexpr int kMaxM = 4;

struct Params {
  const __nv_bfloat16* X;  // [M][4096]
  void* Y;                 // [M][N]
  const uint8_t* codes;    // [N][2048]
  const __half* scales;    // [N][32]
  const __half* zeros;     // [N][32] or null (symmetric)
  int M, N, tiles, y_bf16, pdl;
  uint32_t off_sz;         // [rows of the CTA][33] {scale, 128 + zero} binary32
  uint32_t off_part;       // [tiles of the CTA][16 warps][8 rows][M] binary32
  uint32_t off_ring;       // [16 warps][DEPTH][2][32 lanes][16 bytes]
};

// Two 16-byte copies, of row r and row r + 4 of a unit (8,192 bytes apart).
__device__ __forceinline__ void copy_rows(uint32_t dst, const uint8_t* src) {
  asm volatile(
      "cp.async.cg.shared.global [%0], [%1], 16;\n\t"
      "cp.async.cg.shared.global [%2], [%1+8192], 16;" ::"r"(dst),
      "l"(src), "r"(dst + 512)
      : "memory");
}

// RAGGED: N is not a multiple of 8, so the last tile holds rows past N (they
// read as zeros through the bounds-checked copies).  Without it the refill is
// the two copies alone: measured on B200, the bounds-checked branch cost ~6
// warp instructions per unit even where it was never taken (8.40 -> 8.01 us
// per layer without it).
template <bool SYM, int MT, int DEPTH, bool RAGGED = true>
__global__ void __launch_bounds__(kThreads, 2) gemv_ks_kernel(const Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int kRowBytes = kK / 2;             // 2,048
  constexpr int kGroups = kK / 128;             // 32
  constexpr int kSzStride = kGroups + 1;        // table entries per row (banks differ)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = lane >> 3, c = lane & 7;        // load view
  const int g = lane >> 2, t = lane & 3;        // fragment view
  const int tb0 = int(int64_t(blockIdx.x) * p.tiles / gridDim.x);
  const int tb1 = int(int64_t(blockIdx.x + 1) * p.tiles / gridDim.x);
  const int ntiles = tb1 - tb0;
  const int pair = warp;

  float2* sz = reinterpret_cast<float2*>(smem + p.off_sz);
  float* part = reinterpret_cast<float*>(smem + p.off_part);
  const int per_tile = kTileRows * p.M;

  // this lane's bytes of tile row r of the first tile, and the ring slot
  const uint8_t* src = p.codes + (size_t(tb0) * kTileRows + r) * kRowBytes +
                       size_t(pair) * 128 + size_t(c) * 16;
  constexpr size_t kTileStride = size_t(kTileRows) * kRowBytes;
  const uint32_t ring =
      smem_addr(smem) + p.off_ring + uint32_t(warp * DEPTH * 1024 + lane * 16);
  // tiles [0, nfull) of the CTA have every row < N; only the last may not
  const int nfull = tb1 * kTileRows > p.N ? ntiles - 1 : ntiles;
  int fetched = 0;
  auto fetch = [&](int slot) {
    const uint32_t dst = ring + uint32_t(slot) * 1024;
    static_assert(4 * kRowBytes == 8192, "row r + 4 is 8,192 bytes on");
    if (!RAGGED) {
      if (fetched < ntiles) copy_rows(dst, src);
    } else if (fetched < nfull) {
      copy_rows(dst, src);
    } else if (fetched < ntiles) {
      const int row = (tb0 + fetched) * kTileRows + r;
      ld::cp_async16(dst, row < p.N ? src : p.codes, row < p.N);
      ld::cp_async16(dst + 512, row + 4 < p.N ? src + 4 * kRowBytes : p.codes, row + 4 < p.N);
    }
    src += kTileStride;  // never dereferenced past the CTA's last tile
    ++fetched;
    ld::cp_async_commit();
  };

  const int row_lo = tb0 * kTileRows;
  const int rows = min(p.N, tb1 * kTileRows) - row_lo;
  auto weight_setup = [&]() {
#pragma unroll
    for (int j = 0; j < DEPTH; ++j) fetch(j);
    const int meta4 = rows * kGroups / 4;
    for (int i = int(threadIdx.x); i < meta4; i += kThreads) {
      const uint2 a = ld::ldg_stream64(p.scales + size_t(row_lo) * kGroups + 4 * size_t(i));
      const uint2 z = SYM ? make_uint2(0, 0)
                          : ld::ldg_stream64(p.zeros + size_t(row_lo) * kGroups + 4 * size_t(i));
      const int e = 4 * i, row = e / kGroups, gi = e - row * kGroups;
      float2* d = sz + row * kSzStride + gi;
      const uint32_t sw[2] = {a.x, a.y}, zw[2] = {z.x, z.y};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t sk = (sw[k >> 1] >> (16 * (k & 1))) & 0xFFFFu;
        const uint32_t zk = (zw[k >> 1] >> (16 * (k & 1))) & 0xFFFFu;
        const float bias =
            SYM ? 136.f : 128.f + __half2float(__ushort_as_half(static_cast<unsigned short>(zk)));
        d[k] = make_float2(__half2float(__ushort_as_half(static_cast<unsigned short>(sk))), bias);
      }
    }
  };
  if (p.pdl) weight_setup();
  grid_dependents_launch();
  grid_dependency_wait();
  if (!p.pdl) weight_setup();

  // B fragments of this warp's pair, loaded once: lane (g, t) holds token
  // bm = g % 4 of group 2 pair + g / 4 at k = 32 t .. 32 t + 31, permuted to
  // (x0, x4, x1, x5, x2, x6, x3, x7) per 8 values; and the group sums this
  // lane's outputs need
  const int bm = g & 3, bh = g >> 2;
  const bool has_x = bm < MT && bm < p.M;
  uint4 xf[4];
  float sum = 0.f;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 o = make_uint4(0, 0, 0, 0);
    if (has_x) {
      const uint4 v = *reinterpret_cast<const uint4*>(
          p.X + size_t(bm) * kK + size_t(2 * pair + bh) * 128 + 32 * t + 8 * q);
      o.x = __byte_perm(v.x, v.z, 0x5410);
      o.y = __byte_perm(v.x, v.z, 0x7632);
      o.z = __byte_perm(v.y, v.w, 0x5410);
      o.w = __byte_perm(v.y, v.w, 0x7632);
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j)
        sum += __uint_as_float(w4[j] << 16) + __uint_as_float(w4[j] & 0xFFFF0000u);
    }
    xf[q] = o;
  }
  sum += __shfl_xor_sync(0xffffffffu, sum, 1);
  sum += __shfl_xor_sync(0xffffffffu, sum, 2);
  const int hh = g & 1;                   // group half of this lane's A rows
  const bool owner = hh == (t >> 1);      // this lane's D entries are meaningful
  const int m0 = (2 * t) & 3, m1 = m0 + 1;
  const bool use0 = owner && m0 < MT && m0 < p.M;
  const bool use1 = owner && m1 < MT && m1 < p.M;
  const float sx0 = __shfl_sync(0xffffffffu, sum, 4 * (4 * hh + m0));
  const float sx1 = __shfl_sync(0xffffffffu, sum, 4 * (4 * hh + (m1 & 3)));
  const int rr0 = g >> 1;
  const int gi = 2 * pair + hh;
  // this lane's two table entries for the first tile; successive tiles are
  // 8 rows further
  // 32-bit shared addresses: this lane's two table entries for the first
  // tile (successive tiles are 8 rows further) and its partial-sum slots
  const int mrow = MT == 1 ? 1 : p.M;
  uint32_t sz_a = smem_addr(sz + rr0 * kSzStride + gi);
  uint32_t dst0 = smem_addr(part + warp * per_tile + rr0 * mrow + m0);
  uint32_t dst1 = smem_addr(part + warp * per_tile + rr0 * mrow + (m1 & 3));
  const uint32_t part_tile_bytes = uint32_t(kWarps * per_tile) * 4u;
  const uint32_t row4_bytes = uint32_t(4 * mrow) * 4u;
  // the partial sums of this warp's slots: every slot of every tile is
  // written below (rows past N included), so no clearing is needed; the
  // {s, 128 + z} table was written by all threads
  __syncthreads();

  // Every lane computes its epilogue values (a lane and its partner L ^ 6
  // are both owners or both not; only owners' sums are stored), so the loop
  // has no branch but its end; slots are compile-time constants.
  const bool st0 = hh == 0 && use0, st1 = hh == 0 && use1;
  for (int it0 = 0; it0 < ntiles; it0 += DEPTH) {
#pragma unroll
    for (int slot = 0; slot < DEPTH; ++slot) {
      if (it0 + slot >= ntiles) break;
      ld::cp_async_wait<DEPTH - 1>();
      const uint32_t a = ring + uint32_t(slot) * 1024;
      const uint4 c0 = lds128(a);
      const uint4 c1 = lds128(a + 512);
      float d[4] = {0.f, 0.f, 0.f, 0.f};
      const uint32_t w0[4] = {c0.x, c0.y, c0.z, c0.w};
      const uint32_t w1[4] = {c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t pa[4], pb[4];
        unpack_u4(w0[q], pa);
        unpack_u4(w1[q], pb);
        const uint32_t a_even[4] = {pa[0], pb[0], pa[1], pb[1]};
        const uint32_t b_even[2] = {xf[q].x, xf[q].y};
        const uint32_t a_odd[4] = {pa[2], pb[2], pa[3], pb[3]};
        const uint32_t b_odd[2] = {xf[q].z, xf[q].w};
        mma_bf16_16816(d, a_even, b_even);
        mma_bf16_16816(d, a_odd, b_odd);
      }
      // the slot's bytes are used: refill it with the unit DEPTH tiles on
      fetch(slot);
      // y = s (C - (128 + z) Sx) for tile rows rr0 and rr0 + 4, in binary32;
      // the row's two groups are then added (lanes L and L ^ 6; binary32
      // addition commutes, so both lanes hold the same sum)
      const uint2 e0b = lds64(sz_a);
      const uint2 e1b = lds64(sz_a + 4 * kSzStride * 8);
      sz_a += kTileRows * kSzStride * 8;
      const float2 e0 = make_float2(__uint_as_float(e0b.x), __uint_as_float(e0b.y));
      const float2 e1 = make_float2(__uint_as_float(e1b.x), __uint_as_float(e1b.y));
      float y0 = e0.x * fmaf(-e0.y, sx0, d[0]);
      float y2 = e1.x * fmaf(-e1.y, sx0, d[2]);
      y0 += __shfl_xor_sync(0xffffffffu, y0, 6);
      y2 += __shfl_xor_sync(0xffffffffu, y2, 6);
      if (st0) {
        sts32(dst0, y0);
        sts32(dst0 + row4_bytes, y2);
      }
      if constexpr (MT > 1) {
        float y1 = e0.x * fmaf(-e0.y, sx1, d[1]);
        float y3 = e1.x * fmaf(-e1.y, sx1, d[3]);
        y1 += __shfl_xor_sync(0xffffffffu, y1, 6);
        y3 += __shfl_xor_sync(0xffffffffu, y3, 6);
        if (st1) {
          sts32(dst1, y1);
          sts32(dst1 + row4_bytes, y3);
        }
      }
      dst0 += part_tile_bytes;
      dst1 += part_tile_bytes;
    }
  }
  ld::cp_async_wait<0>();
  __syncthreads();

  // Y[m][row] = sum over the warps in order
  const int outs = ntiles * per_tile;
  for (int i = threadIdx.x; i < outs; i += kThreads) {
    const int tl = i / per_tile, rem = i - tl * per_tile;
    const float* s = part + size_t(tl) * kWarps * per_tile + rem;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) v += s[w * per_tile];
    const int row = (tb0 + tl) * kTileRows + rem / p.M, m = rem % p.M;
    if (row < p.N) {
      if (p.y_bf16)
        static_cast<__nv_bfloat16*>(p.Y)[size_t(m) * p.N + row] = __float2bfloat16_rn(v);
      else
        static_cast<float*>(p.Y)[size_t(m) * p.N + row] = v;
    }
  }
}

}  // namespace ks
}  // namespace wq
