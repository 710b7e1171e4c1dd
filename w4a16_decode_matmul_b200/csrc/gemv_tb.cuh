// gemv_tb.cuh -- the bulk-staged small-batch matmul Y = X * What^T for 4-bit
// codes in groups of 128 (M <= 4): "vLLM 量化与推测解码" section 2 (W4A16:
// packed INT4 weights and their group scales are unpacked and scaled on
// chip, multiplied with 16-bit activations, accumulated in higher precision)
// and "量化" (llminference s08) section 实现 (each group's block is
// dequantized inside the accumulation; full-precision weights never exist
// in memory).
//
// Decode time is bytes over bandwidth ("量化" section 问题).  Reaching the HBM
// rate needs ~100 KB of reads in flight per SM at all times, issued with
// few operations, so the weights arrive by TMA in large stages:
//
//   * A stage is one 8-row tile x one chunk of 16 pairs of groups (2,048
//     bytes of codes per row): the codes as one 3-D box (256 bytes x 8
//     blocks x 8 rows, 16 KB) and the tile's 32 scales and 32 zeros per row
//     as one 2-D box each -- three TMA operations, 17 KB, one mbarrier.  Rows
//     and chunks past the tensor's end are filled with zeros.
//   * One producer thread keeps a ring of DEPTH stages full.  With static
//     weights it starts before the wait on the previous grid, so a launch
//     streams its first DEPTH stages while the previous kernel finishes;
//     the CTA is small enough (under half an SM's registers and shared
//     memory) that the next launch's CTA can do the same on the same SM.
//   * Eight consumer warps; in each stage warp w computes pairs w and w + 8
//     of the chunk (8 rows x 256 codes each: a "unit").  Lane L = 8 r + c
//     reads bytes 16 c .. 16 c + 15 of rows r and r + 4 of the pair (whole
//     128-byte lines per quarter warp: no bank conflicts).
//   * Fragments as in gemv_ld.cuh: lane L holds A row g = 2 r + c / 4 of an
//     mma.sync m16n8k16 (tile row g / 2, group g % 2 of the pair); one LOP3
//     turns two codes into the exact bfloat16 pair 128 + u; B column
//     n = 4 h + m carries token m of group h; D[g][n] is used where
//     g % 2 == n / 4.  Per group in binary32: y += s (C - (128 + z) Sx),
//     s and z read from the stage (symmetric codes: 128 + 8).
//   * Activations: when K is one chunk (K = 4096 and below), each warp's two
//     pairs never change, and their B fragments and group sums stay in
//     registers for the whole launch, loaded straight from X after the
//     wait.  Otherwise X is staged once in shared memory, permuted so that
//     a B fragment is one 16-byte load, with its group sums.
//   * Deterministic reduction: the two lanes of a row's two groups add
//     their sums (a shuffle); a warp keeps a tile's sum over its units and
//     chunks in registers and leaves it in shared memory when the tile
//     changes; after one barrier each output is the sum over the warps in
//     warp order.
#pragma once

#include "common.cuh"
#include "unpack.cuh"

namespace wq {
namespace tb {

constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;  // + one producer warp
constexpr int kTileRows = 8;
constexpr int kGroup = 128;
constexpr int kPairBytes = 128;                        // a pair of groups, one row
constexpr int kChunkPairs = 16;                        // pairs per stage
constexpr int kRowBytes = kChunkPairs * kPairBytes;    // 2,048 bytes of codes per row
constexpr int kCodesStage = kTileRows * kRowBytes;     // 16 KB
constexpr int kMetaRow = 2 * kChunkPairs * 2;          // 32 binary16 per row: 64 bytes
constexpr int kMetaStage = kTileRows * kMetaRow;       // 512 bytes
constexpr int kStageBytes = kCodesStage + 2 * kMetaStage;  // 17,408 (a multiple of 128)
constexpr int kMaxDepth = 8;
constexpr int kMaxM = 4;
// barrier slots in the first KB of shared memory
constexpr int kBarFull = 0, kBarEmpty = kMaxDepth;
constexpr int kAbortSlot = 2 * kMaxDepth * 8;

struct Params {
  const __nv_bfloat16* X;  // [M][K]
  void* Y;                 // [M][N]
  int M, N, K, ngroups, pairs, tiles;
  int nch;                 // chunks per row: ceil(pairs / 16)
  int depth;               // stages in the ring
  int y_bf16;
  int pdl;                 // weights may be read before the previous grid completes
  uint32_t xs_row_bytes;   // staged activation row (when K is more than one chunk)
  uint32_t off_part, off_x, off_sx, off_ring;
};

template <bool SYM, int MT, bool XREG>
__global__ void __launch_bounds__(kThreads, 1)
    gemv_tb_kernel(const __grid_constant__ CUtensorMap tm_codes,
                   const __grid_constant__ CUtensorMap tm_scales,
                   const __grid_constant__ CUtensorMap tm_zeros, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kAbortSlot);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tb0 = int(int64_t(blockIdx.x) * p.tiles / gridDim.x);
  const int tb1 = int(int64_t(blockIdx.x + 1) * p.tiles / gridDim.x);
  const int nstages = (tb1 - tb0) * p.nch;
  const int D = p.depth;

  if (threadIdx.x == 0) {
    for (int i = 0; i < D; ++i) {
      mbar_init(&bars[kBarFull + i], 1);
      mbar_init(&bars[kBarEmpty + i], kConsumerWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  grid_dependents_launch();

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tm_codes);
      prefetch_tensormap(&tm_scales);
      if (!SYM) prefetch_tensormap(&tm_zeros);
      // the weights may be written by the previous kernel unless promised static
      if (!p.pdl) grid_dependency_wait();
      const uint64_t policy = l2_policy_evict_first();
      const uint32_t tx = uint32_t(kCodesStage + (SYM ? 1 : 2) * kMetaStage);
      for (int i = 0; i < nstages; ++i) {
        const int slot = i % D;
        if (i >= D && (*abort_flag || !mbar_wait_idle(&bars[kBarEmpty + slot],
                                                      uint32_t((i / D) - 1) & 1u))) {
          *abort_flag = 1;
          break;
        }
        const int tile = tb0 + i / p.nch, ch = i % p.nch;
        uint8_t* st = smem + p.off_ring + size_t(slot) * kStageBytes;
        mbar_arrive_expect_tx(&bars[kBarFull + slot], tx);
        tma_load_3d(st, &tm_codes, &bars[kBarFull + slot], 0, ch * (kRowBytes / 256),
                    tile * kTileRows, policy);
        tma_load_2d(st + kCodesStage, &tm_scales, &bars[kBarFull + slot], ch * 2 * kChunkPairs,
                    tile * kTileRows, policy);
        if (!SYM)
          tma_load_2d(st + kCodesStage + kMetaStage, &tm_zeros, &bars[kBarFull + slot],
                      ch * 2 * kChunkPairs, tile * kTileRows, policy);
      }
      // the copies of the last D stages land before the CTA can finish
      for (int i = max(0, nstages - D); i < nstages; ++i)
        mbar_wait_idle(&bars[kBarFull + i % D], uint32_t(i / D) & 1u);
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  const int r = lane >> 3, c = lane & 7;  // load view: tile row r (and r + 4), chunk c
  const int g = lane >> 2, t = lane & 3;  // fragment view
  const int bm = g & 3, bh = g >> 2;      // B column g: token bm of group half bh
  const bool has_x = bm < MT && bm < p.M;
  const int hh = g & 1;                   // group half of this lane's A rows
  const bool owner = hh == (t >> 1);      // this lane's D entries are meaningful
  const int m0 = (2 * t) & 3, m1 = m0 + 1;
  const bool use0 = owner && m0 < MT && m0 < p.M;
  const bool use1 = owner && m1 < MT && m1 < p.M;
  const int rr0 = g >> 1;                 // tile rows rr0 and rr0 + 4
  float* part = reinterpret_cast<float*>(smem + p.off_part);
  const int per_tile = kTileRows * p.M;

  // partial sums of this warp, cleared (they do not depend on the inputs)
  for (int i = lane; i < (tb1 - tb0) * per_tile; i += 32)
    part[(size_t(i / per_tile) * kConsumerWarps + warp) * per_tile + i % per_tile] = 0.f;
  grid_dependency_wait();

  // B fragments: xf[u][q] = {b_even, b_odd} of step q of this warp's unit u
  // (pair w or w + 8 of the chunk), and the group sums this lane's outputs
  // need.  Lane (g, t) loads x[bm][gi * 128 + 32 t .. + 31], permuted.
  uint4 xf[2][4];
  float sxu[2][2];  // [unit][m0 / m1] group sum of group 2 pair + hh
  auto frags_from_global = [&](int u, int pair) {
    float sum = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 o = make_uint4(0, 0, 0, 0);
      if (has_x && pair < p.pairs) {
        const uint4 v = *reinterpret_cast<const uint4*>(
            p.X + size_t(bm) * p.K + size_t(2 * pair + bh) * kGroup + 32 * t + 8 * q);
        o.x = __byte_perm(v.x, v.z, 0x5410);  // x0, x4
        o.y = __byte_perm(v.x, v.z, 0x7632);  // x1, x5
        o.z = __byte_perm(v.y, v.w, 0x5410);  // x2, x6
        o.w = __byte_perm(v.y, v.w, 0x7632);  // x3, x7
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
          sum += __uint_as_float(w4[j] << 16) + __uint_as_float(w4[j] & 0xFFFF0000u);
      }
      xf[u][q] = o;
    }
    // the group's sum over its four t-lanes
    sum += __shfl_xor_sync(0xffffffffu, sum, 1);
    sum += __shfl_xor_sync(0xffffffffu, sum, 2);
    // this lane's outputs need token m0 / m1 of group half hh: held by lane
    // 4 (4 hh + m) + t'
    sxu[u][0] = __shfl_sync(0xffffffffu, sum, 4 * (4 * hh + (m0 & 3)));
    sxu[u][1] = __shfl_sync(0xffffffffu, sum, 4 * (4 * hh + (m1 & 3)));
  };

  const float* sx = reinterpret_cast<const float*>(smem + p.off_sx);
  if constexpr (XREG) {
    frags_from_global(0, warp);
    frags_from_global(1, warp + kConsumerWarps);
  } else {
    // activations staged once, permuted as in gemv_ld.cuh, with group sums
    const int total8 = p.M * p.K / 8;
    float* sxw = reinterpret_cast<float*>(smem + p.off_sx);
    for (int base = 0; base < total8; base += kConsumerWarps * 32) {
      const int i = base + int(threadIdx.x);
      const bool ok = i < total8;
      float sum = 0.f;
      if (ok) {
        const int e = 8 * i, n = e / p.K, k = e - n * p.K;
        const uint4 v = *reinterpret_cast<const uint4*>(p.X + e);
        const int gi = k / kGroup, kg = k % kGroup;
        const int tt = kg / 32, q = (kg % 32) / 8;
        uint4 o;
        o.x = __byte_perm(v.x, v.z, 0x5410);
        o.y = __byte_perm(v.x, v.z, 0x7632);
        o.z = __byte_perm(v.y, v.w, 0x5410);
        o.w = __byte_perm(v.y, v.w, 0x7632);
        const int slot = (((gi >> 1) * 4 + q) * 2 + (gi & 1)) * 4 + tt;
        *reinterpret_cast<uint4*>(smem + p.off_x + size_t(n) * p.xs_row_bytes +
                                  (size_t(slot) << 4)) = o;
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
          sum += __uint_as_float(w4[j] << 16) + __uint_as_float(w4[j] & 0xFFFF0000u);
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (ok && (threadIdx.x & 15) == 0) sxw[(8 * i) / kGroup] = sum;  // [n][gi]
    }
    named_barrier_sync(1, kConsumerWarps * 32);
  }
  const uint32_t xs_lane = smem_addr(smem) + p.off_x + uint32_t(bm) * p.xs_row_bytes +
                           uint32_t((bh * 4 + t) * 16);

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  int cur_tile = tb0;
  auto flush = [&]() {
    // lanes L and L ^ 6 hold a row's two groups: add them (group A's first)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float other = __shfl_xor_sync(0xffffffffu, acc[i], 6);
      acc[i] = hh == 0 ? acc[i] + other : other + acc[i];
    }
    float* dst = part + (size_t(cur_tile - tb0) * kConsumerWarps + warp) * per_tile;
    if (hh == 0 && use0) {
      dst[rr0 * p.M + m0] = acc[0];
      dst[(rr0 + 4) * p.M + m0] = acc[2];
    }
    if (hh == 0 && use1) {
      dst[rr0 * p.M + m1] = acc[1];
      dst[(rr0 + 4) * p.M + m1] = acc[3];
    }
    acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
  };

  for (int i = 0; i < nstages; ++i) {
    const int slot = i % D;
    const int tile = tb0 + i / p.nch, ch = i % p.nch;
    if (tile != cur_tile) {
      flush();
      cur_tile = tile;
    }
    if (*abort_flag || !mbar_wait(&bars[kBarFull + slot], uint32_t(i / D) & 1u)) {
      *abort_flag = 1;
      break;
    }
    const uint32_t st = smem_addr(smem) + p.off_ring + uint32_t(slot) * kStageBytes;
    const uint8_t* stp = smem + p.off_ring + size_t(slot) * kStageBytes;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int pl = warp + u * kConsumerWarps;  // pair within the chunk
      const int pair = ch * kChunkPairs + pl;
      if (pair < p.pairs) {
        const uint32_t row_a = st + uint32_t(r * kRowBytes + pl * kPairBytes + c * 16);
        const uint4 c0 = lds128(row_a);
        const uint4 c1 = lds128(row_a + 4 * kRowBytes);
        float d[4] = {0.f, 0.f, 0.f, 0.f}, e[4] = {0.f, 0.f, 0.f, 0.f};
        const uint32_t w0[4] = {c0.x, c0.y, c0.z, c0.w};
        const uint32_t w1[4] = {c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t pa[4], pb[4];
          unpack_u4(w0[q], pa);
          unpack_u4(w1[q], pb);
          uint4 xv;
          if constexpr (XREG) {
            xv = xf[u][q];
          } else {
            xv = make_uint4(0, 0, 0, 0);
            if (has_x) xv = lds128(xs_lane + (uint32_t(pair * 4 + q) << 7));
          }
          const uint32_t a_even[4] = {pa[0], pb[0], pa[1], pb[1]};
          const uint32_t b_even[2] = {xv.x, xv.y};
          const uint32_t a_odd[4] = {pa[2], pb[2], pa[3], pb[3]};
          const uint32_t b_odd[2] = {xv.z, xv.w};
          mma_bf16_16816(d, a_even, b_even);
          mma_bf16_16816(e, a_odd, b_odd);
        }
        if (owner) {
          // y += s (C - (128 + z) Sx) for rows rr0 and rr0 + 4, group 2 pair + hh
          const int gl = 2 * pl + hh;  // group within the chunk
          const __half* ms = reinterpret_cast<const __half*>(stp + kCodesStage);
          const __half* mz = reinterpret_cast<const __half*>(stp + kCodesStage + kMetaStage);
          const float s0 = __half2float(ms[rr0 * (kMetaRow / 2) + gl]);
          const float s1 = __half2float(ms[(rr0 + 4) * (kMetaRow / 2) + gl]);
          const float b0 = SYM ? 136.f : 128.f + __half2float(mz[rr0 * (kMetaRow / 2) + gl]);
          const float b1 =
              SYM ? 136.f : 128.f + __half2float(mz[(rr0 + 4) * (kMetaRow / 2) + gl]);
          float x0, x1;
          if constexpr (XREG) {
            x0 = sxu[u][0];
            x1 = sxu[u][1];
          } else {
            x0 = sx[m0 * p.ngroups + 2 * pair + hh];
            x1 = m1 < p.M ? sx[m1 * p.ngroups + 2 * pair + hh] : 0.f;
          }
          if (use0) {
            acc[0] = fmaf(s0, fmaf(-b0, x0, d[0] + e[0]), acc[0]);
            acc[2] = fmaf(s1, fmaf(-b1, x0, d[2] + e[2]), acc[2]);
          }
          if (use1) {
            acc[1] = fmaf(s0, fmaf(-b0, x1, d[1] + e[1]), acc[1]);
            acc[3] = fmaf(s1, fmaf(-b1, x1, d[3] + e[3]), acc[3]);
          }
        }
      }
    }
    // the stage is read: the producer may refill it
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars[kBarEmpty + slot]);
  }
  if (nstages > 0) flush();
  named_barrier_sync(1, kConsumerWarps * 32);

  // Y[m][row] = sum over the warps in order
  const int outs = (tb1 - tb0) * per_tile;
  for (int i = threadIdx.x; i < outs; i += kConsumerWarps * 32) {
    const int tl = i / per_tile, rem = i - tl * per_tile;
    const float* src = part + size_t(tl) * kConsumerWarps * per_tile + rem;
    float y = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) y += src[w * per_tile];
    const int row = (tb0 + tl) * kTileRows + rem / p.M, m = rem % p.M;
    if (row < p.N && !*abort_flag) {
      if (p.y_bf16)
        static_cast<__nv_bfloat16*>(p.Y)[size_t(m) * p.N + row] = __float2bfloat16_rn(y);
      else
        static_cast<float*>(p.Y)[size_t(m) * p.N + row] = y;
    }
  }
}

}  // namespace tb
}  // namespace wq
