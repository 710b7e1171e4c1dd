// gemv_ld.cuh -- the direct-load small-batch matmul Y = X * What^T for 4-bit
// codes in groups of 128 (M <= 4): "vLLM 量化与推测解码" section 2 (W4A16:
// packed INT4 weights and their group scales are unpacked and scaled on
// chip, multiplied with 16-bit activations and accumulated in higher
// precision) and "量化" (llminference s08) section 实现 (each group's block
// is dequantized inside the accumulation).
//
// Decode moves bytes ("量化" section 问题: time = bytes / bandwidth).  A plain
// read of a layer's bytes reaches the HBM copy rate at this size when every
// SM keeps many independent 16-byte loads in flight and every load
// instruction covers whole 128-byte lines, so this kernel is shaped like
// such a read:
//
//   * One CTA of 16 warps per SM; CTA b owns a contiguous range of 8-row
//     tiles.  A "unit" is one tile x one pair of groups: 8 rows x 128 bytes
//     of codes (1 KB).  The units of the CTA's range, tile-major, are cut
//     into 16 contiguous ranges, one per warp.
//   * Lane L = 8 r + c of a warp copies bytes 16 c .. 16 c + 15 of the
//     unit's row r (one instruction: rows 0-3, whole lines) and of row r + 4
//     (a second one) into its own 32 bytes of a per-warp ring of DEPTH units
//     in shared memory (cp.async: no registers held while in flight), and
//     reads them back itself when the unit is computed.  The CTA's scales
//     and zeros (a contiguous block of each tensor) are read once, coalesced,
//     into a shared-memory table of binary32 pairs {s, 128 + z}.  When the
//     caller promises the weights are static, the first DEPTH units, the
//     table and the clearing of the partial sums all happen before the wait
//     on the previous grid; only the activations are read after it.
//   * Seen as mma.sync m16n8k16 fragments (lane = 4 g + t), lane L holds row
//     g of the A operand with g = 2 r + (c / 4), i.e. A row g is (tile row
//     g / 2, group g % 2 of the pair) and rows g + 8 are tile rows 4 + g / 2.
//     The two groups of a pair need different activations, so they use
//     different columns of B: column n = 4 h + m carries token m of group h.
//     D[g][n] is meaningful where g % 2 == n / 4; the other half is unused.
//   * Unpacking: one LOP3 turns two codes u into the exact bfloat16 pair
//     (128 + u).  A group is eight k16 steps in one accumulator, and its
//     scale applies after it, in binary32: y += s * (C - (128 + z) * Sx), Sx
//     the group's activation sum (for symmetric codes the bias is 128 + 8).
//   * The activations are staged once per CTA in shared memory, each 8-value
//     block permuted to (x0, x4, x1, x5, x2, x6, x3, x7) to match the pairs,
//     laid out so that the lanes of one B column read 64 contiguous bytes;
//     the group sums Sx are formed at the same time.
//   * Deterministic reduction: the two lanes holding a row's two groups add
//     their sums (a shuffle), every warp leaves its per-tile partial sums in
//     shared memory, and after one barrier each output is the sum over the
//     warps in warp order.
#pragma once

#include "common.cuh"
#include "unpack.cuh"

namespace wq {
namespace ld {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kDepth = 3;        // default units in flight per warp (shared-memory ring)
constexpr int kMaxDepth = 8;
constexpr int kMaxM = 4;
constexpr int kGroup = 128;      // codes per group (4-bit: 64 bytes of a row)
constexpr int kTileRows = 8;
constexpr int kUnitBytes = 128;  // bytes of one tile row in a unit (a pair of groups)

struct Params {
  const __nv_bfloat16* X;  // [M][K]
  void* Y;                 // [M][N] binary32 or bfloat16
  const uint8_t* codes;    // [N][K/2]
  const __half* scales;    // [N][ngroups]
  const __half* zeros;     // [N][ngroups] or null (symmetric)
  int M, N, K, ngroups;    // ngroups even
  int tiles;               // ceil(N / 8)
  int y_bf16;
  int pdl;                 // weights may be read before the previous grid completes
  // 2^28, 2^24, 2^20: the high word of w times these is w >> 4, 8, 12.  Given
  // as parameters (values the compiler cannot see), the right shifts of the
  // unpack run as integer multiplies on the FMA pipe instead of the ALU pipe.
  uint32_t mul_shr4, mul_shr8, mul_shr12;
  uint32_t xs_row_bytes;   // K * 2 + 64: shared-memory bytes per activation row
  uint32_t off_sx;         // [M][ngroups] binary32 group sums
  uint32_t off_sz;         // [rows of the CTA][ngroups + 1] {scale, 128 + zero} binary32
  uint32_t off_part;       // [tiles per CTA][kWarps][8][M] binary32 partials
  uint32_t off_ring;       // [kWarps][DEPTH][2][32 lanes][16 bytes] codes ring
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  // 16 bytes global -> shared through L2 only; zero-filled when !valid
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint2 ldg_stream64(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];"
               : "=r"(v.x), "=r"(v.y)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t mul_hi(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.hi.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Eight 4-bit codes of one word -> four bfloat16 pairs (128 + u), as
// unpack_u4, with the three right shifts either on the ALU pipe (SHF) or as
// multiplies by 2^(32-s) keeping the high word (the FMA pipe).
template <bool FMA_SHIFT>
__device__ __forceinline__ void unpack_u4_pipe(uint32_t w, uint32_t (&r)[4], const Params& p) {
  constexpr uint32_t kMask = 0x000F000Fu, kMagic = 0x43004300u;  // bf16 128.0 pair
  r[0] = lop3_and_or(w, kMask, kMagic);
  if constexpr (FMA_SHIFT) {
    r[1] = lop3_and_or(mul_hi(w, p.mul_shr4), kMask, kMagic);
    r[2] = lop3_and_or(mul_hi(w, p.mul_shr8), kMask, kMagic);
    r[3] = lop3_and_or(mul_hi(w, p.mul_shr12), kMask, kMagic);
  } else {
    r[1] = lop3_and_or(w >> 4, kMask, kMagic);
    r[2] = lop3_and_or(w >> 8, kMask, kMagic);
    r[3] = lop3_and_or(w >> 12, kMask, kMagic);
  }
}

// The fetch side of a warp's units: the byte offset of this lane's 16 bytes
// of tile row r in the codes, and whether rows r and r + 4 exist.
struct FetchWalk {
  const uint8_t* ptr;  // this lane's 16 bytes of tile row r
  int pair, left;
  bool ok0, ok1;
  int row0;
  __device__ __forceinline__ void set_rows(int N) {
    ok0 = row0 < N;
    ok1 = row0 + 4 < N;
  }
  __device__ __forceinline__ void next(int pairs, size_t row_bytes, int N) {
    --left;
    ptr += kUnitBytes;
    if (++pair == pairs) {  // next tile: 8 rows down, back to the first pair
      pair = 0;
      ptr += 7 * row_bytes;
      row0 += kTileRows;
      set_rows(N);
    }
  }
};

// One unit's 32 bytes for this lane into ring slot `dst` (row r at dst, row
// r + 4 at dst + 512); rows past N are zero-filled without reading.
__device__ __forceinline__ void load_unit(const uint8_t* codes, const FetchWalk& f,
                                          size_t row_bytes, uint32_t dst) {
  cp_async16(dst, f.ok0 ? f.ptr : codes, f.ok0);
  cp_async16(dst + 512, f.ok1 ? f.ptr + 4 * row_bytes : codes, f.ok1);
}

// Units in order: tile-major, pair-minor.
struct UnitWalk {
  int tile, pair, left;
  __device__ __forceinline__ void next(int pairs) {
    --left;
    if (++pair == pairs) {
      pair = 0;
      ++tile;
    }
  }
};

// MT: a compile-time bound on M (1, 2 or 4), so that lanes whose token
// columns cannot exist keep no accumulators.  DEPTH: units in flight per
// warp.  FMA_SHIFT: the unpack's right shifts as multiplies (FMA pipe).
// MINB: CTAs per SM the register allocation must allow (2 lets the next
// launch's CTA start streaming while this one finishes).
template <bool SYM, int MT, int DEPTH, bool FMA_SHIFT, int MINB>
__global__ void __launch_bounds__(kThreads, MINB) gemv_ld_kernel(const Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = lane >> 3, c = lane & 7;  // load view: tile row r (and r + 4), chunk c
  const int g = lane >> 2, t = lane & 3;  // fragment view
  const int ng = p.ngroups, pairs = ng / 2;
  const int tb0 = int(int64_t(blockIdx.x) * p.tiles / gridDim.x);
  const int tb1 = int(int64_t(blockIdx.x + 1) * p.tiles / gridDim.x);
  const int units = (tb1 - tb0) * pairs;
  const int ub = int(int64_t(warp) * units / kWarps);
  const int ue = int(int64_t(warp + 1) * units / kWarps);

  const size_t row_bytes = size_t(p.K) / 2;
  UnitWalk use{tb0 + ub / pairs, ub % pairs, ue - ub};
  FetchWalk fetch;
  fetch.pair = use.pair;
  fetch.left = use.left;
  fetch.row0 = use.tile * kTileRows + r;
  fetch.ptr = p.codes + size_t(fetch.row0) * row_bytes + size_t(use.pair) * kUnitBytes +
              size_t(c) * 16;
  fetch.set_rows(p.N);
  // this lane's 16 bytes of slot 0 (row r); slot j at + 1024 j
  const uint32_t ring = smem_addr(smem) + p.off_ring + uint32_t(warp * DEPTH * 1024 + lane * 16);
  // one commit group per unit (empty past the end) keeps the wait count fixed
  auto prefetch = [&](int slot) {
    if (fetch.left > 0) {
      load_unit(p.codes, fetch, row_bytes, ring + uint32_t(slot) * 1024);
      fetch.next(pairs, row_bytes, p.N);
    }
    cp_async_commit();
  };

  float* sx = reinterpret_cast<float*>(smem + p.off_sx);
  float2* sz = reinterpret_cast<float2*>(smem + p.off_sz);
  float* part = reinterpret_cast<float*>(smem + p.off_part);
  const int sz_stride = ng + 1;  // entries per row: rows land on different banks

  // The weight-side set-up, which reads no input the previous kernel may
  // write: the first DEPTH units of every warp are requested, the CTA's
  // scales and zeros -- rows [8 tb0, min(N, 8 tb1)) x ngroups, contiguous
  // blocks of 4 binary16 values (ngroups is even and rows start at a
  // multiple of 8: every block is 8-byte aligned and inside one row) -- are
  // turned into the {s, 128 + z} table (symmetric: 128 + 8), and the partial
  // sums are cleared.  With static weights all of this happens before the
  // wait on the previous grid.
  const int row_lo = tb0 * kTileRows;
  const int rows = min(p.N, tb1 * kTileRows) - row_lo;
  const int meta4 = rows * ng / 4;
  auto weight_setup = [&]() {
#pragma unroll
    for (int j = 0; j < DEPTH; ++j) prefetch(j);
    for (int i = int(threadIdx.x); i < meta4; i += kThreads) {
      const uint2 a = ldg_stream64(p.scales + size_t(row_lo) * ng + 4 * size_t(i));
      const uint2 z = SYM ? make_uint2(0, 0)
                          : ldg_stream64(p.zeros + size_t(row_lo) * ng + 4 * size_t(i));
      const int e = 4 * i, row = e / ng, gi = e - row * ng;
      float2* d = sz + row * sz_stride + gi;
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
    const int nparts = (tb1 - tb0) * kWarps * kTileRows * p.M;
    for (int i = threadIdx.x; i < nparts; i += kThreads) part[i] = 0.f;
  };
  if (p.pdl) weight_setup();
  grid_dependents_launch();
  grid_dependency_wait();
  if (!p.pdl) weight_setup();

  {
    // activations, permuted, and their group sums
    const int total8 = p.M * p.K / 8;  // a multiple of 16: groups of 128 never straddle
    for (int base = 0; base < total8; base += kThreads) {
      const int i = base + int(threadIdx.x);
      const bool ok = i < total8;
      float sum = 0.f;
      if (ok) {
        const int e = 8 * i, n = e / p.K, k = e - n * p.K;
        const uint4 v = *reinterpret_cast<const uint4*>(p.X + e);
        const int gi = k / kGroup, kg = k % kGroup;
        const int tt = kg / 32, q = (kg % 32) / 8;
        uint4 o;
        o.x = __byte_perm(v.x, v.z, 0x5410);  // x0, x4
        o.y = __byte_perm(v.x, v.z, 0x7632);  // x1, x5
        o.z = __byte_perm(v.y, v.w, 0x5410);  // x2, x6
        o.w = __byte_perm(v.y, v.w, 0x7632);  // x3, x7
        const int slot = (((gi >> 1) * 4 + q) * 2 + (gi & 1)) * 4 + tt;
        *reinterpret_cast<uint4*>(smem + size_t(n) * p.xs_row_bytes + (size_t(slot) << 4)) = o;
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
          sum += __uint_as_float(w[j] << 16) + __uint_as_float(w[j] & 0xFFFF0000u);
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (ok && (threadIdx.x & 15) == 0) sx[(8 * i) / kGroup] = sum;  // [n][gi] flattened
    }
  }
  __syncthreads();

  // B column g carries token g % 4 of group half g / 4
  const int bm = g & 3, bh = g >> 2;
  const bool has_x = bm < MT && bm < p.M;
  const uint32_t xs_lane =
      smem_addr(smem) + uint32_t(bm) * p.xs_row_bytes + uint32_t((bh * 4 + t) * 16);
  // outputs of this lane: D[g][2t], D[g][2t+1] (tile row g / 2) and the same
  // for tile row 4 + g / 2, valid where the group half g % 2 == t / 2
  const int hh = g & 1;
  const bool owner = hh == (t >> 1);
  const int m0 = (2 * t) & 3, m1 = m0 + 1;
  const bool use0 = owner && m0 < MT && m0 < p.M;
  const bool use1 = owner && m1 < MT && m1 < p.M;
  const int rr0 = g >> 1, rr1 = rr0 + 4;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  int cur_tile = use.tile;
  // this lane's rows of the {s, 128 + z} table for the current tile, and its
  // tokens' group sums
  const float2* sz0 = sz + ((cur_tile - tb0) * kTileRows + rr0) * sz_stride;
  const float* sx0 = sx + m0 * ng;
  const float* sx1 = sx + m1 * ng;

  // Lanes L and L ^ 6 own the same outputs for the two groups of a pair:
  // their sums are added (group A's lane first) and group A's lane stores.
  auto flush = [&]() {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float other = __shfl_xor_sync(0xffffffffu, acc[i], 6);
      acc[i] = hh == 0 ? acc[i] + other : other + acc[i];
    }
    float* dst = part + size_t((cur_tile - tb0) * kWarps + warp) * kTileRows * p.M;
    if (hh == 0 && use0) {
      dst[rr0 * p.M + m0] = acc[0];
      dst[rr1 * p.M + m0] = acc[2];
    }
    if (hh == 0 && use1) {
      dst[rr0 * p.M + m1] = acc[1];
      dst[rr1 * p.M + m1] = acc[3];
    }
    acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
  };

  while (use.left > 0) {
#pragma unroll
    for (int j = 0; j < DEPTH; ++j) {
      if (use.left > 0) {
        if (use.tile != cur_tile) {
          flush();
          cur_tile = use.tile;
          sz0 = sz + ((cur_tile - tb0) * kTileRows + rr0) * sz_stride;
        }
        cp_async_wait<DEPTH - 1>();  // this unit's copies (issued by this lane) landed
        const uint4 c0 = lds128(ring + uint32_t(j) * 1024);
        const uint4 c1 = lds128(ring + uint32_t(j) * 1024 + 512);
        const int pair = use.pair;
        float d[4] = {0.f, 0.f, 0.f, 0.f}, e[4] = {0.f, 0.f, 0.f, 0.f};  // two chains
        const uint32_t w0[4] = {c0.x, c0.y, c0.z, c0.w};
        const uint32_t w1[4] = {c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t pa[4], pb[4];
          unpack_u4_pipe<FMA_SHIFT>(w0[q], pa, p);
          unpack_u4_pipe<FMA_SHIFT>(w1[q], pb, p);
          uint4 xv = make_uint4(0, 0, 0, 0);
          if (has_x) xv = lds128(xs_lane + (uint32_t(pair * 4 + q) << 7));
          const uint32_t a_even[4] = {pa[0], pb[0], pa[1], pb[1]};
          const uint32_t b_even[2] = {xv.x, xv.y};
          const uint32_t a_odd[4] = {pa[2], pb[2], pa[3], pb[3]};
          const uint32_t b_odd[2] = {xv.z, xv.w};
          mma_bf16_16816(d, a_even, b_even);
          mma_bf16_16816(e, a_odd, b_odd);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) d[i] += e[i];
        // the slot's bytes are in registers and used: refill it
        prefetch(j);
        if (owner) {
          // y += s * (C - (128 + z) * Sx), per row, in binary32
          const int gi = 2 * pair + hh;
          const float2 e0 = sz0[gi];                       // tile row rr0
          const float2 e1 = sz0[4 * sz_stride + gi];       // tile row rr0 + 4
          if (use0) {
            const float x = sx0[gi];
            acc[0] = fmaf(e0.x, fmaf(-e0.y, x, d[0]), acc[0]);
            acc[2] = fmaf(e1.x, fmaf(-e1.y, x, d[2]), acc[2]);
          }
          if (use1) {
            const float x = sx1[gi];
            acc[1] = fmaf(e0.x, fmaf(-e0.y, x, d[1]), acc[1]);
            acc[3] = fmaf(e1.x, fmaf(-e1.y, x, d[3]), acc[3]);
          }
        }
        use.next(pairs);
      }
    }
  }
  if (ue > ub) flush();
  cp_async_wait<0>();
  __syncthreads();

  // Y[m][row] = sum over the warps in order
  const int per_tile = kTileRows * p.M;
  const int outs = (tb1 - tb0) * per_tile;
  for (int i = threadIdx.x; i < outs; i += kThreads) {
    const int tl = i / per_tile, rem = i - tl * per_tile;
    const float* src = part + size_t(tl) * kWarps * per_tile + rem;
    float y = 0.f;
#pragma unroll 8
    for (int w = 0; w < kWarps; ++w) y += src[w * per_tile];
    const int row = (tb0 + tl) * kTileRows + rem / p.M, m = rem % p.M;
    if (row < p.N) {
      if (p.y_bf16)
        static_cast<__nv_bfloat16*>(p.Y)[size_t(m) * p.N + row] = __float2bfloat16_rn(y);
      else
        static_cast<float*>(p.Y)[size_t(m) * p.N + row] = y;
    }
  }
}

}  // namespace ld
}  // namespace wq
