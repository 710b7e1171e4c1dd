// gemv.cuh -- fused dequant-in-register small-batch matmul Y = X * What^T
// (M <= 32): "vLLM 量化与推测解码" section 2 (W4A16: packed INT4 weights and
// group scales are unpacked and scaled on chip, multiplied with 16-bit
// activations, accumulated in higher precision; the full-precision weights
// are never materialised) and "量化" (llminference s08) section 实现 (each
// group's block is dequantized inside the accumulation).
//
// Decode is bound by the bytes of the packed weights ("量化" section 问题:
// time = bytes / bandwidth), so the kernel is built around streaming the
// codes exactly once at HBM speed with as few instructions per weight as
// possible:
//
//   * Persistent CTAs, one per SM.  Work item = RT row tiles of 16 rows; the
//     CTA's K range (all of K, or 1/C of it when a cluster of C CTAs splits
//     K) is cut into stages.  One producer warp streams each row's segment
//     of a stage with one bulk copy (cp.async.bulk, the rows' segments are
//     contiguous in memory; one warp instruction issues a whole row tile)
//     into a ring of DEPTH stages (mbarrier full/empty pairs), together with
//     the stage's [16 rows x groups] scale and zero tiles (TMA boxes), so
//     ~200 KB per SM are in flight regardless of register pressure.  Rows
//     land an odd multiple of 64 bytes apart, so the consumers' 16-byte
//     code loads are bank-conflict free.
//   * 16 consumer warps.  Warp (rt, sk) owns row tile rt and BPW boxes of
//     every stage.  Lane (g, t) of a warp holds rows g and g+8 and one
//     quarter of every group, so each tensor-core step stays inside one group.
//   * Unpacking: one LOP3 turns two 4-bit codes u into the bfloat16 pair
//     (128 + u) (exponent 2^7, code in the low mantissa bits: exact); 8-bit
//     codes go through a binary32 exponent trick and a paired conversion.
//     The integer-valued operands enter mma.sync m16n8k16 (weights as the
//     16-row A operand, activations as the 8-column B operand, binary32
//     accumulation), which replaces 8 scalar FMAs per lane and step.
//   * Per group, in binary32: y += s * (C - (128 + z) * Sx), where C is the
//     group's tensor-core sum of x * (128 + u) and Sx the group's sum of x
//     (precomputed once per CTA).  For 8-bit codes the bias is z.
//   * The activations are staged in shared memory once per CTA, permuted so
//     that every B fragment is one 8-byte load.
//   * Deterministic reductions: warps of a row tile add their partial sums
//     through shared memory in a fixed order; cluster ranks add theirs
//     through distributed shared memory in rank order.
#pragma once

#include "common.cuh"
#include "unpack.cuh"

namespace wq {
namespace gemv {

constexpr int kNumConsumerWarps = 16;
constexpr int kThreads = (kNumConsumerWarps + 1) * 32;
constexpr int kBoxRows = 16;
constexpr int kBoxRowBytes = 64;
constexpr int kBoxBytes = kBoxRows * kBoxRowBytes;  // 1 KB

struct Params {
  const __nv_bfloat16* X;  // [M][K]
  void* Y;                 // [M][N]
  const __half* scales;    // [N][ngroups] (used by the plain-load metadata path)
  const __half* zeros;     // [N][ngroups] or null
  int M, N, K, ngroups;
  int row_tiles;           // ceil(N / 16)
  int items;               // ceil(row_tiles / RT)
  int RT, SKW, BPW;        // row tiles per item, warps per row tile, boxes per warp per stage
  int depth;               // ring stages
  int kc;                  // K extent of one cluster rank (multiple of max(box k, G))
  int stage_k;             // SKW * BPW * box_k
  int stages_per_item;     // ceil(kc / stage_k)
  int meta_tma;            // 1: metadata tiles by TMA; 0: loaded by the producer warp
  int y_bf16;
  uint32_t stage_bytes;    // codes + metadata of one stage
  uint32_t meta_offset;    // offset of the metadata inside a stage
  uint32_t off_ring, off_x, off_sx, off_red, off_part;
  uint32_t x_row_stride;   // bytes per activation row in shared memory (odd multiple of 64)
  int red_bufs;            // 0: every item's partials kept, one reduction at the end;
                           // 2: double-buffered per item; 1: single buffer, two barriers
  const uint8_t* codes;    // [N][K*BITS/8]
  uint32_t row_stride;     // bytes between rows of a stage in shared memory
  int contig;              // 1: a stage is whole rows (C == 1, one stage of all K): the
                           // item's codes and metadata are contiguous and arrive by one
                           // bulk copy each
};

// Shared-memory loads as plain C++ accesses (offsets from the dynamic
// shared-memory base): ordered after the mbarrier waits, whose asm carries a
// memory clobber, but otherwise free for the compiler to schedule early.
template <typename T>
__device__ __forceinline__ T sld(const uint8_t* smem, uint32_t off) {
  return *reinterpret_cast<const T*>(smem + off);
}

// Load N consecutive 32-bit words (N = 1, 2, 4) from shared memory.
template <int N>
__device__ __forceinline__ void load_words(const uint8_t* smem, uint32_t off, uint32_t (&w)[N]) {
  if constexpr (N == 4) {
    const uint4 v = sld<uint4>(smem, off);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (N == 2) {
    const uint2 v = sld<uint2>(smem, off);
    w[0] = v.x; w[1] = v.y;
  } else {
    w[0] = sld<uint32_t>(smem, off);
  }
}

template <int BITS, int G>
struct Geometry {
  static constexpr int kBoxK = kBoxRowBytes * 8 / BITS;           // k per box row
  static constexpr int kGroupBytes = G * BITS / 8;                 // bytes of one group row
  static constexpr int kU = kGroupBytes < kBoxRowBytes ? kGroupBytes : kBoxRowBytes;
  static constexpr int kUk = kU * 8 / BITS;                        // k per sub-unit
  static constexpr int kQB = kU / 4;                               // bytes per lane quarter
  static constexpr int kQk = kUk / 4;                              // k per lane quarter
  static constexpr int kWords = kQB / 4;                           // 32-bit words per quarter
  static constexpr int kSubUnits = kBoxRowBytes / kU;              // sub-units per box
  static constexpr int kStepsPerSubUnit = kUk / 16;
  static constexpr int kSubUnitsPerGroup = G / kUk;                // 1, or 2 (8-bit, G = 128)
  static_assert(kQB == 4 || kQB == 8 || kQB == 16, "quarter size");
  static_assert(kQk % 8 == 0, "activation staging works in blocks of 8");
};

// FAST: M <= 8 (MT == 1), one stage per item, and the warps' box count is
// kFastBPW: every warp then covers the same K slice for every item, so its
// activation fragments are loaded into registers once, and the whole stage
// (codes loads, unpack, tensor-core steps, sweeps, epilogues) is unrolled
// with compile-time offsets.
template <int BITS>
struct FastShape {
  static constexpr int kBPW = BITS == 4 ? 2 : 4;
};

template <int BITS, bool SYM, int G, int MT, int MEFF, bool FAST>
__global__ void __launch_bounds__(kThreads, 1)
    gemv_kernel(const __grid_constant__ CUtensorMap tmap_codes,
                const __grid_constant__ CUtensorMap tmap_scales,
                const __grid_constant__ CUtensorMap tmap_zeros, const Params p) {
  using Geo = Geometry<BITS, G>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + 32;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 512);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Cluster geometry: rank splits K; cluster id walks the items.
  const uint32_t rank = cluster_ctarank();
  uint32_t csize;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(csize));
  const int cid = int(cluster_id_x());
  const int ncl = int(num_clusters_x());
  const int k_begin = int(rank) * p.kc;
  const int k_end = min(p.K, k_begin + p.kc);

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.depth; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kNumConsumerWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // Kernels launched after this one may be scheduled; they wait for this
  // grid before touching its outputs.  The weights are read before the wait
  // for the previous grid (they are not written by it, as the caller
  // promises when it asks for programmatic dependent launch).
  grid_dependents_launch();

  uint8_t* ring = smem + p.off_ring;
  constexpr bool kAsymMeta = !SYM;

  if (warp == kNumConsumerWarps) {
    // ------------------------------------------------------------ producer
    // Per stage: lane 0 posts the byte count on the full barrier, then lanes
    // issue one bulk copy each (row r of row tile rt: its segment of the
    // stage's K range, contiguous in memory), so a 16-row x 2 KB stage takes
    // one warp instruction; the scale/zero tiles come by two TMA boxes.
    if (lane == 0 && p.meta_tma) {
      prefetch_tensormap(&tmap_scales);
      if (kAsymMeta) prefetch_tensormap(&tmap_zeros);
    }
    const uint64_t policy = l2_policy_evict_first();
    const uint32_t meta_rt_bytes = uint32_t(kBoxRows * (p.stage_k / G) * 2);
    const size_t row_bytes = size_t(p.K) * BITS / 8;
    const uint8_t* codes = p.codes;
    int slot = 0;
    uint32_t phase = 0;
    for (int item = cid; item < p.items; item += ncl) {
      const int rows_total = min(p.RT * kBoxRows, p.N - item * p.RT * kBoxRows);
      for (int st = 0; st < p.stages_per_item; ++st) {
        if (!*abort_flag && !mbar_wait(&empty[slot], phase ^ 1)) *abort_flag = 1;
        uint8_t* stage = ring + size_t(slot) * p.stage_bytes;
        uint8_t* meta = stage + p.meta_offset;
        const int stage_k0 = k_begin + st * p.stage_k;
        const int g0 = stage_k0 / G;
        // a rank's last stage may lie past its K range: then nothing is copied
        const bool has_k = stage_k0 < k_end;
        const uint32_t seg = has_k ? uint32_t(min(p.stage_k, k_end - stage_k0) * BITS / 8) : 0u;
        const int tiles_here = (rows_total + kBoxRows - 1) / kBoxRows;
        const uint32_t meta_bytes_tma =
            p.contig ? uint32_t(rows_total) * uint32_t(p.ngroups) * 2 : uint32_t(tiles_here) * meta_rt_bytes;
        const uint32_t bytes =
            uint32_t(rows_total) * seg +
            (has_k && p.meta_tma ? meta_bytes_tma * (kAsymMeta ? 2 : 1) : 0u);
        if (!p.meta_tma) {
          // plain loads of the stage's metadata by the whole warp
          const int sg = p.stage_k / G;
          for (int rt = 0; rt < tiles_here; ++rt) {
            const int tile = item * p.RT + rt;
            __half* ms = reinterpret_cast<__half*>(meta + rt * meta_rt_bytes);
            __half* mz = reinterpret_cast<__half*>(meta + (p.RT + rt) * meta_rt_bytes);
            for (int e = lane; e < kBoxRows * sg; e += 32) {
              const int r = e / sg, gl = e % sg;
              const int row = tile * kBoxRows + r, gi = g0 + gl;
              const bool ok = row < p.N && gi < p.ngroups;
              ms[e] = ok ? p.scales[size_t(row) * p.ngroups + gi] : __float2half(0.f);
              if (kAsymMeta) mz[e] = ok ? p.zeros[size_t(row) * p.ngroups + gi] : __float2half(0.f);
            }
          }
        }
        if (lane == 0) mbar_arrive_expect_tx(&full[slot], bytes);
        __syncwarp();
        if (!*abort_flag && has_k && p.contig) {
          // whole rows: one copy each for the codes, the scales and the zeros
          if (lane == 0) {
            const size_t row0 = size_t(item) * p.RT * kBoxRows;
            bulk_load(stage, codes + row0 * row_bytes, uint32_t(rows_total) * seg, &full[slot],
                      policy);
            const uint32_t mbytes = uint32_t(rows_total) * uint32_t(p.ngroups) * 2;
            bulk_load(meta, p.scales + row0 * p.ngroups, mbytes, &full[slot], policy);
            if (kAsymMeta)
              bulk_load(meta + p.RT * meta_rt_bytes, p.zeros + row0 * p.ngroups, mbytes, &full[slot],
                        policy);
          }
        } else if (!*abort_flag && has_k) {
          const size_t src0 = size_t(item) * p.RT * kBoxRows * row_bytes + size_t(stage_k0) * BITS / 8;
          for (int r = lane; r < rows_total; r += 32)
            bulk_load(stage + size_t(r) * p.row_stride, codes + src0 + size_t(r) * row_bytes, seg,
                      &full[slot], policy);
          if (lane == 0 && p.meta_tma) {
            for (int rt = 0; rt < tiles_here; ++rt) {
              const int row0 = (item * p.RT + rt) * kBoxRows;
              tma_load_2d(meta + rt * meta_rt_bytes, &tmap_scales, &full[slot], g0, row0, policy);
              if (kAsymMeta)
                tma_load_2d(meta + (p.RT + rt) * meta_rt_bytes, &tmap_zeros, &full[slot], g0, row0,
                            policy);
            }
          }
        }
        __syncwarp();
        if (++slot == p.depth) {
          slot = 0;
          phase ^= 1;
        }
      }
    }
    // Drain: every issued stage must have landed before the CTA may exit.
    if (*abort_flag && lane == 0) {
      for (int i = 0; i < p.depth; ++i) {
        int s2 = slot - 1 - i;
        uint32_t ph = phase;
        if (s2 < 0) {
          s2 += p.depth;
          ph ^= 1;
        }
        mbar_wait(&full[s2], ph);
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    grid_dependency_wait();  // activations and outputs belong to the previous grid until then
    const int tid = threadIdx.x;  // 0 .. 16*32-1
    const int nthr = kNumConsumerWarps * 32;
    const int M = p.M;
    uint8_t* xs = smem + p.off_x;
    float* sx = reinterpret_cast<float*>(smem + p.off_sx);
    const int sx_stride = p.kc / G;                    // Sx is [m][group]
    constexpr int kSxRows = 8 * MT;
    constexpr int kChunksPerQuarter = Geo::kQk / 8;  // 8-k chunks per lane quarter of a sub-unit

    // Stage X for this rank's K range as [m][chunk][quarter][8 values] (one
    // 16-byte load feeds two tensor-core steps), plus one row of zeros that
    // B-fragment lanes without an activation row read.  Each thread takes 8
    // consecutive k; the G/8 threads of a group add their sums by shuffles
    // (a fixed order), giving the per-group sums Sx.
    {
      const int nq = (k_end - k_begin) / 8;
      const int total = M * nq;
      for (int base = warp * 32; base < total; base += nthr) {
        const int idx = base + lane;
        const bool valid = idx < total;
        float part_sum = 0.f;
        int m = 0, r = 0;
        if (valid) {
          m = idx / nq;
          r = (idx % nq) * 8;
          const uint4 v = *reinterpret_cast<const uint4*>(p.X + size_t(m) * p.K + k_begin + r);
          const int su = r / Geo::kUk, rr = r % Geo::kUk;
          const int tq = rr / Geo::kQk, rq = rr % Geo::kQk;
          const int chunk = su * kChunksPerQuarter + rq / 8;
          uint4 o = v;
          if (BITS == 4) {  // [x0 x4 x1 x5 x2 x6 x3 x7]
            o.x = __byte_perm(v.x, v.z, 0x5410);
            o.y = __byte_perm(v.x, v.z, 0x7632);
            o.z = __byte_perm(v.y, v.w, 0x5410);
            o.w = __byte_perm(v.y, v.w, 0x7632);
          }
          *reinterpret_cast<uint4*>(xs + size_t(m) * p.x_row_stride + chunk * 64 + tq * 16) = o;
          const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.x));
          const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.y));
          const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.z));
          const float2 f3 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.w));
          part_sum = ((f0.x + f0.y) + (f1.x + f1.y)) + ((f2.x + f2.y) + (f3.x + f3.y));
        }
#pragma unroll
        for (int off = 1; off < G / 8; off <<= 1)
          part_sum += __shfl_xor_sync(0xffffffffu, part_sum, off);
        if (valid && (r % G) == 0) sx[m * sx_stride + r / G] = part_sum;
      }
      // the zero row, and zero sums for the padding rows m >= M
      for (int e = tid; e < int(p.x_row_stride / 16); e += nthr)
        *reinterpret_cast<uint4*>(xs + size_t(M) * p.x_row_stride + e * 16) = make_uint4(0, 0, 0, 0);
      for (int e = M * sx_stride + tid; e < kSxRows * sx_stride; e += nthr) sx[e] = 0.f;
    }
    named_barrier_sync(1, nthr);

    const int rt = warp / p.SKW, sk = warp % p.SKW;
    const int g = lane >> 2, t = lane & 3;
    const uint32_t sx_off = p.off_sx;
    const uint32_t zero_row = p.off_x + uint32_t(M) * p.x_row_stride + t * 16;
    float* red = reinterpret_cast<float*>(smem + p.off_red);
    float* part = reinterpret_cast<float*>(smem + p.off_part);
    const uint32_t meta_rt_bytes = uint32_t(kBoxRows * (p.stage_k / G) * 2);
    const int sg = p.stage_k / G;
    const int per_tile = kBoxRows * M;
    const int red_stride = p.RT * p.SKW * per_tile;  // floats per buffer

    // Columns of the 8-wide B operand.  MT == 1: column = jj * MEFF + m, so
    // one accumulator sweeps kJ = 8 / MEFF consecutive groups of this warp
    // (group jj of the sweep in column block jj) before one epilogue.
    // MT > 1: column = m within each n8 tile, one group per sweep.
    constexpr int kJ = MT == 1 ? 8 / MEFF : 1;
    // this lane's B column: activation row and sweep slot
    const int col_m = MT == 1 ? g % MEFF : g;
    const int col_jj = MT == 1 ? g / MEFF : 0;
    uint32_t xrow[MT];
#pragma unroll
    for (int nt = 0; nt < MT; ++nt) {
      const int m = col_m + 8 * nt;
      xrow[nt] = m < M ? p.off_x + uint32_t(m) * p.x_row_stride + t * 16 : zero_row;
    }

    // Sum the SKW partials of one item's row tiles (buffer rb) in a fixed
    // order and write Y (one CTA) or this rank's cluster partials.  Threads
    // rotate with the item so the work spreads over the warps.
    auto reduce_item = [&](const float* rb, int item, int li, int tid_) {
      const int rot = (li * 32 * 5) % nthr;
      const int me = (tid_ + nthr - rot) % nthr;
      for (int o = me; o < p.RT * per_tile; o += nthr) {
        const int rto = o / per_tile, rem = o % per_tile;
        const float* src = rb + rto * p.SKW * per_tile + rem;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        int s2 = 0;
        for (; s2 + 4 <= p.SKW; s2 += 4) {
          acc[0] += src[(s2 + 0) * per_tile];
          acc[1] += src[(s2 + 1) * per_tile];
          acc[2] += src[(s2 + 2) * per_tile];
          acc[3] += src[(s2 + 3) * per_tile];
        }
        for (; s2 < p.SKW; ++s2) acc[0] += src[s2 * per_tile];
        const float sum = (acc[0] + acc[1]) + (acc[2] + acc[3]);
        if (csize == 1) {
          const int row = (item * p.RT + rto) * kBoxRows + rem / M;
          const int m = rem % M;
          if (row < p.N) {
            if (p.y_bf16)
              reinterpret_cast<__nv_bfloat16*>(p.Y)[size_t(m) * p.N + row] = __float2bfloat16_rn(sum);
            else
              reinterpret_cast<float*>(p.Y)[size_t(m) * p.N + row] = sum;
          }
        } else {
          part[size_t(li) * p.RT * per_tile + o] = sum;
        }
      }
    };

    // FAST path constants and the warp's activation fragments (constant over items)
    constexpr int kFBPW = FastShape<BITS>::kBPW;
    constexpr int kFSub = kFBPW * Geo::kSubUnits;                 // sub-units per warp and stage
    constexpr int kFNG = kFSub / Geo::kSubUnitsPerGroup;          // groups per warp and stage
    constexpr int kFFrag = BITS == 4 ? kFBPW * 4 : kFBPW * 2;     // 16-byte B fragments
    static_assert(Geo::kSubUnits * Geo::kWords == 4, "four code words per lane, row and box");
    uint4 breg[FAST ? kFFrag : 1];
    if constexpr (FAST) {
      const int kw0 = k_begin + sk * kFBPW * Geo::kBoxK;  // this warp's first k of the stage
#pragma unroll
      for (int bb = 0; bb < kFBPW; ++bb)
#pragma unroll
        for (int j = 0; j < Geo::kSubUnits; ++j) {
          const int su = bb * Geo::kSubUnits + j;
          const int q = su / Geo::kSubUnitsPerGroup;  // group of this warp
          const int jj = q % kJ;                      // its column slot in the sweep
          const int ksu = kw0 + bb * Geo::kBoxK + j * Geo::kUk;
          const uint32_t base = (col_jj == jj ? xrow[0] : zero_row) +
                                uint32_t((ksu - k_begin) / Geo::kUk * kChunksPerQuarter) * 64;
#pragma unroll
          for (int wi = 0; wi < Geo::kWords; wi += (BITS == 4 ? 1 : 2)) {
            const int f = BITS == 4 ? su * Geo::kWords + wi : (su * Geo::kWords + wi) / 2;
            breg[f] = (ksu < k_end) ? sld<uint4>(smem, base + (BITS == 4 ? wi : wi / 2) * 64)
                                    : make_uint4(0, 0, 0, 0);
          }
        }
    }

    int slot = 0;
    uint32_t phase = 0;
    int local_item = 0;
    for (int item = cid; item < p.items; item += ncl, ++local_item) {
      const int tile = item * p.RT + rt;
      const bool tile_ok = tile < p.row_tiles;
      float y[MT][4];
#pragma unroll
      for (int nt = 0; nt < MT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) y[nt][e] = 0.f;

      if constexpr (FAST) {
        // ---- one stage, fully unrolled
        if (!*abort_flag && !mbar_wait(&full[slot], phase)) *abort_flag = 1;
        const uint32_t stage_addr = p.off_ring + uint32_t(slot) * p.stage_bytes;
        const uint32_t meta_s = stage_addr + p.meta_offset + rt * meta_rt_bytes;
        const uint32_t meta_z = stage_addr + p.meta_offset + (p.RT + rt) * meta_rt_bytes;
        const int gw0 = sk * kFBPW * Geo::kBoxK / G;  // warp's first group, stage-relative
        if (tile_ok && !*abort_flag) {
          uint32_t wa[kFBPW][4], wb[kFBPW][4];
          const uint32_t box0 = stage_addr + uint32_t(rt * kBoxRows + g) * p.row_stride +
                                uint32_t(sk * kFBPW) * kBoxRowBytes + t * Geo::kQB;
#pragma unroll
          for (int bb = 0; bb < kFBPW; ++bb)
#pragma unroll
            for (int j = 0; j < Geo::kSubUnits; ++j) {
              uint32_t ta[Geo::kWords], tb[Geo::kWords];
              const uint32_t a = box0 + bb * kBoxRowBytes + j * Geo::kU;
              load_words<Geo::kWords>(smem, a, ta);
              load_words<Geo::kWords>(smem, a + 8 * p.row_stride, tb);
#pragma unroll
              for (int wi = 0; wi < Geo::kWords; ++wi) {
                wa[bb][j * Geo::kWords + wi] = ta[wi];
                wb[bb][j * Geo::kWords + wi] = tb[wi];
              }
            }
          float c[2][4];
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int e = 0; e < 4; ++e) c[h][e] = 0.f;
#pragma unroll
          for (int su = 0; su < kFSub; ++su) {
            const int bb = su / Geo::kSubUnits, j = su % Geo::kSubUnits;
            if constexpr (BITS == 4) {
#pragma unroll
              for (int wi = 0; wi < Geo::kWords; ++wi) {
                uint32_t ua[4], ub[4];
                unpack_u4(wa[bb][j * Geo::kWords + wi], ua);
                unpack_u4(wb[bb][j * Geo::kWords + wi], ub);
                const uint32_t a0[4] = {ua[0], ub[0], ua[1], ub[1]};
                const uint32_t a1[4] = {ua[2], ub[2], ua[3], ub[3]};
                const uint4 bv = breg[su * Geo::kWords + wi];
                const uint32_t b0[2] = {bv.x, bv.y};
                const uint32_t b1[2] = {bv.z, bv.w};
                mma_bf16_16816(c[0], a0, b0);
                mma_bf16_16816(c[1], a1, b1);
              }
            } else {
#pragma unroll
              for (int wi = 0; wi < Geo::kWords; wi += 2) {
                uint32_t ua0[2], ub0[2], ua1[2], ub1[2];
                unpack_u8(wa[bb][j * Geo::kWords + wi], ua0);
                unpack_u8(wb[bb][j * Geo::kWords + wi], ub0);
                unpack_u8(wa[bb][j * Geo::kWords + wi + 1], ua1);
                unpack_u8(wb[bb][j * Geo::kWords + wi + 1], ub1);
                const uint32_t a0[4] = {ua0[0], ub0[0], ua0[1], ub0[1]};
                const uint32_t a1[4] = {ua1[0], ub1[0], ua1[1], ub1[1]};
                const uint4 bv = breg[(su * Geo::kWords + wi) / 2];
                const uint32_t b0[2] = {bv.x, bv.y};
                const uint32_t b1[2] = {bv.z, bv.w};
                mma_bf16_16816(c[0], a0, b0);
                mma_bf16_16816(c[1], a1, b1);
              }
            }
            // end of a group, and of a sweep: epilogue over the sweep's groups
            if ((su + 1) % Geo::kSubUnitsPerGroup == 0) {
              const int q = (su + 1) / Geo::kSubUnitsPerGroup - 1;  // group just finished
              if ((q + 1) % kJ == 0 || q + 1 == kFNG) {
                const int s0 = q - q % kJ;                              // sweep's first group
                const int ngs = q - s0 + 1;                             // groups in the sweep
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int col = 2 * t + (e & 1);
                  const int jj = col / MEFF;
                  const int m = col % MEFF;
                  const int row = g + 8 * (e >> 1);
                  const int gls = gw0 + s0 + jj;                        // stage-relative group
                  if (jj < ngs && (k_begin + gls * G) < k_end) {
                    const uint32_t me = uint32_t(row * sg + gls) * 2;
                    const float sc = __half2float(sld<__half>(smem, meta_s + me));
                    const float z =
                        SYM ? float(1 << (BITS - 1)) : __half2float(sld<__half>(smem, meta_z + me));
                    const float bias = (BITS == 4 ? 128.f : 0.f) + z;
                    const float sxv = sld<float>(smem, sx_off + uint32_t(m * sx_stride + gls) * 4);
                    y[0][e] = fmaf(sc, fmaf(-bias, sxv, c[0][e] + c[1][e]), y[0][e]);
                  }
                  c[0][e] = 0.f;
                  c[1][e] = 0.f;
                }
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
        if (++slot == p.depth) {
          slot = 0;
          phase ^= 1;
        }
      } else
      for (int st = 0; st < p.stages_per_item; ++st) {
        if (!*abort_flag && !mbar_wait(&full[slot], phase)) *abort_flag = 1;
        const uint32_t stage_addr = p.off_ring + uint32_t(slot) * p.stage_bytes;  // offset in smem
        const int stage_k0 = k_begin + st * p.stage_k;
        const int g0 = stage_k0 / G;
        const uint32_t meta_s = stage_addr + p.meta_offset + rt * meta_rt_bytes;
        const uint32_t meta_z = stage_addr + p.meta_offset + (p.RT + rt) * meta_rt_bytes;
        if (tile_ok && !*abort_flag) {
          float c[2][MT][4];
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int nt = 0; nt < MT; ++nt)
#pragma unroll
              for (int e = 0; e < 4; ++e) c[h][nt][e] = 0.f;
          int sw_n = 0;    // groups accumulated in the current sweep
          int sw_gi = 0;   // global index of the sweep's first group
          // B base for the current group: this lane's row if its column
          // belongs to the group's slot of the sweep, else the zero row
          uint32_t bbase[MT];
#pragma unroll
          for (int nt = 0; nt < MT; ++nt) bbase[nt] = col_jj == 0 ? xrow[nt] : zero_row;

          // Epilogue of a sweep: y += s * (C - bias * Sx), in binary32.
          auto epilogue = [&]() {
#pragma unroll
            for (int nt = 0; nt < MT; ++nt)
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int col = 2 * t + (e & 1);
                const int jj = MT == 1 ? col / MEFF : 0;
                const int m = (MT == 1 ? col % MEFF : col) + 8 * nt;
                const int row = g + 8 * (e >> 1);
                if (jj < sw_n) {
                  const int gi = sw_gi + jj;
                  const uint32_t me = uint32_t(row * sg + gi - g0) * 2;
                  const float sc = __half2float(sld<__half>(smem, meta_s + me));
                  const float z =
                      SYM ? float(1 << (BITS - 1)) : __half2float(sld<__half>(smem, meta_z + me));
                  const float bias = (BITS == 4 ? 128.f : 0.f) + z;
                  const float sxv = sld<float>(smem, sx_off + uint32_t(m * sx_stride + gi - k_begin / G) * 4);
                  const float d = c[0][nt][e] + c[1][nt][e];
                  y[nt][e] = fmaf(sc, fmaf(-bias, sxv, d), y[nt][e]);
                }
                c[0][nt][e] = 0.f;
                c[1][nt][e] = 0.f;
              }
            sw_n = 0;
          };

          for (int bb = 0; bb < p.BPW; ++bb) {
            const int b = sk * p.BPW + bb;
            const int kb = stage_k0 + b * Geo::kBoxK;
            if (kb >= k_end) break;
            // this warp's 64-byte column block of the row tile (rows p.row_stride apart)
            const uint32_t box = stage_addr + uint32_t(rt * kBoxRows) * p.row_stride +
                                 uint32_t(b) * kBoxRowBytes;
#pragma unroll
            for (int j = 0; j < Geo::kSubUnits; ++j) {
              const int ksu = kb + j * Geo::kUk;
              if (ksu >= k_end) break;
              if (sw_n == 0 && ((ksu % G) == 0)) sw_gi = ksu / G;
              // codes of rows g and g+8, this lane's quarter of the sub-unit
              uint32_t wa[Geo::kWords], wb[Geo::kWords];
              const uint32_t ra = box + g * p.row_stride + j * Geo::kU + t * Geo::kQB;
              load_words<Geo::kWords>(smem, ra, wa);
              load_words<Geo::kWords>(smem, ra + 8 * p.row_stride, wb);
              const uint32_t chunk_off =
                  uint32_t((ksu - k_begin) / Geo::kUk * kChunksPerQuarter) * 64;
              if constexpr (BITS == 4) {
#pragma unroll
                for (int wi = 0; wi < Geo::kWords; ++wi) {
                  uint32_t ua[4], ub[4];
                  unpack_u4(wa[wi], ua);
                  unpack_u4(wb[wi], ub);
                  const uint32_t a0[4] = {ua[0], ub[0], ua[1], ub[1]};
                  const uint32_t a1[4] = {ua[2], ub[2], ua[3], ub[3]};
#pragma unroll
                  for (int nt = 0; nt < MT; ++nt) {
                    const uint4 bv = sld<uint4>(smem, bbase[nt] + chunk_off + wi * 64);
                    const uint32_t b0[2] = {bv.x, bv.y};
                    const uint32_t b1[2] = {bv.z, bv.w};
                    mma_bf16_16816(c[0][nt], a0, b0);
                    mma_bf16_16816(c[1][nt], a1, b1);
                  }
                }
              } else {
#pragma unroll
                for (int wi = 0; wi < Geo::kWords; wi += 2) {
                  uint32_t ua0[2], ub0[2], ua1[2], ub1[2];
                  unpack_u8(wa[wi], ua0);
                  unpack_u8(wb[wi], ub0);
                  unpack_u8(wa[wi + 1], ua1);
                  unpack_u8(wb[wi + 1], ub1);
                  const uint32_t a0[4] = {ua0[0], ub0[0], ua0[1], ub0[1]};
                  const uint32_t a1[4] = {ua1[0], ub1[0], ua1[1], ub1[1]};
#pragma unroll
                  for (int nt = 0; nt < MT; ++nt) {
                    const uint4 bv = sld<uint4>(smem, bbase[nt] + chunk_off + (wi / 2) * 64);
                    const uint32_t b0[2] = {bv.x, bv.y};
                    const uint32_t b1[2] = {bv.z, bv.w};
                    mma_bf16_16816(c[0][nt], a0, b0);
                    mma_bf16_16816(c[1][nt], a1, b1);
                  }
                }
              }
              if (((ksu + Geo::kUk) % G) == 0) {  // a group ends here
                ++sw_n;
                if (sw_n == kJ) epilogue();
#pragma unroll
                for (int nt = 0; nt < MT; ++nt)
                  bbase[nt] = col_jj == sw_n ? xrow[nt] : zero_row;
              }
            }
          }
          if (sw_n > 0) epilogue();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
        if (++slot == p.depth) {
          slot = 0;
          phase ^= 1;
        }
      }

      // Lanes whose columns hold the same activation row add their sums
      // (the sweep put different groups of one row in different columns).
      if constexpr (MT == 1 && MEFF < 8) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (MEFF == 1 && (e & 1)) continue;
          float v = y[0][e] + (MEFF == 1 ? y[0][e | 1] : 0.f);
          if (MEFF <= 2) v += __shfl_xor_sync(0xffffffffu, v, 1);
          v += __shfl_xor_sync(0xffffffffu, v, 2);
          y[0][e] = v;
        }
      }

      // Add the SKW partial sums of each row tile in a fixed order.  With
      // red_bufs == 0 every item has its own slot and the sums are added
      // once after the last item (no barrier between items, so warps drift
      // apart and overlap their phases); otherwise the partials go to one of
      // red_bufs buffers with one or two barriers per item.
      const int rslot = p.red_bufs == 0 ? local_item : (p.red_bufs == 2 ? (local_item & 1) : 0);
      float* rb = red + rslot * red_stride;
#pragma unroll
      for (int nt = 0; nt < MT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int col = 2 * t + (e & 1);
          int m;
          bool owner;
          if (MT == 1 && MEFF < 8) {
            m = col % MEFF;
            // after the shuffles, lanes t < MEFF/2 (t = 0 when MEFF <= 2) hold the totals
            owner = (MEFF == 1) ? (t == 0 && (e & 1) == 0) : (t < MEFF / 2);
          } else {
            m = col + 8 * nt;
            owner = true;
          }
          const int r = g + 8 * (e >> 1);
          if (owner && m < M) rb[(rt * p.SKW + sk) * per_tile + r * M + m] = y[nt][e];
        }
      if (p.red_bufs != 0) {
        named_barrier_sync(1, nthr);
        reduce_item(rb, item, local_item, tid);
        if (p.red_bufs == 1) named_barrier_sync(1, nthr);  // buffer reused by the next item
      }
    }
    if (p.red_bufs == 0) {
      named_barrier_sync(1, nthr);
      for (int li = 0; li < local_item; ++li)
        reduce_item(red + li * red_stride, cid + li * ncl, li, tid);
    }
    // the last item's reducers must finish before the cluster exchange
    named_barrier_sync(1, nthr);
  }

  if (csize > 1) {
    // Add the ranks' partial sums in rank order through distributed shared
    // memory; rank r writes the outputs with index % csize == r.
    cluster_sync();
    if (warp < kNumConsumerWarps) {
      const int per_item = p.RT * kBoxRows * p.M;
      int n_local = 0;
      for (int item = cid; item < p.items; item += ncl) ++n_local;
      const uint32_t part_local = smem_addr(smem + p.off_part);
      for (int e = int(threadIdx.x) * int(csize) + int(rank); e < n_local * per_item;
           e += kNumConsumerWarps * 32 * int(csize)) {
        float sum = 0.f;
        for (uint32_t r2 = 0; r2 < csize; ++r2)
          sum += ld_dsmem_f32(map_to_rank(part_local + uint32_t(e) * 4, r2));
        const int li = e / per_item, rem = e % per_item;
        const int item = cid + li * ncl;
        const int rto = rem / (kBoxRows * p.M), rr = rem % (kBoxRows * p.M);
        const int row = (item * p.RT + rto) * kBoxRows + rr / p.M;
        const int m = rr % p.M;
        if (row < p.N) {
          if (p.y_bf16)
            reinterpret_cast<__nv_bfloat16*>(p.Y)[size_t(m) * p.N + row] = __float2bfloat16_rn(sum);
          else
            reinterpret_cast<float*>(p.Y)[size_t(m) * p.N + row] = sum;
        }
      }
    }
    cluster_sync();
  }
}

}  // namespace gemv
}  // namespace wq
