// gemv_sk.cuh -- balanced small-batch matmul Y = X * What^T for M <= 8:
// "vLLM 量化与推测解码" section 2 (W4A16: packed codes and group scales are
// unpacked and scaled on chip, multiplied with 16-bit activations and
// accumulated in higher precision; the full-precision weights never exist in
// memory) and "量化" (llminference s08) section 实现 (each group's block is
// dequantized inside the accumulation).
//
// Decode time is the packed bytes over the bandwidth ("量化" section 问题), so
// the kernel streams every byte of codes and metadata exactly once and gives
// every SM the same number of bytes:
//
//   * Work unit = (row tile of 16 rows, slice of 128 bytes of each row).
//     Whole tiles are dealt round-robin to the CTAs (one per SM), so each
//     wave of CTAs reads one contiguous stretch of the codes; the tiles left
//     over after the last full wave are cut into equal ranges of units, one
//     per CTA.  A tile whose slices fall into two or more ranges is summed
//     across CTAs: the CTAs that hold its later slices publish their partial
//     sums in a workspace (a flag per CTA) once all their copies have
//     landed, and the CTA that holds slice 0 adds them in CTA order (fixed,
//     so the result is deterministic) and writes Y.
//   * A stage is up to 16 consecutive slices of one tile (never crossing a
//     multiple of 16 slices).  One producer lane loads it with one 3-D TMA box
//     (128 bytes x 16 rows x 16 slices, 128-byte swizzle) for the codes and
//     one 3-D box per metadata tensor (8 groups x 16 rows x blocks); stages
//     that are cut short at a range end take one box per slice / per 8-group
//     block, so no byte of another CTA's range is read.  The ring holds
//     nearly all of a CTA's stages, so the copies are issued at once.
//   * 16 consumer warps; warp w owns slice w of every 16-slice block.  Lanes
//     read their codes with ldmatrix from the swizzled slice (bank-conflict
//     free): lane (g, t) gets word t of every 16-byte chunk of rows g and
//     g + 8, the A-fragment layout of mma.sync m16n8k16.
//   * Tensor-core operands are binary16.  Codes become the exact small
//     integers u (asymmetric; the zero is applied in the epilogue) or u - 8 /
//     u - 128 (symmetric) with one shift, four LOP3s and four packed FMA-pipe
//     ops per word of eight 4-bit codes.  The activations of each group are
//     scaled by 2^sigma (sigma per activation row and group, putting the
//     group's largest magnitude in [2^14, 2^15)) and rounded to binary16:
//     exact for every element within 2^32 of that largest magnitude
//     (bfloat16 has 8 significant bits); smaller elements are rounded to the
//     binary16 grid (absolute error below 2^-40 of the group's largest
//     magnitude).  Products are exact in binary32 and accumulate in binary32.
//   * The B operand puts kJ = 8 / MEFF consecutive groups of MEFF activation
//     rows in its 8 columns (column = group slot * MEFF + row), so one
//     accumulator collects a whole sweep of groups before one binary32
//     epilogue y += s * (2^-sigma C - z Sx) (symmetric: y += s 2^-sigma C),
//     Sx being the group's sum of the rounded activations at their own
//     scale.
//   * With programmatic dependent launch the weights stream in before the
//     previous kernel of the stream has finished; activations, outputs and
//     the workspace are touched only after griddepcontrol.wait.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "unpack.cuh"

namespace wq {
namespace sk {

constexpr int kWarps = 16;
constexpr int kThreads = (kWarps + 1) * 32;
constexpr int kRows = 16;                                    // rows per tile
constexpr int kSliceBytes = 128;                             // bytes of a row per unit
constexpr int kSlicesPerStage = 16;                          // one per consumer warp
constexpr int kSliceSmem = kRows * kSliceBytes;              // 2 KB
constexpr int kCodesStage = kSlicesPerStage * kSliceSmem;    // 32 KB
constexpr int kBlockGroups = 8;                              // metadata block: 8 groups x 16 rows
constexpr int kBlockBytes = kRows * kBlockGroups * 2;        // 256 B
constexpr int kWsRowsMax = kRows * 8;                        // workspace floats per CTA (M <= 8)
constexpr int kWsCtasMax = 1024;                             // CTAs the workspace has room for
constexpr int kMaxDepth = 32;
constexpr int kMaxM = 8;

struct Params {
  const __nv_bfloat16* X;   // [M][K]
  void* Y;                  // [M][N]
  float* ws_part;           // [ctas][kWsRowsMax] partial sums of split tiles
  unsigned int* ws_flag;    // [ctas] 1 = partial published; reset to 0 by its reader
  int M, N, K, ngroups;
  int tiles;                // ceil(N / 16)
  int nk;                   // slices per tile = K * bits / 8 / 128
  int ctas;                 // grid size
  int waves;                // whole tiles per CTA, dealt round-robin: tiles / ctas
  int tail_tiles;           // tiles left after the waves: tiles % ctas
  int split;                // 1: the tail is cut into equal unit ranges; 0: whole tail tiles
  int pdl;                  // launched as a programmatic dependent (weights may stream early)
  int depth;                // ring stages
  int red_mode;             // 0: one partial slot per local tile, reduced at the end; 2: two
  int box_slices;           // slices of the whole-stage codes box: min(16, nk)
  int box_blocks;           // 8-group blocks of the whole-stage metadata box
  int y_bf16;
  uint32_t stage_bytes;     // codes, scale blocks, zero blocks
  uint32_t off_ring, off_x, off_sx, off_red;
  uint32_t x_stride;        // bytes per staged activation row
  // Test hooks of the timeout path (set only through an internal export):
  // the CTA that does not publish its split-tile flag (-1: none), and the
  // limit of the wait for published flags, in nanoseconds.  That wait comes
  // after every copy and product of the waiting CTA has completed, so giving
  // up there leaves nothing in flight.
  int test_skip_publish;
  unsigned long long flag_wait_ns;
};

struct Stage {
  int tile, s0, s1;  // slices [s0, s1) of row tile `tile`
};

// Absolute unit (tile * nk + slice) where CTA c's share of the tail starts;
// c = ctas gives the end of the tail.
__host__ __device__ __forceinline__ long long tail_begin(int c, const Params& p) {
  const long long base = (long long)p.waves * p.ctas * p.nk;
  if (p.split) return base + (long long)c * ((long long)p.tail_tiles * p.nk) / p.ctas;
  return base + (long long)(c < p.tail_tiles ? c : p.tail_tiles) * p.nk;
}

// Walk over a run of units, one stage at a time: up to the next multiple of
// 16 slices, the end of the tile, or the end of the run.  32-bit state.
struct Walk {
  int tile, s, left;  // current tile and slice, units left in the run

  __host__ __device__ __forceinline__ Walk(int tile_, int s_, int left_)
      : tile(tile_), s(s_), left(left_) {}

  __host__ __device__ __forceinline__ bool done() const { return left <= 0; }

  __host__ __device__ __forceinline__ Stage next(int nk) {
    Stage st;
    st.tile = tile;
    st.s0 = s;
    int lim = (s & ~(kSlicesPerStage - 1)) + kSlicesPerStage;
    if (lim > nk) lim = nk;
    st.s1 = lim - s <= left ? lim : s + left;
    left -= st.s1 - s;
    s = st.s1;
    if (s == nk) {
      ++tile;
      s = 0;
    }
    return st;
  }
};

// Every stage of CTA c in order: its whole tiles c, c + ctas, ..., then its
// share of the tail.  fn(stage, last stage of a tile in this CTA).
template <typename Fn>
__host__ __device__ __forceinline__ void for_each_stage(int c, const Params& p, Fn&& fn) {
  for (int w = 0; w < p.waves; ++w) {
    Walk wk(c + w * p.ctas, 0, p.nk);
    while (!wk.done()) {
      const Stage st = wk.next(p.nk);
      fn(st, wk.done());
    }
  }
  const long long tb = tail_begin(c, p), te = tail_begin(c + 1, p);
  if (te > tb) {
    Walk wk(int(tb / p.nk), int(tb % p.nk), int(te - tb));
    while (!wk.done()) {
      const Stage st = wk.next(p.nk);
      fn(st, st.s1 == p.nk || wk.done());
    }
  }
}

// Wait until *flag == 1; false (and the status word set to WQ_ERR_TIMEOUT)
// after limit_ns of wall time.
__device__ __forceinline__ bool wait_flag_for(const unsigned int* flag,
                                              unsigned long long limit_ns) {
  if (ld_acquire_gpu(flag) == 1u) return true;
  const unsigned long long start = global_timer_ns();
  while (true) {
    if (ld_acquire_gpu(flag) == 1u) return true;
    if (global_timer_ns() - start > limit_ns) {
      record_status(kStatusTimeout);
      return false;
    }
  }
}

template <int BITS, int MEFF>
struct Shape {
  static constexpr int kSliceK = kSliceBytes * 8 / BITS;   // k per slice: 256 | 128
  static constexpr int kChunkK = 16 * 8 / BITS;            // k per 16-byte chunk: 32 | 16
  static constexpr int kJ = 8 / MEFF;                      // groups per sweep
};

// x * 2^e in binary32 through two exact power-of-two factors (e may lie
// outside the normal exponent range).
__device__ __forceinline__ float scale_pow2(float x, int e) {
  const int e1 = e / 2, e2 = e - e1;
  return x * __int_as_float((e1 + 127) << 23) * __int_as_float((e2 + 127) << 23);
}

template <int BITS, bool SYM, int G, int MEFF, bool RESIDENT>
__global__ void __launch_bounds__(kThreads, 1)
    gemv_sk_kernel(const __grid_constant__ CUtensorMap tm_codes16,
                   const __grid_constant__ CUtensorMap tm_codes1,
                   const __grid_constant__ CUtensorMap tm_s16,
                   const __grid_constant__ CUtensorMap tm_s1,
                   const __grid_constant__ CUtensorMap tm_z16,
                   const __grid_constant__ CUtensorMap tm_z1, const Params params) {
  using Sh = Shape<BITS, MEFF>;
  constexpr int kGPS = Sh::kSliceK / G;            // groups per slice
  constexpr int kCPG = G / Sh::kChunkK;            // chunks per group
  constexpr int kJ = Sh::kJ;
  constexpr int kSweepChunks = kCPG * kJ;          // chunks per sweep (may exceed 8)
  constexpr int kMetaBlocks = kSlicesPerStage * kGPS / kBlockGroups;  // per metadata tensor
  constexpr int kZC = SYM ? (1 << (BITS - 1)) : 0;  // zero folded into the operand
  static_assert(kGPS >= 1 && kCPG >= 1 && kMetaBlocks >= 1, "slice geometry");
  using Frag = typename std::conditional<BITS == 4, uint4, uint2>::type;

  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kMaxDepth;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 512);
  // The parameters are copied to shared memory once: later reads (some only
  // at the end of the kernel) then never wait on the constant cache.
  static_assert(sizeof(Params) % 4 == 0 && sizeof(Params) <= 1024 - 640, "params copy");
  if (threadIdx.x < sizeof(Params) / 4)
    reinterpret_cast<uint32_t*>(smem + 640)[threadIdx.x] =
        reinterpret_cast<const uint32_t*>(&params)[threadIdx.x];
  const Params& p = *reinterpret_cast<const Params*>(smem + 640);  // valid after the barrier

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cta = int(blockIdx.x);
  const int nk = params.nk;

  if (threadIdx.x == 0) {
    for (int i = 0; i < params.depth; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // Every CTA is resident: kernels launched after this one may be scheduled
  // (they wait for this grid before touching its outputs).
  grid_dependents_launch();

  if (warp == kWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tm_codes16);
      prefetch_tensormap(&tm_codes1);
      prefetch_tensormap(&tm_s16);
      prefetch_tensormap(&tm_s1);
      if (!SYM) {
        prefetch_tensormap(&tm_z16);
        prefetch_tensormap(&tm_z1);
      }
      const uint64_t policy = l2_policy_evict_first();
      int issued = 0, slot = 0;
      uint32_t phase = 0;
      bool stop = false;
      for_each_stage(cta, p, [&](const Stage& st, bool) {
        if (stop) return;
        if (*abort_flag || !mbar_wait_idle(&empty[slot], phase ^ 1u)) {
          *abort_flag = 1;
          stop = true;
          return;
        }
        uint8_t* stage = smem + p.off_ring + size_t(slot) * p.stage_bytes;
        uint8_t* ms = stage + kCodesStage;
        uint8_t* mz = ms + kMetaBlocks * kBlockBytes;
        const int a16 = st.s0 & ~(kSlicesPerStage - 1);
        // one box for the whole block of 16 slices when the stage is exactly
        // that block (or its part inside the tile: the rest lies past the
        // tensor's extent and is filled with zeros, not read)
        const bool whole = st.s0 == a16 && st.s1 == min(a16 + kSlicesPerStage, nk);
        const int base_blk = a16 * kGPS / kBlockGroups;
        const int b_lo = st.s0 * kGPS / kBlockGroups;
        const int b_hi = (st.s1 * kGPS + kBlockGroups - 1) / kBlockGroups;
        // the transaction count is the box size, zero-filled parts included
        const uint32_t codes_bytes =
            uint32_t(whole ? p.box_slices : st.s1 - st.s0) * kSliceSmem;
        const uint32_t meta_bytes = uint32_t(whole ? p.box_blocks : b_hi - b_lo) * kBlockBytes;
        mbar_arrive_expect_tx(&full[slot], codes_bytes + meta_bytes * (SYM ? 1u : 2u));
        const int row0 = st.tile * kRows;
        if (whole) {
          tma_load_3d(stage, &tm_codes16, &full[slot], 0, row0, a16, policy);
          tma_load_3d(ms, &tm_s16, &full[slot], 0, row0, base_blk, policy);
          if (!SYM) tma_load_3d(mz, &tm_z16, &full[slot], 0, row0, base_blk, policy);
        } else {
          for (int s = st.s0; s < st.s1; ++s)
            tma_load_3d(stage + (s - a16) * kSliceSmem, &tm_codes1, &full[slot], 0, row0, s,
                        policy);
          for (int b = b_lo; b < b_hi; ++b) {
            tma_load_3d(ms + (b - base_blk) * kBlockBytes, &tm_s1, &full[slot], 0, row0, b,
                        policy);
            if (!SYM)
              tma_load_3d(mz + (b - base_blk) * kBlockBytes, &tm_z1, &full[slot], 0, row0, b,
                          policy);
          }
        }
        ++issued;
        if (++slot == p.depth) {
          slot = 0;
          phase ^= 1u;
        }
      });
      // Every issued copy must land before the CTA exits (the consumers
      // have waited for them unless they gave up after a timeout).
      for (int j = max(0, issued - p.depth); j < issued; ++j)
        mbar_wait_idle(&full[j % p.depth], uint32_t(j / p.depth) & 1u);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int tid = threadIdx.x;
  constexpr int nthr = kWarps * 32;
  const int M = p.M;
  const int g = lane >> 2, t = lane & 3;
  const uint32_t smem_base = smem_addr(smem);
  // per (activation row, group): {2^-sigma, scaled-back sum of the group}
  float2* gsc = reinterpret_cast<float2*>(smem + p.off_sx);

  // activations, outputs and the workspace belong to the previous kernel
  // until it has finished
  grid_dependency_wait();

  // Stage X in one pass.  Each thread takes a block of 8 activations; the
  // G/8 threads of a group find the group's largest magnitude (exponent e)
  // by shuffles, scale by 2^sigma with sigma = 14 - e, round to binary16 and
  // store the block permuted to match the code pairs (4-bit: x0 x4 x1 x5 x2
  // x6 x3 x7; 8-bit: x0 x2 x1 x3 x4 x6 x5 x7).  Per (row, group) the pair
  // {2^-sigma, sum of the rounded values times 2^-sigma} goes to gsc for the
  // epilogue.  Shuffles add in a fixed order.
  {
    const int nq = p.K / 8;
    const int total = M * nq;
    for (int base = warp * 32; base < total; base += nthr) {
      const int idx = base + lane;
      const bool valid = idx < total;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (valid) v = *reinterpret_cast<const uint4*>(p.X + size_t(idx) * 8);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      float f[8];
      float mx = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 t2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[j]));
        f[2 * j] = t2.x;
        f[2 * j + 1] = t2.y;
        mx = fmaxf(mx, fmaxf(fabsf(t2.x), fabsf(t2.y)));
      }
#pragma unroll
      for (int off = 1; off < G / 8; off <<= 1)
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const unsigned int mb = __float_as_uint(mx);
      const int sg = mb == 0u ? 0 : 14 - (int((mb >> 23) & 0xffu) - 127);
      uint32_t hp[4];
      float part = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __half2 h = __floats2half2_rn(scale_pow2(f[2 * j], sg), scale_pow2(f[2 * j + 1], sg));
        const float2 back = __half22float2(h);
        part += back.x + back.y;
        hp[j] = *reinterpret_cast<const uint32_t*>(&h);
      }
#pragma unroll
      for (int off = 1; off < G / 8; off <<= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
      if (valid) {
        const int m = idx / nq;
        const int b = idx - m * nq;
        uint4 o;
        if (BITS == 4) {
          o.x = __byte_perm(hp[0], hp[2], 0x5410);
          o.y = __byte_perm(hp[0], hp[2], 0x7632);
          o.z = __byte_perm(hp[1], hp[3], 0x5410);
          o.w = __byte_perm(hp[1], hp[3], 0x7632);
        } else {
          o.x = __byte_perm(hp[0], hp[1], 0x5410);
          o.y = __byte_perm(hp[0], hp[1], 0x7632);
          o.z = __byte_perm(hp[2], hp[3], 0x5410);
          o.w = __byte_perm(hp[2], hp[3], 0x7632);
        }
        *reinterpret_cast<uint4*>(smem + p.off_x + size_t(m) * p.x_stride + size_t(b) * 16) = o;
        if ((b % (G / 8)) == 0) {
          const float inv = scale_pow2(1.f, -sg);
          gsc[m * p.ngroups + b / (G / 8)] = make_float2(inv, part * inv);
        }
      }
    }
  }
  named_barrier_sync(1, nthr);

  // B fragments of slice s: chunk c of the slice, this lane's column.  The
  // column holds activation row m = g % MEFF for the group slot g / MEFF of
  // the sweep; the lane loads only if chunk c's group sits in that slot.
  const int col_jj = g / MEFF;
  const int col_m = g % MEFF;
  Frag bf[8];
  auto load_frags = [&](int s) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int q = c / kCPG;
      const bool active = (q % kJ) == col_jj && col_m < M && s < nk;
      if constexpr (BITS == 4) {
        const uint32_t a =
            p.off_x + uint32_t(col_m) * p.x_stride + uint32_t(32 * s + 4 * c + t) * 16;
        bf[c] = active ? *reinterpret_cast<const uint4*>(smem + a) : make_uint4(0, 0, 0, 0);
      } else {
        const uint32_t a =
            p.off_x + uint32_t(col_m) * p.x_stride + uint32_t(256 * s + 32 * c + 8 * t);
        bf[c] = active ? *reinterpret_cast<const uint2*>(smem + a) : make_uint2(0, 0);
      }
    }
  };

  // Epilogue addressing of this lane's four accumulator elements e: row g
  // (e < 2) or g + 8, column 2t + (e & 1) -> group slot jj and activation
  // row m.  A slice's groups lie in one 8-group metadata block, so sweep sw
  // adds sw * kJ to the group of every element.
  int e_jj[4], e_m[4];
  uint32_t e_off[4], e_sx[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int col = 2 * t + (e & 1);
    e_jj[e] = col / MEFF;
    e_m[e] = col % MEFF;
  }
  auto epilogue_setup = [&](int s, int a16) {
    const int gbase = s * kGPS;  // the slice's first group along K
    const int blk = gbase / kBlockGroups - a16 * kGPS / kBlockGroups;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int row = g + 8 * (e >> 1);
      e_off[e] = uint32_t(
          ((blk * kRows + row) * kBlockGroups + (gbase % kBlockGroups) + e_jj[e]) * 2);
      e_sx[e] = uint32_t(e_m[e] * p.ngroups + gbase + e_jj[e]);
    }
  };
  if constexpr (RESIDENT) {
    load_frags(warp);
    epilogue_setup(warp, 0);
  }

  // ldmatrix addressing: lane l names row (l % 8) + 8 * ((l / 8) % 2) and
  // chunk offset l / 16; the 128-byte swizzle stores logical chunk c of row r
  // at physical chunk c ^ (r % 8).
  const int lrow = (lane & 7) + ((lane >> 3) & 1) * 8;
  const int lsel = lane >> 4;
  const int lkey = lane & 7;

  float* red = reinterpret_cast<float*>(smem + p.off_red);
  const int per_tile = kRows * M;
  const long long tail_b = tail_begin(cta, p), tail_e = tail_begin(cta + 1, p);
  const int tail_first = int(tail_b / nk);

  // Local tile li: the waves' tiles, then the tail's.  Sum the 16 warps'
  // partials in warp order and finish it: write Y, publish it, or add the
  // published partials of later CTAs.  kind: 0 whole, 1 publish, 2 finish.
  auto tile_of = [&](int li) {
    return li < p.waves ? cta + li * p.ctas : tail_first + li - p.waves;
  };
  auto kind_of = [&](int li) {
    if (li < p.waves) return 0;
    const long long t0 = (long long)tile_of(li) * nk, t1 = t0 + nk;
    if (t0 < tail_b) return 1;
    return t1 <= tail_e ? 0 : 2;
  };
  auto warp_sum = [&](int li, int o) {
    const float* rb = red + size_t(p.red_mode == 2 ? (li & 1) : li) * kWarps * per_tile;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int w = 0; w < kWarps; w += 4) {
      acc[0] += rb[(w + 0) * per_tile + o];
      acc[1] += rb[(w + 1) * per_tile + o];
      acc[2] += rb[(w + 2) * per_tile + o];
      acc[3] += rb[(w + 3) * per_tile + o];
    }
    return (acc[0] + acc[1]) + (acc[2] + acc[3]);
  };
  auto write_y = [&](int tile, int o, float v) {
    const int row = tile * kRows + o / M;
    const int m = o % M;
    if (row < p.N) {
      if (p.y_bf16)
        reinterpret_cast<__nv_bfloat16*>(p.Y)[size_t(m) * p.N + row] = __float2bfloat16_rn(v);
      else
        reinterpret_cast<float*>(p.Y)[size_t(m) * p.N + row] = v;
    }
  };
  // Split tiles (kind 1 and 2), by warp 0.  Split tiles exist only with a
  // workspace (the plan deals whole tail tiles otherwise); refuse rather than
  // touch a missing one.
  auto reduce_split = [&](int li, int kind) {
    if (p.ws_flag == nullptr || p.ws_part == nullptr) {
      if (tid == 0) record_status(kStatusInternal);
      return;
    }
    if (warp != 0) return;
    const int tile = tile_of(li);
    if (kind == 1) {
      // publish: partial sums, then the flag (a release store after them)
      for (int o = lane; o < per_tile; o += 32)
        __stcg(p.ws_part + size_t(cta) * kWsRowsMax + o, warp_sum(li, o));
      __syncwarp();
      if (lane == 0 && cta != p.test_skip_publish) st_release_gpu(p.ws_flag + cta, 1u);
      return;
    }
    // finish: own partial plus those of the CTAs whose (non-empty) tail
    // ranges start inside this tile, added in CTA (= k) order.  Lanes wait
    // on the flags of 32 candidates at once; loads go four CTAs at a time.
    constexpr int kV = kWsRowsMax / 32;
    const long long t1 = (long long)(tile + 1) * nk;
    float v[kV];
#pragma unroll
    for (int j = 0; j < kV; ++j) {
      const int o = lane + 32 * j;
      v[j] = o < per_tile ? warp_sum(li, o) : 0.f;
    }
    for (int base = cta + 1; base < p.ctas; base += 32) {
      const int c2 = base + lane;
      const long long b2 = c2 < p.ctas ? tail_begin(c2, p) : t1;
      const bool in = b2 < t1;
      const bool pub = in && tail_begin(c2 + 1, p) > b2;
      const unsigned int in_mask = __ballot_sync(0xffffffffu, in);
      if (in_mask == 0u) break;
      const bool ok = !pub || (*abort_flag == 0 && wait_flag_for(p.ws_flag + c2, p.flag_wait_ns));
      if (__ballot_sync(0xffffffffu, !ok) != 0u) {
        *abort_flag = 1;
        break;
      }
      unsigned int pub_mask = __ballot_sync(0xffffffffu, pub);
      while (pub_mask != 0u) {
        int cc[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          cc[q] = pub_mask != 0u ? base + __ffs(pub_mask) - 1 : -1;
          pub_mask &= pub_mask - 1u;
        }
        float tmp[4][kV];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int j = 0; j < kV; ++j) {
            const int o = lane + 32 * j;
            tmp[q][j] = (cc[q] >= 0 && o < per_tile)
                            ? __ldcg(p.ws_part + size_t(cc[q]) * kWsRowsMax + o)
                            : 0.f;
          }
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int j = 0; j < kV; ++j)
            if (cc[q] >= 0) v[j] += tmp[q][j];
      }
      __syncwarp();
      if (pub) p.ws_flag[c2] = 0u;  // ready for the next call
      if (in_mask != 0xffffffffu) break;
    }
#pragma unroll
    for (int j = 0; j < kV; ++j) {
      const int o = lane + 32 * j;
      if (o < per_tile) write_y(tile, o, v[j]);
    }
  };

  float y[4] = {0.f, 0.f, 0.f, 0.f};
  int li = 0;
  int slot = 0;
  uint32_t phase = 0;
  for_each_stage(cta, p, [&](const Stage& st, bool tile_end) {
    bool ok = *abort_flag == 0;
    if (ok && !mbar_wait(&full[slot], phase)) {
      *abort_flag = 1;
      ok = false;
    }
    const int a16 = st.s0 & ~(kSlicesPerStage - 1);
    const int s = a16 + warp;
    if (ok && s >= st.s0 && s < st.s1) {
      if constexpr (!RESIDENT) {
        load_frags(s);
        epilogue_setup(s, a16);
      }
      const uint32_t stage = smem_base + p.off_ring + uint32_t(slot) * p.stage_bytes;
      const uint32_t row_addr =
          stage + uint32_t(warp) * kSliceSmem + uint32_t(lrow) * kSliceBytes;
      uint32_t wa[8], wb[8];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        ldmatrix_x4(row_addr + (uint32_t((2 * q + lsel) ^ lkey) << 4), wa[2 * q], wb[2 * q],
                    wa[2 * q + 1], wb[2 * q + 1]);
      const uint32_t ms = p.off_ring + uint32_t(slot) * p.stage_bytes + kCodesStage;
      const uint32_t mz = ms + kMetaBlocks * kBlockBytes;
      float acc[2][4];
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[h][e] = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        if constexpr (BITS == 4) {
          uint32_t ua[4], ub[4];
          unpack_u4_h<kZC>(wa[c], ua);
          unpack_u4_h<kZC>(wb[c], ub);
          const uint32_t a0[4] = {ua[0], ub[0], ua[1], ub[1]};
          const uint32_t a1[4] = {ua[2], ub[2], ua[3], ub[3]};
          const uint32_t b0[2] = {bf[c].x, bf[c].y};
          const uint32_t b1[2] = {bf[c].z, bf[c].w};
          mma_f16_16816(acc[0], a0, b0);
          mma_f16_16816(acc[1], a1, b1);
        } else {
          uint32_t ua[2], ub[2];
          unpack_u8_h<kZC>(wa[c], ua);
          unpack_u8_h<kZC>(wb[c], ub);
          const uint32_t a0[4] = {ua[0], ub[0], ua[1], ub[1]};
          const uint32_t b0[2] = {bf[c].x, bf[c].y};
          mma_f16_16816(acc[c & 1], a0, b0);
        }
        // end of a sweep: y += s * (C - z * Sx) (symmetric: s * C) for each
        // (row, group) column of the sweep
        if ((c + 1) % kSweepChunks == 0 || c == 7) {
          const int sw = c / kSweepChunks;
          const int ng = kJ < kGPS - sw * kJ ? kJ : kGPS - sw * kJ;  // groups in the sweep
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (e_jj[e] < ng && e_m[e] < M) {
              const uint32_t off = e_off[e] + uint32_t(sw * kJ * 2);
              const float sc = __half2float(*reinterpret_cast<const __half*>(smem + ms + off));
              const float cv = acc[0][e] + acc[1][e];
              const float2 gs = gsc[e_sx[e] + sw * kJ];
              if constexpr (SYM) {
                y[e] = fmaf(sc * gs.x, cv, y[e]);
              } else {
                const float z = __half2float(*reinterpret_cast<const __half*>(smem + mz + off));
                y[e] = fmaf(sc, fmaf(gs.x, cv, -z * gs.y), y[e]);
              }
            }
            acc[0][e] = 0.f;
            acc[1][e] = 0.f;
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
    if (++slot == p.depth) {
      slot = 0;
      phase ^= 1u;
    }

    if (tile_end) {
      // end of this CTA's part of the tile: combine the columns that hold the
      // same activation row, store the warp's partial sums
      if constexpr (MEFF < 8) {
        // lanes t < kUsedT hold columns (kUsedT = columns in use / 2)
        constexpr int kUsedT = ((kGPS < kJ ? kGPS : kJ) * MEFF + 1) / 2;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (MEFF == 1 && (e & 1)) continue;
          float v = y[e] + (MEFF == 1 ? y[e | 1] : 0.f);
          if (MEFF <= 2 && kUsedT > 1) v += __shfl_xor_sync(0xffffffffu, v, 1);
          if (kUsedT > 2) v += __shfl_xor_sync(0xffffffffu, v, 2);
          y[e] = v;
        }
      }
      float* rb = red + size_t(p.red_mode == 2 ? (li & 1) : li) * kWarps * per_tile +
                  size_t(warp) * per_tile;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int m = e_m[e];
        const bool owner = MEFF == 1 ? (t == 0 && (e & 1) == 0)
                                     : (MEFF == 2 ? t == 0 : (MEFF == 4 ? t < 2 : true));
        const int row = g + 8 * (e >> 1);
        if (owner && m < M) rb[row * M + m] = y[e];
        y[e] = 0.f;
      }
      if (p.red_mode == 2) {
        named_barrier_sync(1, nthr);
        const int kind = kind_of(li);
        if (kind == 0)
          for (int o = tid; o < per_tile; o += nthr) write_y(tile_of(li), o, warp_sum(li, o));
        else
          reduce_split(li, kind);
      }
      ++li;
    }
  });
  if (p.red_mode == 0 && li > 0) {
    // publish first (so no CTA waits on one that is itself waiting), then
    // every whole tile at once, then the finished split tile.  Only the
    // first tail tile (local index p.waves) can be published and only the
    // last local tile can be finished here.
    named_barrier_sync(1, nthr);
    if (li > p.waves && kind_of(p.waves) == 1) reduce_split(p.waves, 1);
    for (int it = tid; it < li * per_tile; it += nthr) {
      const int r = it / per_tile, o = it - r * per_tile;
      if (kind_of(r) == 0) write_y(tile_of(r), o, warp_sum(r, o));
    }
    if (kind_of(li - 1) == 2) reduce_split(li - 1, 2);
  }
}

}  // namespace sk
}  // namespace wq
