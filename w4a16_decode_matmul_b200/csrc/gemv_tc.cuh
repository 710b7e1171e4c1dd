// gemv_tc.cuh -- the small-batch matmul Y = X * What^T (M <= 2) for 4- or
// 8-bit codes in groups of 128 with K = 4096 on the fifth-generation tensor
// cores: "vLLM 量化与推测解码" section 2 (W4A16: packed INT4 weights and their
// group scales are unpacked and scaled on chip, multiplied with 16-bit
// activations and accumulated in higher precision), section 3 ("FP8、INT8 与
// INT4": INT8 codes with an explicit scale and zero) and "量化" (llminference
// s08) section 实现 (each group's block is dequantized inside the
// accumulation).
//
// Why the tensor-memory path: a warp-level mma.sync m16n8k16 costs about
// eight warp instructions on sm_100 (measured with the k-sliced kernel: 73.6
// instructions per 1 KB of 4-bit codes with the MMAs replaced by an empty
// asm, 141.7 with them).  Here a warp's share of an MMA is one tcgen05.st of
// its unpacked codes, and one thread issues the MMAs for the CTA.  The
// issuing thread is then the limit: measured on B200, a tcgen05.mma
// (M = 128, K = 16, A in tensor memory) takes ~49 cycles at any N up to 64,
// ~63 with ALU-heavy warps on the same sub-partition, and it consumes 2048
// weights -- 1 KB of 4-bit codes, 2 KB of 8-bit codes.  For 4-bit codes that
// ceiling is near the HBM rate (the k-sliced kernel stays the default); for
// 8-bit codes it is far above it.
//
// Mapping.  A tile is 8 rows of W; K = 4096 is two halves j of 16 groups.
// The MMA's 128 rows (tensor-memory lanes) are the 8 rows x 16 groups of a
// half: lane 32 q + 4 r + i holds row r, group 16 j + 4 q + i, its 128 codes
// as exact bfloat16 values (64 columns): 128 + u for 4-bit codes (one LOP3
// per two), u for 8-bit codes (through binary32 2^23 + u).  The MMA's
// N = 16 MT columns are the same 16 groups of the activations, column
// MT s + m holding token m's 128 values of group 16 j + s in the codes'
// column order.  D[lane][MT s + m] is then the dot product of the lane's
// codes with group s of token m; the lane keeps only the diagonal s = its
// own group.  The other 15/16 of the products are waste, but the tensor
// pipe runs such an MMA (128 x 16 x 16) in a few cycles and is otherwise
// idle.
//
// Per tile and half: warp (q, j) copies its 8 rows x 4 groups with cp.async
// into its own ring (each copy instruction reads 64 contiguous bytes of a
// row, 16 per lane, for the lanes that own them; lane L's chunk c sits at
// 16-byte unit 32 c + (L ^ (c & 3)) of the slot, conflict-free for the
// copies and the reads), unpacks them into 64 columns and stores them to
// one of two A slots of its half in tensor memory; one thread (warp 8)
// issues the half's eight MMAs (M = 128, N = 16 MT, K = 16) into one of two
// accumulators and commits them to one barrier, which frees the A slot and
// hands the accumulator to the epilogue; a tile later the warp reads its
// four groups' accumulators back, applies y = s (C - b Sx) in binary32 (b
// = 128 + z for 4-bit codes, z for 8-bit; Sx the group's activation sum),
// adds its four groups by shuffles and leaves the row's partial sum in
// shared memory.  At the end each output is the sum of the 8 warps'
// partials in a fixed order (deterministic).  A warp arrives at "A written"
// only after reading the accumulator the MMAs are about to reuse, so that
// barrier also frees the accumulator.
//
// The weight-side set-up (the first DEPTH stages of every warp, the
// {s, b} table, tensor-memory allocation) happens before the wait on the
// previous grid when the weights are static; a CTA takes at most half an
// SM's shared memory, so the next launch's CTA streams its first stages
// while this one finishes (its allocation of the 512 tensor-memory columns
// waits until this CTA frees them).  Every wait is bounded in time; a
// timeout records WQ_ERR_TIMEOUT, the roles stop, copies and MMAs are
// drained and tensor memory is freed.
#pragma once

#include "common.cuh"
#include "unpack.cuh"
#include "gemv_ld.cuh"
#include "gemm2.cuh"

namespace wq {
namespace tc {

constexpr int kK = 4096;
constexpr int kGroups = kK / 128;       // 32
constexpr int kTileRows = 8;
constexpr int kDqWarps = 8;             // warp w: lane quarter w % 4, half w / 4
constexpr int kMmaWarp = kDqWarps;      // allocation and MMA issue
constexpr int kThreads = (kDqWarps + 1) * 32;
constexpr int kACols = 64;              // one group of bfloat16 pairs per lane
constexpr int kASlots = 2;              // A stages per half (tiles in flight)
constexpr int kSzStride = 36;           // {s, z} entries per row (32-bit loads conflict-free)
constexpr int kTmemCols = 512;          // A: 2 halves x 2 slots x 64; accumulators after
constexpr int kMaxMT = 2;

// Bytes of a row, of a group, and of one warp's stage (32 lanes x a group).
__host__ __device__ constexpr int row_bytes(int bits) { return kK * bits / 8; }
__host__ __device__ constexpr int group_bytes(int bits) { return 128 * bits / 8; }
__host__ __device__ constexpr int slot_bytes(int bits) { return 32 * group_bytes(bits); }

// shared-memory head: mbarriers, then the tensor-memory base and abort flag
constexpr int kBarAFull = 0;            // [2 halves][2 slots] A written (one arrival per quarter)
constexpr int kBarDone = 4;             // [2 halves][2 slots] the MMAs finished (commit)
constexpr int kBarMmaDone = 8;          // every MMA of the CTA finished
constexpr int kTmemSlot = 128;
constexpr int kAbortSlot = 132;
constexpr int kHeadBytes = 1024;

struct Params {
  const __nv_bfloat16* X;  // [M][4096]
  void* Y;                 // [M][N]
  const uint8_t* codes;    // [N][4096 * bits / 8]
  const __half* scales;    // [N][32]
  const __half* zeros;     // [N][32] or null (symmetric)
  int M, N, tiles, y_bf16, pdl;
  uint32_t off_b;     // activation operand: [2 halves][2 boxes of 64 k][16 MT rows][128 bytes]
  uint32_t off_sz;    // [rows of the CTA][36] {scale, zero} binary16 pairs
  uint32_t off_part;  // [tiles of the CTA][2 halves][4 quarters][8 rows][MT] binary32
  uint32_t off_ring;  // [8 warps][DEPTH][slot_bytes]
};

// Bytes of the activation operand and of one of its 64-k boxes.
__host__ __device__ constexpr int box_bytes(int mt) { return 16 * mt * 128; }
__host__ __device__ constexpr int b_bytes(int mt) { return 4 * box_bytes(mt); }

// tcgen05.ld of 4 or 8 consecutive binary32 columns of this warp's lanes.
__device__ __forceinline__ void tmem_ld4(uint32_t taddr, float (&v)[4]) {
  uint32_t r[4];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// Four 8-bit codes -> (u0, u1), (u2, u3) as exact bfloat16 pairs: binary32
// 2^23 + u by byte permutes, minus 2^23 two at a time (exact), then one
// packing conversion per pair (exact: u < 256).
__device__ __forceinline__ void unpack_u8_pairs(uint32_t w, uint32_t (&r)[2]) {
  asm("{\n\t"
      ".reg .b32 f0, f1, f2, f3;\n\t"
      ".reg .b64 p, q;\n\t"
      "prmt.b32 f0, %2, %3, 0x7650;\n\t"
      "prmt.b32 f1, %2, %3, 0x7651;\n\t"
      "prmt.b32 f2, %2, %3, 0x7652;\n\t"
      "prmt.b32 f3, %2, %3, 0x7653;\n\t"
      "mov.b64 p, {f0, f1};\n\t"
      "mov.b64 q, {f2, f3};\n\t"
      "sub.rn.f32x2 p, p, %4;\n\t"
      "sub.rn.f32x2 q, q, %4;\n\t"
      "mov.b64 {f0, f1}, p;\n\t"
      "mov.b64 {f2, f3}, q;\n\t"
      "cvt.rn.bf16x2.f32 %0, f1, f0;\n\t"
      "cvt.rn.bf16x2.f32 %1, f3, f2;\n\t"
      "}"
      : "=r"(r[0]), "=r"(r[1])
      : "r"(w), "r"(0x4B000000u), "l"(0x4B0000004B000000ull));
}

// The eight MMAs of one half and tile (M = 128, N from idesc, K = 16 each):
// A columns a, a + 8, ..., a + 56 in tensor memory, B descriptors bd[k];
// the first overwrites the accumulator d, the rest add to it.
__device__ __forceinline__ void mma8(uint32_t d, uint32_t a, const uint64_t (&bd)[8],
                                     uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b32 ak;\n\t"
      "setp.ne.b32 p, %11, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %10, p;\n\t"
      "setp.eq.b32 p, %11, 0;\n\t"
      "add.u32 ak, %1, 8;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ak], %3, %10, p;\n\t"
      "add.u32 ak, %1, 16;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ak], %4, %10, p;\n\t"
      "add.u32 ak, %1, 24;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ak], %5, %10, p;\n\t"
      "add.u32 ak, %1, 32;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ak], %6, %10, p;\n\t"
      "add.u32 ak, %1, 40;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ak], %7, %10, p;\n\t"
      "add.u32 ak, %1, 48;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ak], %8, %10, p;\n\t"
      "add.u32 ak, %1, 56;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [ak], %9, %10, p;\n\t}" ::"r"(d),
      "r"(a), "l"(bd[0]), "l"(bd[1]), "l"(bd[2]), "l"(bd[3]), "l"(bd[4]), "l"(bd[5]),
      "l"(bd[6]), "l"(bd[7]), "r"(idesc), "r"(0u)
      : "memory");
}

// Four 16-byte copies: dst[g] + off <- src + STRIDE g.
template <int STRIDE>
__device__ __forceinline__ void copy4(const uint32_t (&dst)[4], uint32_t off, const uint8_t* src) {
  asm volatile(
      "cp.async.cg.shared.global [%0], [%4], 16;\n\t"
      "cp.async.cg.shared.global [%1], [%4+%5], 16;\n\t"
      "cp.async.cg.shared.global [%2], [%4+%6], 16;\n\t"
      "cp.async.cg.shared.global [%3], [%4+%7], 16;" ::"r"(dst[0] + off),
      "r"(dst[1] + off), "r"(dst[2] + off), "r"(dst[3] + off), "l"(src), "n"(STRIDE),
      "n"(2 * STRIDE), "n"(3 * STRIDE)
      : "memory");
}

// RAGGED: N is not a multiple of 8, so the CTA's last tile may hold rows past
// N (read as zeros through bounds-checked copies; their sums are not stored).
template <int BITS, bool SYM, int MT, int DEPTH, bool RAGGED = true>
__global__ void __launch_bounds__(kThreads, 2) gemv_tc_kernel(const Params p) {
  static_assert(BITS == 4 || BITS == 8, "bits");
  static_assert(MT >= 1 && MT <= kMaxMT, "tokens");
  constexpr int kN = 16 * MT;                 // MMA N: 16 groups x MT tokens
  constexpr int kBox = box_bytes(MT);
  constexpr uint32_t kIdesc = gemm2::instr_desc(kN);
  constexpr int kDCol0 = 2 * kASlots * kACols;  // accumulators after the A stages
  static_assert(kDCol0 + 4 * kN <= kTmemCols, "tensor memory");
  constexpr int kRowBytes = row_bytes(BITS);
  constexpr int kGroupBytes = group_bytes(BITS);
  constexpr int kSlotBytes = slot_bytes(BITS);
  constexpr int kChunks = kGroupBytes / 16;   // 16-byte chunks of a lane's group
  constexpr int kCpg = kChunks / 4;           // copy instructions per group of a row
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kTmemSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kAbortSlot);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tb0 = int(int64_t(blockIdx.x) * p.tiles / gridDim.x);
  const int tb1 = int(int64_t(blockIdx.x + 1) * p.tiles / gridDim.x);
  const int ntiles = tb1 - tb0;
  uint32_t* sz = reinterpret_cast<uint32_t*>(smem + p.off_sz);
  float* part = reinterpret_cast<float*>(smem + p.off_part);

  if (threadIdx.x == 0) {
    for (int b = 0; b < 4; ++b) {
      mbar_init(&bars[kBarAFull + b], 4);
      mbar_init(&bars[kBarDone + b], 1);
    }
    mbar_init(&bars[kBarMmaDone], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }

  // dequantize warps: lane quarter q, half j; lane (r, i4) = tile row r,
  // group 16 j + 4 q + i4
  const int q = warp & 3, j = (warp >> 2) & 1;
  const int r = lane >> 2, i4 = lane & 3;
  // copy instruction c of lane (r, i4) brings bytes 64 c + 16 i4 of row r's
  // four groups: chunk 4 (c % kCpg) + i4 of group g = c / kCpg, for reader
  // lane 4 r + g, to unit 32 chunk + ((4 r + g) ^ i4)
  const uint8_t* src = p.codes + (size_t(tb0) * kTileRows + r) * kRowBytes +
                       16 * kGroupBytes * j + 4 * kGroupBytes * q + 16 * i4;
  const uint32_t ring = smem_addr(smem) + p.off_ring + uint32_t(warp * DEPTH * kSlotBytes);
  uint32_t dst[4];
#pragma unroll
  for (int g = 0; g < 4; ++g) dst[g] = ring + uint32_t(512 * i4 + 16 * (4 * r + (g ^ i4)));
  // tiles [0, nfull) of the CTA have every row < N; only the last may not
  const int nfull = tb1 * kTileRows > p.N ? ntiles - 1 : ntiles;
  int fetched = 0;
  auto fetch = [&](int slot) {
    const uint32_t so = uint32_t(slot * kSlotBytes);
    if (!RAGGED ? fetched < ntiles : fetched < nfull) {
#pragma unroll
      for (int h = 0; h < kCpg; ++h) copy4<64 * kCpg>(dst, so + uint32_t(2048 * h), src + 64 * h);
    } else if (RAGGED && fetched < ntiles) {
      const bool ok = (tb0 + fetched) * kTileRows + r < p.N;
#pragma unroll
      for (int c = 0; c < kChunks; ++c)
        ld::cp_async16(dst[c / kCpg] + so + uint32_t(2048 * (c % kCpg)),
                       ok ? src + 64 * c : p.codes, ok);
    }
    src += kTileRows * kRowBytes;  // never dereferenced past the CTA's last tile
    ++fetched;
    ld::cp_async_commit();
  };

  const int row_lo = tb0 * kTileRows;
  const int rows = min(p.N, tb1 * kTileRows) - row_lo;
  auto weight_setup = [&]() {
    if (warp < kDqWarps) {
#pragma unroll
      for (int s = 0; s < DEPTH; ++s) fetch(s);
    }
    // the row's {scale, zero} pairs as stored (binary16; zero 0 if symmetric)
    const int meta4 = rows * kGroups / 4;
    for (int i = int(threadIdx.x); i < meta4; i += kThreads) {
      const uint2 a = ld::ldg_stream64(p.scales + size_t(row_lo) * kGroups + 4 * size_t(i));
      const uint2 z = SYM ? make_uint2(0, 0)
                          : ld::ldg_stream64(p.zeros + size_t(row_lo) * kGroups + 4 * size_t(i));
      const int e = 4 * i, row = e / kGroups, gi = e - row * kGroups;
      uint32_t* d = sz + row * kSzStride + gi;
      d[0] = __byte_perm(a.x, z.x, 0x5410);
      d[1] = __byte_perm(a.x, z.x, 0x7632);
      d[2] = __byte_perm(a.y, z.y, 0x5410);
      d[3] = __byte_perm(a.y, z.y, 0x7632);
    }
  };
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(smem + kTmemSlot)),
                 "r"(uint32_t(kTmemCols))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (p.pdl) weight_setup();
  grid_dependents_launch();
  grid_dependency_wait();
  if (!p.pdl) weight_setup();

  // the activation operand B: for half h and 64-k box b, row n = MT s + m
  // holds token m's values of group 16 h + s in the codes' column order
  // (4-bit: x0, x4, x1, x5, x2, x6, x3, x7 per 8; 8-bit: k order), 128-byte
  // swizzled
  {
    uint8_t* bs = smem + p.off_b;
    for (int ci = int(threadIdx.x); ci < 4 * kN * 8; ci += kThreads) {
      const int c16 = ci & 7, n = (ci >> 3) % kN, hb = (ci >> 3) / kN;
      const int sg = n / MT, m = n - sg * MT;
      uint4 o = make_uint4(0, 0, 0, 0);
      if (m < p.M) {
        const uint4 v = *reinterpret_cast<const uint4*>(
            p.X + size_t(m) * kK + 2048 * (hb >> 1) + 128 * sg + 64 * (hb & 1) + 8 * c16);
        if (BITS == 4) {
          o.x = __byte_perm(v.x, v.z, 0x5410);
          o.y = __byte_perm(v.x, v.z, 0x7632);
          o.z = __byte_perm(v.y, v.w, 0x5410);
          o.w = __byte_perm(v.y, v.w, 0x7632);
        } else {
          o = v;
        }
      }
      *reinterpret_cast<uint4*>(bs + hb * kBox + n * 128 + ((c16 ^ (n & 7)) << 4)) = o;
    }
    gemm2::fence_async_shared();  // the tensor cores read B through the async proxy
  }
  // this lane's group sums, one per token: 16 values per lane, then the 8
  // lanes of the group (xor 4, 8, 16)
  float sx[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    float acc = 0.f;
    if (warp < kDqWarps && m < p.M) {
      const __nv_bfloat16* xg = p.X + size_t(m) * kK + 128 * (16 * j + 4 * q + i4) + 16 * r;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint4 v = *reinterpret_cast<const uint4*>(xg + 8 * h);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k)
          acc += __uint_as_float(w4[k] << 16) + __uint_as_float(w4[k] & 0xFFFF0000u);
      }
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 4);
    acc += __shfl_xor_sync(0xffffffffu, acc, 8);
    acc += __shfl_xor_sync(0xffffffffu, acc, 16);
    sx[m] = acc;
  }
  gemm2::tc_fence_before();
  __syncthreads();
  gemm2::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // Waits poll with test_wait, reading the time limit and the abort flag
  // every 64 polls; the dequantize warps (idle) sleep briefly between polls
  // so as to leave issue slots to the MMA thread of their sub-partition.
  auto wait = [&](int bar, uint32_t parity, bool idle) {
    if (mbar_test_wait(&bars[bar], parity)) return true;
    const unsigned long long start = global_timer_ns();
    for (uint32_t n = 1;; ++n) {
      if (idle) __nanosleep(32);
      if (mbar_test_wait(&bars[bar], parity)) return true;
      if ((n & 63u) == 0) {
        if (*abort_flag) return false;
        if (global_timer_ns() - start > kWaitLimitNs) {
          record_status(kStatusTimeout);
          *abort_flag = 1;
          return false;
        }
      }
    }
  };

  if (warp == kMmaWarp) {
    // ---------------------------------------------------------- MMA issue
    if (lane == 0) {
      // B never changes: both halves' eight descriptors, once (k step k: box
      // k / 4 of the half, 32 bytes further per step in it)
      uint64_t bd[2][8];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint64_t base = gemm2::umma_desc_sw128(smem_addr(smem + p.off_b) + uint32_t(2 * h * kBox));
#pragma unroll
        for (int k = 0; k < 8; ++k) bd[h][k] = base + uint64_t((k >> 2) * (kBox >> 4) + 2 * (k & 3));
      }
      bool stop = false;
      for (int e = 0; e < ntiles && !stop; ++e) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int sl = 2 * h + (e & 1);  // A slot, accumulator and barrier of this tile
          // the half's A is written (and the accumulator's previous use read)
          if (!wait(kBarAFull + sl, uint32_t(e >> 1) & 1u, false)) {
            stop = true;
            break;
          }
          gemm2::tc_fence_after();
          mma8(tmem_base + uint32_t(kDCol0 + sl * kN), tmem_base + uint32_t(sl * kACols), bd[h],
               kIdesc);
          gemm2::tc_commit(&bars[kBarDone + sl]);
        }
      }
      // every MMA of the CTA completes before tensor memory is freed
      gemm2::tc_commit(&bars[kBarMmaDone]);
      mbar_wait(&bars[kBarMmaDone], 0);
    }
  }
  else {
    // ---------------------------------------------------------- dequantize
    const uint32_t lane_bits = uint32_t(32 * q) << 16;
    const uint32_t a_tmem = tmem_base + lane_bits + uint32_t(2 * j * kACols);
    const uint32_t d_tmem = tmem_base + lane_bits + uint32_t(kDCol0 + 2 * j * kN + 4 * MT * q);
    // chunk c of this lane's group: 16-byte unit 32 c + (lane ^ (c & 3))
    uint32_t rd[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) rd[c] = ring + uint32_t(16 * (lane ^ c));
    // the {s, z} entry of this lane's row and group in the first tile;
    // successive tiles are 8 rows further
    uint32_t sz_a = smem_addr(sz + r * kSzStride + 16 * j + 4 * q + i4);
    // b = 128 + z (4-bit codes enter as 128 + u) or z (8-bit codes, as u);
    // symmetric codes have z = 2^(bits - 1)
    constexpr float kCodeBias = (BITS == 4 ? 128.f : 0.f) + (SYM ? float(1 << (BITS - 1)) : 0.f);
    uint32_t part_a = smem_addr(part + (j * 4 + q) * kTileRows * MT + r * MT);
    constexpr uint32_t kPartTileBytes = uint32_t(8 * kTileRows * MT * 4);
    bool stop = false;
    for (int it0 = 0; it0 <= ntiles && !stop; it0 += DEPTH) {
#pragma unroll
      for (int slot = 0; slot < DEPTH; ++slot) {
        const int it = it0 + slot;
        if (it > ntiles) break;
        if (it < ntiles) {
          // tile it: codes -> A slot it % 2 of this half, once the MMAs of
          // tile it - 2 have finished with it
          ld::cp_async_wait<DEPTH - 1>();
          __syncwarp();
          const uint32_t so = uint32_t(slot * kSlotBytes);
          const int sl = 2 * j + (it & 1);
          const uint32_t a_cols = a_tmem + uint32_t((it & 1) * kACols);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            // 32 columns: 8 words of 4-bit codes or 16 words of 8-bit codes
            constexpr int kHalfChunks = kChunks / 2;
            uint4 cw[kHalfChunks];
#pragma unroll
            for (int c = 0; c < kHalfChunks; ++c) {
              const int ch = kHalfChunks * hh + c;
              cw[c] = lds128(rd[ch & 3] + so + uint32_t(512 * ch));
            }
            uint32_t a[32];
#pragma unroll
            for (int c = 0; c < kHalfChunks; ++c) {
              const uint32_t w4[4] = {cw[c].x, cw[c].y, cw[c].z, cw[c].w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                if constexpr (BITS == 4) {
                  uint32_t u[4];
                  unpack_u4(w4[e], u);  // (128 + u_t, 128 + u_{t+4}), t = 0..3
#pragma unroll
                  for (int t = 0; t < 4; ++t) a[16 * c + 4 * e + t] = u[t];
                } else {
                  uint32_t u[2];
                  unpack_u8_pairs(w4[e], u);  // (u0, u1), (u2, u3)
#pragma unroll
                  for (int t = 0; t < 2; ++t) a[8 * c + 2 * e + t] = u[t];
                }
              }
            }
            if (hh == 0) {
              // warp-uniform: the tensor-memory stores below are .aligned
              const bool ok = wait(kBarDone + sl, (uint32_t(it >> 1) & 1u) ^ 1u, true);
              if (!__all_sync(0xffffffffu, ok)) {
                stop = true;
                break;
              }
              gemm2::tc_fence_after();
            }
            gemm2::tmem_st32(a_cols + uint32_t(32 * hh), a);
          }
          if (stop) break;
          gemm2::tmem_wait_st();
          gemm2::tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[kBarAFull + sl]);
          // every lane's reads of the slot are done: refill it DEPTH tiles on
          fetch(slot);
        }
        if (it > 0) {
          // tile it - 1: this lane's group sums -> the row's partial sum
          const int e = it - 1, sl = 2 * j + (e & 1);
          const bool ok = wait(kBarDone + sl, uint32_t(e >> 1) & 1u, true);
          if (!__all_sync(0xffffffffu, ok)) {
            stop = true;
            break;
          }
          gemm2::tc_fence_after();
          float dv[4 * MT];
          if constexpr (MT == 1)
            tmem_ld4(d_tmem + uint32_t((e & 1) * kN), dv);
          else
            tmem_ld8(d_tmem + uint32_t((e & 1) * kN), dv);
          gemm2::tmem_wait_ld();
          // the accumulator is read; "A written" of tile it + 1 tells the
          // MMA thread so (after this warp's fence and arrival there)
          const uint32_t eb = lds32(sz_a);
          sz_a += uint32_t(kTileRows * kSzStride * 4);
          const float sc = __half2float(__ushort_as_half(static_cast<unsigned short>(eb & 0xFFFFu)));
          const float bias =
              SYM ? kCodeBias
                  : kCodeBias + __half2float(__ushort_as_half(static_cast<unsigned short>(eb >> 16)));
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const float c01 = (i4 & 1) ? dv[MT + m] : dv[m];
            const float c23 = (i4 & 1) ? dv[3 * MT + m] : dv[2 * MT + m];
            float y = sc * fmaf(-bias, sx[m], (i4 & 2) ? c23 : c01);
            y += __shfl_xor_sync(0xffffffffu, y, 1);
            y += __shfl_xor_sync(0xffffffffu, y, 2);
            if (i4 == 0) sts32(part_a + uint32_t(4 * m), y);
          }
          part_a += kPartTileBytes;
        }
      }
    }
    ld::cp_async_wait<0>();
  }

  gemm2::tc_fence_before();
  __syncthreads();
  // Y[m][row] = the 8 warps' partial sums in order (half, quarter)
  if (!*abort_flag) {
    constexpr int kPerTile = kTileRows * MT;
    const int outs = ntiles * kPerTile;
    for (int o = int(threadIdx.x); o < outs; o += kThreads) {
      const int tl = o / kPerTile, rem = o - tl * kPerTile;
      const float* s = part + tl * 8 * kPerTile + rem;
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) v += s[w * kPerTile];
      const int row = (tb0 + tl) * kTileRows + rem / MT, m = rem % MT;
      if (m < p.M && row < p.N) {
        if (p.y_bf16)
          static_cast<__nv_bfloat16*>(p.Y)[size_t(m) * p.N + row] = __float2bfloat16_rn(v);
        else
          static_cast<float*>(p.Y)[size_t(m) * p.N + row] = v;
      }
    }
  }
  // tensor memory is freed by the warp that allocated it, after every MMA
  // and every reader is done
  if (warp == kMmaWarp) {
    gemm2::tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(uint32_t(kTmemCols))
                 : "memory");
  }
}

}  // namespace tc
}  // namespace wq
