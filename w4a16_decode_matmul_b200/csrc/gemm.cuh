// gemm.cuh -- prefill-sized matmul Y = X * What^T (M > 32) on the fifth
// generation tensor cores: "vLLM 量化与推测解码" section 2 (W4A16: weights kept
// packed in memory with group scales, dequantized on chip, multiplied with
// 16-bit activations and accumulated in higher precision) with the prefill
// observation of "量化" (llminference s08) section 实现 (large batches are
// bound by the multiply, so the weights are dequantized in on-chip tiles that
// feed the tensor cores).
//
// Exactness.  A dequantized weight s (q - z) needs up to 16 significant bits
// and is not a bfloat16 in general, so the tensor cores multiply the exact
// integers (q - z) (bfloat16 holds them exactly) and each group's partial sum
// D_g = sum over the group of x (q - z) is scaled in binary32:
// y = sum_g s_g D_g.  Products are exact; D_g accumulates in binary32.
//
// One CTA computes a 128 x 128 tile of Y over all of K, per stage of 64 k
// (a ring of 4 stages, each holding the activation tile, the codes and the
// dequantized weight tile):
//   warp 0      TMA: the 128 x 64 activation tile (128-byte swizzle) and the
//               128 rows x 64 codes; once per tile the tile's scales/zeros;
//   warps 2-9   dequantize: half a row of codes per thread (the two halves of
//               a row on adjacent lanes) -> 32 bfloat16
//               (q - z) written in the same swizzled K-major layout, then an
//               async-proxy fence and an arrive;
//   warp 1      one thread issues tcgen05.mma (M=128, N=128, K=16, bfloat16
//               in, binary32 accumulator in tensor memory) per 16 k; a
//               group's MMAs accumulate into one of three 128-column TMEM
//               buffers, whose commit hands it to the epilogue;
//   warps 10-17 epilogue: each thread owns one row and 64 columns; per group
//               it reads D_g from TMEM, releases the buffer and adds s_g D_g
//               into the running sum S, kept in TMEM next to the group
//               buffers (binary32); at the end it writes S to Y.
// Every wait is bounded in time; a timeout records WQ_ERR_TIMEOUT, the other
// roles skip their work, issued copies and MMAs are drained and TMEM is freed.
#pragma once

#include "common.cuh"

namespace wq {
namespace gemm {

constexpr int kBM = 128;                 // rows of X per tile (MMA M)
constexpr int kBN = 128;                 // rows of W per tile (MMA N)
constexpr int kBK = 64;                  // k per stage (one 128-byte swizzled row)
constexpr int kStages = 4;
constexpr int kDequantWarp0 = 2, kNumDequantWarps = 8;
constexpr int kEpilogueWarp0 = 10, kNumEpilogueWarps = 8;
constexpr int kThreads = (kEpilogueWarp0 + kNumEpilogueWarps) * 32;  // 576
constexpr int kTileBytes = kBM * kBK * 2;                              // 16 KB (A and B alike)
constexpr int kAccBufs = 3;                   // group accumulators in TMEM
constexpr int kTmemCols = (kAccBufs + 1) * kBN;  // 512: the buffers and the running sum
constexpr int kSumCol = kAccBufs * kBN;        // first TMEM column of the running sum S
constexpr int kColsPerThread = kBN / 2;                                // epilogue: 64 columns

// mbarrier slots in the first KB of shared memory
constexpr int kBarLdFull = 0;            // [kStages] activation + codes tile landed
constexpr int kBarEmpty = 4;             // [kStages] MMAs of the stage done (commit)
constexpr int kBarBFull = 8;             // [kStages] dequantized tile written
constexpr int kBarAccFull = 12;          // [kAccBufs] group accumulator ready (commit)
constexpr int kBarAccEmpty = 15;         // [kAccBufs] group accumulator read
constexpr int kBarMeta = 18;             // tile's scales / zeros landed
constexpr int kBarMmaDone = 19;          // every MMA of the CTA finished
constexpr int kTmemSlot = 576;           // byte offset of the TMEM base address
constexpr int kAbortSlot = 580;          // byte offset of the abort flag

struct Params {
  __nv_bfloat16* Y_bf16;    // one of Y_bf16 / Y_f32 is set
  float* Y_f32;
  int M, N, K, ngroups;
  int tiles_m;
  uint32_t codes_stage_bytes;  // kBN * kBK * bits / 8
  uint32_t meta_bytes;         // kBN * ngroups * 2 (one metadata tensor)
  uint32_t off_a, off_b, off_codes, off_meta_s, off_meta_z, off_stab;
};

// UMMA shared-memory descriptor of a K-major tile in the canonical 128-byte
// swizzled layout (8-row atoms of 1024 bytes): start address, leading byte
// offset 1 (unused for swizzled K-major), stride byte offset 1024 (between
// 8-row groups), descriptor version 1, layout type 2 (128-byte swizzle).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_addr_bytes) {
  return uint64_t((smem_addr_bytes >> 4) & 0x3FFFu) | (uint64_t(1) << 16) |
         (uint64_t(1024 >> 4) << 32) | (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// Instruction descriptor: binary32 accumulator, bfloat16 A and B, both
// K-major, N = 128, M = 128.
constexpr uint32_t kInstrDesc = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(kBN >> 3) << 17) |
                                (uint32_t(kBM >> 4) << 24);

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}"
      :
      : "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(kInstrDesc), "r"(accumulate), "r"(0u)
      : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void fence_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 32 consecutive binary32 columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32};"
      ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])),
      "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])),
      "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
      "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
      "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])),
      "r"(__float_as_uint(v[17])), "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])),
      "r"(__float_as_uint(v[20])), "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])),
      "r"(__float_as_uint(v[23])), "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])),
      "r"(__float_as_uint(v[26])), "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])),
      "r"(__float_as_uint(v[29])), "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Eight 4-bit codes of a word (k = 0..7) -> four bfloat16 pairs in k order,
// each code minus zc: (u0-zc, u1-zc), (u2-zc, u3-zc), (u4-zc, u5-zc),
// (u6-zc, u7-zc).  zc2 holds 128 + zc in both halves (the codes enter as
// 128 + u, exact).
__device__ __forceinline__ void dequant_u4_kord(uint32_t w, uint32_t zc2, uint32_t (&o)[4]) {
  constexpr uint32_t kMask = 0x000F000Fu, kMagic = 0x43004300u;
  uint32_t t[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(r) : "r"(w >> (4 * i)), "r"(kMask), "r"(kMagic));
    t[i] = r;  // (128 + u_i, 128 + u_{i+4})
  }
  o[0] = bf16x2_sub(__byte_perm(t[0], t[1], 0x5410), zc2);
  o[1] = bf16x2_sub(__byte_perm(t[2], t[3], 0x5410), zc2);
  o[2] = bf16x2_sub(__byte_perm(t[0], t[1], 0x7632), zc2);
  o[3] = bf16x2_sub(__byte_perm(t[2], t[3], 0x7632), zc2);
}

// Four 8-bit codes -> two bfloat16 pairs (u0 - zc, u1 - zc), (u2 - zc, u3 - zc):
// 2^23 + u in binary32 minus 2^23 + zc is exact, and so is the conversion
// of the integer (|u - zc| < 256) to bfloat16.
__device__ __forceinline__ void dequant_u8_kord(uint32_t w, float zc, uint32_t (&o)[2]) {
  float f[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    f[i] = __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7650 | i)) - (8388608.0f + zc);
  const __nv_bfloat162 p0 = __floats2bfloat162_rn(f[0], f[1]);
  const __nv_bfloat162 p1 = __floats2bfloat162_rn(f[2], f[3]);
  o[0] = *reinterpret_cast<const uint32_t*>(&p0);
  o[1] = *reinterpret_cast<const uint32_t*>(&p1);
}

template <int BITS, bool SYM, int G>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_codes,
                const __grid_constant__ CUtensorMap tm_scales,
                const __grid_constant__ CUtensorMap tm_zeros, const Params p) {
  static_assert(G % kBK == 0, "a group spans whole stages");
  constexpr int kKbPerGroup = G / kBK;
  constexpr int kCodesRowBytes = kBK * BITS / 8;  // 32 | 64

  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kTmemSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kAbortSlot);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tm = int(blockIdx.x) % p.tiles_m;
  const int tn = int(blockIdx.x) / p.tiles_m;
  const int m0 = tm * kBM, n0 = tn * kBN;
  const int nkb = p.K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars[kBarLdFull + s], 1);
      mbar_init(&bars[kBarEmpty + s], 1);
      mbar_init(&bars[kBarBFull + s], kNumDequantWarps);
    }
    for (int b = 0; b < kAccBufs; ++b) {
      mbar_init(&bars[kBarAccFull + b], 1);
      mbar_init(&bars[kBarAccEmpty + b], kNumEpilogueWarps);
    }
    mbar_init(&bars[kBarMeta], 1);
    mbar_init(&bars[kBarMmaDone], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    // the whole warp allocates the two group buffers in tensor memory
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(smem + kTmemSlot)),
                 "r"(uint32_t(kTmemCols))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  auto wait = [&](int bar, uint32_t parity) {
    if (mbar_test_wait(&bars[bar], parity)) return true;  // completed: no flag read
    if (*abort_flag) return false;
    if (!mbar_wait(&bars[bar], parity)) {
      *abort_flag = 1;
      return false;
    }
    return true;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tm_x);
      prefetch_tensormap(&tm_codes);
      prefetch_tensormap(&tm_scales);
      if (!SYM) prefetch_tensormap(&tm_zeros);
      const uint64_t keep = l2_policy_evict_last();   // X and W tiles are read by many CTAs
      mbar_arrive_expect_tx(&bars[kBarMeta], p.meta_bytes * (SYM ? 1u : 2u));
      tma_load_2d(smem + p.off_meta_s, &tm_scales, &bars[kBarMeta], 0, n0, keep);
      if (!SYM) tma_load_2d(smem + p.off_meta_z, &tm_zeros, &bars[kBarMeta], 0, n0, keep);
      int issued = 0;
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % kStages;
        const uint32_t ph = uint32_t(kb / kStages) & 1u;
        if (!wait(kBarEmpty + s, ph ^ 1u)) break;
        mbar_arrive_expect_tx(&bars[kBarLdFull + s], uint32_t(kTileBytes) + p.codes_stage_bytes);
        tma_load_2d(smem + p.off_a + s * kTileBytes, &tm_x, &bars[kBarLdFull + s], kb * kBK, m0,
                    keep);
        tma_load_2d(smem + p.off_codes + s * p.codes_stage_bytes, &tm_codes,
                    &bars[kBarLdFull + s], kb * kCodesRowBytes, n0, keep);
        ++issued;
      }
      // every issued copy lands before the CTA can finish
      mbar_wait(&bars[kBarMeta], 0);
      for (int j = max(0, issued - kStages); j < issued; ++j)
        mbar_wait(&bars[kBarLdFull + j % kStages], uint32_t(j / kStages) & 1u);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t a0 = smem_addr(smem + p.off_a);
      const uint32_t b0 = smem_addr(smem + p.off_b);
      int kb = 0;
      for (int gi = 0; gi < p.ngroups && !*abort_flag; ++gi) {
        const int buf = gi % kAccBufs;
        if (!wait(kBarAccEmpty + buf, (uint32_t(gi / kAccBufs) & 1u) ^ 1u)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + uint32_t(buf * kBN);
        bool ok = true;
        for (int j = 0; j < kKbPerGroup; ++j, ++kb) {
          const int s = kb % kStages;
          const uint32_t ph = uint32_t(kb / kStages) & 1u;
          if (!wait(kBarLdFull + s, ph) || !wait(kBarBFull + s, ph)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t da = umma_desc_sw128(a0 + uint32_t(s) * kTileBytes);
          const uint64_t db = umma_desc_sw128(b0 + uint32_t(s) * kTileBytes);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)  // 32 bytes of each swizzled row per step
            tc_mma(d, da + uint64_t(2 * k), db + uint64_t(2 * k), (j > 0 || k > 0) ? 1u : 0u);
          tc_commit(&bars[kBarEmpty + s]);
        }
        if (!ok) break;
        tc_commit(&bars[kBarAccFull + buf]);
      }
      // all MMAs of this CTA complete before TMEM is freed
      tc_commit(&bars[kBarMmaDone]);
      mbar_wait(&bars[kBarMmaDone], 0);
    }
  } else if (warp < kEpilogueWarp0) {
    // ------------------------------------------------------------ dequantize
    // Two lanes per row, side by side: a warp's code reads are contiguous and
    // the swizzled tile writes stay free of bank conflicts.
    const int dt = threadIdx.x - kDequantWarp0 * 32;  // 0..255
    const int r = dt >> 1;                            // row of the W tile
    const int part = dt & 1;                          // 16-byte chunks 4*part .. 4*part+3
    const bool have_meta = wait(kBarMeta, 0);
    const __half* zrow = reinterpret_cast<const __half*>(smem + p.off_meta_z) + r * p.ngroups;
    int zc_group = -1;  // the zero point is read once per group
    float zc = float(1 << (BITS - 1));
    for (int kb = 0; kb < nkb && have_meta; ++kb) {
      const int s = kb % kStages;
      const uint32_t ph = uint32_t(kb / kStages) & 1u;
      // codes landed, and the previous MMAs of this slot are done with B
      if (!wait(kBarLdFull + s, ph) || !wait(kBarEmpty + s, ph ^ 1u)) break;
      const int gi = kb / kKbPerGroup;
      if (!SYM && gi != zc_group) {
        zc = __half2float(zrow[gi]);
        zc_group = gi;
      }
      const uint8_t* crow = smem + p.off_codes + s * p.codes_stage_bytes + r * kCodesRowBytes;
      uint8_t* brow = smem + p.off_b + s * kTileBytes + r * 128;
      if constexpr (BITS == 4) {
        const __nv_bfloat162 zz = __floats2bfloat162_rn(128.f + zc, 128.f + zc);
        const uint32_t zc2 = *reinterpret_cast<const uint32_t*>(&zz);
        const uint4 c = *reinterpret_cast<const uint4*>(crow + 16 * part);
        const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {  // word j: k = 8j .. 8j + 7 of this half = chunk 4*part + j
          uint32_t o[4];
          dequant_u4_kord(w[j], zc2, o);
          const int ch = 4 * part + j;
          *reinterpret_cast<uint4*>(brow + ((ch ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {  // 8 bytes of codes -> 16-byte chunk 4*part + j
          const int ch = 4 * part + j;
          const uint2 c = *reinterpret_cast<const uint2*>(crow + 8 * ch);
          uint32_t o0[2], o1[2];
          dequant_u8_kord(c.x, zc, o0);
          dequant_u8_kord(c.y, zc, o1);
          *reinterpret_cast<uint4*>(brow + ((ch ^ (r & 7)) << 4)) = make_uint4(o0[0], o0[1], o1[0], o1[1]);
        }
      }
      fence_async_shared();  // the tensor cores read B through the async proxy
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarBFull + s]);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int e = warp - kEpilogueWarp0;             // 0..7
    const int quarter = warp & 3;                    // TMEM lanes 32*quarter ..
    const int half = e >> 2;                         // columns 64*half ..
    const int row = 32 * quarter + lane;             // row of the Y tile
    const int etid = e * 32 + lane;                  // 0..255
    float* stab = reinterpret_cast<float*>(smem + p.off_stab);  // [group][128 columns]
    const bool have_meta = wait(kBarMeta, 0);
    if (have_meta) {
      const __half* ms = reinterpret_cast<const __half*>(smem + p.off_meta_s);
      for (int i = etid; i < p.ngroups * kBN; i += kNumEpilogueWarps * 32) {
        const int gi = i / kBN, n = i - gi * kBN;
        stab[i] = __half2float(ms[n * p.ngroups + gi]);
      }
    }
    named_barrier_sync(2, kNumEpilogueWarps * 32);
    const uint32_t lanes = uint32_t(32 * quarter) << 16;
    const uint32_t sum_addr = tmem_base + lanes + uint32_t(kSumCol + half * kColsPerThread);
    int done = 0;
    for (int gi = 0; gi < p.ngroups && have_meta; ++gi) {
      const int buf = gi % kAccBufs;
      if (!wait(kBarAccFull + buf, uint32_t(gi / kAccBufs) & 1u)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + lanes + uint32_t(buf * kBN + half * kColsPerThread);
      const float* sg = stab + gi * kBN + half * kColsPerThread;
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // 32 columns at a time: S += s_g D_g
        float d[32], acc[32];
        tmem_ld32(taddr + 32 * h, d);
        if (gi > 0) tmem_ld32(sum_addr + 32 * h, acc);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const float4 sv = *reinterpret_cast<const float4*>(sg + 32 * h + j);
          acc[j + 0] = fmaf(sv.x, d[j + 0], gi > 0 ? acc[j + 0] : 0.f);
          acc[j + 1] = fmaf(sv.y, d[j + 1], gi > 0 ? acc[j + 1] : 0.f);
          acc[j + 2] = fmaf(sv.z, d[j + 2], gi > 0 ? acc[j + 2] : 0.f);
          acc[j + 3] = fmaf(sv.w, d[j + 3], gi > 0 ? acc[j + 3] : 0.f);
        }
        tmem_st32(sum_addr + 32 * h, acc);
      }
      tmem_wait_st();
      // D_g is read: the MMA warp may overwrite this buffer
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarAccEmpty + buf]);
      done = gi + 1;
    }
    const int m = m0 + row;
    const int nb = n0 + half * kColsPerThread;
    if (!*abort_flag && done == p.ngroups) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float acc[32];
        tmem_ld32(sum_addr + 32 * h, acc);
        tmem_wait_ld();
        const int nh = nb + 32 * h;
        if (m < p.M) {
          if (p.Y_f32 != nullptr) {
            float* yrow = p.Y_f32 + size_t(m) * p.N + nh;
            if (nh + 32 <= p.N && (p.N % 4) == 0) {
#pragma unroll
              for (int j = 0; j < 32; j += 4)
                *reinterpret_cast<float4*>(yrow + j) =
                    make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (nh + j < p.N) yrow[j] = acc[j];
            }
          } else {
            __nv_bfloat16* yrow = p.Y_bf16 + size_t(m) * p.N + nh;
            if (nh + 32 <= p.N && (p.N % 8) == 0) {
#pragma unroll
              for (int j = 0; j < 32; j += 8) {
                uint4 o;
                __nv_bfloat162 h0 = __floats2bfloat162_rn(acc[j], acc[j + 1]);
                __nv_bfloat162 h1 = __floats2bfloat162_rn(acc[j + 2], acc[j + 3]);
                __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[j + 4], acc[j + 5]);
                __nv_bfloat162 h3 = __floats2bfloat162_rn(acc[j + 6], acc[j + 7]);
                o.x = *reinterpret_cast<uint32_t*>(&h0);
                o.y = *reinterpret_cast<uint32_t*>(&h1);
                o.z = *reinterpret_cast<uint32_t*>(&h2);
                o.w = *reinterpret_cast<uint32_t*>(&h3);
                *reinterpret_cast<uint4*>(yrow + j) = o;
              }
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (nh + j < p.N) yrow[j] = __float2bfloat16_rn(acc[j]);
            }
          }
        }
      }
    }
  }

  // TMEM is freed by the warp that allocated it, after every reader and
  // every MMA is done
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(uint32_t(kTmemCols))
                 : "memory");
  }
}

}  // namespace gemm
}  // namespace wq
