// gemm2.cuh -- prefill-sized matmul Y = X * What^T (M > 32) on the fifth
// generation tensor cores, weights as the tensor-memory operand: "vLLM 量化与
// 推测解码" section 2 (W4A16: packed weights and group scales dequantized on
// chip, multiplied with 16-bit activations, accumulated in higher precision)
// and "量化" (llminference s08) section 实现 (large batches are bound by the
// multiply: the weights are dequantized in on-chip tiles that feed the
// tensor cores).
//
// Exactness: the tensor cores multiply the exact integers (q - z) (bfloat16
// holds them) by the activations, one group at a time, into a binary32
// accumulator D_g; y = sum_g s_g D_g is formed in binary32.  Products are
// exact; only the binary32 sums round.
//
// Orientation (the transpose of Y is computed): the MMA's M dimension is 128
// rows of W, its N dimension 128 tokens (rows of X), K runs along the
// reduction.  A -- the dequantized weights -- lives in tensor memory,
// written there by the dequantize warps with tcgen05.st, so the weight tile
// never passes through shared memory; only the activation tile (B, from
// shared memory, loaded by TMA) and the packed codes do.  Per 16 k step the
// shared-memory traffic is the activation tile read by the MMA and written by
// TMA plus the codes, about half that of a kernel with both operands in
// shared memory.
//
// Persistent CTAs walk 128 x 128 tiles (token tile major, so that the CTAs of
// a wave share one activation tile and the whole weight matrix stays in L2).
// A load stage is 128 k: two activation boxes (128 tokens x 64 k, 128-byte
// swizzle, K-major) and the codes box (128 rows x 128 k of codes, 64- or
// 128-byte swizzle).  128 k is eight MMAs per barrier hand-off: with four
// (64 k) the issuing thread's per-stage wait and commit left the tensor pipe
// idle most of the time (measured on B200: ~240 cycles per 64-cycle MMA
// against ~90 with eight per stage).
// Warp roles:
//   warp 0      TMA producer (one thread);
//   warp 1      tensor-memory allocation; one thread issues tcgen05.mma
//               (M=128, N=128, K=16) per 16 k from A in tensor memory and B
//               in shared memory, into one of two 128-column group
//               accumulators, and commits it to the epilogue after a group;
//   warps 2-5   dequantize: one row of W per thread; a stage's codes ->
//               64 columns of bfloat16 pairs (q - z) -> tensor memory
//               (A stage s sits beside load stage s: both are freed by the
//               one commit of the stage's MMAs);
//   warps 6-13  epilogue: one row of W and 64 tokens per thread; per group
//               S += s_g D_g in registers (the row's eight scales of a
//               block in one 16-byte load); at the end of the tile S goes
//               out through shared memory by tensor stores, 16 tokens at a
//               time in two buffers per warp, so that the warps are free for
//               the next tile's groups while it is written (plain stores
//               where Y's pitch or shared memory does not allow it).
// Every wait is bounded in time; a timeout records WQ_ERR_TIMEOUT, sets the
// CTA's abort flag, the roles stop, issued copies and MMAs are drained and
// tensor memory is freed.
#pragma once

#include "common.cuh"
#include "gemm.cuh"

namespace wq {
namespace gemm2 {

using gemm::fence_async_shared;
using gemm::tc_commit;
using gemm::tc_fence_after;
using gemm::tc_fence_before;
using gemm::tmem_ld32;
using gemm::tmem_wait_ld;
using gemm::umma_desc_sw128;

constexpr int kBW = 128;     // rows of W per tile (MMA M)
constexpr int kBK = 128;     // k per load stage (8 MMAs of K = 16)
constexpr int kMaxLoadStages = 8;
constexpr int kMaxAStages = 8;  // barrier slots for A stages in tensor memory
constexpr int kDequantWarp0 = 2;
// threads of a CTA with DW dequantize and EW epilogue warps (and the
// producer and MMA warps)
__host__ __device__ constexpr int threads_for(int dw, int ew) { return (2 + dw + ew) * 32; }
constexpr int kTmemCols = 512;
constexpr int kAStageCols = kBK / 2;              // 128 k of bfloat16 pairs
// Bytes of one activation stage (BT tokens x 128 k of bfloat16: two boxes
// of 64 k, as the 128-byte swizzle spans 64 bfloat16).
__host__ __device__ constexpr int x_stage_bytes(int bt) { return bt * kBK * 2; }
// Instruction descriptor: binary32 accumulator, bfloat16 A and B, both
// K-major, N = BT tokens, M = 128 rows of W.
__host__ __device__ constexpr uint32_t instr_desc(int bt) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(bt >> 3) << 17) |
         (uint32_t(kBW >> 4) << 24);
}

// mbarrier slots (8 bytes each) in the first KB of shared memory
constexpr int kBarFull = 0;                    // [kMaxLoadStages] X + codes landed (tx)
constexpr int kBarEmpty = 8;                   // [kMaxLoadStages] MMAs + dequantize done
constexpr int kBarAFull = 16;                  // [kMaxAStages] A stage written
constexpr int kBarDFull = 32;                  // [2] group accumulator ready
constexpr int kBarDEmpty = 34;                 // [2] group accumulator read
constexpr int kBarMmaDone = 36;                // every MMA of the CTA finished
// Ring of 8-group blocks of scales and zeros.  Eight blocks (64 groups) are
// more than the producer can run ahead of the epilogue (the load ring, the
// eight A stages and the two accumulators hold at most 34 groups of k at
// group 32), so the producer never waits on a block the epilogue still needs
// for work it has not been given.
constexpr int kMetaSlots = 8;
constexpr int kMetaGroups = 8;                 // groups per block (16 bytes of a row)
constexpr int kBarMetaFull = 38;               // [kMetaSlots] block landed (tx)
constexpr int kBarMetaEmpty = 46;              // [kMetaSlots] block read by every user
constexpr int kMetaTensorBytes = kBW * kMetaGroups * 2;  // 2 KB: 128 rows x 8 binary16
constexpr int kMetaSlotBytes = 2 * kMetaTensorBytes;     // scales, then zeros
// Output staging: each epilogue warp writes its 32 rows x 16 tokens of Y
// into one of two buffers and one lane copies it out with a tensor store,
// so the tile's results leave while the warp starts on the next tile.
constexpr int kOutChunk = 16;                          // tokens per store
constexpr int kOutBufBytes = kOutChunk * 32 * 4;       // 2 KB (binary32; bfloat16 uses half)
constexpr int kOutWarpBytes = 2 * kOutBufBytes;
__host__ __device__ constexpr int out_stage_bytes(int ew) { return ew * kOutWarpBytes; }
constexpr int kTmemSlot = 512;                 // byte offset of the TMEM base address
constexpr int kAbortSlot = 516;                // byte offset of the abort flag
constexpr int kSmemHead = 1024;

struct Params {
  __nv_bfloat16* Y_bf16;   // one of Y_bf16 / Y_f32 is set
  float* Y_f32;
  const __half* scales;    // [N][ngroups]
  const __half* zeros;     // [N][ngroups] (asymmetric)
  int M, N, K, ngroups;
  int tiles_t, tiles_w, num_tiles;
  uint32_t codes_stage_bytes;  // kBW * kBK * bits / 8
  uint32_t off_x, off_codes;   // rings (1024-byte aligned)
  uint32_t off_meta;           // ring of scale / zero blocks (with MT)
  uint32_t off_out;            // output staging buffers; 0: plain stores
};

// A in tensor memory (M = 128 lanes, K = 16 as eight 32-bit columns of
// bfloat16 pairs), B from a shared-memory descriptor.
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      :
      : "r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 consecutive 32-bit columns of this warp's 32 lanes from registers.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32};"
      ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
      "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]),
      "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]),
      "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

// 16 consecutive 32-bit columns of this warp's 32 lanes from registers.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};"
      ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
      "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]),
      "r"(v[14]), "r"(v[15])
      : "memory");
}

// 16 consecutive binary32 columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
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
// (u0-z, u1-z), (u2-z, u3-z), (u4-z, u5-z), (u6-z, u7-z); zb2 holds 128 + z
// in both halves (the codes enter as the exact bfloat16 128 + u).
__device__ __forceinline__ void dq4(uint32_t w, uint32_t zb2, uint32_t* o) {
  constexpr uint32_t kMask = 0x000F000Fu, kMagic = 0x43004300u;
  uint32_t t[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(r) : "r"(w >> (4 * i)), "r"(kMask), "r"(kMagic));
    t[i] = r;  // (128 + u_i, 128 + u_{i+4})
  }
  o[0] = bf16x2_sub(__byte_perm(t[0], t[1], 0x5410), zb2);
  o[1] = bf16x2_sub(__byte_perm(t[2], t[3], 0x5410), zb2);
  o[2] = bf16x2_sub(__byte_perm(t[0], t[1], 0x7632), zb2);
  o[3] = bf16x2_sub(__byte_perm(t[2], t[3], 0x7632), zb2);
}

// Four 8-bit codes -> two bfloat16 pairs (u0 - z, u1 - z), (u2 - z, u3 - z):
// 2^23 + u in binary32 minus 2^23 + z is exact, and so is the conversion of
// the integer (|u - z| < 256) to bfloat16.
__device__ __forceinline__ void dq8(uint32_t w, float z, uint32_t* o) {
  float f[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    f[i] = __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7650 | i)) - (8388608.0f + z);
  const __nv_bfloat162 p0 = __floats2bfloat162_rn(f[0], f[1]);
  const __nv_bfloat162 p1 = __floats2bfloat162_rn(f[2], f[3]);
  o[0] = *reinterpret_cast<const uint32_t*>(&p0);
  o[1] = *reinterpret_cast<const uint32_t*>(&p1);
}

// LS: load stages in the shared-memory ring; DW: dequantize warps (4: one
// per tensor-memory lane quarter, a whole stage each; 8: two per quarter,
// half of a stage's k each).
// MT: scales and zeros arrive by TMA in blocks of 8 groups x 128 rows (K /
// group a multiple of 8, as the tensor maps' row pitch needs); otherwise the
// dequantize and epilogue threads read them from global memory directly.
template <int BITS, bool SYM, int G, int LS, int DW, int EW, int BT, bool MT>
__global__ void __launch_bounds__(threads_for(DW, EW), 1)
    gemm2_kernel(const __grid_constant__ CUtensorMap tm_x,
                 const __grid_constant__ CUtensorMap tm_codes,
                 const __grid_constant__ CUtensorMap tm_scales,
                 const __grid_constant__ CUtensorMap tm_zeros,
                 const __grid_constant__ CUtensorMap tm_y, const Params p) {
  static_assert(G == 32 || G == 64 || G == 128, "group");
  static_assert(LS >= 2 && LS <= kMaxLoadStages && (DW == 4 || DW == 8) &&
                    (EW == 8 || EW == 16), "roles");
  constexpr int kLoadStages = LS;
  constexpr int kNumDequantWarps = DW;
  constexpr int kEpilogueWarp0 = kDequantWarp0 + DW;
  constexpr int kNumEpilogueWarps = EW;
  static_assert(BT == 64 || BT == 128, "token tile");
  constexpr int kBT = BT;
  constexpr int kXStageBytes = x_stage_bytes(BT);
  constexpr int kDCols = BT;                       // one group accumulator
  constexpr int kACol0 = 2 * kDCols;               // A stages after the two accumulators
  // A stages of 64 columns in the rest of tensor memory: 4 (BT = 128), 6 (BT = 64)
  constexpr int kAStages = (kTmemCols - kACol0) / kAStageCols;
  static_assert(kAStages >= 2 && kAStages <= kMaxAStages, "A stages");
  static_assert(LS == kAStages, "one ring: load stage s and A stage s are freed together");
  constexpr int kXBoxBytes = BT * 64 * 2;          // one 64-k activation box
  constexpr uint32_t kIdesc = instr_desc(BT);
  constexpr int kEpiCols = kBT / (EW / 4);         // tokens per epilogue thread
  constexpr int kStagesPerBlock = kMetaGroups * G / kBK;  // load stages per metadata block
  constexpr int kStepsPerGroup = G / 16;        // 16-k MMA steps per group
  constexpr int kCodesRowBytes = kBK * BITS / 8;  // 64 | 128 bytes of a row per stage
  constexpr int kChunks = kCodesRowBytes / 16;     // 4 | 8 chunks of 16 bytes
  constexpr int kMyChunks = kChunks * 4 / DW;      // chunks of a row per dequantize thread
  constexpr int kMyCols = kAStageCols * 4 / DW;    // A columns per dequantize thread

  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kTmemSlot);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kAbortSlot);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nkb = p.K / kBK;  // load stages per tile

  if (threadIdx.x == 0) {
    for (int s = 0; s < kLoadStages; ++s) {
      mbar_init(&bars[kBarFull + s], 1);
      mbar_init(&bars[kBarEmpty + s], 1 + kNumDequantWarps);
    }
    for (int s = 0; s < kAStages; ++s) {
      mbar_init(&bars[kBarAFull + s], kNumDequantWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars[kBarDFull + b], 1);
      mbar_init(&bars[kBarDEmpty + b], kNumEpilogueWarps);
    }
    mbar_init(&bars[kBarMmaDone], 1);
    for (int b = 0; b < kMetaSlots; ++b) {
      mbar_init(&bars[kBarMetaFull + b], 1);
      mbar_init(&bars[kBarMetaEmpty + b], DW + EW);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
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
      if (MT) {
        prefetch_tensormap(&tm_scales);
        if (!SYM) prefetch_tensormap(&tm_zeros);
      }
      const uint64_t keep = l2_policy_evict_last();  // both operands are reread by other CTAs
      int issued = 0, mb = 0;
      bool stop = false;
      for (int tile = blockIdx.x; tile < p.num_tiles && !stop; tile += gridDim.x) {
        const int t0 = (tile / p.tiles_w) * kBT, w0 = (tile % p.tiles_w) * kBW;
        for (int kb = 0; kb < nkb; ++kb, ++issued) {
          if (MT && kb % kStagesPerBlock == 0) {
            // the next 8-group block of scales and zeros, ahead of its stages
            const int ms = mb % kMetaSlots;
            if (!wait(kBarMetaEmpty + ms, (uint32_t(mb / kMetaSlots) & 1u) ^ 1u)) {
              stop = true;
              break;
            }
            uint8_t* dst = smem + p.off_meta + ms * kMetaSlotBytes;
            mbar_arrive_expect_tx(&bars[kBarMetaFull + ms],
                                  uint32_t((SYM ? 1 : 2) * kMetaTensorBytes));
            tma_load_2d(dst, &tm_scales, &bars[kBarMetaFull + ms],
                        (kb / kStagesPerBlock) * kMetaGroups, w0, keep);
            if (!SYM)
              tma_load_2d(dst + kMetaTensorBytes, &tm_zeros, &bars[kBarMetaFull + ms],
                          (kb / kStagesPerBlock) * kMetaGroups, w0, keep);
            ++mb;
          }
          const int s = issued % kLoadStages;
          const uint32_t ph = uint32_t(issued / kLoadStages) & 1u;
          if (!wait(kBarEmpty + s, ph ^ 1u)) {
            stop = true;
            break;
          }
          mbar_arrive_expect_tx(&bars[kBarFull + s], uint32_t(kXStageBytes) + p.codes_stage_bytes);
          tma_load_2d(smem + p.off_x + s * kXStageBytes, &tm_x, &bars[kBarFull + s], kb * kBK,
                      t0, keep);
          tma_load_2d(smem + p.off_x + s * kXStageBytes + kXBoxBytes, &tm_x, &bars[kBarFull + s],
                      kb * kBK + 64, t0, keep);
          tma_load_2d(smem + p.off_codes + s * p.codes_stage_bytes, &tm_codes,
                      &bars[kBarFull + s], kb * kCodesRowBytes, w0, keep);
        }
      }
      // every issued copy lands before the CTA can finish
      for (int j = max(0, issued - kLoadStages); j < issued; ++j)
        mbar_wait(&bars[kBarFull + j % kLoadStages], uint32_t(j / kLoadStages) & 1u);
      for (int j = max(0, mb - kMetaSlots); j < mb; ++j)
        mbar_wait(&bars[kBarMetaFull + j % kMetaSlots], uint32_t(j / kMetaSlots) & 1u);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t xs0 = smem_addr(smem + p.off_x);
      int ld = 0;       // load stages consumed
      int gcount = 0;   // groups accumulated (selects the D buffer)
      bool stop = false;
      for (int tile = blockIdx.x; tile < p.num_tiles && !stop; tile += gridDim.x) {
        int step_in_group = 0;
        uint32_t d = 0;
        for (int kb = 0; kb < nkb && !stop; ++kb, ++ld) {
          const int s = ld % kLoadStages;
          const int as = s;  // the A stages are the load stages' slots
          // A written implies the stage's activations landed: the dequantize
          // warps wait for the stage's copies before they arrive here
          if (!wait(kBarAFull + as, uint32_t(ld / kAStages) & 1u)) {
            stop = true;
            break;
          }
          tc_fence_after();
          const uint64_t xdesc = umma_desc_sw128(xs0 + uint32_t(s) * kXStageBytes);
          const uint32_t a_addr = tmem_base + uint32_t(kACol0 + as * kAStageCols);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            if (step_in_group == 0) {
              const int db = gcount & 1;
              if (!wait(kBarDEmpty + db, (uint32_t(gcount >> 1) & 1u) ^ 1u)) {
                stop = true;
                break;
              }
              tc_fence_after();
              d = tmem_base + uint32_t(db * kDCols);
            }
            // k step k: box k / 4 of the stage, 32 bytes further per step in it
            tc_mma_ts(d, a_addr + uint32_t(8 * k),
                      xdesc + uint64_t((k / 4) * (kXBoxBytes >> 4) + 2 * (k % 4)), kIdesc,
                      step_in_group > 0 ? 1u : 0u);
            if (++step_in_group == kStepsPerGroup) {
              tc_commit(&bars[kBarDFull + (gcount & 1)]);
              step_in_group = 0;
              ++gcount;
            }
          }
          if (stop) break;
          // the stage's activations, codes and A columns are free once these
          // MMAs finish (one commit: the A stages are the load stages' slots)
          tc_commit(&bars[kBarEmpty + s]);
        }
      }
      // all MMAs of this CTA complete before tensor memory is freed
      tc_commit(&bars[kBarMmaDone]);
      mbar_wait(&bars[kBarMmaDone], 0);
    }
  } else if (warp < kEpilogueWarp0) {
    // ------------------------------------------------------------ dequantize
    // one row of the weight tile per thread; the warp's lanes are its 32
    // rows of tensor memory
    const int quarter = warp & 3;
    const int r = 32 * quarter + lane;  // row of the W tile = TMEM lane
    const uint32_t lanes = uint32_t(32 * quarter) << 16;
    const int part = (warp - kDequantWarp0) >> 2;  // which share of the stage's k (DW = 8)
    int ld = 0, mb = 0;
    bool stop = false;
    for (int tile = blockIdx.x; tile < p.num_tiles && !stop; tile += gridDim.x) {
      const int w0 = (tile % p.tiles_w) * kBW;
      const int row = w0 + r;
      const bool row_ok = row < p.N;
      const __half* zrow = p.zeros + size_t(row_ok ? row : 0) * p.ngroups;
      for (int kb = 0; kb < nkb; ++kb, ++ld) {
        const int s = ld % kLoadStages;
        const int as = ld % kAStages;
        // the stage's copies landed; then A stage `as` is free as well: the
        // copies were issued after the MMAs of its previous use committed
        if (!wait(kBarFull + s, uint32_t(ld / kLoadStages) & 1u)) {
          stop = true;
          break;
        }
        tc_fence_after();
        // with MT: this stage's zero points come from the ring's block
        const __half* zsm = nullptr;
        if constexpr (MT && !SYM) {
          const int ms = mb % kMetaSlots;
          if (kb % kStagesPerBlock == 0 &&
              !wait(kBarMetaFull + ms, uint32_t(mb / kMetaSlots) & 1u)) {
            stop = true;
            break;
          }
          zsm = reinterpret_cast<const __half*>(smem + p.off_meta + ms * kMetaSlotBytes +
                                                kMetaTensorBytes) +
                r * kMetaGroups;
        }
        // the stage's codes of row r, unswizzled: chunk c sits at chunk
        // c ^ key (64-byte swizzle: bits 4-5 of the address XOR bits 7-8;
        // 128-byte swizzle: bits 4-6 XOR bits 7-9)
        const uint8_t* crow = smem + p.off_codes + s * p.codes_stage_bytes + r * kCodesRowBytes;
        const int key = kChunks == 4 ? ((r >> 1) & 3) : (r & 7);
        uint32_t o[kMyCols];
        if constexpr (BITS == 4) {
#pragma unroll
          for (int cc = 0; cc < kMyChunks; ++cc) {  // 16 bytes = 32 k
            const int c = part * kMyChunks + cc;
            const uint4 v = *reinterpret_cast<const uint4*>(crow + ((c ^ key) << 4));
            const int k0 = kb * kBK + 32 * c;
            float zf = SYM ? 8.f : 0.f;
            if constexpr (!SYM) {
              if constexpr (MT)
                zf = __half2float(zsm[(k0 / G) % kMetaGroups]);
              else
                zf = row_ok ? __half2float(zrow[k0 / G]) : 0.f;
            }
            const __nv_bfloat162 zz = __floats2bfloat162_rn(128.f + zf, 128.f + zf);
            const uint32_t zb2 = *reinterpret_cast<const uint32_t*>(&zz);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) dq4(w[j], zb2, o + 16 * cc + 4 * j);
          }
        } else {
#pragma unroll
          for (int cc = 0; cc < kMyChunks; ++cc) {  // 16 bytes = 16 k
            const int c = part * kMyChunks + cc;
            const uint4 v = *reinterpret_cast<const uint4*>(crow + ((c ^ key) << 4));
            const int k0 = kb * kBK + 16 * c;
            float zf = SYM ? 128.f : 0.f;
            if constexpr (!SYM) {
              if constexpr (MT)
                zf = __half2float(zsm[(k0 / G) % kMetaGroups]);
              else
                zf = row_ok ? __half2float(zrow[k0 / G]) : 0.f;
            }
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) dq8(w[j], zf, o + 8 * cc + 2 * j);
          }
        }
        if (!row_ok) {
#pragma unroll
          for (int i = 0; i < kMyCols; ++i) o[i] = 0u;
        }
        // the codes of this stage are consumed, and with MT the block of zero
        // points once its last stage is
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kBarEmpty + s]);
        if (MT && (kb % kStagesPerBlock == kStagesPerBlock - 1 || kb == nkb - 1)) {
          if (lane == 0) mbar_arrive(&bars[kBarMetaEmpty + mb % kMetaSlots]);
          ++mb;
        }
        const uint32_t col = uint32_t(kACol0 + as * kAStageCols + part * kMyCols);
        if constexpr (kMyCols == 64) {
          uint32_t lo[32], hi[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            lo[i] = o[i];
            hi[i] = o[32 + i];
          }
          tmem_st32(tmem_base + lanes + col, lo);
          tmem_st32(tmem_base + lanes + col + 32, hi);
        } else if constexpr (kMyCols == 32) {
          tmem_st32(tmem_base + lanes + col, o);
        } else {
          tmem_st16(tmem_base + lanes + col, o);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kBarAFull + as]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int e = warp - kEpilogueWarp0;  // 0 .. EW-1
    const int quarter = warp & 3;         // TMEM lanes 32 * quarter ..
    const int half = e >> 2;              // tokens kEpiCols * half .. of the tile
    const int r = 32 * quarter + lane;    // row of the W tile
    const uint32_t lanes = uint32_t(32 * quarter) << 16;
    const bool staged = p.off_out != 0;
    const bool out_bf16 = p.Y_f32 == nullptr;
    const uint32_t out0 = smem_addr(smem + p.off_out) + uint32_t(e * kOutWarpBytes);
    int gcount = 0, mb = 0, chunks = 0;
    bool stop = false;
    float S[kEpiCols];
    // S += sg * D_g for the next group's accumulator, read in loads of up to
    // 32 columns; the buffer is handed back once its last load has landed
    // in registers, before the last multiply-adds.  False if a wait gave up.
    auto group = [&](float sg) -> bool {
      const int db = gcount & 1;
      if (!wait(kBarDFull + db, uint32_t(gcount >> 1) & 1u)) return false;
      tc_fence_after();
      const uint32_t taddr = tmem_base + lanes + uint32_t(db * kDCols + half * kEpiCols);
      constexpr int kLd = kEpiCols < 32 ? kEpiCols : 32;
#pragma unroll
      for (int h = 0; h < kEpiCols / kLd; ++h) {
        float dv[kLd];
        if constexpr (kLd == 32)
          tmem_ld32(taddr + uint32_t(32 * h), dv);
        else
          tmem_ld16(taddr + uint32_t(16 * h), dv);
        tmem_wait_ld();
        if (h == kEpiCols / kLd - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[kBarDEmpty + db]);
        }
#pragma unroll
        for (int j = 0; j < kLd; ++j) S[kLd * h + j] = fmaf(sg, dv[j], S[kLd * h + j]);
      }
      ++gcount;
      return true;
    };
    for (int tile = blockIdx.x; tile < p.num_tiles && !stop; tile += gridDim.x) {
      const int t0 = (tile / p.tiles_w) * kBT, w0 = (tile % p.tiles_w) * kBW;
      const int row = w0 + r;
      const bool row_ok = row < p.N;
#pragma unroll
      for (int j = 0; j < kEpiCols; ++j) S[j] = 0.f;
      if constexpr (MT) {
        // the row's eight scales of a block in one 16-byte load; the block
        // is released as soon as they are in registers
        for (int gb = 0; gb < p.ngroups && !stop; gb += kMetaGroups) {
          const int ms = mb % kMetaSlots;
          if (!wait(kBarMetaFull + ms, uint32_t(mb / kMetaSlots) & 1u)) {
            stop = true;
            break;
          }
          const uint4 sv = lds128(smem_addr(smem + p.off_meta + ms * kMetaSlotBytes) +
                                  uint32_t(r * kMetaGroups * 2));
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars[kBarMetaEmpty + ms]);
          ++mb;
          const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
          for (int u = 0; u < kMetaGroups; ++u) {
            const uint32_t bits16 = (u & 1) ? (sw[u >> 1] >> 16) : (sw[u >> 1] & 0xFFFFu);
            if (!group(__half2float(__ushort_as_half(static_cast<unsigned short>(bits16))))) {
              stop = true;
              break;
            }
          }
        }
      } else {
        const __half* srow = p.scales + size_t(row_ok ? row : 0) * p.ngroups;
        for (int gi = 0; gi < p.ngroups; ++gi) {
          if (!group(row_ok ? __half2float(srow[gi]) : 0.f)) {
            stop = true;
            break;
          }
        }
      }
      if (stop || *abort_flag) break;
      const int tb = t0 + half * kEpiCols;
      if (staged) {
        // chunk c of 16 tokens into buffer (chunks & 1), once the store that
        // last read that buffer (two chunks ago) has read it; the tensor
        // store leaves out the rows past N and the tokens past M
#pragma unroll
        for (int c = 0; c < kEpiCols / kOutChunk; ++c, ++chunks) {
          const uint32_t buf = out0 + uint32_t(chunks & 1) * kOutBufBytes;
          if (lane == 0) bulk_wait_group_read<1>();
          __syncwarp();
          if (out_bf16) {
#pragma unroll
            for (int j = 0; j < kOutChunk; ++j)
              sts16(buf + uint32_t(j * 64 + lane * 2),
                    __bfloat16_as_ushort(__float2bfloat16_rn(S[kOutChunk * c + j])));
          } else {
#pragma unroll
            for (int j = 0; j < kOutChunk; ++j)
              sts32(buf + uint32_t(j * 128 + lane * 4), S[kOutChunk * c + j]);
          }
          fence_async_shared();
          __syncwarp();
          if (lane == 0) {
            if (tb + kOutChunk * c < p.M && w0 + 32 * quarter < p.N)
              tma_store_2d(&tm_y, buf, w0 + 32 * quarter, tb + kOutChunk * c);
            bulk_commit_group();
          }
        }
      } else if (row_ok) {
#pragma unroll
        for (int j = 0; j < kEpiCols; ++j) {
          const int m = tb + j;
          if (m < p.M) {
            if (!out_bf16)
              p.Y_f32[size_t(m) * p.N + row] = S[j];
            else
              p.Y_bf16[size_t(m) * p.N + row] = __float2bfloat16_rn(S[j]);
          }
        }
      }
    }
    // every tensor store has finished before the CTA's shared memory goes
    if (staged && lane == 0) bulk_wait_group<0>();
  }

  // tensor memory is freed by the warp that allocated it, after every reader
  // and every MMA is done
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(uint32_t(kTmemCols))
                 : "memory");
  }
}

}  // namespace gemm2
}  // namespace wq
