// k_gemm2.cu -- plan and launch of the prefill matmul with the weights as
// the tensor-memory operand (gemm2.cuh).
#include <algorithm>

#include "host.h"
#include "gemm2.cuh"

namespace wqh {
namespace {

struct Gemm2Plan {
  wq::gemm2::Params p;
  int grid = 1;
  size_t smem = 0;
  size_t smem_rings = 0;  // without the output staging
  int variant = 0;
  int bt = 128;   // tokens per tile: 64 for M <= 64 (the MMA's N), else 128
  bool meta_tma = false;  // scales / zeros by TMA (K / group a multiple of 8)
};

// Build variants (load stages, dequantize warps, epilogue warps), chosen
// through an internal tuning hook.  Eight dequantize warps (two per lane
// quarter, half of a stage's k each) measured slower on B200 (658 against
// 757 TFLOP/s at M = 2048: at 576 threads the registers run out and the
// epilogue spills), so one build remains.
struct Gemm2Variant {
  int load_stages, dequant_warps, epilogue_warps;
};
constexpr Gemm2Variant kGemm2Variants[] = {{4, 4, 8}};
constexpr int kNumGemm2Variants = int(sizeof(kGemm2Variants) / sizeof(kGemm2Variants[0]));
int g_gemm2_variant = 0;

// Scope: groups of 32, 64 or 128, K a multiple of 128; any M and N.
bool plan_gemm2(int M, int N, int K, int bits, int group, const DeviceInfo& dev,
                Gemm2Plan* plan, int variant) {
  using namespace wq::gemm2;
  if (variant < 0 || variant >= kNumGemm2Variants) return false;
  plan->variant = variant;
  // the 64-token tile has one build: 6 load stages, 4 dequantize and 8
  // epilogue warps
  const int stages = M <= 64 ? 6 : kGemm2Variants[variant].load_stages;
  if (group != 32 && group != 64 && group != 128) return false;
  if (bits != 4 && bits != 8) return false;
  if (K % kBK != 0 || K % group != 0 || M < 1 || N < 1) return false;
  wq::gemm2::Params& p = plan->p;
  p = wq::gemm2::Params{};
  plan->bt = M <= 64 ? 64 : 128;
  const int bt = plan->bt;
  p.M = M;
  p.N = N;
  p.K = K;
  p.ngroups = K / group;
  p.tiles_t = (M + bt - 1) / bt;
  p.tiles_w = (N + kBW - 1) / kBW;
  const long long tiles = (long long)p.tiles_t * p.tiles_w;
  if (tiles > 0x7fffffffLL) return false;
  p.num_tiles = int(tiles);
  p.codes_stage_bytes = uint32_t(kBW * kBK * bits / 8);
  p.off_x = kSmemHead;
  p.off_codes = p.off_x + uint32_t(stages * x_stage_bytes(bt));
  p.off_meta = p.off_codes + uint32_t(stages) * p.codes_stage_bytes;
  plan->meta_tma = p.ngroups % kMetaGroups == 0;
  plan->smem = p.off_meta + (plan->meta_tma ? size_t(kMetaSlots) * kMetaSlotBytes : 0);
  if (plan->smem > size_t(dev.max_smem_optin)) return false;
  plan->smem_rings = plan->smem;
  // the epilogue's output staging after the rings, where it fits (not with
  // 8-bit codes and 128-token tiles)
  const int ew = M <= 64 ? 8 : kGemm2Variants[variant].epilogue_warps;
  const size_t off_out = (plan->smem + 1023) & ~size_t(1023);
  if (off_out + size_t(out_stage_bytes(ew)) <= size_t(dev.max_smem_optin)) {
    p.off_out = uint32_t(off_out);
    plan->smem = off_out + size_t(out_stage_bytes(ew));
  }
  plan->grid = std::min(p.num_tiles, dev.sms);
  return true;
}

template <int BITS, bool SYM, int G, int LS, int DW, int EW, int BT, bool MT>
cudaError_t launch_gemm2(Gemm2Plan* plan, const DeviceInfo* dev, const void* X, const void* c,
                         const void* sc, const void* z, cudaStream_t s) {
  using namespace wq::gemm2;
  auto kernel = &gemm2_kernel<BITS, SYM, G, LS, DW, EW, BT, MT>;
  static int configured[kMaxDevices] = {};
  {
    const cudaError_t e = configure_smem(kernel, configured, size_t(dev->max_smem_optin));
    if (e != cudaSuccess) return e;
  }
  const wq::gemm2::Params& p = plan->p;
  CUtensorMap tx, tc;
  // X [M][K] bfloat16, boxes of 64 k x BT tokens (two per 128-k stage), 128-byte swizzle (the
  // K-major canonical layout of the MMA's B operand)
  if (!encode_2d_ex(&tx, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, uint64_t(p.K), uint64_t(p.M),
                    64u, uint32_t(BT), CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
    return cudaErrorInvalidValue;
  // codes [N][K*bits/8] bytes, boxes of 128 k x 128 rows, swizzled so that
  // the dequantize threads (one row each) read without bank conflicts
  const uint32_t row_box = uint32_t(kBK * BITS / 8);
  if (!encode_2d_ex(&tc, c, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, uint64_t(p.K) * BITS / 8,
                    uint64_t(p.N), row_box, uint32_t(kBW),
                    BITS == 4 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
    return cudaErrorInvalidValue;
  // scales / zeros [N][ngroups] binary16, boxes of 8 groups x 128 rows
  CUtensorMap ts, tz;
  std::memcpy(&ts, &tx, sizeof(tx));
  std::memcpy(&tz, &tx, sizeof(tx));
  if (MT) {
    if (!encode_2d(&ts, sc, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, uint64_t(p.ngroups),
                   uint64_t(p.N), uint32_t(kMetaGroups), uint32_t(kBW)))
      return cudaErrorInvalidValue;
    if (!SYM && !encode_2d(&tz, z, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, uint64_t(p.ngroups),
                           uint64_t(p.N), uint32_t(kMetaGroups), uint32_t(kBW)))
      return cudaErrorInvalidValue;
  }
  // Y [M][N] for the epilogue's tensor stores: boxes of 32 rows of W x 16
  // tokens; without the staging (or a map) the epilogue stores directly
  CUtensorMap ty;
  std::memcpy(&ty, &tx, sizeof(tx));
  wq::gemm2::Params pl = p;
  size_t smem = plan->smem;
  if (pl.off_out != 0) {
    const bool f32 = pl.Y_f32 != nullptr;
    const void* y = f32 ? static_cast<const void*>(pl.Y_f32) : static_cast<const void*>(pl.Y_bf16);
    const int esz = f32 ? 4 : 2;
    if (reinterpret_cast<uintptr_t>(y) % 16 != 0 || (int64_t(p.N) * esz) % 16 != 0 ||
        !encode_2d(&ty, y, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                   esz, uint64_t(p.N), uint64_t(p.M), 32u, uint32_t(kOutChunk))) {
      pl.off_out = 0;
      smem = plan->smem_rings;
      std::memcpy(&ty, &tx, sizeof(tx));
    }
  }
  kernel<<<plan->grid, threads_for(DW, EW), smem, s>>>(tx, tc, ts, tz, ty, pl);
  return cudaGetLastError();
}

template <int BITS, bool SYM, int G, bool MT>
cudaError_t launch_gemm2_v(Gemm2Plan* plan, const DeviceInfo* dev, const void* X, const void* c,
                           const void* sc, const void* z, cudaStream_t s) {
  if (plan->bt == 64) return launch_gemm2<BITS, SYM, G, 6, 4, 8, 64, MT>(plan, dev, X, c, sc, z, s);
  return launch_gemm2<BITS, SYM, G, 4, 4, 8, 128, MT>(plan, dev, X, c, sc, z, s);
}

template <int BITS, bool SYM, int G>
struct Gemm2Op {
  static cudaError_t run(Gemm2Plan* plan, const DeviceInfo* dev, const void* X, const void* c,
                         const void* sc, const void* z, cudaStream_t s) {
    return plan->meta_tma ? launch_gemm2_v<BITS, SYM, G, true>(plan, dev, X, c, sc, z, s)
                          : launch_gemm2_v<BITS, SYM, G, false>(plan, dev, X, c, sc, z, s);
  }
};

}  // namespace

bool run_gemm2(const MatmulArgs& a, cudaError_t* err) {
  Gemm2Plan gp;
  if (!plan_gemm2(a.M, a.N, a.K, a.bits, a.group, a.dev, &gp, g_gemm2_variant) &&
      (g_gemm2_variant == 0 || !plan_gemm2(a.M, a.N, a.K, a.bits, a.group, a.dev, &gp, 0)))
    return false;
  if (a.y_bf16)
    gp.p.Y_bf16 = static_cast<__nv_bfloat16*>(a.Y);
  else
    gp.p.Y_f32 = static_cast<float*>(a.Y);
  gp.p.scales = static_cast<const __half*>(a.scales);
  gp.p.zeros = static_cast<const __half*>(a.zeros);
  *err = dispatch_format<Gemm2Op>(a.bits, a.sym, a.group, &gp, &a.dev, a.X, a.codes, a.scales,
                                 a.zeros, a.stream);
  return true;
}

}  // namespace wqh

extern "C" {

// Test hook, not part of the public ABI: the prefill plan with the weights in
// tensor memory, written to out[0..10] (M, N, K, ngroups, tiles_t, tiles_w,
// num_tiles, codes_stage_bytes, smem, grid, off_out).  Returns 0 if the shape is
// outside the kernel's scope.
int wq_internal_plan_gemm2(int M, int N, int K, int bits, int group, int sms, int smem_optin,
                           int64_t* out) {
  wqh::DeviceInfo dev;
  dev.sms = sms;
  dev.max_smem_optin = smem_optin;
  wqh::Gemm2Plan plan;
  if (!wqh::plan_gemm2(M, N, K, bits, group, dev, &plan, 0)) return 0;
  const wq::gemm2::Params& p = plan.p;
  const int64_t v[] = {p.M,         p.N,         p.K,         p.ngroups,         p.tiles_t,
                       p.tiles_w,   p.num_tiles, p.codes_stage_bytes, int64_t(plan.smem),
                       plan.grid,   p.off_out};
  for (size_t i = 0; i < sizeof(v) / sizeof(v[0]); ++i) out[i] = v[i];
  return 1;
}

// Tuning hook, not part of the public ABI: the build variant of the prefill
// kernel with the weights in tensor memory (see kGemm2Variants; one that
// does not fit falls back to 0).  Returns the number of variants.
int wq_internal_set_gemm2_variant(int variant) {
  if (variant >= 0 && variant < wqh::kNumGemm2Variants) wqh::g_gemm2_variant = variant;
  return wqh::kNumGemm2Variants;
}

}  // extern "C"
