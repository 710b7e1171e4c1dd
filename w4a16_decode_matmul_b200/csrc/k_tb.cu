// k_tb.cu -- plan and launch of the bulk-staged small-batch matmul
// (gemv_tb.cuh).
#include <algorithm>

#include "host.h"
#include "gemv_tb.cuh"

namespace wqh {
namespace {

struct TbPlan {
  wq::tb::Params p;
  int grid = 1;
  size_t smem = 0;
  bool xreg = false;
};

// Scope: 4-bit codes in groups of 128, M <= 4, K a multiple of 1,024 (whole
// 256-byte blocks of codes per row, and scale rows of a multiple of 16
// bytes, as the tensor maps need).  One CTA per SM (at most one per 8-row
// tile), sized to at most half an SM so that the next launch's CTA can
// stream on the same SM before this one ends.
bool plan_tb(int M, int N, int K, int bits, int group, const DeviceInfo& dev, TbPlan* plan) {
  using namespace wq::tb;
  if (bits != 4 || group != kGroup || M < 1 || M > kMaxM || N < 1 || K < 1024 || K % 1024 != 0)
    return false;
  wq::tb::Params& p = plan->p;
  p = wq::tb::Params{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.ngroups = K / kGroup;
  p.pairs = p.ngroups / 2;
  p.nch = (p.pairs + kChunkPairs - 1) / kChunkPairs;
  p.tiles = (N + kTileRows - 1) / kTileRows;
  plan->xreg = p.nch == 1;
  plan->grid = std::min(p.tiles, dev.sms);
  const size_t max_tiles = size_t((p.tiles + plan->grid - 1) / plan->grid);
  p.off_part = 1024;
  size_t off = p.off_part + max_tiles * kConsumerWarps * kTileRows * size_t(M) * 4;
  p.xs_row_bytes = uint32_t(K) * 2 + 64;  // rows 64 bytes apart modulo 128
  p.off_x = uint32_t(round_up(off, 16));
  p.off_sx = p.off_x;
  if (!plan->xreg) {
    p.off_sx = uint32_t(round_up(p.off_x + size_t(M) * p.xs_row_bytes, 16));
    off = p.off_sx + size_t(M) * p.ngroups * 4;
  }
  p.off_ring = uint32_t(round_up(off, 1024));
  const size_t half_sm = size_t(dev.max_smem_optin) / 2 - 1024;
  const int fit = int((half_sm - std::min(half_sm, size_t(p.off_ring))) / kStageBytes);
  p.depth = std::min(kMaxDepth, fit);
  if (p.depth < 3) return false;
  plan->smem = p.off_ring + size_t(p.depth) * kStageBytes;
  return true;
}

template <bool SYM, int MT, bool XREG>
cudaError_t launch_tb(TbPlan* plan, const DeviceInfo& dev, const void* codes, const void* scales,
                      const void* zeros, cudaStream_t s, bool pdl) {
  using namespace wq::tb;
  auto kernel = &gemv_tb_kernel<SYM, MT, XREG>;
  static int configured[kMaxDevices] = {};
  cudaError_t e = configure_smem(kernel, configured, size_t(dev.max_smem_optin));
  if (e != cudaSuccess) return e;
  const wq::tb::Params& p = plan->p;
  CUtensorMap tc, ts, tz;
  // codes [N][K/2] bytes seen as [N][K/512 blocks][256 bytes]; one box is 8
  // rows x 8 blocks x 256 bytes (one stage)
  if (!encode_3d(&tc, codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 256, uint64_t(p.K) / 512,
                 uint64_t(p.N), 256, uint64_t(p.K) / 2, 256, kRowBytes / 256, kTileRows,
                 CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
    return cudaErrorInvalidValue;
  // scales / zeros [N][ngroups] binary16; one box is 8 rows x 32 groups
  if (!encode_2d(&ts, scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, uint64_t(p.ngroups),
                 uint64_t(p.N), 2 * kChunkPairs, kTileRows))
    return cudaErrorInvalidValue;
  std::memcpy(&tz, &ts, sizeof(ts));
  if (!SYM && !encode_2d(&tz, zeros, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, uint64_t(p.ngroups),
                         uint64_t(p.N), 2 * kChunkPairs, kTileRows))
    return cudaErrorInvalidValue;
  plan->p.pdl = pdl ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attrs[1];
  cfg.gridDim = dim3(unsigned(plan->grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = plan->smem;
  cfg.stream = s;
  if (pdl) {
    attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, kernel, tc, ts, tz, plan->p);
}

template <bool SYM, int MT>
cudaError_t launch_tb_x(TbPlan* plan, const DeviceInfo& dev, const void* c, const void* sc,
                        const void* z, cudaStream_t s, bool pdl) {
  return plan->xreg ? launch_tb<SYM, MT, true>(plan, dev, c, sc, z, s, pdl)
                    : launch_tb<SYM, MT, false>(plan, dev, c, sc, z, s, pdl);
}

template <bool SYM>
cudaError_t launch_tb_m(TbPlan* plan, const DeviceInfo& dev, const void* c, const void* sc,
                        const void* z, cudaStream_t s, bool pdl) {
  const int M = plan->p.M;
  if (M == 1) return launch_tb_x<SYM, 1>(plan, dev, c, sc, z, s, pdl);
  if (M == 2) return launch_tb_x<SYM, 2>(plan, dev, c, sc, z, s, pdl);
  return launch_tb_x<SYM, 4>(plan, dev, c, sc, z, s, pdl);
}

}  // namespace

bool run_tb(const MatmulArgs& a, cudaError_t* err) {
  TbPlan tp;
  if (!plan_tb(a.M, a.N, a.K, a.bits, a.group, a.dev, &tp)) return false;
  tp.p.X = static_cast<const __nv_bfloat16*>(a.X);
  tp.p.Y = a.Y;
  tp.p.y_bf16 = a.y_bf16 ? 1 : 0;
  *err = a.sym ? launch_tb_m<true>(&tp, a.dev, a.codes, a.scales, a.zeros, a.stream, a.pdl)
               : launch_tb_m<false>(&tp, a.dev, a.codes, a.scales, a.zeros, a.stream, a.pdl);
  return true;
}

}  // namespace wqh

extern "C" {

// Test hook, not part of the public ABI: the bulk-staged kernel's plan for a
// device with `sms` SMs and `smem_optin` bytes of shared memory per block,
// written to out[0..14] (M, N, K, ngroups, pairs, nch, tiles, depth,
// xs_row_bytes, off_part, off_x, off_sx, off_ring, smem, grid, xreg).
// Returns 0 if the shape is outside the kernel's scope.
int wq_internal_plan_tb(int M, int N, int K, int bits, int group, int sms, int smem_optin,
                        int64_t* out) {
  wqh::DeviceInfo dev;
  dev.sms = sms;
  dev.max_smem_optin = smem_optin;
  wqh::TbPlan plan;
  if (!wqh::plan_tb(M, N, K, bits, group, dev, &plan)) return 0;
  const wq::tb::Params& p = plan.p;
  const int64_t v[] = {p.M,       p.N,          p.K,        p.ngroups, p.pairs,   p.nch,
                       p.tiles,   p.depth,      p.xs_row_bytes, p.off_part, p.off_x, p.off_sx,
                       p.off_ring, int64_t(plan.smem), plan.grid, plan.xreg ? 1 : 0};
  for (size_t i = 0; i < sizeof(v) / sizeof(v[0]); ++i) out[i] = v[i];
  return 1;
}

}  // extern "C"
