// k_tc.cu -- plan and launch of the tensor-memory small-batch matmul
// (gemv_tc.cuh).
#include <algorithm>

#include "host.h"
#include "gemv_tc.cuh"

namespace wqh {

struct TcPlan {
  wq::tc::Params p;
  int grid = 1;
  int depth = 3;
  size_t smem = 0;
};

// Scope: 4- or 8-bit codes in groups of 128, K = 4096, M <= 2.  One CTA per
// SM (at most one per 8-row tile), at most half of the SM's shared memory so
// that the next launch's CTA fits beside it and prefetches its first
// stages; a ring of 4 stages per warp for 4-bit codes (2 KB each), 2 for
// 8-bit codes (4 KB each).  Layers whose CTAs hold too many tiles for that
// are out of scope.
int tc_depth(int bits) { return bits == 4 ? 4 : 2; }

bool plan_tc(int M, int N, int K, int bits, int group, const DeviceInfo& dev, TcPlan* plan) {
  using namespace wq::tc;
  if ((bits != 4 && bits != 8) || group != 128 || K != kK || M < 1 || M > kMaxMT || N < 1)
    return false;
  wq::tc::Params& p = plan->p;
  p = wq::tc::Params{};
  p.M = M;
  p.N = N;
  p.tiles = (N + kTileRows - 1) / kTileRows;
  plan->grid = std::min(p.tiles, dev.sms);
  const size_t max_tiles = size_t((p.tiles + plan->grid - 1) / plan->grid);
  p.off_b = uint32_t(kHeadBytes);
  p.off_sz = p.off_b + uint32_t(b_bytes(M));
  p.off_part = uint32_t(round_up(p.off_sz + max_tiles * kTileRows * kSzStride * 4, 16));
  p.off_ring = uint32_t(round_up(p.off_part + max_tiles * 8 * kTileRows * size_t(M) * 4, 128));
  const size_t limit = size_t(dev.max_smem_optin) / 2 - 1024;
  plan->depth = tc_depth(bits);
  plan->smem = p.off_ring + size_t(kDqWarps) * plan->depth * slot_bytes(bits);
  return plan->smem <= limit;
}

namespace {

template <int BITS, bool SYM, int MT>
cudaError_t launch_tc(TcPlan* plan, const DeviceInfo& dev, cudaStream_t s, bool pdl) {
  constexpr int kDepth = BITS == 4 ? 4 : 2;
  // the build without the bounds-checked refill where every tile is whole
  const bool whole = plan->p.N % wq::tc::kTileRows == 0;
  auto kernel = whole ? &wq::tc::gemv_tc_kernel<BITS, SYM, MT, kDepth, false>
                      : &wq::tc::gemv_tc_kernel<BITS, SYM, MT, kDepth, true>;
  static int configured[2][kMaxDevices] = {};  // per build
  cudaError_t e = configure_smem(kernel, configured[whole ? 0 : 1], size_t(dev.max_smem_optin));
  if (e != cudaSuccess) return e;
  plan->p.pdl = pdl ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attrs[1];
  cfg.gridDim = dim3(unsigned(plan->grid));
  cfg.blockDim = dim3(wq::tc::kThreads);
  cfg.dynamicSmemBytes = plan->smem;
  cfg.stream = s;
  if (pdl) {
    attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, kernel, plan->p);
}

template <int BITS, bool SYM>
cudaError_t launch_tc_m(TcPlan* plan, const DeviceInfo& dev, cudaStream_t s, bool pdl) {
  return plan->p.M == 1 ? launch_tc<BITS, SYM, 1>(plan, dev, s, pdl)
                        : launch_tc<BITS, SYM, 2>(plan, dev, s, pdl);
}

}  // namespace

bool run_tc(const MatmulArgs& a, cudaError_t* err) {
  TcPlan tp;
  if (!plan_tc(a.M, a.N, a.K, a.bits, a.group, a.dev, &tp)) return false;
  tp.p.X = static_cast<const __nv_bfloat16*>(a.X);
  tp.p.Y = a.Y;
  tp.p.codes = static_cast<const uint8_t*>(a.codes);
  tp.p.scales = static_cast<const __half*>(a.scales);
  tp.p.zeros = static_cast<const __half*>(a.zeros);
  tp.p.y_bf16 = a.y_bf16 ? 1 : 0;
  if (a.bits == 4)
    *err = a.sym ? launch_tc_m<4, true>(&tp, a.dev, a.stream, a.pdl)
                 : launch_tc_m<4, false>(&tp, a.dev, a.stream, a.pdl);
  else
    *err = a.sym ? launch_tc_m<8, true>(&tp, a.dev, a.stream, a.pdl)
                 : launch_tc_m<8, false>(&tp, a.dev, a.stream, a.pdl);
  return true;
}

}  // namespace wqh

extern "C" {

// Test hook, not part of the public ABI: the tensor-memory small-batch
// kernel's plan for a device with `sms` SMs and `smem_optin` bytes of shared
// memory per block, written to out[0..9] (M, N, tiles, off_b, off_sz,
// off_part, off_ring, depth, smem, grid).  Returns 0 if the shape is outside
// the kernel's scope.
int wq_internal_plan_tc(int M, int N, int K, int bits, int group, int sms, int smem_optin,
                        int64_t* out) {
  wqh::DeviceInfo dev;
  dev.sms = sms;
  dev.max_smem_optin = smem_optin;
  wqh::TcPlan plan;
  if (!wqh::plan_tc(M, N, K, bits, group, dev, &plan)) return 0;
  const wq::tc::Params& p = plan.p;
  const int64_t v[] = {p.M,      p.N,        p.tiles,    p.off_b,           p.off_sz,
                       p.off_part, p.off_ring, plan.depth, int64_t(plan.smem), plan.grid};
  for (size_t i = 0; i < sizeof(v) / sizeof(v[0]); ++i) out[i] = v[i];
  return 1;
}

}  // extern "C"
