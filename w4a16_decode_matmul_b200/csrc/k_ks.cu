// k_ks.cu -- plan and launch of the k-sliced direct-load small-batch matmul
// (gemv_ks.cuh).
#include <algorithm>

#include "host.h"
#include "gemv_ks.cuh"

namespace wqh {
namespace {

struct KsPlan {
  wq::ks::Params p;
  int grid = 1;
  int depth = 3;
  size_t smem = 0;
};

// 0: one CTA per SM with at most half an SM of shared memory, so that the
// next launch's CTA can stream on the same SM (ring 3 to 5 units deep);
// 1: one CTA per SM with the whole SM (ring up to 8 units deep); 2: two
// CTAs per SM, each with at most half of it.
int g_ks_mode = 0;

// Scope: 4-bit codes in groups of 128, K = 4096, M <= 4.  One CTA per SM (at
// most one per 8-row tile); the ring is as deep as the shared memory of the
// mode allows.
bool plan_ks(int M, int N, int K, int bits, int group, const DeviceInfo& dev, KsPlan* plan) {
  using namespace wq::ks;
  if (bits != 4 || group != 128 || K != kK || M < 1 || M > kMaxM || N < 1) return false;
  wq::ks::Params& p = plan->p;
  p = wq::ks::Params{};
  p.M = M;
  p.N = N;
  p.tiles = (N + kTileRows - 1) / kTileRows;
  plan->grid = std::min(p.tiles, (g_ks_mode == 2 ? 2 : 1) * dev.sms);
  const size_t max_tiles = size_t((p.tiles + plan->grid - 1) / plan->grid);
  p.off_sz = 0;
  p.off_part = uint32_t(round_up(max_tiles * kTileRows * (kK / 128 + 1) * 8, 16));
  p.off_ring = uint32_t(round_up(p.off_part + max_tiles * kWarps * kTileRows * size_t(M) * 4, 128));
  const size_t limit = g_ks_mode == 1 ? size_t(dev.max_smem_optin)
                                       : size_t(dev.max_smem_optin) / 2 - 1024;
  int depth = g_ks_mode == 1 ? 8 : 5;
  while (depth >= 3 && p.off_ring + size_t(kWarps) * depth * 1024 > limit) --depth;
  if (depth == 7) depth = 6;
  if (depth < 3) return false;
  plan->depth = depth;
  plan->smem = p.off_ring + size_t(kWarps) * depth * 1024;
  return true;
}

template <bool SYM, int MT, int DEPTH>
cudaError_t launch_ks(KsPlan* plan, const DeviceInfo& dev, cudaStream_t s, bool pdl) {
  // the build without the bounds-checked refill where every tile is whole
  auto kernel = plan->p.N % wq::ks::kTileRows == 0 ? &wq::ks::gemv_ks_kernel<SYM, MT, DEPTH, false>
                                                   : &wq::ks::gemv_ks_kernel<SYM, MT, DEPTH, true>;
  static int configured[2][kMaxDevices] = {};  // per build
  cudaError_t e = configure_smem(kernel, configured[plan->p.N % wq::ks::kTileRows == 0 ? 0 : 1],
                                 size_t(dev.max_smem_optin));
  if (e != cudaSuccess) return e;
  plan->p.pdl = pdl ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attrs[1];
  cfg.gridDim = dim3(unsigned(plan->grid));
  cfg.blockDim = dim3(wq::ks::kThreads);
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

template <bool SYM, int MT>
cudaError_t launch_ks_d(KsPlan* plan, const DeviceInfo& dev, cudaStream_t s, bool pdl) {
  switch (plan->depth) {
    case 8: return launch_ks<SYM, MT, 8>(plan, dev, s, pdl);
    case 6: return launch_ks<SYM, MT, 6>(plan, dev, s, pdl);
    case 5: return launch_ks<SYM, MT, 5>(plan, dev, s, pdl);
    case 4: return launch_ks<SYM, MT, 4>(plan, dev, s, pdl);
    default: return launch_ks<SYM, MT, 3>(plan, dev, s, pdl);
  }
}

template <bool SYM>
cudaError_t launch_ks_m(KsPlan* plan, const DeviceInfo& dev, cudaStream_t s, bool pdl) {
  const int M = plan->p.M;
  if (M == 1) return launch_ks_d<SYM, 1>(plan, dev, s, pdl);
  if (M == 2) return launch_ks_d<SYM, 2>(plan, dev, s, pdl);
  return launch_ks_d<SYM, 4>(plan, dev, s, pdl);
}

}  // namespace

bool run_ks(const MatmulArgs& a, cudaError_t* err) {
  KsPlan kp;
  if (!plan_ks(a.M, a.N, a.K, a.bits, a.group, a.dev, &kp)) return false;
  kp.p.X = static_cast<const __nv_bfloat16*>(a.X);
  kp.p.Y = a.Y;
  kp.p.codes = static_cast<const uint8_t*>(a.codes);
  kp.p.scales = static_cast<const __half*>(a.scales);
  kp.p.zeros = static_cast<const __half*>(a.zeros);
  kp.p.y_bf16 = a.y_bf16 ? 1 : 0;
  *err = a.sym ? launch_ks_m<true>(&kp, a.dev, a.stream, a.pdl)
               : launch_ks_m<false>(&kp, a.dev, a.stream, a.pdl);
  return true;
}

}  // namespace wqh

extern "C" {

// Tuning hook, not part of the public ABI: the k-sliced kernel's shared
// memory mode (0: one CTA per SM in half of it, 1: one CTA per SM, the whole
// SM, 2: two CTAs per SM).
void wq_internal_set_ks_mode(int mode) { wqh::g_ks_mode = mode >= 0 && mode <= 2 ? mode : 0; }

// Test hook, not part of the public ABI: the k-sliced kernel's plan for a
// device with `sms` SMs and `smem_optin` bytes of shared memory per block,
// written to out[0..7] (M, N, tiles, off_sz, off_part, off_ring, depth,
// smem, grid).  Returns 0 if the shape is outside the kernel's scope.
int wq_internal_plan_ks(int M, int N, int K, int bits, int group, int sms, int smem_optin,
                        int64_t* out) {
  wqh::DeviceInfo dev;
  dev.sms = sms;
  dev.max_smem_optin = smem_optin;
  wqh::KsPlan plan;
  if (!wqh::plan_ks(M, N, K, bits, group, dev, &plan)) return 0;
  const wq::ks::Params& p = plan.p;
  const int64_t v[] = {p.M,        p.N,         p.tiles,    p.off_sz, p.off_part,
                       p.off_ring, plan.depth,  int64_t(plan.smem), plan.grid};
  for (size_t i = 0; i < sizeof(v) / sizeof(v[0]); ++i) out[i] = v[i];
  return 1;
}

}  // extern "C"
