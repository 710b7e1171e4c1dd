// k_ld.cu -- plan and launch of the direct-load small-batch matmul
// (gemv_ld.cuh).
#include <algorithm>

#include "host.h"
#include "gemv_ld.cuh"

namespace wqh {
namespace {

struct LdPlan {
  wq::ld::Params p;
  int grid = 1;
  size_t smem = 0;
  int variant = 0;
};

// Build variants of the kernel (ring depth, pipe of the unpack shifts, CTAs
// per SM the registers must allow), chosen through an internal tuning hook.
struct LdVariant {
  int depth;
  bool fma_shift;
  int min_blocks;
};
constexpr LdVariant kLdVariants[] = {
    {3, false, 1}, {3, true, 1}, {4, true, 2}, {6, true, 1}, {4, false, 2}, {6, false, 1},
};
constexpr int kNumLdVariants = int(sizeof(kLdVariants) / sizeof(kLdVariants[0]));
int g_ld_variant = 4;  // measured fastest (4-deep ring, two CTAs per SM)

// Plan the direct-load kernel: 4-bit codes in groups of 128 with K a
// multiple of 512 (groups come in pairs; a CTA's scales load in blocks of
// four), M <= 4; one CTA per SM (at most one per 8-row tile) with the
// activations, their group sums, the CTA's scales and zeros and the per-warp
// partial sums of its tiles in shared memory, next to the per-warp rings of
// codes.
bool plan_ld(int M, int N, int K, int bits, int group, const DeviceInfo& dev, LdPlan* plan,
             int variant) {
  using namespace wq::ld;
  if (bits != 4 || group != kGroup || M < 1 || M > kMaxM || N < 1 || K < 4 * kGroup ||
      K % (4 * kGroup) != 0)
    return false;
  wq::ld::Params& p = plan->p;
  p = wq::ld::Params{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.ngroups = K / kGroup;
  p.tiles = (N + kTileRows - 1) / kTileRows;
  plan->grid = std::min(p.tiles, dev.sms);
  const size_t max_tiles = size_t((p.tiles + plan->grid - 1) / plan->grid);
  const size_t max_rows = max_tiles * kTileRows;
  p.xs_row_bytes = uint32_t(K) * 2 + 64;  // rows 64 bytes apart modulo 128: no bank conflicts
  p.off_sx = uint32_t(round_up(size_t(M) * p.xs_row_bytes, 16));
  p.off_sz = uint32_t(round_up(p.off_sx + size_t(M) * p.ngroups * 4, 16));
  p.off_part = uint32_t(round_up(p.off_sz + max_rows * (p.ngroups + 1) * 8, 16));
  p.off_ring =
      uint32_t(round_up(p.off_part + max_tiles * kWarps * kTileRows * size_t(M) * 4, 128));
  if (variant < 0 || variant >= kNumLdVariants) return false;
  const LdVariant v = kLdVariants[variant];
  plan->variant = variant;
  plan->smem = p.off_ring + size_t(kWarps) * v.depth * 1024;
  p.mul_shr4 = 1u << 28;
  p.mul_shr8 = 1u << 24;
  p.mul_shr12 = 1u << 20;
  // CTAs of two launches share an SM only if each takes at most half of it
  // (1 KB of every CTA's shared memory is reserved by the hardware)
  const size_t limit = v.min_blocks == 2 ? size_t(dev.max_smem_optin) / 2 - 1024
                                         : size_t(dev.max_smem_optin);
  return plan->smem <= limit;
}

template <bool SYM, int MT, int DEPTH, bool FMA_SHIFT, int MINB>
cudaError_t launch_ld(LdPlan* plan, const DeviceInfo& dev, cudaStream_t s, bool pdl) {
  auto kernel = &wq::ld::gemv_ld_kernel<SYM, MT, DEPTH, FMA_SHIFT, MINB>;
  static int configured[kMaxDevices] = {};
  cudaError_t e = configure_smem(kernel, configured, size_t(dev.max_smem_optin));
  if (e != cudaSuccess) return e;
  plan->p.pdl = pdl ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attrs[1];
  cfg.gridDim = dim3(unsigned(plan->grid));
  cfg.blockDim = dim3(wq::ld::kThreads);
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
cudaError_t launch_ld_v(LdPlan* plan, const DeviceInfo& dev, cudaStream_t s, bool pdl) {
  switch (plan->variant) {
    case 1: return launch_ld<SYM, MT, 3, true, 1>(plan, dev, s, pdl);
    case 2: return launch_ld<SYM, MT, 4, true, 2>(plan, dev, s, pdl);
    case 3: return launch_ld<SYM, MT, 6, true, 1>(plan, dev, s, pdl);
    case 4: return launch_ld<SYM, MT, 4, false, 2>(plan, dev, s, pdl);
    case 5: return launch_ld<SYM, MT, 6, false, 1>(plan, dev, s, pdl);
    default: return launch_ld<SYM, MT, 3, false, 1>(plan, dev, s, pdl);
  }
}

template <bool SYM>
cudaError_t launch_ld_m(LdPlan* plan, const DeviceInfo& dev, cudaStream_t s, bool pdl) {
  const int M = plan->p.M;
  if (M == 1) return launch_ld_v<SYM, 1>(plan, dev, s, pdl);
  if (M == 2) return launch_ld_v<SYM, 2>(plan, dev, s, pdl);
  return launch_ld_v<SYM, 4>(plan, dev, s, pdl);
}

}  // namespace

bool run_ld(const MatmulArgs& a, cudaError_t* err) {
  LdPlan lp;
  if (!plan_ld(a.M, a.N, a.K, a.bits, a.group, a.dev, &lp, g_ld_variant) &&
      (g_ld_variant == 0 || !plan_ld(a.M, a.N, a.K, a.bits, a.group, a.dev, &lp, 0)))
    return false;
  lp.p.X = static_cast<const __nv_bfloat16*>(a.X);
  lp.p.Y = a.Y;
  lp.p.codes = static_cast<const uint8_t*>(a.codes);
  lp.p.scales = static_cast<const __half*>(a.scales);
  lp.p.zeros = static_cast<const __half*>(a.zeros);
  lp.p.y_bf16 = a.y_bf16 ? 1 : 0;
  *err = a.sym ? launch_ld_m<true>(&lp, a.dev, a.stream, a.pdl)
               : launch_ld_m<false>(&lp, a.dev, a.stream, a.pdl);
  return true;
}

}  // namespace wqh

extern "C" {

// Test hook, not part of the public ABI: the direct-load kernel's plan for a
// device with `sms` SMs and `smem_optin` bytes of shared memory per block,
// written to out[0..11] (see tests/test_plan_ld.py for the field order).
// Returns 0 if the shape is outside that kernel's scope.
int wq_internal_plan_ld(int M, int N, int K, int bits, int group, int sms, int smem_optin,
                        int64_t* out) {
  wqh::DeviceInfo dev;
  dev.sms = sms;
  dev.max_smem_optin = smem_optin;
  wqh::LdPlan plan;
  if (!wqh::plan_ld(M, N, K, bits, group, dev, &plan, 0)) return 0;
  const wq::ld::Params& p = plan.p;
  const int64_t v[] = {p.M,      p.N,      p.K,        p.ngroups, p.tiles,
                       p.xs_row_bytes, p.off_sx, p.off_sz, p.off_part, p.off_ring,
                       int64_t(plan.smem), plan.grid};
  for (size_t i = 0; i < sizeof(v) / sizeof(v[0]); ++i) out[i] = v[i];
  return 1;
}

// Tuning hook, not part of the public ABI: the build variant of the
// direct-load kernel used by the next calls (0 .. 5; see kLdVariants; a
// variant that does not fit a shape falls back to 0).  Returns the number
// of variants.
int wq_internal_set_ld_variant(int variant) {
  if (variant >= 0 && variant < wqh::kNumLdVariants) wqh::g_ld_variant = variant;
  return wqh::kNumLdVariants;
}

}  // extern "C"
