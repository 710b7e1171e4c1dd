// k_sk.cu -- plan and launch of the balanced small-batch matmul
// (gemv_sk.cuh).
#include <algorithm>

#include "host.h"
#include "gemv_sk.cuh"

namespace wqh {
namespace {

// Test hooks of the timeout path (wq_internal_timeout_test).
int g_test_skip_publish = -1;
unsigned long long g_flag_wait_ns = wq::kWaitLimitNs;

struct SkPlan {
  wq::sk::Params p;
  int grid = 1;
  size_t smem = 0;
  int resident = 0;     // B fragments loaded once (all of K in one 16-slice block)
  int max_stages = 0;   // most stages any CTA walks
  int max_tiles = 0;    // most row tiles any CTA touches
};

// Plan the balanced kernel; false if the shape is outside its scope (M <= 8,
// K a multiple of one 128-byte slice of codes, groups a multiple of 8 per
// row, activations resident in shared memory next to a ring of >= 3 stages).
bool plan_sk(int M, int N, int K, int bits, int group, bool symmetric, const DeviceInfo& dev,
             bool split, SkPlan* plan) {
  using namespace wq::sk;
  auto round_up = [](size_t a, size_t b) { return (a + b - 1) / b * b; };
  if (M < 1 || M > 8) return false;
  const int slice_k = kSliceBytes * 8 / bits;
  if (K % slice_k != 0 || group > slice_k) return false;
  const int ngroups = K / group;
  if (ngroups % kBlockGroups != 0) return false;
  const int nk = K / slice_k;
  const int tiles = (N + kRows - 1) / kRows;
  const long long units = (long long)tiles * nk;
  const int gps = slice_k / group;
  const int meta_blocks = kSlicesPerStage * gps / kBlockGroups;

  wq::sk::Params& p = plan->p;
  p = wq::sk::Params{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.ngroups = ngroups;
  p.tiles = tiles;
  p.nk = nk;
  p.split = split ? 1 : 0;
  p.ctas = int(split ? std::min<long long>(dev.sms, units) : std::min(dev.sms, tiles));
  p.waves = tiles / p.ctas;
  p.tail_tiles = tiles % p.ctas;

  // walk every CTA's stages as the kernel does
  int max_stages = 0, max_tiles = 0;
  for (int c = 0; c < p.ctas; ++c) {
    int n = 0, nt = 0;
    for_each_stage(c, p, [&](const Stage&, bool tile_end) {
      ++n;
      nt += tile_end ? 1 : 0;
    });
    max_stages = std::max(max_stages, n);
    max_tiles = std::max(max_tiles, nt);
  }
  plan->max_stages = max_stages;
  plan->max_tiles = max_tiles;
  plan->resident = nk <= kSlicesPerStage ? 1 : 0;
  p.box_slices = std::min(kSlicesPerStage, nk);
  p.box_blocks = std::min(meta_blocks, ngroups / kBlockGroups);

  const size_t meta_bytes = size_t(meta_blocks) * kBlockBytes * (symmetric ? 1 : 2);
  p.stage_bytes = uint32_t(round_up(kCodesStage + meta_bytes, 1024));
  // activation rows an odd multiple of 64 bytes apart (bank halves alternate)
  p.x_stride = uint32_t(2 * K + (((2 * K) / 64) % 2 == 0 ? 64 : 0));
  const size_t fixed_x = round_up(size_t(M) * p.x_stride, 128);
  const size_t fixed_sx = round_up(size_t(M) * ngroups * 8, 128);  // {2^-sigma, sum} per group
  const size_t per_slot = size_t(kWarps) * kRows * M * 4;
  p.red_mode = size_t(max_tiles) * per_slot <= 32 * 1024 ? 0 : 2;
  const size_t fixed_red = round_up((p.red_mode == 0 ? max_tiles : 2) * per_slot, 128);
  const size_t head = 1024;  // barriers and the abort flag
  const size_t fixed = head + fixed_x + fixed_sx + fixed_red;
  const size_t budget = size_t(dev.max_smem_optin);
  if (fixed + p.stage_bytes > budget) return false;
  int depth = int((budget - fixed) / p.stage_bytes);
  depth = std::min(depth, std::min(kMaxDepth, max_stages));
  if (depth < std::min(3, max_stages)) return false;
  p.depth = depth;
  p.off_ring = uint32_t(head);
  p.off_x = uint32_t(head + size_t(depth) * p.stage_bytes);
  p.off_sx = uint32_t(p.off_x + fixed_x);
  p.off_red = uint32_t(p.off_sx + fixed_sx);
  plan->smem = p.off_red + fixed_red;
  plan->grid = p.ctas;
  return true;
}

template <int BITS, bool SYM, int G, int MEFF, bool RES>
cudaError_t launch_sk_t(SkPlan& plan, const DeviceInfo& dev, const void* codes,
                        const void* scales, const void* zeros, cudaStream_t s, bool pdl) {
  using namespace wq::sk;
  auto kernel = &gemv_sk_kernel<BITS, SYM, G, MEFF, RES>;
  static int configured[kMaxDevices] = {};
  {
    const cudaError_t e = configure_smem(kernel, configured, size_t(dev.max_smem_optin));
    if (e != cudaSuccess) return e;
  }
  const wq::sk::Params& p = plan.p;
  const uint64_t row_bytes = uint64_t(p.K) * BITS / 8;
  const uint64_t nblk = uint64_t(p.ngroups) / kBlockGroups;
  CUtensorMap c16, c1, s16, s1, z16, z1;
  if (!encode_3d(&c16, codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, kSliceBytes, uint64_t(p.N),
                 uint64_t(p.nk), row_bytes, kSliceBytes, kSliceBytes, kRows,
                 uint32_t(p.box_slices), CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B) ||
      !encode_3d(&c1, codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, kSliceBytes, uint64_t(p.N),
                 uint64_t(p.nk), row_bytes, kSliceBytes, kSliceBytes, kRows, 1,
                 CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B) ||
      !encode_3d(&s16, scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, kBlockGroups, uint64_t(p.N), nblk,
                 uint64_t(p.ngroups) * 2, kBlockGroups * 2, kBlockGroups, kRows,
                 uint32_t(p.box_blocks), CU_TENSOR_MAP_SWIZZLE_NONE,
                 CU_TENSOR_MAP_L2_PROMOTION_NONE) ||
      !encode_3d(&s1, scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, kBlockGroups, uint64_t(p.N), nblk,
                 uint64_t(p.ngroups) * 2, kBlockGroups * 2, kBlockGroups, kRows, 1,
                 CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE))
    return cudaErrorInvalidValue;
  std::memcpy(&z16, &s16, sizeof(s16));
  std::memcpy(&z1, &s1, sizeof(s1));
  if (!SYM &&
      (!encode_3d(&z16, zeros, CU_TENSOR_MAP_DATA_TYPE_UINT16, kBlockGroups, uint64_t(p.N), nblk,
                  uint64_t(p.ngroups) * 2, kBlockGroups * 2, kBlockGroups, kRows,
                  uint32_t(p.box_blocks), CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE) ||
       !encode_3d(&z1, zeros, CU_TENSOR_MAP_DATA_TYPE_UINT16, kBlockGroups, uint64_t(p.N), nblk,
                  uint64_t(p.ngroups) * 2, kBlockGroups * 2, kBlockGroups, kRows, 1,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE)))
    return cudaErrorInvalidValue;

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attrs[1];
  cfg.gridDim = dim3(unsigned(plan.grid), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = plan.smem;
  cfg.stream = s;
  plan.p.pdl = pdl ? 1 : 0;
  if (pdl) {
    attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, kernel, c16, c1, s16, s1, z16, z1, plan.p);
}

template <int BITS, bool SYM, int G>
struct SkOp {
  static cudaError_t run(SkPlan* plan, const DeviceInfo* dev, const void* c, const void* sc,
                         const void* z, cudaStream_t s, bool pdl) {
    const int M = plan->p.M;
    if (plan->resident) {
      if (M == 1) return launch_sk_t<BITS, SYM, G, 1, true>(*plan, *dev, c, sc, z, s, pdl);
      if (M == 2) return launch_sk_t<BITS, SYM, G, 2, true>(*plan, *dev, c, sc, z, s, pdl);
      if (M <= 4) return launch_sk_t<BITS, SYM, G, 4, true>(*plan, *dev, c, sc, z, s, pdl);
      return launch_sk_t<BITS, SYM, G, 8, true>(*plan, *dev, c, sc, z, s, pdl);
    }
    if (M == 1) return launch_sk_t<BITS, SYM, G, 1, false>(*plan, *dev, c, sc, z, s, pdl);
    if (M == 2) return launch_sk_t<BITS, SYM, G, 2, false>(*plan, *dev, c, sc, z, s, pdl);
    if (M <= 4) return launch_sk_t<BITS, SYM, G, 4, false>(*plan, *dev, c, sc, z, s, pdl);
    return launch_sk_t<BITS, SYM, G, 8, false>(*plan, *dev, c, sc, z, s, pdl);
  }
};

}  // namespace

bool run_sk(const MatmulArgs& a, bool split, cudaError_t* err) {
  SkPlan sk;
  if (!plan_sk(a.M, a.N, a.K, a.bits, a.group, a.sym, a.dev, split, &sk)) return false;
  sk.p.X = static_cast<const __nv_bfloat16*>(a.X);
  sk.p.Y = a.Y;
  sk.p.y_bf16 = a.y_bf16 ? 1 : 0;
  sk.p.test_skip_publish = g_test_skip_publish;
  sk.p.flag_wait_ns = g_flag_wait_ns;
  if (split) {
    sk.p.ws_flag = static_cast<unsigned int*>(a.workspace);
    sk.p.ws_part = reinterpret_cast<float*>(static_cast<uint8_t*>(a.workspace) +
                                            size_t(wq::sk::kWsCtasMax) * 4);
  }
  *err = dispatch_format<SkOp>(a.bits, a.sym, a.group, &sk, &a.dev, a.codes, a.scales, a.zeros,
                               a.stream, a.pdl);
  return true;
}

size_t sk_workspace_bytes() { return size_t(wq::sk::kWsCtasMax) * (wq::sk::kWsRowsMax * 4 + 4); }
int sk_workspace_ctas() { return wq::sk::kWsCtasMax; }

}  // namespace wqh

extern "C" {

// Test hook, not part of the public ABI: make the timeout path of the
// balanced kernel's split tiles run.  CTA `skip_publish_cta` (-1: none) then
// never publishes its partial sums, and the CTA that waits for them gives up
// after `wait_ns` nanoseconds (0 restores the default limit), records
// WQ_ERR_TIMEOUT and returns.  Only that wait is shortened: it follows the
// completion of every copy and product of the waiting CTA.
void wq_internal_timeout_test(int skip_publish_cta, unsigned long long wait_ns) {
  wqh::g_test_skip_publish = skip_publish_cta;
  wqh::g_flag_wait_ns = wait_ns > 0 ? wait_ns : wq::kWaitLimitNs;
}

// Test hook, not part of the public ABI: the balanced kernel's plan for a
// device with `sms` SMs and `smem_optin` bytes of shared memory per block,
// written to out[0..24] (see tests/test_plan_sk.py for the field order).
// Returns 0 if the shape is outside the kernel's scope.
int wq_internal_plan_sk(int M, int N, int K, int bits, int group, int symmetric, int sms,
                        int smem_optin, int split, int64_t* out) {
  wqh::DeviceInfo dev;
  dev.sms = sms;
  dev.max_smem_optin = smem_optin;
  wqh::SkPlan plan;
  if (!wqh::plan_sk(M, N, K, bits, group, symmetric != 0, dev, split != 0, &plan)) return 0;
  const wq::sk::Params& p = plan.p;
  const int64_t v[] = {p.M,           p.N,          p.K,           p.ngroups,   p.tiles,
                       p.nk,          p.waves,      p.ctas,        p.split,     p.depth,
                       p.red_mode,    p.stage_bytes, p.off_ring,   p.off_x,     p.off_sx,
                       p.off_red,     p.x_stride,   p.box_slices,  p.box_blocks, int64_t(plan.smem),
                       plan.grid,     plan.resident, plan.max_stages, plan.max_tiles,
                       p.tail_tiles};
  for (size_t i = 0; i < sizeof(v) / sizeof(v[0]); ++i) out[i] = v[i];
  return 1;
}

}  // extern "C"
