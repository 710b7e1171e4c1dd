// k_q4k.cu -- launchers of the nested-superblock (4.5 bits per weight)
// quantize and fused small-batch matmul kernels.
#include <algorithm>

#include "host.h"
#include "q4k.cuh"
#include "q4k_ks.cuh"

namespace wqh {

// 0: the tensor-core kernel where it applies (M = 1, K = 4096), else the
// scalar one; 1: always the scalar one.  Tuning and test hook.
int g_q4k_kernel = 0;

cudaError_t run_q4k_quantize(const void* W, int64_t nblocks, void* blocks, cudaStream_t s,
                             int sms) {
  const int64_t grid =
      std::max<int64_t>(1, std::min<int64_t>((nblocks + 7) / 8, int64_t(sms) * 16));
  wq::q4k::quantize_kernel<<<unsigned(grid), 256, 0, s>>>(static_cast<const __half*>(W),
                                                           nblocks,
                                                           static_cast<uint8_t*>(blocks));
  return cudaGetLastError();
}

namespace {

struct Q4ksPlan {
  wq::q4ks::Params p;
  int grid = 1;
  int depth = 2;
  size_t smem = 0;
};

// The tensor-core kernel's scope: M = 1, K = 4096.  One CTA per SM (at most
// one per 16-row tile), at most half an SM of shared memory; the ring is as
// deep (2 to 4 units per warp) as that allows.
bool plan_q4ks(int M, int N, int K, const DeviceInfo& dev, Q4ksPlan* plan) {
  using namespace wq::q4ks;
  if (M != 1 || K != kK || N < 1) return false;
  wq::q4ks::Params& p = plan->p;
  p = wq::q4ks::Params{};
  p.N = N;
  p.tiles = (N + kTileRows - 1) / kTileRows;
  plan->grid = std::min(p.tiles, dev.sms);
  const size_t max_tiles = size_t((p.tiles + plan->grid - 1) / plan->grid);
  p.off_part = 0;
  p.off_ring = uint32_t(round_up(max_tiles * kWarps * kTileRows * 4, 128));
  const size_t half_sm = size_t(dev.max_smem_optin) / 2 - 1024;
  int depth = 4;
  while (depth >= 2 && p.off_ring + size_t(kWarps) * depth * kUnitBytes > half_sm) --depth;
  if (depth < 2) return false;
  plan->depth = depth;
  plan->smem = p.off_ring + size_t(kWarps) * depth * kUnitBytes;
  return true;
}

template <int DEPTH>
cudaError_t launch_q4ks(Q4ksPlan* plan, const DeviceInfo& dev, cudaStream_t s) {
  // the build without the bounds-checked copies where every tile is whole
  const bool whole = plan->p.N % wq::q4ks::kTileRows == 0;
  auto kernel = whole ? &wq::q4ks::gemv_q4k_kernel<DEPTH, false>
                      : &wq::q4ks::gemv_q4k_kernel<DEPTH, true>;
  static int configured[2][kMaxDevices] = {};  // per build
  const cudaError_t e = configure_smem(kernel, configured[whole ? 0 : 1], size_t(dev.max_smem_optin));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attrs[1];
  cfg.gridDim = dim3(unsigned(plan->grid));
  cfg.blockDim = dim3(wq::q4ks::kThreads);
  cfg.dynamicSmemBytes = plan->smem;
  cfg.stream = s;
  if (plan->p.pdl) {
    attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, kernel, plan->p);
}

}  // namespace

cudaError_t run_q4k_matmul(const void* X, int M, const void* blocks, int N, int K, void* Y,
                           bool y_bf16, bool pdl, cudaStream_t s, int sms) {
  DeviceInfo dev;
  Q4ksPlan qp;
  if (g_q4k_kernel == 0 && device_info(&dev) && plan_q4ks(M, N, K, dev, &qp)) {
    qp.p.X = static_cast<const __nv_bfloat16*>(X);
    qp.p.Y = Y;
    qp.p.blocks = static_cast<const uint8_t*>(blocks);
    qp.p.y_bf16 = y_bf16 ? 1 : 0;
    qp.p.pdl = pdl ? 1 : 0;
    switch (qp.depth) {
      case 4: return launch_q4ks<4>(&qp, dev, s);
      case 3: return launch_q4ks<3>(&qp, dev, s);
      default: return launch_q4ks<2>(&qp, dev, s);
    }
  }
  const int64_t grid = std::max<int64_t>(1, std::min<int64_t>((N + 7) / 8, int64_t(sms) * 8));
  const auto* x = static_cast<const __nv_bfloat16*>(X);
  const auto* b = static_cast<const uint8_t*>(blocks);
  const int yb = y_bf16 ? 1 : 0;
  const unsigned g = unsigned(grid);
  if (M == 1)
    wq::q4k::matmul_kernel<1><<<g, 256, 0, s>>>(x, M, b, N, K, Y, yb);
  else if (M == 2)
    wq::q4k::matmul_kernel<2><<<g, 256, 0, s>>>(x, M, b, N, K, Y, yb);
  else if (M <= 4)
    wq::q4k::matmul_kernel<4><<<g, 256, 0, s>>>(x, M, b, N, K, Y, yb);
  else
    wq::q4k::matmul_kernel<8><<<g, 256, 0, s>>>(x, M, b, N, K, Y, yb);
  return cudaGetLastError();
}

}  // namespace wqh

extern "C" {

// Tuning and test hook, not part of the public ABI: 1 forces the scalar
// superblock matmul kernel, 0 lets wq_q4k_matmul choose.
void wq_internal_set_q4k_kernel(int choice) { wqh::g_q4k_kernel = choice == 1 ? 1 : 0; }

// Test hook, not part of the public ABI: the tensor-core superblock kernel's
// plan for a device with `sms` SMs and `smem_optin` bytes of shared memory per
// block, written to out[0..6] (N, tiles, off_part, off_ring, depth, smem,
// grid).  Returns 0 if the shape is outside the kernel's scope.
int wq_internal_plan_q4ks(int M, int N, int K, int sms, int smem_optin, int64_t* out) {
  wqh::DeviceInfo dev;
  dev.sms = sms;
  dev.max_smem_optin = smem_optin;
  wqh::Q4ksPlan plan;
  if (!wqh::plan_q4ks(M, N, K, dev, &plan)) return 0;
  const wq::q4ks::Params& p = plan.p;
  const int64_t v[] = {p.N, p.tiles, p.off_part, p.off_ring, plan.depth, int64_t(plan.smem),
                       plan.grid};
  for (size_t i = 0; i < sizeof(v) / sizeof(v[0]); ++i) out[i] = v[i];
  return 1;
}

}  // extern "C"
