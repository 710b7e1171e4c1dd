// k_gemm.cu -- plan and launch of the prefill tensor-core matmul (gemm.cuh).
#include <algorithm>

#include "host.h"
#include "gemm.cuh"

namespace wqh {
namespace {

struct GemmPlan {
  wq::gemm::Params p;
  int grid = 1;
  size_t smem = 0;
};

// Shared-memory layout of the prefill kernel; false if the shape is outside
// its scope (group 64 or 128, K a multiple of 64 with at most 256 groups, a
// multiple of 8 groups per row, the tile's metadata resident next to the
// ring).
bool plan_gemm(int M, int N, int K, int bits, int group, bool symmetric, const DeviceInfo& dev,
               GemmPlan* plan) {
  using namespace wq::gemm;
  auto round_up = [](size_t a, size_t b) { return (a + b - 1) / b * b; };
  if (group != 64 && group != 128) return false;
  if (K % kBK != 0 || K % group != 0) return false;
  const int ngroups = K / group;
  if (ngroups > 256 || ngroups % 8 != 0) return false;
  wq::gemm::Params& p = plan->p;
  p = wq::gemm::Params{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.ngroups = ngroups;
  p.tiles_m = (M + kBM - 1) / kBM;
  p.codes_stage_bytes = uint32_t(kBN * kBK * bits / 8);
  p.meta_bytes = uint32_t(kBN * ngroups * 2);
  p.off_a = 1024;
  p.off_b = p.off_a + uint32_t(kStages * kTileBytes);
  p.off_codes = p.off_b + uint32_t(kStages * kTileBytes);
  p.off_meta_s = p.off_codes + uint32_t(kStages) * p.codes_stage_bytes;
  p.off_meta_z = p.off_meta_s + uint32_t(round_up(p.meta_bytes, 128));
  p.off_stab = p.off_meta_z + (symmetric ? 0u : uint32_t(round_up(p.meta_bytes, 128)));
  plan->smem = p.off_stab + size_t(ngroups) * kBN * 4;
  if (plan->smem > size_t(dev.max_smem_optin)) return false;
  const long long tiles = (long long)p.tiles_m * ((N + kBN - 1) / kBN);
  if (tiles > 0x7fffffffLL) return false;
  plan->grid = int(tiles);
  return true;
}

template <int BITS, bool SYM, int G>
struct GemmOp {
  static cudaError_t run(GemmPlan* plan, const DeviceInfo* dev, const void* X, const void* c,
                         const void* sc, const void* z, cudaStream_t s) {
    if constexpr (G % wq::gemm::kBK != 0) {
      return cudaErrorNotSupported;
    } else {
      using namespace wq::gemm;
      auto kernel = &gemm_kernel<BITS, SYM, G>;
      static int configured[kMaxDevices] = {};
      {
        const cudaError_t e = configure_smem(kernel, configured, size_t(dev->max_smem_optin));
        if (e != cudaSuccess) return e;
      }
      const wq::gemm::Params& p = plan->p;
      CUtensorMap tx, tc, ts, tz;
      // X [M][K] bfloat16, boxes of 64 k x 128 rows, 128-byte swizzle
      if (!encode_2d_ex(&tx, X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, uint64_t(p.K), uint64_t(p.M),
                        uint32_t(kBK), uint32_t(kBM), CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
        return cudaErrorInvalidValue;
      const uint64_t row_bytes = uint64_t(p.K) * BITS / 8;
      if (!encode_2d(&tc, c, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, row_bytes, uint64_t(p.N),
                     uint32_t(kBK * BITS / 8), uint32_t(kBN)) ||
          !encode_2d(&ts, sc, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, uint64_t(p.ngroups),
                     uint64_t(p.N), uint32_t(p.ngroups), uint32_t(kBN)))
        return cudaErrorInvalidValue;
      std::memcpy(&tz, &ts, sizeof(ts));
      if (!SYM && !encode_2d(&tz, z, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, uint64_t(p.ngroups),
                             uint64_t(p.N), uint32_t(p.ngroups), uint32_t(kBN)))
        return cudaErrorInvalidValue;
      gemm_kernel<BITS, SYM, G><<<plan->grid, kThreads, plan->smem, s>>>(tx, tc, ts, tz, p);
      return cudaGetLastError();
    }
  }
};

}  // namespace

bool run_gemm(const MatmulArgs& a, cudaError_t* err) {
  GemmPlan gp;
  if (!plan_gemm(a.M, a.N, a.K, a.bits, a.group, a.sym, a.dev, &gp)) return false;
  if (a.y_bf16)
    gp.p.Y_bf16 = static_cast<__nv_bfloat16*>(a.Y);
  else
    gp.p.Y_f32 = static_cast<float*>(a.Y);
  *err = dispatch_format<GemmOp>(a.bits, a.sym, a.group, &gp, &a.dev, a.X, a.codes, a.scales,
                                 a.zeros, a.stream);
  return true;
}

}  // namespace wqh

extern "C" {

// Test hook, not part of the public ABI: the prefill plan, written to
// out[0..14] (see tests/test_plan_gemm.py for the field order).  Returns 0
// if the shape is outside the prefill kernel's scope.
int wq_internal_plan_gemm(int M, int N, int K, int bits, int group, int symmetric,
                          int smem_optin, int64_t* out) {
  wqh::DeviceInfo dev;
  dev.sms = 148;
  dev.max_smem_optin = smem_optin;
  wqh::GemmPlan plan;
  if (!wqh::plan_gemm(M, N, K, bits, group, symmetric != 0, dev, &plan)) return 0;
  const wq::gemm::Params& p = plan.p;
  const int64_t v[] = {p.M, p.N, p.K, p.ngroups, p.tiles_m, p.codes_stage_bytes, p.meta_bytes,
                       p.off_a, p.off_b, p.off_codes, p.off_meta_s, p.off_meta_z, p.off_stab,
                       int64_t(plan.smem), plan.grid};
  for (size_t i = 0; i < sizeof(v) / sizeof(v[0]); ++i) out[i] = v[i];
  return 1;
}

}  // extern "C"
