// k_gemv.cu -- plan and launch of the cluster-split small-batch matmul
// (gemv.cuh).
#include <algorithm>

#include "host.h"
#include "gemv.cuh"

namespace wqh {
namespace {

using wq::gemv::Params;

struct GemvPlan {
  Params p;
  int C = 1;
  int grid = 1;
  size_t smem = 0;
};

// Shared-memory layout and work split for one call with K split over C
// cluster ranks and `bpw` boxes per warp and stage.  False if it does not fit
// with at least `min_depth` ring stages.
bool plan_gemv_with(int M, int N, int K, int bits, int group, const DeviceInfo& dev,
                    int cluster_cap, int C, int bpw, int min_depth, int red_bufs, bool pad,
                    GemvPlan* plan) {
  auto round_up = [](int a, int b) { return (a + b - 1) / b * b; };
  const int box_k = wq::gemv::kBoxRowBytes * 8 / bits;
  const int granule = std::max(box_k, group);
  const int tiles = (N + 15) / 16;
  const size_t budget = size_t(dev.max_smem_optin);
  const int MT = M <= 8 ? 1 : (M <= 16 ? 2 : 4);

  const int kc = round_up((K + C - 1) / C, granule);
  C = (K + kc - 1) / kc;  // ranks that have work
  int skw = wq::gemv::kNumConsumerWarps;
  while (skw > 1 && skw * box_k * bpw > kc) skw /= 2;
  if (skw * box_k * bpw > kc && bpw > 1) return false;
  const int RT = wq::gemv::kNumConsumerWarps / skw;
  const int stage_k = skw * bpw * box_k;
  const int sg = stage_k / group;
  const int ngroups = K / group;

  Params& p = plan->p;
  p.M = M;
  p.N = N;
  p.K = K;
  p.ngroups = ngroups;
  p.row_tiles = tiles;
  p.RT = RT;
  p.SKW = skw;
  p.BPW = bpw;
  p.items = (tiles + RT - 1) / RT;
  p.kc = kc;
  p.stage_k = stage_k;
  p.stages_per_item = (kc + stage_k - 1) / stage_k;
  p.meta_tma = (ngroups % 8 == 0 && sg % 8 == 0 && (kc / group) % 8 == 0) ? 1 : 0;

  // rows of a stage: stage_k*bits/8 bytes, padded to an odd multiple of 64;
  // whole-row stages (one cluster rank, one stage of all K) stay dense so the
  // item arrives by single bulk copies
  const uint32_t seg = uint32_t(stage_k * bits / 8);
  p.contig = (C == 1 && stage_k == K && p.meta_tma) ? 1 : 0;
  p.row_stride = seg + (pad && !p.contig && (seg / 64) % 2 == 0 ? 64u : 0u);
  const uint32_t codes_bytes = uint32_t(round_up(int(RT * 16 * p.row_stride), 128));
  const uint32_t meta_bytes = uint32_t(2 * RT * 16 * sg * 2);  // scales + zeros
  p.meta_offset = codes_bytes;
  p.stage_bytes = uint32_t(round_up(int(codes_bytes + meta_bytes), 1024));

  const size_t off = 1024;  // barriers + flags
  int clusters = std::max(1, dev.sms / C);
  if (cluster_cap > 0) clusters = std::min(clusters, cluster_cap);
  const int items_per_cluster_max = (p.items + clusters - 1) / clusters;
  // activation rows: 2*kc bytes padded to an odd multiple of 64 B so that
  // rows m and m+1 fall in different shared-memory bank halves
  p.x_row_stride = uint32_t(2 * kc + (pad && ((2 * kc) / 64) % 2 == 0 ? 64 : 0));
  const size_t fixed_x = size_t(round_up(int(p.x_row_stride) * (M + 1), 128));  // + a zero row
  const size_t fixed_sx = size_t(round_up((kc / group) * 8 * MT * 4, 128));
  // red_bufs == 0: one partial-sum slot per item of the CTA (no per-item barrier)
  p.red_bufs = red_bufs;
  const int red_slots = red_bufs == 0 ? items_per_cluster_max : red_bufs;
  const size_t fixed_red = size_t(round_up(red_slots * 16 * 16 * M * 4, 128));
  const size_t fixed_part =
      C > 1 ? size_t(round_up(items_per_cluster_max * RT * 16 * M * 4, 128)) : 0;
  const size_t fixed = off + fixed_x + fixed_sx + fixed_red + fixed_part;
  if (fixed + size_t(min_depth) * p.stage_bytes > budget) return false;
  int depth = int((budget - fixed) / p.stage_bytes);
  depth = std::min(depth, 32);
  // no point holding more stages than the CTA will ever consume
  depth = std::min(depth, std::max(2, items_per_cluster_max * p.stages_per_item));
  p.depth = depth;
  p.off_ring = uint32_t(off);
  p.off_x = uint32_t(off + size_t(depth) * p.stage_bytes);
  p.off_sx = uint32_t(p.off_x + fixed_x);
  p.off_red = uint32_t(p.off_sx + fixed_sx);
  p.off_part = uint32_t(p.off_red + fixed_red);
  plan->smem = p.off_part + fixed_part;
  plan->C = C;
  plan->grid = std::min(p.items, clusters) * C;
  return true;
}

// Choose the cluster split and stage size.  K is split across a cluster when
// there are too few row tiles to fill the SMs, or when the activations would
// not fit in shared memory; stages shrink before the ring gets shallow.
// Tuning hook (internal, off by default): force the cluster split, boxes per
// warp and ring depth of the next plans; 0 keeps the heuristic's choice.
int g_force_C = 0, g_force_bpw = 0, g_force_depth = 0;

bool plan_gemv(int M, int N, int K, int bits, int group, const DeviceInfo& dev, int cluster_cap,
               GemvPlan* plan) {
  const int tiles = (N + 15) / 16;
  if (g_force_C > 0 || g_force_bpw > 0) {
    const int C = g_force_C > 0 ? g_force_C : 1;
    const int bpw = g_force_bpw > 0 ? g_force_bpw : 1;
    for (int red_bufs : {2, 1})
      if (plan_gemv_with(M, N, K, bits, group, dev, cluster_cap, C, bpw, 2, red_bufs, true, plan)) {
        if (g_force_depth > 0 && g_force_depth < plan->p.depth) {
          const int d = g_force_depth;
          const uint32_t shift = uint32_t(plan->p.depth - d) * plan->p.stage_bytes;
          plan->p.depth = d;
          plan->p.off_x -= shift;
          plan->p.off_sx -= shift;
          plan->p.off_red -= shift;
          plan->p.off_part -= shift;
          plan->smem -= shift;
        }
        return true;
      }
    return false;
  }
  const int sms = dev.sms;
  int C0 = 1;
  if (tiles < 3 * sms) C0 = 2;
  if (tiles < sms) C0 = 4;
  if (tiles < sms / 4) C0 = 8;
  const int bpw_min = (bits == 8 && group == 128) ? 2 : 1;
  const int bpw_max = bits == 8 ? 4 : 2;
  for (int min_depth : {3, 2}) {
    for (int red_bufs : {0, 2, 1}) {
      for (int C = C0; C <= 16; C *= 2) {
        const int box_k = wq::gemv::kBoxRowBytes * 8 / bits;
        const int granule = std::max(box_k, group);
        const int kc = (((K + C - 1) / C) + granule - 1) / granule * granule;
        if (size_t(kc) * M * 2 > 128 * 1024 && C < 16) continue;
        for (int bpw = bpw_max; bpw >= bpw_min; bpw /= 2)
          for (bool pad : {true, false})  // unpadded rows (bank conflicts) only as a last resort
            if (plan_gemv_with(M, N, K, bits, group, dev, cluster_cap, C, bpw, min_depth, red_bufs,
                               pad, plan))
              return true;
      }
    }
  }
  return false;
}

template <int BITS, bool SYM, int G, int MT, int MEFF, bool FAST>
cudaError_t launch_gemv_t(GemvPlan& plan, const DeviceInfo& dev, const void* codes,
                          const void* scales, const void* zeros, cudaStream_t s, bool pdl) {
  auto kernel = &wq::gemv::gemv_kernel<BITS, SYM, G, MT, MEFF, FAST>;
  static int configured_smem[kMaxDevices] = {};  // per instantiation and device
  {
    int device = 0;
    cudaGetDevice(&device);
    if (device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
    if (configured_smem[device] == 0) {
      cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
    }
    const cudaError_t e = configure_smem(kernel, configured_smem, size_t(dev.max_smem_optin));
    if (e != cudaSuccess) return e;
  }

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attrs[2];
  cfg.blockDim = dim3(wq::gemv::kThreads, 1, 1);
  cfg.stream = s;
  if (plan.C > 1) {
    // Size the grid to the clusters that can be resident at once.
    attrs[0].id = cudaLaunchAttributeClusterDimension;
    attrs[0].val.clusterDim.x = unsigned(plan.C);
    attrs[0].val.clusterDim.y = 1;
    attrs[0].val.clusterDim.z = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(unsigned(plan.grid), 1, 1);
    cfg.dynamicSmemBytes = plan.smem;
    int max_clusters = 0;
    cudaError_t e = cudaOccupancyMaxActiveClusters(&max_clusters, kernel, &cfg);
    if (e != cudaSuccess) return e;
    if (max_clusters < 1) return cudaErrorNotSupported;
    if (plan.grid / plan.C > max_clusters) {
      const Params keep = plan.p;
      if (!plan_gemv(keep.M, keep.N, keep.K, BITS, G, dev, max_clusters, &plan))
        return cudaErrorNotSupported;
      plan.p.X = keep.X;
      plan.p.Y = keep.Y;
      plan.p.scales = keep.scales;
      plan.p.zeros = keep.zeros;
      plan.p.codes = keep.codes;
      plan.p.y_bf16 = keep.y_bf16;
    }
  }
  cfg.gridDim = dim3(unsigned(plan.grid), 1, 1);
  cfg.dynamicSmemBytes = plan.smem;
  if (pdl) {
    attrs[cfg.numAttrs].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[cfg.numAttrs].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attrs;
    ++cfg.numAttrs;
  }

  const Params& p = plan.p;
  const int row_bytes = p.K * BITS / 8;
  CUtensorMap tc, ts, tz;
  const int sg = p.stage_k / G;
  if (!encode_2d(&tc, codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, uint64_t(row_bytes),
                 uint64_t(p.N), wq::gemv::kBoxRowBytes, wq::gemv::kBoxRows))
    return cudaErrorInvalidValue;
  std::memcpy(&ts, &tc, sizeof(tc));
  std::memcpy(&tz, &tc, sizeof(tc));
  if (p.meta_tma) {
    if (!encode_2d(&ts, scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, uint64_t(p.ngroups),
                   uint64_t(p.N), uint32_t(sg), wq::gemv::kBoxRows))
      return cudaErrorInvalidValue;
    if (!SYM && !encode_2d(&tz, zeros, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, uint64_t(p.ngroups),
                           uint64_t(p.N), uint32_t(sg), wq::gemv::kBoxRows))
      return cudaErrorInvalidValue;
  }
  return cudaLaunchKernelEx(&cfg, kernel, tc, ts, tz, p);
}

template <int BITS, bool SYM, int G>
struct GemvOp {
  static cudaError_t run(GemvPlan* plan, const DeviceInfo* dev, const void* c, const void* sc,
                         const void* z, cudaStream_t s, bool pdl) {
    // M <= 8: one n8 tile whose columns hold up to 8/MEFF groups of MEFF rows
    const int M = plan->p.M;
    // the unrolled path: one stage per item with the format's natural box count
    const bool fast = M <= 8 && plan->p.stages_per_item == 1 &&
                      plan->p.BPW == wq::gemv::FastShape<BITS>::kBPW;
    if (fast) {
      if (M == 1) return launch_gemv_t<BITS, SYM, G, 1, 1, true>(*plan, *dev, c, sc, z, s, pdl);
      if (M == 2) return launch_gemv_t<BITS, SYM, G, 1, 2, true>(*plan, *dev, c, sc, z, s, pdl);
      if (M <= 4) return launch_gemv_t<BITS, SYM, G, 1, 4, true>(*plan, *dev, c, sc, z, s, pdl);
      return launch_gemv_t<BITS, SYM, G, 1, 8, true>(*plan, *dev, c, sc, z, s, pdl);
    }
    if (M == 1) return launch_gemv_t<BITS, SYM, G, 1, 1, false>(*plan, *dev, c, sc, z, s, pdl);
    if (M == 2) return launch_gemv_t<BITS, SYM, G, 1, 2, false>(*plan, *dev, c, sc, z, s, pdl);
    if (M <= 4) return launch_gemv_t<BITS, SYM, G, 1, 4, false>(*plan, *dev, c, sc, z, s, pdl);
    if (M <= 8) return launch_gemv_t<BITS, SYM, G, 1, 8, false>(*plan, *dev, c, sc, z, s, pdl);
    if (M <= 16) return launch_gemv_t<BITS, SYM, G, 2, 8, false>(*plan, *dev, c, sc, z, s, pdl);
    return launch_gemv_t<BITS, SYM, G, 4, 8, false>(*plan, *dev, c, sc, z, s, pdl);
  }
};

}  // namespace

bool run_gemv(const MatmulArgs& a, cudaError_t* err) {
  GemvPlan plan;
  if (!plan_gemv(a.M, a.N, a.K, a.bits, a.group, a.dev, 0, &plan)) return false;
  plan.p.X = static_cast<const __nv_bfloat16*>(a.X);
  plan.p.Y = a.Y;
  plan.p.scales = static_cast<const __half*>(a.scales);
  plan.p.zeros = static_cast<const __half*>(a.zeros);
  plan.p.codes = static_cast<const uint8_t*>(a.codes);
  plan.p.y_bf16 = a.y_bf16 ? 1 : 0;
  *err = dispatch_format<GemvOp>(a.bits, a.sym, a.group, &plan, &a.dev, a.codes, a.scales,
                                 a.zeros, a.stream, a.pdl);
  return true;
}

}  // namespace wqh

extern "C" {

// Tuning hook, not part of the public ABI (see g_force_C).
void wq_internal_force_gemv_plan(int C, int bpw, int depth) {
  wqh::g_force_C = C;
  wqh::g_force_bpw = bpw;
  wqh::g_force_depth = depth;
}

// Test hook, not part of the public ABI: the matmul plan for a device with
// `sms` SMs and `smem_optin` bytes of shared memory per block, written to
// out[0..27] (see tests/test_plan.py for the field order).  Returns 0 if no
// plan exists.
int wq_internal_plan_gemv(int M, int N, int K, int bits, int group, int sms, int smem_optin,
                          int cluster_cap, int64_t* out) {
  wqh::DeviceInfo dev;
  dev.sms = sms;
  dev.max_smem_optin = smem_optin;
  wqh::GemvPlan plan;
  if (!wqh::plan_gemv(M, N, K, bits, group, dev, cluster_cap, &plan)) return 0;
  const wq::gemv::Params& p = plan.p;
  const int64_t v[] = {p.M,       p.N,           p.K,         p.ngroups,     p.row_tiles,
                       p.items,   p.RT,          p.SKW,       p.BPW,         p.depth,
                       p.kc,      p.stage_k,     p.stages_per_item, p.meta_tma, p.stage_bytes,
                       p.meta_offset, p.off_ring, p.off_x,    p.off_sx,      p.off_red,
                       p.off_part, int64_t(plan.smem), plan.C, plan.grid, p.x_row_stride,
                       p.red_bufs, p.row_stride, p.contig};
  for (size_t i = 0; i < sizeof(v) / sizeof(v[0]); ++i) out[i] = v[i];
  return 1;
}

}  // extern "C"
