// wq.cu -- the C ABI declared in include/wq.h: argument checks, TMA
// descriptor encoding, launch configuration, kernel dispatch.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "wq.h"
#include "common.cuh"
#include "quantize.cuh"
#include "gemv.cuh"
#include "gemv_sk.cuh"
#include "gemm.cuh"
#include "gemv_ld.cuh"
#include "stream.cuh"
#include "q4k.cuh"

namespace {

using wq::gemv::Params;

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  int sms = 0;
  int max_smem_optin = 0;
};

DeviceInfo g_devices[kMaxDevices];
std::mutex g_mutex;

bool device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& d = g_devices[dev];
  if (d.sms == 0) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return false;
    if (cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin,
                               dev) != cudaSuccess)
      return false;
  }
  *out = d;
  return true;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D row-major tensor [rows][cols] of `elem_bytes`-byte elements.
bool encode_2d(CUtensorMap* map, const void* base, CUtensorMapDataType type, int elem_bytes,
               uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * uint64_t(elem_bytes)};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, type, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D view: dims {d0, d1, d2} (d0 innermost, contiguous), byte strides of d1
// and d2 (any order), box {b0, b1, b2}.
bool encode_3d(CUtensorMap* map, const void* base, CUtensorMapDataType type, uint64_t d0,
               uint64_t d1, uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t b0,
               uint32_t b1, uint32_t b2, CUtensorMapSwizzle swizzle,
               CUtensorMapL2promotion promotion) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride1, stride2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, type, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, promotion,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_format(int64_t N, int64_t K, int bits, int group) {
  if (bits != 4 && bits != 8) return false;
  if (group != 32 && group != 64 && group != 128) return false;
  if (N < 1 || K < 32 || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31)) return false;
  if (K % 32 != 0 || K % group != 0) return false;
  return true;
}

unsigned grid_for_elements(int64_t total, int sms) {
  const int64_t warps_needed = (total + 1023) / 1024;
  const int64_t blocks = (warps_needed + 7) / 8;
  return unsigned(std::max<int64_t>(1, std::min<int64_t>(blocks, int64_t(sms) * 16)));
}

// ---------------------------------------------------------------- quantize

template <int BITS, bool SYM, int G>
cudaError_t launch_quantize(const void* W, int64_t total, void* codes, void* scales, void* zeros,
                            cudaStream_t s, int sms) {
  wq::quantize_kernel<BITS, SYM, G><<<grid_for_elements(total, sms), 256, 0, s>>>(
      static_cast<const __half*>(W), total, static_cast<uint8_t*>(codes),
      static_cast<__half*>(scales), static_cast<__half*>(zeros));
  return cudaGetLastError();
}

template <int BITS, bool SYM, int G>
cudaError_t launch_dequantize(const void* codes, const void* scales, const void* zeros,
                              int64_t total, void* out, cudaStream_t s, int sms) {
  wq::dequantize_kernel<BITS, SYM, G><<<grid_for_elements(total, sms), 256, 0, s>>>(
      static_cast<const uint8_t*>(codes), static_cast<const __half*>(scales),
      static_cast<const __half*>(zeros), total, static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

template <template <int, bool, int> class F, typename... Args>
cudaError_t dispatch_format(int bits, bool sym, int group, Args... args) {
#define WQ_CASE(B, S, G)                                        \
  if (bits == B && sym == S && group == G) return F<B, S, G>::run(args...);
  WQ_CASE(4, false, 32) WQ_CASE(4, false, 64) WQ_CASE(4, false, 128)
  WQ_CASE(4, true, 32) WQ_CASE(4, true, 64) WQ_CASE(4, true, 128)
  WQ_CASE(8, false, 32) WQ_CASE(8, false, 64) WQ_CASE(8, false, 128)
  WQ_CASE(8, true, 32) WQ_CASE(8, true, 64) WQ_CASE(8, true, 128)
#undef WQ_CASE
  return cudaErrorInvalidValue;
}

template <int B, bool S, int G>
struct QuantizeOp {
  static cudaError_t run(const void* W, int64_t total, void* c, void* sc, void* z,
                         cudaStream_t s, int sms) {
    return launch_quantize<B, S, G>(W, total, c, sc, z, s, sms);
  }
};

template <int B, bool S, int G>
struct DequantizeOp {
  static cudaError_t run(const void* c, const void* sc, const void* z, int64_t total, void* out,
                         cudaStream_t s, int sms) {
    return launch_dequantize<B, S, G>(c, sc, z, total, out, s, sms);
  }
};

// ---------------------------------------------------------------- matmul

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
  int device = 0;
  cudaGetDevice(&device);
  if (device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
  if (configured_smem[device] == 0) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         dev.max_smem_optin);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    configured_smem[device] = dev.max_smem_optin;
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

// --------------------------------------------------- direct-load kernel

struct LdPlan {
  wq::ld::Params p;
  int grid = 1;
  size_t smem = 0;
};

// Plan the direct-load kernel: 4-bit codes in groups of 128 with K a
// multiple of 512 (groups come in pairs; a CTA's scales load in blocks of
// four), M <= 4; one CTA per SM (at most one per 8-row tile) with the
// activations, their group sums, the CTA's scales and zeros and the per-warp
// partial sums of its tiles in shared memory, next to the per-warp rings of
// codes.
bool plan_ld(int M, int N, int K, int bits, int group, const DeviceInfo& dev, LdPlan* plan) {
  using namespace wq::ld;
  if (bits != 4 || group != kGroup || M < 1 || M > kMaxM || N < 1 || K < 4 * kGroup ||
      K % (4 * kGroup) != 0)
    return false;
  auto round_up = [](size_t a, size_t b) { return (a + b - 1) / b * b; };
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
  p.off_ring = uint32_t(round_up(p.off_part + max_tiles * kWarps * kTileRows * size_t(M) * 4, 128));
  plan->smem = p.off_ring + size_t(kWarps) * kDepth * 1024;
  return plan->smem <= size_t(dev.max_smem_optin);
}

template <int BITS, bool SYM, int G>
struct LdOp {
  static cudaError_t run(LdPlan* plan, const DeviceInfo* dev, cudaStream_t s, bool pdl) {
    if constexpr (BITS != 4 || G != wq::ld::kGroup) {
      return cudaErrorInvalidValue;
    } else {
      const int M = plan->p.M;
      if (M == 1) return launch<1>(plan, dev, s, pdl);
      if (M == 2) return launch<2>(plan, dev, s, pdl);
      return launch<4>(plan, dev, s, pdl);
    }
  }

  template <int MT>
  static cudaError_t launch(LdPlan* plan, const DeviceInfo* dev, cudaStream_t s, bool pdl) {
    {
      auto kernel = &wq::ld::gemv_ld_kernel<SYM, MT>;
      static int configured[kMaxDevices] = {};
      int device = 0;
      cudaGetDevice(&device);
      if (device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
      if (!configured[device]) {
        const cudaError_t e = cudaFuncSetAttribute(
            kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dev->max_smem_optin);
        if (e != cudaSuccess) return e;
        configured[device] = 1;
      }
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
  }
};

// ------------------------------------------------------- balanced kernel

struct SkPlan {
  wq::sk::Params p;
  int grid = 1;
  size_t smem = 0;
  int resident = 0;     // B fragments loaded once (all of K in one 16-slice block)
  int max_stages = 0;   // most stages any CTA walks
  int max_tiles = 0;    // most row tiles any CTA touches
};

// Which small-batch kernel wq_matmul uses: 0 chooses, 1 forces the
// cluster-split kernel, 2 forces the balanced kernel, 3 forces it with split
// row tiles, 4 forces the direct-load kernel (tuning and tests).
int g_kernel_choice = 0;

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
  int device = 0;
  cudaGetDevice(&device);
  if (device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
  if (configured[device] == 0) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         dev.max_smem_optin);
    if (e != cudaSuccess) return e;
    configured[device] = 1;
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

// ------------------------------------------------------- prefill GEMM

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
      int device = 0;
      cudaGetDevice(&device);
      if (device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
      if (configured[device] == 0) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             dev->max_smem_optin);
        if (e != cudaSuccess) return e;
        configured[device] = 1;
      }
      const wq::gemm::Params& p = plan->p;
      CUtensorMap tx, tc, ts, tz;
      auto fn = tensor_map_encoder();
      if (!fn) return cudaErrorInvalidValue;
      {
        // X [M][K] bfloat16, boxes of 64 k x 128 rows, 128-byte swizzle
        cuuint64_t dims[2] = {cuuint64_t(p.K), cuuint64_t(p.M)};
        cuuint64_t strides[1] = {cuuint64_t(p.K) * 2};
        cuuint32_t box[2] = {uint32_t(kBK), uint32_t(kBM)};
        cuuint32_t estr[2] = {1, 1};
        if (fn(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(X), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
          return cudaErrorInvalidValue;
      }
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

// The last CUDA error a call returned (reported by an internal export).
cudaError_t g_last_cuda_error = cudaSuccess;

wq_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return WQ_OK;
  g_last_cuda_error = e;
  if (e == cudaErrorInvalidValue) return WQ_ERR_INVALID_ARG;
  if (e == cudaErrorNotSupported) return WQ_ERR_UNSUPPORTED;
  return WQ_ERR_CUDA;
}

}  // namespace

extern "C" {

size_t wq_codes_bytes(int64_t N, int64_t K, int bits) {
  if ((bits != 4 && bits != 8) || N < 1 || K < 1 || (K * bits) % 8 != 0) return 0;
  return size_t(N) * size_t(K) * size_t(bits) / 8;
}

size_t wq_meta_elems(int64_t N, int64_t K, int group) {
  if (group < 1 || N < 1 || K < 1 || K % group != 0) return 0;
  return size_t(N) * size_t(K / group);
}

wq_status wq_quantize(const void* W, int64_t N, int64_t K, int bits, int group, int symmetric,
                      void* codes, void* scales, void* zeros, wq_stream_t stream) {
  if (!valid_format(N, K, bits, group)) return WQ_ERR_INVALID_ARG;
  if (symmetric != 0 && symmetric != 1) return WQ_ERR_INVALID_ARG;
  if (!W || !codes || !scales || (symmetric ? zeros != nullptr : zeros == nullptr))
    return WQ_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(codes) || !aligned16(scales) || (zeros && !aligned16(zeros)))
    return WQ_ERR_ALIGNMENT;
  DeviceInfo dev;
  if (!device_info(&dev)) return WQ_ERR_CUDA;
  const cudaError_t e = dispatch_format<QuantizeOp>(bits, symmetric != 0, group, W, N * K, codes,
                                                    scales, zeros,
                                                    reinterpret_cast<cudaStream_t>(stream), dev.sms);
  return from_cuda(e);
}

wq_status wq_dequantize(const void* codes, const void* scales, const void* zeros, int64_t N,
                        int64_t K, int bits, int group, int symmetric, void* W_out,
                        wq_stream_t stream) {
  if (!valid_format(N, K, bits, group)) return WQ_ERR_INVALID_ARG;
  if (symmetric != 0 && symmetric != 1) return WQ_ERR_INVALID_ARG;
  if (!W_out || !codes || !scales || (symmetric ? zeros != nullptr : zeros == nullptr))
    return WQ_ERR_INVALID_ARG;
  if (!aligned16(W_out) || !aligned16(codes) || !aligned16(scales) ||
      (zeros && !aligned16(zeros)))
    return WQ_ERR_ALIGNMENT;
  DeviceInfo dev;
  if (!device_info(&dev)) return WQ_ERR_CUDA;
  const cudaError_t e =
      dispatch_format<DequantizeOp>(bits, symmetric != 0, group, codes, scales, zeros, N * K,
                                    W_out, reinterpret_cast<cudaStream_t>(stream), dev.sms);
  return from_cuda(e);
}

size_t wq_matmul_workspace_bytes(void) {
  return size_t(wq::sk::kWsCtasMax) * (wq::sk::kWsRowsMax * 4 + 4);
}

wq_status wq_matmul(const void* X, int64_t M, const void* codes, const void* scales,
                    const void* zeros, int64_t N, int64_t K, int bits, int group, int symmetric,
                    void* Y, int out_dtype, void* workspace, size_t workspace_bytes,
                    unsigned int flags, wq_stream_t stream) {
  if (!valid_format(N, K, bits, group) || M < 1 || M >= (int64_t(1) << 31))
    return WQ_ERR_INVALID_ARG;
  if (symmetric != 0 && symmetric != 1) return WQ_ERR_INVALID_ARG;
  if (out_dtype != WQ_OUT_F32 && out_dtype != WQ_OUT_BF16) return WQ_ERR_INVALID_ARG;
  if ((flags & ~unsigned(WQ_MATMUL_STATIC_WEIGHTS)) != 0) return WQ_ERR_INVALID_ARG;
  if (!X || !codes || !scales || !Y || (symmetric ? zeros != nullptr : zeros == nullptr))
    return WQ_ERR_INVALID_ARG;
  if (workspace == nullptr && workspace_bytes != 0) return WQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(codes) || !aligned16(scales) || !aligned16(Y) ||
      (zeros && !aligned16(zeros)) || (workspace && !aligned16(workspace)))
    return WQ_ERR_ALIGNMENT;
  DeviceInfo dev;
  if (!device_info(&dev)) return WQ_ERR_CUDA;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (M > 32) {
    // prefill: tensor-core GEMM on exact integer weights, binary32 group scaling
    GemmPlan gp;
    if (!plan_gemm(int(M), int(N), int(K), bits, group, symmetric != 0, dev, &gp))
      return WQ_ERR_UNSUPPORTED;
    if (out_dtype == WQ_OUT_BF16)
      gp.p.Y_bf16 = static_cast<__nv_bfloat16*>(Y);
    else
      gp.p.Y_f32 = static_cast<float*>(Y);
    return from_cuda(dispatch_format<GemmOp>(bits, symmetric != 0, group, &gp, &dev, X, codes,
                                             scales, zeros, s));
  }
  const bool have_ws = workspace != nullptr && workspace_bytes >= wq_matmul_workspace_bytes() &&
                       dev.sms <= wq::sk::kWsCtasMax;

  const bool pdl = (flags & WQ_MATMUL_STATIC_WEIGHTS) != 0;
  const int tiles = int((N + 15) / 16);
  // Kernel choice (measured on B200, back-to-back launches): the direct-load
  // kernel wherever it applies (4-bit codes, groups of 128, M <= 4, K a
  // multiple of 512): faster than both others on every Llama-8B layer shape
  // at M = 1, 2, 4.  Otherwise: the balanced kernel for 8-bit codes, group
  // 32, and layers with fewer than three waves of row tiles per SM; the
  // cluster-split kernel otherwise.  Splitting row tiles across CTAs through
  // the workspace measured slower than whole tiles on every shape tried (the
  // end-of-kernel gather costs more than the balance gains), so it is used
  // only when forced through the tuning hook.
  if (g_kernel_choice == 4 || g_kernel_choice == 0) {
    LdPlan lp;
    if (plan_ld(int(M), int(N), int(K), bits, group, dev, &lp)) {
      lp.p.X = static_cast<const __nv_bfloat16*>(X);
      lp.p.Y = Y;
      lp.p.codes = static_cast<const uint8_t*>(codes);
      lp.p.scales = static_cast<const __half*>(scales);
      lp.p.zeros = static_cast<const __half*>(zeros);
      lp.p.y_bf16 = out_dtype == WQ_OUT_BF16;
      return from_cuda(dispatch_format<LdOp>(bits, symmetric != 0, group, &lp, &dev, s, pdl));
    }
    if (g_kernel_choice == 4) return WQ_ERR_UNSUPPORTED;
  }
  const bool prefer_balanced = bits == 8 || group == 32 || tiles < 3 * dev.sms;
  const bool use_balanced =
      g_kernel_choice == 2 || g_kernel_choice == 3 || (g_kernel_choice == 0 && prefer_balanced);
  const bool split = have_ws && g_kernel_choice == 3;
  SkPlan sk;
  if (use_balanced &&
      plan_sk(int(M), int(N), int(K), bits, group, symmetric != 0, dev, split, &sk)) {
    sk.p.X = static_cast<const __nv_bfloat16*>(X);
    sk.p.Y = Y;
    sk.p.y_bf16 = out_dtype == WQ_OUT_BF16;
    if (split) {
      sk.p.ws_flag = static_cast<unsigned int*>(workspace);
      sk.p.ws_part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                              size_t(wq::sk::kWsCtasMax) * 4);
    }
    return from_cuda(dispatch_format<SkOp>(bits, symmetric != 0, group, &sk, &dev, codes, scales,
                                           zeros, s, pdl));
  }
  if (g_kernel_choice >= 2) return WQ_ERR_UNSUPPORTED;

  GemvPlan plan;
  if (!plan_gemv(int(M), int(N), int(K), bits, group, dev, 0, &plan)) return WQ_ERR_UNSUPPORTED;
  plan.p.X = static_cast<const __nv_bfloat16*>(X);
  plan.p.Y = Y;
  plan.p.scales = static_cast<const __half*>(scales);
  plan.p.zeros = static_cast<const __half*>(zeros);
  plan.p.codes = static_cast<const uint8_t*>(codes);
  plan.p.y_bf16 = out_dtype == WQ_OUT_BF16;
  const cudaError_t e = dispatch_format<GemvOp>(bits, symmetric != 0, group, &plan, &dev, codes,
                                                scales, zeros, s, pdl);
  return from_cuda(e);
}

// ------------------------------------------------------ no-allocation entry

}  // extern "C"

namespace {

// Scratch of wq_matmul_noalloc: the matmul workspace of any call (flags for
// kWsCtasMax CTAs and their binary32 partial sums, M <= 8), in device memory
// that the module brings with it.  Zero at load; every completed call leaves
// it zero.
constexpr size_t kNoallocScratchBytes =
    size_t(wq::sk::kWsCtasMax) * (size_t(wq::sk::kWsRowsMax) * 4 + 4);
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

void* g_noalloc_address[kMaxDevices] = {};

// The scratch address on the current device, looked up once per device (with
// that device current) and cleared once; null on failure.
void* noalloc_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_noalloc_address[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return nullptr;
    if (cudaMemset(p, 0, kNoallocScratchBytes) != cudaSuccess) return nullptr;
    g_noalloc_address[dev] = p;
  }
  return g_noalloc_address[dev];
}

}  // namespace

extern "C" {

size_t wq_matmul_noalloc_scratch_bytes(void) { return kNoallocScratchBytes; }

wq_status wq_matmul_noalloc(const void* X, int64_t M, const void* codes, const void* scales,
                            const void* zeros, int64_t N, int64_t K, int bits, int group,
                            int symmetric, void* Y, int out_dtype, unsigned int flags,
                            wq_stream_t stream) {
  // the scratch holds any workspace the matmul asks for; refuse otherwise
  if (wq_matmul_workspace_bytes() > kNoallocScratchBytes) return WQ_ERR_UNSUPPORTED;
  DeviceInfo dev;
  if (!device_info(&dev)) return WQ_ERR_CUDA;
  if (dev.sms > wq::sk::kWsCtasMax) return WQ_ERR_UNSUPPORTED;
  void* scratch = noalloc_scratch();
  if (scratch == nullptr) return WQ_ERR_CUDA;
  return wq_matmul(X, M, codes, scales, zeros, N, K, bits, group, symmetric, Y, out_dtype,
                   scratch, kNoallocScratchBytes, flags, stream);
}

wq_status wq_get_device_error(wq_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return WQ_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, wq::g_status, sizeof(v)) != cudaSuccess) return WQ_ERR_CUDA;
  const unsigned int zero = 0;
  if (cudaMemcpyToSymbol(wq::g_status, &zero, sizeof(zero)) != cudaSuccess) return WQ_ERR_CUDA;
  return static_cast<wq_status>(v);
}

const char* wq_status_string(wq_status status) {
  switch (status) {
    case WQ_OK: return "ok";
    case WQ_ERR_INVALID_ARG: return "invalid argument";
    case WQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case WQ_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case WQ_ERR_CUDA: return "CUDA runtime error";
    case WQ_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

const char* wq_version(void) { return "wq 0.1.0 (sm_100a)"; }

// Tuning hook, not part of the public ABI (see g_force_C).
void wq_internal_force_gemv_plan(int C, int bpw, int depth) {
  g_force_C = C;
  g_force_bpw = bpw;
  g_force_depth = depth;
}

// Diagnostic hook, not part of the public ABI: the name of the last CUDA
// error behind a WQ_ERR_CUDA status.
const char* wq_internal_last_cuda_error(void) { return cudaGetErrorName(g_last_cuda_error); }

// Tuning and test hook, not part of the public ABI: 0 lets wq_matmul choose
// the small-batch kernel, 1 forces the cluster-split kernel, 2 forces the
// balanced kernel, 3 forces the balanced kernel with row tiles split across
// CTAs whenever a workspace is given, 4 forces the direct-load kernel (2, 3
// and 4 return WQ_ERR_UNSUPPORTED where the forced kernel does not apply).
void wq_internal_set_kernel(int choice) { g_kernel_choice = choice; }

// Test hook, not part of the public ABI: the balanced kernel's plan for a
// device with `sms` SMs and `smem_optin` bytes of shared memory per block,
// written to out[0..24] (see tests/test_plan_sk.py for the field order).
// Returns 0 if the shape is outside the kernel's scope.
int wq_internal_plan_sk(int M, int N, int K, int bits, int group, int symmetric, int sms,
                        int smem_optin, int split, int64_t* out) {
  DeviceInfo dev;
  dev.sms = sms;
  dev.max_smem_optin = smem_optin;
  SkPlan plan;
  if (!plan_sk(M, N, K, bits, group, symmetric != 0, dev, split != 0, &plan)) return 0;
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

// Test hook, not part of the public ABI: the prefill plan, written to
// out[0..14] (see tests/test_plan_gemm.py for the field order).  Returns 0
// if the shape is outside the prefill kernel's scope.
int wq_internal_plan_gemm(int M, int N, int K, int bits, int group, int symmetric,
                          int smem_optin, int64_t* out) {
  DeviceInfo dev;
  dev.sms = 148;
  dev.max_smem_optin = smem_optin;
  GemmPlan plan;
  if (!plan_gemm(M, N, K, bits, group, symmetric != 0, dev, &plan)) return 0;
  const wq::gemm::Params& p = plan.p;
  const int64_t v[] = {p.M, p.N, p.K, p.ngroups, p.tiles_m, p.codes_stage_bytes, p.meta_bytes,
                       p.off_a, p.off_b, p.off_codes, p.off_meta_s, p.off_meta_z, p.off_stab,
                       int64_t(plan.smem), plan.grid};
  for (size_t i = 0; i < sizeof(v) / sizeof(v[0]); ++i) out[i] = v[i];
  return 1;
}

// Test hook, not part of the public ABI: the direct-load kernel's plan for a
// device with `sms` SMs and `smem_optin` bytes of shared memory per block,
// written to out[0..11] (see tests/test_plan_ld.py for the field order).
// Returns 0 if the shape is outside that kernel's scope.
int wq_internal_plan_ld(int M, int N, int K, int bits, int group, int sms, int smem_optin,
                        int64_t* out) {
  DeviceInfo dev;
  dev.sms = sms;
  dev.max_smem_optin = smem_optin;
  LdPlan plan;
  if (!plan_ld(M, N, K, bits, group, dev, &plan)) return 0;
  const wq::ld::Params& p = plan.p;
  const int64_t v[] = {p.M,      p.N,      p.K,        p.ngroups, p.tiles,
                       p.xs_row_bytes, p.off_sx, p.off_sz, p.off_part, p.off_ring,
                       int64_t(plan.smem), plan.grid};
  for (size_t i = 0; i < sizeof(v) / sizeof(v[0]); ++i) out[i] = v[i];
  return 1;
}

// Test hook, not part of the public ABI: the matmul plan for a device with
// `sms` SMs and `smem_optin` bytes of shared memory per block, written to
// out[0..27] (see tests/test_plan.py for the field order).  Returns 0 if no
// plan exists.
int wq_internal_plan_gemv(int M, int N, int K, int bits, int group, int sms, int smem_optin,
                          int cluster_cap, int64_t* out) {
  DeviceInfo dev;
  dev.sms = sms;
  dev.max_smem_optin = smem_optin;
  GemvPlan plan;
  if (!plan_gemv(M, N, K, bits, group, dev, cluster_cap, &plan)) return 0;
  const Params& p = plan.p;
  const int64_t v[] = {p.M,       p.N,           p.K,         p.ngroups,     p.row_tiles,
                       p.items,   p.RT,          p.SKW,       p.BPW,         p.depth,
                       p.kc,      p.stage_k,     p.stages_per_item, p.meta_tma, p.stage_bytes,
                       p.meta_offset, p.off_ring, p.off_x,    p.off_sx,      p.off_red,
                       p.off_part, int64_t(plan.smem), plan.C, plan.grid, p.x_row_stride,
                       p.red_bufs, p.row_stride, p.contig};
  for (size_t i = 0; i < sizeof(v) / sizeof(v[0]); ++i) out[i] = v[i];
  return 1;
}

// Measurement hook, not part of the public ABI: one launch of the read-only
// streaming kernel over up to three spans (a, b, c; byte counts multiples of
// 16, pointers 16-byte aligned; a null pointer with size 0 skips a span).  It
// writes one word per block to `out`, which must hold
// wq_internal_stream_read_out_bytes() bytes.  `pdl` launches it with
// programmatic dependent launch, like the fused matmul.
size_t wq_internal_stream_read_out_bytes(void) {
  DeviceInfo dev;
  if (!device_info(&dev)) return 0;
  return size_t(dev.sms) * wq::stream::kBlocksPerSm * 4;
}

wq_status wq_internal_stream_read(const void* a, size_t na, const void* b, size_t nb,
                                  const void* c, size_t nc, void* out, int pdl,
                                  wq_stream_t stream) {
  const void* ptrs[3] = {a, b, c};
  const size_t sizes[3] = {na, nb, nc};
  for (int i = 0; i < 3; ++i) {
    if (sizes[i] % 16 != 0 || (sizes[i] != 0 && ptrs[i] == nullptr)) return WQ_ERR_INVALID_ARG;
    if (ptrs[i] && !aligned16(ptrs[i])) return WQ_ERR_ALIGNMENT;
  }
  if (!out) return WQ_ERR_INVALID_ARG;
  DeviceInfo dev;
  if (!device_info(&dev)) return WQ_ERR_CUDA;
  using wq::stream::Span;
  const Span sa{reinterpret_cast<const uint4*>(a), na / 16};
  const Span sb{reinterpret_cast<const uint4*>(b), nb / 16};
  const Span sc{reinterpret_cast<const uint4*>(c), nc / 16};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(dev.sms * wq::stream::kBlocksPerSm));
  cfg.blockDim = dim3(wq::stream::kThreads);
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  if (pdl) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  return from_cuda(cudaLaunchKernelEx(&cfg, wq::stream::stream_read_kernel, sa, sb, sc,
                                      reinterpret_cast<uint32_t*>(out)));
}

}  // extern "C"

// ------------------------------------------------------ nested superblocks

extern "C" {

size_t wq_q4k_bytes(int64_t N, int64_t K) {
  if (N < 1 || K < wq::q4k::kBlockWeights || K % wq::q4k::kBlockWeights != 0 ||
      N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31))
    return 0;
  return size_t(N) * size_t(K / wq::q4k::kBlockWeights) * wq::q4k::kBlockBytes;
}

wq_status wq_q4k_quantize(const void* W, int64_t N, int64_t K, void* blocks,
                          wq_stream_t stream) {
  if (wq_q4k_bytes(N, K) == 0 || !W || !blocks) return WQ_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(blocks)) return WQ_ERR_ALIGNMENT;
  DeviceInfo dev;
  if (!device_info(&dev)) return WQ_ERR_CUDA;
  const int64_t nblocks = N * (K / wq::q4k::kBlockWeights);
  const int64_t grid = std::max<int64_t>(1, std::min<int64_t>((nblocks + 7) / 8,
                                                               int64_t(dev.sms) * 16));
  wq::q4k::quantize_kernel<<<unsigned(grid), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const __half*>(W), nblocks, static_cast<uint8_t*>(blocks));
  return from_cuda(cudaGetLastError());
}

wq_status wq_q4k_matmul(const void* X, int64_t M, const void* blocks, int64_t N, int64_t K,
                        void* Y, int out_dtype, wq_stream_t stream) {
  if (wq_q4k_bytes(N, K) == 0 || M < 1 || M > 8 || !X || !blocks || !Y)
    return WQ_ERR_INVALID_ARG;
  if (out_dtype != WQ_OUT_F32 && out_dtype != WQ_OUT_BF16) return WQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(blocks) || !aligned16(Y)) return WQ_ERR_ALIGNMENT;
  DeviceInfo dev;
  if (!device_info(&dev)) return WQ_ERR_CUDA;
  const int64_t grid = std::max<int64_t>(1, std::min<int64_t>((N + 7) / 8, int64_t(dev.sms) * 8));
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const auto* x = static_cast<const __nv_bfloat16*>(X);
  const auto* b = static_cast<const uint8_t*>(blocks);
  const int yb = out_dtype == WQ_OUT_BF16;
  const unsigned g = unsigned(grid);
  if (M == 1)
    wq::q4k::matmul_kernel<1><<<g, 256, 0, s>>>(x, int(M), b, int(N), int(K), Y, yb);
  else if (M == 2)
    wq::q4k::matmul_kernel<2><<<g, 256, 0, s>>>(x, int(M), b, int(N), int(K), Y, yb);
  else if (M <= 4)
    wq::q4k::matmul_kernel<4><<<g, 256, 0, s>>>(x, int(M), b, int(N), int(K), Y, yb);
  else
    wq::q4k::matmul_kernel<8><<<g, 256, 0, s>>>(x, int(M), b, int(N), int(K), Y, yb);
  return from_cuda(cudaGetLastError());
}

}  // extern "C"
