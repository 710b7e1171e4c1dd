// k_quantize.cu -- launchers of the quantize kernel and of the unfused
// dequantize kernel (the traffic baseline), one instantiation per format.
#include <algorithm>

#include "host.h"
#include "quantize.cuh"
#include "quantize2.cuh"

namespace wqh {
namespace {

unsigned grid_for_elements(int64_t total, int sms) {
  const int64_t warps_needed = (total + 1023) / 1024;
  const int64_t blocks = (warps_needed + 7) / 8;
  return unsigned(std::max<int64_t>(1, std::min<int64_t>(blocks, int64_t(sms) * 16)));
}

// 0: quantize2_kernel (prefetching, paired binary32 rounding, exact ties
// fixed per word); 1: the first quantize kernel.  Tuning hook.
int g_quantize_variant = 0;

template <int B, bool S, int G>
struct QuantizeOp {
  static cudaError_t run(const void* W, int64_t total, void* c, void* sc, void* z,
                         cudaStream_t s, int sms) {
    if (g_quantize_variant == 1) {
      wq::quantize_kernel<B, S, G><<<grid_for_elements(total, sms), 256, 0, s>>>(
          static_cast<const __half*>(W), total, static_cast<uint8_t*>(c),
          static_cast<__half*>(sc), static_cast<__half*>(z));
    } else {
      // one warp per 1,024 weights at a time; three CTAs of 8 warps per SM
      const int64_t chunks = (total + 1023) / 1024;
      const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((chunks + 7) / 8,
                                                                  int64_t(sms) * 3));
      wq::quantize2_kernel<B, S, G><<<unsigned(blocks), 256, 0, s>>>(
          static_cast<const __half*>(W), total, static_cast<uint8_t*>(c),
          static_cast<__half*>(sc), static_cast<__half*>(z));
    }
    return cudaGetLastError();
  }
};

template <int B, bool S, int G>
struct DequantizeOp {
  static cudaError_t run(const void* c, const void* sc, const void* z, int64_t total, void* out,
                         cudaStream_t s, int sms) {
    wq::dequantize_kernel<B, S, G><<<grid_for_elements(total, sms), 256, 0, s>>>(
        static_cast<const uint8_t*>(c), static_cast<const __half*>(sc),
        static_cast<const __half*>(z), total, static_cast<__nv_bfloat16*>(out));
    return cudaGetLastError();
  }
};

}  // namespace

cudaError_t run_quantize(int bits, bool sym, int group, const void* W, int64_t total,
                         void* codes, void* scales, void* zeros, cudaStream_t s, int sms) {
  return dispatch_format<QuantizeOp>(bits, sym, group, W, total, codes, scales, zeros, s, sms);
}

cudaError_t run_dequantize(int bits, bool sym, int group, const void* codes, const void* scales,
                           const void* zeros, int64_t total, void* out, cudaStream_t s,
                           int sms) {
  return dispatch_format<DequantizeOp>(bits, sym, group, codes, scales, zeros, total, out, s,
                                       sms);
}

}  // namespace wqh

extern "C" {

// Tuning hook, not part of the public ABI: 0 quantizes with quantize2_kernel
// (the default), 1 with the first quantize kernel.
void wq_internal_set_quantize_variant(int variant) { wqh::g_quantize_variant = variant; }

}  // extern "C"
