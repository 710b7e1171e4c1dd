// k_quantize.cu -- launchers of the quantize kernel and of the unfused
// dequantize kernel (the traffic baseline), one instantiation per format.
#include <algorithm>

#include "host.h"
#include "quantize.cuh"

namespace wqh {
namespace {

unsigned grid_for_elements(int64_t total, int sms) {
  const int64_t warps_needed = (total + 1023) / 1024;
  const int64_t blocks = (warps_needed + 7) / 8;
  return unsigned(std::max<int64_t>(1, std::min<int64_t>(blocks, int64_t(sms) * 16)));
}

template <int B, bool S, int G>
struct QuantizeOp {
  static cudaError_t run(const void* W, int64_t total, void* c, void* sc, void* z,
                         cudaStream_t s, int sms) {
    wq::quantize_kernel<B, S, G><<<grid_for_elements(total, sms), 256, 0, s>>>(
        static_cast<const __half*>(W), total, static_cast<uint8_t*>(c),
        static_cast<__half*>(sc), static_cast<__half*>(z));
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
