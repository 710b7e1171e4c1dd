// k_q4k.cu -- launchers of the nested-superblock (4.5 bits per weight)
// quantize and fused small-batch matmul kernels.
#include <algorithm>

#include "host.h"
#include "q4k.cuh"

namespace wqh {

cudaError_t run_q4k_quantize(const void* W, int64_t nblocks, void* blocks, cudaStream_t s,
                             int sms) {
  const int64_t grid =
      std::max<int64_t>(1, std::min<int64_t>((nblocks + 7) / 8, int64_t(sms) * 16));
  wq::q4k::quantize_kernel<<<unsigned(grid), 256, 0, s>>>(static_cast<const __half*>(W),
                                                           nblocks,
                                                           static_cast<uint8_t*>(blocks));
  return cudaGetLastError();
}

cudaError_t run_q4k_matmul(const void* X, int M, const void* blocks, int N, int K, void* Y,
                           bool y_bf16, cudaStream_t s, int sms) {
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
