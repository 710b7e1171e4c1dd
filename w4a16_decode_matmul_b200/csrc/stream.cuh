// stream.cuh -- a read-only streaming kernel: the practical ceiling for
// reading a decode layer's bytes (codes, scales, zeros) once from HBM in one
// launch, with the same launch pattern as the fused matmul (persistent grid,
// programmatic dependent launch).  It does none of the method's arithmetic;
// it exists so that the fused kernel's bandwidth can be read against what a
// plain read of the same bytes achieves at the same size.
#pragma once

#include "common.cuh"

namespace wq {
namespace stream {

constexpr int kThreads = 512;
constexpr int kBlocksPerSm = 4;
constexpr int kUnroll = 4;  // 16-byte loads in flight per thread

struct Span {
  const uint4* p;
  size_t n;  // 16-byte words
};

__device__ __forceinline__ uint32_t read_span(Span s, size_t first, size_t stride) {
  uint32_t acc = 0;
  for (size_t base = first; base < s.n; base += kUnroll * stride) {
    uint4 v[kUnroll];
#pragma unroll
    for (int j = 0; j < kUnroll; ++j) {
      const size_t i = base + size_t(j) * stride;
      v[j] = i < s.n ? ldg_stream128(s.p + i) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int j = 0; j < kUnroll; ++j) acc ^= v[j].x ^ v[j].y ^ v[j].z ^ v[j].w;
  }
  return acc;
}

// Every thread folds its words into one XOR; one word per block is written
// (after the previous launch on the stream has finished, so that
// back-to-back launches never write the same words concurrently).
__global__ void __launch_bounds__(kThreads) stream_read_kernel(Span a, Span b, Span c,
                                                               uint32_t* out) {
  grid_dependents_launch();
  const size_t first = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t stride = size_t(gridDim.x) * blockDim.x;
  uint32_t acc = read_span(a, first, stride) ^ read_span(b, first, stride) ^
                 read_span(c, first, stride);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
  __shared__ uint32_t warp_acc[kThreads / 32];
  if ((threadIdx.x & 31) == 0) warp_acc[threadIdx.x >> 5] = acc;
  __syncthreads();
  grid_dependency_wait();
  if (threadIdx.x == 0) {
    uint32_t r = 0;
    for (int w = 0; w < kThreads / 32; ++w) r ^= warp_acc[w];
    out[blockIdx.x] = r;
  }
}

}  // namespace stream
}  // namespace wq
