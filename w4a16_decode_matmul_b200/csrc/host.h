// host.h -- host-side pieces shared by the library's translation units: the
// device description, TMA descriptor encoding, the arguments of one matmul
// call, and the launcher of each kernel family.  Each family (quantize,
// direct-load, cluster-split, balanced, prefill, superblocks) is compiled in
// its own translation unit; wq.cu holds the C ABI and chooses among them.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>

namespace wqh {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  int sms = 0;
  int max_smem_optin = 0;
};

// SM count and opt-in shared memory of the current device (cached per
// device); false if the runtime cannot say.
bool device_info(DeviceInfo* out);

// 2-D row-major tensor [rows][cols] of `elem_bytes`-byte elements, no swizzle.
bool encode_2d(CUtensorMap* map, const void* base, CUtensorMapDataType type, int elem_bytes,
               uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows);

// 2-D row-major tensor with an explicit swizzle and L2 promotion.
bool encode_2d_ex(CUtensorMap* map, const void* base, CUtensorMapDataType type, int elem_bytes,
                  uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows,
                  CUtensorMapSwizzle swizzle, CUtensorMapL2promotion promotion);

// 3-D view: dims {d0, d1, d2} (d0 innermost, contiguous), byte strides of d1
// and d2 (any order), box {b0, b1, b2}.
bool encode_3d(CUtensorMap* map, const void* base, CUtensorMapDataType type, uint64_t d0,
               uint64_t d1, uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t b0,
               uint32_t b1, uint32_t b2, CUtensorMapSwizzle swizzle,
               CUtensorMapL2promotion promotion);

// Raise a kernel's dynamic shared-memory limit once per device.
template <typename K>
cudaError_t configure_smem(K kernel, int* configured, size_t bytes) {
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess || device < 0 || device >= kMaxDevices)
    return cudaErrorInvalidDevice;
  if (configured[device] == 0) {
    const cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
    if (e != cudaSuccess) return e;
    configured[device] = 1;
  }
  return cudaSuccess;
}

// One wq_matmul call, after the host-side checks.
struct MatmulArgs {
  const void* X;
  int M, N, K, bits, group;
  bool sym;
  const void* codes;
  const void* scales;
  const void* zeros;
  void* Y;
  bool y_bf16;
  void* workspace;      // null, or wq_matmul_workspace_bytes() zero-filled bytes
  bool pdl;             // launch as a programmatic dependent (static weights)
  cudaStream_t stream;
  DeviceInfo dev;
};

// Each runner returns false (launching nothing) when the call is outside its
// kernel's scope, true otherwise with the launch result in *err.
bool run_ld(const MatmulArgs& a, cudaError_t* err);
bool run_tb(const MatmulArgs& a, cudaError_t* err);
bool run_ks(const MatmulArgs& a, cudaError_t* err);
bool run_tc(const MatmulArgs& a, cudaError_t* err);
bool run_sk(const MatmulArgs& a, bool split, cudaError_t* err);
bool run_gemv(const MatmulArgs& a, cudaError_t* err);
bool run_gemm(const MatmulArgs& a, cudaError_t* err);
bool run_gemm2(const MatmulArgs& a, cudaError_t* err);

cudaError_t run_quantize(int bits, bool sym, int group, const void* W, int64_t total,
                         void* codes, void* scales, void* zeros, cudaStream_t s, int sms);
cudaError_t run_dequantize(int bits, bool sym, int group, const void* codes, const void* scales,
                           const void* zeros, int64_t total, void* out, cudaStream_t s, int sms);

cudaError_t run_q4k_quantize(const void* W, int64_t nblocks, void* blocks, cudaStream_t s,
                             int sms);
cudaError_t run_q4k_matmul(const void* X, int M, const void* blocks, int N, int K, void* Y,
                           bool y_bf16, bool pdl, cudaStream_t s, int sms);

// Balanced-kernel workspace geometry (flags, then partial sums).
size_t sk_workspace_bytes();
int sk_workspace_ctas();

// Kernel choice for wq_matmul (tuning and test hook): 0 chooses, 1 forces
// the cluster-split kernel, 2 the balanced kernel, 3 the balanced kernel
// with row tiles split across CTAs, 4 the direct-load kernel, 5 the
// bulk-staged kernel, 6 the k-sliced direct-load kernel.
extern int g_kernel_choice;

// Prefill kernel for wq_matmul at M > 32 (tuning and test hook): 0 chooses
// (the weights-in-tensor-memory kernel wherever it applies), 1 forces the
// kernel with both operands in shared memory, 2 forces the former.
extern int g_prefill_choice;

// Calls every format the library supports through F<BITS, SYM, G>::run.
template <template <int, bool, int> class F, typename... Args>
cudaError_t dispatch_format(int bits, bool sym, int group, Args... args) {
#define WQ_CASE(B, S, G) \
  if (bits == B && sym == S && group == G) return F<B, S, G>::run(args...);
  WQ_CASE(4, false, 32) WQ_CASE(4, false, 64) WQ_CASE(4, false, 128)
  WQ_CASE(4, true, 32) WQ_CASE(4, true, 64) WQ_CASE(4, true, 128)
  WQ_CASE(8, false, 32) WQ_CASE(8, false, 64) WQ_CASE(8, false, 128)
  WQ_CASE(8, true, 32) WQ_CASE(8, true, 64) WQ_CASE(8, true, 128)
#undef WQ_CASE
  return cudaErrorInvalidValue;
}

inline size_t round_up(size_t a, size_t b) { return (a + b - 1) / b * b; }

}  // namespace wqh
