// wq.cu -- the C ABI declared in include/wq.h: argument checks, the choice
// of matmul kernel, the device status word, and the host pieces shared by
// the kernel families (device description, TMA descriptor encoding).  Each
// kernel family is planned and launched in its own translation unit
// (k_*.cu).
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "wq.h"
#include "host.h"
#include "common.cuh"
#include "stream.cuh"

namespace wq {
// The device status word (see common.cuh); one for the whole library.
__device__ unsigned int g_status;
}  // namespace wq

namespace wqh {

namespace {
DeviceInfo g_devices[kMaxDevices];
std::mutex g_mutex;

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
}  // namespace

int g_kernel_choice = 0;
int g_prefill_choice = 0;  // 0: tensor-memory kernel first (measured faster at every M), then shared

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

bool encode_2d_ex(CUtensorMap* map, const void* base, CUtensorMapDataType type, int elem_bytes,
                  uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows,
                  CUtensorMapSwizzle swizzle, CUtensorMapL2promotion promotion) {
  auto fn = tensor_map_encoder();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * uint64_t(elem_bytes)};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, type, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, promotion,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_2d(CUtensorMap* map, const void* base, CUtensorMapDataType type, int elem_bytes,
               uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows) {
  return encode_2d_ex(map, base, type, elem_bytes, cols, rows, box_cols, box_rows,
                      CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
}

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

}  // namespace wqh

namespace {

using wqh::DeviceInfo;
using wqh::kMaxDevices;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_format(int64_t N, int64_t K, int bits, int group) {
  if (bits != 4 && bits != 8) return false;
  if (group != 32 && group != 64 && group != 128) return false;
  if (N < 1 || K < 32 || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31)) return false;
  if (K % 32 != 0 || K % group != 0) return false;
  return true;
}

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
  if (!wqh::device_info(&dev)) return WQ_ERR_CUDA;
  return from_cuda(wqh::run_quantize(bits, symmetric != 0, group, W, N * K, codes, scales, zeros,
                                     reinterpret_cast<cudaStream_t>(stream), dev.sms));
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
  if (!wqh::device_info(&dev)) return WQ_ERR_CUDA;
  return from_cuda(wqh::run_dequantize(bits, symmetric != 0, group, codes, scales, zeros, N * K,
                                       W_out, reinterpret_cast<cudaStream_t>(stream), dev.sms));
}

size_t wq_matmul_workspace_bytes(void) { return wqh::sk_workspace_bytes(); }

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
  wqh::MatmulArgs a{};
  if (!wqh::device_info(&a.dev)) return WQ_ERR_CUDA;
  a.X = X;
  a.M = int(M);
  a.N = int(N);
  a.K = int(K);
  a.bits = bits;
  a.group = group;
  a.sym = symmetric != 0;
  a.codes = codes;
  a.scales = scales;
  a.zeros = zeros;
  a.Y = Y;
  a.y_bf16 = out_dtype == WQ_OUT_BF16;
  a.pdl = (flags & WQ_MATMUL_STATIC_WEIGHTS) != 0;
  a.stream = reinterpret_cast<cudaStream_t>(stream);
  const bool have_ws = workspace != nullptr && workspace_bytes >= wq_matmul_workspace_bytes() &&
                       a.dev.sms <= wqh::sk_workspace_ctas();
  a.workspace = have_ws ? workspace : nullptr;
  cudaError_t e = cudaSuccess;
  const int choice = wqh::g_kernel_choice;

  if (M > 32) {
    // prefill: tensor-core GEMM on exact integer weights, binary32 group scaling
    const int pc = wqh::g_prefill_choice;
    if (pc != 1 && wqh::run_gemm2(a, &e)) return from_cuda(e);
    if (pc == 2) return WQ_ERR_UNSUPPORTED;
    if (!wqh::run_gemm(a, &e)) return WQ_ERR_UNSUPPORTED;
    return from_cuda(e);
  }
  // Kernel choice (measured on B200, back-to-back launches from CUDA graphs):
  // for 4-bit codes in groups of 128 with K = 4096 and M <= 4 the k-sliced
  // kernel, where the layer has at least one 8-row tile per SM (8.5 us
  // against 10.2 for the direct-load kernel at N = 14336; slower at N =
  // 1024); the direct-load kernel wherever it applies (4-bit codes, groups of
  // 128, M <= 4, K a multiple of 512): faster than both others on every
  // Llama-8B layer shape at M = 1, 2, 4.  Otherwise: the balanced kernel for
  // 8-bit codes, group 32, and layers with fewer than three waves of row
  // tiles per SM; the cluster-split kernel otherwise.  Splitting row tiles
  // across CTAs through the workspace measured slower than whole tiles on
  // every shape tried (the end-of-kernel gather costs more than the balance
  // gains), so it is used only when forced through the tuning hook.
  if (choice == 0 && N >= 8 * int64_t(a.dev.sms) && wqh::run_ks(a, &e)) return from_cuda(e);
  if (choice == 5) {
    if (wqh::run_tb(a, &e)) return from_cuda(e);
    return WQ_ERR_UNSUPPORTED;
  }
  if (choice == 6) {
    if (wqh::run_ks(a, &e)) return from_cuda(e);
    return WQ_ERR_UNSUPPORTED;
  }
  if (choice == 7) {
    if (wqh::run_tc(a, &e)) return from_cuda(e);
    return WQ_ERR_UNSUPPORTED;
  }
  if (choice == 4 || choice == 0) {
    if (wqh::run_ld(a, &e)) return from_cuda(e);
    if (choice == 4) return WQ_ERR_UNSUPPORTED;
  }
  const int tiles = int((N + 15) / 16);
  const bool prefer_balanced = bits == 8 || group == 32 || tiles < 3 * a.dev.sms;
  const bool use_balanced = choice == 2 || choice == 3 || (choice == 0 && prefer_balanced);
  const bool split = have_ws && choice == 3;
  if (use_balanced && wqh::run_sk(a, split, &e)) return from_cuda(e);
  if (choice >= 2) return WQ_ERR_UNSUPPORTED;
  if (!wqh::run_gemv(a, &e)) return WQ_ERR_UNSUPPORTED;
  return from_cuda(e);
}

}  // extern "C"

// ------------------------------------------------------ no-allocation entry

namespace {

// Scratch of wq_matmul_noalloc: the matmul workspace of any call (a flag for
// each of up to 1,024 CTAs, then their binary32 partial sums), in device
// memory that the module brings with it.  Zero at load; every completed
// call leaves it zero.
constexpr size_t kNoallocFlagBytes = 1024 * 4;
constexpr size_t kNoallocScratchBytes = kNoallocFlagBytes + size_t(1024) * 128 * 4;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

void* g_noalloc_address[kMaxDevices] = {};
// Set when wq_get_device_error reports a timed-out wait on a device: a
// kernel may then have left a flag of the block set, so the next call clears
// the block before use.
bool g_noalloc_dirty[kMaxDevices] = {};
std::mutex g_noalloc_mutex;

// The scratch address on the current device, looked up once per device (with
// that device current) and cleared then, synchronously; null on failure.
void* noalloc_scratch(int dev) {
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_address[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return nullptr;
    if (cudaMemset(p, 0, kNoallocScratchBytes) != cudaSuccess) return nullptr;
    // the memset runs on the legacy stream: finish it before any kernel on
    // another stream can touch the block
    if (cudaDeviceSynchronize() != cudaSuccess) return nullptr;
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
  if (!wqh::device_info(&dev)) return WQ_ERR_CUDA;
  if (dev.sms > wqh::sk_workspace_ctas()) return WQ_ERR_UNSUPPORTED;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess || device < 0 || device >= kMaxDevices)
    return WQ_ERR_CUDA;
  void* scratch = noalloc_scratch(device);
  if (scratch == nullptr) return WQ_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_dirty[device]) {
      // ordered before this call's kernel on the same stream
      if (cudaMemsetAsync(scratch, 0, kNoallocFlagBytes,
                          reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return WQ_ERR_CUDA;
      g_noalloc_dirty[device] = false;
    }
  }
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
  if (v == WQ_ERR_TIMEOUT) {
    int device = 0;
    if (cudaGetDevice(&device) == cudaSuccess && device >= 0 && device < kMaxDevices) {
      std::lock_guard<std::mutex> lock(g_noalloc_mutex);
      g_noalloc_dirty[device] = true;
    }
  }
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

const char* wq_version(void) { return "wq 0.2.0 (sm_100a)"; }

// Diagnostic hook, not part of the public ABI: the name of the last CUDA
// error behind a WQ_ERR_CUDA status.
const char* wq_internal_last_cuda_error(void) { return cudaGetErrorName(g_last_cuda_error); }

// Tuning and test hook, not part of the public ABI: 0 lets wq_matmul choose
// the small-batch kernel, 1 forces the cluster-split kernel, 2 forces the
// balanced kernel, 3 forces the balanced kernel with row tiles split across
// CTAs whenever a workspace is given, 4 forces the direct-load kernel, 5 the
// bulk-staged kernel, 6 the k-sliced direct-load kernel, 7 the tensor-memory
// small-batch kernel (2 to 7 return
// WQ_ERR_UNSUPPORTED where the forced kernel does not apply).
void wq_internal_set_kernel(int choice) { wqh::g_kernel_choice = choice; }

// Tuning and test hook, not part of the public ABI: the prefill kernel at
// M > 32 (0 chooses, 1 forces the kernel with both operands in shared
// memory, 2 forces the kernel with the weights in tensor memory; a forced
// kernel that does not apply returns WQ_ERR_UNSUPPORTED).
void wq_internal_set_prefill(int choice) { wqh::g_prefill_choice = choice; }

// Test hook, not part of the public ABI: the number of non-zero flag words
// in the no-allocation scratch block of the current device (0 when every
// completed call has left it clear), or -1 if it cannot be read.
int wq_internal_noalloc_flags_set(void) {
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess || device < 0 || device >= kMaxDevices) return -1;
  if (noalloc_scratch(device) == nullptr) return -1;
  unsigned int flags[kNoallocFlagBytes / 4];
  if (cudaMemcpyFromSymbol(flags, g_noalloc_scratch, kNoallocFlagBytes) != cudaSuccess) return -1;
  int n = 0;
  for (unsigned int f : flags) n += f != 0u;
  return n;
}

// Measurement hook, not part of the public ABI: one launch of the read-only
// streaming kernel over up to three spans (a, b, c; byte counts multiples of
// 16, pointers 16-byte aligned; a null pointer with size 0 skips a span).  It
// writes one word per block to `out`, which must hold
// wq_internal_stream_read_out_bytes() bytes.  `pdl` launches it with
// programmatic dependent launch, like the fused matmul.
size_t wq_internal_stream_read_out_bytes(void) {
  DeviceInfo dev;
  if (!wqh::device_info(&dev)) return 0;
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
  if (!wqh::device_info(&dev)) return WQ_ERR_CUDA;
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

// ------------------------------------------------------ nested superblocks

size_t wq_q4k_bytes(int64_t N, int64_t K) {
  constexpr int64_t kBlockWeights = 256, kBlockBytes = 144;
  if (N < 1 || K < kBlockWeights || K % kBlockWeights != 0 || N >= (int64_t(1) << 31) ||
      K >= (int64_t(1) << 31))
    return 0;
  return size_t(N) * size_t(K / kBlockWeights) * size_t(kBlockBytes);
}

wq_status wq_q4k_quantize(const void* W, int64_t N, int64_t K, void* blocks,
                          wq_stream_t stream) {
  if (wq_q4k_bytes(N, K) == 0 || !W || !blocks) return WQ_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(blocks)) return WQ_ERR_ALIGNMENT;
  DeviceInfo dev;
  if (!wqh::device_info(&dev)) return WQ_ERR_CUDA;
  return from_cuda(wqh::run_q4k_quantize(W, N * (K / 256), blocks,
                                         reinterpret_cast<cudaStream_t>(stream), dev.sms));
}

wq_status wq_q4k_matmul_ex(const void* X, int64_t M, const void* blocks, int64_t N,
                           int64_t K, void* Y, int out_dtype, unsigned int flags,
                           wq_stream_t stream) {
  if (wq_q4k_bytes(N, K) == 0 || M < 1 || M > 8 || !X || !blocks || !Y)
    return WQ_ERR_INVALID_ARG;
  if (out_dtype != WQ_OUT_F32 && out_dtype != WQ_OUT_BF16) return WQ_ERR_INVALID_ARG;
  if ((flags & ~unsigned(WQ_MATMUL_STATIC_WEIGHTS)) != 0) return WQ_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(blocks) || !aligned16(Y)) return WQ_ERR_ALIGNMENT;
  DeviceInfo dev;
  if (!wqh::device_info(&dev)) return WQ_ERR_CUDA;
  return from_cuda(wqh::run_q4k_matmul(X, int(M), blocks, int(N), int(K), Y,
                                       out_dtype == WQ_OUT_BF16,
                                       (flags & WQ_MATMUL_STATIC_WEIGHTS) != 0,
                                       reinterpret_cast<cudaStream_t>(stream), dev.sms));
}

wq_status wq_q4k_matmul(const void* X, int64_t M, const void* blocks, int64_t N, int64_t K,
                        void* Y, int out_dtype, wq_stream_t stream) {
  return wq_q4k_matmul_ex(X, M, blocks, N, K, Y, out_dtype, 0u, stream);
}

}  // extern "C"
