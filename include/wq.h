/*
 * wq.h -- C ABI of the B200 (sm_100a) library for groupwise affine low-bit
 * weight quantization and the fused dequant-in-register W4A16 matmul.
 *
 * Operations and where they are defined:
 *   quantize    q = clamp(round(w/s) + z, qmin, qmax), one binary16 scale s
 *               and one binary16 integer zero z per group of `group`
 *               consecutive weights along K.  Asymmetric: "vLLM 量化与推测解码"
 *               section 1 (affine map, min-max scale s = (xmax - xmin)/(qmax
 *               - qmin), zero z = round(qmin - xmin/s), qmin = 0, qmax =
 *               2^b - 1, range widened to contain 0, scale 1.0 for a
 *               degenerate range, zero clamped).  Symmetric: "量化"
 *               (llminference s08) section 解法 (z = 0, s = max|w| /
 *               (2^(b-1) - 1), codes clipped to [-2^(b-1), 2^(b-1) - 1]).
 *   dequantize  x^ = s (q - z)  (same section 1); materialises the weights.
 *   matmul      Y = X * What^T with What = s (q - z) formed on chip
 *               ("vLLM 量化与推测解码" section 2, W4A16: packed INT4 weights
 *               and group scales are unpacked and scaled in registers /
 *               on-chip tiles, multiplied with 16-bit activations and
 *               accumulated in higher precision; "量化" (llminference s08)
 *               section 实现: dequantize inside the accumulation, never write
 *               full-precision weights back to memory).
 *   q4k_*       the same two operations for nested superblocks of 256
 *               weights at 4.5 bits per weight ("量化" (llminference s08),
 *               the Q4_K superblock figure); the format is given with those
 *               entry points below.
 *
 * Numerics (fixed where the pages leave them open):
 *   - round() is round-half-to-even; the arithmetic that decides each code
 *     is exact for binary16 inputs;
 *   - the stored scale is the binary16 value obtained by rounding the scale
 *     toward +infinity, and codes are computed with that stored scale, so
 *     |w - x^| <= s/2 holds for every element;
 *   - the zero point is stored as a binary16 holding an integer;
 *   - symmetric codes are stored offset-binary: u = q + 2^(b-1);
 *   - matmul accumulates in binary32; |y - y_ref| <= 1e-4 * sum_k |x_k w^_k|
 *     (binary32 output), plus one bfloat16 ulp for bfloat16 output.
 *
 * Layouts (all row-major, all device memory, all owned by the caller):
 *   W      [N][K]              binary16 weights (quantize input)
 *   codes  [N][K*bits/8]       bytes; bits = 4: byte j of a row holds
 *                              k = 2j in bits 0-3 and k = 2j + 1 in bits 4-7;
 *                              bits = 8: one byte per weight
 *   scales [N][K/group]        binary16
 *   zeros  [N][K/group]        binary16 (integers 0..2^b-1); asymmetric only,
 *                              NULL when symmetric
 *   X      [M][K]              bfloat16 activations
 *   Y      [M][N]              binary32 or bfloat16 (fully overwritten)
 *   What   [N][K]              bfloat16 (dequantize output)
 *
 * Ownership and streams: the caller allocates and frees every buffer.  No
 * entry point allocates, frees or synchronizes; all work is enqueued on
 * `stream` (a cudaStream_t; NULL is the legacy default stream).  Every
 * pointer must be 16-byte aligned.  Inputs and outputs must not overlap.
 *
 * Errors: arguments are checked on the host before anything is launched; a
 * failed check returns a non-zero status and launches nothing.  A launch
 * failure returns WQ_ERR_CUDA.  Kernels never trap: a wait that exceeds its
 * time limit records WQ_ERR_TIMEOUT in a device status word that
 * wq_get_device_error() reads.  Weights containing NaN or Inf give
 * unspecified codes.
 */
#ifndef WQ_H
#define WQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st *wq_stream_t;

typedef enum wq_status {
    WQ_OK = 0,
    WQ_ERR_INVALID_ARG = 1,  /* a size, pointer or option is out of range   */
    WQ_ERR_UNSUPPORTED = 2,  /* valid request this build does not implement */
    WQ_ERR_ALIGNMENT = 3,    /* a pointer is not 16-byte aligned            */
    WQ_ERR_CUDA = 4,         /* a CUDA runtime call failed                  */
    WQ_ERR_TIMEOUT = 5       /* a device-side wait ran out of time          */
} wq_status;

/* Output element types for wq_matmul. */
enum { WQ_OUT_F32 = 0, WQ_OUT_BF16 = 1 };

/* Supported formats: bits in {4, 8}; group in {32, 64, 128}; K a multiple of
 * 32 and of group; 1 <= N, K < 2^31; 1 <= M. */

/* Bytes of the packed codes of an [N][K] matrix: N*K*bits/8 ("vLLM 量化与推测
 * 解码" section 2, payload N_param * b_w / 8).  Returns 0 for invalid sizes. */
size_t wq_codes_bytes(int64_t N, int64_t K, int bits);

/* Elements of each metadata tensor (scales, and zeros when asymmetric):
 * N*(K/group).  Each element is 2 bytes.  Returns 0 for invalid sizes. */
size_t wq_meta_elems(int64_t N, int64_t K, int group);

/* Quantize W [N][K] binary16 into codes / scales / zeros (layouts above).
 * symmetric = 0: asymmetric, zeros required; symmetric = 1: zeros must be
 * NULL.  One pass over W; the result is bit-exact with the definition in
 * the file header. */
wq_status wq_quantize(const void *W, int64_t N, int64_t K, int bits, int group,
                      int symmetric, void *codes, void *scales, void *zeros,
                      wq_stream_t stream);

/* Materialise What [N][K] bfloat16 = round-to-nearest-even(s (q - z)).
 * Kept only as the traffic baseline of the unfused path (dequantize, then an
 * ordinary matmul), which moves more bytes than the 16-bit weights it
 * replaces ("量化" (llminference s08) section 实现). */
wq_status wq_dequantize(const void *codes, const void *scales, const void *zeros,
                        int64_t N, int64_t K, int bits, int group, int symmetric,
                        void *W_out, wq_stream_t stream);

/* Flags of wq_matmul. */
enum {
    /* The weights (codes, scales, zeros) are not written by the kernel that
     * precedes this call on `stream`.  The call may then be launched as a
     * programmatic dependent of that kernel: it starts streaming the weights
     * while the previous kernel finishes, and reads X, writes Y and touches
     * the workspace only after the previous kernel has completed.  Use it for
     * the static weights of a model's layers, not right after wq_quantize of
     * the same weights. */
    WQ_MATMUL_STATIC_WEIGHTS = 1
};

/* Bytes of the matmul workspace (a device buffer, 16-byte aligned, filled
 * with zeros by the caller before its first use; every completed call leaves
 * it filled with zeros again). */
size_t wq_matmul_workspace_bytes(void);

/* Y [M][N] = X [M][K] * What^T, weights formed on chip from codes, scales
 * and zeros and never written to memory.  out_dtype is WQ_OUT_F32 or
 * WQ_OUT_BF16 (round-to-nearest-even from the binary32 accumulator).
 *
 * M <= 32 runs the small-batch decode kernels: codes streamed once from
 * HBM, tensor-core products of integer-valued 16-bit codes, binary32 group
 * scaling.  Every supported format is accepted.
 *
 * M > 32 runs the prefill kernel: the exact integers q - z on the tcgen05
 * tensor cores with binary32 accumulators in tensor memory, one per group,
 * scaled by s in binary32 ("量化" (llminference s08) section 实现: large
 * batches are bound by the multiply).  Its scope in this build: groups of
 * 32, 64 or 128, 4- or 8-bit codes, K a multiple of 128 (a load stage is
 * 128 k); other shapes at M > 32 return WQ_ERR_UNSUPPORTED.
 *
 * workspace / workspace_bytes: NULL and 0, or a buffer of at least
 * wq_matmul_workspace_bytes() bytes as described there.  With it, every SM
 * streams the same number of bytes (row tiles may be summed across CTAs
 * through the workspace, in a fixed order); without it, whole row tiles are
 * divided among the SMs.  Calls that may run at the same time on the GPU
 * (different streams) need different workspaces.  After a call that recorded
 * WQ_ERR_TIMEOUT the workspace must be zero-filled again.
 *
 * flags: 0 or WQ_MATMUL_STATIC_WEIGHTS.
 *
 * Deterministic: the same inputs give the same bits on every call. */
wq_status wq_matmul(const void *X, int64_t M, const void *codes, const void *scales,
                    const void *zeros, int64_t N, int64_t K, int bits, int group,
                    int symmetric, void *Y, int out_dtype, void *workspace,
                    size_t workspace_bytes, unsigned int flags, wq_stream_t stream);

/* As wq_matmul, without a workspace argument and without allocating:
 * the workspace is a fixed block of device memory inside the library
 * (wq_matmul_noalloc_scratch_bytes() bytes: flags and partial sums for up to
 * 1,024 CTAs), zero at load and left zero by every completed call.  The
 * pages have no counterpart of this entry point.  It is for callers that
 * cannot call cudaMalloc: code that runs where the allocator must not be
 * entered (a host callback, a real-time or signal-safe path, a custom
 * allocator that owns all device memory), or that must not grow its memory
 * after start-up.
 *   - The first call on a device looks up the block's address with
 *     cudaGetSymbolAddress (with that device current) and clears the block,
 *     synchronously (cudaMemset, then cudaDeviceSynchronize): make that
 *     first call before any stream capture.
 *   - All calls on a device share the block: calls whose kernels overlap on
 *     the GPU (different streams, or graphs replayed concurrently) race.
 *   - After wq_get_device_error has reported WQ_ERR_TIMEOUT on a device, the
 *     next call there first clears the block's flags (cudaMemsetAsync on its
 *     stream), since a timed-out call can leave one set.
 *   - A device with more SMs than the block has room for gets
 *     WQ_ERR_UNSUPPORTED, as does a workspace larger than the block.
 * Results are bit-identical to wq_matmul given a workspace. */
size_t wq_matmul_noalloc_scratch_bytes(void);
wq_status wq_matmul_noalloc(const void *X, int64_t M, const void *codes, const void *scales,
                            const void *zeros, int64_t N, int64_t K, int bits, int group,
                            int symmetric, void *Y, int out_dtype, unsigned int flags,
                            wq_stream_t stream);

/* ---- nested superblocks, 4.5 bits per weight -----------------------------
 * "量化" (llminference s08), the Q4_K superblock figure: 256 weights in 8
 * sub-blocks of 32, a 6-bit scale and a 6-bit minimum per sub-block
 * quantized against a binary16 super-scale d and super-minimum dmin, 4-bit
 * codes.  The page fixes the nesting and the bit counts only; this format
 * is the library's reading (not GGUF-compatible):
 *   sub-block j: lo = min(0, min w), hi = max(0, max w) ("vLLM 量化与推测
 *   解码" section 1's range); s_j = (hi - lo)/15; m_j = -lo;
 *   d = smallest binary16 >= max s_j / 63, dmin likewise for m_j (0 when the
 *   maximum is 0); sc_j = clamp(round(s_j/d), 1, 63) (1 when d = 0);
 *   mq_j = clamp(round(m_j/dmin), 0, 63) (0 when dmin = 0);
 *   q = clamp(round((w + M_j)/S_j), 0, 15) with S_j = d sc_j, M_j = dmin mq_j
 *   (0 when S_j = 0); reconstruction w^ = S_j q - M_j.
 * Every rounding is half-to-even of the exact value.
 * Layout: row-major [N][K/256] blocks of 144 bytes: d, dmin (binary16,
 * little-endian), 12 bytes of sixteen 6-bit fields (sc_0..7 then mq_0..7,
 * least significant bit first), 128 bytes of codes (byte i holds weight 2i
 * in its low nibble, 2i+1 in its high nibble).  K a multiple of 256.
 * Errors, checked on the host before any launch: WQ_ERR_INVALID_ARG for a
 * size outside that scope, M outside 1..8, a null pointer or an unknown
 * out_dtype; WQ_ERR_ALIGNMENT for a pointer not 16-byte aligned. */

/* Bytes of the blocks of an [N][K] matrix: N*(K/256)*144 (4.5 bits per
 * weight); 0 for invalid sizes. */
size_t wq_q4k_bytes(int64_t N, int64_t K);

/* Quantize W [N][K] binary16 into blocks (wq_q4k_bytes(N, K) bytes, 16-byte
 * aligned, caller-owned).  Bit-exact with the definition above. */
wq_status wq_q4k_quantize(const void *W, int64_t N, int64_t K, void *blocks,
                          wq_stream_t stream);

/* Y [M][N] = X [M][K] (bfloat16) * What^T for superblock weights, 1 <= M <=
 * 8, binary32 accumulation (per sub-block: d sc (sum x q) - dmin mq (sum x));
 * Y binary32 or bfloat16 (out_dtype as for wq_matmul).  The full-precision
 * weights are never written.  Pointers 16-byte aligned; nothing is
 * allocated; the call is enqueued on `stream`. */
wq_status wq_q4k_matmul(const void *X, int64_t M, const void *blocks, int64_t N, int64_t K,
                        void *Y, int out_dtype, wq_stream_t stream);

/* As wq_q4k_matmul, with flags: 0 or WQ_MATMUL_STATIC_WEIGHTS, which means
 * as for wq_matmul that nothing enqueued before the call on `stream` writes
 * the blocks: the kernel is launched as a programmatic dependent of the
 * previous work and may read the blocks before that work has finished (X and
 * Y only after).  Errors as wq_q4k_matmul, and WQ_ERR_INVALID_ARG for an
 * unknown flag. */
wq_status wq_q4k_matmul_ex(const void *X, int64_t M, const void *blocks, int64_t N,
                           int64_t K, void *Y, int out_dtype, unsigned int flags,
                           wq_stream_t stream);

/* Read and clear the device status word (WQ_OK if no kernel recorded an
 * error).  Synchronizes `stream` first. */
wq_status wq_get_device_error(wq_stream_t stream);

/* Static text for a status code. */
const char *wq_status_string(wq_status status);

/* Library version string. */
const char *wq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* WQ_H */
