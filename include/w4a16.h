/*
 * w4a16.h -- C ABI of the B200 (sm_100a) weight-only int4 matmul library.
 *
 * The operation: Y = X_bf16 . dequant(W_int4)^T, where each 4-bit code q
 * of W carries a per-group fp16 scale s and zero point z and dequantizes as
 * w = (q - z) * s (llm-quantization, "Objectives" 1 and 2: quantize FP16 to
 * INT4 and pack into INT8/INT32; Y = X_bf16 @ W_int4^T).  The same packed
 * weights also serve the transposed product dX = dY . dequant(W) used in
 * fine-tuning backward ("Re-write HQQ Fused Gemm Transpose": pack once, pass
 * transposed=True, no repacking and no reshaping of scales or zeros).
 *
 * Conventions shared by every entry point
 *   - All array arguments are DEVICE pointers owned by the caller; the
 *     library never frees or keeps them.  Calls are asynchronous on
 *     `stream` (a cudaStream_t; NULL = the legacy default stream).
 *   - N and K always name W's dimensions: W is [N, K] row-major.
 *   - packed: uint32 [N, K/8]; code i of word j of row n holds k = 8j + i
 *     in bits 4i..4i+3 (byte-identical to two codes per byte, low nibble =
 *     even k).
 *   - scales / zeros: fp16 [N, K/g] row-major (GROUPWISE), [N, 1]
 *     (ROWWISE), [1, 1] (GLOBAL).  zeros hold integer values 0..15.
 *   - Activations, gradients, bias and outputs are bf16, row-major, dense.
 *   - Accumulation is fp32; each output is rounded to bf16 once, after the
 *     optional bias has been added in fp32.
 *   - Arguments are validated before any launch, in the order listed in
 *     each comment; the first failure is returned and nothing is launched.
 *     After each launch the library checks cudaGetLastError() and returns
 *     W4_ERR_CUDA if it reports a launch failure.
 *   - The library allocates no device memory at run time.  Kernels that
 *     need scratch take it from the caller's `workspace`; query the size
 *     first.  The one exception is w4a16_gemv_noalloc, whose scratch is a
 *     fixed 8 MiB array compiled into the library (see there).
 *   - Pointers must be 16-byte aligned (W4_ERR_ALIGNMENT otherwise).
 */
#ifndef W4A16_H
#define W4A16_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum w4_status {
    W4_OK = 0,
    W4_ERR_INVALID_ARG = 1,  /* a size, mode or group size out of range */
    W4_ERR_UNSUPPORTED = 2,  /* valid, but no kernel here handles it */
    W4_ERR_ALIGNMENT = 3,    /* a pointer is not 16-byte aligned */
    W4_ERR_WORKSPACE = 4,    /* workspace missing or smaller than required */
    W4_ERR_CUDA = 5,         /* a CUDA runtime call or launch failed */
    W4_ERR_TIMEOUT = 6       /* a kernel gave up on a bounded wait (see w4_device_error) */
} w4_status;

typedef enum w4_mode {
    W4_MODE_GLOBAL = 0,    /* one (s, z) for the whole matrix */
    W4_MODE_ROWWISE = 1,   /* one (s, z) per row; group_size is ignored (g = K) */
    W4_MODE_GROUPWISE = 2  /* one (s, z) per g consecutive k of a row */
} w4_mode;

/*
 * Format flags, or-ed into the `mode` argument of every call (the quantizer
 * and the matmuls must be given the same ones).  Without flags the zero
 * point is an integer in [0, 15] and s, z are fp16.
 *   W4_ZERO_FLOAT  fractional zero point, the HQQ-style quantizer ("Re-write
 *                  HQQ Fused Gemm Transpose": its fused GEMM keeps a float
 *                  zero):  z = meta(-min / s), neither rounded to an integer
 *                  nor clamped to [0, 15] (only kept finite in its type), and
 *                  q = clamp(rint(w / s + z), 0, 15).
 *   W4_META_BF16   s and z are stored as bf16 instead of fp16 (every fp16
 *                  rounding of the quantizer becomes a bf16 rounding).
 * With W4_ZERO_FLOAT, q - z is no longer a small integer: the kernels round
 * it once (to bf16 on the bf16-mma and tensor-core paths, in fp32 on the
 * CUDA-core ones), except the int8 forward GEMV and the transposed GEMV,
 * which keep the integer part zi = clamp(rint(z), 0, 15) exact and add the
 * rest, (z - zi) times the activation sum, in fp32.
 */
enum { W4_ZERO_FLOAT = 0x10, W4_META_BF16 = 0x20 };

/*
 * Workspace bytes w4_quantize_pack needs for (N, K, mode): non-zero only for
 * GLOBAL, whose min/max runs as a separate grid-wide pass.
 */
size_t w4_quantize_workspace_bytes(int N, int K, int mode);

/*
 * w4_quantize_pack -- quantize bf16 W [N, K] to uint4 and pack eight codes
 * per uint32 along K (llm-quantization, "Objectives" 1: a kernel that
 * quantizes a 2-D matrix to INT4 and packs it into INT32; modes GLOBAL,
 * ROWWISE and GROUPWISE from its mode table).  Per group:
 *     s = fp16((max - min) / 15); if s == 0: s = fp16(max(|min|, 2^-14))
 *     z = clamp(rint(-min / s), 0, 15)
 *     q = clamp(rint(w / s) + z, 0, 15)
 * in IEEE fp32 with round-half-even (with the format flags above: the
 * fractional zero point and / or bf16 metadata); results are bit-exact
 * against the CPU oracle.  Inputs must be finite and, for fp16 metadata,
 * satisfy (max - min) / 15 <= 65504.
 *
 * Outputs: packed uint32 [N, K/8]; scales, zeros fp16 or bf16 bits (see
 * conventions).
 * Validation: N, K > 0; K % 8 == 0; mode in range (unknown flag bits are
 * W4_ERR_INVALID_ARG); GROUPWISE needs
 * group_size >= 8, group_size % 8 == 0, K % group_size == 0; pointers
 * non-NULL and 16-byte aligned; workspace_bytes >=
 * w4_quantize_workspace_bytes(N, K, mode).
 */
w4_status w4_quantize_pack(const void *W, int N, int K, int mode, int group_size,
                           uint32_t *packed, void *scales, void *zeros,
                           void *workspace, size_t workspace_bytes, void *stream);

/*
 * Workspace bytes w4a16_gemm / w4a16_gemv need for this problem (0 when the
 * chosen kernels need none).  Depends only on (M, N, K, transposed).
 */
size_t w4_workspace_bytes(int M, int N, int K, int transposed);

/*
 * w4a16_gemm -- weight-only int4 matmul with in-register dequantization.
 *   transposed = 0:  A = X  [M, K] -> Y  [M, N]:  Y  = X  . w_hat^T (+ bias[N])
 *       (llm-quantization, "Objectives" 2: Y = X_bf16 @ W_int4^T)
 *   transposed = 1:  A = dY [M, N] -> Y = dX [M, K]:  dX = dY . w_hat (+ bias[K])
 *       ("Re-write HQQ Fused Gemm Transpose": the backward product from the
 *       same packed weights, scales and zeros)
 *   bias: bf16 vector over the output columns, or NULL (vLLM "Adding bias
 *       epilogue support for cutlass_scaled_mm": bias dtype = output dtype).
 * Fused QKV weights (torchao "Add fused QKV HQQ triton_mm test") are just
 * the row-wise concatenation of the Q, K and V packed weights, scales and
 * zeros; they need no special call.
 * M <= 4 runs the small-batch GEMV kernels (same results as w4a16_gemv);
 * M > 4 runs the tcgen05 tensor-core kernel, which needs a workspace only
 * when it splits the tiles of a last partial wave (or of a grid smaller
 * than the GPU) into k slices: their fp32 partial tiles, added by a second
 * kernel.  Results do not depend on timing (fixed summation order).
 * Validation: M, N, K > 0; K % 8 == 0; mode/group rules as for
 * w4_quantize_pack; pointers (bias may be NULL) non-NULL and 16-byte
 * aligned; workspace_bytes >= w4_workspace_bytes(M, N, K, transposed).
 * The tensor-core path also needs K % 32 == 0 and, when transposed,
 * N % 8 == 0 (W4_ERR_UNSUPPORTED otherwise).
 */
w4_status w4a16_gemm(const void *A, int M, int N, int K, const uint32_t *packed,
                     const void *scales, const void *zeros, int mode, int group_size,
                     const void *bias, int transposed, void *Y,
                     void *workspace, size_t workspace_bytes, void *stream);

/*
 * w4a16_gemv -- the small-batch path (TensorRT-LLM "Modify small-batched
 * weight only quantization": a batch <= 4 GEMV is bound by global memory
 * loads): TMA-streamed packed weights with their dot products on the tensor
 * pipe.  Every product of a code and an activation is exact and the sums are
 * fp32:
 *   forward, g a multiple of 128 or one group per row: int8 mma on the
 *     activations as exact 24-bit integers per 128-k granule (three digits);
 *     a granule whose values span more than 15 binades takes bf16 mma on
 *     exact (q - z) codes instead;
 *   forward, other g multiples of 32: bf16 mma on exact (q - z) codes;
 *   transposed: bf16 mma, dY * s split into three exact bf16 parts;
 *   K or g not a multiple of 32 (or scale layouts the TMA boxes do not
 *     take): CUDA-core kernels with exact (q - z) and fp32 fma.
 * With W4_ZERO_FLOAT the int8 and transposed paths keep the integer part of
 * z exact and add the rest in fp32; the other paths round q - z once.
 * Same arguments and results as w4a16_gemm; M must be 1..4
 * (W4_ERR_INVALID_ARG otherwise).
 */
w4_status w4a16_gemv(const void *A, int M, int N, int K, const uint32_t *packed,
                     const void *scales, const void *zeros, int mode, int group_size,
                     const void *bias, int transposed, void *Y,
                     void *workspace, size_t workspace_bytes, void *stream);

/*
 * Act-order: weights quantized in a permuted input-channel order (the GPTQ
 * "desc_act" variant that TensorRT-LLM "Modify small-batched weight only
 * quantization" names beside channel-wise and group-wise AWQ/GPTQ).  When
 * packed column j holds input channel perm[j] (perm a permutation of
 * [0, K)), the products are
 *     forward     Y = X[:, perm] . w_hat^T:  gather X's columns, then the matmul;
 *     transposed  dX[:, perm] = dY . w_hat:  the matmul (with bias[perm] when a
 *                                            bias is given), then the columns
 *                                            put back (a gather by the inverse
 *                                            permutation).
 * The packed layout itself is unchanged; quantizing W[:, perm] gives it.
 *
 * w4_gather_columns -- out[m, j] = A[m, idx[j]] for m < M, j < L.
 *   A: bf16 [M, src_cols] row-major; idx: int32 [L] (device); out: bf16
 *   [M, L].  An idx[j] outside [0, src_cols) gives 0 there and records
 *   code 5 in the device error word (w4_device_error then returns
 *   W4_ERR_INVALID_ARG).
 * w4_scatter_columns -- out[m, idx[j]] = A[m, j] for m < M, j < L.
 *   A: bf16 [M, L]; out: bf16 [M, dst_cols]; idx must not repeat (a
 *   repeated index is a race); an index outside [0, dst_cols) is skipped
 *   and recorded as above.  Columns of out that no idx names are left as
 *   they are.
 * Both are asynchronous on `stream`; M, L and the column counts must be
 * > 0 and the pointers non-NULL (W4_ERR_INVALID_ARG otherwise).
 *
 * Two-per-byte view: the packed uint32 [N, K/8] array is byte-identical to
 * uint8 [N, K/2] with two codes per byte, the even k in the low nibble, so a
 * caller holding that byte layout passes its pointer as `packed` unchanged.
 */
w4_status w4_gather_columns(const void *A, int M, int src_cols, const int32_t *idx, int L,
                            void *out, void *stream);
w4_status w4_scatter_columns(const void *A, int M, int L, const int32_t *idx, int dst_cols,
                             void *out, void *stream);
/*
 * w4_invert_permutation -- inv[perm[j]] = j for j < n: int32 [n] device
 * arrays; perm must be a permutation of [0, n) (an entry outside it is
 * skipped and recorded as code 5).  A scatter by perm of a whole row is then
 * the gather by inv, whose writes are contiguous.  Asynchronous on `stream`.
 */
w4_status w4_invert_permutation(const int32_t *perm, int n, int32_t *inv, void *stream);

/* Human-readable name of a status code (static storage, never NULL). */
const char *w4_status_string(int status);

/*
 * w4_device_error -- read and clear the device-side error word of the
 * current device.  Kernels whose waits are bounded set it instead of
 * hanging (codes 1..4: which wait gave up); the column gather / scatter set
 * code 5 for an index out of range; *code receives 0 when nothing was
 * recorded.  Synchronizes the device.  Returns W4_ERR_INVALID_ARG for code 5,
 * W4_ERR_TIMEOUT for the other non-zero codes, W4_ERR_CUDA on a CUDA
 * failure, W4_OK otherwise.
 */
w4_status w4_device_error(int *code);

/*
 * w4_last_cuda_error -- text of the last CUDA error behind a W4_ERR_CUDA
 * returned on the calling host thread ("no error" if none).  Static
 * storage, never NULL.
 */
const char *w4_last_cuda_error(void);

/*
 * w4_launch_count -- number of kernel launches this library has issued in
 * the calling process since it was loaded (all devices, all entry points).
 * Host-side counter; launches replayed from a captured CUDA graph are not
 * re-counted.
 */
uint64_t w4_launch_count(void);

/*
 * w4a16_gemv_noalloc -- the forward GEMV of w4a16_gemv (M = 1..4,
 * transposed = 0) for callers that cannot allocate device memory: code that
 * runs where cudaMalloc is off limits or unsafe, such as inside an engine
 * that owns every byte of the GPU through its own pool, a plugin handed
 * only its input and output buffers, or a path that must not block on the
 * allocator.  The pages have no counterpart of this call.
 *
 * Instead of a caller workspace it uses a scratch array compiled into the
 * library: 8 MiB of device memory per GPU, held from the moment the library
 * is loaded on that device until the process exits.  The call allocates
 * nothing (no cudaMalloc, cudaFree or allocating library routine).  The
 * caller still passes X [M, K], the packed weights, scales, zeros, the
 * optional bias [N] and Y [M, N], with the layouts and validation of
 * w4a16_gemv.
 *
 * Limits and sharing:
 *   - The scratch holds the fp32 partial sums of a plan that splits K (few
 *     output rows and a long K).  Every problem with
 *     w4_workspace_bytes(M, N, K, 0) <= 8 MiB
 *     runs; a larger one runs when the plan for its own group length fits,
 *     else the call returns W4_ERR_WORKSPACE and launches nothing.
 *   - Every call on a device shares the one array.  Calls that may overlap
 *     on the GPU (other streams, other host threads) race on it and give
 *     wrong results; order them on one stream.  Each call writes all the
 *     scratch it later reads, so nothing needs clearing between calls.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current and keeps it; make
 *     that first call before any stream capture.  The address is kept for
 *     the life of the process, so do not call cudaDeviceReset (or otherwise
 *     destroy the device's primary context) between calls: the array may
 *     then sit elsewhere.
 */
w4_status w4a16_gemv_noalloc(const void *X, int M, int N, int K, const uint32_t *packed,
                             const void *scales, const void *zeros, int mode, int group_size,
                             const void *bias, void *Y, void *stream);

/*
 * w4_set_debug_checks -- debug mode for input checks (off by default;
 * process-wide).  When on, w4_quantize_pack first scans W for NaN and
 * infinities and returns W4_ERR_INVALID_ARG, quantizing nothing, if it
 * finds any; the scan synchronizes the call's stream, so keep it out of
 * stream capture.  With it off, non-finite weights give undefined codes.
 * (vLLM "Adding bias epilogue support for cutlass_scaled_mm": an opaque
 * "Error Internal" is what distinct statuses avoid.)
 */
w4_status w4_set_debug_checks(int on);

/*
 * Failure injection for testing the bounded waits (current device; both
 * synchronous).  w4_debug_set_wait_limit sets how long a kernel's bounded
 * wait may last before the kernel gives up (0 restores the default, 2 s).
 * w4_debug_withhold_stage makes the producer of every CTA of the GEMV
 * kernels skip the copy of its stage number `stage` (-1: none, the default)
 * without issuing it, so the consumers' waits run out, the kernel unwinds,
 * and w4_device_error reports W4_ERR_TIMEOUT.  Nothing is left in flight and
 * the context stays usable.  For tests only.
 */
w4_status w4_debug_set_wait_limit(unsigned long long ns);
w4_status w4_debug_withhold_stage(int stage);

#ifdef __cplusplus
}
#endif

#endif /* W4A16_H */
