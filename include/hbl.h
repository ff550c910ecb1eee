/*
 * hbl.h -- C ABI of the B200 (sm_100a) H-BitLinear forward (and backward) library.
 *
 * The layer is the H-BitLinear module of "BitNet v2: Native 4-bit
 * Activations with Hadamard Transformation for 1-bit LLMs" (arXiv 2504.18415;
 * section "H-BitLinear", the matrix-operation formula Y = Q(H(LN(X))) . Qw(W)).
 * Per token row of length K it computes
 *   1. LN: plain LayerNorm, no affine, eps_ln = 1e-5, biased variance;
 *   2. H : the Sylvester-order Walsh-Hadamard transform of length K (a power of
 *          two) scaled by 1/sqrt(K), computed as a fast Hadamard transform;
 *   3. Q : per-token activation quantization, INT4 absmean
 *          (beta = mean|t|, q = clip(rint(sqrt(7) t/(beta+eps)), -8, 7),
 *          scale = beta/sqrt(7)) or INT8 absmax (gamma = max|t|,
 *          q = clip(rint(127 t/(gamma+eps)), -128, 127), scale = gamma/127);
 *   4. an exact integer GEMM with the ternary weight codes, int32 accumulation;
 *   5. dequantisation y[m][n] = (float)acc[m][n] * (scale[m] * alpha).
 * Weights are ternarised once by per-tensor absmean (alpha = mean|W|,
 * w = clip(rint(W/(alpha+eps)), -1, 1)).  eps = 1e-5; rint rounds half to even.
 *
 * Conventions for every entry point:
 *  - All memory is owned by the caller.  Pointers marked "device" must point
 *    to device memory of the current CUDA device, 16-byte aligned.  The library
 *    never allocates or frees memory, never synchronises the stream (except
 *    hbl_last_device_error) and keeps no state between calls other than the
 *    device status (the error word read by hbl_last_device_error and the
 *    kernels' wait limit, hbl_debug_set_wait_limit_ns), each host thread's
 *    last CUDA error code (hbl_last_cuda_error), per-device caches of queried
 *    values (SM count, kernel attributes, cluster occupancy, symbol addresses;
 *    atomics filled on first use with the same value whichever thread fills
 *    them, so concurrent first calls only repeat the query), and the fixed
 *    scratch area of hbl_forward_noalloc.
 *  - Work is enqueued on `stream` (0 = legacy default stream) and is
 *    asynchronous; outputs are valid once the stream reaches that point.
 *  - Arguments are checked on the host before any launch.  A failed check
 *    returns an error status and enqueues nothing.  Launch failures return
 *    HBL_ERR_CUDA.  Nothing traps, asserts or exits.
 *  - Supported sizes: K a power of two with 64 <= K <= 32768; 1 <= M <= 2^26;
 *    N a multiple of 16 with 16 <= N <= 2^20 (forward, ternary packing).
 *    Entry points that differ say so below.
 *  - Row-major layouts throughout.  x is [M][K]; W is [N][K] (out x in, the
 *    layout of a PyTorch Linear weight); y is [M][N].
 */
#ifndef HBL_H_
#define HBL_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HBL_OK = 0,
  HBL_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, bad bits/dtype, misaligned */
  HBL_ERR_UNSUPPORTED = 2, /* a size outside the supported set (e.g. K not a power of two) */
  HBL_ERR_WORKSPACE = 3,   /* workspace pointer null or smaller than required */
  HBL_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
  HBL_ERR_TIMEOUT = 5      /* a kernel gave up a bounded wait (see hbl_last_device_error) */
} hbl_status;

typedef enum { HBL_F32 = 0, HBL_BF16 = 1 } hbl_dtype;

/* ---------------------------------------------------------------- sizes */

/* Bytes of the packed ternary weight: N rows of K/4 bytes (2 bits per code:
 * element 4j+i of a row sits at bits 2i..2i+1 of byte j; 00 = 0, 01 = +1,
 * 11 = -1).  Returns 0 for invalid sizes. */
size_t hbl_packed_ternary_bytes(int64_t K, int64_t N);

/* Bytes of activation codes for M rows: bits = 4 -> M*K/2 (two's-complement
 * nibbles, element 2j of a row in the low nibble of byte j, 2j+1 in the high
 * nibble); bits = 8 -> M*K (int8).  Returns 0 for invalid arguments. */
size_t hbl_codes_bytes(int64_t M, int64_t K, int bits);

/* Workspace bytes needed by hbl_pack_ternary (partial sums of |W|). */
size_t hbl_pack_ternary_workspace_bytes(int64_t K, int64_t N);

/* Workspace bytes needed by hbl_forward: int8 activation codes [M][K],
 * per-row scales [M] and the int8 weight codes [N][K] the tensor cores read.
 * Returns 0 for invalid arguments. */
size_t hbl_forward_workspace_bytes(int64_t M, int64_t K, int64_t N, int bits);

/* ---------------------------------------------------------------- compute */

/* Ternary weight quantization (the weights are quantized per tensor by
 * absmean to {-1, 0, 1}: the weight-quantization formula of section
 * "H-BitLinear").
 *   W         device, [N][K] of dtype wt (HBL_F32 or HBL_BF16)
 *   packed    device, hbl_packed_ternary_bytes(K, N) bytes (output)
 *   alpha_dev device, one float (output): alpha = mean|W| (accumulated in
 *             double, rounded once to float)
 *   workspace device, >= hbl_pack_ternary_workspace_bytes(K, N) bytes
 * Codes: w = clip(rint(W * (1/(alpha+eps))), -1, 1), the reciprocal one float
 * division, the product one float multiply. */
hbl_status hbl_pack_ternary(const void* W, hbl_dtype wt, int64_t K, int64_t N, uint8_t* packed,
                            float* alpha_dev, void* workspace, size_t workspace_bytes,
                            cudaStream_t stream);

/* LN -> H -> per-token quantization of M rows (the activation path of
 * H-BitLinear: LayerNorm, online Hadamard transformation, then per-token
 * absmean quantization for 4 bits or absmax quantization for 8 bits).
 *   x      device, [M][K] of dtype xt
 *   bits   4 or 8
 *   codes  device, hbl_codes_bytes(M, K, bits) bytes (output, layout above)
 *   scales device, M floats (output): beta/sqrt(7) (bits 4) or gamma/127
 *          (bits 8) per row
 * Per row: beta (or gamma) from the float transform output t; the mean of |t|
 * is accumulated in double and rounded once to float; r = c/(stat+eps) is one
 * float division (c = sqrt(7) rounded to float, or 127); q = rint(t*r),
 * clipped. */
hbl_status hbl_fht_quant(const void* x, hbl_dtype xt, int64_t M, int64_t K, int bits,
                         uint8_t* codes, float* scales, cudaStream_t stream);

/* Whole H-BitLinear forward: y = dequant(Q(H(LN(x))) . w^T).
 *   x          device, [M][K] of dtype xt
 *   packed     device, packed ternary weight from hbl_pack_ternary ([N][K/4])
 *   alpha_dev  device, the float alpha written by hbl_pack_ternary
 *   bits       4 or 8
 *   y          device, [M][N] of dtype yt (HBL_F32 or HBL_BF16, round to
 *              nearest even): y = (float)acc * (scale[m] * alpha)
 *   workspace  device, >= hbl_forward_workspace_bytes(M, K, N, bits) bytes,
 *              256-byte aligned; its contents are scratch
 * The integer GEMM runs on the tcgen05 tensor cores (kind::i8) with exact
 * int32 accumulation; decode-sized batches (M <= 4, M * K <= 65536) take exact
 * dp4a products straight from the packed weights instead, with the same y
 * (see "forward stages" below). */
hbl_status hbl_forward(const void* x, hbl_dtype xt, int64_t M, int64_t K, const uint8_t* packed,
                       const float* alpha_dev, int64_t N, int bits, void* y, hbl_dtype yt,
                       void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------- the transform alone; rotated weights
 * The Hadamard ablation of the pages compares rotating only the activations
 * (H-BitLinear) with rotating weights and activations.  Rotating each weight
 * row by the same orthogonal H/sqrt(K) leaves the product unchanged before
 * quantization, (H x).(H w) = x.w, so the rotated weight runs through
 * hbl_forward unchanged. */

/* t = H_K x / sqrt(K) per row (Sylvester order), float out [M][K] (device);
 * K a power of two in [64, 32768]. */
hbl_status hbl_fht(const void* x, hbl_dtype xt, int64_t M, int64_t K, float* t, cudaStream_t stream);

/* Workspace bytes of hbl_pack_ternary_rotated: the float rotated weight
 * [N][K] plus the partial sums of hbl_pack_ternary. */
size_t hbl_pack_ternary_rotated_workspace_bytes(int64_t K, int64_t N);

/* Ternary quantization of the rotated weight W' = W H_K / sqrt(K) (each row
 * of W [N][K] transformed along K in float), then exactly hbl_pack_ternary on
 * W': alpha = mean|W'|, w = clip(rint(W' / (alpha + eps)), -1, 1), packed.
 * Same arguments and layouts as hbl_pack_ternary; workspace device, >=
 * hbl_pack_ternary_rotated_workspace_bytes(K, N) bytes, 256-byte aligned. */
hbl_status hbl_pack_ternary_rotated(const void* W, hbl_dtype wt, int64_t K, int64_t N, uint8_t* packed,
                                    float* alpha_dev, void* workspace, size_t workspace_bytes,
                                    cudaStream_t stream);

/* ---------------------------------------------------------------- BitLinear without the transform
 * The activation path of the BitLinear layers that have no Hadamard
 * transform (every linear layer but the input and output embeddings moves to
 * 4-bit activations, and H-BitLinear replaces only Wo and Wdown;
 * BitNet b1.58 keeps 8-bit absmax activations): normalisation, then the same
 * per-token quantizer as hbl_fht_quant. */
typedef enum { HBL_NORM_LAYER = 0, HBL_NORM_RMS = 1 } hbl_norm;

/* t = LN(x) (HBL_NORM_LAYER: mean subtraction, biased variance) or
 * RMSNorm(x) (HBL_NORM_RMS: x / sqrt(mean x^2 + eps)), eps 1e-5, no affine;
 * then INT4 absmean (bits 4, codes packed two per byte) or INT8 absmax
 * (bits 8) exactly as hbl_fht_quant.  K a power of two in [256, 32768];
 * codes and scales as in hbl_fht_quant. */
hbl_status hbl_norm_quant(const void* x, hbl_dtype xt, int64_t M, int64_t K, hbl_norm norm, int bits,
                          uint8_t* codes, float* scales, cudaStream_t stream);

/* The normalisation alone: t as float [M][K] (device), the same kernel code as
 * hbl_norm_quant up to its quantizer (test hook). */
hbl_status hbl_debug_norm(const void* x, hbl_dtype xt, int64_t M, int64_t K, hbl_norm norm, float* t,
                          cudaStream_t stream);

/* ---------------------------------------------------------------- forward stages
 * hbl_forward is made of these calls on slices of its workspace:
 * hbl_fht_quant_i8, hbl_widen_ternary and hbl_gemm_dequant.  For
 * decode-sized batches (M <= 4 and M * K <= 65536) it runs hbl_fht_quant_i8
 * then hbl_gemv_ternary_dequant instead, and when M * K <= 16384 one kernel
 * that does what those two do, with the same arithmetic (y bit-identical),
 * keeping the codes in shared memory and leaving the workspace untouched.
 * hbl_fht_quant then hbl_gemm_tern_dequant is another
 * route to the identical y that needs no int8 buffers (it measured slower, so
 * hbl_forward does not take it).  They are public so that callers can overlap
 * stages or time each kernel on their own stream. */

/* The integer GEMM and its dequantisation straight from the packed operands:
 * y[m][n] = (float)(sum_k q[m][k] w[n][k]) * (scales[m] * alpha_dev[0]),
 * stored as yt, with q the INT4 codes of hbl_fht_quant (device, [M][K/2],
 * two per byte, element 2j in the low nibble) and w the 2-bit codes of
 * hbl_pack_ternary (device, [N][K/4]).  Converter warps widen both to int8 in
 * shared memory for the tcgen05 tensor cores (kind::i8); y is bit-identical
 * to hbl_gemm_dequant on the widened codes.  Requires M >= 256 and K a
 * multiple of 64 up to 32768 (else HBL_ERR_UNSUPPORTED), N a multiple of 16;
 * scales, alpha_dev, y as in hbl_gemm_dequant. */
hbl_status hbl_gemm_tern_dequant(const uint8_t* A, const uint8_t* packed, int64_t M, int64_t N, int64_t K,
                                 const float* scales, const float* alpha_dev, void* y, hbl_dtype yt,
                                 cudaStream_t stream);

/* Activation path with one int8 per code (the layout the tensor cores read):
 * the same LN -> H -> quantizer as hbl_fht_quant, codes device int8 [M][K]
 * (INT4 codes in [-8, 7], INT8 codes in [-128, 127]), scales device [M]. */
hbl_status hbl_fht_quant_i8(const void* x, hbl_dtype xt, int64_t M, int64_t K, int bits, int8_t* codes,
                            float* scales, cudaStream_t stream);

/* Packed 2-bit ternary codes [N][K/4] -> int8 codes [N][K] (device). */
hbl_status hbl_widen_ternary(const uint8_t* packed, int64_t K, int64_t N, int8_t* w, cudaStream_t stream);

/* The integer GEMM with the dequantisation fused into its epilogue:
 * y[m][n] = (float)(sum_k A[m][k] w[n][k]) * (scales[m] * alpha_dev[0]),
 * stored as yt.  A device int8 [M][K], w device int8 [N][K], scales device
 * float [M], alpha_dev device float, y device [M][N].  K a multiple of 16 up
 * to 65536, N a multiple of 16. */
hbl_status hbl_gemm_dequant(const int8_t* A, const int8_t* w, int64_t M, int64_t N, int64_t K,
                            const float* scales, const float* alpha_dev, void* y, hbl_dtype yt,
                            cudaStream_t stream);

/* The same product and dequantisation for decode-sized batches, straight
 * from the packed 2-bit weights (no widened copy): y[m][n] = (float)(sum_k
 * A[m][k] w[n][k]) * (scales[m] * alpha_dev[0]) with w the ternary codes of
 * packed [N][K/4] (hbl_pack_ternary's layout).  The int32 sums are exact and
 * the rescaling is hbl_gemm_dequant's, so y is bit-identical to it.  A device
 * int8 [M][K] (16-byte aligned), packed device (16-byte aligned), scales,
 * alpha_dev, y as in hbl_gemm_dequant.  Requires M <= 4, M * K <= 65536 and
 * K a power of two in [64, 32768] (HBL_ERR_UNSUPPORTED otherwise), N a
 * multiple of 16. */
hbl_status hbl_gemv_ternary_dequant(const int8_t* A, const uint8_t* packed, int64_t M, int64_t N, int64_t K,
                                    const float* scales, const float* alpha_dev, void* y, hbl_dtype yt,
                                    cudaStream_t stream);

/* ---------------------------------------------------------------- no caller workspace
 * The paper has no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory when they run a layer (a fixed memory
 * budget reserved up front, allocator-free runtimes or plugins handed only a
 * layer's tensors, hosts where cudaMalloc may block or fail late).
 *
 * hbl_forward_noalloc computes exactly what hbl_forward computes, with the
 * same arguments minus the workspace: it uses a fixed 32 MiB area of device
 * memory that belongs to the library (a file-scope __device__ array that every
 * GPU loading the library holds until the process exits).  Shapes whose
 * hbl_forward_workspace_bytes(M, K, N, bits) exceeds 32 MiB are rejected with
 * HBL_ERR_WORKSPACE before anything is launched; other argument errors are
 * those of hbl_forward.  It calls no allocator.
 *  - Each call made outside stream capture (with the device current) looks
 *    up the area's device address (cudaGetSymbolAddress, a query) and
 *    remembers it; a call made during capture uses the remembered address,
 *    so make the first call on a device before any stream capture (a
 *    captured first call returns HBL_ERR_CUDA).  The lookup on every
 *    uncaptured call keeps the address valid after cudaDeviceReset.
 *  - All calls share the area, which keeps the last call's contents; nothing
 *    in it needs to start at zero.  Calls whose kernels overlap on the GPU
 *    (other streams, unordered host threads) race on it: serialise them. */
hbl_status hbl_forward_noalloc(const void* x, hbl_dtype xt, int64_t M, int64_t K, const uint8_t* packed,
                               const float* alpha_dev, int64_t N, int bits, void* y, hbl_dtype yt,
                               cudaStream_t stream);

/* ---------------------------------------------------------------- backward pass
 * "BitNet v2: Native 4-bit Activations with Hadamard Transformation for 1-bit
 * LLMs", training strategy: gradients bypass the non-differentiable
 * quantizers (straight-through estimator) and are carried through the
 * Hadamard transform by its orthogonality.  With the forward's t, (q, s) and
 * (w, alpha) as in hbl_forward (y = (s q) (alpha w)^T) and u = LN(x):
 *   g_t = alpha g_y w                    (the quantizer of t passed straight through)
 *   g_u = H g_t / sqrt(K)                (H symmetric: the same scaled transform)
 *   g_x = (g_u - mean(g_u) - u mean(g_u u)) / sqrt(var(x) + 1e-5)   (LayerNorm backward, no affine)
 *   g_W = g_y^T (s q)                    (the ternary quantizer passed straight through)
 * The products run on the tensor cores in bf16 with float accumulation: w and
 * q are exact in bf16, g_y is used as given (rounded to bf16 first when it is
 * float), and s g_y is rounded to bf16 once for g_W. */

/* Workspace bytes of hbl_backward (0 for unsupported shapes). */
size_t hbl_backward_workspace_bytes(int64_t M, int64_t K, int64_t N, int bits);

/* x, M, K, packed, alpha_dev, N, bits as in hbl_forward (the forward's codes
 * and scales are recomputed from x).  g_y device [M][N] of dtype gyt (16-byte
 * aligned); outputs g_x device [M][K] of x's dtype and g_W device float
 * [N][K] (both 16-byte aligned, caller-owned).  workspace device, 256-byte
 * aligned, >= hbl_backward_workspace_bytes(M, K, N, bits) bytes.  Shape and
 * argument errors as in hbl_forward. */
hbl_status hbl_backward(const void* x, hbl_dtype xt, int64_t M, int64_t K, const uint8_t* packed,
                        const float* alpha_dev, int64_t N, int bits, const void* g_y, hbl_dtype gyt, void* g_x,
                        float* g_W, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* The backward's products alone: D[r][c] = scale * sum_k A[r][k] B[k][c] on
 * the tcgen05 tensor cores (bf16 operands, float accumulation).  A device
 * bf16: a_mn = 0 stored [R][Kc] (K-major), a_mn = 1 stored [Kc][R]; B device
 * bf16 stored [Kc][C]; D device float [R][C]; scale_dev a device float or
 * NULL for 1.  All 16-byte aligned; C a multiple of 8, and R (a_mn = 1) or Kc
 * (a_mn = 0) a multiple of 8, R * C at most 2^40 (HBL_ERR_UNSUPPORTED
 * otherwise). */
hbl_status hbl_gemm_bf16_f32(const uint16_t* A, int a_mn, const uint16_t* B, int64_t R, int64_t C, int64_t Kc,
                             float* D, const float* scale_dev, cudaStream_t stream);

/* The LayerNorm backward alone: g_x from x [M][K] (dtype xt) and g_u float
 * [M][K], as in hbl_backward; g_x of x's dtype.  K a power of two in
 * [64, 32768]; device pointers, 16-byte aligned. */
hbl_status hbl_ln_backward(const void* x, hbl_dtype xt, int64_t M, int64_t K, const float* g_u, void* g_x,
                           cudaStream_t stream);

/* The transform and the LayerNorm backward of hbl_backward in one pass:
 * g_x = LayerNorm backward at x of H g / sqrt(K), g float [M][K], x [M][K] of
 * dtype xt, g_x [M][K] of x's dtype (device, 16-byte aligned).  K a power of
 * two in [64, 32768]. */
hbl_status hbl_fht_ln_backward(const float* g, const void* x, hbl_dtype xt, int64_t M, int64_t K, void* g_x,
                               cudaStream_t stream);

/* ---------------------------------------------------------------- low-bit QKV states
 * The low-bit attention experiments of the pages quantize the QKV states after
 * RoPE: the heads go to unsigned integers through the absmax function, with no
 * calibration data (a 3-bit KV cache matches full precision).  The pages give
 * no formula; this library reads it as a linear map of [-gamma, gamma] onto
 * the 2^b unsigned levels, per head vector (one token, one head):
 *   gamma = max|x|, L = 2^b - 1, r = L / (2 (gamma + eps)) (float division),
 *   q = clip(rint(fl(fl(x r) + L/2)), 0, L),  scale = gamma,
 * so that x ~ (2 q - L) gamma / L.  RoPE itself and the attention are the
 * caller's.
 *   x      device, [rows][D] of dtype xt (each row one head vector, post-RoPE)
 *   D      head dimension: 32, 64, 128 or 256 (else HBL_ERR_UNSUPPORTED)
 *   bits   2 .. 8
 *   codes  device, [rows][D] bytes, one unsigned code per byte (output)
 *   scales device, rows floats: gamma per head vector (output) */
hbl_status hbl_kv_quant(const void* x, hbl_dtype xt, int64_t rows, int64_t D, int bits, uint8_t* codes,
                        float* scales, cudaStream_t stream);

/* ---------------------------------------------------------------- test hooks */

/* Stages 1-2 alone: t = H LN(x) / sqrt(K) as float [M][K] (device output).
 * The same kernel code as hbl_fht_quant up to the quantizer. */
hbl_status hbl_debug_ln_fht(const void* x, hbl_dtype xt, int64_t M, int64_t K, float* t,
                            cudaStream_t stream);

/* Stage 3 alone on given float rows t [M][K] (device): the same quantizer as
 * hbl_fht_quant.  K any multiple of 16 in [16, 65536]. */
hbl_status hbl_quant_from_f32(const float* t, int64_t M, int64_t K, int bits, uint8_t* codes,
                              float* scales, cudaStream_t stream);

/* Integer GEMM alone: acc[m][n] = sum_k A[m][k] * B[n][k] (exact int32) on the
 * tcgen05 tensor cores.  A device int8 [M][K], B device int8 [N][K],
 * acc device int32 [M][N]; K a multiple of 16, N a multiple of 16. */
hbl_status hbl_gemm_i8_i32(const int8_t* A, const int8_t* B, int64_t M, int64_t N, int64_t K,
                           int32_t* acc, cudaStream_t stream);

/* ---------------------------------------------------------------- errors */

/* Synchronises `stream`, then reports and clears the device error word that
 * kernels set when a bounded wait runs out: HBL_ERR_TIMEOUT if one did,
 * HBL_ERR_CUDA if the synchronisation failed, else HBL_OK.  The word is one
 * per device, shared by every stream and host thread that uses the library
 * there: a timeout is reported to the first caller that reads it after the
 * kernel that set it has run (work still running on other streams is not
 * waited for). */
hbl_status hbl_last_device_error(cudaStream_t stream);

/* Sets the device error word as a kernel would on a bounded-wait timeout
 * (used by the tests of the error path; enqueued on `stream`). */
hbl_status hbl_debug_raise_device_error(cudaStream_t stream);

/* Limit, in nanoseconds, of the kernels' pipeline waits on the current device
 * (each mbarrier wait of a producer, MMA issuer or epilogue gives up after it,
 * sets the device error word and leaves; its CTA then waits, for at most 2 s,
 * for the copies it issued before it exits).  0 restores the default of 2 s.
 * A test hook: a limit shorter than a kernel's run makes a wait run out so
 * that the error path can be tested without a fault.  Synchronises the device
 * before it changes the limit. */
hbl_status hbl_debug_set_wait_limit_ns(uint64_t ns);

/* Static string for a status code. */
const char* hbl_status_string(hbl_status status);

/* The CUDA runtime error code (a cudaError_t value) behind the most recent
 * HBL_ERR_CUDA returned on this host thread, 0 if there was none.  Reading it
 * does not clear it. */
int hbl_last_cuda_error(void);

/* Static name of a CUDA runtime error code, e.g. "cudaErrorInvalidValue". */
const char* hbl_cuda_error_name(int code);

#ifdef __cplusplus
}
#endif

#endif /* HBL_H_ */
