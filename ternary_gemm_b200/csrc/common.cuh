// Internal declarations shared by the translation units of libhbl.so.
// Nothing here is part of the public ABI (include/hbl.h is).
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "hbl.h"

namespace hbl {

// K1 output modes of the fused LN -> Hadamard -> quantize kernel.
enum K1Mode : int {
  K1_T_F32 = 0,      // t = H LN(x)/sqrt(K) as float (no quantizer)
  K1_Q4_PACKED = 1,  // INT4 absmean codes, two per byte
  K1_Q4_I8 = 2,      // INT4 absmean codes widened to one int8 per element
  K1_Q8_I8 = 3,      // INT8 absmax codes, one int8 per element
  K1_FHT_F32 = 4,    // the plain scaled transform H x / sqrt(K) as float (no LN, no quantizer)
  K1_LNBWD = 5,      // backward: LayerNorm backward at x of H g / sqrt(K) (g float; register kernel only)
};

constexpr int kMinLogK = 6;   // K = 64
constexpr int kMaxLogK = 15;  // K = 32768

// Fused K1.  x: [M][K] (bf16 bits if in_bf16 else float).  out: float t,
// packed nibbles or int8 codes as `mode` says; scales: [M] (ignored for
// K1_T_F32).  Returns cudaSuccess or the launch error.
cudaError_t launch_ln_fht_quant(const void* x, bool in_bf16, int64_t M, int log2k, K1Mode mode,
                                void* out, float* scales, cudaStream_t stream);

// The same operation with the high Hadamard factor on the tensor cores
// (bf16 input, K in [128, 32768], 16-byte aligned x and out, not
// K1_FHT_F32); launch_ln_fht_quant dispatches to it when supported and M is
// above kRegisterKernelMaxRows.
constexpr int64_t kRegisterKernelMaxRows = 4;
bool ln_fht_quant_tc_supports(bool in_bf16, int log2k, K1Mode mode, const void* x, const void* out);
cudaError_t launch_ln_fht_quant_tc(const void* x, int64_t M, int log2k, K1Mode mode, void* out, float* scales,
                                   cudaStream_t stream);
// The same launch with the ternary weight widening (2-bit [N][K/4] -> int8
// [N][K]) done by the kernel's two otherwise idle warps per CTA alongside
// the transform (hbl_forward's first two stages in one kernel) when the
// kernel has a CTA on every SM; for shorter batches the widening kernel runs
// after it.
cudaError_t launch_ln_fht_quant_tc_widen(const void* x, int64_t M, int log2k, K1Mode mode, void* out,
                                         float* scales, const uint8_t* packed, int64_t N, int64_t K, int8_t* w,
                                         cudaStream_t stream);

// LayerNorm (rms = false) or RMSNorm (rms = true) then the quantizer, without
// the Hadamard transform; K a power of two in [256, 32768].
cudaError_t launch_norm_quant(const void* x, bool in_bf16, int64_t M, int64_t K, bool rms, K1Mode mode,
                              void* out, float* scales, cudaStream_t stream);

// The quantizer alone on float rows t [M][K] (K % 16 == 0).
cudaError_t launch_quant_from_f32(const float* t, int64_t M, int64_t K, int bits, bool packed,
                                  uint8_t* codes, float* scales, cudaStream_t stream);

// Ternary weights: partial sums of |W| into ws (double[kTernaryPartials]),
// then alpha and the 2-bit codes.
constexpr int kTernaryPartials = 1184;  // 8 blocks per SM of a 148-SM B200
cudaError_t launch_pack_ternary(const void* W, bool in_bf16, int64_t N, int64_t K, uint8_t* packed,
                                float* alpha, double* partials, cudaStream_t stream);

// 2-bit ternary codes [N][K/4] -> int8 codes [N][K] for the tensor cores.
// With overlap_previous the kernel is a programmatic dependent of the
// previous kernel of the stream (which it does not read from): it runs
// alongside it and completes only after it.
cudaError_t launch_widen_ternary(const uint8_t* packed, int64_t N, int64_t K, int8_t* out, cudaStream_t stream,
                                 bool overlap_previous = false);

// tcgen05 int8 GEMM: acc[m][n] = sum_k A[m][k] B[n][k].  Epilogue: either the
// raw int32 (y_mode 0) or y = (float)acc * (scales[m] * alpha[0]) as float
// (y_mode 1) or bf16 (y_mode 2).
// ab_max: a bound on |A[m][k] B[n][k]| known to the caller (8 for INT4 codes
// times ternary weights), or 0; it lets short batches exchange int16 partials
cudaError_t launch_gemm_i8(const int8_t* A, const int8_t* B, int64_t M, int64_t N, int64_t K,
                           int y_mode, void* y, const float* scales, const float* alpha,
                           cudaStream_t stream, int ab_max = 0);

// The same product straight from packed INT4 codes A [M][K/2] and packed
// ternary weights W [N][K/4] (gemm_packed.cu): M >= 256, K % 64 == 0;
// y_mode 1 float, 2 bf16.  y is bit for bit that of launch_gemm_i8 on the
// widened codes.
bool gemm_tern_supports(int64_t M, int64_t K);
cudaError_t launch_gemm_tern(const uint8_t* A, const uint8_t* W, int64_t M, int64_t N, int64_t K, int y_mode,
                             void* y, const float* scales, const float* alpha, cudaStream_t stream);

// Small-M product straight from the packed 2-bit weights with the same
// dequantisation (y_mode 1 float, 2 bf16): M <= kGemvMaxRows,
// M * K <= kGemvMaxCodeBytes (the code rows live in shared memory), K a power
// of two in 64 .. 32768.  `early`: the codes come from the stream's previous
// kernel, which started after all earlier work, so the weight copies may
// begin before the programmatic dependency wait.
constexpr int64_t kGemvMaxRows = 4;
constexpr int64_t kGemvMaxCodeBytes = 65536;
bool gemv_ternary_supports(int64_t M, int64_t K);
cudaError_t launch_gemv_ternary(const int8_t* A, const float* scales, const uint8_t* packed, const float* alpha,
                                int64_t M, int64_t N, int64_t K, int y_mode, void* y, cudaStream_t stream,
                                bool early = false);
// The decode-sized forward in one launch (x -> LN -> transform -> quantize ->
// product -> y), every CTA quantizing the rows itself: gemv_ternary_supports
// and M * K <= kDecodeFusedMaxCodes (beyond that the redundant transforms cost
// more than a second launch); x bf16 or float, bits 4 or 8, y_mode 1 float /
// 2 bf16.
constexpr int64_t kDecodeFusedMaxCodes = 16384;
bool decode_forward_supports(int64_t M, int64_t K);
cudaError_t launch_decode_forward(const void* x, bool x_bf16, int64_t M, int log2k, int bits, const uint8_t* packed,
                                  const float* alpha, int64_t N, int y_mode, void* y, cudaStream_t stream);

// Device error word (bounded-wait timeouts) -- lives in gemm_i8.cu; kernels in
// other translation units receive its device address.
int* device_error_word();

// backward pass (gemm_bf16.cu, backward.cu)
cudaError_t launch_gemm_bf16(const uint16_t* A, bool a_mn, const uint16_t* B, int64_t R, int64_t C, int64_t Kc,
                             float* d, const float* scale, cudaStream_t stream);
cudaError_t launch_ternary_to_bf16(const uint8_t* packed, int64_t N, int64_t K, uint16_t* out, cudaStream_t stream);
cudaError_t launch_codes_to_bf16(const int8_t* q, int64_t count, uint16_t* out, cudaStream_t stream);
cudaError_t launch_scale_rows_bf16(const void* g, bool g_bf16, const float* s, int64_t M, int64_t N, uint16_t* out,
                                   cudaStream_t stream);
cudaError_t launch_ln_backward(const void* x, bool x_bf16, const float* gu, int64_t M, int log2k, void* gx,
                               cudaStream_t stream);
// low-bit QKV-state quantizer (kv_quant.cu): D in {32, 64, 128, 256}, bits in [2, 8]
cudaError_t launch_kv_quant(const void* x, bool bf16, int64_t rows, int64_t D, int bits, uint8_t* codes,
                            float* scales, cudaStream_t stream);
// g_x = LayerNorm backward at x of H g / sqrt(K), in one pass (fht_quant.cu)
cudaError_t launch_fht_ln_backward(const float* g, const void* x, bool x_bf16, int64_t M, int log2k, void* gx,
                                   cudaStream_t stream);
// Records e as the thread's last CUDA error (hbl_last_cuda_error) and maps it
// to a status: HBL_OK for cudaSuccess, else HBL_ERR_CUDA.
hbl_status note_cuda_error(cudaError_t e);
cudaError_t read_and_clear_device_error(cudaStream_t stream, int* value);
cudaError_t raise_device_error(cudaStream_t stream);
// Limit of the kernels' pipeline waits on the current device (0: the 2 s
// default); synchronizes the device first.
cudaError_t set_wait_limit(unsigned long long ns);

}  // namespace hbl
