// C ABI of libhbl.so (declarations and contracts in include/hbl.h): argument
// checks, workspace carving and the launch sequence of each entry point.
#include <cstdint>

#include "common.cuh"

namespace {

using hbl::K1Mode;

constexpr int64_t kMaxRows = int64_t(1) << 26;
constexpr int64_t kMaxN = int64_t(1) << 20;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int log2_exact(int64_t K) {
  if (K <= 0 || (K & (K - 1))) return -1;
  int l = 0;
  while ((int64_t(1) << l) < K) ++l;
  return l;
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

bool dtype_ok(hbl_dtype t) { return t == HBL_F32 || t == HBL_BF16; }

thread_local int g_last_cuda_error = 0;

hbl_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return HBL_OK;
  g_last_cuda_error = (int)e;
  return HBL_ERR_CUDA;
}

// K a power of two in [64, 32768] -> log2 K, else -1 / -2 (unsupported)
hbl_status check_k(int64_t K, int* log2k) {
  if (K <= 0) return HBL_ERR_INVALID_ARG;
  int l = log2_exact(K);
  if (l < hbl::kMinLogK || l > hbl::kMaxLogK) return HBL_ERR_UNSUPPORTED;
  *log2k = l;
  return HBL_OK;
}

hbl_status check_rows(int64_t M) {
  if (M <= 0) return HBL_ERR_INVALID_ARG;
  if (M > kMaxRows) return HBL_ERR_UNSUPPORTED;
  return HBL_OK;
}

hbl_status check_n(int64_t N) {
  if (N <= 0) return HBL_ERR_INVALID_ARG;
  if (N % 16 != 0 || N > kMaxN) return HBL_ERR_UNSUPPORTED;
  return HBL_OK;
}

hbl_status check_norm_k(int64_t K) {
  if (K <= 0) return HBL_ERR_INVALID_ARG;
  if (K < 256 || K > 32768 || (K & (K - 1))) return HBL_ERR_UNSUPPORTED;
  return HBL_OK;
}

// hbl_forward's workspace: int8 codes [M][K], scales [M], int8 weight codes
// [N][K].  (The GEMM that reads packed codes, hbl_gemm_tern_dequant, needs
// neither int8 buffer but measured slower at every size, so the forward keeps
// the int8 operands.)
struct ForwardLayout {
  size_t a_off, s_off, b_off, total;
};

ForwardLayout forward_layout(int64_t M, int64_t K, int64_t N, int bits) {
  (void)bits;
  ForwardLayout L;
  L.a_off = 0;
  L.s_off = align256((size_t)M * (size_t)K);
  L.b_off = L.s_off + align256((size_t)M * 4);
  L.total = L.b_off + align256((size_t)N * (size_t)K);
  return L;
}

// hbl_backward's workspace: codes int8 [M][K], scales [M], bf16 copies of
// w [N][K], g_y [M][N], s g_y [M][N] and q [M][K], g_t f32 [M][K]
struct BackwardLayout {
  size_t q_off, s_off, w16_off, gy16_off, gys_off, q16_off, gt_off, total;
};

BackwardLayout backward_layout(int64_t M, int64_t K, int64_t N) {
  const size_t m = (size_t)M, k = (size_t)K, n = (size_t)N;
  BackwardLayout L;
  L.q_off = 0;
  L.s_off = L.q_off + align256(m * k);
  L.w16_off = L.s_off + align256(m * 4);
  L.gy16_off = L.w16_off + align256(n * k * 2);
  L.gys_off = L.gy16_off + align256(m * n * 2);
  L.q16_off = L.gys_off + align256(m * n * 2);
  L.gt_off = L.q16_off + align256(m * k * 2);
  L.total = L.gt_off + align256(m * k * 4);
  return L;
}

}  // namespace

namespace hbl {
hbl_status note_cuda_error(cudaError_t e) { return cuda_status(e); }
}  // namespace hbl

extern "C" {

size_t hbl_packed_ternary_bytes(int64_t K, int64_t N) {
  int l;
  if (check_k(K, &l) != HBL_OK || check_n(N) != HBL_OK) return 0;
  return (size_t)N * (size_t)(K / 4);
}

size_t hbl_codes_bytes(int64_t M, int64_t K, int bits) {
  int l;
  if (check_k(K, &l) != HBL_OK || check_rows(M) != HBL_OK || (bits != 4 && bits != 8)) return 0;
  return bits == 4 ? (size_t)M * (size_t)(K / 2) : (size_t)M * (size_t)K;
}

size_t hbl_pack_ternary_workspace_bytes(int64_t K, int64_t N) {
  int l;
  if (check_k(K, &l) != HBL_OK || check_n(N) != HBL_OK) return 0;
  return sizeof(double) * hbl::kTernaryPartials;
}

size_t hbl_forward_workspace_bytes(int64_t M, int64_t K, int64_t N, int bits) {
  int l;
  if (check_k(K, &l) != HBL_OK || check_rows(M) != HBL_OK || check_n(N) != HBL_OK || (bits != 4 && bits != 8))
    return 0;
  return forward_layout(M, K, N, bits).total;
}

hbl_status hbl_pack_ternary(const void* W, hbl_dtype wt, int64_t K, int64_t N, uint8_t* packed, float* alpha_dev,
                            void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!W || !packed || !alpha_dev || !dtype_ok(wt)) return HBL_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(packed, 16) || !aligned(alpha_dev, 4)) return HBL_ERR_INVALID_ARG;
  int l;
  hbl_status s = check_k(K, &l);
  if (s != HBL_OK) return s;
  if ((s = check_n(N)) != HBL_OK) return s;
  if (!workspace || !aligned(workspace, 16) || workspace_bytes < hbl_pack_ternary_workspace_bytes(K, N))
    return HBL_ERR_WORKSPACE;
  return cuda_status(hbl::launch_pack_ternary(W, wt == HBL_BF16, N, K, packed, alpha_dev,
                                              reinterpret_cast<double*>(workspace), stream));
}

hbl_status hbl_fht_quant(const void* x, hbl_dtype xt, int64_t M, int64_t K, int bits, uint8_t* codes, float* scales,
                         cudaStream_t stream) {
  if (!x || !codes || !scales || !dtype_ok(xt) || (bits != 4 && bits != 8)) return HBL_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(codes, 16) || !aligned(scales, 4)) return HBL_ERR_INVALID_ARG;
  int l;
  hbl_status s = check_k(K, &l);
  if (s != HBL_OK) return s;
  if ((s = check_rows(M)) != HBL_OK) return s;
  const K1Mode mode = bits == 4 ? hbl::K1_Q4_PACKED : hbl::K1_Q8_I8;
  return cuda_status(hbl::launch_ln_fht_quant(x, xt == HBL_BF16, M, l, mode, codes, scales, stream));
}

hbl_status hbl_forward(const void* x, hbl_dtype xt, int64_t M, int64_t K, const uint8_t* packed,
                       const float* alpha_dev, int64_t N, int bits, void* y, hbl_dtype yt, void* workspace,
                       size_t workspace_bytes, cudaStream_t stream) {
  if (!x || !packed || !alpha_dev || !y || !dtype_ok(xt) || !dtype_ok(yt) || (bits != 4 && bits != 8))
    return HBL_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(packed, 16) || !aligned(alpha_dev, 4) || !aligned(y, 16))
    return HBL_ERR_INVALID_ARG;
  int l;
  hbl_status s = check_k(K, &l);
  if (s != HBL_OK) return s;
  if ((s = check_rows(M)) != HBL_OK) return s;
  if ((s = check_n(N)) != HBL_OK) return s;
  const ForwardLayout L = forward_layout(M, K, N, bits);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < L.total) return HBL_ERR_WORKSPACE;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  int8_t* A = reinterpret_cast<int8_t*>(ws + L.a_off);
  float* scales = reinterpret_cast<float*>(ws + L.s_off);
  int8_t* B = reinterpret_cast<int8_t*>(ws + L.b_off);
  cudaError_t e;
  const K1Mode mode = bits == 4 ? hbl::K1_Q4_I8 : hbl::K1_Q8_I8;
  if (hbl::decode_forward_supports(M, K)) {
    // decode-sized batch: one launch quantizes x and takes the product
    // straight from the packed weights (the workspace is not touched)
    return cuda_status(hbl::launch_decode_forward(x, xt == HBL_BF16, M, l, bits, packed, alpha_dev, N,
                                                  yt == HBL_BF16 ? 2 : 1, y, stream));
  }
  if (hbl::gemv_ternary_supports(M, K)) {
    // a few longer rows: the quantizer once, then the product from the packed
    // weights, whose copies start while the quantizer runs
    e = hbl::launch_ln_fht_quant(x, xt == HBL_BF16, M, l, mode, A, scales, stream);
    if (e == cudaSuccess)
      e = hbl::launch_gemv_ternary(A, scales, packed, alpha_dev, M, N, K, yt == HBL_BF16 ? 2 : 1, y, stream,
                                   /*early=*/true);
    return cuda_status(e);
  }
  if (hbl::ln_fht_quant_tc_supports(xt == HBL_BF16, l, mode, x, A)) {
    // the quantizer, with the weight widening in its idle warps when the
    // quantizer's traffic dominates, else in a kernel that overlaps it
    e = hbl::launch_ln_fht_quant_tc_widen(x, M, l, mode, A, scales, packed, N, K, B, stream);
  } else {
    e = hbl::launch_ln_fht_quant(x, xt == HBL_BF16, M, l, mode, A, scales, stream);
    if (e == cudaSuccess) e = hbl::launch_widen_ternary(packed, N, K, B, stream, /*overlap_previous=*/true);
  }
  // |code x weight| <= 8 (INT4 codes, ternary weights) or 128 (INT8)
  if (e == cudaSuccess)
    e = hbl::launch_gemm_i8(A, B, M, N, K, yt == HBL_BF16 ? 2 : 1, y, scales, alpha_dev, stream, bits == 4 ? 8 : 128);
  return cuda_status(e);
}

hbl_status hbl_fht_quant_i8(const void* x, hbl_dtype xt, int64_t M, int64_t K, int bits, int8_t* codes,
                            float* scales, cudaStream_t stream) {
  if (!x || !codes || !scales || !dtype_ok(xt) || (bits != 4 && bits != 8)) return HBL_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(codes, 16) || !aligned(scales, 4)) return HBL_ERR_INVALID_ARG;
  int l;
  hbl_status s = check_k(K, &l);
  if (s != HBL_OK) return s;
  if ((s = check_rows(M)) != HBL_OK) return s;
  const K1Mode mode = bits == 4 ? hbl::K1_Q4_I8 : hbl::K1_Q8_I8;
  return cuda_status(hbl::launch_ln_fht_quant(x, xt == HBL_BF16, M, l, mode, codes, scales, stream));
}

hbl_status hbl_widen_ternary(const uint8_t* packed, int64_t K, int64_t N, int8_t* w, cudaStream_t stream) {
  if (!packed || !w) return HBL_ERR_INVALID_ARG;
  if (!aligned(packed, 16) || !aligned(w, 16)) return HBL_ERR_INVALID_ARG;
  int l;
  hbl_status s = check_k(K, &l);
  if (s != HBL_OK) return s;
  if ((s = check_n(N)) != HBL_OK) return s;
  return cuda_status(hbl::launch_widen_ternary(packed, N, K, w, stream));
}

hbl_status hbl_gemm_dequant(const int8_t* A, const int8_t* w, int64_t M, int64_t N, int64_t K, const float* scales,
                            const float* alpha_dev, void* y, hbl_dtype yt, cudaStream_t stream) {
  if (!A || !w || !scales || !alpha_dev || !y || !dtype_ok(yt)) return HBL_ERR_INVALID_ARG;
  if (!aligned(A, 16) || !aligned(w, 16) || !aligned(scales, 4) || !aligned(alpha_dev, 4) || !aligned(y, 16))
    return HBL_ERR_INVALID_ARG;
  if (K <= 0) return HBL_ERR_INVALID_ARG;
  if (K % 16 != 0 || K > 65536) return HBL_ERR_UNSUPPORTED;
  hbl_status s = check_rows(M);
  if (s != HBL_OK) return s;
  if ((s = check_n(N)) != HBL_OK) return s;
  return cuda_status(hbl::launch_gemm_i8(A, w, M, N, K, yt == HBL_BF16 ? 2 : 1, y, scales, alpha_dev, stream));
}

hbl_status hbl_gemm_tern_dequant(const uint8_t* A, const uint8_t* packed, int64_t M, int64_t N, int64_t K,
                                 const float* scales, const float* alpha_dev, void* y, hbl_dtype yt,
                                 cudaStream_t stream) {
  if (!A || !packed || !scales || !alpha_dev || !y || !dtype_ok(yt)) return HBL_ERR_INVALID_ARG;
  if (!aligned(A, 16) || !aligned(packed, 16) || !aligned(scales, 4) || !aligned(alpha_dev, 4) || !aligned(y, 16))
    return HBL_ERR_INVALID_ARG;
  if (K <= 0) return HBL_ERR_INVALID_ARG;
  if (K % 64 != 0 || K > 32768) return HBL_ERR_UNSUPPORTED;
  hbl_status s = check_rows(M);
  if (s != HBL_OK) return s;
  if ((s = check_n(N)) != HBL_OK) return s;
  if (!hbl::gemm_tern_supports(M, K)) return HBL_ERR_UNSUPPORTED;
  return cuda_status(hbl::launch_gemm_tern(A, packed, M, N, K, yt == HBL_BF16 ? 2 : 1, y, scales, alpha_dev,
                                           stream));
}

hbl_status hbl_gemv_ternary_dequant(const int8_t* A, const uint8_t* packed, int64_t M, int64_t N, int64_t K,
                                    const float* scales, const float* alpha_dev, void* y, hbl_dtype yt,
                                    cudaStream_t stream) {
  if (!A || !packed || !scales || !alpha_dev || !y || !dtype_ok(yt)) return HBL_ERR_INVALID_ARG;
  if (!aligned(A, 16) || !aligned(packed, 16) || !aligned(scales, 4) || !aligned(alpha_dev, 4) || !aligned(y, 4))
    return HBL_ERR_INVALID_ARG;
  int l;
  hbl_status s = check_k(K, &l);
  if (s != HBL_OK) return s;
  if ((s = check_rows(M)) != HBL_OK) return s;
  if ((s = check_n(N)) != HBL_OK) return s;
  if (!hbl::gemv_ternary_supports(M, K)) return HBL_ERR_UNSUPPORTED;
  return cuda_status(hbl::launch_gemv_ternary(A, scales, packed, alpha_dev, M, N, K, yt == HBL_BF16 ? 2 : 1, y,
                                              stream));
}

hbl_status hbl_fht(const void* x, hbl_dtype xt, int64_t M, int64_t K, float* t, cudaStream_t stream) {
  if (!x || !t || !dtype_ok(xt)) return HBL_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(t, 16)) return HBL_ERR_INVALID_ARG;
  int l;
  hbl_status s = check_k(K, &l);
  if (s != HBL_OK) return s;
  if ((s = check_rows(M)) != HBL_OK) return s;
  return cuda_status(hbl::launch_ln_fht_quant(x, xt == HBL_BF16, M, l, hbl::K1_FHT_F32, t, nullptr, stream));
}

size_t hbl_pack_ternary_rotated_workspace_bytes(int64_t K, int64_t N) {
  const size_t base = hbl_pack_ternary_workspace_bytes(K, N);
  if (base == 0) return 0;
  return align256((size_t)N * (size_t)K * 4) + base;
}

hbl_status hbl_pack_ternary_rotated(const void* W, hbl_dtype wt, int64_t K, int64_t N, uint8_t* packed,
                                    float* alpha_dev, void* workspace, size_t workspace_bytes,
                                    cudaStream_t stream) {
  if (!W || !packed || !alpha_dev || !dtype_ok(wt)) return HBL_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(packed, 16) || !aligned(alpha_dev, 4)) return HBL_ERR_INVALID_ARG;
  int l;
  hbl_status s = check_k(K, &l);
  if (s != HBL_OK) return s;
  if ((s = check_n(N)) != HBL_OK) return s;
  const size_t need = hbl_pack_ternary_rotated_workspace_bytes(K, N);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < need) return HBL_ERR_WORKSPACE;
  float* rotated = reinterpret_cast<float*>(workspace);
  double* partials = reinterpret_cast<double*>(reinterpret_cast<uint8_t*>(workspace) +
                                               align256((size_t)N * (size_t)K * 4));
  cudaError_t e = hbl::launch_ln_fht_quant(W, wt == HBL_BF16, N, l, hbl::K1_FHT_F32, rotated, nullptr, stream);
  if (e == cudaSuccess) e = hbl::launch_pack_ternary(rotated, false, N, K, packed, alpha_dev, partials, stream);
  return cuda_status(e);
}

hbl_status hbl_norm_quant(const void* x, hbl_dtype xt, int64_t M, int64_t K, hbl_norm norm, int bits,
                          uint8_t* codes, float* scales, cudaStream_t stream) {
  if (!x || !codes || !scales || !dtype_ok(xt) || (bits != 4 && bits != 8) ||
      (norm != HBL_NORM_LAYER && norm != HBL_NORM_RMS))
    return HBL_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(codes, 16) || !aligned(scales, 4)) return HBL_ERR_INVALID_ARG;
  hbl_status s = check_norm_k(K);
  if (s != HBL_OK) return s;
  if ((s = check_rows(M)) != HBL_OK) return s;
  const K1Mode mode = bits == 4 ? hbl::K1_Q4_PACKED : hbl::K1_Q8_I8;
  return cuda_status(hbl::launch_norm_quant(x, xt == HBL_BF16, M, K, norm == HBL_NORM_RMS, mode, codes, scales,
                                            stream));
}

hbl_status hbl_debug_norm(const void* x, hbl_dtype xt, int64_t M, int64_t K, hbl_norm norm, float* t,
                          cudaStream_t stream) {
  if (!x || !t || !dtype_ok(xt) || (norm != HBL_NORM_LAYER && norm != HBL_NORM_RMS)) return HBL_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(t, 16)) return HBL_ERR_INVALID_ARG;
  hbl_status s = check_norm_k(K);
  if (s != HBL_OK) return s;
  if ((s = check_rows(M)) != HBL_OK) return s;
  return cuda_status(hbl::launch_norm_quant(x, xt == HBL_BF16, M, K, norm == HBL_NORM_RMS, hbl::K1_T_F32, t,
                                            nullptr, stream));
}

hbl_status hbl_debug_ln_fht(const void* x, hbl_dtype xt, int64_t M, int64_t K, float* t, cudaStream_t stream) {
  if (!x || !t || !dtype_ok(xt)) return HBL_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(t, 16)) return HBL_ERR_INVALID_ARG;
  int l;
  hbl_status s = check_k(K, &l);
  if (s != HBL_OK) return s;
  if ((s = check_rows(M)) != HBL_OK) return s;
  return cuda_status(hbl::launch_ln_fht_quant(x, xt == HBL_BF16, M, l, hbl::K1_T_F32, t, nullptr, stream));
}

hbl_status hbl_quant_from_f32(const float* t, int64_t M, int64_t K, int bits, uint8_t* codes, float* scales,
                              cudaStream_t stream) {
  if (!t || !codes || !scales || (bits != 4 && bits != 8)) return HBL_ERR_INVALID_ARG;
  if (!aligned(t, 16) || !aligned(codes, 16) || !aligned(scales, 4)) return HBL_ERR_INVALID_ARG;
  if (K <= 0) return HBL_ERR_INVALID_ARG;
  if (K % 16 != 0 || K > 65536) return HBL_ERR_UNSUPPORTED;
  hbl_status s = check_rows(M);
  if (s != HBL_OK) return s;
  return cuda_status(hbl::launch_quant_from_f32(t, M, K, bits, bits == 4, codes, scales, stream));
}

hbl_status hbl_gemm_i8_i32(const int8_t* A, const int8_t* B, int64_t M, int64_t N, int64_t K, int32_t* acc,
                           cudaStream_t stream) {
  if (!A || !B || !acc) return HBL_ERR_INVALID_ARG;
  if (!aligned(A, 16) || !aligned(B, 16) || !aligned(acc, 16)) return HBL_ERR_INVALID_ARG;
  if (K <= 0) return HBL_ERR_INVALID_ARG;
  if (K % 16 != 0 || K > 65536) return HBL_ERR_UNSUPPORTED;
  hbl_status s = check_rows(M);
  if (s != HBL_OK) return s;
  if ((s = check_n(N)) != HBL_OK) return s;
  return cuda_status(hbl::launch_gemm_i8(A, B, M, N, K, 0, acc, nullptr, nullptr, stream));
}

size_t hbl_backward_workspace_bytes(int64_t M, int64_t K, int64_t N, int bits) {
  int l;
  if (check_k(K, &l) != HBL_OK || check_rows(M) != HBL_OK || check_n(N) != HBL_OK || (bits != 4 && bits != 8))
    return 0;
  return backward_layout(M, K, N).total;
}

hbl_status hbl_backward(const void* x, hbl_dtype xt, int64_t M, int64_t K, const uint8_t* packed,
                        const float* alpha_dev, int64_t N, int bits, const void* g_y, hbl_dtype gyt, void* g_x,
                        float* g_W, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!x || !packed || !alpha_dev || !g_y || !g_x || !g_W || !dtype_ok(xt) || !dtype_ok(gyt) ||
      (bits != 4 && bits != 8))
    return HBL_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(packed, 16) || !aligned(alpha_dev, 4) || !aligned(g_y, 16) || !aligned(g_x, 16) ||
      !aligned(g_W, 16))
    return HBL_ERR_INVALID_ARG;
  int l;
  hbl_status s = check_k(K, &l);
  if (s != HBL_OK) return s;
  if ((s = check_rows(M)) != HBL_OK) return s;
  if ((s = check_n(N)) != HBL_OK) return s;
  const BackwardLayout L = backward_layout(M, K, N);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < L.total) return HBL_ERR_WORKSPACE;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  int8_t* q = reinterpret_cast<int8_t*>(ws + L.q_off);
  float* scales = reinterpret_cast<float*>(ws + L.s_off);
  uint16_t* w16 = reinterpret_cast<uint16_t*>(ws + L.w16_off);
  uint16_t* gy16 = reinterpret_cast<uint16_t*>(ws + L.gy16_off);
  uint16_t* gys = reinterpret_cast<uint16_t*>(ws + L.gys_off);
  uint16_t* q16 = reinterpret_cast<uint16_t*>(ws + L.q16_off);
  float* gt = reinterpret_cast<float*>(ws + L.gt_off);
  const bool gy_bf16 = gyt == HBL_BF16;
  const K1Mode mode = bits == 4 ? hbl::K1_Q4_I8 : hbl::K1_Q8_I8;
  // the forward's codes and scales, recomputed
  cudaError_t e = hbl::launch_ln_fht_quant(x, xt == HBL_BF16, M, l, mode, q, scales, stream);
  // activation gradient: g_t = alpha g_y w, then g_u = H g_t / sqrt(K) and the LayerNorm backward
  if (e == cudaSuccess) e = hbl::launch_ternary_to_bf16(packed, N, K, w16, stream);
  const uint16_t* gyb = reinterpret_cast<const uint16_t*>(g_y);
  if (e == cudaSuccess && !gy_bf16) {
    e = hbl::launch_scale_rows_bf16(g_y, false, nullptr, M, N, gy16, stream);
    gyb = gy16;
  }
  if (e == cudaSuccess) e = hbl::launch_gemm_bf16(gyb, false, w16, M, K, N, gt, alpha_dev, stream);
  // g_u = H g_t / sqrt(K) and the LayerNorm backward in one pass over the rows
  if (e == cudaSuccess) e = hbl::launch_fht_ln_backward(gt, x, xt == HBL_BF16, M, l, g_x, stream);
  // weight gradient: g_W = (s g_y)^T q
  if (e == cudaSuccess) e = hbl::launch_scale_rows_bf16(g_y, gy_bf16, scales, M, N, gys, stream);
  if (e == cudaSuccess) e = hbl::launch_codes_to_bf16(q, M * K, q16, stream);
  if (e == cudaSuccess) e = hbl::launch_gemm_bf16(gys, true, q16, N, K, M, g_W, nullptr, stream);
  return cuda_status(e);
}

hbl_status hbl_gemm_bf16_f32(const uint16_t* A, int a_mn, const uint16_t* B, int64_t R, int64_t C, int64_t Kc,
                             float* D, const float* scale_dev, cudaStream_t stream) {
  if (!A || !B || !D) return HBL_ERR_INVALID_ARG;
  if (!aligned(A, 16) || !aligned(B, 16) || !aligned(D, 16) || (scale_dev && !aligned(scale_dev, 4)))
    return HBL_ERR_INVALID_ARG;
  if (R <= 0 || C <= 0 || Kc <= 0) return HBL_ERR_INVALID_ARG;
  if (R > kMaxRows || C > kMaxRows || Kc > kMaxRows || C % 8 != 0 || (a_mn ? R % 8 : Kc % 8) != 0)
    return HBL_ERR_UNSUPPORTED;
  if (R * C > (int64_t(1) << 40)) return HBL_ERR_UNSUPPORTED;  // keeps the tile count within int
  return cuda_status(hbl::launch_gemm_bf16(A, a_mn != 0, B, R, C, Kc, D, scale_dev, stream));
}

hbl_status hbl_ln_backward(const void* x, hbl_dtype xt, int64_t M, int64_t K, const float* g_u, void* g_x,
                           cudaStream_t stream) {
  if (!x || !g_u || !g_x || !dtype_ok(xt)) return HBL_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(g_u, 16) || !aligned(g_x, 16)) return HBL_ERR_INVALID_ARG;
  int l;
  hbl_status s = check_k(K, &l);
  if (s != HBL_OK) return s;
  if ((s = check_rows(M)) != HBL_OK) return s;
  return cuda_status(hbl::launch_ln_backward(x, xt == HBL_BF16, g_u, M, l, g_x, stream));
}

hbl_status hbl_fht_ln_backward(const float* g, const void* x, hbl_dtype xt, int64_t M, int64_t K, void* g_x,
                               cudaStream_t stream) {
  if (!g || !x || !g_x || !dtype_ok(xt)) return HBL_ERR_INVALID_ARG;
  if (!aligned(g, 16) || !aligned(x, 16) || !aligned(g_x, 16)) return HBL_ERR_INVALID_ARG;
  int l;
  hbl_status s = check_k(K, &l);
  if (s != HBL_OK) return s;
  if ((s = check_rows(M)) != HBL_OK) return s;
  return cuda_status(hbl::launch_fht_ln_backward(g, x, xt == HBL_BF16, M, l, g_x, stream));
}

hbl_status hbl_kv_quant(const void* x, hbl_dtype xt, int64_t rows, int64_t D, int bits, uint8_t* codes,
                        float* scales, cudaStream_t stream) {
  if (!x || !codes || !scales || !dtype_ok(xt)) return HBL_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(codes, 16) || !aligned(scales, 4)) return HBL_ERR_INVALID_ARG;
  if (rows <= 0 || D <= 0 || bits <= 0) return HBL_ERR_INVALID_ARG;
  if ((D != 32 && D != 64 && D != 128 && D != 256) || bits < 2 || bits > 8 || rows > kMaxRows * 64)
    return HBL_ERR_UNSUPPORTED;
  return cuda_status(hbl::launch_kv_quant(x, xt == HBL_BF16, rows, D, bits, codes, scales, stream));
}

hbl_status hbl_last_device_error(cudaStream_t stream) {
  int v = 0;
  cudaError_t e = hbl::read_and_clear_device_error(stream, &v);
  if (e != cudaSuccess) return cuda_status(e);
  return v ? HBL_ERR_TIMEOUT : HBL_OK;
}

hbl_status hbl_debug_raise_device_error(cudaStream_t stream) {
  return cuda_status(hbl::raise_device_error(stream));
}

hbl_status hbl_debug_set_wait_limit_ns(uint64_t ns) { return cuda_status(hbl::set_wait_limit(ns)); }

const char* hbl_status_string(hbl_status status) {
  switch (status) {
    case HBL_OK: return "HBL_OK";
    case HBL_ERR_INVALID_ARG: return "HBL_ERR_INVALID_ARG";
    case HBL_ERR_UNSUPPORTED: return "HBL_ERR_UNSUPPORTED";
    case HBL_ERR_WORKSPACE: return "HBL_ERR_WORKSPACE";
    case HBL_ERR_CUDA: return "HBL_ERR_CUDA";
    case HBL_ERR_TIMEOUT: return "HBL_ERR_TIMEOUT";
  }
  return "HBL_ERR_UNKNOWN";
}

int hbl_last_cuda_error(void) { return g_last_cuda_error; }

const char* hbl_cuda_error_name(int code) { return cudaGetErrorName((cudaError_t)code); }

}  // extern "C"
