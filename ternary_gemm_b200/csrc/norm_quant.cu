// Activation path of a BitLinear layer without the Hadamard transform:
// LayerNorm or RMSNorm per token row, then the same per-token quantizer as
// H-BitLinear ("BitNet v2: Native 4-bit Activations with Hadamard
// Transformation for 1-bit LLMs": the other linear layers of the 4-bit model
// quantize their inputs to INT4 without the rotation, and BitNet b1.58 keeps
// 8-bit absmax activations; section "BitNet v2: native 4-bit activations").
//
// The row layout is the one of the fused transform kernel's first pass: T =
// K/64 threads per row, each holding 64 elements as eight 16-byte vectors
// T*8 elements apart (coalesced loads, runs of 8 codes for the stores), R rows
// per CTA so a CTA has >= 128 threads, 2-3 row-wide reductions and no other
// exchange.  Against the fused kernel this measures what the transform costs.
#include <cstdint>

#include "common.cuh"
#include "quant.cuh"
#include "rowkit.cuh"

namespace hbl {
namespace {

using namespace rowkit;

template <int LOGK>
struct NShape {
  static constexpr int K = 1 << LOGK;
  static constexpr int T = K / 64;
  static constexpr int R = T >= 128 ? 1 : 128 / T;
  static constexpr int THREADS = T * R;
  static constexpr int MINB = THREADS >= 512 ? 1 : (THREADS >= 256 ? 3 : 5);
  static constexpr int WPR = T > 32 ? T / 32 : 1;
};

// MODE: K1_T_F32 (normalised float out), K1_Q4_PACKED, K1_Q4_I8, K1_Q8_I8.
template <int LOGK, bool BF16, int MODE, bool RMS>
__global__ void __launch_bounds__(NShape<LOGK>::THREADS, NShape<LOGK>::MINB)
norm_quant_kernel(const void* __restrict__ x, int64_t M, void* __restrict__ out, float* __restrict__ scales) {
  using S = NShape<LOGK>;
  constexpr int K = S::K, T = S::T, R = S::R;
  __shared__ float red_f[3][R * S::WPR];
  __shared__ double red_d[R * S::WPR];

  const int tid = threadIdx.x;
  const int rl = tid / T;
  const int t = tid % T;
  const int64_t row = (int64_t)blockIdx.x * R + rl;
  const bool active = row < M;
  const size_t esz = BF16 ? 2 : 4;
  const void* xrow = reinterpret_cast<const unsigned char*>(x) + (size_t)(active ? row : 0) * K * esz;

  float e[64];
  float f8[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  if (active) {
    if constexpr (!RMS) load8<BF16>(xrow, 0, f8);
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) load8<BF16>(xrow, (jj * T + t) * 8, &e[jj * 8]);
  } else {
#pragma unroll
    for (int r = 0; r < 64; ++r) e[r] = 0.0f;
  }
  constexpr float invK = 1.0f / (float)K;  // exact: K is a power of two
  if constexpr (!RMS) {
    // shifted two-pass mean: subtract the mean of the row's first 8 values
    // (identical in every thread) so the float sum sees residuals, not a
    // large common offset
    const float shift = (((f8[0] + f8[1]) + (f8[2] + f8[3])) + ((f8[4] + f8[5]) + (f8[6] + f8[7]))) * 0.125f;
#pragma unroll
    for (int r = 0; r < 64; r += 2) sub2(e[r], e[r + 1], shift);
    float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
    for (int r = 0; r < 64; r += 2) {
      a0 += e[r];
      a1 += e[r + 1];
    }
    const float mu = RowReduce<T, S::WPR>::run(a0 + a1, AddF(), red_f[0], rl, t) * invK;
#pragma unroll
    for (int r = 0; r < 64; r += 2) sub2(e[r], e[r + 1], mu);
  }
  float s0 = 0.0f, s1 = 0.0f;
#pragma unroll
  for (int r = 0; r < 64; r += 2) sq_acc2(s0, s1, e[r], e[r + 1]);
  const float ss = RowReduce<T, S::WPR>::run(s0 + s1, AddF(), red_f[1], rl, t);
  const float rstd = __fdiv_rn(1.0f, sqrtf(__fadd_rn(ss * invK, 1e-5f)));
#pragma unroll
  for (int r = 0; r < 64; r += 2) mul2(e[r], e[r + 1], rstd);

  if constexpr (MODE == K1_T_F32) {
    if (active) {
      float* orow = reinterpret_cast<float*>(out) + (size_t)row * K;
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        float4* dst = reinterpret_cast<float4*>(orow + (jj * T + t) * 8);
        dst[0] = make_float4(e[8 * jj], e[8 * jj + 1], e[8 * jj + 2], e[8 * jj + 3]);
        dst[1] = make_float4(e[8 * jj + 4], e[8 * jj + 5], e[8 * jj + 6], e[8 * jj + 7]);
      }
    }
  } else {
    q::RowParams p;
    if constexpr (MODE == K1_Q8_I8) {
      float g = 0.0f;
#pragma unroll
      for (int r = 0; r < 64; ++r) g = fmaxf(g, fabsf(e[r]));
      p = q::params_int8(RowReduce<T, S::WPR>::run(g, MaxF(), red_f[2], rl, t));
    } else {
      double a0 = 0.0, a1 = 0.0;
#pragma unroll
      for (int r = 0; r < 64; r += 2) {
        a0 += q::abs_f64(e[r]);
        a1 += q::abs_f64(e[r + 1]);
      }
      p = q::params_int4(RowReduce<T, S::WPR>::run(a0 + a1, AddD(), red_d, rl, t), K);
    }
    if (!active) return;
    if (t == 0) scales[row] = p.scale();
    uint32_t m[64];
#pragma unroll
    for (int r = 0; r < 64; r += 2) magic2(e[r], e[r + 1], p.r, m[r], m[r + 1]);
    if constexpr (MODE == K1_Q4_PACKED) {
      uint32_t* orow = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(out) + (size_t)row * (K / 2));
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        int n[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) n[u] = (int)m[8 * jj + u] - q::kMagicBits;
        orow[jj * T + t] = q::pack_s4x8(n);
      }
    } else {
      if constexpr (MODE == K1_Q4_I8) {
#pragma unroll
        for (int r = 0; r < 64; ++r) m[r] = q::clip_magic_int4(m[r]);
      }
      uint2* orow = reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(out) + (size_t)row * K);
#pragma unroll
      for (int jj = 0; jj < 8; ++jj)
        orow[jj * T + t] = make_uint2(q::gather_low_bytes(m[8 * jj], m[8 * jj + 1], m[8 * jj + 2], m[8 * jj + 3]),
                                      q::gather_low_bytes(m[8 * jj + 4], m[8 * jj + 5], m[8 * jj + 6], m[8 * jj + 7]));
    }
  }
}

template <int LOGK, bool BF16, bool RMS>
cudaError_t launch_k(const void* x, int64_t M, K1Mode mode, void* out, float* scales, cudaStream_t s) {
  using S = NShape<LOGK>;
  const unsigned grid = (unsigned)((M + S::R - 1) / S::R);
  switch (mode) {
    case K1_T_F32: norm_quant_kernel<LOGK, BF16, K1_T_F32, RMS><<<grid, S::THREADS, 0, s>>>(x, M, out, scales); break;
    case K1_Q4_PACKED:
      norm_quant_kernel<LOGK, BF16, K1_Q4_PACKED, RMS><<<grid, S::THREADS, 0, s>>>(x, M, out, scales);
      break;
    case K1_Q4_I8: norm_quant_kernel<LOGK, BF16, K1_Q4_I8, RMS><<<grid, S::THREADS, 0, s>>>(x, M, out, scales); break;
    case K1_Q8_I8: norm_quant_kernel<LOGK, BF16, K1_Q8_I8, RMS><<<grid, S::THREADS, 0, s>>>(x, M, out, scales); break;
  }
  return cudaGetLastError();
}

template <bool BF16, bool RMS>
cudaError_t launch_norm(const void* x, int64_t M, int64_t K, K1Mode mode, void* out, float* scales,
                        cudaStream_t s) {
  switch (K) {
    case 256: return launch_k<8, BF16, RMS>(x, M, mode, out, scales, s);
    case 512: return launch_k<9, BF16, RMS>(x, M, mode, out, scales, s);
    case 1024: return launch_k<10, BF16, RMS>(x, M, mode, out, scales, s);
    case 2048: return launch_k<11, BF16, RMS>(x, M, mode, out, scales, s);
    case 4096: return launch_k<12, BF16, RMS>(x, M, mode, out, scales, s);
    case 8192: return launch_k<13, BF16, RMS>(x, M, mode, out, scales, s);
    case 16384: return launch_k<14, BF16, RMS>(x, M, mode, out, scales, s);
    case 32768: return launch_k<15, BF16, RMS>(x, M, mode, out, scales, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_norm_quant(const void* x, bool in_bf16, int64_t M, int64_t K, bool rms, K1Mode mode, void* out,
                              float* scales, cudaStream_t stream) {
  if (in_bf16)
    return rms ? launch_norm<true, true>(x, M, K, mode, out, scales, stream)
               : launch_norm<true, false>(x, M, K, mode, out, scales, stream);
  return rms ? launch_norm<false, true>(x, M, K, mode, out, scales, stream)
             : launch_norm<false, false>(x, M, K, mode, out, scales, stream);
}

}  // namespace hbl
