// The H-BitLinear backward pass ("BitNet v2: Native 4-bit Activations with
// Hadamard Transformation for 1-bit LLMs", training strategy: the
// straight-through estimator takes the gradient around the non-differentiable
// quantizers, and the orthogonality of the Hadamard matrix carries it through
// the transform).  With t = H LN(x) / sqrt(K), (q, s) its per-token codes and
// scales, and (w, alpha) the ternary weight, the forward is
// y = (s q) (alpha w)^T; given g_y:
//
//   g_t = alpha g_y w                   [M][K]   (bf16 tensor-core GEMM, f32 out)
//   g_u = H g_t / sqrt(K)               [M][K]   (H symmetric and orthogonal up to sqrt K)
//   g_x = (g_u - mean(g_u) - u mean(g_u u)) / sigma,  u = (x - mu) / sigma   (LayerNorm backward)
//   g_W = g_y^T (s q)                   [N][K]   (bf16 tensor-core GEMM, f32 out)
//
// This file holds the memory-bound steps: the operand conversions to bf16
// (ternary weights, integer codes: both exact; g_y s: one rounding) and the
// LayerNorm backward.  Each is a grid-stride or row-per-CTA streaming kernel.
#include <cstdint>

#include <cuda_bf16.h>

#include "common.cuh"
#include "sm100.cuh"

namespace hbl {
namespace {

constexpr int kEwThreads = 256;

int ew_grid(int64_t work) {
  const int64_t g = (work + kEwThreads - 1) / kEwThreads;
  const int64_t cap = (int64_t)sm100_host::sm_count() * 16;
  return (int)(g < 1 ? 1 : (g < cap ? g : cap));
}

// Ternary 2-bit codes (00 = 0, 01 = +1, 11 = -1, element 4j + i at bits
// 2i .. 2i+1 of byte j) -> bf16, 16 codes per 32-bit word per thread.
__global__ void __launch_bounds__(kEwThreads)
ternary_to_bf16_kernel(const uint32_t* __restrict__ packed, int64_t nwords, uint4* __restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * kEwThreads + threadIdx.x; i < nwords; i += (int64_t)gridDim.x * kEwThreads) {
    const uint32_t v = __ldg(packed + i);
    uint32_t h[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      uint32_t pair = 0;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const uint32_t f = (v >> (4 * e + 2 * u)) & 3u;
        // +1 -> 0x3F80, -1 -> 0xBF80, 0 -> 0
        const uint32_t b = (f & 1u) ? (0x3F80u | ((f & 2u) << 14)) : 0u;
        pair |= b << (16 * u);
      }
      h[e] = pair;
    }
    out[2 * i] = make_uint4(h[0], h[1], h[2], h[3]);
    out[2 * i + 1] = make_uint4(h[4], h[5], h[6], h[7]);
  }
}

// int8 codes -> bf16 (exact: |q| <= 128), 16 per thread and step
__global__ void __launch_bounds__(kEwThreads)
codes_to_bf16_kernel(const int4* __restrict__ q, int64_t n16, uint4* __restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * kEwThreads + threadIdx.x; i < n16; i += (int64_t)gridDim.x * kEwThreads) {
    const int4 v = __ldg(q + i);
    const uint32_t w[4] = {(uint32_t)v.x, (uint32_t)v.y, (uint32_t)v.z, (uint32_t)v.w};
    uint32_t h[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t word = w[e >> 1];
      const int lo = (int)(int8_t)((word >> (16 * (e & 1))) & 0xFFu);
      const int hi = (int)(int8_t)((word >> (16 * (e & 1) + 8)) & 0xFFu);
      h[e] = (uint32_t)__bfloat16_as_ushort(__int2bfloat16_rn(lo)) |
             ((uint32_t)__bfloat16_as_ushort(__int2bfloat16_rn(hi)) << 16);
    }
    out[2 * i] = make_uint4(h[0], h[1], h[2], h[3]);
    out[2 * i + 1] = make_uint4(h[4], h[5], h[6], h[7]);
  }
}

// out[m][n] = bf16(g[m][n] * s[m]) (s null: bf16(g), exact for bf16 g);
// g bf16 or float; 4 elements per thread and step (N % 4 == 0)
template <bool G_BF16>
__global__ void __launch_bounds__(kEwThreads)
scale_rows_bf16_kernel(const void* __restrict__ g, const float* __restrict__ s, int64_t M, int64_t N,
                       uint2* __restrict__ out) {
  const int64_t n4 = M * N / 4;
  for (int64_t i = (int64_t)blockIdx.x * kEwThreads + threadIdx.x; i < n4; i += (int64_t)gridDim.x * kEwThreads) {
    const int64_t m = (4 * i) / N;
    const float sm = s ? __ldg(s + m) : 1.0f;
    float v[4];
    if constexpr (G_BF16) {
      const uint2 u = __ldg(reinterpret_cast<const uint2*>(g) + i);
      v[0] = __uint_as_float(u.x << 16);
      v[1] = __uint_as_float(u.x & 0xFFFF0000u);
      v[2] = __uint_as_float(u.y << 16);
      v[3] = __uint_as_float(u.y & 0xFFFF0000u);
    } else {
      const float4 f = __ldg(reinterpret_cast<const float4*>(g) + i);
      v[0] = f.x;
      v[1] = f.y;
      v[2] = f.z;
      v[3] = f.w;
    }
    uint32_t h[2];
#pragma unroll
    for (int e = 0; e < 2; ++e)
      h[e] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(v[2 * e], sm))) |
             ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(v[2 * e + 1], sm))) << 16);
    out[i] = make_uint2(h[0], h[1]);
  }
}

// Sum of two floats over the block (every thread gets the totals).
template <int T>
__device__ __forceinline__ float2 block_sum2(float2 v, float2* red) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    v.x += __shfl_xor_sync(0xffffffffu, v.x, o);
    v.y += __shfl_xor_sync(0xffffffffu, v.y, o);
  }
  constexpr int W = T / 32;
  if constexpr (W > 1) {
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) red[warp] = v;
    __syncthreads();
    float2 t = red[0];
#pragma unroll
    for (int w = 1; w < W; ++w) {
      t.x += red[w].x;
      t.y += red[w].y;
    }
    __syncthreads();  // the slots are reused by the next reduction
    return t;
  }
  return v;
}

// LayerNorm backward, one CTA of T threads per row, V = K / T values per
// thread (element T j + tid).  Statistics in float: mu and var recomputed from
// x (two passes over the registers, as the forward), then
// g_x = (g_u - mean g_u - u mean(g_u u)) / sigma.  With 1024 threads (64
// registers each) only x stays in registers and g_u is read again in each
// pass (from L1/L2).
template <int T, int V, bool X_BF16>
__global__ void __launch_bounds__(T)
ln_backward_kernel(const void* __restrict__ x, const float* __restrict__ gu, int64_t M, void* __restrict__ gx) {
  constexpr int K = T * V;
  constexpr bool KEEP = T < 1024;  // g_u kept in registers
  __shared__ float2 red[T / 32 > 1 ? T / 32 : 1];
  const int64_t row = blockIdx.x;
  if (row >= M) return;
  const float* gr = gu + row * K + threadIdx.x;
  float xv[V], gv[KEEP ? V : 1];
#pragma unroll
  for (int j = 0; j < V; ++j) {
    const int64_t idx = row * K + (int64_t)T * j + threadIdx.x;
    if constexpr (X_BF16)
      xv[j] = __uint_as_float((uint32_t)__ldg(reinterpret_cast<const uint16_t*>(x) + idx) << 16);
    else
      xv[j] = __ldg(reinterpret_cast<const float*>(x) + idx);
    if constexpr (KEEP) gv[j] = __ldg(gr + T * j);
  }
  auto g_at = [&](int j) -> float {
    if constexpr (KEEP) return gv[j];
    else return __ldg(gr + T * j);
  };
  float2 a = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int j = 0; j < V; ++j) {
    a.x += xv[j];
    a.y += g_at(j);
  }
  a = block_sum2<T>(a, red);
  const float mu = a.x / (float)K;
  const float mg = a.y / (float)K;
  float2 b = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int j = 0; j < V; ++j) {
    const float d = xv[j] - mu;
    b.x = fmaf(d, d, b.x);
    b.y = fmaf(g_at(j), d, b.y);
  }
  b = block_sum2<T>(b, red);
  const float var = b.x / (float)K;
  const float rs = rsqrtf(var + 1e-5f);  // 1 / sigma
  // mean(g_u u) = rs mean(g_u (x - mu))
  const float mgu = rs * (b.y / (float)K);
#pragma unroll
  for (int j = 0; j < V; ++j) {
    const int64_t idx = row * K + (int64_t)T * j + threadIdx.x;
    const float u = (xv[j] - mu) * rs;
    const float r = (g_at(j) - mg - u * mgu) * rs;
    if constexpr (X_BF16)
      reinterpret_cast<__nv_bfloat16*>(gx)[idx] = __float2bfloat16_rn(r);
    else
      reinterpret_cast<float*>(gx)[idx] = r;
  }
}

template <int T, int V>
cudaError_t launch_lnb(const void* x, bool x_bf16, const float* gu, int64_t M, void* gx, cudaStream_t stream) {
  if (x_bf16)
    ln_backward_kernel<T, V, true><<<(unsigned)M, T, 0, stream>>>(x, gu, M, gx);
  else
    ln_backward_kernel<T, V, false><<<(unsigned)M, T, 0, stream>>>(x, gu, M, gx);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ternary_to_bf16(const uint8_t* packed, int64_t N, int64_t K, uint16_t* out, cudaStream_t stream) {
  const int64_t words = N * K / 16;
  if (words <= 0) return cudaSuccess;
  ternary_to_bf16_kernel<<<ew_grid(words), kEwThreads, 0, stream>>>(reinterpret_cast<const uint32_t*>(packed), words,
                                                                      reinterpret_cast<uint4*>(out));
  return cudaGetLastError();
}

cudaError_t launch_codes_to_bf16(const int8_t* q, int64_t count, uint16_t* out, cudaStream_t stream) {
  const int64_t n16 = count / 16;
  if (n16 <= 0) return cudaSuccess;
  codes_to_bf16_kernel<<<ew_grid(n16), kEwThreads, 0, stream>>>(reinterpret_cast<const int4*>(q), n16,
                                                                  reinterpret_cast<uint4*>(out));
  return cudaGetLastError();
}

cudaError_t launch_scale_rows_bf16(const void* g, bool g_bf16, const float* s, int64_t M, int64_t N, uint16_t* out,
                                   cudaStream_t stream) {
  const int64_t n4 = M * N / 4;
  if (n4 <= 0) return cudaSuccess;
  if (g_bf16)
    scale_rows_bf16_kernel<true><<<ew_grid(n4), kEwThreads, 0, stream>>>(g, s, M, N, reinterpret_cast<uint2*>(out));
  else
    scale_rows_bf16_kernel<false><<<ew_grid(n4), kEwThreads, 0, stream>>>(g, s, M, N, reinterpret_cast<uint2*>(out));
  return cudaGetLastError();
}

cudaError_t launch_ln_backward(const void* x, bool x_bf16, const float* gu, int64_t M, int log2k, void* gx,
                               cudaStream_t stream) {
  if (M <= 0) return cudaSuccess;
  if (M > INT32_MAX) return cudaErrorInvalidValue;
  switch (log2k) {  // T = clamp(K / 32, 32, 1024) threads, V = K / T values each
    case 6: return launch_lnb<32, 2>(x, x_bf16, gu, M, gx, stream);
    case 7: return launch_lnb<32, 4>(x, x_bf16, gu, M, gx, stream);
    case 8: return launch_lnb<32, 8>(x, x_bf16, gu, M, gx, stream);
    case 9: return launch_lnb<32, 16>(x, x_bf16, gu, M, gx, stream);
    case 10: return launch_lnb<32, 32>(x, x_bf16, gu, M, gx, stream);
    case 11: return launch_lnb<64, 32>(x, x_bf16, gu, M, gx, stream);
    case 12: return launch_lnb<128, 32>(x, x_bf16, gu, M, gx, stream);
    case 13: return launch_lnb<256, 32>(x, x_bf16, gu, M, gx, stream);
    case 14: return launch_lnb<512, 32>(x, x_bf16, gu, M, gx, stream);
    case 15: return launch_lnb<1024, 32>(x, x_bf16, gu, M, gx, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace hbl
