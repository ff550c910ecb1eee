// Fused LayerNorm -> fast Walsh-Hadamard transform -> per-token quantization
// (the activation path of H-BitLinear in "BitNet v2: Native 4-bit
// Activations with Hadamard Transformation for 1-bit LLMs", section
// "H-BitLinear": the Hadamard-transform definition, computed with the fast
// Hadamard transform in O(n log n), and the activation-quantization formula).
//
// One row of K = 2^k elements is spread over T = K/64 threads holding 64
// floats each in registers; R rows share a CTA so that a CTA has >= 128
// threads, and the register budget is set so that 3-5 CTAs share an SM: the
// butterflies (FMA pipe), the integer work of the quantizer (ALU pipe) and
// the exchanges (shared memory) of different rows then overlap.  The Sylvester transform is the product of
// one 2-point butterfly per index bit and those factors commute, so the k
// stages may run in any order.  Three passes cover all bits with two trips
// through shared memory:
//   pass 1: coalesced 16-byte loads give each thread index bits {0,1,2} (within
//           a 16-byte vector) and the top three bits {k-3,k-2,k-1} (eight
//           vectors T*8 elements apart); those 6 stages run in registers.
//   pass 2: (k >= 10) each thread reads 2^(k-9) vectors of 2^(15-k) contiguous
//           floats spanning bits {6..k-4} and runs those stages.
//   pass 3: each thread reads 64 contiguous elements (bits 0..5) and runs the
//           stages of bits {3,4,5} not done yet; the row is complete and each
//           thread's slice is contiguous, ready for the quantizer and 16-byte
//           stores.
// Shared memory uses an XOR swizzle of index bits 5..8 into bits 2..4; it is
// linear over GF(2), so an address splits into a per-thread part (eight
// precomputed bases) and a compile-time offset.  The accesses of all three
// passes are free of bank conflicts for K = 512, 1024 and K >= 4096; pass 2
// at K = 2048 is 2-way (its threads differ in index bits 4, 5 and 8, and bit
// 8 folds onto bit 4), and at K = 64 .. 256 rows of a quarter-warp share
// banks through the row padding (4-way at 64, 2-way at 128 and 256).
// Butterflies, scaling and the
// quantizer's products run as paired f32x2 instructions (one issue slot for
// two IEEE float operations).
//
// LayerNorm is folded around the transform: a row offset mu~ (the mean of the
// row's first 8 values, identical in every thread) is subtracted first when it
// exceeds their spread, so that large means do not cost precision; then
// Y = H (x - mu~) (mu~ = 0 otherwise).  Because row 0
// of H is all ones, Y_0 = K (mu - mu~) and sum_{i>=1} Y_i^2 = K^2 var, so
//   t_i = Y_i / sqrt(K (var + eps_ln))  for i >= 1,   t_0 = 0,
// which is exactly H LN(x) / sqrt(K) with the biased variance and no affine.
#include <cstdint>

#include <cuda_bf16.h>

#include "common.cuh"
#include "sm100.cuh"
#include "quant.cuh"
#include "rowkit.cuh"
#include "fht_rows.cuh"

namespace hbl {
namespace {

using namespace rowkit;
using namespace fhtrows;

// One CTA handles one group of R rows.
// Sum of four floats over the T threads of a row (the RowReduce pattern with a
// float4 slot per warp; every thread of the row ends with the same totals).
template <int T, int WPR>
__device__ __forceinline__ float4 row_sum4(float4 v, float4* red, int rl, int t) {
  constexpr int W = T < 32 ? T : 32;
#pragma unroll
  for (int o = W / 2; o >= 1; o >>= 1) {
    v.x += __shfl_xor_sync(0xffffffffu, v.x, o);
    v.y += __shfl_xor_sync(0xffffffffu, v.y, o);
    v.z += __shfl_xor_sync(0xffffffffu, v.z, o);
    v.w += __shfl_xor_sync(0xffffffffu, v.w, o);
  }
  if constexpr (T > 32) {
    if ((t & 31) == 0) red[rl * WPR + (t >> 5)] = v;
    __syncthreads();
    float4 s = red[rl * WPR];
#pragma unroll
    for (int w = 1; w < WPR; ++w) {
      s.x += red[rl * WPR + w].x;
      s.y += red[rl * WPR + w].y;
      s.z += red[rl * WPR + w].z;
      s.w += red[rl * WPR + w].w;
    }
    v = s;
  }
  return v;
}

template <int LOGK, bool BF16, int MODE>
__global__ void __launch_bounds__(Shape<LOGK>::THREADS, Shape<LOGK>::MINB)
ln_fht_quant_kernel(const void* __restrict__ x, int64_t M, float sK, void* __restrict__ out,
                    float* __restrict__ scales, const void* __restrict__ aux) {
  using S = Shape<LOGK>;
  constexpr int K = S::K, T = S::T, R = S::R;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* smem = reinterpret_cast<float*>(smem_raw);
  void* red1 = smem_raw + S::XCH;
  void* red2 = smem_raw + S::XCH + S::RED;

  const int tid = threadIdx.x;
  const int rl = tid / T;
  const int t = tid % T;
  const int64_t row = (int64_t)blockIdx.x * R + rl;
  const bool active = row < M;
  // K1_LNBWD transforms a float gradient row; BF16 then describes the
  // LayerNorm input x (aux) and the output
  constexpr bool IN_BF16 = MODE == K1_LNBWD ? false : BF16;
  const size_t esz = IN_BF16 ? 2 : 4;
  const void* xrow = reinterpret_cast<const unsigned char*>(x) + (size_t)(active ? row : 0) * K * esz;
  // the plain transform and the backward transform have no forward LayerNorm
  constexpr bool kLN = MODE != K1_FHT_F32 && MODE != K1_LNBWD;
  // a programmatic dependent of this kernel may start now (it waits for this
  // kernel's results itself before reading them)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  float e[64];
  fht_ln_rows<S, IN_BF16, kLN>(xrow, active, rl, t, smem, reinterpret_cast<float*>(red1), sK, e);
  const int base = t * 64;

  if constexpr (MODE == K1_LNBWD) {
    // e = g_u[base .. base + 63]; the LayerNorm backward at the forward's x of
    // the same elements: g_x = (g_u - mean g_u - u mean(g_u u)) / sigma.
    // Statistics on x - x0 (x0 the row's first value, the same in every
    // thread) so that a large row mean costs no precision; one reduction of
    // four sums: sum d, sum d^2, sum g_u d, sum g_u.
    const unsigned char* xl = reinterpret_cast<const unsigned char*>(aux) + (size_t)(active ? row : 0) * K * (BF16 ? 2 : 4);
    float x0 = 0.0f;
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (active) {
      float f0[8];
      load8<BF16>(xl, 0, f0);
      x0 = f0[0];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float xv[8];
        load8<BF16>(xl, base + 8 * j, xv);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float d = xv[u] - x0;
          acc.x += d;
          acc.y = fmaf(d, d, acc.y);
          acc.z = fmaf(e[8 * j + u], d, acc.z);
          acc.w += e[8 * j + u];
        }
      }
    }
    acc = row_sum4<T, S::WPR>(acc, reinterpret_cast<float4*>(red1), rl, t);
    const float invK = 1.0f / (float)K;
    const float mu = acc.x * invK;                            // mean of x - x0
    const float var = fmaxf(acc.y * invK - mu * mu, 0.0f);
    const float rs = rsqrtf(var + 1e-5f);                     // 1 / sigma
    const float mg = acc.w * invK;                            // mean g_u
    const float mgu = rs * (acc.z * invK - mu * mg);          // mean(g_u u)
    if (active) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float xv[8], r[8];
        load8<BF16>(xl, base + 8 * j, xv);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float uu = (xv[u] - x0 - mu) * rs;
          r[u] = (e[8 * j + u] - mg - uu * mgu) * rs;
        }
        if constexpr (BF16) {
          uint32_t h[4];
#pragma unroll
          for (int u = 0; u < 4; ++u)
            h[u] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(r[2 * u])) |
                   ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(r[2 * u + 1])) << 16);
          reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(out) + (size_t)row * K + base)[j] =
              make_uint4(h[0], h[1], h[2], h[3]);
        } else {
          float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + (size_t)row * K + base + 8 * j);
          dst[0] = make_float4(r[0], r[1], r[2], r[3]);
          dst[1] = make_float4(r[4], r[5], r[6], r[7]);
        }
      }
    }
  } else if constexpr (MODE == K1_T_F32 || MODE == K1_FHT_F32) {
    if (active) {
      float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + (size_t)row * K + base);
#pragma unroll
      for (int j = 0; j < 16; ++j) dst[j] = make_float4(e[4 * j], e[4 * j + 1], e[4 * j + 2], e[4 * j + 3]);
    }
  } else {
    const q::RowParams p = row_params<S, MODE>(e, red2, rl, t);
    if (active) {
      if (t == 0) scales[row] = p.scale();
      if constexpr (MODE == K1_Q4_PACKED) {
        uint32_t m[64];
#pragma unroll
        for (int r = 0; r < 64; r += 2) magic2(e[r], e[r + 1], p.r, m[r], m[r + 1]);
        uint32_t w[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          int n[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) n[u] = (int)m[8 * j + u] - q::kMagicBits;
          w[j] = q::pack_s4x8(n);
        }
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(out) + (size_t)row * (K / 2) + base / 2);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
      } else {
        uint32_t w[16];
        codes64_i8<MODE>(e, p.r, w);
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(out) + (size_t)row * K + base);
#pragma unroll
        for (int j = 0; j < 4; ++j) dst[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
      }
    }
  }
}

template <int LOGK, bool BF16, int MODE>
cudaError_t launch_one(const void* x, int64_t M, void* out, float* scales, cudaStream_t stream,
                       const void* aux = nullptr) {
  using S = Shape<LOGK>;
  auto kern = ln_fht_quant_kernel<LOGK, BF16, MODE>;
  static std::atomic<bool> smem_set[sm100_host::kMaxDevices];
  cudaError_t e = sm100_host::ensure_smem(kern, (int)S::SMEM, smem_set);
  if (e != cudaSuccess) return e;
  const int64_t grid = (M + S::R - 1) / S::R;
  const float sK = (float)(1.0 / sqrt((double)S::K));
  kern<<<(unsigned)grid, S::THREADS, S::SMEM, stream>>>(x, M, sK, out, scales, aux);
  return cudaGetLastError();
}

template <int LOGK, bool BF16>
cudaError_t launch_mode(const void* x, int64_t M, K1Mode mode, void* out, float* scales, cudaStream_t s) {
  switch (mode) {
    case K1_T_F32: return launch_one<LOGK, BF16, K1_T_F32>(x, M, out, scales, s);
    case K1_Q4_PACKED: return launch_one<LOGK, BF16, K1_Q4_PACKED>(x, M, out, scales, s);
    case K1_Q4_I8: return launch_one<LOGK, BF16, K1_Q4_I8>(x, M, out, scales, s);
    case K1_Q8_I8: return launch_one<LOGK, BF16, K1_Q8_I8>(x, M, out, scales, s);
    case K1_FHT_F32: return launch_one<LOGK, BF16, K1_FHT_F32>(x, M, out, scales, s);
  }
  return cudaErrorInvalidValue;
}

template <int LOGK>
cudaError_t launch_k(const void* x, bool bf16, int64_t M, K1Mode mode, void* out, float* scales,
                     cudaStream_t s) {
  return bf16 ? launch_mode<LOGK, true>(x, M, mode, out, scales, s)
              : launch_mode<LOGK, false>(x, M, mode, out, scales, s);
}

// ---------------------------------------------------------------- quantizer only

constexpr int kQThreads = 256;

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  v = red[0];
#pragma unroll
  for (int w = 1; w < kQThreads / 32; ++w) v = fmaxf(v, red[w]);
  return v;
}

__device__ __forceinline__ double block_sum_d(double v, double* red) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  v = red[0];
#pragma unroll
  for (int w = 1; w < kQThreads / 32; ++w) v += red[w];
  return v;
}

// One CTA per row; chunks of 8 elements.
__global__ void __launch_bounds__(kQThreads)
quant_rows_kernel(const float* __restrict__ t, int64_t K, int bits, int packed, uint8_t* __restrict__ codes,
                  float* __restrict__ scales) {
  __shared__ double red[kQThreads / 32];
  const int64_t row = blockIdx.x;
  const float* trow = t + (size_t)row * K;
  const int64_t nchunk = K / 8;
  q::RowParams p;
  if (bits == 4) {
    double a0 = 0.0, a1 = 0.0;
    for (int64_t c = threadIdx.x; c < nchunk; c += kQThreads) {
      float4 u = __ldg(reinterpret_cast<const float4*>(trow + c * 8));
      float4 v = __ldg(reinterpret_cast<const float4*>(trow + c * 8 + 4));
      a0 += q::abs_f64(u.x); a1 += q::abs_f64(u.y); a0 += q::abs_f64(u.z); a1 += q::abs_f64(u.w);
      a0 += q::abs_f64(v.x); a1 += q::abs_f64(v.y); a0 += q::abs_f64(v.z); a1 += q::abs_f64(v.w);
    }
    p = q::params_int4(block_sum_d(a0 + a1, red), K);
  } else {
    float g = 0.0f;
    for (int64_t c = threadIdx.x; c < nchunk; c += kQThreads) {
      float4 u = __ldg(reinterpret_cast<const float4*>(trow + c * 8));
      float4 v = __ldg(reinterpret_cast<const float4*>(trow + c * 8 + 4));
      g = fmaxf(g, fmaxf(fmaxf(fabsf(u.x), fabsf(u.y)), fmaxf(fabsf(u.z), fabsf(u.w))));
      g = fmaxf(g, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
    p = q::params_int8(block_max(g, reinterpret_cast<float*>(red)));
  }
  if (threadIdx.x == 0) scales[row] = p.scale();
  for (int64_t c = threadIdx.x; c < nchunk; c += kQThreads) {
    float4 u = __ldg(reinterpret_cast<const float4*>(trow + c * 8));
    float4 v = __ldg(reinterpret_cast<const float4*>(trow + c * 8 + 4));
    int n[8] = {q::rint_code(u.x, p.r), q::rint_code(u.y, p.r), q::rint_code(u.z, p.r), q::rint_code(u.w, p.r),
                q::rint_code(v.x, p.r), q::rint_code(v.y, p.r), q::rint_code(v.z, p.r), q::rint_code(v.w, p.r)};
    if (bits == 4 && packed) {
      reinterpret_cast<uint32_t*>(codes + (size_t)row * (K / 2))[c] = q::pack_s4x8(n);
    } else {
      if (bits == 4) {
#pragma unroll
        for (int u8 = 0; u8 < 8; ++u8) n[u8] = q::clip_int4(n[u8]);
      }
      uint2 w = make_uint2(q::pack_s8x4(n[0], n[1], n[2], n[3]), q::pack_s8x4(n[4], n[5], n[6], n[7]));
      reinterpret_cast<uint2*>(codes + (size_t)row * K)[c] = w;
    }
  }
}

}  // namespace

cudaError_t launch_ln_fht_quant(const void* x, bool in_bf16, int64_t M, int log2k, K1Mode mode, void* out,
                                float* scales, cudaStream_t stream) {
  // A few rows (decode-sized batches) go to the register kernel: the
  // tensor-core kernel's setup (TMEM, barriers, the Hadamard operand) and one
  // CTA's TMA/MMA round trips cost ~1 us more than the whole register kernel.
  if (M > kRegisterKernelMaxRows && ln_fht_quant_tc_supports(in_bf16, log2k, mode, x, out))
    return launch_ln_fht_quant_tc(x, M, log2k, mode, out, scales, stream);
  switch (log2k) {
    case 6: return launch_k<6>(x, in_bf16, M, mode, out, scales, stream);
    case 7: return launch_k<7>(x, in_bf16, M, mode, out, scales, stream);
    case 8: return launch_k<8>(x, in_bf16, M, mode, out, scales, stream);
    case 9: return launch_k<9>(x, in_bf16, M, mode, out, scales, stream);
    case 10: return launch_k<10>(x, in_bf16, M, mode, out, scales, stream);
    case 11: return launch_k<11>(x, in_bf16, M, mode, out, scales, stream);
    case 12: return launch_k<12>(x, in_bf16, M, mode, out, scales, stream);
    case 13: return launch_k<13>(x, in_bf16, M, mode, out, scales, stream);
    case 14: return launch_k<14>(x, in_bf16, M, mode, out, scales, stream);
    case 15: return launch_k<15>(x, in_bf16, M, mode, out, scales, stream);
  }
  return cudaErrorInvalidValue;
}

namespace {
template <int LOGK>
cudaError_t launch_lnbwd_k(const float* g, const void* x, bool x_bf16, int64_t M, void* gx, cudaStream_t s) {
  return x_bf16 ? launch_one<LOGK, true, K1_LNBWD>(g, M, gx, nullptr, s, x)
                : launch_one<LOGK, false, K1_LNBWD>(g, M, gx, nullptr, s, x);
}
}  // namespace

cudaError_t launch_fht_ln_backward(const float* g, const void* x, bool x_bf16, int64_t M, int log2k, void* gx,
                                   cudaStream_t stream) {
  if (M <= 0) return cudaSuccess;
  switch (log2k) {
    case 6: return launch_lnbwd_k<6>(g, x, x_bf16, M, gx, stream);
    case 7: return launch_lnbwd_k<7>(g, x, x_bf16, M, gx, stream);
    case 8: return launch_lnbwd_k<8>(g, x, x_bf16, M, gx, stream);
    case 9: return launch_lnbwd_k<9>(g, x, x_bf16, M, gx, stream);
    case 10: return launch_lnbwd_k<10>(g, x, x_bf16, M, gx, stream);
    case 11: return launch_lnbwd_k<11>(g, x, x_bf16, M, gx, stream);
    case 12: return launch_lnbwd_k<12>(g, x, x_bf16, M, gx, stream);
    case 13: return launch_lnbwd_k<13>(g, x, x_bf16, M, gx, stream);
    case 14: return launch_lnbwd_k<14>(g, x, x_bf16, M, gx, stream);
    case 15: return launch_lnbwd_k<15>(g, x, x_bf16, M, gx, stream);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_quant_from_f32(const float* t, int64_t M, int64_t K, int bits, bool packed, uint8_t* codes,
                                  float* scales, cudaStream_t stream) {
  quant_rows_kernel<<<(unsigned)M, kQThreads, 0, stream>>>(t, K, bits, packed ? 1 : 0, codes, scales);
  return cudaGetLastError();
}

}  // namespace hbl
