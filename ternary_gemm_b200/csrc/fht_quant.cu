// Fused LayerNorm -> fast Walsh-Hadamard transform -> per-token quantization
// (the activation path of H-BitLinear in "BitNet v2: Native 4-bit
// Activations with Hadamard Transformation for 1-bit LLMs", section
// "H-BitLinear": the Hadamard-transform definition, computed with the fast
// Hadamard transform in O(n log n), and the activation-quantization formula).
//
// One row of K = 2^k elements is spread over T = K/64 threads holding 64
// floats each in registers; R rows share a CTA so that a CTA has >= 128
// threads.  The Sylvester transform is the product of one 2-point butterfly
// per index bit, and those factors commute, so the k butterfly stages may run
// in any order.  Three passes cover all bits with two trips through shared
// memory:
//   pass 1: coalesced 16-byte loads give each thread index bits {0,1,2} (within
//           a 16-byte vector) and the top three bits {k-3,k-2,k-1} (eight
//           vectors T*8 elements apart); those 6 stages run in registers.
//   pass 2: (k >= 10) each thread reads the 2^(k-9) elements spanning bits
//           {6..k-4} from shared memory and runs those stages.
//   pass 3: each thread reads 64 contiguous elements (bits 0..5) and runs the
//           stages of bits {3,4,5} not done yet; the row is then complete and
//           contiguous per thread, ready for the quantizer and 16-byte stores.
// Shared memory uses an XOR swizzle of index bits 5..8 into bits 2..4 that
// keeps the vector writes of pass 1, the scalar accesses of pass 2 and the
// vector reads of pass 3 free of bank conflicts.
//
// LayerNorm is folded around the transform: a row offset mu~ (the mean of the
// row's first 8 values, identical in every thread) is subtracted first so
// that large means do not cost precision, then Y = H (x - mu~).  Because row 0
// of H is all ones, Y_0 = K (mu - mu~) and sum_{i>=1} Y_i^2 = K^2 var, so
//   t_i = Y_i / sqrt(K (var + eps_ln))  for i >= 1,   t_0 = 0,
// which is exactly H LN(x) / sqrt(K) with the biased variance and no affine.
#include <cstdint>

#include "common.cuh"
#include "quant.cuh"

namespace hbl {
namespace {

template <int LOGK>
struct Shape {
  static constexpr int K = 1 << LOGK;
  static constexpr int E = 64;                          // elements per thread
  static constexpr int T = K / E;                       // threads per row
  static constexpr int R = T >= 128 ? 1 : 128 / T;      // rows per CTA
  static constexpr int THREADS = T * R;
  static constexpr int PAD = T < 32 ? 16 : 0;           // floats of padding per row
  static constexpr int STRIDE = K + PAD;                // floats per row in smem
  static constexpr int WPR = T > 32 ? T / 32 : 1;       // warps per row
  static constexpr size_t SMEM = (size_t)R * STRIDE * 4 + (size_t)R * WPR * 8;
};

__device__ __forceinline__ int swz(int i) {
  int f = ((((i >> 5) ^ (i >> 6)) & 1) << 2) | (((i >> 7) & 1) << 3) | (((i >> 8) & 1) << 4);
  return i ^ f;
}

// Butterfly over register-index bit B: (e[r], e[r + 2^B]) -> (sum, difference).
template <int B, int N>
__device__ __forceinline__ void stage(float (&e)[N]) {
#pragma unroll
  for (int r = 0; r < N; ++r) {
    if (!(r & (1 << B))) {
      float a = e[r], c = e[r | (1 << B)];
      e[r] = a + c;
      e[r | (1 << B)] = a - c;
    }
  }
}

// Row-wide all-reduce over the T threads of a row (deterministic order: every
// thread of the row ends with the identical value).
template <int T, int WPR>
struct RowReduce {
  template <typename V, typename Op>
  __device__ __forceinline__ static V run(V v, Op op, V* red, int rl, int t) {
    constexpr int W = T < 32 ? T : 32;
#pragma unroll
    for (int o = W / 2; o >= 1; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
    if constexpr (T > 32) {
      if ((t & 31) == 0) red[rl * WPR + (t >> 5)] = v;
      __syncthreads();
      v = red[rl * WPR];
#pragma unroll
      for (int w = 1; w < WPR; ++w) v = op(v, red[rl * WPR + w]);
      __syncthreads();
    }
    return v;
  }
};

struct AddF {
  __device__ __forceinline__ float operator()(float a, float b) const { return a + b; }
};
struct AddD {
  __device__ __forceinline__ double operator()(double a, double b) const { return a + b; }
};
struct MaxF {
  __device__ __forceinline__ float operator()(float a, float b) const { return fmaxf(a, b); }
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* o) {
  o[0] = __uint_as_float(u.x << 16);
  o[1] = __uint_as_float(u.x & 0xffff0000u);
  o[2] = __uint_as_float(u.y << 16);
  o[3] = __uint_as_float(u.y & 0xffff0000u);
  o[4] = __uint_as_float(u.z << 16);
  o[5] = __uint_as_float(u.z & 0xffff0000u);
  o[6] = __uint_as_float(u.w << 16);
  o[7] = __uint_as_float(u.w & 0xffff0000u);
}

// 8 consecutive input values starting at element `i` of the row.
template <bool BF16>
__device__ __forceinline__ void load8(const void* xrow, int i, float* o) {
  if constexpr (BF16) {
    uint4 u = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(xrow) + i));
    bf16x8_to_f32(u, o);
  } else {
    const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(xrow) + i);
    float4 a = __ldg(p), b = __ldg(p + 1);
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
    o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
  }
}

// Index bit j of the "other" bits of pass 2: {0,1,2,3,4,5,k-3,k-2,k-1}.
template <int LOGK>
__host__ __device__ constexpr int other_bit(int j) {
  return j < 6 ? j : LOGK - 9 + j;
}

template <int LOGK, bool BF16, int MODE>
__global__ void __launch_bounds__(Shape<LOGK>::THREADS, 1)
ln_fht_quant_kernel(const void* __restrict__ x, int64_t M, float sK, void* __restrict__ out,
                    float* __restrict__ scales) {
  using S = Shape<LOGK>;
  constexpr int K = S::K, T = S::T, R = S::R;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* smem = reinterpret_cast<float*>(smem_raw);
  void* red = smem_raw + (size_t)R * S::STRIDE * 4;

  const int tid = threadIdx.x;
  const int rl = tid / T;
  const int t = tid % T;
  const int64_t row = (int64_t)blockIdx.x * R + rl;
  const bool active = row < M;
  const size_t esz = BF16 ? 2 : 4;
  const void* xrow = reinterpret_cast<const unsigned char*>(x) + (size_t)(active ? row : 0) * K * esz;
  float* srow = smem + rl * S::STRIDE;

  float e[64];

  // ---- pass 1: load, remove the row offset, stages of bits {0,1,2,k-3,k-2,k-1}
  float mu = 0.0f;
  if (active) {
    float f[8];
    load8<BF16>(xrow, 0, f);
    mu = (((f[0] + f[1]) + (f[2] + f[3])) + ((f[4] + f[5]) + (f[6] + f[7]))) * 0.125f;
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) load8<BF16>(xrow, (jj * T + t) * 8, &e[jj * 8]);
  } else {
#pragma unroll
    for (int r = 0; r < 64; ++r) e[r] = 0.0f;
  }
#pragma unroll
  for (int r = 0; r < 64; ++r) e[r] = e[r] - mu;
  stage<0>(e); stage<1>(e); stage<2>(e); stage<3>(e); stage<4>(e); stage<5>(e);
#pragma unroll
  for (int jj = 0; jj < 8; ++jj) {
    int i0 = (jj * T + t) * 8;
    *reinterpret_cast<float4*>(srow + swz(i0)) = make_float4(e[jj * 8 + 0], e[jj * 8 + 1], e[jj * 8 + 2], e[jj * 8 + 3]);
    *reinterpret_cast<float4*>(srow + swz(i0 + 4)) = make_float4(e[jj * 8 + 4], e[jj * 8 + 5], e[jj * 8 + 6], e[jj * 8 + 7]);
  }
  __syncthreads();

  // ---- pass 2: stages of bits {6 .. k-4}
  if constexpr (LOGK >= 10) {
    constexpr int NPB = LOGK - 9;
    constexpr int NP = 1 << NPB;
    constexpr int G = 64 / NP;
    int tb = 0;
#pragma unroll
    for (int j = 0; j < LOGK - 6; ++j) tb |= ((t >> j) & 1) << other_bit<LOGK>(j);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      int gb = 0;
#pragma unroll
      for (int j = 0; j < 15 - LOGK; ++j) gb |= ((g >> j) & 1) << other_bit<LOGK>(LOGK - 6 + j);
#pragma unroll
      for (int p = 0; p < NP; ++p) e[g * NP + p] = srow[swz(tb | gb | (p << 6))];
    }
    if constexpr (NPB > 0) stage<0>(e);
    if constexpr (NPB > 1) stage<1>(e);
    if constexpr (NPB > 2) stage<2>(e);
    if constexpr (NPB > 3) stage<3>(e);
    if constexpr (NPB > 4) stage<4>(e);
    if constexpr (NPB > 5) stage<5>(e);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      int gb = 0;
#pragma unroll
      for (int j = 0; j < 15 - LOGK; ++j) gb |= ((g >> j) & 1) << other_bit<LOGK>(LOGK - 6 + j);
#pragma unroll
      for (int p = 0; p < NP; ++p) srow[swz(tb | gb | (p << 6))] = e[g * NP + p];
    }
    __syncthreads();
  }

  // ---- pass 3: 64 contiguous elements per thread, stages of bits {3,4,5} left
  const int base = t * 64;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    float4 v = *reinterpret_cast<const float4*>(srow + swz(base + 4 * j));
    e[4 * j + 0] = v.x; e[4 * j + 1] = v.y; e[4 * j + 2] = v.z; e[4 * j + 3] = v.w;
  }
  if constexpr (3 < LOGK - 3) stage<3>(e);
  if constexpr (4 < LOGK - 3) stage<4>(e);
  if constexpr (5 < LOGK - 3) stage<5>(e);

  // ---- LayerNorm statistics from the transform: K^2 var = sum_{i>=1} Y_i^2
  float ss = 0.0f;
#pragma unroll
  for (int r = 1; r < 64; ++r) ss = fmaf(e[r], e[r], ss);
  if (t != 0) ss = fmaf(e[0], e[0], ss);
  ss = RowReduce<T, S::WPR>::run(ss, AddF(), reinterpret_cast<float*>(red), rl, t);
  const float var = ss * (1.0f / ((float)K * (float)K));
  const float cmul = __fmul_rn(__fdiv_rn(1.0f, sqrtf(__fadd_rn(var, 1e-5f))), sK);
#pragma unroll
  for (int r = 0; r < 64; ++r) e[r] = __fmul_rn(e[r], cmul);
  if (t == 0) e[0] = 0.0f;

  if constexpr (MODE == K1_T_F32) {
    if (active) {
      float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + (size_t)row * K + base);
#pragma unroll
      for (int j = 0; j < 16; ++j) dst[j] = make_float4(e[4 * j], e[4 * j + 1], e[4 * j + 2], e[4 * j + 3]);
    }
    return;
  } else {
    q::RowParams p;
    if constexpr (MODE == K1_Q8_I8) {
      float g = 0.0f;
#pragma unroll
      for (int r = 0; r < 64; ++r) g = fmaxf(g, fabsf(e[r]));
      g = RowReduce<T, S::WPR>::run(g, MaxF(), reinterpret_cast<float*>(red), rl, t);
      p = q::params_int8(g);
    } else {
      double a0 = 0.0, a1 = 0.0;
#pragma unroll
      for (int r = 0; r < 64; r += 2) {
        a0 += q::abs_f64(e[r]);
        a1 += q::abs_f64(e[r + 1]);
      }
      double a = RowReduce<T, S::WPR>::run(a0 + a1, AddD(), reinterpret_cast<double*>(red), rl, t);
      p = q::params_int4(a, K);
    }
    if (!active) return;
    if (t == 0) scales[row] = p.scale;
    if constexpr (MODE == K1_Q4_PACKED) {
      uint32_t w[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        int n[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) n[u] = q::rint_code(e[8 * j + u], p.r);
        w[j] = q::pack_s4x8(n);
      }
      uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(out) + (size_t)row * (K / 2) + base / 2);
      dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
      dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    } else {
      uint32_t w[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        int n0 = q::rint_code(e[4 * j + 0], p.r), n1 = q::rint_code(e[4 * j + 1], p.r);
        int n2 = q::rint_code(e[4 * j + 2], p.r), n3 = q::rint_code(e[4 * j + 3], p.r);
        if constexpr (MODE == K1_Q4_I8) {
          n0 = q::clip_int4(n0); n1 = q::clip_int4(n1); n2 = q::clip_int4(n2); n3 = q::clip_int4(n3);
        }
        w[j] = q::pack_s8x4(n0, n1, n2, n3);
      }
      uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(out) + (size_t)row * K + base);
#pragma unroll
      for (int j = 0; j < 4; ++j) dst[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
    }
  }
}

template <int LOGK, bool BF16, int MODE>
cudaError_t launch_one(const void* x, int64_t M, void* out, float* scales, cudaStream_t stream) {
  using S = Shape<LOGK>;
  auto kern = ln_fht_quant_kernel<LOGK, BF16, MODE>;
  static cudaError_t attr = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)S::SMEM);
  if (attr != cudaSuccess) return attr;
  const int64_t grid = (M + S::R - 1) / S::R;
  const float sK = (float)(1.0 / sqrt((double)S::K));
  kern<<<(unsigned)grid, S::THREADS, S::SMEM, stream>>>(x, M, sK, out, scales);
  return cudaGetLastError();
}

template <int LOGK, bool BF16>
cudaError_t launch_mode(const void* x, int64_t M, K1Mode mode, void* out, float* scales, cudaStream_t s) {
  switch (mode) {
    case K1_T_F32: return launch_one<LOGK, BF16, K1_T_F32>(x, M, out, scales, s);
    case K1_Q4_PACKED: return launch_one<LOGK, BF16, K1_Q4_PACKED>(x, M, out, scales, s);
    case K1_Q4_I8: return launch_one<LOGK, BF16, K1_Q4_I8>(x, M, out, scales, s);
    case K1_Q8_I8: return launch_one<LOGK, BF16, K1_Q8_I8>(x, M, out, scales, s);
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
  if (threadIdx.x == 0) scales[row] = p.scale;
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

cudaError_t launch_quant_from_f32(const float* t, int64_t M, int64_t K, int bits, bool packed, uint8_t* codes,
                                  float* scales, cudaStream_t stream) {
  quant_rows_kernel<<<(unsigned)M, kQThreads, 0, stream>>>(t, K, bits, packed ? 1 : 0, codes, scales);
  return cudaGetLastError();
}

}  // namespace hbl
