// Ternary weight quantization ("BitNet v2: Native 4-bit Activations with
// Hadamard Transformation for 1-bit LLMs", section "H-BitLinear",
// weight-quantization formula: per-tensor absmean to {-1, 0, 1}):
//   alpha = mean |W|,  w = clip(rint(W / (alpha + eps)), -1, 1).
// alpha is accumulated in double and rounded once to float; the codes use one
// float reciprocal r = 1/(alpha+eps) and rint of the exact product W r.
//
// Kernel 1 writes kTernaryPartials double partial sums (fixed grid, fixed
// per-thread order, fixed tree).  Kernel 2 has every CTA reduce the same
// partials in the same order -- so every CTA holds the identical alpha --
// then packs 16 codes per 32-bit word (2 bits each: 00 = 0, 01 = +1, 11 = -1,
// element 4j+i of a row at bits 2i..2i+1 of byte j).  Both are HBM-bound
// streaming kernels with 16-byte loads.
#include <cstdint>

#include "common.cuh"
#include "quant.cuh"
#include "ternary.cuh"

namespace hbl {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ double block_sum(double v, double* red) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  v = red[0];
#pragma unroll
  for (int w = 1; w < kThreads / 32; ++w) v += red[w];
  __syncthreads();
  return v;
}

// 8 weights per 16-byte chunk (bf16) or 4 (fp32).
template <bool BF16>
__global__ void __launch_bounds__(kThreads)
abs_partials_kernel(const void* __restrict__ W, int64_t nchunks, double* __restrict__ partials) {
  __shared__ double red[kThreads / 32];
  const uint4* src = reinterpret_cast<const uint4*>(W);
  double a0 = 0.0, a1 = 0.0;
  for (int64_t c = (int64_t)blockIdx.x * kThreads + threadIdx.x; c < nchunks; c += (int64_t)gridDim.x * kThreads) {
    uint4 u = __ldg(src + c);
    if constexpr (BF16) {
      a0 += fabs((double)__uint_as_float(u.x << 16)); a1 += fabs((double)__uint_as_float(u.x & 0xffff0000u));
      a0 += fabs((double)__uint_as_float(u.y << 16)); a1 += fabs((double)__uint_as_float(u.y & 0xffff0000u));
      a0 += fabs((double)__uint_as_float(u.z << 16)); a1 += fabs((double)__uint_as_float(u.z & 0xffff0000u));
      a0 += fabs((double)__uint_as_float(u.w << 16)); a1 += fabs((double)__uint_as_float(u.w & 0xffff0000u));
    } else {
      a0 += fabs((double)__uint_as_float(u.x)); a1 += fabs((double)__uint_as_float(u.y));
      a0 += fabs((double)__uint_as_float(u.z)); a1 += fabs((double)__uint_as_float(u.w));
    }
  }
  double s = block_sum(a0 + a1, red);
  if (threadIdx.x == 0) partials[blockIdx.x] = s;
}

__device__ __forceinline__ uint32_t ternary_field(float w, float r) {
  // rint of the exact product w * r, clipped to [-1, 1].  Where |w r| >= 2 the
  // code is the sign; below, the fused multiply-add rounds exactly (see
  // q::rint_code) and only |w r| < 2^22 reaches it.
  int n = __float_as_int(__fmaf_rn(w, r, q::kMagic)) - q::kMagicBits;
  const float p = __fmul_rn(w, r);
  n = fabsf(p) >= 2.0f ? (p > 0.0f ? 1 : -1) : max(-1, min(1, n));
  return (uint32_t)n & 3u;  // 0 -> 00, 1 -> 01, -1 -> 11
}

// Each thread: 16 consecutive weights -> one 32-bit word.
template <bool BF16>
__global__ void __launch_bounds__(kThreads)
pack_kernel(const void* __restrict__ W, int64_t nwords, int64_t count, const double* __restrict__ partials,
            uint32_t* __restrict__ packed, float* __restrict__ alpha_out) {
  __shared__ double red[kThreads / 32];
  double s = 0.0;
  for (int i = threadIdx.x; i < kTernaryPartials; i += kThreads) s += partials[i];
  s = block_sum(s, red);
  const float alpha = (float)(s / (double)count);
  if (blockIdx.x == 0 && threadIdx.x == 0) *alpha_out = alpha;
  const float r = __fdiv_rn(1.0f, __fadd_rn(alpha, q::kEps));
  for (int64_t wi = (int64_t)blockIdx.x * kThreads + threadIdx.x; wi < nwords; wi += (int64_t)gridDim.x * kThreads) {
    float f[16];
    if constexpr (BF16) {
      const uint4* src = reinterpret_cast<const uint4*>(W) + wi * 2;
      uint4 u0 = __ldg(src), u1 = __ldg(src + 1);
      const uint32_t v[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        f[2 * j] = __uint_as_float(v[j] << 16);
        f[2 * j + 1] = __uint_as_float(v[j] & 0xffff0000u);
      }
    } else {
      const float4* src = reinterpret_cast<const float4*>(W) + wi * 4;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float4 a = __ldg(src + j);
        f[4 * j] = a.x; f[4 * j + 1] = a.y; f[4 * j + 2] = a.z; f[4 * j + 3] = a.w;
      }
    }
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) word |= ternary_field(f[j], r) << (2 * j);
    packed[wi] = word;
  }
}

// One word (16 codes -> 16 bytes) per thread and iteration: consecutive
// threads take consecutive words, so every store instruction of a warp writes
// 512 contiguous bytes.
__global__ void __launch_bounds__(kThreads)
widen_kernel(const uint32_t* __restrict__ packed, int64_t nwords, uint4* __restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < nwords; i += (int64_t)gridDim.x * kThreads)
    out[i] = tern::widen16(__ldg(packed + i));
  // Launched as a programmatic dependent of the quantizer kernel (it reads
  // nothing that kernel writes, so it runs alongside it): finishing only
  // after that kernel has finished lets the next kernel of the stream rely on
  // both.  A no-op for an ordinary launch.
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

int grid_for(int64_t work) {
  int64_t g = (work + kThreads - 1) / kThreads;
  return (int)(g < 148 * 16 ? (g < 1 ? 1 : g) : 148 * 16);
}

}  // namespace

cudaError_t launch_pack_ternary(const void* W, bool in_bf16, int64_t N, int64_t K, uint8_t* packed, float* alpha,
                                double* partials, cudaStream_t stream) {
  const int64_t count = N * K;
  const int64_t nchunks = in_bf16 ? count / 8 : count / 4;
  if (in_bf16)
    abs_partials_kernel<true><<<kTernaryPartials, kThreads, 0, stream>>>(W, nchunks, partials);
  else
    abs_partials_kernel<false><<<kTernaryPartials, kThreads, 0, stream>>>(W, nchunks, partials);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t nwords = count / 16;
  if (in_bf16)
    pack_kernel<true><<<grid_for(nwords), kThreads, 0, stream>>>(W, nwords, count, partials,
                                                                 reinterpret_cast<uint32_t*>(packed), alpha);
  else
    pack_kernel<false><<<grid_for(nwords), kThreads, 0, stream>>>(W, nwords, count, partials,
                                                                  reinterpret_cast<uint32_t*>(packed), alpha);
  return cudaGetLastError();
}

cudaError_t launch_widen_ternary(const uint8_t* packed, int64_t N, int64_t K, int8_t* out, cudaStream_t stream,
                                 bool overlap_previous) {
  const int64_t nwords = N * K / 16;  // N K is a multiple of 1024 (K >= 64, N % 16 == 0)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid_for(nwords), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = overlap_previous ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, widen_kernel, reinterpret_cast<const uint32_t*>(packed), nwords,
                            reinterpret_cast<uint4*>(out));
}

}  // namespace hbl
