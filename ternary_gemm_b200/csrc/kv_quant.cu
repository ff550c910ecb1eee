// Low-bit QKV-state quantizer of the low-bit attention experiments ("BitNet
// v2: Native 4-bit Activations with Hadamard Transformation for 1-bit LLMs";
// QbitAI report / Xinzhiyuan article, low-bit attention: after RoPE, the QKV
// heads are quantized directly to unsigned integers by the absmax function,
// with no calibration data; a 3-bit KV cache matches full precision).
// Per head vector of D values (one token, one head):
//
//   gamma = max |x|,   L = 2^b - 1,   r = L / (2 (gamma + eps))   (IEEE division)
//   q     = clip(rint(fl(fl(x r) + L/2)), 0, L)                   (unsigned, one byte)
//   scale = gamma                                                  (x ~ (2 q - L) gamma / L)
//
// i.e. [-gamma, gamma] mapped linearly onto the 2^b levels.  One warp per head
// vector: each lane holds D/32 consecutive values, the absmax is one
// redux.sync over the bit patterns of |x| (non-negative floats order like
// their bits), and each lane stores its D/32 codes (a warp writes D
// contiguous bytes).  A warp takes four consecutive head vectors per step and
// issues their loads together.  Memory-bound: 2 (bf16) or 4 bytes in, 1 byte out per
// value, 4 bytes per head.
#include <cstdint>

#include "common.cuh"
#include "sm100.cuh"

namespace hbl {
namespace {

constexpr int kKvThreads = 256;
constexpr int kKvWarps = kKvThreads / 32;
constexpr int kKvRows = 4;  // head vectors per warp and step

template <int V, bool BF16>
__device__ __forceinline__ void load_v(const void* x, int64_t idx, float (&v)[V]) {
  if constexpr (BF16) {
    const uint16_t* p = reinterpret_cast<const uint16_t*>(x) + idx;
    if constexpr (V == 8) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      }
    } else if constexpr (V == 4) {
      const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
      v[0] = __uint_as_float(u.x << 16);
      v[1] = __uint_as_float(u.x & 0xFFFF0000u);
      v[2] = __uint_as_float(u.y << 16);
      v[3] = __uint_as_float(u.y & 0xFFFF0000u);
    } else if constexpr (V == 2) {
      const uint32_t u = __ldg(reinterpret_cast<const uint32_t*>(p));
      v[0] = __uint_as_float(u << 16);
      v[1] = __uint_as_float(u & 0xFFFF0000u);
    } else {
      v[0] = __uint_as_float((uint32_t)__ldg(p) << 16);
    }
  } else {
    const float* p = reinterpret_cast<const float*>(x) + idx;
    if constexpr (V >= 4) {
#pragma unroll
      for (int i = 0; i < V; i += 4) {
        const float4 f = __ldg(reinterpret_cast<const float4*>(p + i));
        v[i] = f.x;
        v[i + 1] = f.y;
        v[i + 2] = f.z;
        v[i + 3] = f.w;
      }
    } else if constexpr (V == 2) {
      const float2 f = __ldg(reinterpret_cast<const float2*>(p));
      v[0] = f.x;
      v[1] = f.y;
    } else {
      v[0] = __ldg(p);
    }
  }
}

template <int V>
__device__ __forceinline__ void store_codes(uint8_t* dst, const uint32_t (&q)[V]) {
  if constexpr (V == 8) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(q[0] | (q[1] << 8) | (q[2] << 16) | (q[3] << 24),
                                                q[4] | (q[5] << 8) | (q[6] << 16) | (q[7] << 24));
  } else if constexpr (V == 4) {
    *reinterpret_cast<uint32_t*>(dst) = q[0] | (q[1] << 8) | (q[2] << 16) | (q[3] << 24);
  } else if constexpr (V == 2) {
    *reinterpret_cast<uint16_t*>(dst) = (uint16_t)(q[0] | (q[1] << 8));
  } else {
    *dst = (uint8_t)q[0];
  }
}

template <int V, bool BF16>
__global__ void __launch_bounds__(kKvThreads)
kv_quant_kernel(const void* __restrict__ x, int64_t rows, int bits, uint8_t* __restrict__ codes,
                float* __restrict__ scales) {
  constexpr int D = 32 * V;
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * kKvWarps;
  const float L = (float)((1 << bits) - 1);
  const float half = 0.5f * L;
  // kKvRows consecutive head vectors per warp and step, all loaded before any
  // is reduced, so that each warp keeps several loads in flight
  for (int64_t row0 = ((int64_t)blockIdx.x * kKvWarps + (threadIdx.x >> 5)) * kKvRows; row0 < rows;
       row0 += warps * kKvRows) {
    float v[kKvRows][V];
#pragma unroll
    for (int k = 0; k < kKvRows; ++k)
      if (row0 + k < rows) load_v<V, BF16>(x, (row0 + k) * D + lane * V, v[k]);
#pragma unroll
    for (int k = 0; k < kKvRows; ++k) {
      const int64_t row = row0 + k;
      if (row >= rows) break;  // warp-uniform
      float a = 0.0f;
#pragma unroll
      for (int i = 0; i < V; ++i) a = fmaxf(a, fabsf(v[k][i]));
      const float gamma = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(a)));
      const float r = __fdiv_rn(L, __fmul_rn(2.0f, __fadd_rn(gamma, 1e-5f)));
      uint32_t q[V];
#pragma unroll
      for (int i = 0; i < V; ++i) {
        const int c = __float2int_rn(__fadd_rn(__fmul_rn(v[k][i], r), half));
        q[i] = (uint32_t)min(max(c, 0), (int)L);
      }
      store_codes<V>(codes + row * D + lane * V, q);
      if (lane == 0) scales[row] = gamma;
    }
  }
}

template <int V>
cudaError_t launch_v(const void* x, bool bf16, int64_t rows, int bits, uint8_t* codes, float* scales,
                     cudaStream_t stream) {
  const int64_t need = (rows + kKvWarps * kKvRows - 1) / (kKvWarps * kKvRows);
  const int64_t cap = (int64_t)sm100_host::sm_count() * 32;
  const unsigned grid = (unsigned)(need < cap ? need : cap);
  if (bf16)
    kv_quant_kernel<V, true><<<grid, kKvThreads, 0, stream>>>(x, rows, bits, codes, scales);
  else
    kv_quant_kernel<V, false><<<grid, kKvThreads, 0, stream>>>(x, rows, bits, codes, scales);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_kv_quant(const void* x, bool bf16, int64_t rows, int64_t D, int bits, uint8_t* codes,
                            float* scales, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  switch (D) {
    case 32: return launch_v<1>(x, bf16, rows, bits, codes, scales, stream);
    case 64: return launch_v<2>(x, bf16, rows, bits, codes, scales, stream);
    case 128: return launch_v<4>(x, bf16, rows, bits, codes, scales, stream);
    case 256: return launch_v<8>(x, bf16, rows, bits, codes, scales, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace hbl
