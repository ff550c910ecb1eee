// Per-row building blocks shared by the row kernels (the fused transform +
// quantize kernel and the normalise + quantize kernel): paired float
// operations, row-wide all-reduce over the threads of a row, and 16-byte
// loads of 8 bf16 or float values.
#pragma once

#include <cstdint>

#include "quant.cuh"

namespace hbl {
namespace rowkit {

// ---------------------------------------------------------------- paired float ops

__device__ __forceinline__ void bfly2(float& a0, float& a1, float& b0, float& b1) {
  asm("{\n\t.reg .b64 A, B, S, D;\n\t"
      "mov.b64 A, {%0, %1};\n\tmov.b64 B, {%2, %3};\n\t"
      "add.rn.f32x2 S, A, B;\n\tsub.rn.f32x2 D, A, B;\n\t"
      "mov.b64 {%0, %1}, S;\n\tmov.b64 {%2, %3}, D;\n\t}"
      : "+f"(a0), "+f"(a1), "+f"(b0), "+f"(b1));
}

__device__ __forceinline__ void sub2(float& a0, float& a1, float c) {
  asm("{\n\t.reg .b64 A, C;\n\t"
      "mov.b64 A, {%0, %1};\n\tmov.b64 C, {%2, %2};\n\t"
      "sub.rn.f32x2 A, A, C;\n\tmov.b64 {%0, %1}, A;\n\t}"
      : "+f"(a0), "+f"(a1) : "f"(c));
}

__device__ __forceinline__ void mul2(float& a0, float& a1, float c) {
  asm("{\n\t.reg .b64 A, C;\n\t"
      "mov.b64 A, {%0, %1};\n\tmov.b64 C, {%2, %2};\n\t"
      "mul.rn.f32x2 A, A, C;\n\tmov.b64 {%0, %1}, A;\n\t}"
      : "+f"(a0), "+f"(a1) : "f"(c));
}

// (s0, s1) += (a0*a0, a1*a1)
__device__ __forceinline__ void sq_acc2(float& s0, float& s1, float a0, float a1) {
  asm("{\n\t.reg .b64 A, S;\n\t"
      "mov.b64 A, {%2, %3};\n\tmov.b64 S, {%0, %1};\n\t"
      "fma.rn.f32x2 S, A, A, S;\n\tmov.b64 {%0, %1}, S;\n\t}"
      : "+f"(s0), "+f"(s1) : "f"(a0), "f"(a1));
}

// bits of fl(t * r + 1.5*2^23) for a pair, one rounding each (see q::rint_code)
__device__ __forceinline__ void magic2(float t0, float t1, float r, uint32_t& m0, uint32_t& m1) {
  asm("{\n\t.reg .b64 A, R, M;\n\t"
      "mov.b64 A, {%2, %3};\n\tmov.b64 R, {%4, %4};\n\tmov.b64 M, {%5, %5};\n\t"
      "fma.rn.f32x2 A, A, R, M;\n\t"
      "mov.b64 {%0, %1}, A;\n\t}"
      : "=r"(m0), "=r"(m1) : "f"(t0), "f"(t1), "f"(r), "f"(q::kMagic));
}

// Row-wide all-reduce over the T threads of a row (deterministic order: every
// thread of the row ends with the identical value).  `red` must not be reused
// by the CTA afterwards (each reduction has its own slot).
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

}  // namespace rowkit
}  // namespace hbl
