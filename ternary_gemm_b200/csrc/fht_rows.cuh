// The register-resident row transform shared by the fused LayerNorm ->
// Hadamard -> quantize kernel (fht_quant.cu) and the fused decode-sized
// forward (gemv_ternary.cu): the activation path of H-BitLinear in "BitNet v2:
// Native 4-bit Activations with Hadamard Transformation for 1-bit LLMs",
// section "H-BitLinear" (LayerNorm, the Hadamard transform computed with the
// fast transform, the per-token activation quantizers).
//
// A row of K = 2^k floats lives in the registers of T = K/64 threads (64
// floats each) and reaches its Sylvester transform in three passes with two
// trips through shared memory (fht_quant.cu describes the passes, the swizzle
// and the LayerNorm folding).  Every function here is a pure function of the
// row: the same row gives bit-identical t, scale and codes in any kernel and
// for any number of rows per CTA, because the per-row arithmetic and the
// reduction order over the row's T threads do not depend on R.
#pragma once

#include <cstdint>

#include "common.cuh"
#include "quant.cuh"
#include "rowkit.cuh"

namespace hbl {
namespace fhtrows {

using namespace rowkit;

// Rows of K = 2^LOGK floats, T = K/64 threads per row, R rows per CTA.
template <int LOGK, int RR>
struct ShapeR {
  static constexpr int LOG = LOGK;
  static constexpr int K = 1 << LOGK;
  static constexpr int E = 64;                          // elements per thread
  static constexpr int T = K / E;                       // threads per row
  static constexpr int R = RR;                          // rows per CTA
  static constexpr int THREADS = T * R;
  // CTAs per SM the register budget is tuned for: 512 threads -> 128 regs,
  // 256 -> 80 regs (3 CTAs), 128 -> 96 regs (5 CTAs)
  static constexpr int MINB = THREADS >= 512 ? 1 : (THREADS >= 256 ? 3 : 5);
  static constexpr int PAD = T < 32 ? 16 : 0;           // floats of padding per row
  static constexpr int STRIDE = K + PAD;                // floats per row in smem
  static constexpr int WPR = T > 32 ? T / 32 : 1;       // warps per row
  static constexpr size_t XCH = (size_t)R * STRIDE * 4;   // exchange buffer (floats)
  static constexpr size_t RED = (size_t)R * WPR * 8;       // one row-reduction scratch
  static constexpr size_t SMEM = XCH + 2 * RED;            // two reductions, separate slots
  static constexpr int NPB = LOGK >= 10 ? LOGK - 9 : 0;  // pass-2 processed bits {6 .. 5+NPB}
  static constexpr int PB = 6 - NPB;                      // pass-2 vector bits {0 .. PB-1}
  static_assert(NPB >= 0 && NPB <= 6 && PB >= 0 && PB <= 6, "pass-2 split");
};

// The transform kernel's own shape: CTAs of at least 128 threads.
template <int LOGK>
using Shape = ShapeR<LOGK, ((1 << LOGK) / 64 >= 128 ? 1 : 128 / ((1 << LOGK) / 64))>;

// The swizzle: index bits 5..8 XORed into bits 2..4 (linear over GF(2)).
__host__ __device__ constexpr int swz(int i) {
  return i ^ (((((i >> 5) ^ (i >> 6)) & 1) << 2) | (((i >> 7) & 1) << 3) | (((i >> 8) & 1) << 4));
}

// Shared-memory addresses of index (tb | C) for a per-thread tb and a
// compile-time C with disjoint bits: swz(tb | C) = swz(tb) ^ swz(C); the XOR
// part of swz(C) falls in bits 2..4 and selects one of eight bases, the rest
// is an immediate offset.
struct SwzBase {
  int b[8];
  __device__ __forceinline__ SwzBase(int row_off, int tb) {
    const int s = swz(tb);
#pragma unroll
    for (int v = 0; v < 8; ++v) b[v] = row_off + (s ^ (v << 2));
  }
  template <int C>
  __device__ __forceinline__ int at() const {
    constexpr int sc = swz(C);
    return b[(sc >> 2) & 7] + (sc & ~0x1C);
  }
};

// Butterfly over register-index bit B: (e[r], e[r + 2^B]) -> (sum, difference).
template <int B, int N>
__device__ __forceinline__ void stage(float (&e)[N]) {
  if constexpr (B == 0) {
#pragma unroll
    for (int r = 0; r < N; r += 2) {
      float a = e[r], c = e[r + 1];
      e[r] = a + c;
      e[r + 1] = a - c;
    }
  } else {
#pragma unroll
    for (int r = 0; r < N; r += 2)
      if (!(r & (1 << B))) bfly2(e[r], e[r + 1], e[r | (1 << B)], e[(r | (1 << B)) + 1]);
  }
}

template <int N>
__device__ __forceinline__ void stage_range(float (&e)[N], int lo, int hi) {
  // register bits lo..hi-1 (lo, hi compile-time after inlining)
  if (lo <= 0 && 0 < hi) stage<0>(e);
  if (lo <= 1 && 1 < hi) stage<1>(e);
  if (lo <= 2 && 2 < hi) stage<2>(e);
  if (lo <= 3 && 3 < hi) stage<3>(e);
  if (lo <= 4 && 4 < hi) stage<4>(e);
  if (lo <= 5 && 5 < hi) stage<5>(e);
}

// Thread bit j of pass 2 -> index bit: {PB .. 5} then {k-3, k-2, k-1}.
template <int LOGK>
__host__ __device__ constexpr int p2_bit(int j) {
  return j < 6 - Shape<LOGK>::PB ? Shape<LOGK>::PB + j : LOGK - 3 + (j - (6 - Shape<LOGK>::PB));
}

// 4 floats (or fewer, for vectors narrower than 16 bytes) at a smem address.
template <int W>
__device__ __forceinline__ void lds(const float* s, int a, float* o) {
  if constexpr (W == 4) {
    float4 v = *reinterpret_cast<const float4*>(s + a);
    o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
  } else if constexpr (W == 2) {
    float2 v = *reinterpret_cast<const float2*>(s + a);
    o[0] = v.x; o[1] = v.y;
  } else {
    o[0] = s[a];
  }
}

template <int W>
__device__ __forceinline__ void sts(float* s, int a, const float* o) {
  if constexpr (W == 4) {
    *reinterpret_cast<float4*>(s + a) = make_float4(o[0], o[1], o[2], o[3]);
  } else if constexpr (W == 2) {
    *reinterpret_cast<float2*>(s + a) = make_float2(o[0], o[1]);
  } else {
    s[a] = o[0];
  }
}

template <int LOGK, int R0, int NREG>
struct Pass2 {
  // registers r = p * 2^PB + v  <->  index tb | (p << 6) | v; chunks of W floats
  static constexpr int PB = Shape<LOGK>::PB;
  static constexpr int W = PB >= 2 ? 4 : (PB == 1 ? 2 : 1);
  template <int R>
  __device__ __forceinline__ static void load(float (&e)[64], const float* smem, const SwzBase& sb) {
    if constexpr (R < 64) {
      constexpr int p = R >> PB, v = R & ((1 << PB) - 1);
      lds<W>(smem, sb.at<(p << 6) | v>(), &e[R]);
      load<R + W>(e, smem, sb);
    }
  }
  template <int R>
  __device__ __forceinline__ static void store(const float (&e)[64], float* smem, const SwzBase& sb) {
    if constexpr (R < 64) {
      constexpr int p = R >> PB, v = R & ((1 << PB) - 1);
      sts<W>(smem, sb.at<(p << 6) | v>(), &e[R]);
      store<R + W>(e, smem, sb);
    }
  }
};

template <int J>
__device__ __forceinline__ void load_pass3(float (&e)[64], const float* smem, const SwzBase& sb) {
  if constexpr (J < 16) {
    lds<4>(smem, sb.at<4 * J>(), &e[4 * J]);
    load_pass3<J + 1>(e, smem, sb);
  }
}

template <int JJ, int T>
__device__ __forceinline__ void store_pass1(const float (&e)[64], float* smem, const SwzBase& sb) {
  if constexpr (JJ < 8) {
    sts<4>(smem, sb.at<JJ * T * 8>(), &e[JJ * 8]);
    sts<4>(smem, sb.at<JJ * T * 8 + 4>(), &e[JJ * 8 + 4]);
    store_pass1<JJ + 1, T>(e, smem, sb);
  }
}

// Barrier policies for the row functions: the whole CTA, or the first N
// threads of it on a named barrier (for kernels with other warps beside the
// transform).
struct BarCta {
  __device__ __forceinline__ static void sync() { __syncthreads(); }
};
template <int ID, int N>
struct BarNamed {
  __device__ __forceinline__ static void sync() { asm volatile("bar.sync %0, %1;" ::"n"(ID), "n"(N) : "memory"); }
};

// RowReduce with a warp-uniform `compute`: warps that hold no row of
// interest skip the shuffles and the slots but still meet the barrier.
// With compute true it is RowReduce, operation for operation.
template <int T, int WPR, class Bar, typename V, typename Op>
__device__ __forceinline__ V row_reduce(V v, Op op, V* red, int rl, int t, bool compute) {
  constexpr int W = T < 32 ? T : 32;
  if (compute) {
#pragma unroll
    for (int o = W / 2; o >= 1; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
    if constexpr (T > 32) {
      if ((t & 31) == 0) red[rl * WPR + (t >> 5)] = v;
    }
  }
  if constexpr (T > 32) {
    Bar::sync();
    if (compute) {
      v = red[rl * WPR];
#pragma unroll
      for (int w = 1; w < WPR; ++w) v = op(v, red[rl * WPR + w]);
    }
  }
  return v;
}

// Passes 1-3 and the LayerNorm folding for the row of this thread: on return
// e[0..63] = t[64 t .. 64 t + 63], t = H LN(x) / sqrt(K) in float (t_0 = 0),
// or with kLN false the plain scaled transform H x / sqrt(K).  x of an inactive
// row is taken as zeros.  All S::R * S::T threads behind Bar call it (it
// synchronizes them); `red1` is one row-reduction scratch (S::RED bytes).
// Warps with `compute` false (warp-uniform) only meet the barriers: they touch
// no shared memory and leave e undefined.
template <class S, bool IN_BF16, bool kLN, class Bar = BarCta>
__device__ __forceinline__ void fht_ln_rows(const void* xrow, bool active, int rl, int t, float* smem,
                                            float* red1, float sK, float (&e)[64], bool compute = true) {
  constexpr int K = S::K, T = S::T, LOGK = S::LOG;
  const int row_off = rl * S::STRIDE;
  // ---- pass 1: load, remove a large row offset, stages of bits {0,1,2,k-3,k-2,k-1}
  if (compute) {
    float f8[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (active) {
      load8<IN_BF16>(xrow, 0, f8);
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) load8<IN_BF16>(xrow, (jj * T + t) * 8, &e[jj * 8]);
    } else {
#pragma unroll
      for (int r = 0; r < 64; ++r) e[r] = 0.0f;
    }
    // mu~ = mean of the row's first 8 values; subtracted only when it exceeds
    // their spread, i.e. when the row mean could cost float precision
    const float mu = (((f8[0] + f8[1]) + (f8[2] + f8[3])) + ((f8[4] + f8[5]) + (f8[6] + f8[7]))) * 0.125f;
    float lo = f8[0], hi = f8[0];
#pragma unroll
    for (int u = 1; u < 8; ++u) {
      lo = fminf(lo, f8[u]);
      hi = fmaxf(hi, f8[u]);
    }
    if (kLN && fabsf(mu) > hi - lo) {
#pragma unroll
      for (int r = 0; r < 64; r += 2) sub2(e[r], e[r + 1], mu);
    }
    stage_range(e, 0, 6);
    SwzBase sb(row_off, t * 8);
    store_pass1<0, T>(e, smem, sb);
  }
  Bar::sync();

  // ---- pass 2: stages of bits {6 .. k-4} on vectors of 2^PB floats
  if constexpr (LOGK >= 10) {
    if (compute) {
      int tb = 0;
#pragma unroll
      for (int j = 0; j < LOGK - 6; ++j) tb |= ((t >> j) & 1) << p2_bit<LOGK>(j);
      SwzBase sb(row_off, tb);
      Pass2<LOGK, 0, 64>::template load<0>(e, smem, sb);
      stage_range(e, S::PB, 6);
      Pass2<LOGK, 0, 64>::template store<0>(e, smem, sb);
    }
    Bar::sync();
  }

  // ---- pass 3: 64 contiguous elements per thread, stages of bits {3,4,5} left
  if (compute) {
    SwzBase sb(row_off, t * 64);
    load_pass3<0>(e, smem, sb);
    stage_range(e, 3, LOGK - 3 < 6 ? LOGK - 3 : 6);
  }

  // ---- LayerNorm statistics from the transform: K^2 var = sum_{i>=1} Y_i^2
  float cmul = sK;
  if constexpr (kLN) {
    float s0 = 0.0f, s1 = 0.0f;
    if (compute) {
      const float e0 = e[0];
      if (t == 0) e[0] = 0.0f;
#pragma unroll
      for (int r = 0; r < 64; r += 2) sq_acc2(s0, s1, e[r], e[r + 1]);
      if (t == 0) e[0] = e0;
    }
    const float ss = row_reduce<T, S::WPR, Bar>(s0 + s1, AddF(), red1, rl, t, compute);
    const float var = ss * (1.0f / ((float)K * (float)K));
    cmul = __fmul_rn(__fdiv_rn(1.0f, sqrtf(__fadd_rn(var, 1e-5f))), sK);
  }
  if (compute) {
#pragma unroll
    for (int r = 0; r < 64; r += 2) mul2(e[r], e[r + 1], cmul);
    if (kLN && t == 0) e[0] = 0.0f;
  }
}

// The row's quantizer parameters from its t (every thread of the row gets the
// same): INT8 absmax (gamma = max |t|) or INT4 absmean (beta from the double
// sum of |t|, rounded once).  `red2` is a second row-reduction scratch.
template <class S, int MODE, class Bar = BarCta>
__device__ __forceinline__ q::RowParams row_params(const float (&e)[64], void* red2, int rl, int t,
                                                   bool compute = true) {
  if constexpr (MODE == K1_Q8_I8) {
    float gm = 0.0f;
    if (compute) {
#pragma unroll
      for (int r = 0; r < 64; ++r) gm = fmaxf(gm, fabsf(e[r]));
    }
    gm = row_reduce<S::T, S::WPR, Bar>(gm, MaxF(), reinterpret_cast<float*>(red2), rl, t, compute);
    return q::params_int8(gm);
  } else {
    double a0 = 0.0, a1 = 0.0;
    if (compute) {
#pragma unroll
      for (int r = 0; r < 64; r += 2) {
        a0 += q::abs_f64(e[r]);
        a1 += q::abs_f64(e[r + 1]);
      }
    }
    const double a = row_reduce<S::T, S::WPR, Bar>(a0 + a1, AddD(), reinterpret_cast<double*>(red2), rl, t, compute);
    return q::params_int4_mean(a * q::pow2_recip(S::LOG));
  }
}

// The 64 codes rint(t r) of this thread as int8 bytes (w[j] holds codes
// 4j .. 4j + 3, lowest byte first); INT4 codes are clipped to [-8, 7].
template <int MODE>
__device__ __forceinline__ void codes64_i8(const float (&e)[64], float r, uint32_t (&w)[16]) {
  uint32_t m[64];
#pragma unroll
  for (int i = 0; i < 64; i += 2) magic2(e[i], e[i + 1], r, m[i], m[i + 1]);
  if constexpr (MODE == K1_Q4_I8) {
#pragma unroll
    for (int i = 0; i < 64; ++i) m[i] = q::clip_magic_int4(m[i]);
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) w[j] = q::gather_low_bytes(m[4 * j], m[4 * j + 1], m[4 * j + 2], m[4 * j + 3]);
}

}  // namespace fhtrows
}  // namespace hbl
