// Per-token activation quantizer shared by the fused LN+FHT+quant kernels and
// the quantizer-only kernel, so all of them make bit-identical decisions.
//
// "BitNet v2: Native 4-bit Activations with Hadamard Transformation for 1-bit
// LLMs", section "H-BitLinear", activation-quantization formula:
//   4 bit, per-token absmean: beta = mean|t|,
//          q = clip(rint(sqrt(7) t / (beta + eps)), -8, 7), scale = beta / sqrt(7)
//   8 bit, per-token absmax : gamma = max|t|,
//          q = clip(rint(127 t / (gamma + eps)), -128, 127), scale = gamma / 127
// Arithmetic contract (float unless stated): the mean of |t| is accumulated in
// double and rounded once to float; r = c / (stat + eps) is one IEEE division
// per row; each code is rint of the exact product t * r (round half to even,
// a single rounding).  The __f*_rn intrinsics pin every rounding.
#pragma once

#include <cstdint>

namespace hbl {
namespace q {

constexpr float kEps = 1e-5f;
constexpr float kSqrt7 = 2.6457513110645906f;  // sqrt(7) rounded to float
constexpr float kMagic = 12582912.0f;          // 1.5 * 2^23
constexpr int kMagicBits = 0x4B400000;

// |t| as a double, for the absmean accumulation: an exact float -> double
// conversion (it runs on the conversion pipe, which the kernels otherwise
// leave idle, and costs one issue slot) whose absolute value the double add
// takes as an operand modifier.
__device__ __forceinline__ double abs_f64(float t) { return fabs((double)t); }

// |t| * 2^-896 as a double, built from the float's bits with integer shifts
// instead of a conversion (whose pipe is narrow): the float's exponent and
// mantissa fields, shifted right by 3, are a double's fields of the same
// value scaled by 2^(127 - 1023).  Exact for every finite float: a normal
// float gives a normal double, a subnormal float a subnormal double with the
// same scaling, zero gives zero.  Sums of these values round exactly as sums
// of |t| would (every partial sum below 2^-1022 is exact either way), so
// multiplying the sum by kUnscaleAbs (a power of two) gives the double sum of
// |t| itself.
__device__ __forceinline__ double abs_scaled_f64(float t) {
  const uint32_t b = __float_as_uint(t);
  return __hiloint2double((int)((b & 0x7FFFFFFFu) >> 3), (int)(b << 29));
}
constexpr double kUnscaleAbs = 0x1p896;

struct RowParams {
  float r;     // multiplier applied to t before rounding
  float stat;  // beta (INT4) or gamma (INT8)
  float c;     // sqrt(7) or 127
  // dequantisation factor of the row, stat / c (one IEEE division; computed
  // only by the thread that stores it)
  __device__ __forceinline__ float scale() const { return __fdiv_rn(stat, c); }
};

// beta from the mean of |t|, already formed in double and rounded here once.
__device__ __forceinline__ RowParams params_int4_mean(double abs_mean) {
  RowParams p;
  p.stat = (float)abs_mean;
  p.c = kSqrt7;
  p.r = __fdiv_rn(kSqrt7, __fadd_rn(p.stat, kEps));
  return p;
}

// beta from the double sum of |t| over K elements.
__device__ __forceinline__ RowParams params_int4(double abs_sum, int64_t K) {
  return params_int4_mean(abs_sum / (double)K);
}

// The same for K = 2^log2k: dividing by a power of two and multiplying by its
// reciprocal give the identical double (both the correctly rounded value of
// the same real number), without the division sequence.
__device__ __forceinline__ double pow2_recip(int log2k) {
  return __longlong_as_double((long long)(1023 - log2k) << 52);
}

// gamma = max |t| (exact, order free).
__device__ __forceinline__ RowParams params_int8(float gamma) {
  RowParams p;
  p.stat = gamma;
  p.c = 127.0f;
  p.r = __fdiv_rn(127.0f, __fadd_rn(gamma, kEps));
  return p;
}

// rint(t * r) of the exact product, for |t * r| < 2^22: t * r + 1.5 * 2^23
// lies in [2^23, 2^24) where a float's unit in the last place is 1, so the one
// rounding of the fused multiply-add is the rounding of t * r to the nearest
// integer, ties to even (1.5 * 2^23 is even), and the integer sits in the low
// mantissa bits.  Exact over the whole range the callers use: |t r| <= K sqrt(7)
// for absmean, < 127.5 for absmax.
__device__ __forceinline__ int rint_code(float t, float r) {
  return __float_as_int(__fmaf_rn(t, r, kMagic)) - kMagicBits;
}

// Eight codes -> eight 4-bit two's-complement fields, n[0] in the lowest
// nibble; cvt.pack.sat saturates each input to [-8, 7] (the clip).
__device__ __forceinline__ uint32_t pack_s4x8(const int (&n)[8]) {
  uint32_t d;
  asm("cvt.pack.sat.s4.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(n[7]), "r"(n[6]), "r"(0u));
  asm("cvt.pack.sat.s4.s32.b32 %0, %1, %2, %0;" : "+r"(d) : "r"(n[5]), "r"(n[4]));
  asm("cvt.pack.sat.s4.s32.b32 %0, %1, %2, %0;" : "+r"(d) : "r"(n[3]), "r"(n[2]));
  asm("cvt.pack.sat.s4.s32.b32 %0, %1, %2, %0;" : "+r"(d) : "r"(n[1]), "r"(n[0]));
  return d;
}

// Four codes -> four int8 bytes, n[0] in the lowest byte, saturated to
// [-128, 127].
__device__ __forceinline__ uint32_t pack_s8x4(int n0, int n1, int n2, int n3) {
  uint32_t d;
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(n3), "r"(n2), "r"(0u));
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %0;" : "+r"(d) : "r"(n1), "r"(n0));
  return d;
}

__device__ __forceinline__ int clip_int4(int n) { return max(-8, min(7, n)); }

// The bits of fl(t r + 1.5*2^23) are kMagicBits + rint(t r), so clipping
// the bits clips the code, and the low byte is the code as an int8.
__device__ __forceinline__ uint32_t clip_magic_int4(uint32_t m) {
  return (uint32_t)max(kMagicBits - 8, min(kMagicBits + 7, (int)m));
}

// Two codes from the magic-FMA bits of a pair, clipped to the INT4 range,
// as two int16 halves (lo in the low half).  The low 16 bits of the bits are
// the code itself (kMagicBits has zero low halves), so this is exact when
// every |code| < 2^15, which the caller guarantees per row.
__device__ __forceinline__ uint32_t clip_pair_int4_s16(uint32_t m_lo, uint32_t m_hi) {
  uint32_t v = __byte_perm(m_lo, m_hi, 0x5410);
  asm("max.s16x2 %0, %0, %1;" : "+r"(v) : "r"(0xFFF8FFF8u));
  asm("min.s16x2 %0, %0, %1;" : "+r"(v) : "r"(0x00070007u));
  return v;
}

// Low bytes of four words -> one word, a in the lowest byte.
__device__ __forceinline__ uint32_t gather_low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  const uint32_t ab = __byte_perm(a, b, 0x0040);
  const uint32_t cd = __byte_perm(c, d, 0x0040);
  return __byte_perm(ab, cd, 0x5410);
}

}  // namespace q
}  // namespace hbl
