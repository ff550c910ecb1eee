/*
 * hbl_oracle.c -- CPU oracle for the BitNet v2 H-BitLinear forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file: only the tests, __graft_entry__.smoke() and the CPU-baseline
 * leg of bench.py use it.  It shares no code, header, table or constant with
 * the CUDA library in ternary_gemm_b200/csrc.
 *
 * Plain, slow, single-threaded C.  Every function follows one step of the
 * method as the pages state it ("BitNet v2: Native 4-bit Activations with
 * Hadamard Transformation for 1-bit LLMs", arXiv 2504.18415; the news
 * articles on it by QbitAI and Xinzhiyuan, section "H-BitLinear"):
 *
 *   y = Q_w(W) applied to Q_act(H(LN(x)))            (H-BitLinear, eq. "matmul")
 *
 * The pages print the formulas only as images, so the concrete arithmetic is
 * the written specification of the path (one row = one token):
 *   LN      : plain LayerNorm, no affine, eps_ln = 1e-5, biased variance.
 *   H       : Sylvester-order Walsh-Hadamard matrix of size K (a power of
 *             two), scaled by 1/sqrt(K), so H/sqrt(K) is orthogonal.
 *   Q_act 4 : beta = mean|t|, q = clip(rint(sqrt(7) t / (beta+eps)), -8, 7),
 *             scale = beta / sqrt(7)            (per-token absmean)
 *   Q_act 8 : gamma = max|t|, q = clip(rint(127 t / (gamma+eps)), -128, 127),
 *             scale = gamma / 127               (per-token absmax)
 *   Q_w     : alpha = mean|W| over the whole tensor,
 *             w = clip(rint(W / (alpha+eps)), -1, 1)   (per-tensor absmean)
 *   GEMM    : acc[m][n] = sum_k q[m][k] w[n][k], exact integers.
 *   dequant : y[m][n] = (float)acc[m][n] * (scale[m] * alpha).
 * eps = 1e-5 for every quantizer; rint rounds half to even.
 *
 * Beside the forward (the next steps the pages describe):
 *   LN backward : g_x = (g_u - mean g_u - u mean(g_u u)) / sqrt(var + eps_ln),
 *                 the LayerNorm gradient the straight-through estimator needs
 *                 (training strategy: gradients bypass the quantizers);
 *   QKV states  : gamma = max|x| per head vector, L = 2^b - 1,
 *                 q = clip(rint(x L / (2 (gamma+eps)) + L/2), 0, L), scale = gamma
 *                 (low-bit attention: heads to unsigned integers by absmax);
 *   RMSNorm     : x / sqrt(mean x^2 + eps_ln), for the layers without the transform.
 *
 * Precision: LN and the Hadamard transform run in double (the reference
 * precision).  The quantizers take the single-precision FHT output and make
 * their integer decisions in single precision, as the GPU does: the mean of
 * |t| is accumulated in double and rounded once to float, the reciprocal
 * sqrt(7)/(beta+eps) is one IEEE float division per row, and each code is
 * rint of the exact product of the float t and the float reciprocal (one
 * rounding, half to even).
 */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_EPS_LN 1e-5
#define ORC_EPS_Q 1e-5f

/* dtype tags of the oracle's own API (independent of the library's enum) */
#define ORC_F32 0
#define ORC_BF16 1

/* ---------------------------------------------------------------- helpers */

/* bfloat16 -> float: the bf16 bits are the high half of the float bits. */
static float orc_bf16_bits_to_float(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* float -> bfloat16 with round-to-nearest-even (NaN kept quiet). */
uint16_t orc_float_to_bf16_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

void orc_round_to_bf16(const float* in, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_float_to_bf16_bits(in[i]);
}

static double orc_load(const void* x, int dtype, int64_t idx) {
  if (dtype == ORC_BF16) return (double)orc_bf16_bits_to_float(((const uint16_t*)x)[idx]);
  return (double)((const float*)x)[idx];
}

/* round half to even, as a double -> double map (uses the C library's rint
 * under the default rounding mode FE_TONEAREST). */
static double orc_rint(double v) { return rint(v); }

/* -------------------------------------------------------------- LayerNorm */

/* LN of one row in double: mu = mean x, var = mean (x - mu)^2 (two passes),
 * u = (x - mu) / sqrt(var + eps_ln).  The symbol LN of the H-BitLinear
 * matrix-operation formula is LayerNorm; no affine parameters are given, the
 * model has no bias. */
void orc_layernorm_row(const double* x, int64_t K, double* u) {
  double s = 0.0;
  for (int64_t i = 0; i < K; ++i) s += x[i];
  double mu = s / (double)K;
  double v = 0.0;
  for (int64_t i = 0; i < K; ++i) v += (x[i] - mu) * (x[i] - mu);
  v /= (double)K;
  double inv = 1.0 / sqrt(v + ORC_EPS_LN);
  for (int64_t i = 0; i < K; ++i) u[i] = (x[i] - mu) * inv;
}

/* LayerNorm backward of one row in double (no affine, eps 1e-5), the chain
 * rule through u = (x - mu) / sigma with mu and sigma functions of x:
 *   g_x = (g_u - mean(g_u) - u mean(g_u u)) / sigma
 * (the pages' training strategy: the straight-through estimator stands in
 * for the quantizers' gradient and the orthogonal Hadamard matrix carries the
 * gradient through the transform; everything before the transform is
 * ordinary backpropagation). */
void orc_ln_backward_row(const double* x, const double* gu, int64_t K, double* gx) {
  double sum = 0.0;
  for (int64_t i = 0; i < K; ++i) sum += x[i];
  const double mu = sum / (double)K;
  double ss = 0.0;
  for (int64_t i = 0; i < K; ++i) ss += (x[i] - mu) * (x[i] - mu);
  const double var = ss / (double)K;
  const double inv = 1.0 / sqrt(var + ORC_EPS_LN); /* 1 / sigma */
  double mg = 0.0, mgu = 0.0;
  for (int64_t i = 0; i < K; ++i) {
    mg += gu[i];
    mgu += gu[i] * (x[i] - mu) * inv;
  }
  mg /= (double)K;
  mgu /= (double)K;
  for (int64_t i = 0; i < K; ++i) gx[i] = (gu[i] - mg - (x[i] - mu) * inv * mgu) * inv;
}

/* ------------------------------------------------------- Hadamard (Sylvester) */

/* In-place unnormalised fast Walsh-Hadamard transform, natural (Sylvester)
 * order: H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]].  The recursion applied
 * bottom up: at span h every pair (j, j+h) in a block of 2h becomes
 * (a + b, a - b).  O(n log n) additions: the fast transform the pages name. */
void orc_fht_unnormalized(double* v, int64_t n) {
  for (int64_t h = 1; h < n; h *= 2)
    for (int64_t i = 0; i < n; i += 2 * h)
      for (int64_t j = i; j < i + h; ++j) {
        double a = v[j], b = v[j + h];
        v[j] = a + b;
        v[j + h] = a - b;
      }
}

/* Entry (i, j) of the Sylvester Hadamard matrix: (-1)^popcount(i & j). */
int orc_hadamard_entry(int64_t i, int64_t j) {
  return (__builtin_popcountll((unsigned long long)(i & j)) & 1) ? -1 : 1;
}

/* Dense matrix-vector product out = H_n v in double, O(n^2).  A second,
 * independent route to the same transform, used to pin the fast one. */
void orc_hadamard_explicit(const double* v, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) {
    double s = 0.0;
    for (int64_t j = 0; j < n; ++j) s += orc_hadamard_entry(i, j) * v[j];
    out[i] = s;
  }
}

/* t = H_K LN(x) / sqrt(K) for each of M rows of length K (K a power of two).
 * Outputs the double result (t64, may be NULL) and its rounding to float
 * (t32, may be NULL).  Returns 0, or -1 if K is not a power of two. */
int orc_ln_fht(const void* x, int dtype, int64_t M, int64_t K, double* t64, float* t32) {
  if (K < 1 || (K & (K - 1))) return -1;
  double* row = (double*)malloc(sizeof(double) * (size_t)K);
  double* u = (double*)malloc(sizeof(double) * (size_t)K);
  if (!row || !u) { free(row); free(u); return -2; }
  double sc = 1.0 / sqrt((double)K);
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t i = 0; i < K; ++i) row[i] = orc_load(x, dtype, m * K + i);
    orc_layernorm_row(row, K, u);
    orc_fht_unnormalized(u, K);
    for (int64_t i = 0; i < K; ++i) {
      double t = u[i] * sc;
      if (t64) t64[m * K + i] = t;
      if (t32) t32[m * K + i] = (float)t;
    }
  }
  free(row);
  free(u);
  return 0;
}

/* RMSNorm of one row in double: u = x / sqrt(mean x^2 + eps_ln), no affine.
 * (The model around H-BitLinear uses RMSNorm; the BitLinear layers without
 * the Hadamard transform are normalised this way or with LayerNorm.) */
void orc_rmsnorm_row(const double* x, int64_t K, double* u) {
  double s = 0.0;
  for (int64_t i = 0; i < K; ++i) s += x[i] * x[i];
  double inv = 1.0 / sqrt(s / (double)K + ORC_EPS_LN);
  for (int64_t i = 0; i < K; ++i) u[i] = x[i] * inv;
}

/* The activation path of a BitLinear layer without the Hadamard transform:
 * t = LN(x) (norm = 0) or RMSNorm(x) (norm = 1) per row, any K >= 1.
 * Outputs the double result and its rounding to float (either may be NULL). */
int orc_norm_rows(const void* x, int dtype, int64_t M, int64_t K, int norm, double* t64, float* t32) {
  if (K < 1 || (norm != 0 && norm != 1)) return -1;
  double* row = (double*)malloc(sizeof(double) * (size_t)K);
  double* u = (double*)malloc(sizeof(double) * (size_t)K);
  if (!row || !u) { free(row); free(u); return -2; }
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t i = 0; i < K; ++i) row[i] = orc_load(x, dtype, m * K + i);
    if (norm == 0) orc_layernorm_row(row, K, u);
    else orc_rmsnorm_row(row, K, u);
    for (int64_t i = 0; i < K; ++i) {
      if (t64) t64[m * K + i] = u[i];
      if (t32) t32[m * K + i] = (float)u[i];
    }
  }
  free(row);
  free(u);
  return 0;
}

/* t = H_K x / sqrt(K) per row in double (no normalisation): the rotation the
 * Hadamard ablation also applies to the weights.  K a power of two. */
int orc_fht_rows(const void* x, int dtype, int64_t M, int64_t K, double* t64, float* t32) {
  if (K < 1 || (K & (K - 1))) return -1;
  double* row = (double*)malloc(sizeof(double) * (size_t)K);
  if (!row) return -2;
  double inv_sqrt_k = 1.0 / sqrt((double)K);
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t i = 0; i < K; ++i) row[i] = orc_load(x, dtype, m * K + i);
    orc_fht_unnormalized(row, K);
    for (int64_t i = 0; i < K; ++i) {
      double t = row[i] * inv_sqrt_k;
      if (t64) t64[m * K + i] = t;
      if (t32) t32[m * K + i] = (float)t;
    }
  }
  free(row);
  return 0;
}

/* --------------------------------------------------- activation quantizers */

/* Per-token activation quantization of M rows of length K (any K >= 1).
 * bits = 4: absmean, codes in [-8, 7]; bits = 8: absmax, codes in [-128, 127].
 * (the pages: absmax per token for 8-bit activations, absmean per token for
 * 4-bit ones).
 * codes: int8 [M][K] (unpacked); scales: float [M] (dequant factor per row).
 * Returns 0, or -1 on bad bits. */
int orc_quant(const float* t, int64_t M, int64_t K, int bits, int8_t* codes, float* scales) {
  if (bits != 4 && bits != 8) return -1;
  fesetround(FE_TONEAREST);
  const float c = (bits == 4) ? sqrtf(7.0f) : 127.0f;
  const double lo = (bits == 4) ? -8.0 : -128.0;
  const double hi = (bits == 4) ? 7.0 : 127.0;
  for (int64_t m = 0; m < M; ++m) {
    const float* r = t + m * K;
    float stat;
    if (bits == 4) {
      double s = 0.0;                       /* beta = mean |t| */
      for (int64_t i = 0; i < K; ++i) s += (double)fabsf(r[i]);
      stat = (float)(s / (double)K);
    } else {
      float g = 0.0f;                       /* gamma = max |t| */
      for (int64_t i = 0; i < K; ++i) if (fabsf(r[i]) > g) g = fabsf(r[i]);
      stat = g;
    }
    volatile float den = stat + ORC_EPS_Q;  /* one float add */
    volatile float rcp = c / den;           /* one float division per row */
    for (int64_t i = 0; i < K; ++i) {
      /* rint of the exact product t * r: a product of two floats is exact in
       * double, so this is one rounding to the nearest integer */
      double q = orc_rint((double)r[i] * (double)rcp);
      if (q < lo) q = lo;
      if (q > hi) q = hi;
      codes[m * K + i] = (int8_t)q;
    }
    volatile float sc = stat / c;
    scales[m] = sc;
  }
  return 0;
}

/* ------------------------------------------------------ ternary weights */

/* Per-tensor absmean ternarization of W [N][K] (row-major, out x in):
 * alpha = mean|W| (double sum, rounded once to float),
 * w = clip(rint(W / (alpha + eps)), -1, 1) computed as rint of the exact
 * product W * r with the float reciprocal r = 1/(alpha+eps).
 * (the pages: the weights go to {-1, 0, 1} by a per-tensor absmean) */
void orc_ternary(const void* W, int dtype, int64_t N, int64_t K, int8_t* w, float* alpha) {
  fesetround(FE_TONEAREST);
  double s = 0.0;
  int64_t n = N * K;
  for (int64_t i = 0; i < n; ++i) s += fabs(orc_load(W, dtype, i));
  float a = (float)(s / (double)n);
  volatile float den = a + ORC_EPS_Q;
  volatile float rcp = 1.0f / den;
  for (int64_t i = 0; i < n; ++i) {
    double q = orc_rint(orc_load(W, dtype, i) * (double)rcp);   /* exact product, one rounding */
    if (q < -1.0) q = -1.0;
    if (q > 1.0) q = 1.0;
    w[i] = (int8_t)q;
  }
  *alpha = a;
}

/* ---------------------------------------------------------- integer GEMM */

/* acc[m][n] = sum_k A[m][k] * B[n][k] with exact 64-bit accumulation.
 * Returns 0, or -1 if a result does not fit in int32. */
int orc_gemm_i32(const int8_t* A, const int8_t* B, int64_t M, int64_t N, int64_t K, int32_t* acc) {
  int bad = 0;
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      int64_t s = 0;
      for (int64_t k = 0; k < K; ++k) s += (int64_t)A[m * K + k] * (int64_t)B[n * K + k];
      if (s > INT32_MAX || s < INT32_MIN) bad = 1;
      acc[m * N + n] = (int32_t)s;
    }
  return bad ? -1 : 0;
}

/* y[m][n] = (float)acc[m][n] * (scale[m] * alpha), all in float. */
void orc_dequant(const int32_t* acc, const float* scales, float alpha, int64_t M, int64_t N, float* y) {
  for (int64_t m = 0; m < M; ++m) {
    volatile float sa = scales[m] * alpha;
    for (int64_t n = 0; n < N; ++n) {
      volatile float v = (float)acc[m * N + n] * sa;
      y[m * N + n] = v;
    }
  }
}

/* ------------------------------------------------------------ code packing */

/* INT4 codes -> bytes: element 2j in the low nibble, 2j+1 in the high
 * nibble, each as a 4-bit two's-complement number.  K even. */
void orc_pack_int4(const int8_t* q, int64_t M, int64_t K, uint8_t* out) {
  for (int64_t m = 0; m < M; ++m)
    for (int64_t j = 0; j < K / 2; ++j) {
      unsigned lo = (unsigned)(q[m * K + 2 * j] & 0xF);
      unsigned hi = (unsigned)(q[m * K + 2 * j + 1] & 0xF);
      out[m * (K / 2) + j] = (uint8_t)(lo | (hi << 4));
    }
}

void orc_unpack_int4(const uint8_t* in, int64_t M, int64_t K, int8_t* q) {
  for (int64_t m = 0; m < M; ++m)
    for (int64_t j = 0; j < K / 2; ++j) {
      int lo = in[m * (K / 2) + j] & 0xF;
      int hi = (in[m * (K / 2) + j] >> 4) & 0xF;
      q[m * K + 2 * j] = (int8_t)(lo >= 8 ? lo - 16 : lo);
      q[m * K + 2 * j + 1] = (int8_t)(hi >= 8 ? hi - 16 : hi);
    }
}

/* Ternary codes -> 2-bit fields: element 4j+i at bits 2i..2i+1 of byte j,
 * 0 -> 00, +1 -> 01, -1 -> 11.  K a multiple of 4. */
void orc_pack_ternary(const int8_t* w, int64_t N, int64_t K, uint8_t* out) {
  for (int64_t n = 0; n < N; ++n)
    for (int64_t j = 0; j < K / 4; ++j) {
      unsigned byte = 0;
      for (int i = 0; i < 4; ++i) {
        int8_t v = w[n * K + 4 * j + i];
        unsigned f = (v == 0) ? 0u : (v == 1 ? 1u : 3u);
        byte |= f << (2 * i);
      }
      out[n * (K / 4) + j] = (uint8_t)byte;
    }
}

/* Returns the number of fields holding the unused pattern 10 (0 if valid). */
int64_t orc_unpack_ternary(const uint8_t* in, int64_t N, int64_t K, int8_t* w) {
  int64_t bad = 0;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t j = 0; j < K / 4; ++j)
      for (int i = 0; i < 4; ++i) {
        unsigned f = (in[n * (K / 4) + j] >> (2 * i)) & 3u;
        int8_t v = 0;
        if (f == 1u) v = 1;
        else if (f == 3u) v = -1;
        else if (f == 2u) ++bad;
        w[n * K + 4 * j + i] = v;
      }
  return bad;
}

/* ------------------------------------------------------------- forward */

/* Whole H-BitLinear forward for the rows of x listed in `rows` (or all M rows
 * if rows == NULL, nrows = M): LN -> H -> Q_act -> integer GEMM against the
 * ternary codes w [N][K] -> dequant by scale * alpha.  Writes y [nrows][N]
 * float, and optionally the codes [nrows][K] and scales [nrows].
 * Returns 0 or a negative error. */
int orc_forward_rows(const void* x, int dtype, int64_t M, int64_t K, const int64_t* rows, int64_t nrows,
                     const int8_t* w, float alpha, int64_t N, int bits, float* y, int8_t* codes_out,
                     float* scales_out) {
  if (K < 1 || (K & (K - 1))) return -1;
  size_t esz = dtype == ORC_BF16 ? 2 : 4;
  unsigned char* xr = (unsigned char*)malloc(esz * (size_t)K);
  float* t = (float*)malloc(sizeof(float) * (size_t)K);
  int8_t* q = (int8_t*)malloc((size_t)K);
  int32_t* acc = (int32_t*)malloc(sizeof(int32_t) * (size_t)N);
  if (!xr || !t || !q || !acc) { free(xr); free(t); free(q); free(acc); return -2; }
  int rc = 0;
  for (int64_t r = 0; r < nrows && rc == 0; ++r) {
    int64_t m = rows ? rows[r] : r;
    if (m < 0 || m >= M) { rc = -3; break; }
    memcpy(xr, (const unsigned char*)x + esz * (size_t)(m * K), esz * (size_t)K);
    orc_ln_fht(xr, dtype, 1, K, NULL, t);
    float s;
    orc_quant(t, 1, K, bits, q, &s);
    if (orc_gemm_i32(q, w, 1, N, K, acc) != 0) rc = -4;
    orc_dequant(acc, &s, alpha, 1, N, y + r * N);
    if (codes_out) memcpy(codes_out + r * K, q, (size_t)K);
    if (scales_out) scales_out[r] = s;
  }
  free(xr); free(t); free(q); free(acc);
  return rc;
}

/* ------------------------------------------------------- low-bit QKV states */

/* Post-RoPE QKV-state quantizer of the low-bit attention experiments (QbitAI
 * report / Xinzhiyuan article, section on low-bit attention: the QKV heads are quantized
 * to unsigned integers by the absmax function, with no calibration data; a
 * 3-bit KV cache matches full precision).  Reading of the open steps: one head
 * vector of D values (one token, one head) at a time; gamma = max|x|; the
 * range [-gamma, gamma] maps linearly onto the 2^b unsigned levels 0 .. 2^b-1:
 *   L = 2^b - 1,  r = L / (2 (gamma + eps))  (one float division),
 *   q = clip(rint(fl(fl(x r) + L/2)), 0, L),  scale = gamma,
 * so x ~ (2 q - L) gamma / L.  rint rounds half to even. */
int orc_kv_quant(const void* x, int dtype, int64_t rows, int64_t D, int bits, uint8_t* codes, float* scales) {
  if (rows < 0 || D <= 0 || bits < 2 || bits > 8) return -1;
  const float L = (float)((1 << bits) - 1);
  const float half = 0.5f * L;
  for (int64_t m = 0; m < rows; ++m) {
    float g = 0.0f;
    for (int64_t i = 0; i < D; ++i) {
      float a = fabsf((float)orc_load(x, dtype, m * D + i));
      if (a > g) g = a;
    }
    volatile float den = 2.0f * (g + ORC_EPS_Q);
    volatile float r = L / den;
    for (int64_t i = 0; i < D; ++i) {
      volatile float t = (float)orc_load(x, dtype, m * D + i) * r;
      volatile float u = t + half;
      double q = orc_rint((double)u);
      if (q < 0.0) q = 0.0;
      if (q > (double)L) q = (double)L;
      codes[m * D + i] = (uint8_t)q;
    }
    scales[m] = g;
  }
  return 0;
}
