// Fused LayerNorm -> fast Walsh-Hadamard transform -> per-token quantization
// with the transform split between the tensor cores and the FMA pipe
// ("BitNet v2: Native 4-bit Activations with Hadamard Transformation for
// 1-bit LLMs", section "H-BitLinear": the Hadamard-transform definition and
// the activation-quantization formula).  bf16 input, K = 128 .. 32768.
//
// Sylvester's matrix factors over the index bits: with i = C i_hi + i_lo,
// j = C j_hi + j_lo and KH = K / C,
//   H_K[i][j] = H_KH[i_hi][j_hi] * H_C[i_lo][j_lo],
// so Y = H_K x is two smaller transforms.  The high one is a dense
// contraction whose operands are exact in bf16 (x itself and +-1), so it runs
// on the tensor cores; the low one runs as butterflies in registers.  The
// chunk width is C = 64 for K <= 8192 (KH = 2 .. 128) and C = 128 for
// K = 16384 (KH = 128), so KH never exceeds the MMA's 128:
//
//   x viewed as chunk rows Xc[M*KH][C] (row-major, no copy);
//   box     = 128 chunk rows x 64 columns of bf16 (16 KB), one TMA copy;
//   group   = two boxes side by side: C = 64, two consecutive 128-row units;
//             C = 128, the two column halves of one 128-row tile;
//   MMA     D[m][n] = sum_k A[m][k] B[k][n], tcgen05.mma kind::f16,
//           M = 128, N = 128 (the group's two boxes), K = 8 x 16, f32
//           accumulator in TMEM; A = blockdiag(H_KH, ..., H_KH) (+-1 / 0)
//           is written into TMEM once, so the tensor core reads only x from
//           shared memory.  Lane m of a box = (token row m / KH, i_hi =
//           m % KH).  Wide MMAs matter: an N = 64 MMA costs about as long as
//           an N = 128 one, and at N = 64 the MMA time did not hide under
//           the loads.
//   C = 64  each 64-column half of D is one unit, taken by one epilogue
//           warpgroup: 64 columns per thread, 6 butterfly stages.
//   C = 128 a pair of epilogue warpgroups shares the tile: warpgroup h loads
//           columns 64h .. 64h + 63 of its lanes, runs the 6 stages of the
//           low 6 column bits, keeps columns 32h .. 32h + 31 and
//           64 + 32h .. 95 + 32h, and swaps the other 32 with its partner
//           through TMEM (behind a pair barrier) for the stage on column
//           bit 6.  Each thread ends with 64 values.
// The tensor-core sums are exact whenever the bf16 terms of a sum span < 2^9
// in magnitude (their common unit in the last place then divides the
// result), and otherwise round in float like the butterflies would.
//
// LayerNorm is folded around the transform: row 0 of H is all ones, so
// sum_{i>=1} Y_i^2 = K^2 var and t_i = Y_i / sqrt(K (var + eps_ln)) for
// i >= 1, t_0 = 0.  A large row mean only reaches the lanes with i_hi = 0
// (the other rows of H_KH sum to zero); those subtract their own column-0
// value from all C columns before the butterflies, which changes only Y_0
// (discarded) and keeps the float sums on the deviations.
//
// CTA (one per SM, persistent over groups), five warpgroups:
//   warp 0     TMA producer: two boxes per group into a 4-group ring;
//   warp 1     TMEM allocation (512 columns: A in the last 64, three
//              128-column accumulator regions) and one thread issuing the
//              MMAs of a group;
//   warps 2-3  otherwise idle (registers are granted to whole warpgroups);
//              in hbl_forward they widen the ternary weights to int8 for the
//              GEMM that follows (a grid-stride loop, 16 codes per thread
//              and step), which the issue-bound epilogue leaves room for;
//   warps 4-19 four epilogue warpgroups in two pairs; pair p takes every
//              other group: TMEM -> registers, butterflies, LayerNorm
//              statistics, quantizer, codes stored straight to global memory
//              (each warp writes whole consecutive chunk rows).
// Row statistics reduce over the threads of a token row: warp shuffles, then
// per-warp slots behind a named barrier of the row's warpgroup (pair).  The
// first reduction gives sum Y^2 (and for INT8 max |y| of the transformed but
// unscaled y), hence cmul; every mode then forms t = fl(cmul y), the value the
// debug mode writes out.  INT8 is exact from the first reduction: gamma =
// fl(cmul max|y|) = max|t| (rounding is monotone).  INT4 needs sum |t|
// itself: a second reduction sums |t| in
// double (each |t| made exactly from its bits, scaled by a power of two) and
// rounds the mean once to float, as the quantizer-only kernel does.  Both then take r = c / (stat + eps) and
// the scale stat / c as correctly rounded divisions and the codes as
// rint(t r) of the exact product, so the codes and scales are those of the
// quantizer applied to t.  INT4 codes widened to int8 are clipped on packed
// 16-bit halves when the row bound ||t|| r keeps every code below 2^15, else
// on 32-bit values.
// The block is launched with at most 96 registers per thread and rebalanced
// with setmaxnreg: the first warpgroup gives its share down to 64, the
// epilogue warpgroups take 104 each, which uses the launch's 640 x 96
// registers exactly (the host checks that the launch count covers this split
// before launching).  At 40 the producer, MMA and widening loops spilled.
// Every mbarrier wait is bounded (by the device status's limit, 2 s unless a
// test shortens it; then the CTA abort flag and the device error word are set
// and every role leaves its loop), and the producer waits (bounded by 2 s)
// for the loads it issued before the CTA exits.
#include <cstdint>

#include "common.cuh"
#include "quant.cuh"
#include "rowkit.cuh"
#include "sm100.cuh"
#include "ternary.cuh"

namespace hbl {
namespace {

using namespace sm100;
using namespace rowkit;

constexpr int kBoxCols = 64;                         // bf16 columns per box (one 128-byte swizzle row)
constexpr int kBoxRows = 128;                        // chunk rows per box (MMA M and K)
constexpr int kBoxBytes = kBoxRows * kBoxCols * 2;   // 16 KB
constexpr int kSlots = 4;                            // ring slots of two boxes (one group)
constexpr int kSlotBytes = 2 * kBoxBytes;
constexpr int kEpiGroups = 4;                        // epilogue warpgroups
constexpr int kThreads = 128 + 128 * kEpiGroups;
constexpr int kCtrlRegs = 64;  // registers per thread of the first warpgroup after setmaxnreg
constexpr int kEpiRegs = 104;  // registers per thread of an epilogue warpgroup after setmaxnreg
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAcol = 448;  // TMEM column of A (64 columns: 128 bf16 per lane)
constexpr int kRegions = 3;      // 128-column accumulators below kAcol
constexpr size_t kSmemBytes = 1024 + (size_t)kSlots * kSlotBytes + 1024;

// instruction descriptor, kind::f16: D f32, A and B bf16, A K-major, B
// MN-major, N = 128, M = 128
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

struct TcParams {
  int64_t M;         // token rows
  int64_t nchunk;    // chunk rows, M * KH
  int num_groups;    // MMA groups
  float sK;          // 1 / sqrt(K) rounded to float
  float* t_out;      // K1_T_F32: t [M][K]
  uint8_t* codes;    // quantizing modes: codes [M][K/2] (packed) or [M][K] (int8)
  int codes_al32;    // codes 32-byte aligned (256-bit stores allowed)
  const uint32_t* wpacked;  // weight widening by the idle warps: 2-bit codes (16-byte aligned)
  uint4* wout;              // int8 codes out, 16 per uint4
  int64_t wwords;           // 32-bit words of 2-bit codes, a multiple of 4 (0: no widening)
  float* scales;     // [M]
  int* err;          // device error word
};

// D (TMEM) (+)= A (TMEM) x B (shared memory descriptor)
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(kIdesc), "r"(accumulate));
}

// 32 bytes to global memory in one 256-bit store (p 32-byte aligned)
__device__ __forceinline__ void st_global_32B(void* p, const uint4& a, const uint4& b) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a.x), "r"(a.y), "r"(a.z),
               "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
               : "memory");
}

// one TMEM column of this warp's lane quarter
__device__ __forceinline__ uint32_t tmem_ld1(uint32_t taddr) {
  uint32_t v;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(v) : "r"(taddr));
  return v;
}

// Butterfly over register-index bit B of an N-float array.
template <int B, int N>
__device__ __forceinline__ void stage(float (&e)[N]) {
  if constexpr (B == 0) {
#pragma unroll
    for (int r = 0; r < N; r += 2) {
      const float a = e[r], c = e[r + 1];
      e[r] = a + c;
      e[r + 1] = a - c;
    }
  } else {
#pragma unroll
    for (int r = 0; r < N; r += 2)
      if (!(r & (1 << B))) bfly2(e[r], e[r + 1], e[r | (1 << B)], e[(r | (1 << B)) + 1]);
  }
}

// All-reduce of a pair of values over the RT threads of one token row, in
// one round: .x summed, .y summed or, with MAXY, maximized.  RT consecutive
// lanes when RT <= 32, else RT / 32 whole warps numbered wq (their slots)
// inside the barrier's `bar_n` threads.  Every thread of the row ends with
// the identical pair.  `failed` (a bounded wait of this group gave up) is
// or-ed over the barrier's threads, so they all leave the loop together.
template <int RT, bool MAXY>
__device__ __forceinline__ float2 group_reduce2(float2 v, float2* slots, int wq, int lane, int bar_id, int bar_n,
                                                bool& failed) {
  constexpr int W = RT < 32 ? RT : 32;
#pragma unroll
  for (int o = W / 2; o >= 1; o >>= 1) {
    const float a = __shfl_xor_sync(0xffffffffu, v.x, o);
    const float b = __shfl_xor_sync(0xffffffffu, v.y, o);
    v.x += a;
    v.y = MAXY ? fmaxf(v.y, b) : v.y + b;
  }
  if constexpr (RT > 32) {
    constexpr int NW = RT / 32;
    slots[wq] = v;  // every lane holds the same value
    failed = named_bar_any(bar_id, bar_n, failed);
    const int w0 = wq & ~(NW - 1);
    v = slots[w0];
#pragma unroll
    for (int i = 1; i < NW; ++i) {
      const float2 u = slots[w0 + i];
      v.x += u.x;
      v.y = MAXY ? fmaxf(v.y, u.y) : v.y + u.y;
    }
  }
  return v;
}

// The same all-reduce for one float sum.
template <int RT>
__device__ __forceinline__ float group_reduce1(float v, float* slots, int wq, int lane, int bar_id, int bar_n,
                                               bool& failed) {
  constexpr int W = RT < 32 ? RT : 32;
#pragma unroll
  for (int o = W / 2; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if constexpr (RT > 32) {
    constexpr int NW = RT / 32;
    slots[wq] = v;  // every lane holds the same value
    failed = named_bar_any(bar_id, bar_n, failed);
    const int w0 = wq & ~(NW - 1);
    v = slots[w0];
#pragma unroll
    for (int i = 1; i < NW; ++i) v += slots[w0 + i];
  }
  return v;
}

// The same all-reduce for one double sum (the INT4 absmean's second round).
// Additions commute exactly, so the butterfly leaves every lane with the
// identical value, and every thread reads the slots in the same order.
template <int RT>
__device__ __forceinline__ double group_reduce_d(double v, double* slots, int wq, int lane, int bar_id, int bar_n) {
  constexpr int W = RT < 32 ? RT : 32;
#pragma unroll
  for (int o = W / 2; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if constexpr (RT > 32) {
    constexpr int NW = RT / 32;
    slots[wq] = v;  // every lane holds the same value
    named_bar_sync(bar_id, bar_n);
    const int w0 = wq & ~(NW - 1);
    v = slots[w0];
#pragma unroll
    for (int i = 1; i < NW; ++i) v += slots[w0 + i];
  }
  return v;
}

// Per-thread reductions over y[0..63] with 8 independent accumulators (8
// short dependency chains) and a final tree, so they do not serialize on
// the add latency.
__device__ __forceinline__ float sum_sq64(const float (&y)[64]) {
  float s[8];
#pragma unroll
  for (int a = 0; a < 8; ++a) s[a] = 0.0f;
#pragma unroll
  for (int r = 0; r < 64; r += 2) sq_acc2(s[(r >> 1) & 6], s[((r >> 1) & 6) + 1], y[r], y[r + 1]);
#pragma unroll
  for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
    for (int a = 0; a < w; ++a) s[a] += s[a + w];
  return s[0];
}

// sum |t| over t[0..63] in double, scaled by 2^-896 (q::abs_scaled_f64: each
// |t| exact, no conversion instruction); eight independent accumulators keep
// the dependency chains short
__device__ __forceinline__ double sum_abs64_scaled(const float (&t)[64]) {
  double v[8];
#pragma unroll
  for (int a = 0; a < 8; ++a) v[a] = q::abs_scaled_f64(t[a]);
#pragma unroll
  for (int r = 8; r < 64; ++r) v[r & 7] += q::abs_scaled_f64(t[r]);
#pragma unroll
  for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
    for (int a = 0; a < w; ++a) v[a] += v[a + w];
  return v[0];
}

// max |y| (order-free and exact)
__device__ __forceinline__ float max_abs64(const float (&y)[64]) {
  float v[8];
#pragma unroll
  for (int a = 0; a < 8; ++a) v[a] = fabsf(y[a]);
#pragma unroll
  for (int r = 8; r < 64; ++r) v[r & 7] = fmaxf(v[r & 7], fabsf(y[r]));
#pragma unroll
  for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
    for (int a = 0; a < w; ++a) v[a] = fmaxf(v[a], v[a + w]);
  return v[0];
}

// Row m of A = blockdiag(H_KH, ..., H_KH) (128 x 128, bf16 +-1 / 0) as 64
// TMEM words: word c holds A[m][2c] in its low half and A[m][2c + 1] in its
// high half; written by the warp that owns lane m.
template <int KH>
__device__ __forceinline__ void store_a_row(uint32_t taddr, int m) {
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    uint32_t w[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      uint32_t hv[2];
#pragma unroll
      for (int v = 0; v < 2; ++v) {
        const int k = 64 * half + 2 * c + v;
        const bool same = (m / KH) == (k / KH);
        hv[v] = !same ? 0u : (0x3F80u ^ ((uint32_t)(__popc((m % KH) & (k % KH)) & 1) << 15));
      }
      w[c] = hv[0] | (hv[1] << 16);
    }
    tmem_st32(taddr + (uint32_t)(32 * half), w);
  }
}

// 16 int8 codes of y[0..15] (INT8 absmax, or INT4 codes widened to int8).
// INT4 with S16: clip on packed 16-bit halves (every |code| < 2^15).
template <int MODE, bool S16 = false>
__device__ __forceinline__ uint4 codes16_i8(const float* y, float r) {
  uint32_t w[4];
#pragma unroll
  for (int hh = 0; hh < 4; ++hh) {
    uint32_t mm[4];
    magic2(y[4 * hh], y[4 * hh + 1], r, mm[0], mm[1]);
    magic2(y[4 * hh + 2], y[4 * hh + 3], r, mm[2], mm[3]);
    if constexpr (MODE == K1_Q4_I8 && S16) {
      w[hh] = __byte_perm(q::clip_pair_int4_s16(mm[0], mm[1]), q::clip_pair_int4_s16(mm[2], mm[3]), 0x6420);
    } else {
      if constexpr (MODE == K1_Q4_I8) {
#pragma unroll
        for (int u = 0; u < 4; ++u) mm[u] = q::clip_magic_int4(mm[u]);
      }
      w[hh] = q::gather_low_bytes(mm[0], mm[1], mm[2], mm[3]);
    }
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// 32 INT4 codes of y[0..31] as packed nibbles (y[0] in the lowest nibble)
__device__ __forceinline__ uint4 codes32_s4(const float* y, float r) {
  uint32_t w[4];
#pragma unroll
  for (int hh = 0; hh < 4; ++hh) {
    uint32_t mm[8];
#pragma unroll
    for (int u = 0; u < 8; u += 2) magic2(y[8 * hh + u], y[8 * hh + u + 1], r, mm[u], mm[u + 1]);
    int n[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) n[u] = (int)mm[u] - q::kMagicBits;
    w[hh] = q::pack_s4x8(n);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Warps 2-3 (w = 0, 1) widen the ternary weights to int8 for hbl_forward's
// GEMM (its next stage; the issue-bound epilogue leaves slots to spare).  Only
// 64 threads per SM do it, so each keeps two 16-byte loads (128 codes) in
// flight; every warp store covers 2 KB of contiguous output.
__device__ __forceinline__ void widen_in_idle_warps(const TcParams& p, int w, int lane) {
  constexpr int kU = 2;
  const uint4* src = reinterpret_cast<const uint4*>(p.wpacked);
  const int64_t n4 = p.wwords / 4;  // 64 codes per uint4
  const int64_t stride = (int64_t)gridDim.x * 64;
  for (int64_t i = (int64_t)blockIdx.x * 64 + w * 32 + lane; i < n4; i += stride * kU) {
    uint4 v[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) v[u] = i + u * stride < n4 ? __ldg(src + i + u * stride) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (i + u * stride < n4) {
        uint4* d = p.wout + 4 * (i + u * stride);
        d[0] = tern::widen16(v[u].x);
        d[1] = tern::widen16(v[u].y);
        d[2] = tern::widen16(v[u].z);
        d[3] = tern::widen16(v[u].w);
      }
    }
  }
}

template <int LOGK, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
ln_fht_quant_tc_kernel(const __grid_constant__ CUtensorMap tmX, TcParams p) {
  constexpr int K = 1 << LOGK;
  constexpr int C = LOGK >= 14 ? 128 : 64;  // chunk width
  constexpr int KH = K / C;                 // chunk rows per token row
  static_assert(KH >= 2 && KH <= 128, "K out of range");
  constexpr bool PAIR = C == 128;           // a warpgroup pair shares each tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sB = base;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kSlots * kSlotBytes);
  uint64_t* empty = full + kSlots;
  uint64_t* tfull = empty + kSlots;
  uint64_t* tempty = tfull + kRegions;
  uint64_t* drain = tempty + kRegions;
  // [pair][group parity][8]: (sum of squares, |y| sum or max).  Two sets:
  // with no barrier between one group's reduction and the next group's, a
  // fast warp writes the other set while a slow one still reads this one.
  float2* red2 = reinterpret_cast<float2*>(drain + 1);
  double* redd = reinterpret_cast<double*>(red2 + 32);  // the same layout for the INT4 double sums
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(redd + 32);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < kRegions; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 8);  // the 8 warps of the pair that reads the region
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // A into TMEM: the first epilogue warpgroup writes its four lane quarters
  if (warp >= 4 && warp < 8) {
    store_a_row<KH>(tmem_base + kAcol + ((uint32_t)((warp & 3) * 32) << 16), (warp & 3) * 32 + lane);
    tmem_wait_st();
  }
  fence_before();
  __syncthreads();
  fence_after();
  // Launched as a programmatic dependent, the setup above overlapped the
  // previous kernel's tail; global memory is touched only after that kernel
  // completes (x may be its output, the codes and weights its input).  Only
  // then may this kernel's own dependents start (they wait for this kernel's
  // results themselves): a trigger before the wait would let them run beside
  // the kernel before this one.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtrlRegs));
    if (warp == 0) {
      // ---------------------------------------------- TMA producer
      if (lane == 0) {
        prefetch_tensormap(&tmX);
        int j = 0;  // groups issued
        for (;; ++j) {
          const int q = blockIdx.x + j * gridDim.x;
          if (q >= p.num_groups) break;
          const int slot = j % kSlots;
          if (!wait_bounded(&empty[slot], ((uint32_t)(j / kSlots) & 1u) ^ 1u, abort_flag, p.err)) break;
          mbar_expect_tx(&full[slot], (uint32_t)kSlotBytes);
          uint8_t* dst = sB + slot * kSlotBytes;
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            if constexpr (PAIR)
              tma_load_2d(dst + u * kBoxBytes, &tmX, kBoxCols * u, q * kBoxRows, &full[slot]);
            else
              tma_load_2d(dst + u * kBoxBytes, &tmX, 0, (2 * q + u) * kBoxRows, &full[slot]);
          }
        }
        // the copies issued have landed before the CTA may exit
        drain_loads(full, kSlots, j, p.err);
      }
    } else if (warp == 1) {
      // ---------------------------------------------- MMA issuer
      if (lane == 0) {
        const uint32_t a_tm = tmem_base + kAcol;
        for (int j = 0;; ++j) {
          const int q = blockIdx.x + j * gridDim.x;
          if (q >= p.num_groups) break;
          const int slot = j % kSlots, region = j % kRegions;
          if (!wait_bounded(&tempty[region], ((uint32_t)(j / kRegions) & 1u) ^ 1u, abort_flag, p.err)) break;
          if (!wait_bounded(&full[slot], (uint32_t)(j / kSlots) & 1u, abort_flag, p.err)) break;
          fence_after();
          const uint32_t d = tmem_base + (uint32_t)(region * 128);
          // B: MN-major, the two boxes are the two 64-column atoms (16 KB
          // apart); 16 chunk rows (2048 bytes) per K=16 step.  A: 8 TMEM
          // columns (16 bf16 per lane) per K=16 step.
          const uint64_t b = sdesc_mn_sw128(smem_u32(sB + slot * kSlotBytes), kBoxBytes);
#pragma unroll
          for (int s = 0; s < 8; ++s) mma_bf16_ts(d, a_tm + 8u * s, b + (uint64_t)(128 * s), s > 0 ? 1u : 0u);
          umma_commit(&empty[slot]);
          umma_commit(&tfull[region]);
        }
        // all MMAs issued by this thread are complete once this commit arrives
        umma_commit(drain);
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < 200000000ull) {
        }
      }
    } else {
      widen_in_idle_warps(p, warp - 2, lane);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kEpiRegs));
    // ------------------------------------------------ epilogue warpgroups
    const int g = (warp - 4) >> 2;    // epilogue warpgroup
    const int quarter = warp & 3;     // its TMEM lane quarter
    const int pr = g >> 1;            // pair: groups j = pr, pr + 2, ...
    const int h = g & 1;              // column half of the group's accumulator
    const int m = quarter * 32 + lane;
    const int bar_wg = 1 + g;
    const int bar_pair = 1 + kEpiGroups + pr;
    constexpr int RT = PAIR ? 256 : KH;          // threads of a token row
    const int bar_row = PAIR ? bar_pair : bar_wg;
    const int bar_row_n = PAIR ? 256 : 128;
    const int wq = PAIR ? 4 * h + quarter : quarter;  // warp number among the row's warps
    const int i_hi = PAIR ? m : m % KH;
    for (int j = pr;; j += 2) {
      const int q = blockIdx.x + j * gridDim.x;
      if (q >= p.num_groups) break;
      const int region = j % kRegions;
      // A wait that gives up does not leave at once: the group runs on (on
      // stale TMEM contents, same addresses, bounded waits) to the row
      // reduction, whose barrier ors the failure over every thread that
      // shares a barrier with this one, and all of them leave there.
      bool failed = !wait_bounded_warp(&tfull[region], (uint32_t)(j / kRegions) & 1u, abort_flag, p.err);
      fence_after();
      const uint32_t tl = tmem_base + (uint32_t)(region * 128) + ((uint32_t)(quarter * 32) << 16);

      float y[64];
      int64_t row;     // token row of this thread's values
      int64_t unit0;   // first chunk row of the box this warpgroup stores (C = 64)
      if constexpr (!PAIR) {
        const int unit = 2 * q + h;
        unit0 = (int64_t)unit * kBoxRows;
        row = (int64_t)unit * (kBoxRows / KH) + m / KH;
        {
          uint32_t u[64];
          tmem_ld32_nowait(tl + (uint32_t)(64 * h), &u[0]);
          tmem_ld32_nowait(tl + (uint32_t)(64 * h + 32), &u[32]);
          tmem_wait_ld();
#pragma unroll
          for (int r = 0; r < 64; ++r) y[r] = __uint_as_float(u[r]);
        }
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[region]);
        // a large row mean sits only in the i_hi = 0 lanes: remove it there
        if (i_hi == 0) {
          const float c0 = y[0];
#pragma unroll
          for (int r = 0; r < 64; r += 2) sub2(y[r], y[r + 1], c0);
        }
        stage<0>(y);
        stage<1>(y);
        stage<2>(y);
        stage<3>(y);
        stage<4>(y);
        stage<5>(y);
        y[0] = i_hi == 0 ? 0.0f : y[0];  // t_0 = 0 (the mean's coefficient)
      } else {
        unit0 = 0;
        row = q;
        {
          uint32_t u[64];
          uint32_t c0w = 0;
          tmem_ld32_nowait(tl + (uint32_t)(64 * h), &u[0]);
          tmem_ld32_nowait(tl + (uint32_t)(64 * h + 32), &u[32]);
          if (h == 1 && quarter == 0) c0w = tmem_ld1(tl);  // column 0 of lane 0 for the mean removal
          tmem_wait_ld();
#pragma unroll
          for (int r = 0; r < 64; ++r) y[r] = __uint_as_float(u[r]);
          if (m == 0) {
            const float c0 = h == 0 ? y[0] : __uint_as_float(c0w);
#pragma unroll
            for (int r = 0; r < 64; r += 2) sub2(y[r], y[r + 1], c0);
          }
        }
        // column bits 0..5
        stage<0>(y);
        stage<1>(y);
        stage<2>(y);
        stage<3>(y);
        stage<4>(y);
        stage<5>(y);
        // Exchange through TMEM: warpgroup 0 keeps columns 0..31 and hands
        // over 32..63; warpgroup 1 keeps 96..127 and hands over 64..95.
        // Column 0 is never rewritten (warpgroup 1 read it above).
        if (h == 0) {
          uint32_t u[32];
#pragma unroll
          for (int r = 0; r < 32; ++r) u[r] = __float_as_uint(y[32 + r]);
          tmem_st32(tl + 32u, u);
        } else {
          uint32_t u[32];
#pragma unroll
          for (int r = 0; r < 32; ++r) u[r] = __float_as_uint(y[r]);
          tmem_st32(tl + 64u, u);
        }
        tmem_wait_st();
        fence_before();
        named_bar_sync(bar_pair, 256);
        fence_after();
        if (h == 0) {
          uint32_t u[32];
          tmem_ld32_nowait(tl + 64u, u);
          tmem_wait_ld();
#pragma unroll
          for (int r = 0; r < 32; ++r) y[32 + r] = __uint_as_float(u[r]);
        } else {
          uint32_t u[32];
          tmem_ld32_nowait(tl + 32u, u);
          tmem_wait_ld();
#pragma unroll
          for (int r = 0; r < 32; ++r) y[r] = __uint_as_float(u[r]);
        }
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[region]);
        // column bit 6: y[r] = column 32h + r, y[32 + r] = column 64 + 32h + r
#pragma unroll
        for (int r = 0; r < 32; r += 2) bfly2(y[r], y[r + 1], y[32 + r], y[33 + r]);
        y[0] = (m == 0 && h == 0) ? 0.0f : y[0];  // t_0 = 0
      }

      // Row statistics.  First reduction: K^2 var = sum_{i>=1} Y_i^2, and for
      // INT8 max |y| (max |t| = fl(cmul max |y|) exactly, rounding being
      // monotone).  INT4 needs sum |t| over t = fl(cmul y) itself, which
      // exists only once cmul is known: a second reduction sums it in double.
      const int rset = 16 * pr + 8 * ((j >> 1) & 1) + (PAIR ? 0 : 4 * h);
      float ss, gmax = 0.0f;
      if constexpr (MODE == K1_Q8_I8) {
        const float2 red = group_reduce2<RT, true>(make_float2(sum_sq64(y), max_abs64(y)), red2 + rset, wq, lane,
                                                   bar_row, bar_row_n, failed);
        ss = red.x;
        gmax = red.y;
      } else {
        ss = group_reduce1<RT>(sum_sq64(y), reinterpret_cast<float*>(red2) + rset, wq, lane, bar_row, bar_row_n,
                               failed);
      }
      if (failed) break;
      const float var = ss * (1.0f / ((float)K * (float)K));
      // 1 / sqrt(K (var + eps)): a correctly rounded reciprocal square root
      // (one rounding) times 1/sqrt(K); the debug and quantizing modes share it
      const float cmul = __fmul_rn(__frsqrt_rn(__fadd_rn(var, 1e-5f)), p.sK);
      const bool row_ok = row < p.M;
      // this thread's chunk row: C = 64, unit row m; C = 128, tile row m
      const int64_t crow = (PAIR ? (int64_t)q * kBoxRows : unit0) + m;
      // t = fl(cmul y) in place: the transform output every mode starts from
#pragma unroll
      for (int r = 0; r < 64; r += 2) mul2(y[r], y[r + 1], cmul);

      if constexpr (MODE == K1_T_F32) {
        if (row_ok) {
          float* trow = p.t_out + (size_t)row * K;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            // C = 64: columns 64 i_hi + 32 half + r; C = 128: 128 i_hi + 64 half + 32 h + r
            const size_t col = PAIR ? (size_t)i_hi * 128 + 64 * half + 32 * h : (size_t)i_hi * 64 + 32 * half;
            float4* dst = reinterpret_cast<float4*>(trow + col);
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
              const int r = 32 * half + 4 * jj;
              dst[jj] = make_float4(y[r], y[r + 1], y[r + 2], y[r + 3]);
            }
          }
        }
      } else {
        q::RowParams qp;
        if constexpr (MODE == K1_Q8_I8) {
          qp = q::params_int8(__fmul_rn(cmul, gmax));
        } else {
          // second reduction: beta = (float)(sum |t| / K) from a double sum, as the
          // quantizer-only kernel computes it; the sum is scaled by 2^-896,
          // so one multiply by 2^(896 - log2 K) gives the mean exactly
          const double sa = group_reduce_d<RT>(sum_abs64_scaled(y), redd + rset, wq, lane, bar_row, bar_row_n);
          qp = q::params_int4_mean(sa * (q::kUnscaleAbs * q::pow2_recip(LOGK)));
        }
        const float cq = qp.r;  // codes are rint(t r)
        if (row_ok && i_hi == 0 && (!PAIR || h == 0)) p.scales[row] = qp.scale();
        if (row_ok) {
          uint8_t* crow_out = p.codes + crow * (MODE == K1_Q4_PACKED ? C / 2 : C);
          if constexpr (MODE == K1_Q4_PACKED) {
            // 32 codes (16 bytes) per half: C = 64 at bytes 0 and 16 of the
            // 32-byte chunk row; C = 128 at 16h and 32 + 16h of 64 bytes
            uint4* d0 = reinterpret_cast<uint4*>(crow_out + (PAIR ? 16 * h : 0));
            uint4* d1 = reinterpret_cast<uint4*>(crow_out + (PAIR ? 32 + 16 * h : 16));
            *d0 = codes32_s4(&y[0], cq);
            *d1 = codes32_s4(&y[32], cq);
          } else {
            // 16 codes per 16 bytes: C = 64 at 0, 16, 32, 48; C = 128 at
            // 32h, 32h + 16, 64 + 32h, 80 + 32h
            // ||t||^2 = cmul^2 ss (up to the roundings of t), so every
            // |t r| < 3e4 when cmul^2 r^2 ss < 9e8
            const float cr = cmul * cq;
            const bool s16 = MODE == K1_Q4_I8 && ss * cr * cr < 9.0e8f;
            if (PAIR && p.codes_al32) {
              // two whole 32-byte sectors per thread, not four half sectors
#pragma unroll
              for (int c = 0; c < 4; c += 2) {
                const uint4 v0 = s16 ? codes16_i8<MODE, true>(&y[16 * c], cq) : codes16_i8<MODE>(&y[16 * c], cq);
                const uint4 v1 =
                    s16 ? codes16_i8<MODE, true>(&y[16 * c + 16], cq) : codes16_i8<MODE>(&y[16 * c + 16], cq);
                st_global_32B(crow_out + (c == 0 ? 32 * h : 64 + 32 * h), v0, v1);
              }
            } else {
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                const int off = PAIR ? (c < 2 ? 32 * h + 16 * c : 64 + 32 * h + 16 * (c - 2)) : 16 * c;
                const uint4 v = s16 ? codes16_i8<MODE, true>(&y[16 * c], cq) : codes16_i8<MODE>(&y[16 * c], cq);
                *reinterpret_cast<uint4*>(crow_out + off) = v;
              }
            }
          }
        }
      }
    }
  }

  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// ---------------------------------------------------------------- K = 32768
// 256-column chunks (KH = 128, so the high factor is still H_128): a tile is
// one token row, 128 chunk rows x 256 columns = four 64-column boxes (64 KB),
// and one N = 256 MMA per K step.  A (H_128 in bf16) stays in shared memory
// so that TMEM holds two 256-column accumulators (the MMA of the next tile
// overlaps this tile's epilogue).  All four epilogue warpgroups share each
// tile: warpgroup g loads columns 64 g .. 64 g + 63 of its lanes and runs
// the 6 low stages; two exchange rounds through TMEM, each behind a barrier
// of the two warpgroups involved, bring the partners of column bit 6 and
// then of bit 7 together.  In 32-column units u (columns 32 u ..), warpgroup
// g starts with units {2g, 2g+1}, holds {0,2} {1,3} {4,6} {5,7} after
// exchange 1 and the final outputs {g, g+4} after exchange 2.  Every exchange write goes
// to a unit nobody reads again except its receiver, and unit 0 (whose first
// column the i_hi = 0 lanes of every warpgroup read for the mean removal) is
// never written.
constexpr int k256Cols = 256;
constexpr int k256TileBytes = 4 * kBoxBytes;  // 64 KB
constexpr int k256Slots = 2;
constexpr int k256ABytes = 128 * 128 * 2;
constexpr size_t k256SmemBytes = 1024 + (size_t)k256ABytes + (size_t)k256Slots * k256TileBytes + 1024;
// kind::f16: D f32, A and B bf16, A K-major, B MN-major, N = 256, M = 128
constexpr uint32_t kIdesc256 =
    (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((256u >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(kIdesc256), "r"(accumulate));
}

// H_128 as bf16 in the K-major 128B-swizzled layout: two 64-column blocks of
// 128 rows x 128 bytes; 16-byte chunk c of row m at chunk position c ^ (m & 7).
__device__ __forceinline__ void build_h128_smem(uint8_t* sA, int tid, int nthreads) {
  for (int c = tid; c < 2048; c += nthreads) {
    const int blk = c >> 10, m = (c >> 3) & 127, cc = c & 7;
    uint32_t w[4];
#pragma unroll
    for (int u = 0; u < 8; u += 2) {
      uint32_t hv[2];
#pragma unroll
      for (int v = 0; v < 2; ++v) {
        const int k = blk * 64 + cc * 8 + u + v;
        hv[v] = 0x3F80u ^ ((uint32_t)(__popc(m & k) & 1) << 15);
      }
      w[u >> 1] = hv[0] | (hv[1] << 16);
    }
    *reinterpret_cast<uint4*>(sA + blk * 16384 + m * 128 + ((cc ^ (m & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// 32 TMEM columns from registers r[0..31] / into them
__device__ __forceinline__ void tm_put32(uint32_t taddr, const float* r) {
  uint32_t u[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(r[i]);
  tmem_st32(taddr, u);
}
__device__ __forceinline__ void tm_get32(uint32_t taddr, float* r) {
  uint32_t u[32];
  tmem_ld32_nowait(taddr, u);
  tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 32; ++i) r[i] = __uint_as_float(u[i]);
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
ln_fht_quant_tc256_kernel(const __grid_constant__ CUtensorMap tmX, TcParams p) {
  constexpr int K = 32768;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = base;
  uint8_t* sB = sA + k256ABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + k256Slots * k256TileBytes);
  uint64_t* empty = full + k256Slots;
  uint64_t* tfull = empty + k256Slots;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  float2* red2 = reinterpret_cast<float2*>(drain + 1);  // [tile parity][16 warps]
  double* redd = reinterpret_cast<double*>(red2 + 32);  // the same for the INT4 double sums
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(redd + 32);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s2 = 0; s2 < k256Slots; ++s2) {
      mbar_init(&full[s2], 1);
      mbar_init(&empty[s2], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 16);  // every epilogue warp reads every tile
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  if (warp >= 4) {
    build_h128_smem(sA, threadIdx.x - 128, kThreads - 128);
    fence_proxy_async_smem();
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem_base = *tmem_slot;
  asm volatile("griddepcontrol.wait;" ::: "memory");  // as in ln_fht_quant_tc_kernel
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtrlRegs));
    if (warp == 0) {
      if (lane == 0) {
        prefetch_tensormap(&tmX);
        int j = 0;  // tiles issued
        for (;; ++j) {
          const int q = blockIdx.x + j * gridDim.x;
          if (q >= p.num_groups) break;
          const int slot = j % k256Slots;
          if (!wait_bounded(&empty[slot], ((uint32_t)(j / k256Slots) & 1u) ^ 1u, abort_flag, p.err)) break;
          mbar_expect_tx(&full[slot], (uint32_t)k256TileBytes);
#pragma unroll
          for (int u = 0; u < 4; ++u)
            tma_load_2d(sB + slot * k256TileBytes + u * kBoxBytes, &tmX, kBoxCols * u, q * kBoxRows, &full[slot]);
        }
        drain_loads(full, k256Slots, j, p.err);
      }
    } else if (warp == 1) {
      if (lane == 0) {
        const uint32_t a_addr = smem_u32(sA);
        for (int j = 0;; ++j) {
          const int q = blockIdx.x + j * gridDim.x;
          if (q >= p.num_groups) break;
          const int slot = j % k256Slots, region = j & 1;
          if (!wait_bounded(&tempty[region], ((uint32_t)(j >> 1) & 1u) ^ 1u, abort_flag, p.err)) break;
          if (!wait_bounded(&full[slot], (uint32_t)(j / k256Slots) & 1u, abort_flag, p.err)) break;
          fence_after();
          const uint32_t d = tmem_base + (uint32_t)(region * k256Cols);
          // B: four 64-column atoms 16 KB apart, 2048 bytes per K=16 step
          const uint64_t b = sdesc_mn_sw128(smem_u32(sB + slot * k256TileBytes), kBoxBytes);
#pragma unroll
          for (int s2 = 0; s2 < 8; ++s2) {
            const uint64_t a = sdesc_k_sw128(a_addr + (uint32_t)((s2 >> 2) * 16384)) + (uint64_t)(2 * (s2 & 3));
            mma_bf16_ss(d, a, b + (uint64_t)(128 * s2), s2 > 0 ? 1u : 0u);
          }
          umma_commit(&empty[slot]);
          umma_commit(&tfull[region]);
        }
        umma_commit(drain);
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < 200000000ull) {
        }
      }
    } else {
      widen_in_idle_warps(p, warp - 2, lane);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kEpiRegs));
    const int g = (warp - 4) >> 2;    // epilogue warpgroup: starting columns 64 g ..
    const int quarter = warp & 3;
    const int m = quarter * 32 + lane;  // lane = i_hi
    const int wq = 4 * g + quarter;
    const int h1 = g & 1;               // role in exchange 1 (pairs {0,1}, {2,3})
    const int bar_r1 = 1 + (g >> 1);
    const int bar_r2 = 3 + (g & 1);     // exchange 2 pairs {0,2}, {1,3}
    const int bar_row = 5;
    // exchange 2: location written, location read, and whether the kept 32
    // values are y[0..31] (else y[32..63])
    const int w2 = g == 0 ? 3 : g == 1 ? 1 : g == 2 ? 4 : 7;
    const int r2 = g == 0 ? 4 : g == 1 ? 7 : g == 2 ? 3 : 1;
    const bool keep_lo2 = g < 2;
    for (int j = 0;; ++j) {
      const int q = blockIdx.x + j * gridDim.x;
      if (q >= p.num_groups) break;
      const int region = j & 1;
      bool failed = !wait_bounded_warp(&tfull[region], (uint32_t)(j >> 1) & 1u, abort_flag, p.err);
      fence_after();
      const uint32_t tl = tmem_base + (uint32_t)(region * k256Cols) + ((uint32_t)(quarter * 32) << 16);

      float y[64];
      {
        uint32_t u[64];
        uint32_t c0w = 0;
        tmem_ld32_nowait(tl + (uint32_t)(64 * g), &u[0]);
        tmem_ld32_nowait(tl + (uint32_t)(64 * g + 32), &u[32]);
        if (g > 0 && quarter == 0) c0w = tmem_ld1(tl);  // column 0 of lane 0 for the mean removal
        tmem_wait_ld();
#pragma unroll
        for (int r = 0; r < 64; ++r) y[r] = __uint_as_float(u[r]);
        if (m == 0) {
          const float c0 = g == 0 ? y[0] : __uint_as_float(c0w);
#pragma unroll
          for (int r = 0; r < 64; r += 2) sub2(y[r], y[r + 1], c0);
        }
      }
      stage<0>(y);
      stage<1>(y);
      stage<2>(y);
      stage<3>(y);
      stage<4>(y);
      stage<5>(y);
      // exchange 1 (column bit 6): units 2g, 2g+1 -> {4(g>>1) + h1, 4(g>>1) + h1 + 2}
      if (h1 == 0) tm_put32(tl + (uint32_t)(64 * g + 32), &y[32]);  // hand over unit 2g+1
      else tm_put32(tl + (uint32_t)(64 * g), &y[0]);                 // hand over unit 2g
      tmem_wait_st();
      fence_before();
      named_bar_sync(bar_r1, 256);
      fence_after();
      if (h1 == 0) tm_get32(tl + (uint32_t)(64 * g + 64), &y[32]);   // partner's unit 2g+2
      else tm_get32(tl + (uint32_t)(64 * g - 32), &y[0]);            // partner's unit 2g-1
#pragma unroll
      for (int r = 0; r < 32; r += 2) bfly2(y[r], y[r + 1], y[32 + r], y[33 + r]);
      // exchange 2 (column bit 7)
      if (keep_lo2) tm_put32(tl + (uint32_t)(32 * w2), &y[32]);
      else tm_put32(tl + (uint32_t)(32 * w2), &y[0]);
      tmem_wait_st();
      fence_before();
      named_bar_sync(bar_r2, 256);
      fence_after();
      if (keep_lo2) tm_get32(tl + (uint32_t)(32 * r2), &y[32]);
      else tm_get32(tl + (uint32_t)(32 * r2), &y[0]);
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[region]);
#pragma unroll
      for (int r = 0; r < 32; r += 2) bfly2(y[r], y[r + 1], y[32 + r], y[33 + r]);
      // now y[r] = column 32 g + r, y[32 + r] = column 128 + 32 g + r
      y[0] = (m == 0 && g == 0) ? 0.0f : y[0];  // t_0 = 0

      // the two statistic rounds of ln_fht_quant_tc_kernel, over all 512
      // epilogue threads
      const int rset = 16 * (j & 1);
      float ss, gmax = 0.0f;
      if constexpr (MODE == K1_Q8_I8) {
        const float2 red = group_reduce2<512, true>(make_float2(sum_sq64(y), max_abs64(y)), red2 + rset, wq, lane,
                                                    bar_row, 512, failed);
        ss = red.x;
        gmax = red.y;
      } else {
        ss = group_reduce1<512>(sum_sq64(y), reinterpret_cast<float*>(red2) + rset, wq, lane, bar_row, 512, failed);
      }
      if (failed) break;
      const float var = ss * (1.0f / ((float)K * (float)K));
      const float cmul = __fmul_rn(__frsqrt_rn(__fadd_rn(var, 1e-5f)), p.sK);
      const int64_t row = q;
      const int64_t crow = (int64_t)q * kBoxRows + m;
#pragma unroll
      for (int r = 0; r < 64; r += 2) mul2(y[r], y[r + 1], cmul);  // t = fl(cmul y)

      if constexpr (MODE == K1_T_F32) {
        float* trow = p.t_out + (size_t)row * K + (size_t)m * k256Cols;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          float4* dst = reinterpret_cast<float4*>(trow + 128 * half + 32 * g);
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const int r = 32 * half + 4 * jj;
            dst[jj] = make_float4(y[r], y[r + 1], y[r + 2], y[r + 3]);
          }
        }
      } else {
        q::RowParams qp;
        if constexpr (MODE == K1_Q8_I8)
          qp = q::params_int8(__fmul_rn(cmul, gmax));
        else
          qp = q::params_int4_mean(group_reduce_d<512>(sum_abs64_scaled(y), redd + rset, wq, lane, bar_row, 512) *
                                   (q::kUnscaleAbs * q::pow2_recip(15)));
        const float cq = qp.r;
        if (m == 0 && g == 0) p.scales[row] = qp.scale();
        uint8_t* crow_out = p.codes + crow * (MODE == K1_Q4_PACKED ? k256Cols / 2 : k256Cols);
        if constexpr (MODE == K1_Q4_PACKED) {
          // 32 codes (16 bytes) per half, at bytes 16 g and 64 + 16 g
          *reinterpret_cast<uint4*>(crow_out + 16 * g) = codes32_s4(&y[0], cq);
          *reinterpret_cast<uint4*>(crow_out + 64 + 16 * g) = codes32_s4(&y[32], cq);
        } else {
          const float cr = cmul * cq;
          const bool s16 = MODE == K1_Q4_I8 && ss * cr * cr < 9.0e8f;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const uint4 v0 = s16 ? codes16_i8<MODE, true>(&y[32 * half], cq) : codes16_i8<MODE>(&y[32 * half], cq);
            const uint4 v1 =
                s16 ? codes16_i8<MODE, true>(&y[32 * half + 16], cq) : codes16_i8<MODE>(&y[32 * half + 16], cq);
            uint8_t* dst = crow_out + 128 * half + 32 * g;
            if (p.codes_al32) {
              st_global_32B(dst, v0, v1);
            } else {
              reinterpret_cast<uint4*>(dst)[0] = v0;
              reinterpret_cast<uint4*>(dst)[1] = v1;
            }
          }
        }
      }
    }
  }

  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

struct WidenJob {
  const uint32_t* packed = nullptr;
  uint4* out = nullptr;
  int64_t words = 0;
};

template <int LOGK, int MODE>
cudaError_t launch_tc(const void* x, int64_t M, void* out, float* scales, int* err, const WidenJob& wjob,
                      cudaStream_t stream) {
  constexpr int C = LOGK >= 14 ? 128 : 64;
  constexpr int KH = (1 << LOGK) / C;
  constexpr bool PAIR = C == 128;
  const int64_t nchunk = M * KH;
  const int64_t groups = PAIR ? nchunk / kBoxRows : (nchunk + 2 * kBoxRows - 1) / (2 * kBoxRows);
  if (groups > (int64_t)INT32_MAX / 4 || nchunk > (int64_t)INT32_MAX / 2) return cudaErrorInvalidValue;
  CUtensorMap tmX;
  if (!sm100_host::encode_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, C, (uint64_t)nchunk, C * 2, kBoxCols,
                             kBoxRows, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  TcParams p;
  p.M = M;
  p.nchunk = nchunk;
  p.num_groups = (int)groups;
  p.sK = (float)(1.0 / sqrt((double)(1 << LOGK)));
  p.t_out = reinterpret_cast<float*>(out);
  p.codes = reinterpret_cast<uint8_t*>(out);
  p.codes_al32 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0;
  p.wpacked = wjob.packed;
  p.wout = wjob.out;
  p.wwords = wjob.words;
  p.scales = scales;
  p.err = err;
  auto kern = ln_fht_quant_tc_kernel<LOGK, MODE>;
  // setmaxnreg.inc waits until the registers it asks for are free in the
  // block's own allocation: never launch a split the launch count cannot cover
  static const bool split_ok = [&]() {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return false;
    return (int64_t)fa.numRegs * kThreads >= (int64_t)128 * kCtrlRegs + (int64_t)128 * kEpiGroups * kEpiRegs;
  }();
  if (!split_ok) return cudaErrorInvalidConfiguration;
  static std::atomic<bool> smem_set[sm100_host::kMaxDevices];
  cudaError_t e = sm100_host::ensure_smem(kern, (int)kSmemBytes, smem_set);
  if (e != cudaSuccess) return e;
  const int nsm = sm100_host::sm_count();
  const int grid = p.num_groups < nsm ? p.num_groups : nsm;
  return sm100_host::launch_pdl(kern, (unsigned)grid, kThreads, kSmemBytes, stream, 1, tmX, p);
}

template <int MODE>
cudaError_t launch_tc256(const void* x, int64_t M, void* out, float* scales, int* err, const WidenJob& wjob,
                         cudaStream_t stream) {
  const int64_t nchunk = M * 128;
  if (M > (int64_t)INT32_MAX / 4) return cudaErrorInvalidValue;
  CUtensorMap tmX;
  if (!sm100_host::encode_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, k256Cols, (uint64_t)nchunk, k256Cols * 2,
                             kBoxCols, kBoxRows, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  TcParams p;
  p.M = M;
  p.nchunk = nchunk;
  p.num_groups = (int)M;
  p.sK = (float)(1.0 / sqrt(32768.0));
  p.t_out = reinterpret_cast<float*>(out);
  p.scales = scales;
  p.err = err;
  p.codes = reinterpret_cast<uint8_t*>(out);
  p.codes_al32 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0;
  p.wpacked = wjob.packed;
  p.wout = wjob.out;
  p.wwords = wjob.words;
  auto kern = ln_fht_quant_tc256_kernel<MODE>;
  static const bool split_ok = [&]() {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return false;
    return (int64_t)fa.numRegs * kThreads >= (int64_t)128 * kCtrlRegs + (int64_t)128 * kEpiGroups * kEpiRegs;
  }();
  if (!split_ok) return cudaErrorInvalidConfiguration;
  static std::atomic<bool> smem_set[sm100_host::kMaxDevices];
  cudaError_t e = sm100_host::ensure_smem(kern, (int)k256SmemBytes, smem_set);
  if (e != cudaSuccess) return e;
  const int nsm = sm100_host::sm_count();
  const int grid = p.num_groups < nsm ? p.num_groups : nsm;
  return sm100_host::launch_pdl(kern, (unsigned)grid, kThreads, k256SmemBytes, stream, 1, tmX, p);
}

template <int LOGK>
cudaError_t launch_tc_mode(const void* x, int64_t M, K1Mode mode, void* out, float* scales, int* err,
                           const WidenJob& w, cudaStream_t s) {
  if constexpr (LOGK == 15) {
    switch (mode) {
      case K1_T_F32: return launch_tc256<K1_T_F32>(x, M, out, scales, err, w, s);
      case K1_Q4_PACKED: return launch_tc256<K1_Q4_PACKED>(x, M, out, scales, err, w, s);
      case K1_Q4_I8: return launch_tc256<K1_Q4_I8>(x, M, out, scales, err, w, s);
      case K1_Q8_I8: return launch_tc256<K1_Q8_I8>(x, M, out, scales, err, w, s);
      default: return cudaErrorInvalidValue;
    }
  } else {
    switch (mode) {
      case K1_T_F32: return launch_tc<LOGK, K1_T_F32>(x, M, out, scales, err, w, s);
      case K1_Q4_PACKED: return launch_tc<LOGK, K1_Q4_PACKED>(x, M, out, scales, err, w, s);
      case K1_Q4_I8: return launch_tc<LOGK, K1_Q4_I8>(x, M, out, scales, err, w, s);
      case K1_Q8_I8: return launch_tc<LOGK, K1_Q8_I8>(x, M, out, scales, err, w, s);
      default: break;
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool ln_fht_quant_tc_supports(bool in_bf16, int log2k, K1Mode mode, const void* x, const void* out) {
  return in_bf16 && log2k >= 7 && log2k <= 15 && mode != K1_FHT_F32 && mode != K1_LNBWD &&
         (reinterpret_cast<uintptr_t>(x) & 15u) == 0 && (reinterpret_cast<uintptr_t>(out) & 15u) == 0;
}

namespace {

cudaError_t launch_tc_any(const void* x, int64_t M, int log2k, K1Mode mode, void* out, float* scales,
                          const WidenJob& w, cudaStream_t stream) {
  if (M <= 0) return cudaSuccess;
  int* err = device_error_word();
  if (!err) return cudaErrorInvalidValue;
  switch (log2k) {
    case 7: return launch_tc_mode<7>(x, M, mode, out, scales, err, w, stream);
    case 8: return launch_tc_mode<8>(x, M, mode, out, scales, err, w, stream);
    case 9: return launch_tc_mode<9>(x, M, mode, out, scales, err, w, stream);
    case 10: return launch_tc_mode<10>(x, M, mode, out, scales, err, w, stream);
    case 11: return launch_tc_mode<11>(x, M, mode, out, scales, err, w, stream);
    case 12: return launch_tc_mode<12>(x, M, mode, out, scales, err, w, stream);
    case 13: return launch_tc_mode<13>(x, M, mode, out, scales, err, w, stream);
    case 14: return launch_tc_mode<14>(x, M, mode, out, scales, err, w, stream);
    case 15: return launch_tc_mode<15>(x, M, mode, out, scales, err, w, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_ln_fht_quant_tc(const void* x, int64_t M, int log2k, K1Mode mode, void* out, float* scales,
                                   cudaStream_t stream) {
  return launch_tc_any(x, M, log2k, mode, out, scales, WidenJob(), stream);
}

cudaError_t launch_ln_fht_quant_tc_widen(const void* x, int64_t M, int log2k, K1Mode mode, void* out,
                                         float* scales, const uint8_t* packed, int64_t N, int64_t K, int8_t* w,
                                         cudaStream_t stream) {
  // The widening needs every SM's idle warps, and enough quantizer work to
  // hide behind: with fewer CTAs than SMs, or when the weights' traffic
  // (1.25 bytes per code) is not well below the quantizer's (3 bytes per
  // element), it runs as its own kernel beside the quantizer instead.
  const int64_t ctas = log2k >= 14 ? M : (M * ((int64_t)1 << (log2k - 6)) + 2 * kBoxRows - 1) / (2 * kBoxRows);
  if (M <= 0 || ctas < sm100_host::sm_count() || 3 * M < 5 * N) {
    cudaError_t e = launch_tc_any(x, M, log2k, mode, out, scales, WidenJob(), stream);
    if (e == cudaSuccess) e = launch_widen_ternary(packed, N, K, w, stream, /*overlap_previous=*/true);
    return e;
  }
  WidenJob job;
  job.packed = reinterpret_cast<const uint32_t*>(packed);
  job.out = reinterpret_cast<uint4*>(w);
  job.words = N * K / 16;
  return launch_tc_any(x, M, log2k, mode, out, scales, job, stream);
}

}  // namespace hbl
