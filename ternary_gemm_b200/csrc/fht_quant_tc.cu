// Fused LayerNorm -> fast Walsh-Hadamard transform -> per-token quantization
// with the transform split between the tensor cores and the FMA pipe
// ("BitNet v2: Native 4-bit Activations with Hadamard Transformation for
// 1-bit LLMs", section "H-BitLinear": the Hadamard-transform definition and
// the activation-quantization formula).  bf16 input, K = 128 .. 16384.
//
// Sylvester's matrix factors over the index bits: with i = 128 i_hi + i_lo,
// j = 128 j_hi + j_lo and KH = K / 128,
//   H_K[i][j] = H_KH[i_hi][j_hi] * H_128[i_lo][j_lo],
// so Y = H_K x is two smaller transforms.  The high one is a dense
// contraction whose operands are exact in bf16 (x itself and +-1), so it runs
// on the tensor cores; the low one (7 butterfly stages) runs in registers:
//
//   x viewed as chunk rows Xc[M*KH][128] (row-major, no copy);
//   tile    = 128 consecutive chunk rows = 128/KH token rows;
//   MMA     D[m][n] = sum_k A[m][k] Xc[tile*128 + k][n],
//           A = blockdiag(H_KH, ..., H_KH) (128 x 128, bf16 +-1/0),
//           tcgen05.mma kind::f16, M = N = 128, K = 16 x 8, f32 in TMEM;
//           lane m = (token row r = m / KH, i_hi = m % KH), column n = j_lo;
//   thread  m loads its 128 columns (one TMEM lane), runs the 7 stages over
//           j_lo in registers and owns Y[r][128 i_hi .. 128 i_hi + 127],
//           a contiguous slice of the transformed row.
// The tensor-core sums are exact whenever the 128 bf16 terms span < 2^9 in
// magnitude (their common unit in the last place then divides the result),
// and otherwise round in float like the butterflies would.
//
// LayerNorm is folded around the transform as in the register kernel: row 0
// of H is all ones, so sum_{i>=1} Y_i^2 = K^2 var and t_i = Y_i / sqrt(K (var
// + eps_ln)) for i >= 1, t_0 = 0.  A large row mean only reaches the lanes
// with i_hi = 0 (the other rows of H_KH sum to zero); those subtract their own
// column-0 value from all 128 columns before the butterflies, which changes
// only Y_0 (discarded) and keeps the float sums on the deviations.
//
// CTA (one per SM, persistent over tiles), three warpgroups:
//   warp 0     TMA producer: two 64-element-wide 128B-swizzled boxes per
//              tile (the MN-major B operand) into a 4-stage ring;
//   warp 1     TMEM allocation (4 accumulators x 128 columns) and one thread
//              issuing the 8 MMAs of a tile;
//   warps 2-3  idle (registers are granted to whole warpgroups);
//   warps 4-11 two epilogue warpgroups taking alternate tiles: TMEM -> 128
//              registers, butterflies, LayerNorm statistics, quantizer, codes
//              into a swizzled staging tile that one TMA store writes out
//              (the tile's codes are contiguous in the output).
// Registers are allocated for 4-warp groups, so the block is launched with
// 168 per thread and rebalanced with setmaxnreg: the first warpgroup gives
// its share down to 40, the epilogue warpgroups take 208 each (the host
// checks that the launch count covers this split before launching).
// Every mbarrier wait is bounded (2 s, then the CTA abort flag and the device
// error word are set and every role leaves its loop).
#include <cstdint>

#include "common.cuh"
#include "quant.cuh"
#include "rowkit.cuh"
#include "sm100.cuh"

namespace hbl {
namespace {

using namespace sm100;
using namespace rowkit;

constexpr int kTileChunks = 128;                      // chunk rows per tile (MMA K)
constexpr int kTileBytes = kTileChunks * 128 * 2;     // 32 KB of bf16
constexpr int kStages = 4;
constexpr int kABytes = 128 * 128 * 2;                // blockdiag(H_KH) in bf16
constexpr int kOutBytes = kTileChunks * 128;          // int8 codes of a tile
constexpr int kEpiGroups = 2;
constexpr int kThreads = 128 + 128 * kEpiGroups;
constexpr int kCtrlRegs = 40;   // registers per thread of the first warpgroup after setmaxnreg
constexpr int kEpiRegs = 208;   // registers per thread of an epilogue warpgroup after setmaxnreg
constexpr int kAcc = 4;
constexpr uint32_t kTmemCols = 128 * kAcc;
constexpr size_t kSmemBytes = 1024 + kABytes + (size_t)kStages * kTileBytes + kEpiGroups * kOutBytes + 512;

// instruction descriptor, kind::f16: D f32, A and B bf16, A K-major, B
// MN-major, N = 128, M = 128
constexpr uint32_t kIdesc =
    (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

struct TcParams {
  int64_t M;         // token rows
  int num_tiles;     // ceil(M * KH / 128)
  float sK;          // 1 / sqrt(K) rounded to float
  float* t_out;      // K1_T_F32: t [M][K]
  float* scales;     // [M]
  int* err;          // device error word
};

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(kIdesc), "r"(accumulate));
}

// Butterfly over register-index bit B of a 128-float array.
template <int B>
__device__ __forceinline__ void stage128(float (&e)[128]) {
  if constexpr (B == 0) {
#pragma unroll
    for (int r = 0; r < 128; r += 2) {
      const float a = e[r], c = e[r + 1];
      e[r] = a + c;
      e[r + 1] = a - c;
    }
  } else {
#pragma unroll
    for (int r = 0; r < 128; r += 2)
      if (!(r & (1 << B))) bfly2(e[r], e[r + 1], e[r | (1 << B)], e[(r | (1 << B)) + 1]);
  }
}

// All-reduce over the KH consecutive TMEM lanes (threads) of one token row.
// Every thread of the row ends with the identical value.  Rows wider than a
// warp combine warp partials through `slots` behind the warpgroup's barrier.
template <int KH, typename V, typename Op>
__device__ __forceinline__ V group_reduce(V v, Op op, V* slots, int quarter, int lane, int bar_id) {
  constexpr int W = KH < 32 ? KH : 32;
#pragma unroll
  for (int o = W / 2; o >= 1; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  if constexpr (KH > 32) {
    if (lane == 0) slots[quarter] = v;
    named_bar_sync(bar_id, 128);
    if constexpr (KH == 128)
      v = op(op(slots[0], slots[1]), op(slots[2], slots[3]));
    else
      v = op(slots[quarter & 2], slots[(quarter & 2) | 1]);
  }
  return v;
}

// blockdiag(H_KH) as bf16 in the K-major 128B-swizzled layout: two 64-column
// blocks of 128 rows x 128 bytes; 16-byte chunk c of row m sits at chunk
// position c ^ (m & 7).
template <int KH>
__device__ __forceinline__ void build_a(uint8_t* sA, int tid, int nthreads) {
  for (int c = tid; c < 2048; c += nthreads) {
    const int blk = c >> 10, m = (c >> 3) & 127, cc = c & 7;
    uint32_t w[4];
#pragma unroll
    for (int u = 0; u < 8; u += 2) {
      uint32_t h[2];
#pragma unroll
      for (int v = 0; v < 2; ++v) {
        const int k = blk * 64 + cc * 8 + u + v;
        const bool same = (m / KH) == (k / KH);
        h[v] = !same ? 0u : ((__popc((m % KH) & (k % KH)) & 1) ? 0xBF80u : 0x3F80u);
      }
      w[u >> 1] = h[0] | (h[1] << 16);
    }
    *reinterpret_cast<uint4*>(sA + blk * 16384 + m * 128 + ((cc ^ (m & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

template <int LOGK, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
ln_fht_quant_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmOut,
                       TcParams p) {
  constexpr int K = 1 << LOGK;
  constexpr int KH = K / 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = base;
  uint8_t* sB = sA + kABytes;
  uint8_t* sOut = sB + kStages * kTileBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sOut + kEpiGroups * kOutBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + kAcc;
  uint64_t* drain = tempty + kAcc;
  double* red_d = reinterpret_cast<double*>(drain + 1);     // [kEpiGroups][4]
  float* red_f = reinterpret_cast<float*>(red_d + 4 * kEpiGroups);  // [kEpiGroups][4]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(red_f + 4 * kEpiGroups);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < kAcc; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  if (warp >= 4) {
    build_a<KH>(sA, threadIdx.x - 128, kThreads - 128);
    fence_proxy_async_smem();
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtrlRegs));
  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tmX);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
        if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.err)) { ok = false; break; }
        mbar_expect_tx(&full[stage], (uint32_t)kTileBytes);
        uint8_t* dst = sB + stage * kTileBytes;
        tma_load_2d(dst, &tmX, 0, tile * kTileChunks, &full[stage]);
        tma_load_2d(dst + kTileBytes / 2, &tmX, 64, tile * kTileChunks, &full[stage]);
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) {
        // give the copies already issued time to land before the CTA exits
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 20000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      const uint32_t a_addr = smem_u32(sA);
      for (int it = 0, tile = blockIdx.x; tile < p.num_tiles; ++it, tile += gridDim.x) {
        const int acc = it & (kAcc - 1);
        const uint32_t acc_phase = (uint32_t)(it / kAcc) & 1u;
        if (!wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, p.err)) break;
        if (!wait_bounded(&full[stage], phase, abort_flag, p.err)) break;
        fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * 128);
        const uint64_t b0 = sdesc_mn_sw128(smem_u32(sB + stage * kTileBytes), kTileBytes / 2);
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          // A: K-major, 32 bytes per K=16 step inside a 64-column block
          const uint64_t a = sdesc_k_sw128(a_addr + (uint32_t)((s >> 2) * 16384)) + (uint64_t)(2 * (s & 3));
          // B: MN-major, 16 chunk rows (2048 bytes) per K=16 step
          mma_bf16(d_tmem, a, b0 + (uint64_t)(128 * s), s > 0 ? 1u : 0u);
        }
        umma_commit(&empty[stage]);
        umma_commit(&tfull[acc]);
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
      // all MMAs issued by this thread are complete once this commit arrives
      umma_commit(drain);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < 200000000ull) {
      }
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kEpiRegs));
    // ------------------------------------------------ epilogue warpgroups
    const int grp = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int m = quarter * 32 + lane;  // TMEM lane = (token row in tile, i_hi)
    const int r_loc = m / KH;
    const int i_hi = m % KH;
    const int bar_id = 1 + grp;
    const bool issuer = (warp == 4 + 4 * grp) && lane == 0;
    uint8_t* stg = sOut + grp * kOutBytes;
    double* slot_d = red_d + 4 * grp;
    float* slot_f = red_f + 4 * grp;
    for (int it = grp, tile = blockIdx.x + grp * gridDim.x; tile < p.num_tiles;
         it += kEpiGroups, tile += kEpiGroups * gridDim.x) {
      const int acc = it & (kAcc - 1);
      const uint32_t acc_phase = (uint32_t)(it / kAcc) & 1u;
      // the previous TMA store of this group has finished reading the staging tile
      if (issuer) bulk_wait_read_all();
      int ok = 1;
      if (lane == 0) ok = wait_bounded(&tfull[acc], acc_phase, abort_flag, p.err) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (named_bar_any(bar_id, 128, ok == 0)) break;
      fence_after();

      float y[128];
      {
        const uint32_t taddr = tmem_base + (uint32_t)(acc * 128) + ((uint32_t)(quarter * 32) << 16);
        uint32_t u[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32_nowait(taddr + (uint32_t)(32 * c), &u[32 * c]);
        tmem_wait_ld();
#pragma unroll
        for (int r = 0; r < 128; ++r) y[r] = __uint_as_float(u[r]);
      }
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);

      // a large row mean sits only in the i_hi = 0 lanes: remove it there
      if (i_hi == 0) {
        const float c0 = y[0];
#pragma unroll
        for (int r = 0; r < 128; r += 2) sub2(y[r], y[r + 1], c0);
      }
      stage128<0>(y);
      stage128<1>(y);
      stage128<2>(y);
      stage128<3>(y);
      stage128<4>(y);
      stage128<5>(y);
      stage128<6>(y);
      if (i_hi == 0) y[0] = 0.0f;  // t_0 = 0 (the mean's coefficient)

      // LayerNorm statistics: K^2 var = sum_{i>=1} Y_i^2
      float s0 = 0.0f, s1 = 0.0f;
#pragma unroll
      for (int r = 0; r < 128; r += 2) sq_acc2(s0, s1, y[r], y[r + 1]);
      const float ss = group_reduce<KH>(s0 + s1, AddF(), slot_f, quarter, lane, bar_id);
      const float var = ss * (1.0f / ((float)K * (float)K));
      const float cmul = __fmul_rn(__fdiv_rn(1.0f, sqrtf(__fadd_rn(var, 1e-5f))), p.sK);
#pragma unroll
      for (int r = 0; r < 128; r += 2) mul2(y[r], y[r + 1], cmul);

      const int64_t row = (int64_t)tile * (128 / KH) + r_loc;
      const bool row_ok = row < p.M;
      if constexpr (MODE == K1_T_F32) {
        if (row_ok) {
          float4* dst = reinterpret_cast<float4*>(p.t_out + (size_t)row * K + (size_t)i_hi * 128);
#pragma unroll
          for (int j = 0; j < 32; ++j) dst[j] = make_float4(y[4 * j], y[4 * j + 1], y[4 * j + 2], y[4 * j + 3]);
        }
      } else {
        q::RowParams qp;
        if constexpr (MODE == K1_Q8_I8) {
          float g = 0.0f;
#pragma unroll
          for (int r = 0; r < 128; ++r) g = fmaxf(g, fabsf(y[r]));
          qp = q::params_int8(group_reduce<KH>(g, MaxF(), slot_f, quarter, lane, bar_id));
        } else {
          double a0 = 0.0, a1 = 0.0;
#pragma unroll
          for (int r = 0; r < 128; r += 2) {
            a0 += q::abs_f64(y[r]);
            a1 += q::abs_f64(y[r + 1]);
          }
          qp = q::params_int4(group_reduce<KH>(a0 + a1, AddD(), slot_d, quarter, lane, bar_id), K);
        }
        if (row_ok && i_hi == 0) p.scales[row] = qp.scale;
        if constexpr (MODE == K1_Q4_PACKED) {
          // 64 bytes per thread, 16-byte chunk c at position c ^ ((m >> 1) & 3) (64B swizzle)
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const int r0 = 32 * c + 8 * h;
              uint32_t mm[8];
#pragma unroll
              for (int u = 0; u < 8; u += 2) magic2(y[r0 + u], y[r0 + u + 1], qp.r, mm[u], mm[u + 1]);
              int n[8];
#pragma unroll
              for (int u = 0; u < 8; ++u) n[u] = (int)mm[u] - q::kMagicBits;
              w[h] = q::pack_s4x8(n);
            }
            *reinterpret_cast<uint4*>(stg + m * 64 + ((c ^ ((m >> 1) & 3)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else {
          // 128 bytes per thread, 16-byte chunk c at position c ^ (m & 7) (128B swizzle)
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const int r0 = 16 * c + 4 * h;
              uint32_t mm[4];
              magic2(y[r0], y[r0 + 1], qp.r, mm[0], mm[1]);
              magic2(y[r0 + 2], y[r0 + 3], qp.r, mm[2], mm[3]);
              if constexpr (MODE == K1_Q4_I8) {
#pragma unroll
                for (int u = 0; u < 4; ++u) mm[u] = q::clip_magic_int4(mm[u]);
              }
              w[h] = q::gather_low_bytes(mm[0], mm[1], mm[2], mm[3]);
            }
            *reinterpret_cast<uint4*>(stg + m * 128 + ((c ^ (m & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
        fence_proxy_async_smem();
        named_bar_sync(bar_id, 128);
        if (issuer) {
          tma_store_2d(&tmOut, stg, 0, tile * kTileChunks);
          bulk_commit();
        }
      }
    }
    if (issuer) bulk_wait_all();
  }

  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

template <int LOGK, int MODE>
cudaError_t launch_tc(const void* x, int64_t M, void* out, float* scales, int* err, cudaStream_t stream) {
  constexpr int KH = (1 << LOGK) / 128;
  const int64_t nchunk = M * KH;
  CUtensorMap tmX, tmOut;
  if (!sm100_host::encode_2d(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, 128, (uint64_t)nchunk, 256, 64, kTileChunks,
                             CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if constexpr (MODE == K1_Q4_PACKED) {
    if (!sm100_host::encode_2d(&tmOut, CU_TENSOR_MAP_DATA_TYPE_UINT8, out, 64, (uint64_t)nchunk, 64, 64, kTileChunks,
                               CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
  } else if constexpr (MODE == K1_Q4_I8 || MODE == K1_Q8_I8) {
    if (!sm100_host::encode_2d(&tmOut, CU_TENSOR_MAP_DATA_TYPE_UINT8, out, 128, (uint64_t)nchunk, 128, 128,
                               kTileChunks, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  } else {
    tmOut = tmX;  // unused
  }
  TcParams p;
  p.M = M;
  p.num_tiles = (int)((nchunk + kTileChunks - 1) / kTileChunks);
  p.sK = (float)(1.0 / sqrt((double)(1 << LOGK)));
  p.t_out = reinterpret_cast<float*>(out);
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
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const int nsm = sm100_host::sm_count();
  const int grid = p.num_tiles < nsm ? p.num_tiles : nsm;
  kern<<<grid, kThreads, kSmemBytes, stream>>>(tmX, tmOut, p);
  return cudaGetLastError();
}

template <int LOGK>
cudaError_t launch_tc_mode(const void* x, int64_t M, K1Mode mode, void* out, float* scales, int* err,
                           cudaStream_t s) {
  switch (mode) {
    case K1_T_F32: return launch_tc<LOGK, K1_T_F32>(x, M, out, scales, err, s);
    case K1_Q4_PACKED: return launch_tc<LOGK, K1_Q4_PACKED>(x, M, out, scales, err, s);
    case K1_Q4_I8: return launch_tc<LOGK, K1_Q4_I8>(x, M, out, scales, err, s);
    case K1_Q8_I8: return launch_tc<LOGK, K1_Q8_I8>(x, M, out, scales, err, s);
    default: break;
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool ln_fht_quant_tc_supports(bool in_bf16, int log2k, K1Mode mode, const void* x, const void* out) {
  return in_bf16 && log2k >= 7 && log2k <= 14 && mode != K1_FHT_F32 &&
         (reinterpret_cast<uintptr_t>(x) & 15u) == 0 && (reinterpret_cast<uintptr_t>(out) & 15u) == 0;
}

cudaError_t launch_ln_fht_quant_tc(const void* x, int64_t M, int log2k, K1Mode mode, void* out, float* scales,
                                   cudaStream_t stream) {
  if (M <= 0) return cudaSuccess;
  int* err = device_error_word();
  if (!err) return cudaErrorInvalidValue;
  switch (log2k) {
    case 7: return launch_tc_mode<7>(x, M, mode, out, scales, err, stream);
    case 8: return launch_tc_mode<8>(x, M, mode, out, scales, err, stream);
    case 9: return launch_tc_mode<9>(x, M, mode, out, scales, err, stream);
    case 10: return launch_tc_mode<10>(x, M, mode, out, scales, err, stream);
    case 11: return launch_tc_mode<11>(x, M, mode, out, scales, err, stream);
    case 12: return launch_tc_mode<12>(x, M, mode, out, scales, err, stream);
    case 13: return launch_tc_mode<13>(x, M, mode, out, scales, err, stream);
    case 14: return launch_tc_mode<14>(x, M, mode, out, scales, err, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace hbl
