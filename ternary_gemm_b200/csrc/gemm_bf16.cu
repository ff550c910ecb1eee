// bf16 x bf16 -> f32 GEMM on the sm_100a tensor cores (tcgen05, kind::f16)
// for the H-BitLinear backward pass ("BitNet v2: Native 4-bit Activations
// with Hadamard Transformation for 1-bit LLMs", training strategy: the
// straight-through estimator passes the gradient around the quantizers, so
// both gradient products are plain dense contractions of bf16 operands that
// hold exact values: the ternary weights, the integer activation codes, and
// the incoming gradient itself).
//
//   D[r][c] = scale * sum_k A[r][k] B[k][c]        D f32 [R][C] row-major
//
// A is either K-major (stored [R][Kc], row r contiguous over k) or MN-major
// (stored [Kc][R], k-row contiguous over r); B is always MN-major (stored
// [Kc][C]).  That covers the two products of the backward pass without any
// transposed copy:
//   activation gradient  g_t[m][k] = alpha sum_n g_y[m][n] w[n][k]
//                         (A = g_y K-major over n, B = w as stored)
//   weight gradient      g_W[n][k] = sum_m (s g_y)[m][n] q[m][k]
//                         (A = s g_y read MN-major, B = q as stored)
//
// Same structure as the 1-SM int8 kernel: one CTA per SM, persistent over
// 128 x 256 output tiles; warp 0 issues TMA loads (128-byte swizzle) into a
// 4-stage ring of 48 KB stages (64 k-elements each); warp 1 allocates 512 TMEM
// columns (two 128 x 256 f32 accumulators) and one thread issues
// tcgen05.mma (M = 128, N = 256, K = 16, four per stage); warps 2-5 read the
// accumulator quarter of their TMEM lanes, scale and store f32 rows (float4
// per thread, streaming).  Every mbarrier wait is bounded, as in the int8
// kernels.
#include <cstdint>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "sm100.cuh"

namespace hbl {
namespace {

using namespace sm100;

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBKe = 64;                 // k elements per stage (128 bytes of bf16)
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBKe * 2;  // 16 KB
constexpr int kBBytes = kBN * kBKe * 2;  // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kAtomBytes = 64 * kBKe * 2;  // one MN-major box: 64 k-rows x 64 elements (8 KB)
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + 256;

// kind::f16 instruction descriptor: D f32, A and B bf16, B MN-major,
// A MN-major when A_MN, N = 256, M = 128
template <bool A_MN>
__host__ __device__ constexpr uint32_t idesc() {
  return (1u << 4) | (1u << 7) | (1u << 10) | (A_MN ? (1u << 15) : 0u) | (1u << 16) | ((uint32_t)(kBN >> 3) << 17) |
         ((uint32_t)(kBM >> 4) << 24);
}

struct BParams {
  int R, C, Kc;
  int num_r, num_c, num_tiles, num_kb;
  float* d;
  const float* scale;  // device scalar, or null for 1
  int* err;            // device error word (bounded waits that gave up)
  int col_major;       // tile order: rows fastest (1) or columns fastest (0)
};

// Output tile of a linear tile index.  The CTAs in flight at once take
// consecutive indices; with rows fastest they share one B column panel and
// cycle through all A row panels, with columns fastest the reverse.  The host
// picks the order whose cycled operand is the smaller one, so that it stays in
// L2 and the other streams from DRAM once.
__device__ __forceinline__ void tile_coords(const BParams& p, int tile, int& r_blk, int& c_blk) {
  if (p.col_major) {
    r_blk = tile % p.num_r;
    c_blk = tile / p.num_r;
  } else {
    r_blk = tile / p.num_c;
    c_blk = tile % p.num_c;
  }
}

template <bool A_MN>
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc<A_MN>()), "r"(accumulate));
}

template <bool A_MN>
__global__ void __launch_bounds__(kThreads, 1)
gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, BParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = base;
  uint8_t* sB = base + kStages * kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem_base = *tmem_slot;
  asm volatile("griddepcontrol.wait;" ::: "memory");  // programmatic dependent: see gemm_i8.cu
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tmA);
      prefetch_tensormap(&tmB);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int issued = 0;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        int r_blk, c_blk;
        tile_coords(p, tile, r_blk, c_blk);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.err)) { ok = false; break; }
          mbar_expect_tx(&full[stage], (uint32_t)kStageBytes);
          uint8_t* a = sA + stage * kABytes;
          uint8_t* b = sB + stage * kBBytes;
          if constexpr (A_MN) {
            tma_load_2d(a, &tmA, r_blk * kBM, kb * kBKe, &full[stage]);
            tma_load_2d(a + kAtomBytes, &tmA, r_blk * kBM + 64, kb * kBKe, &full[stage]);
          } else {
            tma_load_2d(a, &tmA, kb * kBKe, r_blk * kBM, &full[stage]);
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) tma_load_2d(b + j * kAtomBytes, &tmB, c_blk * kBN + 64 * j, kb * kBKe, &full[stage]);
          ++issued;
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      // the copies issued have landed before the CTA may exit
      drain_loads(full, kStages, issued, p.err);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        if (!wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, p.err)) { ok = false; break; }
        fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kBN);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!wait_bounded(&full[stage], phase, abort_flag, p.err)) { ok = false; break; }
          fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * kABytes);
          // A K-major: 32 bytes per K=16 step inside the 128-byte rows; A and B
          // MN-major: 16 k-rows (2048 bytes) per step, 64-element atoms 8 KB apart
          const uint64_t a0 = A_MN ? sdesc_mn_sw128(a_addr, kAtomBytes) : sdesc_k_sw128(a_addr);
          const uint64_t b0 = sdesc_mn_sw128(smem_u32(sB + stage * kBBytes), kAtomBytes);
#pragma unroll
          for (int k = 0; k < kBKe / 16; ++k) {
            const uint64_t a = a0 + (uint64_t)(A_MN ? 128 * k : 2 * k);
            mma_bf16<A_MN>(d_tmem, a, b0 + (uint64_t)(128 * k), (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      umma_commit(drain);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < 200000000ull) {
      }
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2..5)
    const int quarter = warp & 3;
    const float sc = p.scale ? __ldg(p.scale) : 1.0f;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
      int ok = 1;
      if (lane == 0) ok = wait_bounded(&tfull[acc], acc_phase, abort_flag, p.err) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      fence_after();
      int r_blk, c_blk;
      tile_coords(p, tile, r_blk, c_blk);
      const int row = r_blk * kBM + quarter * 32 + lane;
      const uint32_t tbase = tmem_base + (uint32_t)(acc * kBN) + ((uint32_t)(quarter * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < kBN; c += 32) {
        uint32_t v[32];
        tmem_ld32(tbase + (uint32_t)c, v);
        const int col0 = c_blk * kBN + c;
        if (row >= p.R) continue;
        float* drow = p.d + (size_t)row * p.C;
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          if (col0 + j < p.C) {
            const float4 o = make_float4(__fmul_rn(__uint_as_float(v[j]), sc), __fmul_rn(__uint_as_float(v[j + 1]), sc),
                                         __fmul_rn(__uint_as_float(v[j + 2]), sc),
                                         __fmul_rn(__uint_as_float(v[j + 3]), sc));
            __stcs(reinterpret_cast<float4*>(drow + col0 + j), o);
          }
        }
      }
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// ---------------------------------------------------------------- 2-SM variant
// For R >= 256: a cluster of two CTAs (the two SMs of a TPC) computes 256 x
// 256 tiles with tcgen05.mma.cta_group::2 (M = 256), as the int8 2-SM kernel
// does: each CTA stages its 128 rows of A and its 128 of the 256 B columns
// (6 stages of 32 KB), both CTAs' TMA loads complete on the leader's barrier,
// only the leader issues MMAs and its commits reach both CTAs.  Per MMA each SM
// reads 8 KB of operands instead of the 1-SM kernel's 12 KB, which is what
// keeps the shared-memory port below its bandwidth at the tensor rate.
constexpr int k2Stages = 6;
constexpr int k2ABytes = 128 * kBKe * 2;  // 16 KB
constexpr int k2BBytes = 128 * kBKe * 2;  // 16 KB
constexpr int k2StageBytes = k2ABytes + k2BBytes;
constexpr size_t k2SmemBytes = 1024 + (size_t)k2Stages * k2StageBytes + 256;

template <bool A_MN>
__host__ __device__ constexpr uint32_t idesc2() {
  return (1u << 4) | (1u << 7) | (1u << 10) | (A_MN ? (1u << 15) : 0u) | (1u << 16) | ((uint32_t)(256 >> 3) << 17) |
         ((uint32_t)(256 >> 4) << 24);
}

template <bool A_MN>
__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc2<A_MN>()), "r"(accumulate));
}

template <bool A_MN>
__global__ void __launch_bounds__(kThreads, 1)
gemm_bf16_2sm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, BParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = base;
  uint8_t* sB = base + k2Stages * k2ABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(base + k2Stages * k2StageBytes);
  uint64_t* empty = full + k2Stages;
  uint64_t* tfull = empty + k2Stages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* exitb = drain + 1;
  uint64_t* drainb = exitb + 1;
  int* peer_issued = reinterpret_cast<int*>(drainb + 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(peer_issued + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  int issued = 0;  // stages this CTA's producer (thread 0) loaded
  const int cid = blockIdx.x >> 1;
  const int ncl = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < k2Stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8);  // the epilogue warps of both CTAs
    }
    mbar_init(drain, 1);
    mbar_init(exitb, 1);
    mbar_init(drainb, 1);
    *peer_issued = 0;
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  fence_before();
  cluster_sync_all();
  fence_after();
  const uint32_t tmem_base = *tmem_slot;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&tmA);
      prefetch_tensormap(&tmB);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = cid; tile < p.num_tiles && ok; tile += ncl) {
        int r_blk, c_blk;
        tile_coords(p, tile, r_blk, c_blk);
        const int r0 = r_blk * 256 + (int)rank * 128;
        const int c0 = c_blk * 256 + (int)rank * 128;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.err)) { ok = false; break; }
          const uint32_t fbar = mapa_shared(smem_u32(&full[stage]), 0);
          if (leader) mbar_expect_tx(&full[stage], (uint32_t)(2 * k2StageBytes));
          uint8_t* a = sA + stage * k2ABytes;
          uint8_t* b = sB + stage * k2BBytes;
          if constexpr (A_MN) {
            tma_load_2d_pair(a, &tmA, r0, kb * kBKe, fbar);
            tma_load_2d_pair(a + kAtomBytes, &tmA, r0 + 64, kb * kBKe, fbar);
          } else {
            tma_load_2d_pair(a, &tmA, kb * kBKe, r0, fbar);
          }
          tma_load_2d_pair(b, &tmB, c0, kb * kBKe, fbar);
          tma_load_2d_pair(b + kAtomBytes, &tmB, c0 + 64, kb * kBKe, fbar);
          ++issued;
          if (++stage == k2Stages) { stage = 0; phase ^= 1u; }
        }
      }
      // the loads are drained at the pair's exit (pair_exit_drain)
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = cid; tile < p.num_tiles && ok; tile += ncl) {
        if (!wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, p.err)) { ok = false; break; }
        fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * 256);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!wait_bounded(&full[stage], phase, abort_flag, p.err)) { ok = false; break; }
          fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * k2ABytes);
          const uint64_t a0 = A_MN ? sdesc_mn_sw128(a_addr, kAtomBytes) : sdesc_k_sw128(a_addr);
          const uint64_t b0 = sdesc_mn_sw128(smem_u32(sB + stage * k2BBytes), kAtomBytes);
#pragma unroll
          for (int k = 0; k < kBKe / 16; ++k)
            mma_bf16_pair<A_MN>(d_tmem, a0 + (uint64_t)(A_MN ? 128 * k : 2 * k), b0 + (uint64_t)(128 * k),
                                (kb | k) != 0 ? 1u : 0u);
          mma_commit_pair(&empty[stage]);
          if (++stage == k2Stages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        mma_commit_pair(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      mma_commit_local2(drain);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < 200000000ull) {
      }
    }
  } else {
    const int quarter = warp & 3;
    const float sc = p.scale ? __ldg(p.scale) : 1.0f;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = cid; tile < p.num_tiles; tile += ncl) {
      int ok = 1;
      if (lane == 0) ok = wait_bounded(&tfull[acc], acc_phase, abort_flag, p.err) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      fence_after();
      int r_blk, c_blk;
      tile_coords(p, tile, r_blk, c_blk);
      const int row = r_blk * 256 + (int)rank * 128 + quarter * 32 + lane;
      const uint32_t tbase = tmem_base + (uint32_t)(acc * 256) + ((uint32_t)(quarter * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < 256; c += 32) {
        uint32_t v[32];
        tmem_ld32(tbase + (uint32_t)c, v);
        const int col0 = c_blk * 256 + c;
        if (row >= p.R) continue;
        float* drow = p.d + (size_t)row * p.C;
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          if (col0 + j < p.C) {
            const float4 o = make_float4(__fmul_rn(__uint_as_float(v[j]), sc), __fmul_rn(__uint_as_float(v[j + 1]), sc),
                                         __fmul_rn(__uint_as_float(v[j + 2]), sc),
                                         __fmul_rn(__uint_as_float(v[j + 3]), sc));
            __stcs(reinterpret_cast<float4*>(drow + col0 + j), o);
          }
        }
      }
      fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(&tempty[acc]);
        else
          mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  // neither CTA frees its shared memory or TMEM while the pair still uses
  // them, nor exits with loads into its shared memory in flight (the exit
  // handshake and the leader's drain of the stage ring, pair_exit_drain;
  // thread 0 is each CTA's producer)
  fence_before();
  __syncthreads();
  if (threadIdx.x == 0)
    pair_exit_drain(leader, rank, full, k2Stages, (uint32_t)k2StageBytes, issued, peer_issued, exitb, drainb, p.err);
  __syncthreads();
  fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

}  // namespace

cudaError_t launch_gemm_bf16(const uint16_t* A, bool a_mn, const uint16_t* B, int64_t R, int64_t C, int64_t Kc,
                             float* d, const float* scale, cudaStream_t stream) {
  if (R <= 0 || C <= 0 || Kc <= 0) return cudaSuccess;
  if (R > INT32_MAX / 2 || C > INT32_MAX / 2 || Kc > INT32_MAX / 2 || C % 8 != 0 || (a_mn ? R % 8 : Kc % 8) != 0)
    return cudaErrorInvalidValue;
  CUtensorMap ta, tb;
  bool ok = a_mn ? sm100_host::encode_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, (uint64_t)R, (uint64_t)Kc,
                                         (uint64_t)R * 2, 64, kBKe, CU_TENSOR_MAP_SWIZZLE_128B)
                 : sm100_host::encode_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, (uint64_t)Kc, (uint64_t)R,
                                         (uint64_t)Kc * 2, kBKe, kBM, CU_TENSOR_MAP_SWIZZLE_128B);
  ok = ok && sm100_host::encode_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, (uint64_t)C, (uint64_t)Kc,
                                   (uint64_t)C * 2, 64, kBKe, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return cudaErrorInvalidValue;
  BParams p;
  p.R = (int)R;
  p.C = (int)C;
  p.Kc = (int)Kc;
  p.num_r = (int)((R + kBM - 1) / kBM);
  p.num_c = (int)((C + kBN - 1) / kBN);
  p.num_tiles = p.num_r * p.num_c;
  p.num_kb = (int)((Kc + kBKe - 1) / kBKe);
  p.d = d;
  p.scale = scale;
  p.col_major = R <= C ? 1 : 0;  // A (R x Kc) the smaller operand: cycle it, stream B
  p.err = device_error_word();
  if (!p.err) return cudaErrorInvalidValue;
  const int nsm = sm100_host::sm_count();
  if (R >= 256) {
    // 2-SM tiles of 256 x 256 (the A maps' 128-row boxes serve both variants)
    p.num_r = (int)((R + 255) / 256);
    p.num_tiles = p.num_r * p.num_c;
    const int pairs = nsm / 2;
    const unsigned grid2 = 2u * (unsigned)(p.num_tiles < pairs ? p.num_tiles : pairs);
    if (a_mn) {
      static std::atomic<bool> set2[sm100_host::kMaxDevices];
      cudaError_t e = sm100_host::ensure_smem(gemm_bf16_2sm_kernel<true>, (int)k2SmemBytes, set2);
      if (e != cudaSuccess) return e;
      return sm100_host::launch_pdl(gemm_bf16_2sm_kernel<true>, grid2, kThreads, k2SmemBytes, stream, 2, ta, tb, p);
    }
    static std::atomic<bool> set2[sm100_host::kMaxDevices];
    cudaError_t e = sm100_host::ensure_smem(gemm_bf16_2sm_kernel<false>, (int)k2SmemBytes, set2);
    if (e != cudaSuccess) return e;
    return sm100_host::launch_pdl(gemm_bf16_2sm_kernel<false>, grid2, kThreads, k2SmemBytes, stream, 2, ta, tb, p);
  }
  const int grid = p.num_tiles < nsm ? p.num_tiles : nsm;
  if (a_mn) {
    static std::atomic<bool> set[sm100_host::kMaxDevices];
    cudaError_t e = sm100_host::ensure_smem(gemm_bf16_kernel<true>, (int)kSmemBytes, set);
    if (e != cudaSuccess) return e;
    return sm100_host::launch_pdl(gemm_bf16_kernel<true>, (unsigned)grid, kThreads, kSmemBytes, stream, 1, ta, tb, p);
  }
  static std::atomic<bool> set[sm100_host::kMaxDevices];
  cudaError_t e = sm100_host::ensure_smem(gemm_bf16_kernel<false>, (int)kSmemBytes, set);
  if (e != cudaSuccess) return e;
  return sm100_host::launch_pdl(gemm_bf16_kernel<false>, (unsigned)grid, kThreads, kSmemBytes, stream, 1, ta, tb, p);
}

}  // namespace hbl
