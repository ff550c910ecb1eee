// Exact int8 x int8 -> int32 GEMM on the sm_100a tensor cores (tcgen05,
// kind::i8) with the H-BitLinear dequantisation fused into the epilogue
// ("BitNet v2: Native 4-bit Activations with Hadamard Transformation for
// 1-bit LLMs", section "H-BitLinear", matrix-operation formula: the quantised
// activations times the ternary weights, rescaled by the per-token scale and
// the weight scale alpha).
//
//   acc[m][n] = sum_k A[m][k] * B[n][k]     A: [M][K] int8, B: [N][K] int8
//   y[m][n]   = (float)acc[m][n] * (scale[m] * alpha)     (float or bf16)
//
// Int4 activation codes and ternary weight codes are widened to int8 before
// they reach this kernel (sm_100 has no int4 or ternary integer MMA); int8
// products accumulate exactly in int32 (|acc| <= 127 * 32768 < 2^31).
//
// Three variants share the helpers below: the 2-SM kernel (M >= 256, described
// above gemm_i8_2sm_kernel), this 1-SM kernel for short M, and its split-K
// form for short M with few output tiles (described above
// gemm_i8_splitk_kernel).
//
// 1-SM design (one CTA per SM, persistent over 128 x 256 output tiles):
//   warp 0      TMA producer: 128-byte-swizzled boxes of A (128 x 128 B) and
//               B (256 x 128 B) into a kStages-deep shared-memory ring;
//   warp 1      allocates 512 TMEM columns (two 128 x 256 int32
//               accumulators) and one thread issues tcgen05.mma (M=128,
//               N=256, K=32 per instruction, four per 128-byte k-block),
//               committing each stage back to the producer and each finished
//               accumulator to the epilogue;
//   warps 2-5   epilogue: tcgen05.ld 32 columns at a time from the TMEM lane
//               quarter each warp may access, scale, convert, store (as
//               streaming stores: y is not read again here, and evicting it
//               early writes it back while this kernel leaves DRAM idle
//               instead of during the memory-bound kernel that follows).
// The accumulator double buffer lets the epilogue of tile i overlap the main
// loop of tile i+1.  Every mbarrier wait is bounded: after ~2 s a thread sets
// the CTA abort flag and the device error word, every role leaves its loop,
// the MMA thread drains its outstanding MMAs (bounded) and TMEM is freed.
#include <cstdint>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "sm100.cuh"

namespace hbl {

__device__ sm100::DeviceStatus g_status = {0, 0, sm100::kWaitLimitNs};

namespace {

using namespace sm100;

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 128;  // bytes of K per stage (one 128-byte swizzle atom row)
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK;  // 16 KB
constexpr int kBBytes = kBN * kBK;  // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + 256;

// instruction descriptor, kind::i8: D s32, A s8, B s8, both K-major, M=128, N=256
constexpr uint32_t kIdesc = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) |
                            ((uint32_t)(kBM >> 4) << 24);

struct Params {
  int M, N, K;
  int num_m, num_n, num_tiles, num_kb;
  int y_mode;  // 0 int32, 1 float, 2 bf16
  void* y;
  const float* scales;
  const float* alpha;
  int group_n;  // tile order: column tiles in groups of group_n (0: one group)
};

// Output tile of a linear tile index.  The CTAs in flight take consecutive
// indices.  Within a group of group_n column tiles the index walks the columns
// fastest, then the rows, so the clusters in flight share the group's B panels
// (kept in L2 while every row tile passes) and each A row panel is read once
// per group; with one group this is plain row-major order.
__device__ __forceinline__ void tile_mn(const Params& p, int tile, int& m_blk, int& n_blk) {
  const int g = p.group_n > 0 && p.group_n < p.num_n ? p.group_n : p.num_n;
  const int per_group = g * p.num_m;
  const int grp = tile / per_group;
  const int within = tile - grp * per_group;
  const int cols = min(g, p.num_n - grp * g);
  m_blk = within / cols;
  n_blk = grp * g + within % cols;
}

__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  return sm100::wait_bounded(bar, parity, abort_flag, &g_status.error);
}

__device__ __forceinline__ uint64_t sdesc(uint32_t saddr) { return sm100::sdesc_k_sw128(saddr); }

__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(kIdesc), "r"(accumulate));
}

__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
  uint32_t l = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo));
  uint32_t h = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi));
  return l | (h << 16);
}

__global__ void __launch_bounds__(kThreads, 1)
gemm_i8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, Params p) {
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
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Launched as a programmatic dependent, the setup above overlapped the
  // previous kernel's tail; its results (the codes, the weights) are read
  // only after this wait, and this kernel's own dependents may start only
  // after it (so none of them runs beside the kernel before this one).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tmA) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tmB) : "memory");
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int issued = 0;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
        int m_blk, n_blk;
        tile_mn(p, tile, m_blk, n_blk);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          mbar_expect_tx(&full[stage], (uint32_t)kStageBytes);
          tma_load_2d(sA + stage * kABytes, &tmA, kb * kBK, m_blk * kBM, &full[stage]);
          tma_load_2d(sB + stage * kBBytes, &tmB, kb * kBK, n_blk * kBN, &full[stage]);
          ++issued;
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      // the copies issued have landed before the CTA may exit
      drain_loads(full, kStages, issued, &g_status.error);
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
        if (!wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kBN);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!wait_bounded(&full[stage], phase, abort_flag)) { ok = false; break; }
          fence_after();
          const uint64_t a0 = sdesc(smem_u32(sA + stage * kABytes));
          const uint64_t b0 = sdesc(smem_u32(sB + stage * kBBytes));
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k) {
            // advance the start address by 32 bytes (2 x 16 B) per K=32 step
            mma_i8(d_tmem, a0 + (uint64_t)(2 * k), b0 + (uint64_t)(2 * k), (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      // all MMAs issued by this thread are complete once this commit arrives
      umma_commit(drain);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < 200000000ull) {
      }
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2..5)
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
      int ok = 1;
      if (lane == 0) ok = wait_bounded(&tfull[acc], acc_phase, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      fence_after();
      int m_blk, n_blk;
      tile_mn(p, tile, m_blk, n_blk);
      const int row = m_blk * kBM + quarter * 32 + lane;
      const bool row_ok = row < p.M;
      float sa = 0.0f;
      if (p.y_mode != 0 && row_ok) sa = __fmul_rn(__ldg(p.scales + row), __ldg(p.alpha));
      const uint32_t tbase = tmem_base + (uint32_t)(acc * kBN) + ((uint32_t)(quarter * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < kBN; c += 32) {
        uint32_t r[32];
        tmem_ld32(tbase + (uint32_t)c, r);
        const int col0 = n_blk * kBN + c;
        if (!row_ok) continue;
        if (p.y_mode == 0) {
          int32_t* yrow = reinterpret_cast<int32_t*>(p.y) + (size_t)row * p.N;
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            if (col0 + j < p.N)
              __stcs(reinterpret_cast<uint4*>(yrow + col0 + j), make_uint4(r[j], r[j + 1], r[j + 2], r[j + 3]));
        } else if (p.y_mode == 1) {
          float* yrow = reinterpret_cast<float*>(p.y) + (size_t)row * p.N;
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            if (col0 + j < p.N) {
              float4 v;
              v.x = __fmul_rn(__int2float_rn((int)r[j]), sa);
              v.y = __fmul_rn(__int2float_rn((int)r[j + 1]), sa);
              v.z = __fmul_rn(__int2float_rn((int)r[j + 2]), sa);
              v.w = __fmul_rn(__int2float_rn((int)r[j + 3]), sa);
              __stcs(reinterpret_cast<float4*>(yrow + col0 + j), v);
            }
          }
        } else {
          uint16_t* yrow = reinterpret_cast<uint16_t*>(p.y) + (size_t)row * p.N;
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            if (col0 + j < p.N) {
              uint4 v;
              v.x = bf16x2(__fmul_rn(__int2float_rn((int)r[j]), sa), __fmul_rn(__int2float_rn((int)r[j + 1]), sa));
              v.y = bf16x2(__fmul_rn(__int2float_rn((int)r[j + 2]), sa), __fmul_rn(__int2float_rn((int)r[j + 3]), sa));
              v.z = bf16x2(__fmul_rn(__int2float_rn((int)r[j + 4]), sa), __fmul_rn(__int2float_rn((int)r[j + 5]), sa));
              v.w = bf16x2(__fmul_rn(__int2float_rn((int)r[j + 6]), sa), __fmul_rn(__int2float_rn((int)r[j + 7]), sa));
              __stcs(reinterpret_cast<uint4*>(yrow + col0 + j), v);
            }
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
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

// ---------------------------------------------------------------- 2-SM variant
// A cluster of two CTAs (one per SM of a TPC) computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M = 256): each CTA holds 128 rows of A and 128 of
// the 256 B rows in its own shared memory, so each SM streams half the B
// bytes of the 1-SM kernel per MMA, and a 6-stage ring of 32 KB stages fits.
// Both CTAs' TMA loads complete on the leader CTA's full barrier (the leader
// alone expects the 64 KB of a stage); only the leader issues MMAs; its
// commits arrive on the same-offset barriers of both CTAs (commit multicast,
// no multicast loads).  Each CTA's epilogue reads its own TMEM (its 128 rows)
// and arrives on the leader's accumulator-empty barrier.
constexpr int k2Stages = 6;
constexpr int k2ABytes = 128 * kBK;  // 16 KB: this CTA's 128 rows of A
constexpr int k2BBytes = 128 * kBK;  // 16 KB: this CTA's 128 of the 256 B rows
constexpr int k2StageBytes = k2ABytes + k2BBytes;
constexpr size_t k2SmemBytes = 1024 + (size_t)k2Stages * k2StageBytes + 256;
// kind::i8, D s32, A/B s8 K-major, M = 256, N = 256
constexpr uint32_t kIdesc2 = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(256 >> 3) << 17) |
                             ((uint32_t)(256 >> 4) << 24);

__device__ __forceinline__ void mma_i8_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(kIdesc2), "r"(accumulate));
}

__device__ __forceinline__ void epilogue_tile(const Params& p, uint32_t tbase, int row, int n0) {
  const bool row_ok = row < p.M;
  float sa = 0.0f;
  if (p.y_mode != 0 && row_ok) sa = __fmul_rn(__ldg(p.scales + row), __ldg(p.alpha));
#pragma unroll 1
  for (int c = 0; c < 256; c += 32) {
    uint32_t r[32];
    tmem_ld32(tbase + (uint32_t)c, r);
    const int col0 = n0 + c;
    if (!row_ok) continue;
    if (p.y_mode == 0) {
      int32_t* yrow = reinterpret_cast<int32_t*>(p.y) + (size_t)row * p.N;
#pragma unroll
      for (int j = 0; j < 32; j += 4)
        if (col0 + j < p.N)
          __stcs(reinterpret_cast<uint4*>(yrow + col0 + j), make_uint4(r[j], r[j + 1], r[j + 2], r[j + 3]));
    } else if (p.y_mode == 1) {
      float* yrow = reinterpret_cast<float*>(p.y) + (size_t)row * p.N;
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        if (col0 + j < p.N) {
          float4 v;
          v.x = __fmul_rn(__int2float_rn((int)r[j]), sa);
          v.y = __fmul_rn(__int2float_rn((int)r[j + 1]), sa);
          v.z = __fmul_rn(__int2float_rn((int)r[j + 2]), sa);
          v.w = __fmul_rn(__int2float_rn((int)r[j + 3]), sa);
          __stcs(reinterpret_cast<float4*>(yrow + col0 + j), v);
        }
      }
    } else {
      uint16_t* yrow = reinterpret_cast<uint16_t*>(p.y) + (size_t)row * p.N;
#pragma unroll
      for (int j = 0; j < 32; j += 8) {
        if (col0 + j < p.N) {
          uint4 v;
          v.x = bf16x2(__fmul_rn(__int2float_rn((int)r[j]), sa), __fmul_rn(__int2float_rn((int)r[j + 1]), sa));
          v.y = bf16x2(__fmul_rn(__int2float_rn((int)r[j + 2]), sa), __fmul_rn(__int2float_rn((int)r[j + 3]), sa));
          v.z = bf16x2(__fmul_rn(__int2float_rn((int)r[j + 4]), sa), __fmul_rn(__int2float_rn((int)r[j + 5]), sa));
          v.w = bf16x2(__fmul_rn(__int2float_rn((int)r[j + 6]), sa), __fmul_rn(__int2float_rn((int)r[j + 7]), sa));
          __stcs(reinterpret_cast<uint4*>(yrow + col0 + j), v);
        }
      }
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
gemm_i8_2sm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, Params p) {
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
  const int cid = blockIdx.x >> 1;
  const int ncl = gridDim.x >> 1;
  int issued = 0;  // stages this CTA's producer (thread 0) loaded

  if (threadIdx.x == 0) {
    for (int s = 0; s < k2Stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8);
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
  asm volatile("griddepcontrol.wait;" ::: "memory");  // as in gemm_i8_kernel
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == 0) {
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tmA) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&tmB) : "memory");
      // a column group's B panels are read by every row tile: keep them in
      // L2; an A panel's readers run at about the same time: stream it
      // (measured at the 7B shape: DRAM reads 524 -> 460 MB, writes 60 -> 40 MB)
      const uint64_t pol_a = l2_policy_evict_first();
      const uint64_t pol_b = l2_policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = cid; tile < p.num_tiles && ok; tile += ncl) {
        int m_blk, n_blk;
        tile_mn(p, tile, m_blk, n_blk);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          const uint32_t fbar = mapa_shared(smem_u32(&full[stage]), 0);
          if (leader) mbar_expect_tx(&full[stage], (uint32_t)(2 * k2StageBytes));
          tma_load_2d_pair_hint(sA + stage * k2ABytes, &tmA, kb * kBK, m_blk * 256 + (int)rank * 128, fbar, pol_a);
          tma_load_2d_pair_hint(sB + stage * k2BBytes, &tmB, kb * kBK, n_blk * 256 + (int)rank * 128, fbar, pol_b);
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
        if (!wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * 256);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!wait_bounded(&full[stage], phase, abort_flag)) { ok = false; break; }
          fence_after();
          const uint64_t a0 = sdesc(smem_u32(sA + stage * k2ABytes));
          const uint64_t b0 = sdesc(smem_u32(sB + stage * k2BBytes));
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k)
            mma_i8_pair(d_tmem, a0 + (uint64_t)(2 * k), b0 + (uint64_t)(2 * k), (kb | k) != 0 ? 1u : 0u);
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
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = cid; tile < p.num_tiles; tile += ncl) {
      int ok = 1;
      if (lane == 0) ok = wait_bounded(&tfull[acc], acc_phase, abort_flag) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      fence_after();
      int m_blk, n_blk;
      tile_mn(p, tile, m_blk, n_blk);
      const int row = m_blk * 256 + (int)rank * 128 + quarter * 32 + lane;
      epilogue_tile(p, tmem_base + (uint32_t)(acc * 256) + ((uint32_t)(quarter * 32) << 16), row, n_blk * 256);
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

  // neither CTA may free its shared memory or TMEM while the pair still uses
  // them, nor exit with loads into its shared memory in flight: a bounded
  // handshake through each other's exit barrier, then the leader drains the
  // stage ring for both (thread 0 is each CTA's producer)
  fence_before();
  __syncthreads();
  if (threadIdx.x == 0)
    pair_exit_drain(leader, rank, full, k2Stages, (uint32_t)k2StageBytes, issued, peer_issued, exitb, drainb,
                    &g_status.error);
  __syncthreads();
  fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

// ---------------------------------------------------------------- split-K variant
// Short batches with few output tiles (M < 256 and fewer than half as many
// 128 x 256 tiles as SMs) leave most SMs idle and give each CTA the whole K
// loop.  Here a cluster of S CTAs (S = 2, 4 or 8) shares one tile and splits
// its k-blocks: rank r runs the same TMA / MMA pipeline as the 1-SM kernel
// over k-blocks [r num_kb / S, (r + 1) num_kb / S) into one 256-column TMEM
// accumulator, and its epilogue warps copy the int32 partial into the
// CTA's own (now idle) stage ring: 128 rows of 256 words, rows padded to
// 1040 bytes so that a warp's 16-byte stores of 32 rows spread over the
// banks.  Then rank r sums the S partials of columns [256 r / S, 256 (r + 1)
// / S) through distributed shared memory (ld.shared::cluster) and applies
// the same dequantisation as the other kernels; the int32 sums are exact, so
// y is identical.  Two cluster barrier phases separate writing the partials,
// reading them and leaving; every bounded wait of the pipeline comes before
// them, so each thread reaches both.
constexpr int kSplitMax = 8;
constexpr int kPartRowBytes = 256 * 4 + 16;
constexpr int kPart16RowBytes = 256 * 2 + 16;  // int16 partials (the bound allows it)
constexpr uint32_t kSplitTmemCols = 256;
static_assert(128 * kPartRowBytes <= kStages * kStageBytes, "partial must fit in the stage ring");

// cluster-wide barrier phase: this thread's shared-memory writes are visible
// to every CTA of the cluster after it, and its reads of other CTAs' shared
// memory are complete before any of them passes the next one.  Every thread
// of every CTA takes each phase once; every wait before it is bounded.
__device__ __forceinline__ void cluster_phase() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint4 ld_cluster_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// y[row][col .. col + 3] from four int32 sums (col + 3 < N, 16-byte-aligned rows)
__device__ __forceinline__ void store_y4(const Params& p, int row, int col, const int (&v)[4], float sa) {
  if (p.y_mode == 0) {
    __stcs(reinterpret_cast<int4*>(reinterpret_cast<int32_t*>(p.y) + (size_t)row * p.N + col),
           make_int4(v[0], v[1], v[2], v[3]));
  } else if (p.y_mode == 1) {
    float4 o;
    o.x = __fmul_rn(__int2float_rn(v[0]), sa);
    o.y = __fmul_rn(__int2float_rn(v[1]), sa);
    o.z = __fmul_rn(__int2float_rn(v[2]), sa);
    o.w = __fmul_rn(__int2float_rn(v[3]), sa);
    __stcs(reinterpret_cast<float4*>(reinterpret_cast<float*>(p.y) + (size_t)row * p.N + col), o);
  } else {
    uint2 o;
    o.x = bf16x2(__fmul_rn(__int2float_rn(v[0]), sa), __fmul_rn(__int2float_rn(v[1]), sa));
    o.y = bf16x2(__fmul_rn(__int2float_rn(v[2]), sa), __fmul_rn(__int2float_rn(v[3]), sa));
    __stcs(reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(p.y) + (size_t)row * p.N + col), o);
  }
}

template <int S, bool P16>
__global__ void __launch_bounds__(kThreads, 1)
gemm_i8_splitk_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = base;
  uint8_t* sB = base + kStages * kABytes;
  uint8_t* part = base;  // after the main loop: the int32 partial, 128 rows of kPartRowBytes
  uint64_t* full = reinterpret_cast<uint64_t*>(base + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* drain = tfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = (int)cluster_ctarank();
  const int tile = blockIdx.x / S;
  int m_blk, n_blk;
  tile_mn(p, tile, m_blk, n_blk);
  const int kb0 = rank * p.num_kb / S, kb1 = (rank + 1) * p.num_kb / S;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) tmem_alloc(tmem_slot, kSplitTmemCols);
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem_base = *tmem_slot;
  asm volatile("griddepcontrol.wait;" ::: "memory");  // as in gemm_i8_kernel
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&tmA);
      prefetch_tensormap(&tmB);
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag)) break;
        mbar_expect_tx(&full[stage], (uint32_t)kStageBytes);
        tma_load_2d(sA + stage * kABytes, &tmA, kb * kBK, m_blk * kBM, &full[stage]);
        tma_load_2d(sB + stage * kBBytes, &tmB, kb * kBK, n_blk * kBN, &full[stage]);
        ++issued;
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
      // the loads have landed before the stage ring holds the partials
      drain_loads(full, kStages, issued, &g_status.error);
    }
    __syncwarp();
    cluster_phase();  // partials written
    cluster_phase();  // partials read
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!wait_bounded(&full[stage], phase, abort_flag)) break;
        fence_after();
        const uint64_t a0 = sdesc(smem_u32(sA + stage * kABytes));
        const uint64_t b0 = sdesc(smem_u32(sB + stage * kBBytes));
#pragma unroll
        for (int k = 0; k < kBK / 32; ++k)
          mma_i8(tmem_base, a0 + (uint64_t)(2 * k), b0 + (uint64_t)(2 * k), (kb > kb0 || k > 0) ? 1u : 0u);
        umma_commit(&empty[stage]);
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
      umma_commit(tfull);
      umma_commit(drain);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(drain, 0) && globaltimer() - t0 < 200000000ull) {
      }
    }
    __syncwarp();
    cluster_phase();
    cluster_phase();
  } else {
    // ------------------------------------------------ epilogue (warps 2..5)
    const int quarter = warp & 3;
    const int et = threadIdx.x - 64;  // 0 .. 127
    if (lane == 0) wait_bounded(tfull, 0, abort_flag);
    __syncwarp();
    fence_after();
    // The partial's valid rows into shared memory (on a failed wait:
    // whatever TMEM holds; the error word is set and the handshakes below
    // still run).  Two TMEM loads in flight per wait.
    const int rows = min(kBM, p.M - m_blk * kBM);
    // P16: every partial fits in int16 (the host's bound on |a b| times this
    // rank's k-range), so the exchange moves half the bytes
    constexpr int kRowBytes = P16 ? kPart16RowBytes : kPartRowBytes;
    constexpr int kEsz = P16 ? 2 : 4;
    if (quarter * 32 < rows) {
      const int prow = quarter * 32 + lane;
      uint8_t* dst = part + (size_t)prow * kRowBytes;
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < 256; c += 64) {
        uint32_t r[64];
        tmem_ld32_nowait(tbase + (uint32_t)c, &r[0]);
        tmem_ld32_nowait(tbase + (uint32_t)(c + 32), &r[32]);
        tmem_wait_ld();
        if (prow < rows) {
          if constexpr (P16) {
#pragma unroll
            for (int j = 0; j < 64; j += 8)
              *reinterpret_cast<uint4*>(dst + 2 * (c + j)) =
                  make_uint4((r[j] & 0xFFFFu) | (r[j + 1] << 16), (r[j + 2] & 0xFFFFu) | (r[j + 3] << 16),
                             (r[j + 4] & 0xFFFFu) | (r[j + 5] << 16), (r[j + 6] & 0xFFFFu) | (r[j + 7] << 16));
          } else {
#pragma unroll
            for (int j = 0; j < 64; j += 4)
              *reinterpret_cast<uint4*>(dst + 4 * (c + j)) = make_uint4(r[j], r[j + 1], r[j + 2], r[j + 3]);
          }
        }
      }
    }
    cluster_phase();  // every rank's partial is in its shared memory
    {
      // This rank's columns, W = 256 / S, as 4-column groups over 128 rows:
      // 64 / S groups per thread, taken GB at a time with the S loads of each
      // group all issued before any is used (16 remote loads in flight per
      // thread, so the distributed-shared-memory latency is paid 4 times).
      constexpr int W = kBN / S;
      constexpr int GW = 16 / kEsz;     // columns per group: one 16-byte load
      constexpr int GPR = W / GW;       // groups per row
      constexpr int GB = 16 / S;        // groups per batch and thread
      const int total = rows * GPR;     // groups of the valid rows
      const uint32_t part_u32 = smem_u32(part);
#pragma unroll 1
      for (int b = 0; b < total; b += 128 * GB) {
        uint4 u[GB][S];
#pragma unroll
        for (int gi = 0; gi < GB; ++gi) {
          const int g = b + 128 * gi + et;
          if (g < total) {
            const uint32_t off = part_u32 + (uint32_t)((g / GPR) * kRowBytes + kEsz * (rank * W + GW * (g % GPR)));
#pragma unroll
            for (int r = 0; r < S; ++r) u[gi][r] = ld_cluster_v4(mapa_shared(off, (uint32_t)r));
          }
        }
#pragma unroll
        for (int gi = 0; gi < GB; ++gi) {
          const int g = b + 128 * gi + et;
          if (g >= total) continue;
          int v[GW];
#pragma unroll
          for (int i = 0; i < GW; ++i) v[i] = 0;
#pragma unroll
          for (int r = 0; r < S; ++r) {
            const uint32_t w[4] = {u[gi][r].x, u[gi][r].y, u[gi][r].z, u[gi][r].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              if constexpr (P16) {
                v[2 * i] += (int)(w[i] << 16) >> 16;  // sign-extended halves
                v[2 * i + 1] += (int)w[i] >> 16;
              } else {
                v[i] += (int)w[i];
              }
            }
          }
          const int row = m_blk * kBM + g / GPR;
          const int col = n_blk * kBN + rank * W + GW * (g % GPR);
          if (row < p.M) {
            const float sa = p.y_mode != 0 ? __fmul_rn(__ldg(p.scales + row), __ldg(p.alpha)) : 0.0f;
#pragma unroll
            for (int h = 0; h < GW; h += 4) {
              if (col + h < p.N) {
                const int q4[4] = {v[h], v[h + 1], v[h + 2], v[h + 3]};
                store_y4(p, row, col + h, q4, sa);
              }
            }
          }
        }
      }
    }
    cluster_phase();  // no rank leaves while another still reads its partial
  }

  fence_before();
  __syncthreads();
  fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kSplitTmemCols);
}

// 2-D K-major int8 tensor map: rows x K bytes, box kBK x box_rows, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* ptr, int64_t rows, int64_t K, int box_rows) {
  return sm100_host::encode_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, ptr, (uint64_t)K, (uint64_t)rows, (uint64_t)K,
                               (uint32_t)kBK, (uint32_t)box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

int sm_count() { return sm100_host::sm_count(); }

constexpr int kSplitMaxRows = 64;     // int32 partials: the exchange grows with the rows
constexpr int kSplitMaxRows16 = 255;  // int16 partials: every short batch

// clusters of `split` CTAs of `kern` that the device holds at once (cached
// per device and cluster size; 0 when the query fails)
template <typename Kernel>
int max_active_clusters(Kernel kern, int split, int idx) {
  static std::atomic<int> cache[6][sm100_host::kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= sm100_host::kMaxDevices) return 0;
  const int c = cache[idx][dev].load(std::memory_order_acquire);
  if (c > 0) return c;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)split, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)split;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  cache[idx][dev].store(n, std::memory_order_release);
  return n;
}

}  // namespace

cudaError_t launch_gemm_i8(const int8_t* A, const int8_t* B, int64_t M, int64_t N, int64_t K, int y_mode, void* y,
                           const float* scales, const float* alpha, cudaStream_t stream, int ab_max) {
  CUtensorMap ta, tb;
  if (!make_map(&ta, A, M, K, kBM) || !make_map(&tb, B, N, K, kBN)) return cudaErrorInvalidValue;
  Params p;
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.num_m = (int)((M + kBM - 1) / kBM);
  p.num_n = (int)((N + kBN - 1) / kBN);
  p.num_tiles = p.num_m * p.num_n;
  p.num_kb = (int)((K + kBK - 1) / kBK);
  p.y_mode = y_mode;
  p.y = y;
  p.scales = scales;
  p.alpha = alpha;
  p.group_n = 0;
  if (M >= 256) {
    // 2-SM tiles of 256 x 256
    CUtensorMap tb2;
    if (!make_map(&tb2, B, N, K, 128)) return cudaErrorInvalidValue;
    p.num_m = (int)((M + 255) / 256);
    p.num_n = (int)((N + 255) / 256);
    p.num_tiles = p.num_m * p.num_n;
    // column tiles in as few equal groups as keep a group's B panels within
    // about a third of L2 (40 MB), so they stay there while every row tile
    // passes: at the 7B shape (16 panels of 4 MB) two groups of 8 cut DRAM
    // reads from 616 to 513 MB per launch and the time by 2%
    const int64_t panel = (int64_t)256 * K;
    const int64_t groups = (p.num_n * panel + (int64_t(40) << 20) - 1) / (int64_t(40) << 20);
    p.group_n = groups > 1 ? (int)((p.num_n + groups - 1) / groups) : 0;
    static std::atomic<bool> smem_set2[sm100_host::kMaxDevices];
    cudaError_t e = sm100_host::ensure_smem(gemm_i8_2sm_kernel, (int)k2SmemBytes, smem_set2);
    if (e != cudaSuccess) return e;
    const int pairs = sm_count() / 2;
    const int nclusters = p.num_tiles < pairs ? p.num_tiles : pairs;
    return sm100_host::launch_pdl(gemm_i8_2sm_kernel, (unsigned)(2 * nclusters), kThreads, k2SmemBytes, stream, 2,
                                  ta, tb2, p);
  }
  // A few rows and few tiles: split K over a cluster of S CTAs per tile, the
  // largest S whose clusters all fit on the GPU at once.  (With more rows the
  // partials' exchange through distributed shared memory costs more than the
  // split saves.)
  const int nsm = sm_count();
  for (int split = kSplitMax; split >= 2; split /= 2) {
    if (split > p.num_kb || p.num_tiles * split > nsm) continue;
    // int16 partials when |a b| times this split's k-range per rank stays below 2^15
    const int64_t kb_per = (p.num_kb + split - 1) / split;
    const bool p16 = ab_max > 0 && (int64_t)ab_max * kb_per * kBK <= 32767;
    if (M > (p16 ? kSplitMaxRows16 : kSplitMaxRows)) continue;
    auto kern = p16 ? (split == 2 ? gemm_i8_splitk_kernel<2, true>
                       : split == 4 ? gemm_i8_splitk_kernel<4, true> : gemm_i8_splitk_kernel<8, true>)
                    : (split == 2 ? gemm_i8_splitk_kernel<2, false>
                       : split == 4 ? gemm_i8_splitk_kernel<4, false> : gemm_i8_splitk_kernel<8, false>);
    const int idx = (split == 2 ? 0 : split == 4 ? 1 : 2) + (p16 ? 3 : 0);
    static std::atomic<bool> smem_set_s[6][sm100_host::kMaxDevices];
    cudaError_t e = sm100_host::ensure_smem(kern, (int)kSmemBytes, smem_set_s[idx]);
    if (e != cudaSuccess) return e;
    if (p.num_tiles > max_active_clusters(kern, split, idx)) continue;
    return sm100_host::launch_pdl(kern, (unsigned)(p.num_tiles * split), kThreads, kSmemBytes, stream,
                                  (unsigned)split, ta, tb, p);
  }
  static std::atomic<bool> smem_set[sm100_host::kMaxDevices];
  cudaError_t e = sm100_host::ensure_smem(gemm_i8_kernel, (int)kSmemBytes, smem_set);
  if (e != cudaSuccess) return e;
  const int grid = p.num_tiles < nsm ? p.num_tiles : nsm;
  return sm100_host::launch_pdl(gemm_i8_kernel, (unsigned)grid, kThreads, kSmemBytes, stream, 1, ta, tb, p);
}

int* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  static std::atomic<int*> cache[64];
  int* c = cache[dev].load(std::memory_order_acquire);
  if (!c) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
    c = &reinterpret_cast<sm100::DeviceStatus*>(p)->error;
    cache[dev].store(c, std::memory_order_release);
  }
  return c;
}

cudaError_t read_and_clear_device_error(cudaStream_t stream, int* value) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return e;
  int v = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&v, g_status, sizeof(int), offsetof(sm100::DeviceStatus, error));
  if (e != cudaSuccess) return e;
  e = cudaMemcpyToSymbol(g_status, &zero, sizeof(int), offsetof(sm100::DeviceStatus, error));
  *value = v;
  return e;
}

cudaError_t set_wait_limit(unsigned long long ns) {
  // no kernel of the device may be running while the limit changes
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return e;
  const unsigned long long v = ns ? ns : sm100::kWaitLimitNs;
  return cudaMemcpyToSymbol(g_status, &v, sizeof(v), offsetof(sm100::DeviceStatus, wait_limit_ns));
}

namespace {
__global__ void raise_error_kernel() { atomicExch(&g_status.error, 1); }
}  // namespace

cudaError_t raise_device_error(cudaStream_t stream) {
  raise_error_kernel<<<1, 1, 0, stream>>>();
  return cudaGetLastError();
}

}  // namespace hbl
