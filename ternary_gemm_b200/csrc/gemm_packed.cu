// The H-BitLinear product straight from the packed codes on the sm_100a tensor
// cores ("BitNet v2: Native 4-bit Activations with Hadamard Transformation for
// 1-bit LLMs", section "H-BitLinear", matrix-operation formula: the quantised
// activations times the ternary weights, rescaled by the per-token scale and
// alpha):
//
//   acc[m][n] = sum_k q[m][k] w[n][k]    q: INT4 codes [M][K/2] (two per byte,
//                                           element 2j in the low nibble)
//                                        w: 2-bit ternary codes [N][K/4]
//   y[m][n]   = (float)acc[m][n] * (scale[m] * alpha)      (float or bf16)
//
// Neither operand exists as int8 in global memory.  A TMA producer stages the
// packed bytes of each k-block in shared memory (the whole packed A and W of a
// 7B-sized layer, 84 MB, stay in L2 across tiles), and converter warps widen
// them into the 128-byte-swizzled int8 tiles that tcgen05.mma kind::i8 reads:
//   * an INT4 code q becomes the byte 16 q (its nibble moved to the high half:
//     two byte permutes, shifts and masks per 16 codes);
//   * a ternary code w becomes the byte 64 w (its two bits moved to the top of
//     the byte: shifts and masks per 16 codes);
//   * both use the same order of the 16 k values of each 16-byte chunk (code
//     4i + j at byte 4j + i), so the contraction pairs the right values.
// The int32 sums are therefore 1024 acc exactly (|1024 acc| <= 2^28 for
// K <= 32768), and the epilogue multiplies by scale * alpha / 1024 (a power of
// two apart, so every rounding is that of (float)acc * (scale * alpha)): y is
// bit for bit the y of the int8-operand GEMM.
//
// CTA pair (cluster of two, tcgen05.mma.cta_group::2, M = 256, N = 256,
// K = 32 per instruction), persistent over 256 x 256 output tiles:
//   warp 0     TMA producer: per k-block (128 k) this CTA's 128 rows of packed
//              A (64 bytes each) and its 128 of the tile's 256 rows of packed
//              W (32 bytes each), 12 KB, into a 6-slot staging ring;
//   warps 1-8  converters, two groups of four taking alternate stages (two
//              stages are widened at once): staging slot -> registers -> the
//              int8 tiles of a 4-stage ring of 32 KB stages; after its stores a
//              warp fences them for the tensor cores' (async) proxy and signals
//              the stage on the leader's full barrier: an arrive in the leader,
//              a 16-byte bulk copy with complete-tx from the peer.  The
//              converters issue no global loads (an arrive has release
//              semantics and would wait for them);
//   warp 9     TMEM allocation (512 columns: two 128 x 256 int32 accumulators
//              per CTA) and, in the leader, the thread that issues the MMAs and
//              commits each stage back to both CTAs' empty barriers;
//   warps 10-13 epilogue: TMEM -> registers -> scale -> y, streaming stores;
//              the accumulator double buffer overlaps it with the next tile.
// Every wait is bounded (the device status's limit); a CTA that gives up
// leaves its loops, the producer waits for the copies it issued, the MMA
// thread drains its MMAs, and the pair meets at a bounded exit handshake
// before TMEM is freed.  No multicast load is issued (each CTA loads its own
// staging tiles).
#include <cstdint>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "sm100.cuh"

namespace hbl {
namespace {

using namespace sm100;

constexpr int kConvWarps = 4;                         // converter warps per group (one stage)
constexpr int kConvGroups = 2;                        // groups convert alternate stages
constexpr int kConv0 = 1;                             // first converter warp
constexpr int kMmaWarp = kConv0 + kConvGroups * kConvWarps;  // 9
constexpr int kEpi0 = kMmaWarp + 1;                   // 10: epilogue warps 10-13
constexpr int kThreads = 32 * (kEpi0 + 4);            // 448
constexpr int kSignalBytes = 16;                      // one peer warp's readiness signal
constexpr int kStages = 4;                            // int8 stages the MMAs read
constexpr int kABytes = 128 * 128;  // this CTA's 128 rows of A, one 128-byte k-block
constexpr int kBBytes = 128 * 128;  // this CTA's 128 of the tile's 256 W rows
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kSlots = 6;                             // staging slots of packed bytes
constexpr int kPABytes = 128 * 64;                    // 128 rows x 64 bytes of INT4 codes
constexpr int kPWBytes = 128 * 32;                    // 128 rows x 32 bytes of 2-bit codes
constexpr int kSlotBytes = kPABytes + kPWBytes;
constexpr uint32_t kTmemCols = 512;
constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + (size_t)kSlots * kSlotBytes + 512;
constexpr float kAccScale = 1.0f / 1024.0f;  // 16 (A) x 64 (W)
// kind::i8, D s32, A/B s8 K-major, M = 256, N = 256
constexpr uint32_t kIdesc = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(256 >> 3) << 17) |
                            ((uint32_t)(256 >> 4) << 24);

struct PParams {
  const uint8_t* A;  // INT4 codes, [M][K/2]
  const uint8_t* W;  // 2-bit codes, [N][K/4]
  int M, N, K;
  int num_m, num_n, num_tiles, num_kb;
  int group_n;  // tile order: column tiles in groups of group_n (0: one group)
  int y_mode;   // 1 float, 2 bf16
  void* y;
  const float* scales;
  const float* alpha;
  int* err;
};

// Output tile of a linear tile index (the same walk as the int8-operand GEMM:
// within a group of group_n column tiles, columns fastest).
__device__ __forceinline__ void tile_mn(const PParams& p, int tile, int& m_blk, int& n_blk) {
  const int g = p.group_n > 0 && p.group_n < p.num_n ? p.group_n : p.num_n;
  const int per_group = g * p.num_m;
  const int grp = tile / per_group;
  const int within = tile - grp * per_group;
  const int cols = min(g, p.num_n - grp * g);
  m_blk = within / cols;
  n_blk = grp * g + within % cols;
}

// 16 INT4 codes (element 8v + i in nibble i of word v) -> 16 bytes holding
// 16 * code, code 4i + j at byte 4j + i.
__device__ __forceinline__ uint4 widen_s4x16(uint32_t w0, uint32_t w1) {
  const uint32_t x = __byte_perm(w0, w1, 0x6420);  // codes (0,1) (4,5) (8,9) (12,13)
  const uint32_t y = __byte_perm(w0, w1, 0x7531);  // codes (2,3) (6,7) (10,11) (14,15)
  return make_uint4((x << 4) & 0xF0F0F0F0u, x & 0xF0F0F0F0u, (y << 4) & 0xF0F0F0F0u, y & 0xF0F0F0F0u);
}

// 16 ternary codes (element i at bits 2i of w) -> 16 bytes holding 64 * code
// in the same order: code 4i + j sits at bits 8i + 2j, so word j of the
// result is w shifted left by 6 - 2j with the top two bits of each byte kept.
__device__ __forceinline__ uint4 widen_t2x16(uint32_t w) {
  return make_uint4((w << 6) & 0xC0C0C0C0u, (w << 4) & 0xC0C0C0C0u, (w << 2) & 0xC0C0C0C0u, w & 0xC0C0C0C0u);
}

// 16-byte chunk c of row r of a 128-byte-swizzled K-major tile
__device__ __forceinline__ uint32_t sw128(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

__device__ __forceinline__ void sts16(uint32_t addr, const uint4& v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ uint4 lds16(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
               : "memory");
  return v;
}

// One converter thread's share of a staged k-block, widened into a stage.
// The staging slot holds this CTA's packed rows as TMA wrote them (zero beyond
// the operand), swizzled so that the copy engine's writes of consecutive rows
// spread over the banks: A row r at 64 r with its 16-byte chunk c at
// c ^ ((r >> 1) & 3) (the 64-byte swizzle), W row r at 64 x 128 + 32 r with
// chunk c at c ^ ((r >> 2) & 1) (the 32-byte swizzle).  Thread t takes
// A chunks q = t + 128 i (row q / 4, codes 32 (q % 4) ..), each to tile chunks
// 2 (q % 4) and 2 (q % 4) + 1, and W chunks q = t + 128 i (row q / 2, codes
// 64 (q % 2) ..), each to tile chunks 4 (q % 2) .. 4 (q % 2) + 3.  A warp's
// 16-byte loads cover 512 contiguous bytes and its stores hit every bank
// once per phase (rows r, r + 1 with r even fill complementary chunk sets).
__device__ __forceinline__ void widen_stage(uint32_t slot, uint32_t sA, uint32_t sW, int t) {
  uint4 a[4], w[2];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int q = t + 128 * i, r = q >> 2, c = q & 3;
    a[i] = lds16(slot + (uint32_t)(64 * r + ((c ^ ((r >> 1) & 3)) << 4)));
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int q = t + 128 * i, r = q >> 1, c = q & 1;
    w[i] = lds16(slot + (uint32_t)(kPABytes + 32 * r + ((c ^ ((r >> 2) & 1)) << 4)));
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int q = t + 128 * i, row = q >> 2, c = 2 * (q & 3);
    sts16(sA + sw128(row, c), widen_s4x16(a[i].x, a[i].y));
    sts16(sA + sw128(row, c + 1), widen_s4x16(a[i].z, a[i].w));
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int q = t + 128 * i, row = q >> 1, c = 4 * (q & 1);
    sts16(sW + sw128(row, c), widen_t2x16(w[i].x));
    sts16(sW + sw128(row, c + 1), widen_t2x16(w[i].y));
    sts16(sW + sw128(row, c + 2), widen_t2x16(w[i].z));
    sts16(sW + sw128(row, c + 3), widen_t2x16(w[i].w));
  }
}

__device__ __forceinline__ void mma_i8_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(kIdesc), "r"(accumulate));
}

__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
         ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
}

// y row `row`, columns n0 .. n0 + 255, from this warp's TMEM lane quarter
__device__ __forceinline__ void epilogue_row(const PParams& p, uint32_t tbase, int row, int n0) {
  const bool row_ok = row < p.M;
  // scale * alpha / 1024: the power of two undoes the widening's 16 x 64
  const float sa = row_ok ? __fmul_rn(__fmul_rn(__ldg(p.scales + row), __ldg(p.alpha)), kAccScale) : 0.0f;
#pragma unroll 1
  for (int c = 0; c < 256; c += 32) {
    uint32_t r[32];
    tmem_ld32(tbase + (uint32_t)c, r);
    const int col0 = n0 + c;
    if (!row_ok) continue;
    if (p.y_mode == 1) {
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
gemm_tern_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW, PParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = base;
  uint8_t* sW = base + kStages * kABytes;
  uint8_t* sP = base + kStages * kStageBytes;  // staging slots of packed bytes
  uint64_t* full = reinterpret_cast<uint64_t*>(sP + kSlots * kSlotBytes);
  uint64_t* empty = full + kStages;
  uint64_t* pfull = empty + kStages;
  uint64_t* pempty = pfull + kSlots;
  uint64_t* tfull = pempty + kSlots;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* exitb = drain + 1;
  uint64_t* drainb = exitb + 1;
  // 4 x 16 bytes, 16-byte aligned for the bulk copies: peer signals land here
  uint8_t* sig = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(drainb + 1) + 15) & ~(uintptr_t)15);
  int* peer_issued = reinterpret_cast<int*>(sig + kConvWarps * kSignalBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(peer_issued + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cid = blockIdx.x >> 1;
  const int ncl = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      // the leader's converter warps arrive; the peer's signal through
      // complete-tx (see the converters)
      mbar_init(&full[s], kConvWarps);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&pfull[s], 1);
      mbar_init(&pempty[s], kConvWarps);
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
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  fence_before();
  cluster_sync_all();
  fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // a programmatic dependent: the codes are the previous kernel's output
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // k-blocks in this cluster's order: tiles cid, cid + ncl, ..., num_kb each
  const int my_tiles = cid < p.num_tiles ? (p.num_tiles - 1 - cid) / ncl + 1 : 0;
  const int total = my_tiles * p.num_kb;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer (packed bytes)
    if (lane == 0) {
      prefetch_tensormap(&tmA);
      prefetch_tensormap(&tmW);
      int issued = 0;
      for (; issued < total; ++issued) {
        const int slot = issued % kSlots;
        if (!wait_bounded(&pempty[slot], ((uint32_t)(issued / kSlots) & 1u) ^ 1u, abort_flag, p.err)) break;
        int mb, nb;
        tile_mn(p, cid + (issued / p.num_kb) * ncl, mb, nb);
        const int kb = issued % p.num_kb;
        uint8_t* dst = sP + slot * kSlotBytes;
        mbar_expect_tx(&pfull[slot], (uint32_t)kSlotBytes);
        tma_load_2d(dst, &tmA, kb * 64, mb * 256 + (int)rank * 128, &pfull[slot]);
        tma_load_2d(dst + kPABytes, &tmW, kb * 32, nb * 256 + (int)rank * 128, &pfull[slot]);
      }
      // the copies issued have landed before the CTA may exit
      drain_loads(pfull, kSlots, issued, p.err);
    }
  } else if (warp < kMmaWarp) {
    // ------------------------------------------------ converters (warps 1-8)
    const int grp = (warp - kConv0) / kConvWarps;        // stages grp, grp + 2, ...
    const int gw = (warp - kConv0) % kConvWarps;         // warp within the group
    const int t = 32 * gw + lane;                        // 0 .. 127
    const uint32_t sA0 = smem_u32(sA), sW0 = smem_u32(sW), sP0 = smem_u32(sP);
    const uint32_t full_addr0 = mapa_shared(smem_u32(&full[0]), 0);
    const uint32_t sig_leader = mapa_shared(smem_u32(sig), 0);  // the leader's signal area
    const uint32_t sig_own = smem_u32(sig);                      // any 16 bytes of this CTA
    for (int g = grp; g < total; g += kConvGroups) {
      const int slot = g % kSlots, stage = g % kStages;
      if (!wait_bounded_warp(&pfull[slot], (uint32_t)(g / kSlots) & 1u, abort_flag, p.err)) break;
      if (!wait_bounded_warp(&empty[stage], ((uint32_t)(g / kStages) & 1u) ^ 1u, abort_flag, p.err)) break;
      widen_stage(sP0 + (uint32_t)(slot * kSlotBytes), sA0 + (uint32_t)(stage * kABytes),
                  sW0 + (uint32_t)(stage * kBBytes), t);
      // The generic-proxy stores are made visible to the tensor cores' proxy
      // (every lane fences its own), then one lane frees the staging slot and
      // signals the stage.  The leader's warps arrive on their own full
      // barrier (the MMA thread's CTA-scope acquire covers their stores); the
      // first also expects the peer's 4 x 16 signal bytes.  A peer warp
      // signals through the async proxy, as a TMA load would: a 16-byte bulk
      // copy into the leader's shared memory whose complete-tx lands on the
      // leader's barrier, issued after its proxy fence.  (A cluster-scope
      // acquire on the leader's side costs about a microsecond per stage and
      // held the tensor pipe at a third of its rate.)
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&pempty[slot]);
        if (leader) {
          if (gw == 0)
            mbar_expect_tx(&full[stage], (uint32_t)(kConvWarps * kSignalBytes));
          else
            mbar_arrive(&full[stage]);
        } else {
          asm volatile(
              "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                  sig_leader + (uint32_t)(gw * kSignalBytes)),
              "r"(sig_own), "n"(kSignalBytes), "r"(full_addr0 + (uint32_t)(stage * 8))
              : "memory");
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------ MMA issuer (leader)
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
          // every converter warp of the pair has signalled this stage
          if (!wait_bounded(&full[stage], phase, abort_flag, p.err)) { ok = false; break; }
          fence_after();
          const uint64_t a0 = sdesc_k_sw128(smem_u32(sA + stage * kABytes));
          const uint64_t b0 = sdesc_k_sw128(smem_u32(sW + stage * kBBytes));
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_i8_pair(d_tmem, a0 + (uint64_t)(2 * k), b0 + (uint64_t)(2 * k), (kb | k) != 0 ? 1u : 0u);
          mma_commit_pair(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
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
    // ------------------------------------------------ epilogue (warps 10-13)
    const int quarter = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = cid; tile < p.num_tiles; tile += ncl) {
      if (!wait_bounded_warp(&tfull[acc], acc_phase, abort_flag, p.err)) break;
      fence_after();
      int m_blk, n_blk;
      tile_mn(p, tile, m_blk, n_blk);
      const int row = m_blk * 256 + (int)rank * 128 + quarter * 32 + lane;
      epilogue_row(p, tmem_base + (uint32_t)(acc * 256) + ((uint32_t)(quarter * 32) << 16), row, n_blk * 256);
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

  // Neither CTA frees its shared memory or TMEM while the pair still uses
  // them (the leader's MMAs read both CTAs' stages; its MMA thread drained
  // them above): a bounded handshake through each other's exit barrier.  Each
  // producer drained its own copies above (they complete on its own barriers).
  fence_before();
  __syncthreads();
  if (threadIdx.x == 0) pair_exit_drain(leader, rank, full, kStages, 0u, 0, peer_issued, exitb, drainb, p.err);
  __syncthreads();
  fence_after();
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

}  // namespace

bool gemm_tern_supports(int64_t M, int64_t K) { return M >= 256 && K >= 64 && K % 64 == 0; }

cudaError_t launch_gemm_tern(const uint8_t* A, const uint8_t* W, int64_t M, int64_t N, int64_t K, int y_mode,
                             void* y, const float* scales, const float* alpha, cudaStream_t stream) {
  if (!gemm_tern_supports(M, K) || (y_mode != 1 && y_mode != 2)) return cudaErrorInvalidValue;
  int* err = device_error_word();
  if (!err) return cudaErrorInvalidValue;
  PParams p;
  p.A = A;
  p.W = W;
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.num_m = (int)((M + 255) / 256);
  p.num_n = (int)((N + 255) / 256);
  p.num_tiles = p.num_m * p.num_n;
  p.num_kb = (int)((K + 127) / 128);
  p.y_mode = y_mode;
  p.y = y;
  p.scales = scales;
  p.alpha = alpha;
  p.err = err;
  // column tiles in groups whose packed W panels (64 K bytes per tile column)
  // fit in about a third of L2
  const int64_t panel = (int64_t)64 * K;
  const int64_t groups = (p.num_n * panel + (int64_t(40) << 20) - 1) / (int64_t(40) << 20);
  p.group_n = groups > 1 ? (int)((p.num_n + groups - 1) / groups) : 0;
  // packed operands as byte matrices, boxes of one k-block x 128 rows, with the
  // swizzle of their row width (unswizzled 64- and 32-byte rows put
  // consecutive rows on the same banks, and the copies ran ~3x slower)
  CUtensorMap ta, tw;
  if (!sm100_host::encode_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, A, (uint64_t)(K / 2), (uint64_t)M, (uint64_t)(K / 2),
                             64, 128, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !sm100_host::encode_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, W, (uint64_t)(K / 4), (uint64_t)N, (uint64_t)(K / 4),
                             32, 128, CU_TENSOR_MAP_SWIZZLE_32B))
    return cudaErrorInvalidValue;
  static std::atomic<bool> smem_set[sm100_host::kMaxDevices];
  cudaError_t e = sm100_host::ensure_smem(gemm_tern_pair_kernel, (int)kSmemBytes, smem_set);
  if (e != cudaSuccess) return e;
  const int pairs = sm100_host::sm_count() / 2;
  const int nclusters = p.num_tiles < pairs ? p.num_tiles : pairs;
  return sm100_host::launch_pdl(gemm_tern_pair_kernel, (unsigned)(2 * nclusters), kThreads, kSmemBytes, stream, 2,
                                ta, tw, p);
}

}  // namespace hbl
