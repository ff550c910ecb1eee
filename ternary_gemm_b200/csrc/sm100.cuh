// sm_100a building blocks shared by the tensor-core kernels: mbarriers with
// bounded waits, TMA tile copies, bulk-group bookkeeping, tcgen05 (TMEM
// allocation, MMA commit, TMEM loads) and UMMA shared-memory descriptors,
// plus the host-side tensor-map encoder.  Inline PTX only; no multicast
// loads anywhere.
#pragma once

#include <atomic>
#include <cstdint>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

namespace hbl {
namespace sm100 {

constexpr uint64_t kWaitLimitNs = 2000000000ull;   // default limit of the pipeline waits (2 s)
constexpr uint64_t kDrainLimitNs = 2000000000ull;  // limit of the exit-path drains (never shortened)

// The library's device status, one per device: the error flag that a bounded
// wait sets when it gives up, and the limit of the pipeline waits (kernels
// receive the address of `error`).  The limit is kWaitLimitNs unless a test
// shortens it through the host API to make a wait run out.
struct DeviceStatus {
  int error;
  int reserved;
  unsigned long long wait_limit_ns;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarriers

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait that may suspend the thread for up to `hint_ns` (it returns as
// soon as the phase completes): long waits cost a few issue slots instead of
// a spin loop's.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// wait_bounded for a whole warp (every lane executes it and gets the same
// answer), suspending between polls: for consumers whose wait covers a whole
// pipeline step.
__device__ __forceinline__ bool wait_bounded_warp(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                  int* err) {
  if (mbar_try_wait_hint(bar, parity, 20000u)) return true;
  const uint64_t limit = reinterpret_cast<const volatile DeviceStatus*>(err)->wait_limit_ns;
  const uint64_t t0 = globaltimer();
  for (;;) {
    if (mbar_try_wait_hint(bar, parity, 20000u)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > limit) {
      *abort_flag = 1;
      atomicExch(err, 1);
      return false;
    }
  }
}

// Bounded wait for the phase with the given parity.  Returns false if the
// CTA already aborted or the limit (the device status's wait_limit_ns) ran
// out; then the CTA abort flag and the device error word are set.  `err`
// points at DeviceStatus::error.
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t limit = reinterpret_cast<const volatile DeviceStatus*>(err)->wait_limit_ns;
  const uint64_t t0 = globaltimer();
  for (uint32_t i = 1;; ++i) {
    // suspend (up to 2 us, woken when the phase completes) instead of
    // spinning: the polling thread shares its SM sub-partition with the
    // consumers' warps
    if (mbar_try_wait_hint(bar, parity, 2000u)) return true;
    if ((i & 63u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > limit) {
        *abort_flag = 1;
        atomicExch(err, 1);
        return false;
      }
    }
  }
}

// Exit-path wait for a phase that copies or commits already issued will
// complete, bounded by kDrainLimitNs whatever the pipeline limit is, so that
// a CTA that gave up still lets its copies land before it exits.
__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity, int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > kDrainLimitNs) {
      atomicExch(err, 1);
      return false;
    }
  }
  return true;
}

// A producer's exit drain: issue i of a ring of `stages` stages used stage
// i % stages in phase i / stages; the loads of the last min(issued, stages)
// issues are waited for (every earlier phase was consumed before a later
// issue reused its stage).  On the normal path these phases are complete or
// about to be, so the drain costs at most the last loads' latency.
__device__ __forceinline__ void drain_loads(uint64_t* full, int stages, int issued, int* err) {
  for (int i = issued > stages ? issued - stages : 0; i < issued; ++i)
    drain_wait(&full[i % stages], (uint32_t)(i / stages) & 1u, err);
}

// ---------------------------------------------------------------- named barriers

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Barrier over `nthreads` threads that also returns whether any of them
// passed pred != 0.
__device__ __forceinline__ bool named_bar_any(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// ---------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"((uint64_t)map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Shared -> global tile store (x aligned to 16 bytes, x, y >= 0).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"((uint64_t)map),
               "r"(x), "r"(y), "r"(smem_u32(src))
               : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// the shared-memory sources of all committed stores have been read
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// all committed stores have completed
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// generic-proxy writes to shared memory -> visible to the async proxy (TMA, tensor cores)
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)map) : "memory");
}

// ---------------------------------------------------------------- tcgen05

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// whole warp; the allocated base column lands in *slot
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)), "r"(cols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t base, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(cols) : "memory");
}

// arrive once on `bar` when all tcgen05.mma issued so far by this thread complete
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// 32 consecutive columns of this warp's TMEM lane quarter (one lane per thread)
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 consecutive columns of this warp's TMEM lane quarter from registers
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  tmem_ld32_nowait(taddr, r);
  tmem_wait_ld();
}

// ---------------------------------------------------------------- clusters and CTA pairs

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// try_wait with cluster-scope acquire: writes that another CTA of the cluster
// made before its release-arrive on this barrier are visible afterwards
__device__ __forceinline__ bool mbar_try_wait_acq_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// wait_bounded with cluster-scope acquire, for a barrier that threads of the
// other CTA of the cluster arrive on after their own shared-memory stores
__device__ __forceinline__ bool wait_bounded_cluster(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                     int* err) {
  if (mbar_try_wait_acq_cluster(bar, parity)) return true;
  const uint64_t limit = reinterpret_cast<const volatile DeviceStatus*>(err)->wait_limit_ns;
  const uint64_t t0 = globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait_acq_cluster(bar, parity)) return true;
    if ((i & 63u) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > limit) {
        *abort_flag = 1;
        atomicExch(err, 1);
        return false;
      }
    }
  }
}

// complete-tx of `bytes` on a local barrier without a copy: stands in for
// bytes a copy that was never issued would have delivered
__device__ __forceinline__ void mbar_complete_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.complete_tx.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void st_shared_cluster_u32(uint32_t cluster_addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}

// Exit of a CTA pair (cta_group::2 kernels), run by thread 0 of each CTA after
// every role has left its loop.  Both CTAs' loads complete on the leader's
// `full` barriers (the leader arms each phase with both CTAs' bytes), so the
// leader drains for both, after learning how many stages the peer issued:
//   * a phase both issued: wait for it;
//   * a phase the leader armed that the peer never loaded: complete the
//     peer's bytes by hand, then wait for the leader's own;
//   * a phase the peer loaded that the leader never armed: arm it for the
//     peer's bytes (arrive + expect-tx), then wait.
// Each CTA issues at most `stages` stages beyond the other (a stage is reused
// only after the MMA consumed it, which needed both halves), so the last
// `stages` issues of the further one cover every phase that can be open.
// The peer leaves only when the leader reports the drain done, so neither
// CTA frees its shared memory while a copy into it is in flight.  Every wait
// is bounded by kDrainLimitNs.
__device__ __forceinline__ void pair_exit_drain(bool leader, uint32_t rank, uint64_t* full, int stages,
                                                uint32_t peer_stage_bytes, int issued, int* peer_issued,
                                                uint64_t* exitb, uint64_t* drainb, int* err) {
  if (!leader) st_shared_cluster_u32(mapa_shared(smem_u32(peer_issued), 0), (uint32_t)issued);
  mbar_arrive_cluster(mapa_shared(smem_u32(exitb), rank ^ 1u));
  bool met = true;
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait_acq_cluster(exitb, 0)) {
    if (globaltimer() - t0 > kDrainLimitNs) {
      atomicExch(err, 1);
      met = false;
      break;
    }
  }
  if (leader) {
    const int ip = met ? *reinterpret_cast<volatile int*>(peer_issued) : issued;
    const int last = issued > ip ? issued : ip;
    for (int i = last > stages ? last - stages : 0; i < last; ++i) {
      uint64_t* bar = &full[i % stages];
      const bool armed = i < issued, loaded = i < ip;
      if (armed && !loaded) mbar_complete_tx(bar, peer_stage_bytes);
      if (!armed && loaded) mbar_expect_tx(bar, peer_stage_bytes);
      drain_wait(bar, (uint32_t)(i / stages) & 1u, err);
    }
    mbar_arrive_cluster(mapa_shared(smem_u32(drainb), 1));
  } else if (met) {
    const uint64_t t1 = globaltimer();
    while (!mbar_try_wait_acq_cluster(drainb, 0)) {
      if (globaltimer() - t1 > kDrainLimitNs) {
        atomicExch(err, 1);
        break;
      }
    }
  }
}

__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, int x, int y, uint32_t leader_bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(dst)),
      "l"((uint64_t)map), "r"(x), "r"(y), "r"(leader_bar)
      : "memory");
}

// The same load with an L2 eviction priority (a policy from createpolicy).
__device__ __forceinline__ void tma_load_2d_pair_hint(void* dst, const CUtensorMap* map, int x, int y,
                                                      uint32_t leader_bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"((uint64_t)map), "r"(x), "r"(y), "r"(leader_bar), "l"(policy)
      : "memory");
}

// L2 eviction policies for whole accesses: kept past normal lines, or
// evicted first.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// arrive on the barrier at this offset in both CTAs of the pair once the
// leader's outstanding MMAs complete
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"((uint16_t)0x3)
      : "memory");
}

__device__ __forceinline__ void mma_commit_local2(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// UMMA shared-memory descriptor of a K-major tile in the 128-byte-swizzled
// layout TMA writes (rows of 128 bytes, 8-row atoms of 1024 bytes): stride
// byte offset 1024, leading byte offset unused (1), version 1, layout type 2
// (SWIZZLE_128B).  Stepping K inside the 128-byte row adds bytes/16 to it.
__device__ __forceinline__ uint64_t sdesc_k_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// MN-major 128-byte-swizzled tile: 64 contiguous 16-bit MN elements per
// 128-byte row, one row per K index, 8-row atoms of 1024 bytes.  Leading byte
// offset = distance between 64-element MN blocks, stride byte offset =
// distance between 8-row K groups (1024).  Stepping K by 16 adds 2048 bytes.
__device__ __forceinline__ uint64_t sdesc_mn_sw128(uint32_t saddr, uint32_t mn_block_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((mn_block_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

}  // namespace sm100

// ---------------------------------------------------------------- host side

namespace sm100_host {

inline PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }();
  return fn;
}

// 2-D row-major tensor map: `rows` rows of `inner` elements, `row_bytes`
// apart; box `box_inner` x `box_rows`; zero fill out of bounds.
inline bool encode_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* ptr, uint64_t inner, uint64_t rows,
                      uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  auto encode = encoder();
  if (!encode) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, dtype, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

constexpr int kMaxDevices = 64;

// The per-device caches below are arrays of atomics: several host threads
// may make their first calls at once, and each stores the same value.

// SM count of the current device, queried once per device.
inline int sm_count() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < kMaxDevices) {
    const int c = cache[dev].load(std::memory_order_acquire);
    if (c > 0) return c;
  }
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  if (dev >= 0 && dev < kMaxDevices) cache[dev].store(n, std::memory_order_release);
  return n;
}

// Dynamic shared memory limit of a kernel, set once per device: `done` is the
// call site's own per-device flag array (one per kernel instantiation).
template <typename Kernel>
inline cudaError_t ensure_smem(Kernel kern, int bytes, std::atomic<bool> (&done)[kMaxDevices]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < kMaxDevices && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev >= 0 && dev < kMaxDevices) done[dev].store(true, std::memory_order_release);
  return e;
}

// Launch as a programmatic dependent of the stream's previous kernel: the
// grid may be scheduled once that kernel's blocks have all issued
// griddepcontrol.launch_dependents (or exited), so this kernel's setup
// overlaps the other's tail.  The kernel itself must execute
// griddepcontrol.wait before it touches memory the previous kernel reads or
// writes.  `cluster` > 1 adds a cluster dimension.
template <typename Kernel, typename... Args>
inline cudaError_t launch_pdl(Kernel kern, unsigned grid, unsigned block, size_t smem, cudaStream_t stream,
                              unsigned cluster, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(block, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  unsigned n = 1;
  if (cluster > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace sm100_host
}  // namespace hbl
