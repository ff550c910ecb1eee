// Decode-sized H-BitLinear forward: the matrix product straight from the
// packed ternary weights with the dequantisation fused ("BitNet v2: Native
// 4-bit Activations with Hadamard Transformation for 1-bit LLMs", section
// "H-BitLinear", matrix-operation formula):
//
//   acc[m][n] = sum_k A[m][k] w[n][k]   A: int8 codes [M][K], w: 2-bit codes [N][K/4]
//   y[m][n]   = (float)acc[m][n] * (scale[m] * alpha)            (float or bf16)
//
// For M <= 4 the work is streaming N K / 4 bytes of weights and widening
// them; the rest is latency.  Two kernels share one design:
//
//   * gemv_stream_kernel: the product from int8 codes in global memory (the
//     stage entry point, and the forward when M K is too large to quantize in
//     every CTA);
//   * decode_forward_kernel: the whole forward in one launch.  Every CTA
//     quantizes the M rows of x itself with the register transform of
//     fht_rows.cuh (the quantizer kernel's arithmetic: t, scales and codes are
//     bit-identical to that kernel's) while its weights stream in.
//
// A CTA takes groups of 32 weight rows.  One thread of the last warp streams
// a group through a ring of kStages shared-memory stages with 2-D TMA loads
// (boxes of 32 rows x 128 bytes, 128-byte swizzle; mbarriers track them).
// The other 15 warps consume the stages: lane l owns row l of the group and
// keeps its int32 sums in registers across K; the warps split the stage's
// 16-byte pieces (64 codes each).  For a piece, every lane reads its row's 16
// bytes (for K >= 512 the swizzle spreads the rows of a quarter-warp over all
// banks; the narrower unswizzled boxes of K = 128 and 256 read 2- and 4-way
// conflicted), splits each word of
// 16 codes into four signed-byte planes (tern_planes: 10 integer operations,
// no widening to one byte per code) and takes dp4a products with the M code
// rows, which sit in shared memory in 16-byte units ordered (row, 16-code
// group, piece), each 4 x 4-byte transposed to match the planes: all lanes
// read the same unit, one broadcast.  At the end of a group
// the warps' partial sums meet in shared memory by integer atomics (exact and
// order-free) and y is stored as whole 32-column rows with the tensor-core
// epilogue's two float products, so y is bit-identical to that path's.
#include <atomic>
#include <cstdint>

#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "fht_rows.cuh"
#include "sm100.cuh"

namespace hbl {
namespace {

using namespace sm100;

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kConsumers = kWarps - 1;  // warps 0 .. 14; warp 15 issues the copies
constexpr int kTransformThreads = 256;  // warps 0 .. 7 quantize (decode_forward_kernel)
constexpr int kGroupRows = 32;          // weight rows per group (one per lane)
constexpr int kBoxBytes = 128;          // box width: one swizzle span
constexpr int kStageBoxes = 4;
constexpr int kStageBytes = kGroupRows * kBoxBytes * kStageBoxes;  // 16 KB
constexpr int kStages = 4;
constexpr int kRingBytes = kStages * kStageBytes;
constexpr int kAccBytes = 2 * kGroupRows * kGemvMaxRows * 4;  // two groups' sums in flight
constexpr int kBarBytes = 2 * kStages * 8 + 16;             // full[], empty[], abort flag

// Shared memory common to both kernels, after the kernel's own leading part
// (1024-byte aligned for the swizzled boxes):
// [ring][acc][codes M K][scales 4 floats][full][empty][abort]
struct StreamSmem {
  uint8_t* ring;
  int* acc;  // [2][32][M] int32
  int4* codes;
  float* scales;
  uint64_t* full;
  uint64_t* empty;
  volatile int* abort_flag;
  __device__ __forceinline__ StreamSmem(unsigned char* base, int M, int K) {
    ring = base;
    acc = reinterpret_cast<int*>(base + kRingBytes);
    codes = reinterpret_cast<int4*>(base + kRingBytes + kAccBytes);
    scales = reinterpret_cast<float*>(base + kRingBytes + kAccBytes + (size_t)M * K);
    full = reinterpret_cast<uint64_t*>(base + kRingBytes + kAccBytes + (size_t)M * K + 16);
    empty = full + kStages;
    abort_flag = reinterpret_cast<volatile int*>(empty + kStages);
  }
};

constexpr size_t stream_smem_bytes(int64_t M, int64_t K) {
  return kRingBytes + kAccBytes + (size_t)(M * K) + 16 + kBarBytes;
}

// The walk of one CTA: its groups g = blockIdx.x + i gridDim.x, each in nks
// stages (chunks) of bps boxes of `box` bytes per row.
struct Walk {
  int box, bps, nks, pps, stage_bytes, nchunks, P;
  bool swz;
  __device__ __forceinline__ Walk(int N, int K) {
    P = K / 64;
    const int rowbytes = K / 4;
    box = rowbytes < kBoxBytes ? rowbytes : kBoxBytes;
    const int nb = rowbytes / box;  // boxes per row
    bps = nb < kStageBoxes ? nb : kStageBoxes;
    nks = nb / bps;
    pps = bps * box / 16;
    stage_bytes = kGroupRows * box * bps;
    swz = box == kBoxBytes;
    const int ngroups = (N + kGroupRows - 1) / kGroupRows;
    const int mine = ngroups > (int)blockIdx.x ? (ngroups - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    nchunks = mine * nks;
  }
  __device__ __forceinline__ int group_of(int c) const { return (int)blockIdx.x + (c / nks) * (int)gridDim.x; }
};

// 16 ternary codes of one packed word (code i at bits 2i: 00 = 0, 01 = +1,
// 11 = -1) as four words of signed bytes without widening: byte j of X[f] is
// 4^f w_{4j+f}.  Field f's two bits already sit at bits 2f, 2f+1 of byte j;
// for -1 (bits 11) the bits above them are filled by multiplying the high bit
// by a constant that stays inside the byte (2 x 0x7E = 0xFC, 8 x 0x1E = 0xF0,
// 32 x 6 = 0xC0; field 3's 0xC0 is -64 as it stands).
__device__ __forceinline__ void tern_planes(uint32_t W, int (&X)[4]) {
  X[0] = (int)((W & 0x03030303u) | ((W & 0x02020202u) * 0x7Eu));
  X[1] = (int)((W & 0x0C0C0C0Cu) | ((W & 0x08080808u) * 0x1Eu));
  X[2] = (int)((W & 0x30303030u) | ((W & 0x20202020u) * 0x06u));
  X[3] = (int)(W & 0xC0C0C0C0u);
}

// 16 int8 codes (word j = codes 4j .. 4j+3) -> word f = codes f, 4+f, 8+f,
// 12+f: the activation side of tern_planes, so that dp4a(X[f], A[f]) =
// 4^f sum_j w_{4j+f} a_{4j+f}.
__device__ __forceinline__ int4 transpose4x4(int4 u) {
  const uint32_t t0 = __byte_perm((uint32_t)u.x, (uint32_t)u.y, 0x5140);
  const uint32_t t1 = __byte_perm((uint32_t)u.x, (uint32_t)u.y, 0x7362);
  const uint32_t t2 = __byte_perm((uint32_t)u.z, (uint32_t)u.w, 0x5140);
  const uint32_t t3 = __byte_perm((uint32_t)u.z, (uint32_t)u.w, 0x7362);
  return make_int4((int)__byte_perm(t0, t2, 0x5410), (int)__byte_perm(t0, t2, 0x7632),
                   (int)__byte_perm(t1, t3, 0x5410), (int)__byte_perm(t1, t3, 0x7632));
}

// Thread 0 of the CTA: barriers for the ring, sums to zero.
__device__ __forceinline__ void init_ring(const StreamSmem& sm, int M) {
  for (int s = 0; s < kStages; ++s) {
    mbar_init(&sm.full[s], 1);
    mbar_init(&sm.empty[s], kConsumers);
  }
  *sm.abort_flag = 0;
  for (int i = 0; i < 2 * kGroupRows * M; ++i) sm.acc[i] = 0;
  fence_proxy_async_smem();
}

// Warp 15's lane 0: every chunk of the walk, each stage refilled once all
// consumer warps have released it; then it waits for its copies to land (the
// exit drain), so no copy outlives the CTA.
__device__ __forceinline__ void produce(const StreamSmem& sm, const Walk& wk, const CUtensorMap* tm, int* err) {
  prefetch_tensormap(tm);
  int issued = 0;
  for (int c = 0; c < wk.nchunks; ++c) {
    const int s = c % kStages;
    if (c >= kStages && !wait_bounded(&sm.empty[s], (uint32_t)(c / kStages - 1) & 1u, sm.abort_flag, err)) break;
    const int g = wk.group_of(c), ks = c % wk.nks;
    mbar_expect_tx(&sm.full[s], (uint32_t)wk.stage_bytes);
    uint8_t* dst = sm.ring + (size_t)s * kStageBytes;
    for (int b = 0; b < wk.bps; ++b)
      tma_load_2d(dst + b * kGroupRows * wk.box, tm, (ks * wk.bps + b) * wk.box, g * kGroupRows, &sm.full[s]);
    ++issued;
  }
  drain_loads(sm.full, kStages, issued, err);
}

// The consumer warps (0 .. 14) pass through every chunk in order: each waits
// for the chunk, takes pieces warp, warp + 15, ... of it and releases the
// stage.  Every warp waits for and releases every stage, so none can run a
// full ring ahead or be lapped.  At the end of each group the sums meet in
// shared memory (buffer i & 1 for the CTA's i-th group) and, after a barrier
// of the consumer warps, the first 32 M threads store y and clear the buffer
// (its next use comes after the next group's barrier).
template <int MT>
__device__ __forceinline__ void consume(const StreamSmem& sm, const Walk& wk, float alpha, int M, int N, void* y,
                                        int y_mode, int* err) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cpb = wk.box / 16;  // 16-byte pieces per box row
  // acc[m][f]: 4^f times the sums of field f (tern_planes); combined exactly
  // at the end of a group
  int acc[MT][4];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int f = 0; f < 4; ++f) acc[m][f] = 0;
  bool ok = true;
  for (int c = 0; c < wk.nchunks; ++c) {
    const int s = c % kStages;
    const int ks = c % wk.nks;
    if (ok && !wait_bounded_warp(&sm.full[s], (uint32_t)(c / kStages) & 1u, sm.abort_flag, err)) ok = false;
    if (ok) {
      const uint8_t* st = sm.ring + (size_t)s * kStageBytes;
      for (int pl = warp; pl < wk.pps; pl += kConsumers) {
        const int b = pl / cpb, c16 = pl % cpb;
        const int off = b * kGroupRows * wk.box + lane * wk.box + ((wk.swz ? (c16 ^ (lane & 7)) : c16) << 4);
        const uint4 w = *reinterpret_cast<const uint4*>(st + off);
        const int p = ks * wk.pps + pl;  // piece of the row
        const uint32_t wq[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          int X[4];
          tern_planes(wq[jj], X);  // k = 64 p + 16 jj .. + 15
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            if (m < M) {
              const int4 qv = sm.codes[(m * 4 + jj) * wk.P + p];  // the same unit for every lane (transposed)
              acc[m][0] = __dp4a(X[0], qv.x, acc[m][0]);
              acc[m][1] = __dp4a(X[1], qv.y, acc[m][1]);
              acc[m][2] = __dp4a(X[2], qv.z, acc[m][2]);
              acc[m][3] = __dp4a(X[3], qv.w, acc[m][3]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[s]);
    }
    if (ks == wk.nks - 1) {
      // the group's sums: every consumer warp adds its part, then y
      const int i = c / wk.nks;
      int* buf = sm.acc + (i & 1) * kGroupRows * M;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        // each acc[m][f] is a multiple of 4^f: the shifts are exact
        const int v = acc[m][0] + (acc[m][1] >> 2) + (acc[m][2] >> 4) + (acc[m][3] >> 6);
        if (m < M && v != 0) atomicAdd(buf + lane * M + m, v);
#pragma unroll
        for (int f = 0; f < 4; ++f) acc[m][f] = 0;
      }
      named_bar_sync(2, kConsumers * 32);
      if (threadIdx.x < kGroupRows * M) {
        const int r = threadIdx.x % kGroupRows, m = threadIdx.x / kGroupRows;
        const int n = wk.group_of(c) * kGroupRows + r;
        if (ok && n < N) {
          const float yv = (float)buf[r * M + m] * (sm.scales[m] * alpha);
          const size_t o = (size_t)m * N + n;
          if (y_mode == 2)
            reinterpret_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(yv);
          else
            reinterpret_cast<float*>(y)[o] = yv;
        }
        buf[r * M + m] = 0;
      }
    }
  }
}

// ---------------------------------------------------------------- product from int8 codes

// Codes [M][K] int8 and scales [M] from global memory.  `early` (the codes'
// producer is the preceding kernel of the same forward, and everything before
// that kernel has completed): the weight copies start before the programmatic
// dependency wait, overlapping that kernel; otherwise after it.
template <int MT>
__global__ void __launch_bounds__(kThreads, 1)
gemv_stream_kernel(const __grid_constant__ CUtensorMap tmW, const int8_t* __restrict__ A,
                   const float* __restrict__ scales, const float* __restrict__ alpha, void* __restrict__ y, int M,
                   int N, int K, int y_mode, int early, int* err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const StreamSmem sm(base, M, K);
  const Walk wk(N, K);
  const int tid = threadIdx.x;
  if (tid == 0) init_ring(sm, M);
  __syncthreads();
  if (tid >= kConsumers * 32) {
    // the producer warp: the weights do not depend on the codes' kernel
    if (!early) asm volatile("griddepcontrol.wait;" ::: "memory");
    if (tid == kConsumers * 32) produce(sm, wk, &tmW, err);
    return;
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // the code rows into shared memory, reordered into (row, group, piece) units
  const int P = K / 64;
  for (int u = tid; u < M * K / 16; u += kConsumers * 32) {
    const int m = u / (K / 16), q = u % (K / 16);
    sm.codes[(m * 4 + (q & 3)) * P + (q >> 2)] = transpose4x4(__ldg(reinterpret_cast<const int4*>(A) + u));
  }
  if (tid < M) sm.scales[tid] = __ldg(scales + tid);
  named_bar_sync(1, kConsumers * 32);
  consume<MT>(sm, wk, __ldg(alpha), M, N, y, y_mode, err);
}

// ---------------------------------------------------------------- the whole forward in one launch

// Rows of the transform per pass: at least MT, and whole warps.
template <int LOGK, int MT>
struct DecodeShape {
  static constexpr int T = (1 << LOGK) / 64;
  static constexpr int R0 = MT > 32 / T ? MT : (32 / T > 0 ? 32 / T : 1);
  static constexpr int R = R0 * T <= kTransformThreads ? R0 : kTransformThreads / T;
  using S = fhtrows::ShapeR<LOGK, R>;
  static constexpr size_t LEAD = (S::XCH + 2 * S::RED + 15) / 16 * 16;  // exchange + reduction slots
};

template <int LOGK, int MT>
__global__ void __launch_bounds__(kThreads, 1)
decode_forward_kernel(const __grid_constant__ CUtensorMap tmW, const void* __restrict__ x, int x_bf16, int M,
                      float sK, int bits, const float* __restrict__ alpha, void* __restrict__ y, int y_mode, int N,
                      int* err) {
  using D = DecodeShape<LOGK, MT>;
  using S = typename D::S;
  using Bar = fhtrows::BarNamed<1, S::R * S::T>;
  constexpr int K = S::K, T = S::T, R = S::R;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const StreamSmem sm(base, M, K);
  float* xch = reinterpret_cast<float*>(base + stream_smem_bytes(M, K));
  float* red1 = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(xch) + S::XCH);
  void* red2 = reinterpret_cast<unsigned char*>(xch) + S::XCH + S::RED;
  const Walk wk(N, K);
  const int tid = threadIdx.x;
  if (tid == 0) init_ring(sm, M);
  __syncthreads();
  // x and the weights may be the previous kernel's output: wait for it
  // before any load, then let the stream's next kernel begin its setup
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (tid >= kConsumers * 32) {
    // the producer warp: the weights stream in while the rows are quantized
    if (tid == kConsumers * 32) produce(sm, wk, &tmW, err);
    return;
  }

  // ---- quantize the M rows, R at a time, into shared memory
  if (tid < R * T) {
    const int rl = tid / T, t = tid % T;
    const int P = K / 64;
    for (int g = 0; g < M; g += R) {
      const int row = g + rl;
      const bool active = row < M;
      const bool compute = __any_sync(0xffffffffu, active);  // warp-uniform
      float e[64];
      if (x_bf16) {
        const void* xrow = reinterpret_cast<const uint16_t*>(x) + (size_t)(active ? row : 0) * K;
        fhtrows::fht_ln_rows<S, true, true, Bar>(xrow, active, rl, t, xch, red1, sK, e, compute);
      } else {
        const void* xrow = reinterpret_cast<const float*>(x) + (size_t)(active ? row : 0) * K;
        fhtrows::fht_ln_rows<S, false, true, Bar>(xrow, active, rl, t, xch, red1, sK, e, compute);
      }
      uint32_t w[16];
      q::RowParams p;
      if (bits == 4) {
        p = fhtrows::row_params<S, K1_Q4_I8, Bar>(e, red2, rl, t, compute);
        if (active) fhtrows::codes64_i8<K1_Q4_I8>(e, p.r, w);
      } else {
        p = fhtrows::row_params<S, K1_Q8_I8, Bar>(e, red2, rl, t, compute);
        if (active) fhtrows::codes64_i8<K1_Q8_I8>(e, p.r, w);
      }
      if (active) {
        if (t == 0) sm.scales[row] = p.scale();
        // this thread's 64 codes are piece t of the row: units (row, jj, t)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
          sm.codes[(row * 4 + jj) * P + t] = transpose4x4(
              make_int4((int)w[4 * jj], (int)w[4 * jj + 1], (int)w[4 * jj + 2], (int)w[4 * jj + 3]));
      }
      Bar::sync();  // the exchange and reduction slots are free for the next rows
    }
  }
  named_bar_sync(2, kConsumers * 32);  // codes and scales visible to every consumer warp
  consume<MT>(sm, wk, __ldg(alpha), M, N, y, y_mode, err);
}

// ---------------------------------------------------------------- launches

// The packed weight [N][K/4] as a 2-D byte tensor: boxes of 32 rows x
// min(128, K/4) bytes, swizzled when 128 bytes wide.
bool weight_map(CUtensorMap* map, const uint8_t* packed, int64_t N, int64_t K) {
  const uint32_t box = (uint32_t)(K / 4 < kBoxBytes ? K / 4 : kBoxBytes);
  return sm100_host::encode_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, (uint64_t)(K / 4), (uint64_t)N,
                               (uint64_t)(K / 4), box, (uint32_t)kGroupRows,
                               box == kBoxBytes ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE);
}

// One CTA per SM at most, groups of 32 rows dealt round robin.
inline int stream_grid(int64_t N) {
  const int64_t groups = (N + kGroupRows - 1) / kGroupRows;
  const int64_t sms = sm100_host::sm_count();
  return (int)(groups < sms ? groups : sms);
}

constexpr size_t kStreamSmemMax = 1024 + kRingBytes + kAccBytes + kGemvMaxCodeBytes + 16 + kBarBytes;
static_assert(kStreamSmemMax <= 227 * 1024, "shared memory");

template <int MT>
cudaError_t launch_stream(const int8_t* A, const float* scales, const uint8_t* packed, const float* alpha, void* y,
                          int y_mode, int M, int N, int K, bool early, cudaStream_t stream) {
  static std::atomic<bool> smem_set[sm100_host::kMaxDevices];
  cudaError_t e = sm100_host::ensure_smem(gemv_stream_kernel<MT>, (int)kStreamSmemMax, smem_set);
  if (e != cudaSuccess) return e;
  CUtensorMap tm;
  if (!weight_map(&tm, packed, N, K)) return cudaErrorInvalidValue;
  return sm100_host::launch_pdl(gemv_stream_kernel<MT>, (unsigned)stream_grid(N), (unsigned)kThreads,
                                1024 + stream_smem_bytes(M, K), stream, 1u, tm, A, scales, alpha, y, M, N, K, y_mode,
                                early ? 1 : 0, device_error_word());
}

template <int LOGK, int MT>
cudaError_t launch_decode(const void* x, bool x_bf16, int M, int bits, const uint8_t* packed, const float* alpha,
                          void* y, int y_mode, int N, cudaStream_t stream) {
  using D = DecodeShape<LOGK, MT>;
  constexpr int K = 1 << LOGK;
  constexpr size_t max_codes =
      (size_t)MT * K < (size_t)kDecodeFusedMaxCodes ? (size_t)MT * K : (size_t)kDecodeFusedMaxCodes;
  constexpr size_t max_smem = 1024 + stream_smem_bytes(0, 0) + max_codes + D::LEAD;
  static_assert(max_smem <= 227 * 1024, "shared memory");
  auto kern = decode_forward_kernel<LOGK, MT>;
  static std::atomic<bool> smem_set[sm100_host::kMaxDevices];
  cudaError_t e = sm100_host::ensure_smem(kern, (int)max_smem, smem_set);
  if (e != cudaSuccess) return e;
  CUtensorMap tm;
  if (!weight_map(&tm, packed, N, K)) return cudaErrorInvalidValue;
  const float sK = (float)(1.0 / sqrt((double)K));
  return sm100_host::launch_pdl(kern, (unsigned)stream_grid(N), (unsigned)kThreads,
                                1024 + stream_smem_bytes(M, K) + D::LEAD, stream, 1u, tm, x, x_bf16 ? 1 : 0, M, sK,
                                bits, alpha, y, y_mode, N, device_error_word());
}

template <int LOGK>
cudaError_t launch_decode_k(const void* x, bool x_bf16, int M, int bits, const uint8_t* packed, const float* alpha,
                            void* y, int y_mode, int N, cudaStream_t stream) {
  if constexpr ((1 << LOGK) <= kDecodeFusedMaxCodes) {
    if (M <= 1) return launch_decode<LOGK, 1>(x, x_bf16, M, bits, packed, alpha, y, y_mode, N, stream);
    return launch_decode<LOGK, 4>(x, x_bf16, M, bits, packed, alpha, y, y_mode, N, stream);
  }
  return cudaErrorInvalidValue;  // decode_forward_supports excludes these sizes
}

}  // namespace

bool gemv_ternary_supports(int64_t M, int64_t K) {
  return M >= 1 && M <= kGemvMaxRows && M * K <= kGemvMaxCodeBytes && K >= 64 && K <= 32768 && (K & (K - 1)) == 0;
}

cudaError_t launch_gemv_ternary(const int8_t* A, const float* scales, const uint8_t* packed, const float* alpha,
                                int64_t M, int64_t N, int64_t K, int y_mode, void* y, cudaStream_t stream,
                                bool early) {
  if (!gemv_ternary_supports(M, K) || (y_mode != 1 && y_mode != 2)) return cudaErrorInvalidValue;
  const int m = (int)M, n = (int)N, k = (int)K;
  if (m <= 1) return launch_stream<1>(A, scales, packed, alpha, y, y_mode, m, n, k, early, stream);
  return launch_stream<4>(A, scales, packed, alpha, y, y_mode, m, n, k, early, stream);
}

bool decode_forward_supports(int64_t M, int64_t K) {
  return gemv_ternary_supports(M, K) && M * K <= kDecodeFusedMaxCodes;
}

cudaError_t launch_decode_forward(const void* x, bool x_bf16, int64_t M, int log2k, int bits, const uint8_t* packed,
                                  const float* alpha, int64_t N, int y_mode, void* y, cudaStream_t stream) {
  if (!decode_forward_supports(M, (int64_t)1 << log2k) || (y_mode != 1 && y_mode != 2) || (bits != 4 && bits != 8))
    return cudaErrorInvalidValue;
  const int m = (int)M, n = (int)N;
  switch (log2k) {
    case 6: return launch_decode_k<6>(x, x_bf16, m, bits, packed, alpha, y, y_mode, n, stream);
    case 7: return launch_decode_k<7>(x, x_bf16, m, bits, packed, alpha, y, y_mode, n, stream);
    case 8: return launch_decode_k<8>(x, x_bf16, m, bits, packed, alpha, y, y_mode, n, stream);
    case 9: return launch_decode_k<9>(x, x_bf16, m, bits, packed, alpha, y, y_mode, n, stream);
    case 10: return launch_decode_k<10>(x, x_bf16, m, bits, packed, alpha, y, y_mode, n, stream);
    case 11: return launch_decode_k<11>(x, x_bf16, m, bits, packed, alpha, y, y_mode, n, stream);
    case 12: return launch_decode_k<12>(x, x_bf16, m, bits, packed, alpha, y, y_mode, n, stream);
    case 13: return launch_decode_k<13>(x, x_bf16, m, bits, packed, alpha, y, y_mode, n, stream);
    case 14: return launch_decode_k<14>(x, x_bf16, m, bits, packed, alpha, y, y_mode, n, stream);
    case 15: return launch_decode_k<15>(x, x_bf16, m, bits, packed, alpha, y, y_mode, n, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace hbl
