// Small-M H-BitLinear matrix product straight from the packed ternary
// weights, with the dequantisation fused ("BitNet v2: Native 4-bit
// Activations with Hadamard Transformation for 1-bit LLMs", section
// "H-BitLinear", matrix-operation formula):
//
//   acc[m][n] = sum_k A[m][k] w[n][k]   A: int8 codes [M][K], w: 2-bit codes [N][K/4]
//   y[m][n]   = (float)acc[m][n] * (scale[m] * alpha)            (float or bf16)
//
// For decode-sized batches the tensor-core path is dominated by widening the
// whole weight to int8 and by its 256-column output tiles (N / 256 CTAs).
// Here a CTA owns 32 weight rows, one per lane, and its 16 warps split K:
// each lane streams its row 16 bytes (64 codes) at a time, widens them in
// registers (tern::widen16), loads running ahead of their use, and takes
// dp4a products with the M code rows,
// which the CTA first copies into shared memory (M K <= 64 KB) and every lane
// reads at the same address (one broadcast each).  The warps' int32 partial sums meet in
// shared memory and the first warp rescales and stores y with coalesced
// 32-column rows.  The 2-bit weights are read once (N K / 4 bytes); the sums
// are exact and the dequantisation is the tensor-core epilogue's, so y is
// identical to that path's.  It is launched as a programmatic dependent of
// the quantizer kernel before it: the weight loads start while that kernel
// finishes, and griddepcontrol.wait holds the code reads until its results
// are visible.
#include <cstdint>

#include <cuda_bf16.h>

#include "common.cuh"
#include "sm100.cuh"
#include "ternary.cuh"

namespace hbl {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kRowsPerCta = 32;
constexpr int kAhead = 4;  // weight loads in flight per lane

// MT >= M code rows (rows m >= M are skipped); YMODE 1 float, 2 bf16.
template <int MT, int YMODE>
__global__ void __launch_bounds__(kThreads)
gemv_ternary_kernel(const int8_t* __restrict__ A, const float* __restrict__ scales,
                    const uint4* __restrict__ packed, const float* __restrict__ alpha, void* __restrict__ y, int M,
                    int N, int K) {
  __shared__ int part[kWarps][MT][kRowsPerCta];
  extern __shared__ int4 sA[];  // the M code rows, M K bytes
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int n = blockIdx.x * kRowsPerCta + lane;
  const int steps = K / 64;                                // 16-byte loads per weight row
  const int per_warp = (steps + kWarps - 1) / kWarps;      // a contiguous K slice per warp
  const int st0 = warp * per_warp;
  const int st1 = min(steps, st0 + per_warp);
  int acc[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) acc[m] = 0;
  const uint4* wrow = packed + (size_t)(n < N ? n : 0) * steps;
  // kAhead steps of weight codes are requested before any is used, and the
  // next kAhead while these are consumed, so DRAM latency is paid about once
  uint4 wv[kAhead], wn[kAhead];
  auto load = [&](uint4 (&dst)[kAhead], int sc) {
#pragma unroll
    for (int u = 0; u < kAhead; ++u)
      dst[u] = (n < N && sc + u < st1) ? __ldg(wrow + sc + u) : make_uint4(0u, 0u, 0u, 0u);
  };
  load(wv, st0);
  // The weights do not depend on the preceding kernel of the stream; its
  // codes and scales do.  Under a programmatic dependent launch this waits
  // for that kernel's results (a no-op otherwise).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // the code rows into shared memory once per CTA: every weight row of the
  // CTA reads all of them (broadcast reads below)
  for (int i = threadIdx.x; i < M * K / 16; i += kThreads) sA[i] = __ldg(reinterpret_cast<const int4*>(A) + i);
  __syncthreads();
  for (int sc = st0; sc < st1; sc += kAhead) {
    if (sc + kAhead < st1) load(wn, sc + kAhead);
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
      if (n < N && sc + u < st1) {
        const int st = sc + u;  // codes k = 64 st .. 64 st + 63
        const uint32_t wq[4] = {wv[u].x, wv[u].y, wv[u].z, wv[u].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 e = tern::widen16(wq[j]);  // k = 64 st + 16 j .. + 15
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            if (m < M) {
              // the same 16 bytes for every lane: one broadcast read
              const int4 qv = sA[(m * K + 64 * st + 16 * j) / 16];
              acc[m] = __dp4a(qv.x, (int)e.x, acc[m]);
              acc[m] = __dp4a(qv.y, (int)e.y, acc[m]);
              acc[m] = __dp4a(qv.z, (int)e.z, acc[m]);
              acc[m] = __dp4a(qv.w, (int)e.w, acc[m]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kAhead; ++u) wv[u] = wn[u];
  }
#pragma unroll
  for (int m = 0; m < MT; ++m) part[warp][m][lane] = acc[m];
  __syncthreads();
  if (warp == 0 && n < N) {
    const float a = __ldg(alpha);
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      if (m < M) {
        int v = part[0][m][lane];
#pragma unroll
        for (int w = 1; w < kWarps; ++w) v += part[w][m][lane];
        const float yv = (float)v * (__ldg(scales + m) * a);
        if constexpr (YMODE == 2)
          reinterpret_cast<__nv_bfloat16*>(y)[(size_t)m * N + n] = __float2bfloat16_rn(yv);
        else
          reinterpret_cast<float*>(y)[(size_t)m * N + n] = yv;
      }
    }
  }
}

template <int MT>
cudaError_t launch_mt(const int8_t* A, const float* scales, const uint8_t* packed, const float* alpha, void* y,
                      int y_mode, int M, int N, int K, cudaStream_t stream) {
  static std::atomic<bool> smem_set1[sm100_host::kMaxDevices], smem_set2[sm100_host::kMaxDevices];
  cudaError_t e = y_mode == 2
                      ? sm100_host::ensure_smem(gemv_ternary_kernel<MT, 2>, (int)kGemvMaxCodeBytes, smem_set2)
                      : sm100_host::ensure_smem(gemv_ternary_kernel<MT, 1>, (int)kGemvMaxCodeBytes, smem_set1);
  if (e != cudaSuccess) return e;
  const int grid = (N + kRowsPerCta - 1) / kRowsPerCta;
  const uint4* w = reinterpret_cast<const uint4*>(packed);
  // programmatic dependent launch: the kernel may start while the previous
  // kernel of the stream finishes (it waits for that kernel's results itself)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)M * K;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (y_mode == 2) return cudaLaunchKernelEx(&cfg, gemv_ternary_kernel<MT, 2>, A, scales, w, alpha, y, M, N, K);
  return cudaLaunchKernelEx(&cfg, gemv_ternary_kernel<MT, 1>, A, scales, w, alpha, y, M, N, K);
}

}  // namespace

bool gemv_ternary_supports(int64_t M, int64_t K) {
  return M >= 1 && M <= kGemvMaxRows && M * K <= kGemvMaxCodeBytes && K % 64 == 0;
}

cudaError_t launch_gemv_ternary(const int8_t* A, const float* scales, const uint8_t* packed, const float* alpha,
                                int64_t M, int64_t N, int64_t K, int y_mode, void* y, cudaStream_t stream) {
  if (!gemv_ternary_supports(M, K) || (y_mode != 1 && y_mode != 2)) return cudaErrorInvalidValue;
  const int m = (int)M, n = (int)N, k = (int)K;
  if (m <= 1) return launch_mt<1>(A, scales, packed, alpha, y, y_mode, m, n, k, stream);
  if (m <= 2) return launch_mt<2>(A, scales, packed, alpha, y, y_mode, m, n, k, stream);
  return launch_mt<4>(A, scales, packed, alpha, y, y_mode, m, n, k, stream);
}

}  // namespace hbl
