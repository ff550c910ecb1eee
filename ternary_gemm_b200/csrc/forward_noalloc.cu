// hbl_forward_noalloc: the whole H-BitLinear forward without a caller-supplied
// workspace, for callers that cannot allocate device memory at the point of
// the call -- code running under a fixed memory budget that was reserved up
// front, allocator-free inference runtimes and plugins that are handed only
// the tensors of one layer, or hosts where a cudaMalloc could block on the
// device or fail late.  hbl_forward needs a workspace for the int8 activation
// codes, the per-row scales and the int8 weight codes the tensor cores read;
// this entry point uses a fixed area of device memory that belongs to the
// library instead.
//
// The area is a file-scope __device__ array of kNoAllocScratchBytes (32 MiB).
// Every GPU that loads the library holds it until the process exits.  Host
// code cannot use the array's name as a device address, so each call made
// outside stream capture looks the address up with cudaGetSymbolAddress (a
// query, not an allocation; with that device current) and remembers it per
// device.  A call made while its stream is being captured uses the address
// remembered from the last call outside capture instead, because the lookup
// may load the module, which capture does not allow: the first call on a
// device should therefore happen before any stream capture.  Looking the
// address up again on every uncaptured call keeps it valid after a
// cudaDeviceReset, which may place the array elsewhere.
//
// All calls share the one area and it keeps whatever the last call left
// there.  Nothing in it has to start at zero: every call overwrites the parts
// it reads (codes, scales, widened weights) before reading them.  Calls whose
// kernels overlap on the GPU (different streams, or different host threads on
// the same device without ordering) race on the area; callers must serialise
// them.
#include <cstdint>
#include <mutex>

#include "common.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

__device__ __align__(256) unsigned char g_forward_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_ptr[64] = {nullptr};

// Device address of g_forward_scratch on the current device: looked up on
// every call outside stream capture, remembered for calls during capture.
cudaError_t scratch_address(cudaStream_t stream, void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(stream, &cs);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (cs == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_forward_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  } else if (!g_scratch_ptr[dev]) {
    return cudaErrorStreamCaptureUnsupported;  // no uncaptured call on this device yet
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" hbl_status hbl_forward_noalloc(const void* x, hbl_dtype xt, int64_t M, int64_t K, const uint8_t* packed,
                                          const float* alpha_dev, int64_t N, int bits, void* y, hbl_dtype yt,
                                          cudaStream_t stream) {
  // every argument check of hbl_forward, with no workspace: it answers
  // HBL_ERR_WORKSPACE (and launches nothing) only when all else is valid
  hbl_status s = hbl_forward(x, xt, M, K, packed, alpha_dev, N, bits, y, yt, nullptr, 0, stream);
  if (s != HBL_ERR_WORKSPACE) return s;
  if (hbl_forward_workspace_bytes(M, K, N, bits) > kNoAllocScratchBytes) return HBL_ERR_WORKSPACE;
  void* scratch = nullptr;
  cudaError_t e = scratch_address(stream, &scratch);
  if (e != cudaSuccess) return hbl::note_cuda_error(e);
  return hbl_forward(x, xt, M, K, packed, alpha_dev, N, bits, y, yt, scratch, kNoAllocScratchBytes, stream);
}
