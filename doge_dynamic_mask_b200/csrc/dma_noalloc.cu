// Allocation-free variant of the decode step.
//
// Some callers cannot hand this library a workspace: code embedded in a host
// framework that owns every byte of device memory through its own pool (and
// forbids raw cudaMalloc, which synchronises the device and fragments that
// pool), or plain C callers that have no device allocator at hand.  For them,
// dma_decode_step_noalloc runs the ordinary decode step with its scratch
// (per-key scores, kept-key lists, split-K partials) in a fixed array that
// lives in this library's own device memory.
//
// The array is a file-scope __device__ object of kNoAllocScratchBytes; every
// GPU that loads the library holds it until the process exits.  Host code only
// ever sees a host-side stand-in for its name, so its device address is looked
// up once per device with cudaGetSymbolAddress (with that device current) and
// cached.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/dma.h"
#include "dma_internal.h"

namespace dma {
namespace {

// 64 MiB: enough for a decode step with B * Hkv * Lk up to about 15.7 million cached keys.
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

// Device address of g_decode_scratch on the current device (set up once per device).
cudaError_t scratch_address(void** out) {
  static std::mutex mu;
  static void* cached[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!cached[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    cached[dev] = p;
  }
  *out = cached[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace dma

extern "C" dma_status_t dma_decode_step_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                                const float* W_dt, const float* A, const int32_t* lengths, int B,
                                                int Lk, int Hq, int Hkv, int d, int keep_window_size, float scale,
                                                const float* dt_in, void* out, dma_stream_t stream) {
  const size_t need = dma_workspace_size(B, 1, Lk, Hq, Hkv, d, keep_window_size);
  if (need > dma::kNoAllocScratchBytes) return DMA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (dma::scratch_address(&scratch) != cudaSuccess) return DMA_ERR_CUDA;
  if (need > 0) {
    // the status word must start at zero; every other byte used is overwritten by the kernels
    if (cudaMemsetAsync(scratch, 0, 4, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return DMA_ERR_CUDA;
  }
  // need == 0 means the arguments are rejected: the ordinary entry point returns
  // the reason before it launches anything
  return dma_decode_step(q, k_cache, v_cache, W_dt, A, lengths, B, Lk, Hq, Hkv, d, keep_window_size, scale, dt_in,
                         out, scratch, dma::kNoAllocScratchBytes, stream);
}
