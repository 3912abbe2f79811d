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
// up with cudaGetSymbolAddress (with the device current) and cached per
// device.  The module, and with it the array, is loaded again when a device's
// primary context is destroyed and made anew (cudaDeviceReset): the cache is
// keyed by the context's unique id, so a new context gets a fresh lookup.
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/dma.h"
#include "dma_internal.h"

namespace dma {
namespace {

// 64 MiB: enough for a decode step with B * Hkv * Lk up to about 15.7 million cached keys.
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (0 when there is none or
// the driver cannot tell).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_decode_scratch in the current device's context.
cudaError_t scratch_address(void** out) {
  struct Entry {
    unsigned long long ctx_id;
    void* ptr;
  };
  static std::mutex mu;
  static Entry cached[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long id = current_context_id();
  if (id == 0 || cached[dev].ctx_id != id || !cached[dev].ptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);   // makes the context current if it was not
    if (e != cudaSuccess) return e;
    cached[dev] = Entry{current_context_id(), p};
  }
  *out = cached[dev].ptr;
  return cudaSuccess;
}

}  // namespace
}  // namespace dma

extern "C" dma_status_t dma_decode_step_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                                const float* W_dt, const float* A, const int32_t* lengths, int B,
                                                int Lk, int Hq, int Hkv, int d, int keep_window_size, float scale,
                                                const float* dt_in, void* out, dma_stream_t stream) {
  // every check dma_decode_step makes comes first, so a rejected call
  // enqueues nothing (the array's address stands in for the workspace pointer)
  dma_status_t st = dma::check_decode_args(q, k_cache, v_cache, W_dt, A, lengths, B, Lk, Hq, Hkv, d,
                                           keep_window_size, scale, dt_in, out, &dma::g_decode_scratch);
  if (st != DMA_OK) return st;
  const size_t need = dma_workspace_size(B, 1, Lk, Hq, Hkv, d, keep_window_size);
  if (need == 0) return DMA_ERR_UNSUPPORTED;
  if (need > dma::kNoAllocScratchBytes) return DMA_ERR_WORKSPACE;
  void* scratch = nullptr;
  cudaError_t e = dma::scratch_address(&scratch);
  if (e != cudaSuccess) return dma::cuda_fail(e);
  // the status word must start at zero; every other byte used is overwritten by the kernels
  if ((e = cudaMemsetAsync(scratch, 0, 4, reinterpret_cast<cudaStream_t>(stream))) != cudaSuccess)
    return dma::cuda_fail(e);
  return dma_decode_step(q, k_cache, v_cache, W_dt, A, lengths, B, Lk, Hq, Hkv, d, keep_window_size, scale, dt_in,
                         out, scratch, dma::kNoAllocScratchBytes, stream);
}
