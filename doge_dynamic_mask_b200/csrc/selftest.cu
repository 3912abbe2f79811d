// Diagnostic: exercises the library's bounded-wait path on the device.
//
// Every wait in this library's kernels (TMA arrivals, MMA completions, the
// producer / consumer rings) is bounded: after kWaitLimitCycles it records a
// code in the caller's status word and the kernel leaves instead of spinning.
// dma_selftest_wait launches one thread that waits on an mbarrier nothing ever
// arrives on, so that wait runs out; a caller (or a test) then reads
// DMA_ERR_TIMEOUT through dma_check and can check that the context is still
// usable.  Nothing faults, traps or hangs.
#include "common.cuh"
#include "../../include/dma.h"

namespace dma {
namespace {

__global__ void selftest_wait_kernel(uint32_t* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, err, kDevErrTimeoutBase + 99);   // no arrival: gives up
  __syncthreads();
}

}  // namespace
}  // namespace dma

extern "C" dma_status_t dma_selftest_wait(void* workspace, dma_stream_t stream) {
  if (!workspace) return DMA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 15u) != 0) return DMA_ERR_INVALID_ARG;
  int dev = 0;
  cudaDeviceProp prop;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaGetDeviceProperties(&prop, dev) != cudaSuccess)
    return DMA_ERR_CUDA;
  if (prop.major != 10) return DMA_ERR_UNSUPPORTED;
  dma::selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(static_cast<uint32_t*>(workspace));
  return cudaGetLastError() == cudaSuccess ? DMA_OK : DMA_ERR_CUDA;
}
