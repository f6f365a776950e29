// Device error words of the kernels, read back and cleared by the host, and
// a self-test of the bounded wait: a kernel whose barrier nothing completes
// gives up after the wait limit and records a timeout, without hanging or
// faulting the GPU.
#include "kernels.h"
#include "ptx.cuh"

namespace sas {

__device__ uint32_t g_selftest_err = 0;

__global__ void k_wait_selftest() {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &g_selftest_err);  // no arrival: times out
}

cudaError_t launch_wait_selftest(cudaStream_t st) {
  k_wait_selftest<<<1, 32, 0, st>>>();
  return cudaGetLastError();
}

uint32_t* selftest_error_word() {
  void* p = nullptr;
  cudaGetSymbolAddress(&p, g_selftest_err);
  return static_cast<uint32_t*>(p);
}

}  // namespace sas
