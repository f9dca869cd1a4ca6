// Test kernel for the device-side failure path: an mbarrier wait on a phase
// that nothing completes must give up after the library's bounded limit,
// record LA_ERR_TIMEOUT in the status word and return, leaving the context
// usable.  It uses the same wait as every kernel of the library.
#include <cuda_runtime.h>
#include <stdint.h>

#include "sm100.cuh"

namespace {

__global__ void bounded_wait_kernel(int* status, unsigned long long* out) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    la::mbar_init(&bar, 1);
    la::fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = la::globaltimer_ns();
    const bool ok = la::mbar_wait(&bar, 0, status);   // no thread ever arrives
    out[0] = la::globaltimer_ns() - t0;
    out[1] = ok ? 1ull : 0ull;
  }
}

}  // namespace

// Runs the kernel once; returns a cudaError_t value, fills status and
// {elapsed ns, wait succeeded}.
extern "C" int run_bounded_wait(int* status_host, unsigned long long* out_host) {
  int* status = nullptr;
  unsigned long long* out = nullptr;
  cudaError_t e = cudaMalloc(&status, sizeof(int));
  if (e == cudaSuccess) e = cudaMalloc(&out, 2 * sizeof(unsigned long long));
  if (e == cudaSuccess) e = cudaMemset(status, 0, sizeof(int));
  if (e == cudaSuccess) {
    bounded_wait_kernel<<<1, 32>>>(status, out);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(status_host, status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(out_host, out, 2 * sizeof(unsigned long long), cudaMemcpyDeviceToHost);
  cudaFree(status);
  cudaFree(out);
  return static_cast<int>(e);
}
