// Test helper: the fused kernel's grid barrier (grid_barrier.cuh) in a
// cooperative launch of two CTAs.  With skip_second set, the second CTA leaves
// without arriving -- a count that nothing completes -- so the first CTA's
// bounded wait runs out and sets the timeout bit; otherwise both arrive and
// pass.  Reports each CTA's outcome (1 passed, 0 gave up, -1 never arrived),
// the status word and the launch's duration.
#include <cuda_runtime.h>

#include "grid_barrier.cuh"

using namespace sv;

__global__ void barrier_kernel(unsigned* counter, unsigned* status, int* result, int skip_second) {
  if (skip_second && blockIdx.x == 1) return;
  const bool ok = grid_barrier(counter, status);
  if (threadIdx.x == 0) result[blockIdx.x] = ok ? 1 : 0;
}

extern "C" int barrier_probe(int skip_second, unsigned* status_out, int* result_out, float* ms_out) {
  unsigned* counter = nullptr;
  unsigned* status = nullptr;
  int* result = nullptr;
  if (cudaMalloc(&counter, sizeof(unsigned)) != cudaSuccess) return 1;
  if (cudaMalloc(&status, sizeof(unsigned)) != cudaSuccess) return 1;
  if (cudaMalloc(&result, 2 * sizeof(int)) != cudaSuccess) return 1;
  cudaMemset(counter, 0, sizeof(unsigned));
  cudaMemset(status, 0, sizeof(unsigned));
  cudaMemset(result, 0xFF, 2 * sizeof(int));  // -1: the CTA never reached the barrier
  cudaEvent_t e0, e1;
  cudaEventCreate(&e0);
  cudaEventCreate(&e1);
  void* args[] = {&counter, &status, &result, &skip_second};
  cudaEventRecord(e0, 0);
  const cudaError_t le =
      cudaLaunchCooperativeKernel((const void*)barrier_kernel, dim3(2), dim3(128), args, 0, 0);
  cudaEventRecord(e1, 0);
  const cudaError_t se = cudaDeviceSynchronize();
  int rc = (le == cudaSuccess && se == cudaSuccess) ? 0 : 1;
  if (!rc) {
    cudaEventElapsedTime(ms_out, e0, e1);
    cudaMemcpy(status_out, status, sizeof(unsigned), cudaMemcpyDeviceToHost);
    cudaMemcpy(result_out, result, 2 * sizeof(int), cudaMemcpyDeviceToHost);
  }
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  cudaFree(counter);
  cudaFree(status);
  cudaFree(result);
  return rc;
}
