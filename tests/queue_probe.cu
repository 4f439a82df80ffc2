// Test helper: the fused kernel's bounded waits (work_queue.cuh) on their own.
// wait_kernel claims published race `slot` of a queue whose producer never
// publishes it (a slot that nothing fills), and with idle set also runs the
// idle wait of a warp that never gets work; both must give up on their own
// bounds and set the timeout bit, so that the context stays usable.  With
// fill set, the slot is filled first and the wait returns at once.  Reports
// what the wait returned, the status word and the launch's duration.
#include <cuda_runtime.h>

#include "work_queue.cuh"

using namespace sv;

__global__ void wait_kernel(unsigned* pubq, unsigned* status, unsigned* result, int fill, int idle) {
  if (threadIdx.x == 0 && fill) store_release_gpu(&pubq[0], 42u);
  __syncthreads();
  if (threadIdx.x == 0) result[0] = wait_published(pubq, 0, status);
  if (idle && threadIdx.x < 32) {
    WaitClock clock;
    clock.start();
    unsigned turns = 0;
    while (clock.wait(status)) ++turns;
    if (threadIdx.x == 0) result[1] = turns;
  }
}

extern "C" int queue_probe(int fill, int idle, unsigned* status_out, unsigned* result_out,
                           float* ms_out) {
  unsigned* pubq = nullptr;
  unsigned* status = nullptr;
  unsigned* result = nullptr;
  if (cudaMalloc(&pubq, sizeof(unsigned)) != cudaSuccess) return 1;
  if (cudaMalloc(&status, sizeof(unsigned)) != cudaSuccess) return 1;
  if (cudaMalloc(&result, 2 * sizeof(unsigned)) != cudaSuccess) return 1;
  cudaMemset(pubq, 0, sizeof(unsigned));
  cudaMemset(status, 0, sizeof(unsigned));
  cudaMemset(result, 0xFF, 2 * sizeof(unsigned));
  cudaEvent_t e0, e1;
  cudaEventCreate(&e0);
  cudaEventCreate(&e1);
  cudaEventRecord(e0, 0);
  wait_kernel<<<1, 64>>>(pubq, status, result, fill, idle);
  const cudaError_t le = cudaGetLastError();
  cudaEventRecord(e1, 0);
  const cudaError_t se = cudaDeviceSynchronize();
  int rc = (le == cudaSuccess && se == cudaSuccess) ? 0 : 1;
  if (!rc) {
    cudaEventElapsedTime(ms_out, e0, e1);
    cudaMemcpy(status_out, status, sizeof(unsigned), cudaMemcpyDeviceToHost);
    cudaMemcpy(result_out, result, 2 * sizeof(unsigned), cudaMemcpyDeviceToHost);
  }
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  cudaFree(pubq);
  cudaFree(status);
  cudaFree(result);
  return rc;
}
