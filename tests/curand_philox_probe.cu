// Test helper: words of cuRAND's Philox4_32_10 generator, to pin the oracle's
// Philox4x32-10 against an independent implementation (NVIDIA's library).
// curand_init(seed, subsequence, offset) places the generator at counter
// block (offset / 4) of subsequence `subsequence`; curand4 returns one block.
#include <cuda_runtime.h>
#include <curand_kernel.h>
#include <stdint.h>

__global__ void probe_kernel(const unsigned long long* seeds, const unsigned long long* subseq,
                             const unsigned long long* offsets, uint4* out, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  curandStatePhilox4_32_10_t st;
  curand_init(seeds[i], subseq[i], offsets[i], &st);
  out[i] = curand4(&st);
}

extern "C" int curand_philox_words(const unsigned long long* seeds, const unsigned long long* subseq,
                                   const unsigned long long* offsets, unsigned int* words, int n) {
  unsigned long long *d_s = nullptr, *d_q = nullptr, *d_o = nullptr;
  uint4* d_w = nullptr;
  const size_t b8 = sizeof(unsigned long long) * (size_t)n;
  if (cudaMalloc(&d_s, b8) || cudaMalloc(&d_q, b8) || cudaMalloc(&d_o, b8) ||
      cudaMalloc(&d_w, sizeof(uint4) * (size_t)n))
    return 1;
  cudaMemcpy(d_s, seeds, b8, cudaMemcpyHostToDevice);
  cudaMemcpy(d_q, subseq, b8, cudaMemcpyHostToDevice);
  cudaMemcpy(d_o, offsets, b8, cudaMemcpyHostToDevice);
  probe_kernel<<<(n + 127) / 128, 128>>>(d_s, d_q, d_o, d_w, n);
  cudaError_t e = cudaMemcpy(words, d_w, sizeof(uint4) * (size_t)n, cudaMemcpyDeviceToHost);
  cudaFree(d_s);
  cudaFree(d_q);
  cudaFree(d_o);
  cudaFree(d_w);
  return e == cudaSuccess ? 0 : 2;
}
