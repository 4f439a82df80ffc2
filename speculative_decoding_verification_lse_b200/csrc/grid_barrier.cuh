// grid_barrier.cuh -- a grid-wide barrier for cooperative launches, with a
// bounded wait.
//
// The counter lives in global memory and reads zero before the launch; every
// CTA adds one on arrival and polls until the count reaches the grid size.
// Since a cooperative launch has every CTA resident at once, the count is
// reached unless a CTA skips the barrier; the poll is bounded all the same, and
// a CTA that gives up sets the timeout bit of the status word and reports it.
#pragma once
#include "sv_common.cuh"

namespace sv {

constexpr int kBarrierPolls = 1 << 22;  // each a 64 ns sleep and an L2 load: about 1.5 s

__device__ __forceinline__ unsigned load_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Every CTA of the grid at the barrier counting on *counter; false (and the
// timeout bit in *status) if the wait gave up.  Called by every thread of the CTA.
__device__ __forceinline__ bool grid_barrier(unsigned* counter, unsigned* status) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();  // the CTA's writes before its arrival
    atomicAdd(counter, 1u);
    unsigned n = load_acquire_gpu(counter);
    for (int i = 0; n < gridDim.x && i < kBarrierPolls; ++i) {
      __nanosleep(64);
      n = load_acquire_gpu(counter);
    }
    s_ok = n >= gridDim.x;
    if (!s_ok) atomicOr(status, kStatusTimeout);
    __threadfence();
  }
  __syncthreads();
  return s_ok != 0;
}

}  // namespace sv
