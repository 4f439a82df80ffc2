// row_stats.cu -- the first kernel of the split path: the per-row statistics
// pass (stats_device.cuh) on a persistent grid of warps, each item one warp's
// 8 KiB segment of a row.  Three CTAs of 8 warps per multiprocessor (at most 85
// registers a thread): the 24 warps keep about 192 KiB of loads in flight per
// multiprocessor, which the pass needs to stream at the HBM rate.
#include "stats_device.cuh"

namespace sv {

namespace {

template <int DT, bool WITH_TOP>
__global__ void __launch_bounds__(kThreads, 3) row_stats_kernel(VerifyArgs a) {
  stats_pass<DT, WITH_TOP>(a, blockIdx.x * kWarps + (threadIdx.x >> 5), gridDim.x * kWarps);
  allow_next_kernel();
}

}  // namespace

int row_stats_blocks_per_sm(int dtype) {
  int n = 0;
  cudaError_t e = dtype == kF32 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                                      &n, row_stats_kernel<kF32, true>, kThreads, 0)
                                : cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                                      &n, row_stats_kernel<kBF16, true>, kThreads, 0);
  return e == cudaSuccess ? n : 0;
}

// Saguaro requests (the batch's mode, or any per-request mode) need the top lists.
cudaError_t launch_row_stats(const VerifyArgs& a, cudaStream_t s, int grid) {
  const long long items = (long long)a.B * a.slots * a.nseg;
  if (items == 0) return cudaSuccess;
  const long long need = (items + kWarps - 1) / kWarps;
  if (grid > need) grid = (int)need;
  const bool top = a.mode == kSaguaro || a.mode_per_req != nullptr;
  if (a.dtype == kF32) {
    if (top)
      row_stats_kernel<kF32, true><<<grid, kThreads, 0, s>>>(a);
    else
      row_stats_kernel<kF32, false><<<grid, kThreads, 0, s>>>(a);
  } else {
    if (top)
      row_stats_kernel<kBF16, true><<<grid, kThreads, 0, s>>>(a);
    else
      row_stats_kernel<kBF16, false><<<grid, kThreads, 0, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace sv
