// fused_verify.cu -- the whole verification step in one launch.
//
// A cooperative launch (every CTA resident at once) runs the statistics pass
// over all (request, row, segment) items (stats_device.cuh), meets at a grid
// barrier, and then does what the split path's later kernels do
// (tail_device.cuh), in the same layout: either each CTA takes whole requests
// (blockIdx.x, + gridDim.x, ...), or the CTAs take the accept scans, meet at a
// second barrier, and the warps take the (request, segment) race items (whole
// segments: a.rsplit is 1 here).  The partial statistics are read back from L2.
//
// The barriers are counters in the workspace, zero at launch.  Their waits are
// bounded: a CTA that gives up sets SV_STATUS_TIMEOUT, writes -1 for its
// requests and ends.  Since the launch is cooperative, no CTA ever waits for
// one that is not running.
#include "grid_barrier.cuh"
#include "tail_device.cuh"

namespace sv {

namespace {

// The CTA gave up at a barrier: -1 for its requests.
__device__ void fail_requests(const VerifyArgs& a) {
  for (int b = blockIdx.x; b < a.B; b += gridDim.x) {
    for (int j = threadIdx.x; j <= a.D_max; j += blockDim.x)
      a.out_tokens[(size_t)b * (a.D_max + 1) + j] = -1;
    if (threadIdx.x == 0) {
      a.out_al[b] = -1;
      if (a.out_flags) a.out_flags[b] = kStatusTimeout;
    }
  }
}

template <int DT>
__global__ void __launch_bounds__(kThreads, 2) fused_kernel(VerifyArgs a) {
  __shared__ TailShared S;
  __shared__ RaceDesc s_rd[kWarps];
  const int warp = threadIdx.x >> 5;
  stats_pass<DT, true>(a, blockIdx.x * kWarps + warp, gridDim.x * kWarps);
  if (!grid_barrier(&a.barrier[0], a.status)) return fail_requests(a);
  if (a.per_request) {
    for (int b = blockIdx.x; b < a.B; b += gridDim.x) tail_request<DT>(a, b, S);
    return;
  }
  for (int b = blockIdx.x; b < a.B; b += gridDim.x) scan_cta<DT>(a, b, S);
  if (!grid_barrier(&a.barrier[1], a.status)) return fail_requests(a);
  const long long items = (long long)a.B * a.nseg * a.rsplit;
  for (long long it = (long long)blockIdx.x * kWarps + warp; it < items; it += (long long)gridDim.x * kWarps)
    race_item<DT>(a, it, &s_rd[warp]);
}

}  // namespace

// grid: the most CTAs that can be resident at once (fused_blocks_per_sm x SMs).
cudaError_t launch_fused(const VerifyArgs& a, cudaStream_t s, int grid) {
  if (a.B == 0) return cudaSuccess;
  // no more CTAs than there is work for: one per request, or per 8 warps' items
  const long long items = (long long)a.B * a.slots * a.nseg;
  long long want = (items + kWarps - 1) / kWarps;
  if (want < a.B) want = a.B;
  if (grid > want) grid = (int)want;
  VerifyArgs arg = a;
  void* params[] = {&arg};
  const void* fn =
      a.dtype == kF32 ? (const void*)fused_kernel<kF32> : (const void*)fused_kernel<kBF16>;
  return cudaLaunchCooperativeKernel(fn, dim3(grid), dim3(kThreads), params, 0, s);
}

int fused_blocks_per_sm(int dtype) {
  int n = 0;
  const cudaError_t e =
      dtype == kF32
          ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fused_kernel<kF32>, kThreads, 0)
          : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fused_kernel<kBF16>, kThreads, 0);
  return e == cudaSuccess ? n : 0;
}

}  // namespace sv
