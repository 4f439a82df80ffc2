// row_stats.cu -- the per-row statistics pass of the split path.
//
// A persistent grid of warps walks the (request, row, segment) items in
// request-major order, warp w taking items w, w + W, w + 2W, ... so that at any
// moment the whole device streams one contiguous stretch of the logits; each
// item is one warp's 8 KiB segment (stats_device.cuh).
#include "stats_device.cuh"

namespace sv {

namespace {

template <int DT>
__global__ void __launch_bounds__(kThreads) row_stats_kernel(VerifyArgs a) {
  const unsigned W = gridDim.x * kWarps;
  const unsigned w0 = blockIdx.x * kWarps + (threadIdx.x >> 5);
  const unsigned total = (unsigned)a.B * (unsigned)a.slots * (unsigned)a.nseg;
  if (w0 >= total) return;
  ItemWalker it;
  it.init(a, w0, W);
  for (unsigned i = w0; i < total; i += W, it.advance(a)) {
    const ReqParams rp = load_req(a, it.b);
    if (!row_needed(a, it.slot, rp)) continue;  // parameter errors are reported by the scan
    stats_item<DT>(a, it.b, it.slot, it.seg, rp);
  }
}

}  // namespace

int row_stats_blocks_per_sm(int dtype) {
  int n = 0;
  cudaError_t e =
      dtype == kF32 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, row_stats_kernel<kF32>, kThreads, 0)
                    : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, row_stats_kernel<kBF16>, kThreads, 0);
  return e == cudaSuccess ? n : 0;
}

cudaError_t launch_row_stats(const VerifyArgs& a, cudaStream_t s, int grid) {
  const long long items = (long long)a.B * a.slots * a.nseg;
  if (items == 0) return cudaSuccess;
  const long long need = (items + kWarps - 1) / kWarps;
  if (grid > need) grid = (int)need;
  if (a.dtype == kF32)
    row_stats_kernel<kF32><<<grid, kThreads, 0, s>>>(a);
  else
    row_stats_kernel<kBF16><<<grid, kThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace sv
