// race_sampler.cu -- the race of the split path: one warp per (request,
// segment of the sampled row); see race_device.cuh.
#include "race_device.cuh"

namespace sv {

namespace {

template <int DT>
__global__ void __launch_bounds__(kThreads, 3) race_kernel(VerifyArgs a) {
  __shared__ RaceDesc s_rd[kWarps];
  const int warp = threadIdx.x >> 5;
  const long long item = (long long)blockIdx.x * kWarps + warp;
  if (item >= (long long)a.B * a.nseg) return;
  const int b = (int)(item / a.nseg);
  const int seg = (int)(item % a.nseg);
  load_race_desc(a.rdesc + b, &s_rd[warp]);
  if (s_rd[warp].kind == kRaceNone) return;
  race_item<DT>(a, b, seg, s_rd[warp]);
}

}  // namespace

cudaError_t launch_race(const VerifyArgs& a, cudaStream_t s) {
  const long long items = (long long)a.B * a.nseg;
  if (items == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((items + kWarps - 1) / kWarps);
  if (a.dtype == kF32)
    race_kernel<kF32><<<grid, kThreads, 0, s>>>(a);
  else
    race_kernel<kBF16><<<grid, kThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace sv
