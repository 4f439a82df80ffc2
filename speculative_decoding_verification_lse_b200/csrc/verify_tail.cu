// verify_tail.cu -- the kernels of the split path after the statistics pass
// (tail_device.cuh): either one CTA per request for everything, or the accept
// scan (one CTA per request) followed by the race (one warp per request and
// segment of the sampled row).
#include "tail_device.cuh"

namespace sv {

namespace {

template <int DT>
__global__ void __launch_bounds__(kThreads) scan_kernel(VerifyArgs a) {
  __shared__ TailShared S;
  scan_cta<DT>(a, (int)blockIdx.x, S);
}

template <int DT>
__global__ void __launch_bounds__(kThreads, 2) request_kernel(VerifyArgs a) {
  __shared__ TailShared S;
  tail_request<DT>(a, (int)blockIdx.x, S);
}

template <int DT>
__global__ void __launch_bounds__(kThreads, 2) race_kernel(VerifyArgs a) {
  __shared__ RaceDesc s_rd[kWarps];
  const int warp = threadIdx.x >> 5;
  const long long item = (long long)blockIdx.x * kWarps + warp;
  if (item >= (long long)a.B * a.nseg) return;
  race_item<DT>(a, item, &s_rd[warp]);
}

}  // namespace

cudaError_t launch_scan(const VerifyArgs& a, cudaStream_t s) {
  if (a.B == 0) return cudaSuccess;
  if (a.dtype == kF32)
    scan_kernel<kF32><<<a.B, kThreads, 0, s>>>(a);
  else
    scan_kernel<kBF16><<<a.B, kThreads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_requests(const VerifyArgs& a, cudaStream_t s) {
  if (a.B == 0) return cudaSuccess;
  if (a.dtype == kF32)
    request_kernel<kF32><<<a.B, kThreads, 0, s>>>(a);
  else
    request_kernel<kBF16><<<a.B, kThreads, 0, s>>>(a);
  return cudaGetLastError();
}

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
