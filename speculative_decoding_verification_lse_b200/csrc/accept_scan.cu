// accept_scan.cu -- the accept scan of the split path: one warp per request;
// see scan_device.cuh.
#include "scan_device.cuh"

namespace sv {

namespace {

__global__ void __launch_bounds__(32 * kScanWarps) accept_scan_kernel(VerifyArgs a) {
  __shared__ RowRes s_rows[kScanWarps][2 * kMaxDraft + 1];
  const int warp = threadIdx.x >> 5;
  const int b = blockIdx.x * kScanWarps + warp;
  if (b >= a.B) return;
  scan_request(a, b, s_rows[warp]);
  if ((threadIdx.x & 31) == 0) a.rcount[b] = 0u;  // the race kernel counts its chunks from 0
}

}  // namespace

cudaError_t launch_accept_scan(const VerifyArgs& a, cudaStream_t s) {
  if (a.B == 0) return cudaSuccess;
  const int grid = (a.B + kScanWarps - 1) / kScanWarps;
  accept_scan_kernel<<<grid, 32 * kScanWarps, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace sv
