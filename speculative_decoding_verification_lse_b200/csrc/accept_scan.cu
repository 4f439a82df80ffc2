// accept_scan.cu -- the accept scan of the split path: one CTA per request;
// its warps merge the request's rows in parallel, then warp 0 runs the scan
// (scan_device.cuh).
#include "scan_device.cuh"

namespace sv {

namespace {

constexpr int kScanMaxWarps = 16;

__global__ void __launch_bounds__(32 * kScanMaxWarps) accept_scan_kernel(VerifyArgs a) {
  __shared__ RowRes s_rows[2 * kMaxDraft + 1];
  const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int b = blockIdx.x;
  const ReqParams rp = load_req(a, b);
  for (int slot = warp; slot < a.slots; slot += nw)
    if (slot_needed(a, slot, rp)) merge_row_global(a, b, slot, rp);
  __syncthreads();
  if (warp == 0) {
    scan_request(a, b, s_rows);
    if ((threadIdx.x & 31) == 0) a.rcount[b] = 0u;  // the race kernel counts its segments from 0
  }
}

}  // namespace

cudaError_t launch_accept_scan(const VerifyArgs& a, cudaStream_t s) {
  if (a.B == 0) return cudaSuccess;
  const int warps = a.slots < kScanMaxWarps ? a.slots : kScanMaxWarps;
  accept_scan_kernel<<<a.B, 32 * warps, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace sv
