// verify_tail.cu -- the second kernel of the split path: one CTA per request
// merges the request's rows, runs its accept scan and its race
// (tail_device.cuh).
#include "tail_device.cuh"

namespace sv {

namespace {

template <int DT>
__global__ void __launch_bounds__(kTailThreads, 2) verify_tail_kernel(VerifyArgs a) {
  __shared__ TailShared S;
  tail_request<DT>(a, (int)blockIdx.x, S);
}

}  // namespace

cudaError_t launch_tail(const VerifyArgs& a, cudaStream_t s) {
  if (a.B == 0) return cudaSuccess;
  if (a.dtype == kF32)
    verify_tail_kernel<kF32><<<a.B, kTailThreads, 0, s>>>(a);
  else
    verify_tail_kernel<kBF16><<<a.B, kTailThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace sv
