// verify_tail.cu -- the kernels of the split path after the statistics pass
// (tail_device.cuh): either one CTA per request for everything, or the accept
// scan (one CTA per request) followed by the race (one warp per request and
// segment of the sampled row).
#include <cooperative_groups.h>

#include <atomic>
#include <cstring>

#include "tail_device.cuh"

namespace cg = cooperative_groups;

namespace sv {

namespace {

// Each kernel starts by waiting for the kernel before it (they are launched
// as programmatic dependents, so they can be resident while it drains).
template <int DT>
__global__ void __launch_bounds__(kThreads) scan_kernel(VerifyArgs a) {
  __shared__ TailShared S;
  load_scan_inputs(a, (int)blockIdx.x, S.in);
  wait_for_previous_kernel();
  scan_cta<DT>(a, (int)blockIdx.x, S);
  allow_next_kernel();
}

template <int DT>
__global__ void __launch_bounds__(kThreads, 2) request_kernel(VerifyArgs a) {
  __shared__ TailShared S;
  load_scan_inputs(a, (int)blockIdx.x, S.in);
  wait_for_previous_kernel();
  tail_request<DT>(a, (int)blockIdx.x, S);
}

// One cluster of C CTAs per request (tail_request_cluster).
template <int DT>
__global__ void __launch_bounds__(kThreads, 2) request_cluster_kernel(VerifyArgs a) {
  __shared__ TailShared S;
  __shared__ Best rb;
  cg::cluster_group cluster = cg::this_cluster();
  const int b = (int)(blockIdx.x / cluster.num_blocks());
  if (cluster.block_rank() == 0) load_scan_inputs(a, b, S.in);
  wait_for_previous_kernel();
  tail_request_cluster<DT>(a, b, S, cluster, &rb);
}

template <int DT>
__global__ void __launch_bounds__(kThreads, 2) race_kernel(VerifyArgs a) {
  __shared__ RaceDesc s_rd[kWarps];
  wait_for_previous_kernel();
  const int warp = threadIdx.x >> 5;
  const long long item = (long long)blockIdx.x * kWarps + warp;
  if (item >= (long long)a.B * a.nseg * a.rsplit) return;
  race_item<DT>(a, item, &s_rd[warp]);
}

}  // namespace

// Launch as a programmatic dependent of the kernel before it on the stream.
template <typename K>
cudaError_t launch_dependent(K kernel, unsigned grid, cudaStream_t s, const VerifyArgs& a) {
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, a);
}

cudaError_t launch_scan(const VerifyArgs& a, cudaStream_t s) {
  if (a.B == 0) return cudaSuccess;
  return a.dtype == kF32 ? launch_dependent(scan_kernel<kF32>, a.B, s, a)
                         : launch_dependent(scan_kernel<kBF16>, a.B, s, a);
}

// A cluster of C = 4 or 2 CTAs per request while B C fits two CTAs per
// multiprocessor (sms of them) and the row has a segment for every warp of
// the cluster (nseg of them), else one CTA per request.
int request_cluster_size(int B, int nseg, int sms) {
  int C = 4;
  while (C > 1 && ((long long)B * C > 2LL * sms || C * kWarps > nseg)) C /= 2;
  return C;
}

cudaError_t launch_requests(const VerifyArgs& a, cudaStream_t s, int sms) {
  if (a.B == 0) return cudaSuccess;
  const int C = request_cluster_size(a.B, a.nseg, sms);
  if (C == 1)
    return a.dtype == kF32 ? launch_dependent(request_kernel<kF32>, a.B, s, a)
                           : launch_dependent(request_kernel<kBF16>, a.B, s, a);
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3((unsigned)a.B * (unsigned)C);
  cfg.blockDim = dim3(kThreads);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)C;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return a.dtype == kF32 ? cudaLaunchKernelEx(&cfg, request_cluster_kernel<kF32>, a)
                         : cudaLaunchKernelEx(&cfg, request_cluster_kernel<kBF16>, a);
}

// Race items per segment: a race warp is bound by its own chain of Philox
// rounds and loads, not by the SM's throughput, so while the items fit in one
// wave of resident warps, cutting each segment in two halves the race's time.
int race_split(int B, int nseg, int dtype, int sms) {
  // resident race CTAs per SM, by dtype (host threads may race to fill it in;
  // they all store the same value)
  static std::atomic<int> per_sm[2] = {{-1}, {-1}};
  std::atomic<int>& slot = per_sm[dtype == kF32 ? 0 : 1];
  int n = slot.load(std::memory_order_relaxed);
  if (n < 0) {
    int m = 0;
    const cudaError_t e =
        dtype == kF32 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&m, race_kernel<kF32>, kThreads, 0)
                      : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&m, race_kernel<kBF16>, kThreads, 0);
    n = e == cudaSuccess ? m : 0;
    slot.store(n, std::memory_order_relaxed);
  }
  const long long resident = (long long)n * sms * kWarps;
  return (long long)B * nseg * kMaxRaceSplit <= resident ? kMaxRaceSplit : 1;
}

cudaError_t launch_race(const VerifyArgs& a, cudaStream_t s) {
  const long long items = (long long)a.B * a.nseg * a.rsplit;
  if (items == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((items + kWarps - 1) / kWarps);
  return a.dtype == kF32 ? launch_dependent(race_kernel<kF32>, grid, s, a)
                         : launch_dependent(race_kernel<kBF16>, grid, s, a);
}

}  // namespace sv
