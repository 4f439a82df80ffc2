// row_stats.cu -- the first kernel of the split path: the per-row statistics
// pass (stats_device.cuh) on a persistent grid of warps, each item one warp's
// 8 KiB segment of a row.  Three CTAs of 8 warps per multiprocessor (at most 85
// registers a thread): the 24 warps keep about 192 KiB of loads in flight per
// multiprocessor, which the pass needs to stream at the HBM rate.
#include "stats_device.cuh"

namespace sv {

namespace {

constexpr unsigned kBatch = 1;  // consecutive items per ticket

// TICKETS: warps take batches of kBatch consecutive items from ticket counters
// (zero at launch; each warp fetches its next ticket while it works on the
// current batch), so that the warps and SMs that run ahead take more and the
// pass ends together.  Eight counters on separate 128-byte lines share the
// batches (counter c hands out c, c + 8, ...): one counter for every warp
// would serialise its atomics.  Without: the static request-major schedule,
// which costs nothing to set up (for batches with few items per warp).
template <int DT, bool WITH_TOP, bool TICKETS>
__global__ void __launch_bounds__(kThreads, 3) row_stats_kernel(VerifyArgs a) {
  if (!TICKETS) {
    stats_pass<DT, WITH_TOP>(a, blockIdx.x * kWarps + (threadIdx.x >> 5), gridDim.x * kWarps);
  } else {
    // eight counters (128 bytes apart): counter c hands out batches c, c + 8, ...
    const unsigned lane = threadIdx.x & 31;
    const unsigned per_req = (unsigned)a.slots * (unsigned)a.nseg;
    const unsigned total = (unsigned)a.B * per_req;
    const unsigned batches = (total + kBatch - 1) / kBatch;
    const unsigned c = (blockIdx.x * kWarps + (threadIdx.x >> 5)) & 7u;
    unsigned* ctr = a.ticket + 32 * c;
    unsigned t = 0;
    if (lane == 0) t = atomicAdd(ctr, 1u) * 8u + c;
    t = __shfl_sync(0xFFFFFFFFu, t, 0);
    while (t < batches) {
      unsigned tn = 0;
      if (lane == 0) tn = atomicAdd(ctr, 1u) * 8u + c;
      const unsigned end = min(total, (t + 1) * kBatch);
      for (unsigned i = t * kBatch; i < end; ++i) {
        const int b = (int)(i / per_req);
        const unsigned r = i % per_req;
        const int slot = (int)(r / (unsigned)a.nseg), seg = (int)(r % (unsigned)a.nseg);
        const ReqParams rp = load_req(a, b);
        if (row_needed(a, b, slot, rp)) stats_item<DT, WITH_TOP>(a, b, slot, seg, rp);
      }
      t = __shfl_sync(0xFFFFFFFFu, tn, 0);
    }
  }
  allow_next_kernel();
}

}  // namespace

int row_stats_blocks_per_sm(int dtype) {
  int n = 0;
  cudaError_t e = dtype == kF32 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                                      &n, row_stats_kernel<kF32, true, true>, kThreads, 0)
                                : cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                                      &n, row_stats_kernel<kBF16, true, true>, kThreads, 0);
  return e == cudaSuccess ? n : 0;
}

// Tickets once there are at least 8 items for every resident warp.
bool row_stats_tickets(const VerifyArgs& a, int grid) {
  const long long items = (long long)a.B * a.slots * a.nseg;
  return items >= 8LL * grid * kWarps;
}

template <int DT>
static cudaError_t launch_dt(const VerifyArgs& a, cudaStream_t s, int grid, bool top, bool tickets) {
  if (top) {
    if (tickets)
      row_stats_kernel<DT, true, true><<<grid, kThreads, 0, s>>>(a);
    else
      row_stats_kernel<DT, true, false><<<grid, kThreads, 0, s>>>(a);
  } else {
    if (tickets)
      row_stats_kernel<DT, false, true><<<grid, kThreads, 0, s>>>(a);
    else
      row_stats_kernel<DT, false, false><<<grid, kThreads, 0, s>>>(a);
  }
  return cudaGetLastError();
}

// Saguaro requests (the batch's mode, or any per-request mode) need the top
// lists; `tickets` (row_stats_tickets) needs a.ticket zeroed on the stream first.
cudaError_t launch_row_stats(const VerifyArgs& a, cudaStream_t s, int grid, bool tickets) {
  const long long items = (long long)a.B * a.slots * a.nseg;
  if (items == 0) return cudaSuccess;
  const long long need = (items + kWarps - 1) / kWarps;
  if (grid > need) grid = (int)need;
  const bool top = a.mode == kSaguaro || a.mode_per_req != nullptr;
  return a.dtype == kF32 ? launch_dt<kF32>(a, s, grid, top, tickets)
                         : launch_dt<kBF16>(a, s, grid, top, tickets);
}

}  // namespace sv
