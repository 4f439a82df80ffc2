// row_stats.cu -- the per-row statistics pass of the split path.
//
// A persistent grid of warps walks the (request, row, segment) items in
// request-major order, warp w taking items w, w + W, w + 2W, ... so that at any
// moment the whole device streams one contiguous stretch of the logits; each
// item is one warp's 8 KiB segment (stats_device.cuh).
//
// Every warp owns a two-stage ring of 8 KiB shared-memory buffers.  One lane
// starts the bulk copy (cp.async.bulk, completing on an mbarrier) of the warp's
// next segment before the warp reduces the current one, so HBM keeps streaming
// through the warp's compute phase.  Segments a bulk copy cannot take (a row
// not 16-byte aligned, a last segment whose length is not a multiple of 16
// bytes) are read through registers instead.  Waits on the barriers are
// bounded: an expired wait sets SV_STATUS_TIMEOUT, waits (bounded) for the
// warp's copies still in flight and ends the warp.
#include "stats_device.cuh"

namespace sv {

namespace {

constexpr int kStatsWarps = 4;   // warps per CTA (each with its own ring)
constexpr int kMaxPolls = 1 << 22;

struct WarpRing {
  uint4 buf[2][kSegVecs];   // two 8 KiB stages
  uint64_t bar[2];
};

// Bounded wait for one stage (all lanes get the same answer).
__device__ __forceinline__ bool wait_stage(WarpRing* ring, int stage, uint32_t parity) {
  bool ok = false;
  for (int p = 0; p < kMaxPolls && !ok; ++p) ok = mbar_try_wait(&ring->bar[stage], parity);
  return __all_sync(0xFFFFFFFFu, ok);
}

template <int DT>
__device__ __forceinline__ void issue_copy(const VerifyArgs& a, WarpRing* ring, int stage,
                                           const ItemWalker& it, uint32_t bytes) {
  if ((threadIdx.x & 31) == 0) {
    const char* src = row_base(a, it.b, it.slot) + (size_t)it.seg * kSegVecs * 16;
    fence_proxy_async_smem();  // this warp's reads of the stage come before the copy
    mbar_arrive_expect_tx(&ring->bar[stage], bytes);
    bulk_copy_g2s(ring->buf[stage], src, bytes, &ring->bar[stage]);
  }
}

template <int DT>
__global__ void __launch_bounds__(32 * kStatsWarps) row_stats_kernel(VerifyArgs a) {
  extern __shared__ __align__(128) unsigned char s_dyn[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  WarpRing* ring = reinterpret_cast<WarpRing*>(s_dyn) + warp;
  if (lane == 0) {
    mbar_init(&ring->bar[0], 1);
    mbar_init(&ring->bar[1], 1);
    fence_mbar_init();
  }
  __syncwarp();

  const unsigned W = gridDim.x * kStatsWarps;
  const unsigned total = (unsigned)a.B * (unsigned)a.slots * (unsigned)a.nseg;
  unsigned i = blockIdx.x * kStatsWarps + warp;
  if (i >= total) return;
  ItemWalker it;
  it.init(a, i, W);

  // the next item this warp must compute (parameter errors are reported by the scan)
  auto find_needed = [&](ItemWalker& w, unsigned& idx, ReqParams& rp) -> bool {
    for (; idx < total; idx += W, w.advance(a)) {
      rp = load_req(a, w.b);
      if (row_needed(a, w.slot, rp)) return true;
    }
    return false;
  };

  ReqParams rp;
  bool have = find_needed(it, i, rp);
  unsigned issued = 0, consumed = 0;
  uint32_t bytes = 0;
  if (have) {
    bytes = bulk_bytes<DT>(a, row_base(a, it.b, it.slot), it.seg);
    if (bytes) issue_copy<DT>(a, ring, (int)(issued++ & 1u), it, bytes);
  }
  while (have) {
    // start the copy of the next item before reducing this one
    ItemWalker nx = it;
    unsigned ni = i + W;
    nx.advance(a);
    ReqParams rp_nx;
    const bool have_nx = find_needed(nx, ni, rp_nx);
    uint32_t bytes_nx = 0;
    if (have_nx) {
      bytes_nx = bulk_bytes<DT>(a, row_base(a, nx.b, nx.slot), nx.seg);
      if (bytes_nx) issue_copy<DT>(a, ring, (int)(issued++ & 1u), nx, bytes_nx);
    }
    if (bytes) {
      const int stage = (int)(consumed & 1u);
      if (!wait_stage(ring, stage, (consumed >> 1) & 1u)) {
        // a copy did not complete: report, let the copies in flight land, stop
        if (lane == 0) atomicOr(a.status, kStatusTimeout);
        for (unsigned c = consumed + 1; c < issued; ++c) wait_stage(ring, (int)(c & 1u), (c >> 1) & 1u);
        return;
      }
      stats_item_smem<DT>(a, ring->buf[stage], (int)(bytes / 16), it.b, it.slot, it.seg, rp);
      ++consumed;
    } else {
      stats_item<DT>(a, it.b, it.slot, it.seg, rp);
    }
    __syncwarp();
    it = nx;
    i = ni;
    rp = rp_nx;
    have = have_nx;
    bytes = bytes_nx;
  }
}

constexpr size_t kSmem = kStatsWarps * sizeof(WarpRing);

}  // namespace

int row_stats_threads() { return 32 * kStatsWarps; }

int row_stats_blocks_per_sm(int dtype) {
  int n = 0;
  cudaError_t e;
  if (dtype == kF32) {
    cudaFuncSetAttribute(row_stats_kernel<kF32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, row_stats_kernel<kF32>, 32 * kStatsWarps, kSmem);
  } else {
    cudaFuncSetAttribute(row_stats_kernel<kBF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, row_stats_kernel<kBF16>, 32 * kStatsWarps, kSmem);
  }
  return e == cudaSuccess ? n : 0;
}

cudaError_t launch_row_stats(const VerifyArgs& a, cudaStream_t s, int grid) {
  const long long items = (long long)a.B * a.slots * a.nseg;
  if (items == 0) return cudaSuccess;
  const long long need = (items + kStatsWarps - 1) / kStatsWarps;
  if (grid > need) grid = (int)need;
  if (a.dtype == kF32)
    row_stats_kernel<kF32><<<grid, 32 * kStatsWarps, kSmem, s>>>(a);
  else
    row_stats_kernel<kBF16><<<grid, 32 * kStatsWarps, kSmem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace sv
