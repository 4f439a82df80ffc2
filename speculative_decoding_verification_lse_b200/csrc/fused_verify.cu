// fused_verify.cu -- the whole verification step in one launch.
//
// Every warp of a persistent grid takes tickets from one ordered ticket space
// and does what its ticket names:
//   * a statistics ticket: one 8 KiB segment of one row (stats_device.cuh); the
//     warp that finishes a row's last segment merges that row, and the warp
//     that merges a request's last row runs that request's accept scan
//     (scan_device.cuh) and publishes it;
//   * a race ticket: one segment of one request's race (race_device.cuh).
// The ticket space lists, request after request, the statistics segments of
// request r followed by the race segments of request r - L, with a lag of L
// requests (about 64 MiB of logits) so that a race ticket is normally taken
// after its request has been published, while that request's sampled rows are
// still in L2.  A warp holding a race ticket whose request is not yet published
// waits for it, polling with a sleep and a bounded number of polls (an expired
// wait sets SV_STATUS_TIMEOUT and leaves that token at -1).  The wait always
// ends: the request's statistics tickets all come earlier in the order, so they
// were taken by warps that are running, and statistics work never waits.  For
// the same reason a warp prefetches its next ticket only while it works on a
// statistics segment, never while it waits.
//
// All counters live in a workspace region cleared before the launch.
#include "race_device.cuh"
#include "scan_device.cuh"
#include "stats_device.cuh"

namespace sv {

namespace {

constexpr unsigned kReadyNone = 0u;   // request not finished yet
constexpr unsigned kReadyRace = 1u;   // race published
constexpr unsigned kReadyDone = 2u;   // finished, nothing to race (greedy or error)
constexpr unsigned kLagTickets = 8192;  // statistics tickets (64 MiB) between a request and its race
constexpr int kWaitPolls = 1 << 20;     // with a 128 ns sleep each: well over 0.1 s

__device__ __forceinline__ unsigned load_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void store_release(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// The ordered ticket space.
struct Tickets {
  unsigned S, R, L, B;      // stats and race tickets per request, lag, requests
  unsigned p1, p2, total;   // ends of the three phases
  __device__ __forceinline__ void init(const VerifyArgs& a) {
    S = (unsigned)a.slots * (unsigned)a.nseg;
    R = (unsigned)a.nseg;
    B = (unsigned)a.B;
    L = (kLagTickets + S - 1) / S;
    if (L < 1) L = 1;
    if (L > B) L = B;
    p1 = L * S;                      // requests [0, L): statistics only
    p2 = p1 + (B - L) * (S + R);     // requests [L, B): statistics of r, race of r - L
    total = p2 + L * R;              // the races of the last L requests
  }
  // false: race ticket (b, seg); true: statistics ticket (b, slot, seg)
  __device__ __forceinline__ bool decode(const VerifyArgs& a, unsigned t, int& b, int& slot,
                                         int& seg) const {
    unsigned r, off;
    bool stats;
    if (t < p1) {
      r = t / S;
      off = t % S;
      stats = true;
    } else if (t < p2) {
      const unsigned u = t - p1;
      r = L + u / (S + R);
      off = u % (S + R);
      stats = off < S;
      if (!stats) {
        r -= L;
        off -= S;
      }
    } else {
      const unsigned u = t - p2;
      r = B - L + u / R;
      off = u % R;
      stats = false;
    }
    b = (int)r;
    if (stats) {
      slot = (int)(off / (unsigned)a.nseg);
      seg = (int)(off % (unsigned)a.nseg);
    } else {
      slot = 0;
      seg = (int)off;
    }
    return stats;
  }
};

// Number of rows request b reads.
__device__ __forceinline__ unsigned rows_needed(const ReqParams& rp) {
  return (unsigned)((rp.Db + 1) + (rp.mode == kGreedy ? 0 : rp.Db));
}

// The scan of request b by this warp, then its publication.
__device__ __forceinline__ void finish_request(const VerifyArgs& a, int b, RowRes* rows) {
  __threadfence();
  const int kind = scan_request(a, b, rows);
  if ((threadIdx.x & 31) == 0) {
    __threadfence();
    store_release(&a.ready[b], kind == kRaceNone ? kReadyDone : kReadyRace);
  }
  __syncwarp();
}

// Lane 0: the publication state of request b, waiting (bounded) until it is set.
__device__ unsigned wait_ready(const VerifyArgs& a, int b) {
  unsigned st = load_acquire(&a.ready[b]);
  for (int i = 0; st == kReadyNone && i < kWaitPolls; ++i) {
    __nanosleep(128);
    st = load_acquire(&a.ready[b]);
  }
  if (st == kReadyNone) atomicOr(a.status, kStatusTimeout);
  return st;
}

template <int DT>
__global__ void __launch_bounds__(kThreads) fused_kernel(VerifyArgs a) {
  extern __shared__ __align__(16) unsigned char s_dyn[];
  __shared__ RaceDesc s_rd[kWarps];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  RowRes* rows = reinterpret_cast<RowRes*>(s_dyn) + (size_t)warp * a.slots;
  Tickets T;
  T.init(a);

  unsigned t = 0;
  if (lane == 0) t = atomicAdd(&a.fstate->next_ticket, 1u);
  t = __shfl_sync(0xFFFFFFFFu, t, 0);
  while (t < T.total) {
    int b, slot, seg;
    if (T.decode(a, t, b, slot, seg)) {
      // a statistics segment: fetch the next ticket now, use it afterwards
      unsigned tn = 0;
      if (lane == 0) tn = atomicAdd(&a.fstate->next_ticket, 1u);
      const ReqParams rp = load_req(a, b);
      if (rp.err) {
        // invalid request parameters: the request's first ticket reports them
        if (slot == 0 && seg == 0) finish_request(a, b, rows);
      } else if (row_needed(a, slot, rp)) {
        stats_item<DT>(a, b, slot, seg, rp);
        // the warp finishing the row's last segment merges the row ...
        unsigned prev = 0;
        if (lane == 0) {
          __threadfence();
          prev = atomicAdd(&a.row_done[(size_t)b * a.slots + slot], 1u);
        }
        prev = __shfl_sync(0xFFFFFFFFu, prev, 0);
        if (prev + 1u == (unsigned)a.nseg) {
          __threadfence();
          merge_row_global(a, b, slot, rp);
          // ... and the warp merging the request's last row runs the scan
          if (lane == 0) {
            __threadfence();
            prev = atomicAdd(&a.req_rows[b], 1u);
          }
          prev = __shfl_sync(0xFFFFFFFFu, prev, 0);
          if (prev + 1u == rows_needed(rp)) finish_request(a, b, rows);
        }
      }
      t = __shfl_sync(0xFFFFFFFFu, tn, 0);
    } else {
      // a race segment: its request must have been published
      unsigned st = 0;
      if (lane == 0) st = wait_ready(a, b);
      st = __shfl_sync(0xFFFFFFFFu, st, 0);
      if (st == kReadyRace) {
        __threadfence();
        load_race_desc(a.rdesc + b, &s_rd[warp]);
        race_item<DT>(a, b, seg, s_rd[warp]);
      }
      if (lane == 0) t = atomicAdd(&a.fstate->next_ticket, 1u);
      t = __shfl_sync(0xFFFFFFFFu, t, 0);
    }
  }
}

}  // namespace

size_t fused_smem_bytes(int D_max) { return (size_t)kWarps * (2 * D_max + 1) * sizeof(RowRes); }

cudaError_t launch_fused(const VerifyArgs& a, cudaStream_t s, int grid) {
  if (a.B == 0) return cudaSuccess;
  const size_t smem = fused_smem_bytes(a.D_max);
  if (a.dtype == kF32)
    fused_kernel<kF32><<<grid, kThreads, smem, s>>>(a);
  else
    fused_kernel<kBF16><<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

int fused_blocks_per_sm(int dtype) {
  // sized for the largest draft length; smaller D_max only frees shared memory
  const size_t smem = fused_smem_bytes(kMaxDraft);
  int n = 0;
  cudaError_t e;
  if (dtype == kF32) {
    cudaFuncSetAttribute(fused_kernel<kF32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fused_kernel<kF32>, kThreads, smem);
  } else {
    cudaFuncSetAttribute(fused_kernel<kBF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fused_kernel<kBF16>, kThreads, smem);
  }
  return e == cudaSuccess ? n : 0;
}

}  // namespace sv
