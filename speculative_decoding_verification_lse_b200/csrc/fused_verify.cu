// fused_verify.cu -- the whole verification step in one launch.
//
// Every warp of a persistent grid is an independent worker that repeats:
//   1. claim a published race segment, if any, and run it (race_device.cuh);
//   2. otherwise take the next statistics ticket -- (request, row, segment) in
//      request-major order -- and compute that segment's statistics
//      (stats_device.cuh);
//   3. the warp that finishes the last segment of a request runs that
//      request's accept scan (scan_device.cuh) and publishes its race.
// Race work is claimed through a cursor over requests: a warp claims segments
// of the request under the cursor only when that request is published, and
// moves the cursor on once every segment is claimed.  Nothing ever waits for
// another warp: a warp that finds no published race work takes a ticket, and
// one that finds no ticket left exits.  Whoever publishes the request under
// the cursor carries on with every published request behind it, so no race is
// left unclaimed.  The sampled rows of a request were streamed moments earlier,
// so the race mostly reads them again from L2, while other warps keep HBM busy.
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

__device__ __forceinline__ unsigned load_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void store_release(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Number of statistics items request b completes with.
__device__ __forceinline__ unsigned items_needed(const VerifyArgs& a, const ReqParams& rp) {
  const int rows = (rp.Db + 1) + (rp.mode == kGreedy ? 0 : rp.Db);
  return (unsigned)rows * (unsigned)a.nseg;
}

// Lane 0: claim one published race segment; returns the request (or -1).
__device__ int claim_race(const VerifyArgs& a, int* seg) {
  for (int guard = 0; guard < 4 * a.B + 8; ++guard) {  // each pass moves the cursor or returns
    const unsigned r = load_acquire(&a.fstate->cursor);
    if (r >= (unsigned)a.B) return -1;
    const unsigned st = load_acquire(&a.ready[r]);
    if (st == kReadyNone) return -1;  // not published yet: its publisher will run it
    if (st == kReadyRace) {
      const unsigned s = atomicAdd(&a.rclaim[r], 1u);
      if (s < (unsigned)a.nseg) {
        *seg = (int)s;
        return (int)r;
      }
    }
    atomicCAS(&a.fstate->cursor, r, r + 1);  // fully claimed (or nothing to race): move on
  }
  return -1;
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

template <int DT>
__global__ void __launch_bounds__(kThreads) fused_kernel(VerifyArgs a) {
  extern __shared__ __align__(16) unsigned char s_dyn[];
  __shared__ RaceDesc s_rd[kWarps];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  RowRes* rows = reinterpret_cast<RowRes*>(s_dyn) + (size_t)warp * a.slots;
  const unsigned per_req = (unsigned)a.slots * (unsigned)a.nseg;
  const unsigned total = (unsigned)a.B * per_req;

  for (;;) {
    // 1. published race work first
    int rb = -1, rs = 0;
    if (lane == 0) rb = claim_race(a, &rs);
    rb = __shfl_sync(0xFFFFFFFFu, rb, 0);
    if (rb >= 0) {
      rs = __shfl_sync(0xFFFFFFFFu, rs, 0);
      __threadfence();
      load_race_desc(a.rdesc + rb, &s_rd[warp]);
      race_item<DT>(a, rb, rs, s_rd[warp]);
      continue;
    }

    // 2. the next statistics item
    unsigned tk = 0;
    if (lane == 0) tk = atomicAdd(&a.fstate->next_ticket, 1u);
    tk = __shfl_sync(0xFFFFFFFFu, tk, 0);
    if (tk >= total) break;
    const int b = (int)(tk / per_req);
    const unsigned rem = tk % per_req;
    const int slot = (int)(rem / (unsigned)a.nseg);
    const int seg = (int)(rem % (unsigned)a.nseg);
    const ReqParams rp = load_req(a, b);

    if (rp.err) {
      // invalid request parameters: its first ticket reports them
      if (slot == 0 && seg == 0) finish_request(a, b, rows);
      continue;
    }
    if (!row_needed(a, slot, rp)) continue;
    stats_item<DT>(a, b, slot, seg, rp);

    // 3. the warp finishing a request's last item runs its scan and publishes
    unsigned prev = 0;
    if (lane == 0) {
      __threadfence();
      prev = atomicAdd(&a.done[b], 1u);
    }
    prev = __shfl_sync(0xFFFFFFFFu, prev, 0);
    if (prev + 1u == items_needed(a, rp)) finish_request(a, b, rows);
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
