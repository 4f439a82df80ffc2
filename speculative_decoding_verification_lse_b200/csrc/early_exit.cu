// early_exit.cu -- the early-exit schedule: rows read position by position,
// only for the requests that accepted every earlier draft.
//
// The rule stops at the first rejection ("Speculative Speculative Decoding –
// асинхронизируй это.", rule items 1-2; "NVIDIA: öt irányelv ...", "Mit csinál
// a spekulatív dekódolás?": accept in order up to the first mismatch), so the
// rows of the positions after it never enter a decision.  The split path reads
// them all at once, in parallel; this schedule reads the positions in rounds
// -- position 0, then 1-2, then 3 to D_max -- and after each round tests the
// round's positions of the requests still accepting:
//   ee_stats_kernel  the statistics of the round's rows (target rows d <= D_b,
//                    draft rows d < D_b of sampling requests) of the requests
//                    in the round's list, as the statistics pass computes them;
//   ee_step_kernel   one CTA per listed request: merges those rows into the
//                    workspace, tests the round's positions with the scan's own
//                    accept test, and either decides n (the first rejection, or
//                    D_b once every draft is accepted and row D_b is merged) or
//                    puts the request on the next round's list.
// The verification then finishes as usual (the scan, the race, the outputs)
// from the merged rows (gather_rows).  The outputs equal the split path's,
// except that the rows of positions past the outcome report no LSE (NaN) and
// those never read no non-finite flag.
// The bytes read are those of the positions up to each request's n: about
// half of the split path's at the AL distributions of the synthetic workloads.
#include <cstring>

#include "tail_device.cuh"

namespace sv {

namespace {

// The request of list entry k in round r (round 0 lists every request).
__device__ __forceinline__ int ee_request(const VerifyArgs& a, int r, int k) {
  return r == 0 ? k : a.ee_alive[(size_t)(r & 1) * a.B + k];
}

__device__ __forceinline__ int ee_listed(const VerifyArgs& a, int r) {
  return r == 0 ? a.B : (int)*(volatile unsigned*)&a.ee_count[32 * (r & 1)];
}

// Round r's statistics, positions [p0, p1): warp w0 of W takes the items w0,
// w0 + W, ... of (list entry, slot of the round, segment), the round's slots
// being the target and draft rows of each position in turn.
template <int DT, bool WITH_TOP>
__global__ void __launch_bounds__(kThreads, 3) ee_stats_kernel(VerifyArgs a, int r, int p0, int p1) {
  wait_for_previous_kernel();
  // the next round's list starts empty (its last reader, round r - 1, is done)
  if (blockIdx.x == 0 && threadIdx.x == 0) a.ee_count[32 * ((r + 1) & 1)] = 0u;
  const int listed = ee_listed(a, r);
  const int nsl = 2 * (p1 - p0);
  const unsigned per_entry = (unsigned)nsl * (unsigned)a.nseg;
  const unsigned total = (unsigned)listed * per_entry;
  // items from eight ticket counters (zero at launch), counter c handing out
  // c, c + 8, ..., so that the warps that run ahead take more
  const unsigned lane = threadIdx.x & 31;
  const unsigned c = (blockIdx.x * kWarps + (threadIdx.x >> 5)) & 7u;
  unsigned* ctr = a.ticket + 32 * c;
  for (;;) {
    unsigned i = 0;
    if (lane == 0) i = atomicAdd(ctr, 1u) * 8u + c;
    i = __shfl_sync(0xFFFFFFFFu, i, 0);
    if (i >= total) break;
    const int k = (int)(i / per_entry);
    const unsigned rem = i % per_entry;
    const int j = (int)(rem / (unsigned)a.nseg), seg = (int)(rem % (unsigned)a.nseg);
    const int d = p0 + (j >> 1);
    const bool draft = (j & 1) != 0;
    const int b = ee_request(a, r, k);
    const ReqParams rp = load_req(a, b);
    if (rp.err || d > rp.Db || (draft && d >= rp.Db)) continue;
    const int slot = draft ? a.D_max + 1 + d : d;
    if (!slot_needed(a, b, slot, rp)) continue;
    stats_item<DT, WITH_TOP>(a, b, slot, seg, rp);
  }
  allow_next_kernel();
}

// Round r's decisions, positions [p0, p1): CTA k takes list entry k.  CTA 0
// also zeroes the statistics tickets for the next round.
__global__ void __launch_bounds__(kThreads) ee_step_kernel(VerifyArgs a, int r, int p0, int p1) {
  wait_for_previous_kernel();
  if (blockIdx.x == 0 && threadIdx.x < 8) a.ticket[32 * threadIdx.x] = 0u;
  const int k = blockIdx.x;
  if (k >= ee_listed(a, r)) {
    allow_next_kernel();
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = ee_request(a, r, k);
  const ReqParams rp = load_req(a, b);
  if (rp.err) {
    // the scan reports the parameter error; no row is read
    if (threadIdx.x == 0) a.ee_n[b] = -1;
    allow_next_kernel();
    return;
  }
  RowRes* rows = a.rowres + (size_t)b * a.slots;
  // the scan's inputs (draft tokens, their logits, the accept words) by the
  // last warp while the others merge
  __shared__ ScanInputs s_in[32];
  if (warp == kWarps - 1) s_in[lane] = scan_inputs(a, b, rp);
  // the round's rows (a request is listed only while p0 <= D_b)
  const int dend = min(p1 - 1, rp.Db);  // the last position whose target row is read
  for (int j = warp; j < 2 * (dend - p0 + 1); j += kWarps) {
    const int d = p0 + (j >> 1);
    const bool draft = (j & 1) != 0;
    if (draft && d >= rp.Db) continue;
    const int slot = draft ? a.D_max + 1 + d : d;
    if (slot_needed(a, b, slot, rp)) merge_row_into(a, b, slot, rp, &rows[slot]);
  }
  __syncthreads();
  if (warp == 0) {
    const ScanInputs in = s_in[lane];
    // rows without statistics, or inputs out of range: decided here, the scan reports it
    uint32_t err = in.err;
    for (int j = lane; j < 2 * (dend - p0 + 1); j += 32) {
      const int d = p0 + (j >> 1);
      const bool draft = (j & 1) != 0;
      if (draft && d >= rp.Db) continue;
      const int slot = draft ? a.D_max + 1 + d : d;
      if (slot_needed(a, b, slot, rp) && rows[slot].bad) err |= kFlagNonfinite;
    }
    err = __reduce_or_sync(0xFFFFFFFFu, err);
    bool accept = true, near = false;
    if (!err && lane >= p0 && lane <= dend && lane < rp.Db)
      accept = accept_position(a, rp, rows, in, lane, &near);
    const uint32_t rej = __ballot_sync(0xFFFFFFFFu, !accept);
    if (lane == 0) {
      if (err) {
        a.ee_n[b] = dend;  // every row read so far is merged
      } else if (rej) {
        a.ee_n[b] = __ffs(rej) - 1;  // the first rejection
      } else if (rp.Db < p1) {
        a.ee_n[b] = rp.Db;  // every draft accepted; row D_b merged this round
      } else {
        const unsigned idx = atomicAdd(&a.ee_count[32 * ((r + 1) & 1)], 1u);
        a.ee_alive[(size_t)((r + 1) & 1) * a.B + idx] = b;
      }
    }
  }
  allow_next_kernel();
}

template <typename K>
cudaError_t launch_pdl(K kernel, unsigned grid, cudaStream_t s, const VerifyArgs& a, int r, int p0,
                       int p1) {
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, a, r, p0, p1);
}

}  // namespace

// The rounds' position boundaries: {0, 1, 3, D_max + 1}, the ones past
// D_max + 1 dropped.  Returns the number of rounds.
int ee_rounds(int D_max, int* bounds) {
  int n = 0;
  bounds[n++] = 0;
  if (1 < D_max + 1) bounds[n++] = 1;
  if (3 < D_max + 1) bounds[n++] = 3;
  bounds[n++] = D_max + 1;
  return n - 1;
}

// The rounds (statistics then decisions for each), on stream s; grid: the
// statistics kernel's persistent grid.  The verification then finishes with
// a.ee_n set.
cudaError_t launch_early_exit_rounds(const VerifyArgs& a, cudaStream_t s, int grid) {
  if (a.B == 0) return cudaSuccess;
  int bounds[4];
  const int R = ee_rounds(a.D_max, bounds);
  const bool top = a.mode == kSaguaro || a.mode_per_req != nullptr;
  for (int r = 0; r < R; ++r) {
    const int p0 = bounds[r], p1 = bounds[r + 1];
    cudaError_t e;
    if (a.dtype == kF32)
      e = top ? launch_pdl(ee_stats_kernel<kF32, true>, grid, s, a, r, p0, p1)
              : launch_pdl(ee_stats_kernel<kF32, false>, grid, s, a, r, p0, p1);
    else
      e = top ? launch_pdl(ee_stats_kernel<kBF16, true>, grid, s, a, r, p0, p1)
              : launch_pdl(ee_stats_kernel<kBF16, false>, grid, s, a, r, p0, p1);
    if (e != cudaSuccess) return e;
    if ((e = launch_pdl(ee_step_kernel, (unsigned)a.B, s, a, r, p0, p1)) != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace sv
