// fused_verify.cu -- the whole verification step in one launch, with each
// request's tail overlapping the statistics of the requests after it.
//
// Every warp of a persistent grid runs one work loop over three kinds of work:
//   statistics  batches of (request, row, 8 KiB segment) items from eight
//               ticket counters, in request-major order (stats_device.cuh);
//   row merges  the warp that finishes the last segment of a row (a counter per
//               row) merges its partials into the row's LSE / argmax / top list;
//   scans       the warp that merges the last row of a request (a counter per
//               request) runs its accept scan (scan_device.cuh), writes the
//               outputs, and publishes the request's race as parts;
//   race parts  (a segment, or half of one) taken by any warp from the
//               published races (race_device.cuh); the warp that finishes a
//               request's last part combines the parts and writes the token.
// A warp takes a race part whenever one is published and otherwise the next
// statistics batch, so the races (bound by Philox's integer multiplies) run
// beside the statistics (bound by HBM and the exp unit) instead of after them,
// and only the last requests' tails remain once the logits are read.
//
// Sources: "Accélérer Sonar par la Spéculation", sections "Décodage spéculatif"
// and "Cible-Brouillon" (the rows, the extra token, the full-distribution
// comparison); "Speculative Speculative Decoding – асинхронизируй это.", the
// numbered rule (items 1-3) and the saguaro recipe; "NVIDIA: öt irányelv ...",
// "Mit csinál a spekulatív dekódolás?" (accept in order up to the first
// mismatch).  The results are those of the split path, bit for bit.
//
// Ordering.  A finished item is made visible by its writer's fence before the
// counter it increments; the warp that sees a count complete fences before it
// reads what the others wrote (the last-arriver pattern), so no warp ever waits
// for a statistic or a row.  The only waits are for races to be published:
// an idle warp, holding no statistics work, polls for them with a growing
// sleep, and a claimed part's request index appears right after its count
// (written by a warp that never waits in between).  Every wait is bounded by
// time (about two seconds); a warp that gives up sets SV_STATUS_TIMEOUT in the
// status word and leaves, and the call's outputs are then undefined.  The
// launch is cooperative, so every CTA is resident and no wait can be on a CTA
// that is not running.
#include "work_queue.cuh"
#include "tail_device.cuh"

namespace sv {

namespace {

constexpr unsigned kBatch = 2;  // consecutive statistics items per ticket

// Per-warp shared scratch: the merged rows of the request being scanned, the
// scan's inputs and the race description of the part being raced.
struct WarpScratch {
  RaceDesc rd;
  ScanInputs in[32];
};

__device__ __forceinline__ size_t scratch_bytes(int slots) {
  return align_up(sizeof(WarpScratch) + (size_t)slots * sizeof(RowRes), 16);
}

// Race parts of a request: rsplit parts per segment.
__device__ __forceinline__ int race_parts(const VerifyArgs& a) { return a.nseg * a.rsplit; }

// The accept scan of request b, once all its rows are merged (one warp);
// publishes its race, if any, and counts the request as scanned.
template <int DT>
__device__ void scan_and_publish(const VerifyArgs& a, int b, WarpScratch& W, RowRes* rows) {
  const int lane = threadIdx.x & 31;
  const ReqParams rp = load_req(a, b);
  W.in[lane] = scan_inputs(a, b, rp);
  // the merged rows, written by other warps: through L2
  const int n16 = a.slots * (int)(sizeof(RowRes) / 16);
  const uint4* src = reinterpret_cast<const uint4*>(a.rowres + (size_t)b * a.slots);
  uint4* dst = reinterpret_cast<uint4*>(rows);
  for (int i = lane; i < n16; i += 32) dst[i] = __ldcg(src + i);
  __syncwarp();
  const int kind = scan_request(a, b, rows, &W.rd, W.in[lane]);
  unsigned* ctl = a.ctl;
  if (kind != kRaceNone) {
    constexpr int d16 = sizeof(RaceDesc) / 16;
    static_assert(sizeof(RaceDesc) % 16 == 0, "RaceDesc is copied in 16-byte pieces");
    if (lane < d16)
      reinterpret_cast<uint4*>(a.rdesc + b)[lane] = reinterpret_cast<const uint4*>(&W.rd)[lane];
    __syncwarp();
    if (lane == 0) publish_race(ctl, a.pubq, (unsigned)b);
  }
  if (lane == 0) {
    __threadfence();
    atomicAdd(&ctl[kCtlScanned], 1u);
  }
  __syncwarp();
}

// Items finished for one row: count them; the warp that completes the row
// merges it, and the warp that completes the request's last row scans it.
template <int DT>
__device__ __noinline__ void row_done(const VerifyArgs& a, int b, int slot, unsigned cnt, WarpScratch& W,
                         RowRes* rows) {
  const int lane = threadIdx.x & 31;
  const unsigned row = (unsigned)b * a.slots + slot;
  unsigned last = 0;
  if (lane == 0) {
    __threadfence();  // this warp's partials before its count
    last = atomicAdd(&a.rowcnt[row], cnt) + cnt == (unsigned)a.nseg;
    if (last) __threadfence();  // every partial of the row before reading them
  }
  if (!__shfl_sync(0xFFFFFFFFu, last, 0)) return;
  const ReqParams rp = load_req(a, b);
  if (slot_needed(a, b, slot, rp)) merge_row_into(a, b, slot, rp, &a.rowres[row]);
  unsigned req_last = 0;
  if (lane == 0) {
    __threadfence();
    req_last = atomicAdd(&a.reqcnt[b], 1u) + 1 == (unsigned)a.slots;
    if (req_last) __threadfence();
  }
  if (!__shfl_sync(0xFFFFFFFFu, req_last, 0)) return;
  scan_and_publish<DT>(a, b, W, rows);
}

// Statistics batch t (items t*kBatch ...), then the bookkeeping of its rows.
template <int DT, bool WITH_TOP>
__device__ void stats_batch(const VerifyArgs& a, unsigned t, unsigned total, WarpScratch& W,
                            RowRes* rows) {
  const unsigned per_req = (unsigned)a.slots * (unsigned)a.nseg;
  const unsigned end = min(total, (t + 1) * kBatch);
  int cb = -1, cs = -1;
  unsigned cnt = 0;
  for (unsigned i = t * kBatch; i < end; ++i) {
    const int b = (int)(i / per_req);
    const unsigned r = i % per_req;
    const int slot = (int)(r / (unsigned)a.nseg), seg = (int)(r % (unsigned)a.nseg);
    if ((b != cb || slot != cs) && cnt) {
      row_done<DT>(a, cb, cs, cnt, W, rows);
      cnt = 0;
    }
    cb = b;
    cs = slot;
    const ReqParams rp = load_req(a, b);
    if (row_needed(a, b, slot, rp)) stats_item<DT, WITH_TOP>(a, b, slot, seg, rp);
    ++cnt;
  }
  if (cnt) row_done<DT>(a, cb, cs, cnt, W, rows);
}

// Race part `item` of the published races (item / parts-th race, part item % parts).
template <int DT>
__device__ __noinline__ void race_part_item(const VerifyArgs& a, unsigned item, WarpScratch& W) {
  constexpr int VEC = Lanes<DT>::VEC, QV = 32 / VEC, NG = kLaneVecs / QV;
  const int lane = threadIdx.x & 31;
  const int nparts = race_parts(a);
  const unsigned j = item / (unsigned)nparts;
  const int part = (int)(item % (unsigned)nparts);
  unsigned bq = 0;
  if (lane == 0) bq = wait_published(a.pubq, j, a.status);
  bq = __shfl_sync(0xFFFFFFFFu, bq, 0);
  if (bq == 0) return;  // gave up (status set)
  const int b = (int)bq - 1;
  constexpr int d16 = sizeof(RaceDesc) / 16;
  if (lane < d16)
    reinterpret_cast<uint4*>(&W.rd)[lane] = __ldcg(reinterpret_cast<const uint4*>(a.rdesc + b) + lane);
  __syncwarp();
  const RaceDesc& rd = W.rd;
  const bool residual = rd.kind == kRaceResidual;
  const char* trow = row_base(a, b, rd.n);
  const char* qrow = residual ? row_base(a, b, a.D_max + 1 + rd.n) : nullptr;
  const int seg = part / a.rsplit, h = part % a.rsplit;
  const Best sb = race_part<DT>(a, rd, trow, qrow, residual, seg,
                                h * NG / a.rsplit, (h + 1) * NG / a.rsplit, &a.best_key[b]);
  unsigned prev = 0;
  if (lane == 0) {
    if (sb.idx >= 0) atomicMax(&a.best_key[b], ordered_u64(sb.best));
    RacePart p;
    p.best = sb.best;
    p.second = sb.second;
    p.idx = sb.idx;
    p.pad = 0;
    a.rpart[(size_t)b * nparts + part] = p;
    __threadfence();
    prev = atomicAdd(&a.rcount[b], 1u);
    if (prev == (unsigned)(nparts - 1)) __threadfence();
  }
  prev = __shfl_sync(0xFFFFFFFFu, prev, 0);
  if (prev != (unsigned)(nparts - 1)) return;
  // the request's last part: combine every part's result
  Best r{-INFINITY, -INFINITY, -1};
  for (int s = lane; s < nparts; s += 32) {
    const RacePart* pp = a.rpart + (size_t)b * nparts + s;
    Best o;
    o.best = __ldcg(&pp->best);
    o.second = __ldcg(&pp->second);
    o.idx = __ldcg(&pp->idx);
    r = combine(r, o);
  }
  finish_race<DT>(a, b, rd, warp_combine(r));
}

template <int DT, bool WITH_TOP>
__global__ void __launch_bounds__(kThreads, 3) fused_kernel(VerifyArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  WarpScratch& W = *reinterpret_cast<WarpScratch*>(smem + warp * scratch_bytes(a.slots));
  RowRes* rows = reinterpret_cast<RowRes*>(smem + warp * scratch_bytes(a.slots) + sizeof(WarpScratch));

  const unsigned total = (unsigned)a.B * (unsigned)a.slots * (unsigned)a.nseg;
  const unsigned batches = (total + kBatch - 1) / kBatch;
  const unsigned nparts = (unsigned)race_parts(a);
  const unsigned c = (blockIdx.x * kWarps + warp) & 7u;
  unsigned* ctr = a.ticket + 32 * c;
  unsigned t = 0;
  if (lane == 0) t = atomicAdd(ctr, 1u) * 8u + c;
  t = __shfl_sync(0xFFFFFFFFu, t, 0);

  // multiprocessors that race while statistics remain (the rest stream rows
  // until none are left), so that most multiprocessors keep one loop's code in
  // their instruction cache
  unsigned smid;
  asm("mov.u32 %0, %%smid;" : "=r"(smid));
  const bool race_sm = a.race_sm_every <= 0 || smid % (unsigned)a.race_sm_every == 0;

  WaitClock clock;
  clock.start();
  unsigned pend = kNoPart;  // a claimed race part not yet published (or taken)
  for (;;) {
    // a published race part first: claim one when more are published than claimed
    unsigned avail = 0, done = 0;
    if (lane == 0) {
      const unsigned pub = load_acquire_gpu(&a.ctl[kCtlPublished]) * nparts;
      if (pend == kNoPart && (race_sm || t >= batches) && pub > load_volatile(&a.ctl[kCtlClaimed]))
        pend = atomicAdd(&a.ctl[kCtlClaimed], 1u);
      avail = pend != kNoPart && pend < pub;
      if (!avail && t >= batches && load_acquire_gpu(&a.ctl[kCtlScanned]) == (unsigned)a.B) {
        // every race is published: done once each part is claimed and this warp
        // holds none of them (the count is read after the scans' count)
        const unsigned fin = load_acquire_gpu(&a.ctl[kCtlPublished]) * nparts;
        if (pend != kNoPart && pend < fin) avail = 1;
        else done = load_volatile(&a.ctl[kCtlClaimed]) >= fin;
      }
    }
    avail = __shfl_sync(0xFFFFFFFFu, avail, 0);
    if (avail) {
      const unsigned item = __shfl_sync(0xFFFFFFFFu, pend, 0);
      pend = kNoPart;
      race_part_item<DT>(a, item, W);
      clock.start();
      continue;
    }
    if (t < batches) {
      unsigned tn = 0;
      if (lane == 0) tn = atomicAdd(ctr, 1u) * 8u + c;  // the next ticket, while this batch runs
      stats_batch<DT, WITH_TOP>(a, t, total, W, rows);
      t = __shfl_sync(0xFFFFFFFFu, tn, 0);
      clock.start();
      continue;
    }
    if (__shfl_sync(0xFFFFFFFFu, done, 0)) break;
    // nothing to do yet: the last requests' scans are still running elsewhere
    if (!clock.wait(a.status)) break;
  }
}

template <int DT, bool WITH_TOP>
int blocks_per_sm(int slots) {
  int n = 0;
  const size_t smem = (size_t)kWarps * align_up(sizeof(WarpScratch) + (size_t)slots * sizeof(RowRes), 16);
  if (cudaFuncSetAttribute(fused_kernel<DT, WITH_TOP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return 0;
  const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
      &n, fused_kernel<DT, WITH_TOP>, kThreads, smem);
  return e == cudaSuccess ? n : 0;
}

}  // namespace

// Resident fused CTAs per SM (the smaller of the two builds, with and without
// saguaro top lists).
int fused_blocks_per_sm(int dtype, int slots) {
  if (dtype == kF32) return min(blocks_per_sm<kF32, true>(slots), blocks_per_sm<kF32, false>(slots));
  return min(blocks_per_sm<kBF16, true>(slots), blocks_per_sm<kBF16, false>(slots));
}

// While statistics remain, one multiprocessor in kRaceSmEvery takes race parts
// (about a fifth of the device: the races' share of the work on large
// batches); small batches race on every multiprocessor.
constexpr int kRaceSmEvery = 5;

int fused_race_sm_every(const VerifyArgs& a, int grid) {
  const long long items = (long long)a.B * a.slots * a.nseg;
  return items >= 8LL * grid * kWarps ? kRaceSmEvery : 0;
}

// grid: the most CTAs that can be resident at once (fused_blocks_per_sm x SMs);
// the workspace's zero region must read zero (the launcher clears it).
cudaError_t launch_fused(const VerifyArgs& a, cudaStream_t s, int grid) {
  if (a.B == 0) return cudaSuccess;
  // no more CTAs than there is work for: 8 warps' statistics batches, or one per request
  const long long items = (long long)a.B * a.slots * a.nseg;
  long long want = (items + kBatch * kWarps - 1) / (kBatch * kWarps);
  if (want < a.B) want = a.B;
  if (grid > want) grid = (int)want;
  const size_t smem = (size_t)kWarps * align_up(sizeof(WarpScratch) + (size_t)a.slots * sizeof(RowRes), 16);
  VerifyArgs arg = a;
  void* params[] = {&arg};
  const bool top = a.mode == kSaguaro || a.mode_per_req != nullptr;
  const void* fn;
  if (a.dtype == kF32)
    fn = top ? (const void*)fused_kernel<kF32, true> : (const void*)fused_kernel<kF32, false>;
  else
    fn = top ? (const void*)fused_kernel<kBF16, true> : (const void*)fused_kernel<kBF16, false>;
  // the kernel's dynamic shared memory limit is one attribute for every draft
  // length, last set by whichever occupancy query ran last: set it for this one
  const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return cudaLaunchCooperativeKernel(fn, dim3(grid), dim3(kThreads), params, smem, s);
}

}  // namespace sv
