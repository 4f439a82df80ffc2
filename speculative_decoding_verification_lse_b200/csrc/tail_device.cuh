// tail_device.cuh -- everything after the statistics pass, in one of two
// layouts (the launcher picks one per call):
//   per request: one CTA per request merges the request's rows
//     (scan_device.cuh), runs its accept scan, finds a reference key for the
//     race's word filter and races the sampled row, warp w streaming segments
//     w, w + 8, ... and sharing the best key found so far in shared memory
//     (tail_request).  Best when there are at least as many requests as
//     multiprocessors.
//   scan, then race items: one CTA per request does the merge, the scan and the
//     reference key (scan_cta); then one warp per (request, segment) races the
//     segment -- or half of it, while the items fit in one wave of resident
//     warps -- and the warp that finishes a request's last item (an atomic
//     counter, no waiting) combines them and writes the token (race_item).
//     The items are taken rank-major -- every request's segment with the
//     largest logit first, then every request's second, ... -- so that by the
//     later waves each request's best key so far (ordered bits in global
//     memory, raised with an atomic maximum) is usually the row's best and the
//     filter leaves almost no survivors.  Best for small batches, whose races
//     it spreads over the whole GPU.
#pragma once
#include "race_device.cuh"
#include "scan_device.cuh"

namespace sv {

struct TailShared {
  RowRes rows[2 * kMaxDraft + 1];
  ScanInputs in[32];
  float segm[kThreads];  // the sampled row's segment maxima (race order)
  RaceDesc rd;
  double key[kWarps];
  double best[kWarps], second[kWarps];
  int idx[kWarps];
  unsigned long long k0;  // the best exact key so far (per-request layout), as ordered bits
};

// The merged rows of request b into rows[0 .. slots), by the whole CTA: from
// the segment partials, or -- after the early-exit rounds (a.ee_n set) -- from
// the rows those rounds merged, the rows past the decided position n left
// without statistics (never read by the scan's decisions: the first rejection
// is at n, or n = D_b).  Ends with the CTA synchronised.
__device__ __forceinline__ void gather_rows(const VerifyArgs& a, int b, const ReqParams& rp,
                                            RowRes* rows) {
  const int warp = threadIdx.x >> 5;
  if (a.ee_n == nullptr) {
    for (int slot = warp; slot < a.slots; slot += kWarps)
      if (slot_needed(a, b, slot, rp)) merge_row_into(a, b, slot, rp, &rows[slot]);
  } else {
    const int n = a.ee_n[b];
    for (int slot = threadIdx.x; slot < a.slots; slot += kThreads) {
      const int d = slot <= a.D_max ? slot : slot - a.D_max - 1;
      RowRes r;
      if (d <= n) {
        r = a.rowres[(size_t)b * a.slots + slot];
      } else {
        memset(&r, 0, sizeof r);
        r.lse = NAN;
        r.argmax = -1;
      }
      rows[slot] = r;
    }
  }
  __syncthreads();
}

// The scan's inputs of request b into S.in, by the CTA's last warp: the draft
// tokens, their logits and the accept words -- kernel inputs only, so the
// tail kernels load them before they wait for the statistics kernel (while it
// drains); the first barrier of gather_rows makes them visible.
__device__ __forceinline__ void load_scan_inputs(const VerifyArgs& a, int b, ScanInputs* in) {
  if ((threadIdx.x >> 5) == kWarps - 1) in[threadIdx.x & 31] = scan_inputs(a, b, load_req(a, b));
}

// The end of request b's race, by one warp: r is the combination of every
// segment's result.  An empty residual ({p > q} empty through rounding) is
// drawn from p on the same row instead; then the token and the flags are
// written.
template <int DT>
__device__ __forceinline__ void finish_race(const VerifyArgs& a, int b, const RaceDesc& rd, Best r) {
  const int lane = threadIdx.x & 31;
  const bool residual = rd.kind == kRaceResidual;
  uint32_t flags = rd.flags;
  if (r.idx < 0 && residual) {
    flags |= kFlagResidualEmpty;
    const char* trow = row_base(a, b, rd.n);
    Best Bb{-INFINITY, -INFINITY, -1};
    for (int s = 0; s < a.nseg; ++s)
      Bb = combine(Bb, race_segment<DT>(row_ctx(a), rd, trow, nullptr, false, s, -INFINITY, INFINITY));
    r = Bb;
  }
  if (lane == 0) {
    if (r.best - r.second < 1e-6) flags |= kFlagRaceNearTie;
    a.out_tokens[(size_t)b * (a.D_max + 1) + rd.n] = r.idx;
    if (a.out_flags) a.out_flags[b] = flags;
    if (flags & kFlagResidualEmpty) atomicOr(a.status, kFlagResidualEmpty);
  }
}

// Request b, everything after its statistics, by the whole CTA (kThreads
// threads, S in shared memory; S.in holds the scan's inputs, which the kernel
// loads before it waits for the statistics: load_scan_inputs); every thread
// returns at the same point.
template <int DT>
__device__ __forceinline__ void tail_request(const VerifyArgs& a, int b, TailShared& S) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const ReqParams rp = load_req(a, b);
  gather_rows(a, b, rp, S.rows);
  if (warp == 0) scan_request(a, b, S.rows, &S.rd, S.in[lane]);
  __syncthreads();
  const int kind = S.rd.kind;
  if (kind == kRaceNone) {
    __syncthreads();  // S is reused by the next request
    return;
  }

  // the reference key, from the segment holding the sampled row's largest logit
  // (the request's Philox stream from kernel arguments, the same on every thread)
  const RaceStream R = race_stream(seed_of(a), a.request_offset + (uint32_t)b, (uint32_t)a.vocab_offset >> 2);
  const double kw = race_ref_key_warp<DT>(a, S.rd, R, b, S.rd.ref_seg, warp, kWarps);
  if (lane == 0) S.key[warp] = kw;
  if (threadIdx.x == 0) S.k0 = ordered_u64(-INFINITY);
  __syncthreads();
  double K0 = S.key[0];
#pragma unroll
  for (int w = 1; w < kWarps; ++w) K0 = fmax(K0, S.key[w]);

  // the race, warp w taking segments w, w + 8, ... as one stream
  const bool residual = kind == kRaceResidual;
  const char* trow = row_base(a, b, S.rd.n);
  const char* qrow = residual ? row_base(a, b, a.D_max + 1 + S.rd.n) : nullptr;
  const Best B = race_span_in<DT>(a, S.rd, R, trow, qrow, residual, warp, kWarps, K0, &S.k0);
  if (lane == 0) {
    S.best[warp] = B.best;
    S.second[warp] = B.second;
    S.idx[warp] = B.idx;
  }
  __syncthreads();
  if (warp == 0) {
    Best r{-INFINITY, -INFINITY, -1};
    if (lane < kWarps) {
      r.best = S.best[lane];
      r.second = S.second[lane];
      r.idx = S.idx[lane];
    }
    finish_race<DT>(a, b, S.rd, warp_combine(r));
  }
  __syncthreads();  // S is reused by the next request
}

// Request b by the C CTAs of a thread-block cluster (C > 1; rank 0's S.in as
// for tail_request): rank 0 merges the rows, runs the accept scan and finds the
// reference key, as tail_request does; the other ranks copy its race
// description through distributed shared memory, and the cluster's C * kWarps
// warps race the sampled row (warp w of rank r taking segments 8r + w,
// 8r + w + 8C, ...); rank 0 combines the ranks' results in rank order and
// writes the token.  rb: this CTA's slot for its result.  Every thread of the
// cluster returns at the same point.
template <int DT, class Cluster>
__device__ __forceinline__ void tail_request_cluster(const VerifyArgs& a, int b, TailShared& S,
                                                     Cluster& cluster, Best* rb) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C = (int)cluster.num_blocks(), rank = (int)cluster.block_rank();
  const RaceStream R = race_stream(seed_of(a), a.request_offset + (uint32_t)b, (uint32_t)a.vocab_offset >> 2);
  if (rank == 0) {
    const ReqParams rp = load_req(a, b);
    gather_rows(a, b, rp, S.rows);
    if (warp == 0) scan_request(a, b, S.rows, &S.rd, S.in[lane]);
    __syncthreads();
    if (S.rd.kind != kRaceNone) {
      const double kw = race_ref_key_warp<DT>(a, S.rd, R, b, S.rd.ref_seg, warp, kWarps);
      if (lane == 0) S.key[warp] = kw;
      __syncthreads();
      if (threadIdx.x == 0) {
        double K0 = S.key[0];
        for (int w = 1; w < kWarps; ++w) K0 = fmax(K0, S.key[w]);
        S.rd.K0 = K0;
      }
    }
  }
  cluster.sync();  // rank 0's race description is complete
  constexpr int d16 = sizeof(RaceDesc) / 16;
  static_assert(sizeof(RaceDesc) % 16 == 0, "RaceDesc is copied in 16-byte pieces");
  if (rank != 0 && threadIdx.x < d16)
    reinterpret_cast<uint4*>(&S.rd)[threadIdx.x] =
        reinterpret_cast<const uint4*>(cluster.map_shared_rank(&S.rd, 0))[threadIdx.x];
  if (threadIdx.x == 0) S.k0 = ordered_u64(-INFINITY);
  cluster.sync();  // the copies are done before rank 0 goes on
  const int kind = S.rd.kind;
  if (kind == kRaceNone) return;
  const bool residual = kind == kRaceResidual;
  const char* trow = row_base(a, b, S.rd.n);
  const char* qrow = residual ? row_base(a, b, a.D_max + 1 + S.rd.n) : nullptr;
  const Best B = race_span_in<DT>(a, S.rd, R, trow, qrow, residual, rank * kWarps + warp,
                                  C * kWarps, S.rd.K0, &S.k0);
  if (lane == 0) {
    S.best[warp] = B.best;
    S.second[warp] = B.second;
    S.idx[warp] = B.idx;
  }
  __syncthreads();
  if (warp == 0) {
    Best r{-INFINITY, -INFINITY, -1};
    if (lane < kWarps) {
      r.best = S.best[lane];
      r.second = S.second[lane];
      r.idx = S.idx[lane];
    }
    r = warp_combine(r);
    if (lane == 0) *rb = r;
  }
  cluster.sync();  // every rank's result is in place
  if (rank == 0 && warp == 0) {
    Best r{-INFINITY, -INFINITY, -1};
    if (lane < C) r = *cluster.map_shared_rank(rb, lane);
    finish_race<DT>(a, b, S.rd, warp_combine(r));
  }
  cluster.sync();  // the other ranks' shared memory stays until rank 0 has read it
}

// Request b, by the whole CTA (kThreads threads, S in shared memory; S.in as
// for tail_request); every thread returns at the same point.  Writes the
// request's outputs (all of them unless it races), and for a race a.rdesc[b]
// and the race counters.
template <int DT>
__device__ __forceinline__ void scan_cta(const VerifyArgs& a, int b, TailShared& S) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const ReqParams rp = load_req(a, b);
  gather_rows(a, b, rp, S.rows);
  if (warp == 0) scan_request(a, b, S.rows, &S.rd, S.in[lane]);
  __syncthreads();
  const int kind = S.rd.kind;
  if (kind != kRaceNone) {
    // the reference key: each warp ranks a share of the segment holding the
    // sampled row's largest logit and takes the exact key of its best token
    const RaceStream R = race_stream(seed_of(a), S.rd.g, (uint32_t)a.vocab_offset >> 2);
    // the sampled row's segment maxima, for the race order, load while the
    // reference key is searched
    const bool ranked = a.nseg <= kThreads;
    float m = 0.0f;
    if (ranked && threadIdx.x < a.nseg)
      m = __ldcg(&a.pstat[((size_t)b * a.slots + S.rd.n) * a.nseg + threadIdx.x].m);
    const double kw = race_ref_key_warp<DT>(a, S.rd, R, b, S.rd.ref_seg, warp, kWarps);
    if (lane == 0) S.key[warp] = kw;
    if (ranked && threadIdx.x < a.nseg) S.segm[threadIdx.x] = m;
    __syncthreads();
    // the race order: rank of each segment by its largest logit (ties: lower
    // index first); rows of more than kThreads segments keep index order
    for (int sg = threadIdx.x; sg < a.nseg; sg += kThreads) {
      int rank = sg;
      if (ranked) {
        const float ms = S.segm[sg];
        rank = 0;
        for (int j = 0; j < a.nseg; ++j) {
          const float mj = S.segm[j];
          rank += (mj > ms || (mj == ms && j < sg)) ? 1 : 0;
        }
      }
      a.rorder[(size_t)b * a.nseg + rank] = (unsigned short)sg;
    }
    if (warp == 0) {
      double K0 = lane < kWarps ? S.key[lane] : -INFINITY;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) K0 = fmax(K0, __shfl_xor_sync(0xFFFFFFFFu, K0, o));
      if (lane == 0) {
        S.rd.K0 = K0;
        S.rd.cup = filter_offset(K0, S.rd.lse_t);
        a.rcount[b] = 0u;
        a.best_key[b] = K0 > -INFINITY ? ordered_u64(K0) : 0ull;
      }
      __syncwarp();
      constexpr int n16 = sizeof(RaceDesc) / 16;
      static_assert(sizeof(RaceDesc) % 16 == 0, "RaceDesc is copied in 16-byte pieces");
      if (lane < n16)
        reinterpret_cast<uint4*>(a.rdesc + b)[lane] = reinterpret_cast<const uint4*>(&S.rd)[lane];
    }
  } else if (threadIdx.x == 0) {
    a.rdesc[b].kind = kRaceNone;
  }
  __syncthreads();  // S is reused by the next request
}

// Race item `item`, by one warp; rd: the warp's shared slot for the request's
// race description.  Each segment is cut into a.rsplit parts of whole 32-token
// groups; the items are rank-major over the parts (item = (rank * rsplit + h)
// * B + b: part h of request b's segment of rank `rank`).
template <int DT>
__device__ __forceinline__ void race_item(const VerifyArgs& a, long long item, RaceDesc* rd) {
  constexpr int NG = kLaneVecs / (32 / Lanes<DT>::VEC);
  const int lane = threadIdx.x & 31;
  const int b = (int)(item % a.B);
  const int pr = (int)(item / a.B);
  const int rank = pr / a.rsplit, h = pr % a.rsplit;
  const int nparts = a.nseg * a.rsplit;
  constexpr int n16 = sizeof(RaceDesc) / 16;
  if (lane < n16)
    reinterpret_cast<uint4*>(rd)[lane] = __ldcg(reinterpret_cast<const uint4*>(a.rdesc + b) + lane);
  __syncwarp();
  if (rd->kind == kRaceNone) return;
  const int seg = __ldcg(&a.rorder[(size_t)b * a.nseg + rank]);
  const bool residual = rd->kind == kRaceResidual;
  const char* trow = row_base(a, b, rd->n);
  const char* qrow = residual ? row_base(a, b, a.D_max + 1 + rd->n) : nullptr;
  const unsigned long long bk = *(volatile unsigned long long*)&a.best_key[b];
  const double K = fmax(rd->K0, bk ? from_ordered_u64(bk) : -INFINITY);
  const Best sb = race_segment_in<DT>(a, *rd, race_stream(seed_of(a), rd->g, (uint32_t)a.vocab_offset >> 2), trow, qrow, residual,
                                      seg, K, filter_offset(K, rd->lse_t), h * NG / a.rsplit,
                                      (h + 1) * NG / a.rsplit);
  unsigned prev = 0;
  if (lane == 0) {
    if (sb.idx >= 0) atomicMax(&a.best_key[b], ordered_u64(sb.best));
    RacePart p;
    p.best = sb.best;
    p.second = sb.second;
    p.idx = sb.idx;
    p.pad = 0;
    a.rpart[(size_t)b * nparts + seg * a.rsplit + h] = p;
    __threadfence();
    prev = atomicAdd(&a.rcount[b], 1u);
  }
  prev = __shfl_sync(0xFFFFFFFFu, prev, 0);
  if (prev != (unsigned)(nparts - 1)) return;

  // the request's last part: combine every part's result
  __threadfence();
  Best r{-INFINITY, -INFINITY, -1};
  for (int s = lane; s < nparts; s += 32) {
    const RacePart* pp = a.rpart + (size_t)b * nparts + s;
    Best o;
    o.best = __ldcg(&pp->best);
    o.second = __ldcg(&pp->second);
    o.idx = __ldcg(&pp->idx);
    r = combine(r, o);
  }
  finish_race<DT>(a, b, *rd, warp_combine(r));
}

}  // namespace sv
