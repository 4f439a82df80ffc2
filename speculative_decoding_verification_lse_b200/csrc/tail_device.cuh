// tail_device.cuh -- everything after the statistics pass for one request, by
// one CTA: merge the request's rows (scan_device.cuh), run the accept scan,
// find a reference key for the race, then race the sampled row segment by
// segment (race_device.cuh) and write the token.
//
// The CTA's warps share the best exact key found so far in shared memory, so a
// warp's later segments are filtered against the best key of every segment
// finished before them (a larger K0 leaves fewer survivors).  Nothing here
// waits on another CTA.
#pragma once
#include "race_device.cuh"
#include "scan_device.cuh"

namespace sv {

constexpr int kTailWarps = 8;
constexpr int kTailThreads = 32 * kTailWarps;

struct TailShared {
  RowRes rows[2 * kMaxDraft + 1];
  RaceDesc rd;
  double key[kTailWarps];
  double best[kTailWarps], second[kTailWarps];
  int idx[kTailWarps];
  unsigned long long k0;  // the best exact key so far, as ordered bits
};

// Doubles as unsigned integers in the same order (-0 < +0 aside).
__device__ __forceinline__ unsigned long long ordered_u64(double v) {
  const unsigned long long b = (unsigned long long)__double_as_longlong(v);
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

__device__ __forceinline__ double from_ordered_u64(unsigned long long o) {
  const unsigned long long b = (o >> 63) ? (o & 0x7FFFFFFFFFFFFFFFull) : ~o;
  return __longlong_as_double((long long)b);
}

// Request b, by the whole CTA (kTailThreads threads, S in shared memory).
// Every thread returns at the same point.
template <int DT>
__device__ __forceinline__ void tail_request(const VerifyArgs& a, int b, TailShared& S) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int nw = kTailWarps;
  const ReqParams rp = load_req(a, b);
  for (int slot = warp; slot < a.slots; slot += nw)
    if (slot_needed(a, slot, rp)) merge_row_into(a, b, slot, rp, &S.rows[slot]);
  __syncthreads();
  if (warp == 0) scan_request(a, b, S.rows, &S.rd);
  __syncthreads();
  const int kind = S.rd.kind;
  if (kind == kRaceNone) {
    __syncthreads();  // S is reused by the next request
    return;
  }

  // the reference key, from the segment holding the sampled row's largest logit
  const uint32_t g = a.request_offset + (uint32_t)b;
  const RaceStream R = race_stream(a.seed, g);
  const double kw = race_ref_key_warp<DT>(a, S.rd, R, b, S.rd.ref_seg, warp, nw);
  if (lane == 0) S.key[warp] = kw;
  if (threadIdx.x == 0) S.k0 = ordered_u64(-INFINITY);
  __syncthreads();
  double K0 = S.key[0];
#pragma unroll
  for (int w = 1; w < nw; ++w) K0 = fmax(K0, S.key[w]);

  // the race, warp w taking segments w, w + nw, ...
  const bool residual = kind == kRaceResidual;
  const int n = S.rd.n;
  const char* trow = row_base(a, b, n);
  const char* qrow = residual ? row_base(a, b, a.D_max + 1 + n) : nullptr;
  Best B{-INFINITY, -INFINITY, -1};
  for (int seg = warp; seg < a.nseg; seg += nw) {
    const double K = fmax(K0, from_ordered_u64(*(volatile unsigned long long*)&S.k0));
    const Best sb = race_segment_in<DT>(a, S.rd, R, trow, qrow, residual, seg, K,
                                        filter_offset(K, S.rd.lse_t));
    if (lane == 0 && sb.idx >= 0) atomicMax(&S.k0, ordered_u64(sb.best));
    B = combine(B, sb);
  }
  if (lane == 0) {
    S.best[warp] = B.best;
    S.second[warp] = B.second;
    S.idx[warp] = B.idx;
  }
  __syncthreads();
  if (warp == 0) {
    Best r{-INFINITY, -INFINITY, -1};
    if (lane < nw) {
      r.best = S.best[lane];
      r.second = S.second[lane];
      r.idx = S.idx[lane];
    }
    r = warp_combine(r);
    uint32_t flags = S.rd.flags;
    if (r.idx < 0 && residual) {
      // {p > q} was empty through rounding: draw from p on the same row instead
      flags |= kFlagResidualEmpty;
      Best Bb{-INFINITY, -INFINITY, -1};
      for (int s = 0; s < a.nseg; ++s)
        Bb = combine(Bb, race_segment<DT>(a, S.rd, trow, nullptr, false, s, -INFINITY, INFINITY));
      r = Bb;
    }
    if (lane == 0) {
      if (r.best - r.second < 1e-6) flags |= kFlagRaceNearTie;
      a.out_tokens[(size_t)b * (a.D_max + 1) + n] = r.idx;
      if (a.out_flags) a.out_flags[b] = flags;
      if (flags & kFlagResidualEmpty) atomicOr(a.status, kFlagResidualEmpty);
    }
  }
  __syncthreads();  // S is reused by the next request
}

}  // namespace sv
