// scan_device.cuh -- device code of the per-request accept scan, shared by the
// split accept-scan kernel and the fused kernel.
//
// One warp per request.  The warp merges the segment partials of each row it
// reads in double precision (merge_row), then lane d tests draft position d:
//   a_d = min(1, p_d(x_d) / q_d(x_d))  ("Speculative Speculative Decoding –
//   асинхронизируй это.", rule items 1-2, read as acceptance with probability
//   min(1, p/q)), u_d from Philox, accept iff u_d < a_d;
// a ballot gives n, the first rejected position ("NVIDIA: öt irányelv ...",
// "Mit csinál a spekulatív dekódolás?": accept in order up to the first
// mismatch), and AL = n + 1.
// Greedy requests accept while x_d is the target row's argmax and emit the
// argmax of row n.  Stochastic requests leave slot n to the race and describe
// it in the workspace.  Saguaro requests use
//   ln q'(x) = ln q(x) + [x in K] ln c - ln Z,  Z = 1 - (1 - c) sum_{x in K} q(x)
// (saguaro recipe items 1-2: down-weight the draft's top tokens, renormalised).
#pragma once
#include "philox.cuh"
#include "sv_common.cuh"

#include <float.h>
#include <limits.h>
#include <math.h>

namespace sv {

constexpr double kLn2d = 0.69314718055994530942;

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// Merge the segment partials of one row, by the whole warp (lane l takes
// segments l, l+32, ...; the partials were written by other warps, so they are
// read through L2).  Every lane returns the same RowRes.
//   LSE = ln2 * (Mk + log2 sum_s S_s 2^(m_s k2 - Mk)),  Mk = M k2, M = max_s m_s
// PS(s) and TP(s): the partial and the top list of segment s (the row's
// segments in order, wherever they are stored).
template <class PS, class TP>
__device__ inline void merge_row_at(PS ps_at, TP tp_at, bool has_tp, int nseg, bool lse, float k2,
                                    int k, RowRes& r) {
  const int lane = threadIdx.x & 31;
  float mx = -INFINITY;
  int am = INT_MAX, ms = nseg;
  uint32_t bad = 0;
  double Sd = 0.0;  // relative to 2^(mx*k2)
  for (int s = lane; s < nseg; s += 32) {
    const float4 raw = __ldcg(reinterpret_cast<const float4*>(ps_at(s)));
    const float m = raw.x, S = raw.y;
    const int ai = __float_as_int(raw.z);
    bad |= __float_as_uint(raw.w);
    if (m > mx || ms == nseg) {  // segments ascend: strict '>' keeps the lowest one
      if (lse && Sd > 0.0) Sd *= exp2((double)(mx * k2) - (double)(m * k2));
      mx = m;
      am = ai;
      ms = s;
    }
    if (lse && S > 0.0f) Sd += (double)S * exp2((double)(m * k2) - (double)(mx * k2));
  }
  // the lowest segment holding the largest value; its partial has the argmax
  const unsigned long long win = warp_max_u64(value_index_key(mx, ms));
  const float M = key_value(win);
  const int Ms = key_index(win);
  const unsigned src = __ffs(__ballot_sync(0xFFFFFFFFu, ms == Ms)) - 1;
  const int Mi = __shfl_sync(0xFFFFFFFFu, am, src);
  bad = __any_sync(0xFFFFFFFFu, bad) ? 1u : 0u;
  if (M == -INFINITY) bad = 1u;  // every entry masked: no distribution
  r.argmax = Mi;
  r.mseg = Ms < nseg ? Ms : 0;
  r.lse = NAN;
  if (lse) {
    const double Mk = (double)(M * k2);
    double part = 0.0;
    if (Sd > 0.0) part = Sd * exp2((double)(mx * k2) - Mk);
    const double S = warp_sum_d(part);
    if (!bad) r.lse = (Mk + log2(S)) * kLn2d;
  }
  r.ntop = 0;
  if (has_tp) {
    // k rounds: each lane offers the best head of its segments' lists
    int head[kMaxSegs / 32];
    const int mine = (nseg - lane + 31) / 32;
    for (int i = 0; i < mine; ++i) head[i] = 0;
    for (int rd = 0; rd < k; ++rd) {
      unsigned long long best = 0ull;
      int bi = -1;
      for (int i = 0; i < mine; ++i) {
        if (head[i] >= k) continue;
        const TopPart* t = tp_at(lane + 32 * i);
        const int ci = __ldcg(&t->i[head[i]]);
        if (ci == INT_MAX) continue;
        const unsigned long long kk = value_index_key(__ldcg(&t->v[head[i]]), ci);
        if (kk > best) {
          best = kk;
          bi = i;
        }
      }
      const unsigned long long w = warp_max_u64(best);
      if (w == 0ull) break;
      if (best == w) ++head[bi];
      r.top[r.ntop] = key_index(w);
      r.topv[r.ntop] = key_value(w);
      ++r.ntop;
    }
  }
  r.bad = bad;
}

// A row whose segments' partials are consecutive at ps (and top lists at tp).
__device__ inline void merge_row(const PartStat* ps, const TopPart* tp, int nseg, bool lse,
                                 float k2, int k, RowRes& r) {
  merge_row_at([=](int s) { return ps + s; }, [=](int s) { return tp + s; }, tp != nullptr, nseg,
               lse, k2, k, r);
}

// Whether row `slot` of a request with parameters rp is read by the rule.
__device__ __forceinline__ bool slot_needed(const VerifyArgs& a, int b, int slot, const ReqParams& rp) {
  return row_read(a, b, slot, rp);
}

// Merge row `slot` of request b (one full warp) from the partials PS(s) and
// top lists TP(s) of its nseg segments (has_tp: a saguaro draft row); lane 0
// writes the result to dst.
template <class PS, class TP>
__device__ inline void merge_into_at(const VerifyArgs& a, const ReqParams& rp, int slot, PS ps_at,
                                     TP tp_at, bool has_tp, int nseg, RowRes* dst) {
  const bool greedy = rp.mode == kGreedy;
  const float k2 = greedy ? 0.0f : log2e_over_T(rp.T);
  (void)slot;
  RowRes rr;
  merge_row_at(ps_at, tp_at, has_tp, nseg, !greedy, k2, a.saguaro_k, rr);
  rr.lnZ = 0.0;
  if (has_tp && !rr.bad) {
    // Z = 1 - (1 - c) * sum_{x in K} q(x)
    const double Td = (double)rp.T;
    double mass = 0.0;
    for (int i = 0; i < rr.ntop; ++i) mass += exp((double)rr.topv[i] / Td - rr.lse);
    rr.lnZ = log1p(-(1.0 - (double)a.saguaro_c) * mass);
  }
  if ((threadIdx.x & 31) == 0) *dst = rr;
}

// Merge row `slot` of request b from the workspace's partials.
__device__ inline void merge_row_into(const VerifyArgs& a, int b, int slot, const ReqParams& rp,
                                      RowRes* dst) {
  const int Dm = a.D_max;
  const bool is_t = slot <= Dm;
  const int d = is_t ? slot : slot - Dm - 1;
  const PartStat* ps = a.pstat + ((size_t)b * a.slots + slot) * a.nseg;
  const TopPart* tp =
      (!is_t && rp.mode == kSaguaro) ? a.tpart + ((size_t)b * Dm + d) * a.nseg : nullptr;
  merge_into_at(a, rp, slot, [=](int s) { return ps + s; }, [=](int s) { return tp + s; },
                tp != nullptr, a.nseg, dst);
}

// The scan's per-position inputs, which do not depend on the merged rows: lane
// d < D_b holds draft token x_d and, for a sampling request, its target and
// draft logits and its accept word.  Loaded by the scanning warp before it
// merges rows, so that their latency overlaps the merge.
struct ScanInputs {
  int x;
  float zt, zq;
  uint32_t uw;
  uint32_t err;
};

__device__ __forceinline__ ScanInputs scan_inputs(const VerifyArgs& a, int b, const ReqParams& rp) {
  const int lane = threadIdx.x & 31;
  ScanInputs in;
  in.x = -1;
  in.zt = in.zq = 0.0f;
  in.uw = 0u;
  in.err = rp.err;
  if (!rp.err && lane < rp.Db) {
    in.x = a.tokens[(size_t)b * a.D_max + lane];
    if (in.x < 0 || in.x >= a.V_global) {
      in.err |= kFlagBadToken;
    } else if (rp.mode != kGreedy) {
      in.zt = load_logit(a, row_base(a, b, lane), in.x);
      in.zq = load_logit(a, row_base(a, b, a.D_max + 1 + lane), in.x);
      in.uw = accept_word(seed_of(a), a.request_offset + (uint32_t)b, (uint32_t)lane);
    }
  }
  return in;
}

// The accept test of draft position d of a request with parameters rp, from
// its merged rows (rows[d] the target row, rows[D_max + 1 + d] the draft row)
// and the scan inputs of lane d: greedy -- the draft token is the target
// row's argmax; otherwise u_d < min(1, p(x_d) / q'(x_d)).  *near: |u - a| <
// 1e-5 (sampling requests).
__device__ inline bool accept_position(const VerifyArgs& a, const ReqParams& rp,
                                       const RowRes* rows, const ScanInputs& in, int d,
                                       bool* near) {
  *near = false;
  if (rp.mode == kGreedy) return in.x == rows[d].argmax;
  const double Td = (double)rp.T;
  const RowRes& rq = rows[a.D_max + 1 + d];
  const double lp = (double)in.zt / Td - rows[d].lse;
  double lq = (double)in.zq / Td - rq.lse;
  if (rp.mode == kSaguaro && lq != -INFINITY) {
    bool in_k = false;
    for (int i = 0; i < rq.ntop; ++i) in_k |= (rq.top[i] == in.x);
    lq += (in_k ? log((double)a.saguaro_c) : 0.0) - rq.lnZ;
  }
  double acc;
  if (lp == -INFINITY)
    acc = 0.0;  // p(x) = 0: the target never emits x
  else if (lq == -INFINITY)
    acc = 1.0;
  else
    acc = fmin(1.0, exp(lp - lq));
  const double u = (double)(in.uw >> 8) * 0x1p-24;
  *near = fabs(u - acc) < 1e-5;
  return u < acc;
}

// The accept scan of request b by one full warp, once every row it reads has
// been merged into rows (2*D_max+1 entries of shared memory); in: the warp's
// scan_inputs.  Writes the
// outputs (slot n too for greedy), the flags and the row LSEs, and lane 0
// writes the race description to *rd; returns the race kind (same on all
// lanes).
__device__ inline int scan_request(const VerifyArgs& a, int b, const RowRes* rows, RaceDesc* rd,
                                   const ScanInputs& in) {
  const int lane = threadIdx.x & 31;
  const int Dm = a.D_max;
  const ReqParams rp = load_req(a, b);
  const uint32_t g = a.request_offset + (uint32_t)b;
  int32_t* ot = a.out_tokens + (size_t)b * (Dm + 1);
  const int x = in.x;
  uint32_t err = __reduce_or_sync(0xFFFFFFFFu, in.err);

  const bool greedy = rp.mode == kGreedy;
  const bool saguaro = rp.mode == kSaguaro;
  const double Td = (double)rp.T;
  const double c = (double)a.saguaro_c;

  // the merged rows this request reads
  if (!err) {
    uint32_t nonfinite = 0;
    for (int slot = lane; slot < a.slots; slot += 32)
      if (slot_needed(a, b, slot, rp) && rows[slot].bad) nonfinite = kFlagNonfinite;
    err |= __reduce_or_sync(0xFFFFFFFFu, nonfinite);
  }

  if (a.out_draft_top) {
    // the k largest logits of each saguaro draft row tested (the speculation
    // keys of "Speculative Speculative Decoding": the draft's top tokens)
    const int k = a.saguaro_k;
    for (int i = lane; i < Dm * k; i += 32) {
      const int d = i / k, j = i - d * k;
      int v = -1;
      if (!err && saguaro && d < rp.Db && j < rows[Dm + 1 + d].ntop) v = rows[Dm + 1 + d].top[j];
      a.out_draft_top[(size_t)b * Dm * k + i] = v;
    }
  }

  if (err) {
    for (int j = lane; j <= Dm; j += 32) ot[j] = -1;
    if (a.out_row_lse)
      for (int s = lane; s < a.slots; s += 32) a.out_row_lse[(size_t)b * a.slots + s] = NAN;
    if (lane == 0) {
      a.out_al[b] = -1;
      if (a.out_flags) a.out_flags[b] = err;
      atomicOr(a.status, err);
      rd->kind = kRaceNone;
    }
    __syncwarp();
    return kRaceNone;
  }

  // test every draft position in parallel
  bool accept = false, near = false;
  if (lane < rp.Db) accept = accept_position(a, rp, rows, in, lane, &near);
  const uint32_t rej = __ballot_sync(0xFFFFFFFFu, lane < rp.Db && !accept);
  const int n = rej ? __ffs(rej) - 1 : rp.Db;
  const uint32_t nearm = __ballot_sync(0xFFFFFFFFu, near);
  const uint32_t tested = (n < rp.Db) ? (uint32_t)((2ull << n) - 1ull)
                                      : (uint32_t)((1ull << rp.Db) - 1ull);
  const uint32_t flags = (nearm & tested) ? kFlagAcceptNearTie : 0u;
  const int kind = greedy ? kRaceNone : (n < rp.Db ? kRaceResidual : kRaceBonus);

  // outputs: accepted drafts, then slot n, then -1
  for (int j = lane; j <= Dm; j += 32) {
    int v = -1;
    if (j < n)
      v = a.tokens[(size_t)b * Dm + j];
    else if (j == n && greedy)
      v = rows[n].argmax;
    ot[j] = v;
  }
  if (a.out_row_lse) {
    for (int s = lane; s < a.slots; s += 32) {
      const bool is_t = s <= Dm;
      const int d = is_t ? s : s - Dm - 1;
      const bool used = !greedy && (is_t ? d <= rp.Db : d < rp.Db);
      a.out_row_lse[(size_t)b * a.slots + s] = used ? (float)rows[s].lse : NAN;
    }
  }
  if (lane == 0) {
    a.out_al[b] = n + 1;
    if (a.out_flags) a.out_flags[b] = flags;
    rd->kind = kind;
    rd->n = n;
    rd->g = g;
    rd->flags = flags;
    rd->T = Td;
    rd->lse_t = rows[n].lse;
    rd->k2 = log2e_over_T(rp.T);
    rd->K0 = -INFINITY;
    rd->cup = INFINITY;
    rd->lse_q = 0.0;
    rd->ln_c = log(c);
    rd->ln_Z = 0.0;
    rd->ntop = 0;
    rd->ref_seg = rows[n].mseg;
    if (kind == kRaceResidual) {
      const RowRes& rq = rows[Dm + 1 + n];
      rd->lse_q = rq.lse;
      if (saguaro) {
        rd->ln_Z = rq.lnZ;
        rd->ntop = rq.ntop;
        for (int i = 0; i < rq.ntop; ++i) rd->top[i] = rq.top[i];
      }
    }
  }
  __syncwarp();
  return kind;
}

}  // namespace sv
