// accept_scan.cu -- the per-request accept scan.
//
// One warp per request.  Lane s merges the chunk partials of row slot s in
// chunk order, in double precision: LSE = ln2 * (M + log2 sum_c S_c 2^(mk_c - M)).
// Lane d then tests draft position d:
//   a_d = min(1, p_d(x_d) / q_d(x_d))  ("Speculative Speculative Decoding –
//   асинхронизируй это.", rule items 1-2, read as acceptance with probability
//   min(1, p/q)), u_d from Philox, accept iff u_d < a_d;
// a ballot gives n, the first rejected position ("NVIDIA: öt irányelv ...",
// "Mit csinál a spekulatív dekódolás?": accept in order up to the first
// mismatch), and AL = n + 1.
// Greedy requests accept while x_d is the target row's argmax and emit the
// argmax of row n.  Stochastic requests leave slot n to the race kernel and
// describe its race in the workspace.  Saguaro requests use
//   ln q'(x) = ln q(x) + [x in K] ln c - ln Z,  Z = 1 - (1 - c) sum_{x in K} q(x)
// (saguaro recipe items 1-2: down-weight the draft's top tokens, renormalised).
#include "philox.cuh"
#include "sv_common.cuh"

#include <float.h>
#include <limits.h>
#include <math.h>

namespace sv {

namespace {

constexpr double kLn2 = 0.69314718055994530942;

struct RowRes {
  double lse;   // natural-log LSE at T (stochastic rows)
  double lnZ;   // saguaro draft rows: ln Z
  int argmax;   // target rows
  uint32_t bad;
  int ntop;
  int top[kMaxTopK];
  float topv[kMaxTopK];
};

__device__ void merge_row(const ChunkStat* cs, int nch, bool lse, bool top, int k, RowRes& r) {
  float m = -INFINITY;
  int am = INT_MAX;
  uint32_t bad = 0;
  float M = -INFINITY;
  for (int c = 0; c < nch; ++c) {
    const float mc = cs[c].m;
    bad |= cs[c].bad;
    if (mc > m) {  // chunks ascend in index: strict '>' keeps the lowest index
      m = mc;
      am = cs[c].argmax;
    }
    if (lse) M = fmaxf(M, cs[c].mk);
  }
  if (m == -INFINITY) bad = 1;  // every entry masked: no distribution
  r.argmax = am;
  r.lse = NAN;
  if (lse && !bad) {
    double S = 0.0;
    for (int c = 0; c < nch; ++c) {
      const float Sc = cs[c].S;
      if (Sc > 0.0f) S += (double)Sc * exp2((double)cs[c].mk - (double)M);
    }
    r.lse = ((double)M + log2(S)) * kLn2;
  }
  r.ntop = 0;
  if (top) {
    // k rounds over the chunks' lists: largest value, then lowest index
    int head[64];
    const int nc = nch < 64 ? nch : 64;
    for (int c = 0; c < nc; ++c) head[c] = 0;
    for (int i = 0; i < k; ++i) {
      int bc = -1;
      float bv = -INFINITY;
      int bi = INT_MAX;
      for (int c = 0; c < nc; ++c) {
        if (head[c] >= cs[c].ntop) continue;
        const int ci = cs[c].topi[head[c]];
        if (ci == INT_MAX) continue;
        const float cv = cs[c].topv[head[c]];
        if (bc < 0 || cv > bv || (cv == bv && ci < bi)) {
          bc = c;
          bv = cv;
          bi = ci;
        }
      }
      if (bc < 0) break;
      ++head[bc];
      r.top[r.ntop] = bi;
      r.topv[r.ntop] = bv;
      ++r.ntop;
    }
  }
  r.bad = bad;
}

__global__ void __launch_bounds__(32 * kScanWarps) accept_scan_kernel(VerifyArgs a) {
  __shared__ RowRes s_rows[kScanWarps][2 * kMaxDraft + 1];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int b = blockIdx.x * kScanWarps + warp;
  if (b >= a.B) return;
  RowRes* rows = s_rows[warp];
  const int Dm = a.D_max;
  const ReqParams rp = load_req(a, b);
  const uint32_t g = a.request_offset + (uint32_t)b;
  int32_t* ot = a.out_tokens + (size_t)b * (Dm + 1);
  uint32_t err = rp.err;

  // draft tokens of the tested positions
  int x = -1;
  if (!err && lane < rp.Db) {
    x = a.tokens[(size_t)b * Dm + lane];
    if (x < 0 || x >= a.V) err |= kFlagBadToken;
  }
  err = __reduce_or_sync(0xFFFFFFFFu, err);

  const bool greedy = rp.mode == kGreedy;
  const bool saguaro = rp.mode == kSaguaro;
  const double Td = (double)rp.T;
  const double c = (double)a.saguaro_c;

  // merge the rows this request reads
  uint32_t nonfinite = 0;
  if (!err) {
    for (int s = lane; s < a.slots; s += 32) {
      const bool is_t = s <= Dm;
      const int d = is_t ? s : s - Dm - 1;
      const bool needed = is_t ? d <= rp.Db : (d < rp.Db && !greedy);
      if (!needed) continue;
      const ChunkStat* cs = a.cstat + ((size_t)b * a.slots + s) * a.nch;
      merge_row(cs, a.nch, !greedy, !is_t && saguaro, a.saguaro_k, rows[s]);
      nonfinite |= rows[s].bad ? kFlagNonfinite : 0u;
      if (!is_t && saguaro && !rows[s].bad) {
        // Z = 1 - (1 - c) * sum_{x in K} q(x)
        double mass = 0.0;
        for (int i = 0; i < rows[s].ntop; ++i)
          mass += exp((double)rows[s].topv[i] / Td - rows[s].lse);
        rows[s].lnZ = log1p(-(1.0 - c) * mass);
      }
    }
    err |= __reduce_or_sync(0xFFFFFFFFu, nonfinite);
  }
  __syncwarp();

  if (err) {
    for (int j = lane; j <= Dm; j += 32) ot[j] = -1;
    if (a.out_row_lse)
      for (int s = lane; s < a.slots; s += 32) a.out_row_lse[(size_t)b * a.slots + s] = NAN;
    if (lane == 0) {
      a.out_al[b] = -1;
      if (a.out_flags) a.out_flags[b] = err;
      atomicOr(a.status, err);
      a.rdesc[b].kind = kRaceNone;
    }
    return;
  }

  // test every draft position in parallel
  bool accept = false, near = false;
  if (lane < rp.Db) {
    if (greedy) {
      accept = (x == rows[lane].argmax);
    } else {
      const char* trow = row_base(a, b, lane);
      const char* qrow = row_base(a, b, Dm + 1 + lane);
      const RowRes& rq = rows[Dm + 1 + lane];
      const double lp = (double)load_logit(a, trow, x) / Td - rows[lane].lse;
      double lq = (double)load_logit(a, qrow, x) / Td - rq.lse;
      if (saguaro && lq != -INFINITY) {
        bool in_k = false;
        for (int i = 0; i < rq.ntop; ++i) in_k |= (rq.top[i] == x);
        lq += (in_k ? log(c) : 0.0) - rq.lnZ;
      }
      double acc;
      if (lp == -INFINITY)
        acc = 0.0;  // p(x) = 0: the target never emits x
      else if (lq == -INFINITY)
        acc = 1.0;
      else
        acc = fmin(1.0, exp(lp - lq));
      const double u = (double)(accept_word(a.seed, g, (uint32_t)lane) >> 8) * 0x1p-24;
      accept = u < acc;
      near = fabs(u - acc) < 1e-5;
    }
  }
  const uint32_t rej = __ballot_sync(0xFFFFFFFFu, lane < rp.Db && !accept);
  const int n = rej ? __ffs(rej) - 1 : rp.Db;
  const uint32_t nearm = __ballot_sync(0xFFFFFFFFu, near);
  const uint32_t tested = (n < rp.Db) ? (uint32_t)((2ull << n) - 1ull)
                                      : (uint32_t)((1ull << rp.Db) - 1ull);
  uint32_t flags = (nearm & tested) ? kFlagAcceptNearTie : 0u;

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
    RaceDesc rd;
    rd.kind = greedy ? kRaceNone : (n < rp.Db ? kRaceResidual : kRaceBonus);
    rd.n = n;
    rd.g = g;
    rd.flags = flags;
    rd.T = Td;
    rd.lse_t = rows[n].lse;
    rd.k2 = (float)(1.4426950408889634 / Td);
    rd.l2_t = (float)(rows[n].lse * 1.4426950408889634);
    rd.lse_q = 0.0;
    rd.ln_c = log(c);
    rd.ln_Z = 0.0;
    rd.ntop = 0;
    if (rd.kind == kRaceResidual) {
      const RowRes& rq = rows[Dm + 1 + n];
      rd.lse_q = rq.lse;
      if (saguaro) {
        rd.ln_Z = rq.lnZ;
        rd.ntop = rq.ntop;
        for (int i = 0; i < rq.ntop; ++i) rd.top[i] = rq.top[i];
      }
    }
    a.rdesc[b] = rd;
    a.rcount[b] = 0u;
  }
}

}  // namespace

cudaError_t launch_accept_scan(const VerifyArgs& a, cudaStream_t s) {
  if (a.B == 0) return cudaSuccess;
  const int grid = (a.B + kScanWarps - 1) / kScanWarps;
  accept_scan_kernel<<<grid, 32 * kScanWarps, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace sv
