// tree_verify.cu -- tree (multi-candidate) verification after the statistics
// pass: one thread-block cluster per request walks its draft tree from the root.
//
// "Accélérer Sonar par la Spéculation", section "EAGLE": the draft proposes a
// tree whose nodes hold several candidate tokens.  At position p (the root, or
// an accepted node) the candidates hanging under p are tried in node order
// with the rule of "Speculative Speculative Decoding – асинхронизируй это."
// (items 1-3) applied recursively: candidate j is accepted with probability
// min(1, P_j(x) / q(x)); a rejection replaces P_j by norm(max(0, P_j - q)); after
// the last candidate the token is drawn from that residual, and at a position
// with no candidate the bonus token is drawn from p.  With P_0 = p,
//   P_j = max(0, p - c_j q) / N_j,  c_0 = 0, N_0 = 1,
//   c_{j+1} = c_j + N_j,  N_{j+1} = sum_x max(0, p(x) - c_{j+1} q(x)),
// so each rejection that is followed by another candidate costs one pass over
// the position's target and draft rows (the sum N, by the whole CTA, in a fixed
// order), and the final draw is the residual race with q scaled by c_K -- the
// linear path's race with the draft row's log-normaliser lowered by ln c_K.
//
// The C CTAs of a request's cluster (C = 1, 2 or 4) all merge the rows and take
// the same decisions from the same numbers; each residual pass and the race
// are split over all of them: a pass's partial sums are exchanged through
// distributed shared memory and added in rank order (so every CTA holds the
// same N), and rank 0 combines the race results and writes the outputs.
// The accept uniform of candidate node i is word 0 of Philox at counter
// (i, g, 0, 0), so a chain (one candidate per position) is the linear rule
// exactly.  Greedy: the first candidate holding the target row's argmax is
// accepted; otherwise that argmax is emitted.
#include <cooperative_groups.h>

#include <cstring>

#include "specverify.h"
#include "tail_device.cuh"

namespace cg = cooperative_groups;

namespace sv {

namespace {

struct TreeShared {
  int path[kMaxDraft];
  int len, pos, done, emit_kind;  // emit_kind: kRaceNone (a token is known), kRaceBonus, kRaceResidual
  int emitted;
  uint32_t flags;
  double c, N, c_prev;
  double red[kWarps];
  double part[2];  // this CTA's partial of the residual pass, by pass parity
  Best rb;         // this CTA's race result
  // node i's token logits in its parent position's target and draft rows, and
  // its accept word (loaded before the walk, so that its decisions wait on no
  // memory)
  float zt[kMaxDraft], zq[kMaxDraft];
  uint32_t uw[kMaxDraft];
};

// sum over the row of max(0, p(x) - c q(x)) for target row pos and draft row
// pos of request b, by the whole cluster in a fixed order: thread t of rank r
// takes the 16-byte vectors r kThreads + t + i C kThreads of both rows, four of
// each in flight at once, sums each vector's terms in single precision and
// adds that to its double accumulator; then the warps, the CTA (in double),
// and the ranks in order through distributed shared memory.  Every thread of
// the cluster returns the same value; `parity` alternates between calls.
template <int DT>
__device__ double residual_mass(const VerifyArgs& a, int b, int pos, double lse_t, double lse_q,
                                float k2, double c, TreeShared& T, cg::cluster_group& cluster,
                                int parity) {
  const int C = (int)cluster.num_blocks(), r = (int)cluster.block_rank();
  constexpr int VEC = DT == kF32 ? 4 : 8;
  constexpr int U = 4;
  const char* trow = row_base(a, b, pos);
  const char* qrow = row_base(a, b, a.D_max + 1 + pos);
  const float lt = (float)(lse_t * 1.4426950408889634), lq = (float)(lse_q * 1.4426950408889634);
  const float cf = (float)c;
  const int nfull = a.V / VEC;
  const bool aligned = ((uintptr_t)trow & 15u) == 0 && ((uintptr_t)qrow & 15u) == 0;
  const int stride = C * kThreads;
  double acc = 0.0;
  for (int v0 = r * kThreads + threadIdx.x; v0 < a.nvec; v0 += U * stride) {
    uint4 wt[U], wq[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      // past the row's end: -inf, whose terms are 0
      wt[u] = load_vec_checked<DT>(trow, v0 + u * stride, a.V, a.nvec, nfull, aligned);
      wq[u] = load_vec_checked<DT>(qrow, v0 + u * stride, a.V, a.nvec, nfull, aligned);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float sv = 0.0f;
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        const float p = ex2_approx(fmaf(elem<DT>(wt[u], e), k2, -lt));
        const float q = ex2_approx(fmaf(elem<DT>(wq[u], e), k2, -lq));
        sv += fmaxf(0.0f, fmaf(-cf, q, p));
      }
      acc += (double)sv;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
  if ((threadIdx.x & 31) == 0) T.red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int w = 0; w < kWarps; ++w) s += T.red[w];
    T.part[parity] = s;
  }
  // (a pass's slot is written again two passes later, after every rank has
  // read it: each rank reads before it reaches the next pass's barrier)
  cluster.sync();
  double N = 0.0;
  for (int k = 0; k < C; ++k) N += *cluster.map_shared_rank(&T.part[parity], k);
  return N;
}

template <int DT>
__global__ void __launch_bounds__(kThreads, 2) tree_kernel(VerifyArgs a) {
  __shared__ TailShared S;
  __shared__ TreeShared T;
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks(), rank = (int)cluster.block_rank();
  wait_for_previous_kernel();
  const int b = (int)(blockIdx.x / (unsigned)C);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Dm = a.D_max;
  const ReqParams rp = load_req(a, b);
  const uint32_t g = a.request_offset + (uint32_t)b;
  const int32_t* tok = a.tokens + (size_t)b * Dm;
  const int32_t* par = a.parents + (size_t)b * Dm;
  int32_t* ot = a.out_tokens + (size_t)b * (Dm + 1);

  if (warp == kWarps - 1) {
    // errors: parameters, nodes (token range, parent order), unreadable rows;
    // and the nodes' inputs, while the other warps merge the rows
    uint32_t err = rp.err | (rp.mode == kSaguaro ? kFlagBadParam : 0u);
    if (!rp.err)
      for (int i = lane; i < rp.Db; i += 32) {
        const int x = __ldg(&tok[i]), pi = __ldg(&par[i]);
        if (x < 0 || x >= a.V_global) err |= kFlagBadToken;
        if (pi < 0 || pi > i) err |= kFlagBadParam;
        if (x >= 0 && x < a.V && pi >= 0 && pi <= i && rp.mode != kGreedy) {
          T.zt[i] = logit_at<DT>(row_base(a, b, pi), x);
          T.zq[i] = logit_at<DT>(row_base(a, b, Dm + 1 + pi), x);
          T.uw[i] = accept_word(seed_of(a), g, (uint32_t)i);
        }
      }
    err = __reduce_or_sync(0xFFFFFFFFu, err);
    if (lane == 0) {
      T.flags = err;
      T.len = 0;
      T.pos = 0;
      T.done = 0;
    }
  }
  for (int slot = warp; slot < a.slots; slot += kWarps)
    if (slot_needed(a, b, slot, rp)) merge_row_into(a, b, slot, rp, &S.rows[slot]);
  __syncthreads();
  if (!T.flags) {
    // rows the walk may read that hold NaN, +inf or no finite entry
    uint32_t bad = 0;
    for (int slot = threadIdx.x; slot < a.slots; slot += kThreads)
      if (slot_needed(a, b, slot, rp) && S.rows[slot].bad) bad = kFlagNonfinite;
    bad = __syncthreads_or(bad) ? kFlagNonfinite : 0u;
    if (threadIdx.x == 0) T.flags |= bad;
    __syncthreads();
  }
  if (a.out_row_lse && rank == 0) {
    // natural-log LSE of every row the walk may read (stochastic requests), NaN elsewhere
    const bool ok = !(T.flags & kFlagErrors) && rp.mode != kGreedy;
    for (int s = threadIdx.x; s < a.slots; s += kThreads)
      a.out_row_lse[(size_t)b * a.slots + s] =
          ok && slot_needed(a, b, s, rp) ? (float)S.rows[s].lse : NAN;
  }
  if (T.flags & kFlagErrors) {
    // (every rank of the cluster returns here: the flags come from the same numbers)
    if (rank != 0) return;
    for (int j = threadIdx.x; j <= Dm; j += kThreads) ot[j] = -1;
    if (a.out_nodes)
      for (int j = threadIdx.x; j < Dm; j += kThreads) a.out_nodes[(size_t)b * Dm + j] = -1;
    if (threadIdx.x == 0) {
      a.out_al[b] = -1;
      if (a.out_flags) a.out_flags[b] = T.flags;
      atomicOr(a.status, T.flags);
    }
    return;
  }

  const bool greedy = rp.mode == kGreedy;
  const double Td = (double)rp.T;
  const float k2 = greedy ? 0.0f : log2e_over_T(rp.T);
  int passes = 0;
  for (;;) {
    const int pos = T.pos;
    if (greedy) {
      if (threadIdx.x == 0) {
        const int am = S.rows[pos].argmax;
        int found = -1;
        for (int i = 0; i < rp.Db && found < 0; ++i)
          if (__ldg(&par[i]) == pos && __ldg(&tok[i]) == am) found = i;
        if (found >= 0) {
          T.path[T.len++] = found;
          T.pos = found + 1;
        } else {
          T.emitted = am;
          T.emit_kind = kRaceNone;
          T.done = 1;
        }
      }
      __syncthreads();
      if (T.done) break;
      continue;
    }
    // stochastic: the candidates under pos, in node order
    const double lse_t = S.rows[pos].lse;
    const double lse_q = pos < Dm ? S.rows[Dm + 1 + pos].lse : 0.0;  // read only with candidates
    if (threadIdx.x == 0) {
      T.c = 0.0;
      T.N = 1.0;
    }
    __syncthreads();
    int accepted = -1, any = 0;
    for (int i = 0; i < rp.Db; ++i) {
      if (__ldg(&par[i]) != pos) continue;
      if (any) {
        // the previous candidate was rejected: the residual for this one
        const double cn = T.c + T.N;
        const double Nn = residual_mass<DT>(a, b, pos, lse_t, lse_q, k2, cn, T, cluster, passes & 1);
        ++passes;
        if (threadIdx.x == 0) {
          if (Nn > 0.0) {
            T.c = cn;
            T.N = Nn;
          } else {
            T.flags |= kFlagResidualEmpty;  // only through rounding: keep the last residual
          }
        }
        __syncthreads();
      }
      any = 1;
      if (threadIdx.x == 0) {
        const double lp = (double)T.zt[i] / Td - lse_t;
        const double lq = (double)T.zq[i] / Td - lse_q;
        double acc;
        if (T.c == 0.0) {
          // P = p: the linear rule's ratio
          if (lp == -INFINITY)
            acc = 0.0;
          else if (lq == -INFINITY)
            acc = 1.0;
          else
            acc = fmin(1.0, exp(lp - lq));
        } else {
          const double r = exp(lp) - T.c * exp(lq);
          if (!(r > 0.0))
            acc = 0.0;
          else if (lq == -INFINITY)
            acc = 1.0;
          else
            acc = fmin(1.0, r / (T.N * exp(lq)));
        }
        const uint32_t uw = T.uw[i];
        const double u = (double)(uw >> 8) * 0x1p-24;
        if (fabs(u - acc) < 1e-5) T.flags |= kFlagAcceptNearTie;
        T.emitted = u < acc ? i : -1;
      }
      __syncthreads();
      accepted = T.emitted;
      __syncthreads();
      if (accepted >= 0) break;
    }
    if (accepted >= 0) {
      if (threadIdx.x == 0) {
        T.path[T.len++] = accepted;
        T.pos = accepted + 1;
      }
      __syncthreads();
      continue;
    }
    // every candidate rejected (or none): the race on position pos
    if (threadIdx.x == 0) {
      T.emit_kind = any ? kRaceResidual : kRaceBonus;
      T.c_prev = T.c;
      if (any) T.c += T.N;  // the residual after the last rejection
    }
    __syncthreads();
    break;
  }

  const int len = T.len;
  int emitted = T.emitted;
  if (T.emit_kind != kRaceNone) {
    // the race: as the linear path's, with the draft's log-normaliser lowered
    // by ln c so that the residual is max(0, p - c q)
    const int pos = T.pos;
    const bool residual = T.emit_kind == kRaceResidual;
    if (threadIdx.x == 0) {
      RaceDesc& rd = S.rd;
      rd.kind = T.emit_kind;
      rd.n = pos;
      rd.g = g;
      rd.flags = T.flags;
      rd.T = Td;
      rd.lse_t = S.rows[pos].lse;
      rd.lse_q = residual ? S.rows[Dm + 1 + pos].lse - log(T.c) : 0.0;
      rd.ln_c = 0.0;
      rd.ln_Z = 0.0;
      rd.K0 = -INFINITY;
      rd.k2 = k2;
      rd.cup = INFINITY;
      rd.ntop = 0;
      rd.ref_seg = S.rows[pos].mseg;
      S.k0 = ordered_u64(-INFINITY);
    }
    __syncthreads();
    const RaceStream R = race_stream(seed_of(a), g, (uint32_t)a.vocab_offset >> 2);
    const double kw = race_ref_key_warp<DT>(a, S.rd, R, b, S.rd.ref_seg, warp, kWarps);
    if (lane == 0) S.key[warp] = kw;
    __syncthreads();
    double K0 = S.key[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) K0 = fmax(K0, S.key[w]);
    const char* trow = row_base(a, b, pos);
    const char* qrow = residual ? row_base(a, b, Dm + 1 + pos) : nullptr;
    // the cluster's C * kWarps warps race the row's segments
    const Best Bw = race_span_in<DT>(a, S.rd, R, trow, qrow, residual, rank * kWarps + warp,
                                     C * kWarps, K0, &S.k0);
    if (lane == 0) {
      S.best[warp] = Bw.best;
      S.second[warp] = Bw.second;
      S.idx[warp] = Bw.idx;
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
      if (lane == 0) T.rb = r;
    }
    cluster.sync();
    if (rank == 0 && warp == 0) {
      // the ranks' results, in rank order
      Best r{-INFINITY, -INFINITY, -1};
      if (lane < C) r = *cluster.map_shared_rank(&T.rb, lane);
      r = warp_combine(r);
      uint32_t flags = T.flags;
      if (r.idx < 0 && residual) {
        // {p > c q} empty (only through rounding): the residual before the last
        // rejection is kept, as when an earlier residual comes out empty -- with
        // c = 0 that is the bonus race on p
        flags |= kFlagResidualEmpty;
        const bool keep = T.c_prev > 0.0;
        if (lane == 0) S.rd.lse_q = keep ? S.rows[Dm + 1 + pos].lse - log(T.c_prev) : 0.0;
        __syncwarp();
        Best Bb{-INFINITY, -INFINITY, -1};
        for (int s = 0; s < a.nseg; ++s)
          Bb = combine(Bb, race_segment<DT>(row_ctx(a), S.rd, trow, keep ? qrow : nullptr, keep, s,
                                            -INFINITY, INFINITY));
        r = Bb;
      }
      if (r.best - r.second < 1e-6) flags |= kFlagRaceNearTie;
      if (lane == 0) {
        T.emitted = r.idx;
        T.flags = flags;
      }
    }
    // the other ranks' shared memory stays until rank 0 has read it
    cluster.sync();
    emitted = T.emitted;
  }
  if (rank != 0) return;
  // outputs: the accepted path's tokens, then the drawn or argmax token
  for (int j = threadIdx.x; j <= Dm; j += kThreads)
    ot[j] = j < len ? __ldg(&tok[T.path[j]]) : (j == len ? emitted : -1);
  if (a.out_nodes)
    for (int j = threadIdx.x; j < Dm; j += kThreads)
      a.out_nodes[(size_t)b * Dm + j] = j < len ? T.path[j] : -1;
  if (threadIdx.x == 0) {
    a.out_al[b] = len + 1;
    if (a.out_flags) a.out_flags[b] = T.flags;
    if (T.flags & kFlagResidualEmpty) atomicOr(a.status, kFlagResidualEmpty);
  }
}

}  // namespace

cudaError_t launch_tree(const VerifyArgs& a, cudaStream_t s, int sms) {
  if (a.B == 0) return cudaSuccess;
  int C = 4;
  while (C > 1 && (long long)a.B * C > 2LL * sms) C /= 2;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3((unsigned)a.B * (unsigned)C);
  cfg.blockDim = dim3(kThreads);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)C;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return a.dtype == kF32 ? cudaLaunchKernelEx(&cfg, tree_kernel<kF32>, a)
                         : cudaLaunchKernelEx(&cfg, tree_kernel<kBF16>, a);
}

}  // namespace sv
