// shard_verify.cu -- verification with the vocabulary split across devices
// (tensor-parallel logits: each rank holds columns [r V_s, (r + 1) V_s) of every
// target and draft row).
//
// "Accélérer Sonar par la Spéculation", section "Calendrier Brouillon-Cible":
// the verification batch is formed for the target and synchronised with the
// parallel workers; the sampler then works on logits that, in a
// tensor-parallel target, are split by vocabulary.  Each rank does the work
// on its own columns; two small exchanges (the caller's all-gathers, over
// NCCL / NVLink) carry what the other ranks need:
//   stage 1 (sv_shard_stats): the statistics pass over the rank's columns --
//     per 8 KiB segment the partial (max, sum, argmax as a global index) and,
//     for saguaro draft rows, the top list -- and the target and draft logits
//     of the draft tokens this rank owns.  Exchange 1 = these, per rank.
//   stage 2 (sv_shard_race): every rank merges every rank's partials in global
//     order (rank-major, so the merge sees the row's segments in order), runs
//     the same accept scan (so each writes the same accepted lengths and
//     prefixes), and races its own columns with the Philox words of their
//     global indices; if its columns hold no residual candidate it also races
//     them for the bonus (so that an empty residual, which is global exactly
//     when every rank's part is empty, needs no third exchange).  Exchange 2 =
//     one record per request.
//   stage 3 (sv_shard_finish): the records of all ranks are combined (the best
//     key, ties to the lowest global index) and the token is written.
// The decisions are the rule's; the statistics differ from an unsharded call
// only in how the row is cut into segments, i.e. in rounding.
#include <cstring>

#include "tail_device.cuh"

namespace sv {

namespace {

// Stage 1's owned draft-token logits: lane d < D_b of request b (one warp).
__global__ void __launch_bounds__(kThreads) shard_z_kernel(VerifyArgs a, float2* zx) {
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (b >= a.B) return;
  const ReqParams rp = load_req(a, b);
  for (int d = lane; d < a.D_max; d += 32) {
    float2 z = make_float2(0.0f, 0.0f);
    if (!rp.err && d < rp.Db && rp.mode != kGreedy) {
      const int x = a.tokens[(size_t)b * a.D_max + d] - a.vocab_offset;
      if (x >= 0 && x < a.V) {
        z.x = load_logit(a, row_base(a, b, d), x);
        z.y = load_logit(a, row_base(a, b, a.D_max + 1 + d), x);
      }
    }
    zx[(size_t)b * a.D_max + d] = z;
  }
}

// The scan's inputs from the gathered exchange: the owner of token x is rank
// x / V (every rank holds V columns).
__device__ __forceinline__ ScanInputs shard_scan_inputs(const VerifyArgs& a, int b,
                                                        const ReqParams& rp, const char* x1,
                                                        size_t x1_bytes, size_t zx_off) {
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
      const int owner = in.x / a.V;
      const float2 z = __ldcg(reinterpret_cast<const float2*>(x1 + owner * x1_bytes + zx_off) +
                              (size_t)b * a.D_max + lane);
      in.zt = z.x;
      in.zq = z.y;
      in.uw = accept_word(seed_of(a), a.request_offset + (uint32_t)b, (uint32_t)lane);
    }
  }
  return in;
}

// Stage 2: request b, by the whole CTA.  x1: the gathered exchange 1 (n_shards
// consecutive copies of x1_bytes); rec: this rank's exchange 2.
template <int DT>
__global__ void __launch_bounds__(kThreads, 2) shard_tail_kernel(VerifyArgs a, const char* x1,
                                                                 size_t x1_bytes, size_t top_off,
                                                                 size_t zx_off, int n_shards,
                                                                 ShardRace* rec) {
  __shared__ TailShared S;
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const ReqParams rp = load_req(a, b);
  if (warp == kWarps - 1) S.in[lane] = shard_scan_inputs(a, b, rp, x1, x1_bytes, zx_off);
  // every rank's partials, rank-major: segment s of the row is rank s / nseg's
  // local segment s % nseg
  const int nseg = a.nseg, Dm = a.D_max;
  for (int slot = warp; slot < a.slots; slot += kWarps) {
    if (!slot_needed(a, b, slot, rp)) continue;
    const bool is_t = slot <= Dm;
    const int d = is_t ? slot : slot - Dm - 1;
    const bool top = !is_t && rp.mode == kSaguaro;
    const size_t prow = ((size_t)b * a.slots + slot) * nseg;
    const size_t trow = ((size_t)b * Dm + d) * nseg;
    merge_into_at(
        a, rp, slot,
        [=](int s) {
          return reinterpret_cast<const PartStat*>(x1 + (size_t)(s / nseg) * x1_bytes) + prow +
                 s % nseg;
        },
        [=](int s) {
          return reinterpret_cast<const TopPart*>(x1 + (size_t)(s / nseg) * x1_bytes + top_off) +
                 trow + s % nseg;
        },
        top, nseg * n_shards, &S.rows[slot]);
  }
  __syncthreads();
  if (warp == 0) scan_request(a, b, S.rows, &S.rd, S.in[lane]);
  __syncthreads();
  const int kind = S.rd.kind;
  Best rb{-INFINITY, -INFINITY, -1}, bb{-INFINITY, -INFINITY, -1};
  if (kind != kRaceNone) {
    const bool residual = kind == kRaceResidual;
    const char* trowp = row_base(a, b, S.rd.n);
    const char* qrowp = residual ? row_base(a, b, Dm + 1 + S.rd.n) : nullptr;
    const RaceStream R = race_stream(seed_of(a), S.rd.g, (uint32_t)a.vocab_offset >> 2);
    for (int pass = 0; pass < 2; ++pass) {
      // pass 0: the race of kind; pass 1: the bonus race, when no column here
      // is a residual candidate
      const bool res = residual && pass == 0;
      if (threadIdx.x == 0) S.k0 = ordered_u64(-INFINITY);
      __syncthreads();
      const Best Bw = race_span_in<DT>(a, S.rd, R, trowp, res ? qrowp : nullptr, res, warp,
                                       kWarps, -INFINITY, &S.k0);
      if (lane == 0) {
        S.best[warp] = Bw.best;
        S.second[warp] = Bw.second;
        S.idx[warp] = Bw.idx;
      }
      __syncthreads();
      Best c{-INFINITY, -INFINITY, -1};
      if (lane < kWarps) {
        c.best = S.best[lane];
        c.second = S.second[lane];
        c.idx = S.idx[lane];
      }
      c = warp_combine(c);
      if (c.idx >= 0) c.idx += a.vocab_offset;  // global index
      if (pass == 0) rb = c; else bb = c;
      __syncthreads();  // S.best is reused
      if (!residual || rb.idx >= 0) break;
    }
  }
  if (threadIdx.x == 0) {
    ShardRace r;
    r.best = rb.best;
    r.second = rb.second;
    r.idx = rb.idx;
    r.bbest = bb.best;
    r.bsecond = bb.second;
    r.bidx = bb.idx;
    r.kind = kind;
    r.n = S.rd.n;
    r.flags = S.rd.flags;
    r.pad = 0;
    rec[b] = r;
  }
}

// Stage 3: request b by one warp over the gathered records (n_shards x B).
__global__ void __launch_bounds__(kThreads) shard_finish_kernel(const ShardRace* recs, int B,
                                                                int D_max, int n_shards,
                                                                int32_t* out_tokens,
                                                                uint32_t* out_flags,
                                                                unsigned* status) {
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (b >= B) return;
  const ShardRace& r0 = recs[b];
  const int kind = r0.kind;
  if (kind == kRaceNone) return;
  Best c{-INFINITY, -INFINITY, -1}, e{-INFINITY, -INFINITY, -1};
  for (int r = lane; r < n_shards; r += 32) {
    const ShardRace& x = recs[(size_t)r * B + b];
    c = combine(c, Best{x.best, x.second, x.idx});
    e = combine(e, Best{x.bbest, x.bsecond, x.bidx});
  }
  c = warp_combine(c);
  e = warp_combine(e);
  uint32_t flags = r0.flags;
  if (c.idx < 0 && kind == kRaceResidual) {
    // {p > q} empty on every rank (only through rounding): the bonus race on p
    flags |= kFlagResidualEmpty;
    c = e;
  }
  if (lane == 0) {
    if (c.best - c.second < 1e-6) flags |= kFlagRaceNearTie;
    out_tokens[(size_t)b * (D_max + 1) + r0.n] = c.idx;
    if (out_flags) out_flags[b] = flags;
    if (flags & kFlagResidualEmpty) atomicOr(status, kFlagResidualEmpty);
  }
}

}  // namespace

ShardLayout shard_layout(int B, int D_max, int V_local, int dtype) {
  int nvec, nseg;
  row_geometry(V_local, dtype, &nvec, &nseg);
  const size_t slots = 2 * (size_t)D_max + 1;
  ShardLayout L;
  size_t off = 0;
  L.parts = off;
  off = align_up(off + (size_t)B * slots * nseg * sizeof(PartStat), 256);
  L.tops = off;
  off = align_up(off + (size_t)B * D_max * nseg * sizeof(TopPart), 256);
  L.zx = off;
  off = align_up(off + (size_t)B * D_max * sizeof(float2), 256);
  L.x1 = off;
  L.x2 = (size_t)B * sizeof(ShardRace);  // records of consecutive ranks are consecutive
  return L;
}

cudaError_t launch_shard_z(const VerifyArgs& a, void* zx, cudaStream_t s) {
  if (a.B == 0 || a.D_max == 0) return cudaSuccess;
  shard_z_kernel<<<(a.B + kWarps - 1) / kWarps, kThreads, 0, s>>>(a, (float2*)zx);
  return cudaGetLastError();
}

cudaError_t launch_shard_tail(const VerifyArgs& a, const void* gathered1, int n_shards,
                              void* exchange2, cudaStream_t s) {
  if (a.B == 0) return cudaSuccess;
  const ShardLayout L = shard_layout(a.B, a.D_max, a.V, a.dtype);
  const char* x1 = (const char*)gathered1;
  ShardRace* rec = (ShardRace*)exchange2;
  if (a.dtype == kF32)
    shard_tail_kernel<kF32><<<a.B, kThreads, 0, s>>>(a, x1, L.x1, L.tops, L.zx, n_shards, rec);
  else
    shard_tail_kernel<kBF16><<<a.B, kThreads, 0, s>>>(a, x1, L.x1, L.tops, L.zx, n_shards, rec);
  return cudaGetLastError();
}

cudaError_t launch_shard_finish(const void* gathered2, int B, int D_max, int n_shards,
                                int32_t* out_tokens, uint32_t* out_flags, unsigned* status,
                                cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  shard_finish_kernel<<<(B + kWarps - 1) / kWarps, kThreads, 0, s>>>(
      (const ShardRace*)gathered2, B, D_max, n_shards, out_tokens, out_flags, status);
  return cudaGetLastError();
}

}  // namespace sv
