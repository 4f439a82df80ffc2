// cluster_verify.cu -- the whole verification step in one launch, one thread
// block cluster per request.
//
// A cluster of C CTAs (C = 1 .. 8, chosen by the launcher from the request's
// work) does everything for its request, with the cluster's hardware barrier
// as the only synchronisation -- no grid-wide barrier, no global counter, no
// polling:
//   1. statistics: the cluster's 8C warps take the request's (row, 8 KiB
//      segment) items (stats_device.cuh); the partials go to the workspace
//      and stay in L2;
//   2. merges: the same warps merge one row each (scan_device.cuh);
//   3. accept scan and the race's reference key: CTA 0 (scan_device.cuh,
//      race_device.cuh), which publishes the race description;
//   4. race: the 8C warps stream the sampled row's segments (race_span_in),
//      each writing its best keys;
//   5. CTA 0's first warp combines them and writes the token.
// Each step is separated from the next by a cluster barrier (arrive with
// release, wait with acquire semantics at cluster scope), so what one CTA
// wrote is visible to the cluster's other CTAs after it.
//
// Small batches are launch- and latency-bound: this keeps them to one launch
// with no host-visible dependency, and spreads each request over up to eight
// multiprocessors.  Sources: as the split path ("Accélérer Sonar par la
// Spéculation", "Décodage spéculatif", "Cible-Brouillon"; "Speculative
// Speculative Decoding – асинхронизируй это.", rule items 1-3 and the saguaro
// recipe; "NVIDIA: öt irányelv ...", "Mit csinál a spekulatív dekódolás?").
// The results are those of the split path, bit for bit.
#include <cooperative_groups.h>

#include <cstring>

#include "tail_device.cuh"

namespace cg = cooperative_groups;

namespace sv {

namespace {

// CTA 0 of request b's cluster: the accept scan over the merged rows, then the
// race's reference key; publishes the race description (with the key) to
// a.rdesc[b].  Every thread of the CTA returns at the same point.
template <int DT>
__device__ void cluster_scan(const VerifyArgs& a, int b, const ReqParams& rp, TailShared& S) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == kWarps - 1) S.in[lane] = scan_inputs(a, b, rp);
  // the merged rows, written by the whole cluster: through L2
  const int n16 = a.slots * (int)(sizeof(RowRes) / 16);
  const uint4* src = reinterpret_cast<const uint4*>(a.rowres + (size_t)b * a.slots);
  uint4* dst = reinterpret_cast<uint4*>(S.rows);
  for (int i = threadIdx.x; i < n16; i += kThreads) dst[i] = __ldcg(src + i);
  __syncthreads();
  if (warp == 0) scan_request(a, b, S.rows, &S.rd, S.in[lane]);
  __syncthreads();
  if (S.rd.kind != kRaceNone) {
    const RaceStream R = race_stream(seed_of(a), S.rd.g, (uint32_t)a.vocab_offset >> 2);
    const double kw = race_ref_key_warp<DT>(a, S.rd, R, b, S.rd.ref_seg, warp, kWarps);
    if (lane == 0) S.key[warp] = kw;
    __syncthreads();
    if (threadIdx.x == 0) {
      double K0 = S.key[0];
      for (int w = 1; w < kWarps; ++w) K0 = fmax(K0, S.key[w]);
      S.rd.K0 = K0;
      S.rd.cup = filter_offset(K0, S.rd.lse_t);
    }
    __syncthreads();
  }
  constexpr int d16 = sizeof(RaceDesc) / 16;
  static_assert(sizeof(RaceDesc) % 16 == 0, "RaceDesc is copied in 16-byte pieces");
  if (threadIdx.x < d16)
    reinterpret_cast<uint4*>(a.rdesc + b)[threadIdx.x] = reinterpret_cast<const uint4*>(&S.rd)[threadIdx.x];
}

template <int DT, bool WITH_TOP>
__global__ void __launch_bounds__(kThreads, 2) cluster_kernel(VerifyArgs a) {
  __shared__ TailShared S;
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int r = (int)cluster.block_rank();
  const int b = (int)(blockIdx.x / (unsigned)C);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = r * kWarps + warp, nw = C * kWarps;
  const ReqParams rp = load_req(a, b);

  // 1. the statistics of the request's rows
  const int items = a.slots * a.nseg;
  for (int i = gw; i < items; i += nw) {
    const int slot = i / a.nseg, seg = i - slot * a.nseg;
    if (row_needed(a, b, slot, rp)) stats_item<DT, WITH_TOP>(a, b, slot, seg, rp);
  }
  cluster.sync();

  // 2. one row per warp
  for (int slot = gw; slot < a.slots; slot += nw)
    if (slot_needed(a, b, slot, rp)) merge_row_into(a, b, slot, rp, &a.rowres[(size_t)b * a.slots + slot]);
  cluster.sync();

  // 3. the accept scan and the reference key
  if (r == 0) cluster_scan<DT>(a, b, rp, S);
  cluster.sync();

  // 4. the race over the sampled row, segments gw, gw + nw, ...
  constexpr int d16 = sizeof(RaceDesc) / 16;
  if (threadIdx.x < d16)
    reinterpret_cast<uint4*>(&S.rd)[threadIdx.x] =
        __ldcg(reinterpret_cast<const uint4*>(a.rdesc + b) + threadIdx.x);
  if (threadIdx.x == 0) S.k0 = ordered_u64(-INFINITY);
  __syncthreads();
  const int kind = S.rd.kind;
  if (kind != kRaceNone) {
    const bool residual = kind == kRaceResidual;
    const char* trow = row_base(a, b, S.rd.n);
    const char* qrow = residual ? row_base(a, b, a.D_max + 1 + S.rd.n) : nullptr;
    const RaceStream R = race_stream(seed_of(a), S.rd.g, (uint32_t)a.vocab_offset >> 2);
    const Best B = race_span_in<DT>(a, S.rd, R, trow, qrow, residual, gw, nw, S.rd.K0, &S.k0);
    if (lane == 0) {
      RacePart p;
      p.best = B.best;
      p.second = B.second;
      p.idx = B.idx;
      p.pad = 0;
      a.rpart[(size_t)b * kClusterParts + gw] = p;
    }
  }
  cluster.sync();

  // 5. combine and write the token
  if (kind != kRaceNone && r == 0 && warp == 0) {
    Best c{-INFINITY, -INFINITY, -1};
    for (int s = lane; s < nw; s += 32) {
      const RacePart* pp = a.rpart + (size_t)b * kClusterParts + s;
      Best o;
      o.best = __ldcg(&pp->best);
      o.second = __ldcg(&pp->second);
      o.idx = __ldcg(&pp->idx);
      c = combine(c, o);
    }
    finish_race<DT>(a, b, S.rd, warp_combine(c));
  }
}

template <int DT, bool WITH_TOP>
cudaError_t launch_cl(const VerifyArgs& a, cudaStream_t s, int C) {
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3((unsigned)a.B * (unsigned)C);
  cfg.blockDim = dim3(kThreads);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, cluster_kernel<DT, WITH_TOP>, a);
}

}  // namespace

// CTAs per request: enough warps for about one statistics item each, at most 8.
int cluster_size(const VerifyArgs& a) {
  const long long items = (long long)a.slots * a.nseg;
  long long c = (items + kWarps - 1) / kWarps;
  if (c < 1) c = 1;
  if (c > kClusterMax) c = kClusterMax;
  return (int)c;
}

cudaError_t launch_cluster(const VerifyArgs& a, cudaStream_t s) {
  if (a.B == 0) return cudaSuccess;
  const int C = cluster_size(a);
  const bool top = a.mode == kSaguaro || a.mode_per_req != nullptr;
  if (a.dtype == kF32) return top ? launch_cl<kF32, true>(a, s, C) : launch_cl<kF32, false>(a, s, C);
  return top ? launch_cl<kBF16, true>(a, s, C) : launch_cl<kBF16, false>(a, s, C);
}

}  // namespace sv
