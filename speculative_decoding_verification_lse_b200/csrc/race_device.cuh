// race_device.cuh -- device code of the residual / bonus race, shared by the
// split race kernel and the fused kernel.
//
// After a rejection at position n the token is drawn from norm(max(0, p - q))
// ("Speculative Speculative Decoding – асинхронизируй это.", rule item 3);
// when every draft was accepted it is drawn from p at position D_b, the extra
// token the target gives for free ("Accélérer Sonar par la Spéculation",
// section "Décodage spéculatif").  Both draws are exponential races: the token
// is the argmax over candidates x of r(x) / E_x with E_x unit exponentials from
// Philox keyed by (seed, request, token), which picks x with probability
// r(x) / sum r and does not depend on the order of any sum.
//
// Exactness.  The decision is taken on the exact key ln r(x) - ln E_x in double
// precision, with the same formulas as the plain definition, but only for the
// few tokens that can win.  One warp handles an 8 KiB segment of the row:
//   A. every lane computes, for each of its tokens, a single-precision UPPER
//      BOUND of the key in log2 units (ex2/lg2 based, with explicit slack for
//      every rounding and approximation error; race_bounds) and keeps its two
//      largest;
//   B. each lane evaluates the exact key of its best token; S1 = warp maximum;
//   C. a lane whose second bound reaches S1 (less a margin that also covers
//      the 1e-6 near-tie band) evaluates that token too, and if its second
//      bound reached S1 its third might have as well, so it re-scans its tokens
//      and evaluates every one whose bound reaches S1.
// No token whose exact key is within the band of the segment's best is ever
// skipped, so the segment's best and runner-up are those of the exact keys.
//
// Layout: one warp per (request, segment); the warp that completes the last
// segment of a request (atomic counter, no waiting) merges the segment results
// and writes the token.  The counter starts at zero: the split path's scan
// clears it, the fused path clears it before the launch.
#pragma once
#include "philox.cuh"
#include "stats_device.cuh"
#include "sv_common.cuh"

#include <float.h>
#include <limits.h>
#include <math.h>

namespace sv {

struct Best {
  double best;
  double second;
  int idx;
};

__device__ __forceinline__ void offer(Best& B, double key, int x) {
  if (key == -INFINITY) return;
  if (B.idx < 0 || key > B.best || (key == B.best && x < B.idx)) {
    B.second = B.best;
    B.best = key;
    B.idx = x;
  } else if (key > B.second) {
    B.second = key;
  }
}

__device__ __forceinline__ Best combine(const Best& A, const Best& C) {
  const bool c_wins =
      C.idx >= 0 && (A.idx < 0 || C.best > A.best || (C.best == A.best && C.idx < A.idx));
  const Best& w = c_wins ? C : A;
  const Best& l = c_wins ? A : C;
  Best r;
  r.best = w.best;
  r.idx = w.idx;
  r.second = fmax(w.second, l.best);
  return r;
}

__device__ __forceinline__ Best warp_combine(Best v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    Best w;
    w.best = __shfl_xor_sync(0xFFFFFFFFu, v.best, o);
    w.second = __shfl_xor_sync(0xFFFFFFFFu, v.second, o);
    w.idx = __shfl_xor_sync(0xFFFFFFFFu, v.idx, o);
    v = combine(v, w);
  }
  return v;
}

// A lower bound of E = -ln(1 - W), W = (o + 1/2) 2^-32, within 2^-12 of it, for
// two words at once.
//   W < 2^-10 (o < 2^22): E >= W, and W is exact from the low 22 bits of o.
//   otherwise: U = 1 - W <= Uup = 1 - (o >> 9) 2^-23 (exact in single precision),
//   so E >= -ln Uup >= ln2 (-lg2(Uup) - 2^-16) (lg2's error, taken as at most
//   2^-22 (1 + |result|), is below 2^-16 for Uup in [2^-23, 1 - 2^-10]).
__device__ __forceinline__ float2 E_lower2(uint32_t o0, uint32_t o1) {
  const float2 fa = __fadd2_rn(make_float2(__uint_as_float(0x4B000000u | (o0 & 0x3FFFFFu)),
                                           __uint_as_float(0x4B000000u | (o1 & 0x3FFFFFu))),
                               make_float2(-8388608.0f, -8388608.0f));
  const float2 Ws = __ffma2_rn(fa, make_float2(0x1p-32f, 0x1p-32f), make_float2(0x1p-33f, 0x1p-33f));
  const float2 fb = __fadd2_rn(make_float2(__uint_as_float(0x4B000000u | (o0 >> 9)),
                                           __uint_as_float(0x4B000000u | (o1 >> 9))),
                               make_float2(-8388608.0f, -8388608.0f));
  const float2 Uup = __ffma2_rn(fb, make_float2(-0x1p-23f, -0x1p-23f), make_float2(1.0f, 1.0f));
  const float2 El = __ffma2_rn(make_float2(lg2_approx(Uup.x), lg2_approx(Uup.y)),
                               make_float2(-0.693147180559945f, -0.693147180559945f),
                               make_float2(-0.693147180559945f * 0x1p-16f, -0.693147180559945f * 0x1p-16f));
  return make_float2(o0 < 0x400000u ? Ws.x : El.x, o1 < 0x400000u ? Ws.y : El.y);
}

// The exact key ln r(x) - ln E_x in double precision, the plain definition's
// formulas; -inf if x is no candidate.
static __device__ __noinline__ double exact_key(float zt, float zq, int x, uint32_t o,
                                         const RaceDesc& rd, bool residual) {
  const double lp = (double)zt / rd.T - rd.lse_t;
  if (lp == -INFINITY) return -INFINITY;
  double lr = lp;
  if (residual) {
    double lq = (double)zq / rd.T - rd.lse_q;
    if (rd.ntop > 0 && lq != -INFINITY) {
      bool in_k = false;
      for (int i = 0; i < rd.ntop; ++i) in_k |= (rd.top[i] == x);
      lq += (in_k ? rd.ln_c : 0.0) - rd.ln_Z;
    }
    if (!(lp > lq)) return -INFINITY;
    if (lq != -INFINITY) lr = lp + log(-expm1(lq - lp));
  }
  const double W = ((double)o + 0.5) * 0x1p-32;
  return lr - log(-log1p(-W));
}

template <int DT>
__device__ __forceinline__ float logit_at(const char* row, int x) {
  if (DT == kF32) return ((const float*)row)[x];
  return __uint_as_float((uint32_t)((const uint16_t*)row)[x] << 16);
}

// The race word of token x.
__device__ __forceinline__ uint32_t race_word(uint64_t seed, uint32_t g, int x) {
  const uint4 w = race_words(seed, g, (uint32_t)x >> 2);
  const int l = x & 3;
  return l == 0 ? w.x : l == 1 ? w.y : l == 2 ? w.z : w.w;
}

__device__ __forceinline__ double exact_key_of(const VerifyArgs& a, const RaceDesc& rd,
                                               const char* trow, const char* qrow,
                                               bool residual, int x) {
  const float zt = (a.dtype == kF32) ? logit_at<kF32>(trow, x) : logit_at<kBF16>(trow, x);
  float zq = 0.0f;
  if (residual) zq = (a.dtype == kF32) ? logit_at<kF32>(qrow, x) : logit_at<kBF16>(qrow, x);
  return exact_key(zt, zq, x, race_word(a.seed, rd.g, x), rd, residual);
}

// Upper bounds of the keys (log2 units) of one lane's tokens in segment `seg`;
// calls visit(bound, x) for each.  Every rounding and approximation error is
// covered by explicit slack:
//   l2p = z*k2 - l2_t is within (|z| k2 + |l2_t|) 2^-22 of log2 p(x);
//   log2 E >= lg2(E_lower) - 2^-16;
//   residual, x outside K: d = log2 q'(x) - log2 p(x) >= dlo, and
//     log2(1 - 2^d) <= lg2(1 - ex2(dlo)(1 - 2^-21)) + 2^-16;
//   residual, x possibly in K (draft logit >= the smallest logit of K): r <= p.
// Pairs of tokens share packed fp32x2 arithmetic.
template <int DT, typename Visit>
__device__ __forceinline__ void race_bounds(const VerifyArgs& a, const RaceDesc& rd,
                                            const RaceStream& R, const char* trow,
                                            const char* qrow, bool residual, int seg,
                                            Visit&& visit) {
  constexpr int VEC = DT == kF32 ? 4 : 8;
  const int lane = threadIdx.x & 31;
  const float k2 = rd.k2;
  const float l2t = rd.l2_t, l2q = rd.l2_q, kmin = rd.kmin;
  const float2 kk = make_float2(k2, k2);
  const float2 ks = make_float2(k2 * 0x1p-22f, k2 * 0x1p-22f);
  const float2 nt = make_float2(-l2t, -l2t), nq = make_float2(-l2q, -l2q);
  const float st1 = fmaf(fabsf(l2t), 0x1p-22f, 0x1p-16f);  // + the log2 E slack
  const float2 st = make_float2(st1, st1);
  const float sq1 = fabsf(l2q) * 0x1p-22f;
  const float2 sq = make_float2(sq1, sq1);
  const float2 shrink = make_float2(-(1.0f - 0x1p-21f), -(1.0f - 0x1p-21f));
  const float2 one = make_float2(1.0f, 1.0f);
  const int nfull = a.V / VEC;
  const bool aligned =
      ((uintptr_t)trow & 15u) == 0 && (!residual || ((uintptr_t)qrow & 15u) == 0);
#pragma unroll 1
  for (int j = 0; j < kLaneVecs; ++j) {
    const int v = seg * kSegVecs + lane + 32 * j;
    if (v >= a.nvec) break;
    uint4 wt, wq = make_uint4(0u, 0u, 0u, 0u);
    if (aligned && v < nfull) {
      wt = ld_stream16(trow + (size_t)v * 16);
      if (residual) wq = ld_stream16(qrow + (size_t)v * 16);
    } else {
      wt = load_vec_checked<DT>(trow, v, a.V, a.nvec, nfull, aligned);
      if (residual) wq = load_vec_checked<DT>(qrow, v, a.V, a.nvec, nfull, aligned);
    }
#pragma unroll
    for (int h = 0; h < VEC / 4; ++h) {
      const uint32_t base = (uint32_t)(v * VEC + 4 * h);
      const uint4 o4 = race_words_fast(R, base >> 2);
#pragma unroll
      for (int e = 0; e < 4; e += 2) {
        const float2 zt = make_float2(elem<DT>(wt, 4 * h + e), elem<DT>(wt, 4 * h + e + 1));
        const float2 El = e == 0 ? E_lower2(o4.x, o4.y) : E_lower2(o4.z, o4.w);
        // log2 p(x) + slack, an upper bound (the log2 E slack is folded into st)
        const float2 l2pu = __fadd2_rn(__ffma2_rn(zt, kk, nt),
                                       __ffma2_rn(make_float2(fabsf(zt.x), fabsf(zt.y)), ks, st));
        float2 bound = __fadd2_rn(l2pu, make_float2(-lg2_approx(El.x), -lg2_approx(El.y)));
        if (residual) {
          // r = p (1 - q'/p): add an upper bound of log2(1 - 2^d), d = log2 q' - log2 p
          const float2 zq = make_float2(elem<DT>(wq, 4 * h + e), elem<DT>(wq, 4 * h + e + 1));
          const float2 dlo = __fadd2_rn(
              __fadd2_rn(__ffma2_rn(zq, kk, nq),
                         __fmul2_rn(__ffma2_rn(make_float2(fabsf(zq.x), fabsf(zq.y)), ks, sq),
                                    make_float2(-1.0f, -1.0f))),
              make_float2(-l2pu.x, -l2pu.y));
          const float2 t = __ffma2_rn(make_float2(ex2_approx(dlo.x), ex2_approx(dlo.y)), shrink, one);
          const float2 res = __fadd2_rn(bound, make_float2(lg2_approx(t.x) + 0x1p-16f,
                                                           lg2_approx(t.y) + 0x1p-16f));
          // a token of K keeps the bound r <= p; q' >= p excludes the token
          bound.x = zq.x >= kmin ? bound.x : (dlo.x < 0.0f ? res.x : -INFINITY);
          bound.y = zq.y >= kmin ? bound.y : (dlo.y < 0.0f ? res.y : -INFINITY);
        }
        const int x = (int)base + e;
        if (x < a.V && zt.x > -INFINITY) visit(bound.x, x);
        if (x + 1 < a.V && zt.y > -INFINITY) visit(bound.y, x + 1);
      }
    }
  }
}

// The exact best and runner-up of segment `seg` (all lanes get the result).
template <int DT>
__device__ __forceinline__ Best race_segment(const VerifyArgs& a, const RaceDesc& rd,
                                             const char* trow, const char* qrow,
                                             bool residual, int seg) {
  // A. the two largest bounds of each lane
  const RaceStream R = race_stream(a.seed, rd.g);
  float u1 = -INFINITY, u2 = -INFINITY;
  int i1 = -1, i2 = -1;
  race_bounds<DT>(a, rd, R, trow, qrow, residual, seg, [&](float bound, int x) {
    // branch-free: ties keep the earlier (lower) index
    const bool gt1 = bound > u1, gt2 = bound > u2;
    u2 = gt1 ? u1 : (gt2 ? bound : u2);
    i2 = gt1 ? i1 : (gt2 ? x : i2);
    u1 = gt1 ? bound : u1;
    i1 = gt1 ? x : i1;
  });
  // B. the exact key of each lane's best token
  Best B{-INFINITY, -INFINITY, -1};
  if (i1 >= 0) offer(B, exact_key_of(a, rd, trow, qrow, residual, i1), i1);
  double S1 = B.best;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) S1 = fmax(S1, __shfl_xor_sync(0xFFFFFFFFu, S1, o));
  // C. every token whose bound reaches S1 (less the margin) gets its exact key
  const float thr = S1 == -INFINITY ? -INFINITY : (float)(S1 * 1.4426950408889634) - 0x1p-14f;
  if (i2 >= 0 && u2 >= thr) {
    offer(B, exact_key_of(a, rd, trow, qrow, residual, i2), i2);
    // the third bound may have reached thr as well: visit them all
    const int j1 = i1, j2 = i2;
    race_bounds<DT>(a, rd, R, trow, qrow, residual, seg, [&](float bound, int x) {
      if (bound >= thr && x != j1 && x != j2)
        offer(B, exact_key_of(a, rd, trow, qrow, residual, x), x);
    });
  }
  return warp_combine(B);
}

// Copy a request's race description into the warp's shared slot.
__device__ __forceinline__ void load_race_desc(const RaceDesc* src, RaceDesc* dst) {
  const int lane = threadIdx.x & 31;
  constexpr int n16 = sizeof(RaceDesc) / 16;
  static_assert(sizeof(RaceDesc) % 16 == 0, "RaceDesc is copied in 16-byte pieces");
  if (lane < n16)
    reinterpret_cast<uint4*>(dst)[lane] = __ldcg(reinterpret_cast<const uint4*>(src) + lane);
  __syncwarp();
}

// Race segment `seg` of request b, by one warp (rd in the warp's shared slot).
// The warp that completes the request's last segment merges and writes the token.
template <int DT>
__device__ inline void race_item(const VerifyArgs& a, int b, int seg, const RaceDesc& rd) {
  const int lane = threadIdx.x & 31;
  const bool residual = rd.kind == kRaceResidual;
  const char* trow = row_base(a, b, rd.n);
  const char* qrow = residual ? row_base(a, b, a.D_max + 1 + rd.n) : nullptr;
  const Best sb = race_segment<DT>(a, rd, trow, qrow, residual, seg);

  unsigned prev = 0;
  if (lane == 0) {
    RacePart p;
    p.best = sb.best;
    p.second = sb.second;
    p.idx = sb.idx;
    p.pad = 0;
    a.rpart[(size_t)b * a.nseg + seg] = p;
    __threadfence();
    prev = atomicAdd(&a.rcount[b], 1u);
  }
  prev = __shfl_sync(0xFFFFFFFFu, prev, 0);
  if (prev != (unsigned)(a.nseg - 1)) return;

  // the last segment of this request: merge every segment's result
  __threadfence();
  Best r{-INFINITY, -INFINITY, -1};
  for (int s = lane; s < a.nseg; s += 32) {
    const RacePart* pp = a.rpart + (size_t)b * a.nseg + s;
    Best o;
    o.best = __ldcg(&pp->best);
    o.second = __ldcg(&pp->second);
    o.idx = __ldcg(&pp->idx);
    r = combine(r, o);
  }
  r = warp_combine(r);
  uint32_t flags = rd.flags;
  if (r.idx < 0 && residual) {
    // {p > q} was empty through rounding: draw from p on the same row instead
    flags |= kFlagResidualEmpty;
    Best Bb{-INFINITY, -INFINITY, -1};
    for (int s = 0; s < a.nseg; ++s) Bb = combine(Bb, race_segment<DT>(a, rd, trow, nullptr, false, s));
    r = Bb;
  }
  if (lane == 0) {
    if (r.best - r.second < 1e-6) flags |= kFlagRaceNearTie;
    a.out_tokens[(size_t)b * (a.D_max + 1) + rd.n] = r.idx;
    if (a.out_flags) a.out_flags[b] = flags;
    if (flags & kFlagResidualEmpty) atomicOr(a.status, kFlagResidualEmpty);
  }
}

}  // namespace sv
