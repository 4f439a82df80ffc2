// race_sampler.cu -- the residual / bonus token of each stochastic request.
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
// Exactness: the key ln r(x) - ln E_x is evaluated in double precision, with the
// same formulas as the reference definition, but only for tokens that can still
// win.  Every token first gets a cheap single-precision upper bound of its key
// (ln p(x) - ln E_x >= ln r(x) - ln E_x, evaluated with ex2/lg2 and an error
// below 2^-12 in log2 units); a token whose bound is more than kMargin2 below
// the best exact key seen so far in its warp cannot win and is skipped.  The
// winner and the runner-up (for the near-tie flag) are therefore those of the
// exact keys.
//
// Layout: one CTA per (request, 32 KiB chunk of the row), the same chunking as
// the statistics pass; the last CTA of a request to finish (atomic counter, no
// waiting) merges the chunk results and writes the token.
#include "philox.cuh"
#include "sv_common.cuh"

#include <float.h>
#include <limits.h>
#include <math.h>

namespace sv {

namespace {

constexpr float kMargin2 = 0x1p-9f;  // filter margin, log2 units (>> the bound's error)

struct Best {
  double best;
  double second;
  int idx;
};

__device__ __forceinline__ void offer(Best& B, double key, int x) {
  if (key > B.best || (key == B.best && (B.idx < 0 || x < B.idx))) {
    B.second = B.best;
    B.best = key;
    B.idx = x;
  } else if (key > B.second) {
    B.second = key;
  }
}

__device__ __forceinline__ Best combine(const Best& A, const Best& C) {
  const bool c_wins = C.idx >= 0 && (A.idx < 0 || C.best > A.best || (C.best == A.best && C.idx < A.idx));
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

// log2 of E = -ln(1 - W), W = (o + 1/2) 2^-32, to about 2^-12 (relative in E).
__device__ __forceinline__ float approx_log2_E(uint32_t o) {
  // W < 2^-10: E = W + W^2/2 (+ W^3/3..., below 2^-20 relative)
  const float fa = __uint_as_float(0x4B000000u | (o & 0x7FFFFFu)) - 8388608.0f;
  const float Ws = (fa + 0.5f) * 0x1p-32f;
  const float Es = fmaf(0.5f * Ws, Ws, Ws);
  // otherwise E = -ln(U), U = 1 - W: exactly (~o + 1/2) 2^-32 when ~o < 2^23,
  // else 1 - (o >> 9) 2^-23 (absolute error < 2^-23, U >= 2^-9 there)
  const uint32_t no = ~o;
  const float fc = __uint_as_float(0x4B000000u | (no & 0x7FFFFFu)) - 8388608.0f;
  const float fb = __uint_as_float(0x4B000000u | (o >> 9)) - 8388608.0f;
  const float U = no < 0x800000u ? (fc + 0.5f) * 0x1p-32f : fmaf(-fb, 0x1p-23f, 1.0f);
  const float El = -0.693147180559945f * lg2_approx(U);
  return lg2_approx(o < 0x400000u ? Es : El);
}

// The exact key ln r(x) - ln E_x in double precision; false if x is no candidate.
__device__ __noinline__ bool exact_key(float zt, float zq, int x, uint32_t o, const RaceDesc& rd,
                                       bool residual, double* key) {
  const double lp = (double)zt / rd.T - rd.lse_t;
  if (lp == -INFINITY) return false;
  double lr = lp;
  if (residual) {
    double lq = (double)zq / rd.T - rd.lse_q;
    if (rd.ntop > 0 && lq != -INFINITY) {
      bool in_k = false;
      for (int i = 0; i < rd.ntop; ++i) in_k |= (rd.top[i] == x);
      lq += (in_k ? rd.ln_c : 0.0) - rd.ln_Z;
    }
    if (!(lp > lq)) return false;
    if (lq != -INFINITY) lr = lp + log(-expm1(lq - lp));
  }
  const double W = ((double)o + 0.5) * 0x1p-32;
  *key = lr - log(-log1p(-W));
  return true;
}

template <int DT>
__device__ __forceinline__ float elem_at(const char* row, int x) {
  if (DT == kF32) return ((const float*)row)[x];
  return __uint_as_float((uint32_t)((const uint16_t*)row)[x] << 16);
}

// One thread's share of one chunk.
template <int DT>
__device__ __forceinline__ void race_chunk(const VerifyArgs& a, const RaceDesc& rd,
                                           const char* trow, const char* qrow, bool residual,
                                           int chunk, Best& B, float& thr2) {
  constexpr int VEC = DT == kF32 ? 4 : 8;
  const int t = threadIdx.x;
  const int V = a.V, nfull = V / VEC;
  const bool aligned =
      ((uintptr_t)trow & 15u) == 0 && (!residual || ((uintptr_t)qrow & 15u) == 0);
  const uint32_t k0 = (uint32_t)a.seed, k1 = (uint32_t)(a.seed >> 32);
  const float k2 = rd.k2, l2t = rd.l2_t;
#pragma unroll 1
  for (int j = 0; j < kVecsPerThread; ++j) {
    const int v = chunk * kChunkVecs + t + j * kThreads;
    if (v < a.nvec) {
      float zt[VEC], zq[VEC];
      if (aligned && v < nfull) {
        const uint4 wt = ld_stream16(trow + (size_t)v * 16);
        const uint32_t wt4[4] = {wt.x, wt.y, wt.z, wt.w};
#pragma unroll
        for (int e = 0; e < VEC; ++e)
          zt[e] = DT == kF32 ? __uint_as_float(wt4[e]) : ((e & 1) ? bf_hi(wt4[e >> 1]) : bf_lo(wt4[e >> 1]));
        if (residual) {
          const uint4 wq = ld_stream16(qrow + (size_t)v * 16);
          const uint32_t wq4[4] = {wq.x, wq.y, wq.z, wq.w};
#pragma unroll
          for (int e = 0; e < VEC; ++e)
            zq[e] = DT == kF32 ? __uint_as_float(wq4[e]) : ((e & 1) ? bf_hi(wq4[e >> 1]) : bf_lo(wq4[e >> 1]));
        }
      } else {
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          const int x = v * VEC + e;
          zt[e] = x < V ? elem_at<DT>(trow, x) : -INFINITY;
          zq[e] = (residual && x < V) ? elem_at<DT>(qrow, x) : 0.0f;
        }
      }
#pragma unroll
      for (int h = 0; h < VEC / 4; ++h) {
        const uint32_t base = (uint32_t)(v * VEC + 4 * h);
        const uint4 o4 = philox4x32_10(make_uint4(base >> 2, rd.g, 1u, 0u), k0, k1);
        const uint32_t ow[4] = {o4.x, o4.y, o4.z, o4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int x = (int)base + e;
          const float z = zt[4 * h + e];
          const float bound = fmaf(z, k2, -l2t) - approx_log2_E(ow[e]);
          if (bound >= thr2 && z > -INFINITY) {
            double key;
            if (exact_key(z, zq[4 * h + e], x, ow[e], rd, residual, &key)) {
              offer(B, key, x);
              thr2 = fmaxf(thr2, (float)(B.best * 1.4426950408889634) - kMargin2);
            }
          }
        }
      }
    }
    // share the warp's best threshold
    thr2 = warp_max(thr2);
  }
}

template <int DT>
__device__ Best race_block_reduce(Best B) {
  __shared__ double s_best[kThreads / 32], s_second[kThreads / 32];
  __shared__ int s_idx[kThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  B = warp_combine(B);
  if (lane == 0) {
    s_best[warp] = B.best;
    s_second[warp] = B.second;
    s_idx[warp] = B.idx;
  }
  __syncthreads();
  Best r;
  r.best = s_best[0];
  r.second = s_second[0];
  r.idx = s_idx[0];
  for (int w = 1; w < kThreads / 32; ++w) {
    Best o;
    o.best = s_best[w];
    o.second = s_second[w];
    o.idx = s_idx[w];
    r = combine(r, o);
  }
  __syncthreads();
  return r;
}

template <int DT>
__global__ void __launch_bounds__(kThreads) race_kernel(VerifyArgs a) {
  __shared__ RaceDesc rd;
  __shared__ int s_last;
  const int chunk = blockIdx.x % a.nch;
  const int b = blockIdx.x / a.nch;
  if (threadIdx.x == 0) rd = a.rdesc[b];
  __syncthreads();
  if (rd.kind == kRaceNone) return;
  const bool residual = rd.kind == kRaceResidual;
  const char* trow = row_base(a, b, rd.n);
  const char* qrow = residual ? row_base(a, b, a.D_max + 1 + rd.n) : nullptr;

  Best B{-INFINITY, -INFINITY, -1};
  float thr2 = -INFINITY;
  race_chunk<DT>(a, rd, trow, qrow, residual, chunk, B, thr2);
  const Best cb = race_block_reduce<DT>(B);

  if (threadIdx.x == 0) {
    RacePart p;
    p.best = cb.best;
    p.second = cb.second;
    p.idx = cb.idx;
    p.pad = 0;
    a.rpart[(size_t)b * a.nch + chunk] = p;
    __threadfence();
    const unsigned prev = atomicAdd(&a.rcount[b], 1u);
    s_last = prev == (unsigned)(a.nch - 1);
  }
  __syncthreads();
  if (!s_last) return;

  // the last chunk of this request: merge every chunk's result
  __threadfence();
  Best r{-INFINITY, -INFINITY, -1};
  for (int c = 0; c < a.nch; ++c) {
    const RacePart* pp = a.rpart + (size_t)b * a.nch + c;
    Best o;
    o.best = __ldcg(&pp->best);
    o.second = __ldcg(&pp->second);
    o.idx = __ldcg(&pp->idx);
    r = combine(r, o);
  }
  uint32_t flags = rd.flags;
  if (r.idx < 0 && residual) {
    // {p > q} was empty through rounding: draw from p on the same row instead
    flags |= kFlagResidualEmpty;
    Best Bb{-INFINITY, -INFINITY, -1};
    float th = -INFINITY;
    for (int c = 0; c < a.nch; ++c) race_chunk<DT>(a, rd, trow, nullptr, false, c, Bb, th);
    r = race_block_reduce<DT>(Bb);
  }
  if (threadIdx.x == 0) {
    if (r.best - r.second < 1e-6) flags |= kFlagRaceNearTie;
    a.out_tokens[(size_t)b * (a.D_max + 1) + rd.n] = r.idx;
    if (a.out_flags) a.out_flags[b] = flags;
    if (flags & kFlagResidualEmpty) atomicOr(a.status, kFlagResidualEmpty);
  }
}

}  // namespace

cudaError_t launch_race(const VerifyArgs& a, cudaStream_t s) {
  const long long grid = (long long)a.B * a.nch;
  if (grid == 0) return cudaSuccess;
  if (a.dtype == kF32)
    race_kernel<kF32><<<(unsigned)grid, kThreads, 0, s>>>(a);
  else
    race_kernel<kBF16><<<(unsigned)grid, kThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace sv
