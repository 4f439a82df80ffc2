// race_device.cuh -- device code of the residual / bonus race, shared by the
// split race kernel, the accept scan (its reference key) and the fused kernel.
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
// Exactness.  The decision is taken on the exact key
//   key(x) = ln r(x) - ln E_x,   E_x = -ln(1 - W_x),   W_x = (o_x + 1/2) 2^-32
// in double precision, with the same formulas as the plain definition, but only
// for the tokens that can matter.  Since r(x) <= p(x) and E_x >= W_x,
//   key(x) <= ln p(x) - ln W_x,
// so once the exact key K0 of any one real token is known, a token whose key
// reaches K0 - delta must have a small Philox word:
//   o_x + 1/2 <= 2^L(x),   L(x) = log2 p(x) + 32 - (K0 - delta) log2(e) = z_x k2 + C.
// The word filter (word_filter) tests this with four instructions per token:
// a packed FMA and add for L (its single-precision error is covered by slack
// folded into C: filter_offset), a count of leading zeros of o_x, and an
// integer add whose sign bit says "drop".  The race's best key is >= K0, so
// every token within the near-tie band delta of the best survives the filter;
// the survivors (a handful per row) get exact keys.
//
// K0 comes from a search in the segment holding the sampled row's largest
// logit (race_ref_key_warp), and grows as segments finish; where none is known
// (K0 = -inf) a segment first takes the best exact key of its 32 lane-wise
// largest logits, and if that is -inf too every token survives the filter.
// One warp handles an 8 KiB segment, or a run of them (race_segment_in,
// race_span_in); the segments' results are combined by the CTA that owns the
// request or by the warp that finishes its last segment (tail_device.cuh).
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

// The fields of the argument block that the race's out-of-line helpers read,
// passed by value: a reference to the argument block (kernel parameter space)
// would make every thread copy the block to its stack at each call.
struct RowCtx {
  uint64_t seed;
  int dtype, V, nvec, vocab_offset;
};

__device__ __forceinline__ RowCtx row_ctx(const VerifyArgs& a) {
  RowCtx c;
  c.seed = seed_of(a);
  c.dtype = a.dtype;
  c.V = a.V;
  c.nvec = a.nvec;
  c.vocab_offset = a.vocab_offset;
  return c;
}

__device__ __forceinline__ RowCtx row_ctx(const RowCtx& c) { return c; }

__device__ __forceinline__ uint64_t seed_of(const RowCtx& c) { return c.seed; }

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

// Doubles as unsigned integers in the same order (-0 < +0 aside).
__device__ __forceinline__ unsigned long long ordered_u64(double v) {
  const unsigned long long b = (unsigned long long)__double_as_longlong(v);
  return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

__device__ __forceinline__ double from_ordered_u64(unsigned long long o) {
  const unsigned long long b = (o >> 63) ? (o & 0x7FFFFFFFFFFFFFFFull) : ~o;
  return __longlong_as_double((long long)b);
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

// (A: the argument block or a RowCtx)
template <class A>
__device__ __forceinline__ double exact_key_of(const A& a, const RaceDesc& rd,
                                               const char* trow, const char* qrow,
                                               bool residual, int x) {
  const float zt = (a.dtype == kF32) ? logit_at<kF32>(trow, x) : logit_at<kBF16>(trow, x);
  float zq = 0.0f;
  if (residual) zq = (a.dtype == kF32) ? logit_at<kF32>(qrow, x) : logit_at<kBF16>(qrow, x);
  const int gx = x + a.vocab_offset;  // the token's global index (Philox counter, saguaro K)
  return exact_key(zt, zq, gx, race_word(seed_of(a), rd.g, gx), rd, residual);
}

constexpr double kRaceBand = 1e-5;  // delta: the 1e-6 near-tie band plus every rounding error

// The word filter's offset C for the reference key K0 of a race on a target
// row with LSE lse_t, raised by the filter's own error bound:
//   C = 32 + (delta - lse_t - K0) log2(e).
// The filter computes L = fl(fma(z, k2, C)).  k2 is within 2^-23 of log2(e)/T
// (relative), the FMA rounds once, and |z k2| <= |L| + |C|, so where the
// outcome depends on L (|L| <= 64) its error is below (64 + |C|) 2^-21.
// +inf (keep every token) when K0 is -inf or C is too large to resolve.
__device__ __forceinline__ float filter_offset(double K0, double lse_t) {
  if (!(K0 > -INFINITY) || !(fabs(lse_t) < INFINITY)) return INFINITY;
  const double C = 32.0 + (kRaceBand - lse_t - K0) * 1.4426950408889634;
  if (!(fabs(C) < 0x1p24)) return INFINITY;
  return __double2float_ru(C + (64.0 + fabs(C)) * 0x1p-21 + 0x1p-20);
}

// Tokens per 16-byte vector.
template <int DT>
struct Lanes {
  static constexpr int VEC = DT == kF32 ? 4 : 8;
};

// The index of the most significant set bit of o, -1 for o = 0.
__device__ __forceinline__ int msb_index(uint32_t o) {
  int r;
  asm("bfind.u32 %0, %1;" : "=r"(r) : "r"(o));
  return r;
}

// The word filter over one group of 32 tokens of a lane: vectors j0 .. j0 +
// 32/VEC - 1 of the lane (vector j of the lane is vector v0 + 32 j of the row),
// logits in raw.  Returns the drop word: bit 31 - t is set when token t of the
// group (element t mod VEC of vector j0 + t / VEC) cannot reach K0 - delta.
// A token is kept iff o < 2^ceil(L); with o's top set bit at position m
// (m = -1 for o = 0) that is  m + 1 <= ceil(L), i.e.
//   bits(L + 1.5 * 2^23, rounded up) - m - bits(1.5 * 2^23) - 1 >= 0:
// for |L| < 2^22 the float sum holds ceil(L) in its low bits, and below or
// above that range (-inf included) the comparison still comes out right.
template <int DT>
__device__ __forceinline__ uint32_t word_filter(const uint4 (&raw)[32 / Lanes<DT>::VEC], int j0,
                                                const RaceStream& R, int v0, float k2, float cup) {
  constexpr int VEC = Lanes<DT>::VEC, QV = 32 / VEC;
  const float2 kk = make_float2(k2, k2), cc = make_float2(cup, cup);
  const float2 magic = make_float2(12582912.0f, 12582912.0f);
  // one flag accumulator per vector (independent chains), joined at the end
  uint32_t acc[QV];
#pragma unroll
  for (int jj = 0; jj < QV; ++jj) {
    acc[jj] = 0u;
#pragma unroll
    for (int h = 0; h < VEC / 4; ++h) {
      const uint32_t base = (uint32_t)((v0 + 32 * (j0 + jj)) * VEC + 4 * h);
      const uint4 o4 = race_words_fast(R, base >> 2);
#pragma unroll
      for (int e = 0; e < 4; e += 2) {
        const float2 z = make_float2(elem<DT>(raw[jj], 4 * h + e), elem<DT>(raw[jj], 4 * h + e + 1));
        const float2 F = __fadd2_ru(__ffma2_ru(z, kk, cc), magic);
        const uint32_t oa = e == 0 ? o4.x : o4.z, ob = e == 0 ? o4.y : o4.w;
        const int ta = __float_as_int(F.x) - msb_index(oa) - (0x4B400000 + 1);
        const int tb = __float_as_int(F.y) - msb_index(ob) - (0x4B400000 + 1);
        acc[jj] = __funnelshift_l((uint32_t)ta, acc[jj], 1);
        acc[jj] = __funnelshift_l((uint32_t)tb, acc[jj], 1);
      }
    }
  }
  uint32_t drop = 0u;
#pragma unroll
  for (int jj = 0; jj < QV; ++jj) drop = (drop << VEC) + acc[jj];
  return drop;
}

// word_filter with Philox's ten rounds in a loop (the round keys advanced in
// place) over the group's eight counters at once: the same drop word from a
// body a fraction of the unrolled one's size, for code that shares the
// instruction cache with the statistics pass.
template <int DT>
__device__ __forceinline__ uint32_t word_filter_compact(const uint4 (&raw)[32 / Lanes<DT>::VEC],
                                                        int j0, uint64_t seed, uint32_t g,
                                                        uint32_t i0, int v0, float k2, float cup) {
  constexpr int VEC = Lanes<DT>::VEC, QV = 32 / VEC, NC = 8;  // eight blocks of four tokens
  uint4 c[NC];
#pragma unroll
  for (int n = 0; n < NC; ++n) {
    const int jj = n / (VEC / 4), h = n % (VEC / 4);
    c[n] = make_uint4(i0 + ((uint32_t)((v0 + 32 * (j0 + jj)) * VEC + 4 * h) >> 2), g, 1u, 0u);
  }
  uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
#pragma unroll 1
  for (int r = 0; r < 10; ++r) {
#pragma unroll
    for (int n = 0; n < NC; ++n) philox_round(c[n], k0, k1);
    k0 += kWeylA;
    k1 += kWeylB;
  }
  const float2 kk = make_float2(k2, k2), cc = make_float2(cup, cup);
  const float2 magic = make_float2(12582912.0f, 12582912.0f);
  uint32_t drop = 0u;
#pragma unroll
  for (int n = 0; n < NC; ++n) {
    const int jj = n / (VEC / 4), h = n % (VEC / 4);
#pragma unroll
    for (int e = 0; e < 4; e += 2) {
      const float2 z = make_float2(elem<DT>(raw[jj], 4 * h + e), elem<DT>(raw[jj], 4 * h + e + 1));
      const float2 F = __fadd2_ru(__ffma2_ru(z, kk, cc), magic);
      const uint32_t oa = e == 0 ? c[n].x : c[n].z, ob = e == 0 ? c[n].y : c[n].w;
      const int ta = __float_as_int(F.x) - msb_index(oa) - (0x4B400000 + 1);
      const int tb = __float_as_int(F.y) - msb_index(ob) - (0x4B400000 + 1);
      drop = __funnelshift_l((uint32_t)ta, drop, 1);
      drop = __funnelshift_l((uint32_t)tb, drop, 1);
    }
  }
  (void)QV;
  return drop;
}

// Vectors j0 .. j0 + NJ - 1 of one lane's part of segment `seg` (-inf past the
// end of the row).
template <int DT, int NJ, class A>
__device__ __forceinline__ void load_part(const A& a, const char* row, int seg, int j0,
                                          uint4 (&raw)[NJ]) {
  constexpr int VEC = Lanes<DT>::VEC;
  const int nfull = a.V / VEC;
  const int v0 = seg * kSegVecs + (threadIdx.x & 31) + 32 * j0;
  const bool aligned = ((uintptr_t)row & 15u) == 0;
  if (aligned && v0 + 32 * (NJ - 1) < nfull) {
#pragma unroll
    for (int j = 0; j < NJ; ++j) raw[j] = ld_stream16(row + (size_t)(v0 + 32 * j) * 16);
  } else {
#pragma unroll
    for (int j = 0; j < NJ; ++j) raw[j] = load_vec_checked<DT>(row, v0 + 32 * j, a.V, a.nvec, nfull, aligned);
  }
}

// An upper bound, in log2 units, of token x's race key (key / ln 2), from
// single-precision arithmetic with every rounding error covered; -inf when x
// cannot be a candidate (masked, or q'(x) >= p(x) for certain in a residual
// race).  It uses r <= p and E >= W like the word filter, but with the exact
// word and, for a residual, the factor (1 - q'/p):
//   key/ln2 <= log2 p(x) + log2(1 - 2^d) + 32 - log2(o + 1/2),
//   d = log2 q'(x) - log2 p(x),
// each term bounded with slack for its rounding: log2 p from one FMA on k2
// (within 2^-23 of log2(e)/T), log2f and expm1f (1 ulp each), the conversions,
// and the sums (all below the 2^-21 relative slack added to each term).
static __device__ __noinline__ float key2_upper(const RowCtx a, const RaceDesc& rd,
                                                const char* trow, const char* qrow,
                                                bool residual, int x) {
  const bool f32 = a.dtype == kF32;
  const float z = f32 ? logit_at<kF32>(trow, x) : logit_at<kBF16>(trow, x);
  if (!(z > -INFINITY)) return -INFINITY;
  const float k2 = rd.k2;
  const float l2t = (float)(rd.lse_t * 1.4426950408889634);
  float l2p = fmaf(z, k2, -l2t);
  l2p += (fabsf(z) * k2 + fabsf(l2t) + fabsf(l2p)) * 0x1p-21f + 0x1p-40f;
  float h = 0.0f;
  if (residual) {
    const float zq = f32 ? logit_at<kF32>(qrow, x) : logit_at<kBF16>(qrow, x);
    if (zq > -INFINITY) {
      const float l2qb = (float)((rd.lse_q + rd.ln_Z) * 1.4426950408889634);
      float l2q = fmaf(zq, k2, -l2qb);
      float lc = 0.0f;
      if (rd.ntop > 0) {
        bool in_k = false;
        for (int i = 0; i < rd.ntop; ++i) in_k |= (rd.top[i] == x + a.vocab_offset);
        if (in_k) lc = (float)(rd.ln_c * 1.4426950408889634);
      }
      l2q += lc;
      l2q -= (fabsf(zq) * k2 + fabsf(l2qb) + fabsf(lc) + fabsf(l2q)) * 0x1p-21f + 0x1p-40f;
      const float d = __fsub_rd(l2q, l2p);  // a lower bound of d
      if (!(d < 0.0f)) return -INFINITY;
      // log2(1 - 2^d) falls as d rises, so d's lower bound gives an upper bound;
      // d ln 2 is rounded down (more negative), 1 - 2^y = -expm1(y ln 2)
      const float u = -expm1f(__fmul_rd(d, 0.6931471825f));
      const float hl = log2f(u * (1.0f + 0x1p-21f));
      h = hl + fabsf(hl) * 0x1p-21f + 0x1p-40f;
    }
  }
  const uint32_t o = race_word(seed_of(a), rd.g, x + a.vocab_offset);
  const float lw = log2f((float)o + 0.5f);
  const float nlw = 32.0f - lw + fabsf(lw) * 0x1p-21f + 0x1p-20f;
  const float sum = l2p + h + nlw;
  return sum + (fabsf(l2p) + fabsf(h) + fabsf(nlw)) * 0x1p-21f;
}

// The best exact key among the lanes' largest target logits of a segment (one
// token per lane, the lowest index on ties), over the warp; -inf if none.
template <int DT>
__device__ __noinline__ double lane_max_key(const RowCtx a, const RaceDesc& rd,
                                            const char* trow, const char* qrow, bool residual,
                                            int seg) {
  constexpr int VEC = Lanes<DT>::VEC;
  const int v0 = seg * kSegVecs + (threadIdx.x & 31);
  float mv = -INFINITY;
  int xi = -1;
#pragma unroll 1
  for (int j0 = 0; j0 < kLaneVecs; j0 += kLaneVecs / 2) {
    uint4 raw[kLaneVecs / 2];
    load_part<DT>(a, trow, seg, j0, raw);
#pragma unroll
    for (int j = 0; j < kLaneVecs / 2; ++j)
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        const float z = elem<DT>(raw[j], e);
        if (z > mv) {
          mv = z;
          xi = (v0 + 32 * (j0 + j)) * VEC + e;
        }
      }
  }
  double k = -INFINITY;
  if (xi >= 0 && xi < a.V) k = exact_key_of(a, rd, trow, qrow, residual, xi);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) k = fmax(k, __shfl_xor_sync(0xFFFFFFFFu, k, o));
  return k;
}

// The exact best and runner-up of segment `seg` among the tokens that can reach
// K0 - delta (all lanes get the result); K0 and its filter offset cup come
// from the caller, K0 = -inf when unknown.  A runner-up below best - delta may
// come out lower than it is; no decision depends on it.  R is the race's
// Philox stream.  The lane walks its part of the segment in groups of 32
// tokens, loading the next group while it filters the current one, and takes
// exact keys of a group's survivors (rare) right away, so the loop body stays
// small enough for the instruction cache.  Only groups g0 .. g1 - 1 of the
// lane's NG (g1 < 0: to the end) are raced, so that a segment can be split
// into independent items.
template <int DT, class A>
__device__ __forceinline__ Best race_segment_in(const A& a, const RaceDesc& rd,
                                                const RaceStream& R, const char* trow,
                                                const char* qrow, bool residual, int seg,
                                                double K0, float cup, int g0 = 0, int g1 = -1) {
  constexpr int VEC = Lanes<DT>::VEC, QV = 32 / VEC, NG = kLaneVecs / QV;
  if (g1 < 0) g1 = NG;
  const int v0 = seg * kSegVecs + (threadIdx.x & 31);
  if (!(K0 > -INFINITY)) {
    K0 = lane_max_key<DT>(row_ctx(a), rd, trow, qrow, residual, seg);
    cup = filter_offset(K0, rd.lse_t);
  }
  // survivors whose single-precision bound falls below K0 - delta need no exact key
  const float thr2 = K0 > -INFINITY ? __double2float_rd((K0 - kRaceBand) * 1.4426950408889634 - 1e-5)
                                    : -INFINITY;

  Best B{-INFINITY, -INFINITY, -1};
  uint4 cur[QV], nxt[QV];
  load_part<DT>(a, trow, seg, g0 * QV, cur);
#pragma unroll 1
  for (int gi = g0; gi < g1; ++gi) {
    if (gi + 1 < g1) load_part<DT>(a, trow, seg, (gi + 1) * QV, nxt);
    uint32_t keep = ~word_filter<DT>(cur, gi * QV, R, v0, rd.k2, cup);
    // exact keys of the survivors, one token per lane at a time
    while (__any_sync(0xFFFFFFFFu, keep != 0u)) {
      if (keep) {
        const int t = __clz((int)keep);
        keep &= ~(0x80000000u >> t);
        const int x = (v0 + 32 * (gi * QV + t / VEC)) * VEC + t % VEC;
        if (x < a.V && key2_upper(row_ctx(a), rd, trow, qrow, residual, x) >= thr2)
          offer(B, exact_key_of(a, rd, trow, qrow, residual, x), x);
      }
    }
    if (gi + 1 < g1) {
#pragma unroll
      for (int j = 0; j < QV; ++j) cur[j] = nxt[j];
    }
  }
  return warp_combine(B);
}

// Segments seg0, seg0 + step, ... (below a.nseg) of the race, by one warp, as
// one stream of 32-token groups: the next group loads while the current one is
// filtered, across segment boundaries too.  At each boundary the warp raises
// *shared (the request's best key so far, ordered bits, in shared memory) with
// its own best and takes the largest of K0, its own best and *shared as the
// reference key for the next segment.  Returns the combination of all the
// segments' results (all lanes); otherwise as race_segment_in.
template <int DT>
__device__ __forceinline__ Best race_span_in(const VerifyArgs& a, const RaceDesc& rd,
                                             const RaceStream& R, const char* trow,
                                             const char* qrow, bool residual, int seg0, int step,
                                             double K0, unsigned long long* shared) {
  constexpr int VEC = Lanes<DT>::VEC, QV = 32 / VEC, NG = kLaneVecs / QV;
  const int lane = threadIdx.x & 31;
  Best B{-INFINITY, -INFINITY, -1};
  if (seg0 >= a.nseg) return B;
  int seg = seg0;
  double K = fmax(K0, from_ordered_u64(*(volatile unsigned long long*)shared));
  if (!(K > -INFINITY)) K = lane_max_key<DT>(row_ctx(a), rd, trow, qrow, residual, seg);
  float cup = filter_offset(K, rd.lse_t);
  float thr2 = K > -INFINITY ? __double2float_rd((K - kRaceBand) * 1.4426950408889634 - 1e-5)
                             : -INFINITY;
  uint4 cur[QV], nxt[QV];
  load_part<DT>(a, trow, seg, 0, cur);
  int gi = 0;
#pragma unroll 1
  for (;;) {
    const bool seg_end = gi + 1 == NG;
    const int nseg_ = seg_end ? seg + step : seg;
    const int ngi = seg_end ? 0 : gi + 1;
    const bool more = nseg_ < a.nseg;
    if (more) load_part<DT>(a, trow, nseg_, ngi * QV, nxt);
    const int v0 = seg * kSegVecs + lane;
    uint32_t keep = ~word_filter<DT>(cur, gi * QV, R, v0, rd.k2, cup);
    // exact keys of the survivors, one token per lane at a time
    while (__any_sync(0xFFFFFFFFu, keep != 0u)) {
      if (keep) {
        const int t = __clz((int)keep);
        keep &= ~(0x80000000u >> t);
        const int x = (v0 + 32 * (gi * QV + t / VEC)) * VEC + t % VEC;
        if (x < a.V && key2_upper(row_ctx(a), rd, trow, qrow, residual, x) >= thr2)
          offer(B, exact_key_of(a, rd, trow, qrow, residual, x), x);
      }
    }
    if (!more) break;
    if (seg_end) {
      // share the warp's best so far and refresh the reference key
      double wb = B.best;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) wb = fmax(wb, __shfl_xor_sync(0xFFFFFFFFu, wb, o));
      if (lane == 0 && wb > -INFINITY) atomicMax(shared, ordered_u64(wb));
      __syncwarp();
      K = fmax(K, fmax(wb, from_ordered_u64(*(volatile unsigned long long*)shared)));
      if (!(K > -INFINITY)) K = lane_max_key<DT>(row_ctx(a), rd, trow, qrow, residual, nseg_);
      cup = filter_offset(K, rd.lse_t);
      thr2 = K > -INFINITY ? __double2float_rd((K - kRaceBand) * 1.4426950408889634 - 1e-5)
                           : -INFINITY;
      seg = nseg_;
    }
    gi = ngi;
#pragma unroll
    for (int j = 0; j < QV; ++j) cur[j] = nxt[j];
  }
  return warp_combine(B);
}

// Lane groups g0 .. g1 - 1 of segment `seg` of a race, by one warp, with a
// small register budget (the fused kernel runs it beside the statistics pass
// at three CTAs per multiprocessor): one 32-token group per lane in registers
// at a time, no reference-key search beforehand.  The reference key K starts
// at *best (the best exact key any finished part of the request published,
// ordered bits; 0 = none) and, while it is unknown, is taken from the group
// itself -- the best exact key among the lanes' largest logits of the group;
// after each group it rises to the warp's best so far and *best.  Returns the
// part's exact best and runner-up among the tokens that can reach K - delta
// (all lanes), as race_segment_in does.
template <int DT>
__device__ __forceinline__ Best race_part(const VerifyArgs& a, const RaceDesc& rd,
                                          const char* trow, const char* qrow, bool residual,
                                          int seg, int g0, int g1,
                                          const unsigned long long* best) {
  constexpr int VEC = Lanes<DT>::VEC, QV = 32 / VEC;
  const int lane = threadIdx.x & 31;
  const int v0 = seg * kSegVecs + lane;
  unsigned long long bk = *(const volatile unsigned long long*)best;
  double K = bk ? from_ordered_u64(bk) : -INFINITY;
  Best B{-INFINITY, -INFINITY, -1};
#pragma unroll 1
  for (int gi = g0; gi < g1; ++gi) {
    uint4 cur[QV];
    load_part<DT>(a, trow, seg, gi * QV, cur);
    if (!(K > -INFINITY)) {
      float mv = -INFINITY;
      int xi = -1;
#pragma unroll
      for (int j = 0; j < QV; ++j)
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          const float z = elem<DT>(cur[j], e);
          if (z > mv) {
            mv = z;
            xi = (v0 + 32 * (gi * QV + j)) * VEC + e;
          }
        }
      double k = -INFINITY;
      if (xi >= 0 && xi < a.V) k = exact_key_of(a, rd, trow, qrow, residual, xi);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) k = fmax(k, __shfl_xor_sync(0xFFFFFFFFu, k, o));
      K = k;
    }
    const float cup = filter_offset(K, rd.lse_t);
    const float thr2 = K > -INFINITY ? __double2float_rd((K - kRaceBand) * 1.4426950408889634 - 1e-5)
                                     : -INFINITY;
    uint32_t keep = ~word_filter_compact<DT>(cur, gi * QV, seed_of(a), rd.g,
                                             (uint32_t)a.vocab_offset >> 2, v0, rd.k2, cup);
    // exact keys of the survivors, one token per lane at a time
    while (__any_sync(0xFFFFFFFFu, keep != 0u)) {
      if (keep) {
        const int t = __clz((int)keep);
        keep &= ~(0x80000000u >> t);
        const int x = (v0 + 32 * (gi * QV + t / VEC)) * VEC + t % VEC;
        if (x < a.V && key2_upper(row_ctx(a), rd, trow, qrow, residual, x) >= thr2)
          offer(B, exact_key_of(a, rd, trow, qrow, residual, x), x);
      }
    }
    if (gi + 1 < g1) {
      double wb = B.best;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) wb = fmax(wb, __shfl_xor_sync(0xFFFFFFFFu, wb, o));
      bk = *(const volatile unsigned long long*)best;
      K = fmax(K, fmax(wb, bk ? from_ordered_u64(bk) : -INFINITY));
    }
  }
  return warp_combine(B);
}

template <int DT>
__device__ __noinline__ Best race_segment(const RowCtx a, const RaceDesc& rd,
                                          const char* trow, const char* qrow, bool residual,
                                          int seg, double K0, float cup) {
  return race_segment_in<DT>(a, rd, race_stream(seed_of(a), rd.g, (uint32_t)a.vocab_offset >> 2), trow, qrow, residual, seg, K0, cup);
}

// A quick approximate key (natural-log units) with the hardware's approximate
// exp and log; it only ranks tokens in the search for a reference key.
__device__ __forceinline__ float approx_key_fast(float zt, float zq, uint32_t o, float invT,
                                                 float lse_t, float lse_q, bool residual) {
  const float lp = zt * invT - lse_t;
  float lr = lp;
  if (residual) {
    const float lq = zq * invT - lse_q;
    lr = lq < lp ? lp + __logf(1.0f - __expf(lq - lp)) : -INFINITY;
  }
  const float W = ((float)o + 0.5f) * 0x1p-32f;
  const float E = fmaxf(W, -__logf(1.0f - W));  // E >= W always holds
  return lr - __logf(E);
}

// A reference key for the race of rd (request b), by one warp among nw: the
// warp ranks its share of the 16-byte vectors of segment `seg` of the sampled
// row (vectors warp*32 + lane, + 32 nw, ...) by approximate key and returns
// the exact key of its best token (the same on every lane); -inf if none.
template <int DT>
__device__ __forceinline__ double race_ref_key_warp(const VerifyArgs& a, const RaceDesc& rd,
                                                    const RaceStream& R, int b, int seg,
                                                    int warp, int nw) {
  constexpr int VEC = Lanes<DT>::VEC;
  const int lane = threadIdx.x & 31;
  const bool residual = rd.kind == kRaceResidual;
  const char* trow = row_base(a, b, rd.n);
  const char* qrow = residual ? row_base(a, b, a.D_max + 1 + rd.n) : nullptr;
  const int nfull = a.V / VEC;
  const bool aligned =
      ((uintptr_t)trow & 15u) == 0 && (!residual || ((uintptr_t)qrow & 15u) == 0);
  const float invT = (float)(1.0 / rd.T), lse_t = (float)rd.lse_t;
  const float lse_q = (float)(rd.lse_q + rd.ln_Z);
  float best = -INFINITY;
  int bx = INT_MAX;
  const int vend = min(a.nvec, (seg + 1) * kSegVecs);
  for (int v = seg * kSegVecs + 32 * warp + lane; v < vend; v += 32 * nw) {
    const uint4 wt = load_vec_checked<DT>(trow, v, a.V, a.nvec, nfull, aligned);
    uint4 wq = make_uint4(0u, 0u, 0u, 0u);
    if (residual) wq = load_vec_checked<DT>(qrow, v, a.V, a.nvec, nfull, aligned);
#pragma unroll
    for (int h = 0; h < VEC / 4; ++h) {
      const uint4 o4 = race_words_fast(R, (uint32_t)(v * VEC + 4 * h) >> 2);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int x = v * VEC + 4 * h + e;
        const float zt = elem<DT>(wt, 4 * h + e);
        const uint32_t o = e == 0 ? o4.x : e == 1 ? o4.y : e == 2 ? o4.z : o4.w;
        const float k = approx_key_fast(zt, residual ? elem<DT>(wq, 4 * h + e) : 0.0f, o, invT,
                                        lse_t, lse_q, residual);
        if (x < a.V && zt > -INFINITY && k > best) {
          best = k;
          bx = x;
        }
      }
    }
  }
  // the warp's best (ties: the lower index), then its exact key on every lane
  const unsigned long long w = warp_max_u64(value_index_key(best, bx));
  const int x = key_index(w);
  if (x == INT_MAX || !(key_value(w) > -INFINITY)) return -INFINITY;
  return exact_key_of(a, rd, trow, qrow, residual, x);
}

}  // namespace sv
