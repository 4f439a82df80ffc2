// stats_device.cuh -- device code of the per-row statistics pass, shared by the
// split row_stats kernel and the fused kernel.
//
// For every row the rule reads (target rows 0..D_b, draft rows 0..D_b-1 of
// non-greedy requests) one warp computes, per 8 KiB segment, the partial
// log-sum-exp state of softmax(z / T), the lowest-index argmax (target rows)
// and the k largest logits (saguaro draft rows).
//
// Sources: "Accélérer Sonar par la Spéculation", section "Cible-Brouillon"
// (the sampler compares the full draft and target distributions, so both
// normalisers are needed); "Speculative Speculative Decoding – асинхронизируй
// это.", saguaro recipe item 1 (the draft's top tokens).
//
// Each lane issues its sixteen 16-byte loads at once (8 KiB in flight per
// warp), takes its maximum on packed bf16 pairs, the warp agrees on the segment
// maximum with five shuffles, and then every pair of elements costs one packed
// FFMA, two ex2 and one packed FADD relative to that maximum -- no per-element
// rescaling, no barrier, no shared memory.
#pragma once
#include "sv_common.cuh"

#include <float.h>
#include <limits.h>

#include <type_traits>

namespace sv {

constexpr uint32_t kNegInfBf2 = 0xFF80FF80u;  // two bf16 -inf
constexpr uint32_t kNegInfF32 = 0xFF800000u;

// Vector v of a row (VEC elements), -inf past V; element loads where the row
// is not 16-byte aligned or the vector crosses the end of the row.
template <int DT>
__device__ __forceinline__ uint4 load_vec_checked(const char* row, int v, int V, int nvec,
                                                  int nfull, bool aligned) {
  const uint32_t fill = DT == kF32 ? kNegInfF32 : kNegInfBf2;
  if (v >= nvec) return make_uint4(fill, fill, fill, fill);
  if (aligned && v < nfull) return ld_stream16(row + (size_t)v * 16);
  uint32_t w[4];
  if (DT == kF32) {
    const float* r = (const float*)row;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int x = v * 4 + e;
      w[e] = x < V ? __float_as_uint(r[x]) : kNegInfF32;
    }
  } else {
    const uint16_t* r = (const uint16_t*)row;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int x = v * 8 + 2 * e;
      const uint32_t lo = x < V ? (uint32_t)r[x] : 0xFF80u;
      const uint32_t hi = x + 1 < V ? (uint32_t)r[x + 1] : 0xFF80u;
      w[e] = lo | (hi << 16);
    }
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ __nv_bfloat162 as_bf2(uint32_t w) {
  __nv_bfloat162 r;
  memcpy(&r, &w, 4);
  return r;
}

__device__ __forceinline__ uint32_t word(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// Element e (0..VEC-1) of a loaded vector, widened to float.
template <int DT>
__device__ __forceinline__ float elem(const uint4& v, int e) {
  if (DT == kF32) return __uint_as_float(word(v, e));
  const uint32_t w = word(v, e >> 1);
  return (e & 1) ? bf_hi(w) : bf_lo(w);
}

// Load the lane's kLaneVecs vectors of segment `seg` of a row of V elements
// (nvec vectors).
template <int DT>
__device__ __forceinline__ void load_segment_v(const char* row, int V, int nvec, int seg,
                                               uint4 (&raw)[kLaneVecs]) {
  constexpr int VEC = DT == kF32 ? 4 : 8;
  const int lane = threadIdx.x & 31;
  const int nfull = V / VEC;
  const int v0 = seg * kSegVecs + lane;
  const bool aligned = ((uintptr_t)row & 15u) == 0;
  if (aligned && (seg + 1) * kSegVecs <= nfull) {
    // whole segment inside the row: unchecked streaming loads
#pragma unroll
    for (int j = 0; j < kLaneVecs; ++j) raw[j] = ld_stream16(row + (size_t)(v0 + 32 * j) * 16);
  } else {
#pragma unroll
    for (int j = 0; j < kLaneVecs; ++j)
      raw[j] = load_vec_checked<DT>(row, v0 + 32 * j, V, nvec, nfull, aligned);
  }
}

template <int DT>
__device__ __forceinline__ void load_segment(const VerifyArgs& a, const char* row, int seg,
                                             uint4 (&raw)[kLaneVecs]) {
  load_segment_v<DT>(row, a.V, a.nvec, seg, raw);
}

// "Largest value, then lowest index" keys in 32 bits for bf16 values and
// indices below 2^16 (the top half of the value's order-preserving bits, then
// the complemented index), so that one hardware warp reduction finds the
// maximum; 0 is below every real key.
__device__ __forceinline__ uint32_t value_index_key32(float v, int idx) {
  return (ordered_bits(v) & 0xFFFF0000u) | (0xFFFFu - (uint32_t)idx);
}

__device__ __forceinline__ float key32_value(uint32_t k) {
  const uint32_t o = k >> 16;
  const uint32_t b = (o & 0x8000u) ? (o & 0x7FFFu) : (~o & 0xFFFFu);
  return __uint_as_float(b << 16);
}

__device__ __forceinline__ int key32_index(uint32_t k) { return (int)(0xFFFFu - (k & 0xFFFFu)); }

// Statistics of one segment whose lane vectors are raw[0..kLaneVecs-1] (the
// vectors seg*kSegVecs + lane + 32 j of the row, -inf past its end), by one
// full warp; row (V elements) is read again only by the top list, rarely.
template <int DT, bool LSE, bool ARGMAX, bool TOP>
__device__ __forceinline__ void stats_reduce(const uint4 (&raw)[kLaneVecs], const char* row,
                                             int V, int seg, float k2, int topk, PartStat* out,
                                             TopPart* tout, int off = 0) {
  constexpr int VEC = DT == kF32 ? 4 : 8;
  const int lane = threadIdx.x & 31;
  const int v0 = seg * kSegVecs + lane;
  // ---- lane maximum, with NaN / +inf detection
  float m_t;
  uint32_t bad = 0;
  if (DT == kBF16) {
    __nv_bfloat162 mx = as_bf2(raw[0].x);
#pragma unroll
    for (int j = 0; j < kLaneVecs; ++j) {
      mx = __hmax2_nan(mx, as_bf2(raw[j].x));
      mx = __hmax2_nan(mx, as_bf2(raw[j].y));
      mx = __hmax2_nan(mx, as_bf2(raw[j].z));
      mx = __hmax2_nan(mx, as_bf2(raw[j].w));
    }
    const float lo = __low2float(mx), hi = __high2float(mx);
    bad = (lo != lo) | (hi != hi) | (lo == INFINITY) | (hi == INFINITY);
    m_t = fmaxf(lo, hi);
  } else {
    m_t = -INFINITY;
#pragma unroll
    for (int j = 0; j < kLaneVecs; ++j)
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        const float z = elem<DT>(raw[j], e);
        bad |= (z != z) | (z == INFINITY);
        m_t = fmaxf(m_t, z);
      }
  }
  const float m_w = warp_max(m_t);
  const uint32_t bad_w = __any_sync(0xFFFFFFFFu, bad) ? 1u : 0u;

  // ---- sum of 2^(z*k2 - mk): per pair of elements one packed FFMA, two ex2 and
  // one packed FADD (fixed accumulation order: four float2 accumulators)
  float S_w = 0.0f;
  if (LSE) {
    float S_t = 0.0f;
    if (m_w > -INFINITY) {
      const float mk = m_w * k2;
      const float2 kk = make_float2(k2, k2), nm = make_float2(-mk, -mk);
      float2 acc[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int j = 0; j < kLaneVecs; ++j)
#pragma unroll
        for (int e = 0; e < VEC; e += 2) {
          const float2 t = __ffma2_rn(make_float2(elem<DT>(raw[j], e), elem<DT>(raw[j], e + 1)), kk, nm);
          const int q = ((j * VEC + e) >> 1) & 3;
          acc[q] = __fadd2_rn(acc[q], make_float2(ex2_approx(t.x), ex2_approx(t.y)));
        }
      const float2 s01 = __fadd2_rn(acc[0], acc[1]), s23 = __fadd2_rn(acc[2], acc[3]);
      const float2 s = __fadd2_rn(s01, s23);
      S_t = s.x + s.y;
    }
    S_w = warp_sum(S_t);
  }

  // ---- lowest index of the segment maximum (only lanes holding it search)
  int idx_w = INT_MAX;
  if (ARGMAX) {
    int idx_t = INT_MAX;
    if (m_t == m_w) {
#pragma unroll
      for (int j = kLaneVecs - 1; j >= 0; --j)
#pragma unroll
        for (int e = VEC - 1; e >= 0; --e)
          if (elem<DT>(raw[j], e) == m_w) idx_t = (v0 + 32 * j) * VEC + e;
    }
    idx_w = warp_min_int(idx_t);
  }

  // ---- the k largest logits (value desc, index asc), saguaro draft rows.
  // The k largest lane maxima are k distinct elements, so every element of the
  // segment's top k is at least T, the k-th largest lane maximum.  Only the
  // lanes holding the k largest maxima (barring ties) have vectors whose
  // largest element reaches T, mostly just one: a branch-free pass marks them,
  // and those lanes read their marked vectors again, all at once, one 16-byte
  // load each (L2 hits: the segment has just been streamed), inserting their
  // elements >= T into a list of the 8 largest "value, then lower index" keys
  // (sorted by a branch-free max/min network; 32-bit keys for bf16: value bits
  // and the index within the segment).  An element of the segment's top k is
  // in its own lane's top k, which the list keeps; k rounds of a warp maximum
  // then merge the lists.
  if (TOP) {
    using Key = typename std::conditional<DT == kBF16, uint32_t, unsigned long long>::type;
    float T = -INFINITY;
    if constexpr (DT == kBF16) {
      uint32_t mine = value_index_key32(m_t, lane);
      for (int r = 0; r < topk; ++r) {
        const uint32_t win = __reduce_max_sync(0xFFFFFFFFu, mine);
        T = key32_value(win);
        if (mine == win) mine = 0u;  // each lane maximum counts once
      }
    } else {
      unsigned long long mine = value_index_key(m_t, lane);
      for (int r = 0; r < topk; ++r) {
        const unsigned long long win = warp_max_u64(mine);
        T = key_value(win);
        if (mine == win) mine = 0ull;  // each lane maximum counts once
      }
    }
    uint32_t mark = 0u;  // bit 31 - j: vector j of the lane
#pragma unroll
    for (int j = 0; j < kLaneVecs; ++j) {
      float vm;
      if (DT == kBF16) {
        const __nv_bfloat162 p = __hmax2(__hmax2(as_bf2(raw[j].x), as_bf2(raw[j].y)),
                                         __hmax2(as_bf2(raw[j].z), as_bf2(raw[j].w)));
        vm = fmaxf(__low2float(p), __high2float(p));
      } else {
        vm = fmaxf(fmaxf(elem<DT>(raw[j], 0), elem<DT>(raw[j], 1)),
                   fmaxf(elem<DT>(raw[j], 2), elem<DT>(raw[j], 3)));
      }
      const uint32_t hit = (vm >= T && vm > -INFINITY) ? 0x80000000u : 0u;
      mark = __funnelshift_l(hit, mark, 1);
    }
    mark <<= (32 - kLaneVecs);
    Key lk[kMaxTopK];
#pragma unroll
    for (int q = 0; q < kMaxTopK; ++q) lk[q] = 0;
    // the marked vectors again, each with one 16-byte load (the segment has
    // just been streamed through L2), two at a time
    const int nvec = (V + VEC - 1) / VEC, nfull = V / VEC;
    const bool aligned = ((uintptr_t)row & 15u) == 0;
#pragma unroll 1
    while (mark) {
      const int ja = __clz((int)mark);
      mark &= ~(0x80000000u >> ja);
      const int jb = mark ? __clz((int)mark) : -1;
      if (jb >= 0) mark &= ~(0x80000000u >> jb);
      const uint4 wa = load_vec_checked<DT>(row, v0 + 32 * ja, V, nvec, nfull, aligned);
      const uint4 wb = jb >= 0 ? load_vec_checked<DT>(row, v0 + 32 * jb, V, nvec, nfull, aligned)
                               : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll 1
      for (int t = 0; t < 2 * VEC; ++t) {
        const int j = t < VEC ? ja : jb;
        if (j < 0) break;
        const int e = t < VEC ? t : t - VEC;
        const float z = elem<DT>(t < VEC ? wa : wb, e);
        if (z >= T && z > -INFINITY) {
          Key k;
          if constexpr (DT == kBF16) k = value_index_key32(z, (lane + 32 * j) * VEC + e);
          else k = value_index_key(z, (lane + 32 * j) * VEC + e);
#pragma unroll
          for (int q = 0; q < kMaxTopK; ++q) {
            const Key hi = lk[q] > k ? lk[q] : k;
            k = lk[q] > k ? k : lk[q];
            lk[q] = hi;
          }
        }
      }
    }
    const int base = seg * kSegVecs * VEC;  // indices in the keys are relative to it
    int h = 0;
    for (int r = 0; r < topk; ++r) {
      Key mine = 0;
#pragma unroll
      for (int q = 0; q < kMaxTopK; ++q)
        if (q == h) mine = lk[q];
      if constexpr (DT == kBF16) {
        const uint32_t win = __reduce_max_sync(0xFFFFFFFFu, mine);
        if (win != 0u && mine == win) ++h;
        if (lane == 0) {
          tout->v[r] = win ? key32_value(win) : -INFINITY;
          tout->i[r] = win ? off + base + key32_index(win) : INT_MAX;
        }
      } else {
        const unsigned long long win = warp_max_u64(mine);
        if (win != 0ull && mine == win) ++h;
        if (lane == 0) {
          tout->v[r] = win ? key_value(win) : -INFINITY;
          tout->i[r] = win ? off + base + key_index(win) : INT_MAX;
        }
      }
    }
  }

  if (lane == 0) {
    PartStat p;
    p.m = m_w;
    p.S = S_w;
    p.argmax = idx_w == INT_MAX ? INT_MAX : off + idx_w;  // global index
    p.bad = bad_w;
    *out = p;
  }
}

// Statistics of segment `seg` of one row, by one full warp, loading through registers.
template <int DT, bool LSE, bool ARGMAX, bool TOP>
__device__ __forceinline__ void stats_segment(const VerifyArgs& a, const char* row, int seg,
                                              float k2, int topk, PartStat* out, TopPart* tout) {
  uint4 raw[kLaneVecs];
  load_segment<DT>(a, row, seg, raw);
  stats_reduce<DT, LSE, ARGMAX, TOP>(raw, row, a.V, seg, k2, topk, out, tout, a.vocab_offset);
}

// The statistics of a saguaro draft-row segment (with its top list), compiled
// on its own so that the common path keeps its registers.
// It takes scalars, not the argument block: a reference to that would make
// every thread copy it to its stack at each call.
template <int DT>
__device__ __noinline__ void stats_segment_top(const char* row, int V, int nvec, int seg, float k2,
                                               int topk, int off, PartStat* out, TopPart* tout) {
  uint4 raw[kLaneVecs];
  load_segment_v<DT>(row, V, nvec, seg, raw);
  stats_reduce<DT, true, false, true>(raw, row, V, seg, k2, topk, out, tout, off);
}

// Whether row `slot` of a request with parameters rp is read by the rule.
__device__ __forceinline__ bool row_needed(const VerifyArgs& a, int b, int slot, const ReqParams& rp) {
  return row_read(a, b, slot, rp);
}

// Statistics of segment `seg` of row `slot` of request b (one full warp).
// WITH_TOP: the batch may hold saguaro requests (their draft rows need the top
// list); the launcher compiles the pass both ways and picks by the batch, so
// the common path carries no code for it.  A saguaro row met without it is a
// launcher error, reported as a bad parameter.
template <int DT, bool WITH_TOP>
__device__ __forceinline__ void stats_item(const VerifyArgs& a, int b, int slot, int seg,
                                           const ReqParams& rp) {
  const bool is_target = slot <= a.D_max;
  const char* row = row_base(a, b, slot);
  PartStat* out = a.pstat + ((size_t)b * a.slots + slot) * a.nseg + seg;
  const float k2 = rp.mode == kGreedy ? 0.0f : log2e_over_T(rp.T);
  if (is_target) {
    // the argmax is only used by greedy requests
    if (rp.mode == kGreedy)
      stats_segment<DT, false, true, false>(a, row, seg, k2, 0, out, nullptr);
    else
      stats_segment<DT, true, false, false>(a, row, seg, k2, 0, out, nullptr);
  } else if (rp.mode == kSaguaro) {
    if (WITH_TOP) {
      TopPart* tout = a.tpart + ((size_t)b * a.D_max + (slot - a.D_max - 1)) * a.nseg + seg;
      stats_segment_top<DT>(row, a.V, a.nvec, seg, k2, a.saguaro_k, a.vocab_offset, out, tout);
    } else if ((threadIdx.x & 31) == 0) {
      atomicOr(a.status, kFlagBadParam);
    }
  } else {
    stats_segment<DT, true, false, false>(a, row, seg, k2, 0, out, nullptr);
  }
}

// (b, slot, seg) of work item `it` of the request-major item order, advanced
// in steps of `stride` items without divisions.
struct ItemWalker {
  int b, slot, seg;
  int d_b, d_slot, d_seg;  // the stride decomposed the same way
  __device__ __forceinline__ void init(const VerifyArgs& a, unsigned it, unsigned stride) {
    const unsigned per_req = (unsigned)a.slots * (unsigned)a.nseg;
    b = (int)(it / per_req);
    const unsigned r = it % per_req;
    slot = (int)(r / (unsigned)a.nseg);
    seg = (int)(r % (unsigned)a.nseg);
    d_b = (int)(stride / per_req);
    const unsigned dr = stride % per_req;
    d_slot = (int)(dr / (unsigned)a.nseg);
    d_seg = (int)(dr % (unsigned)a.nseg);
  }
  __device__ __forceinline__ void advance(const VerifyArgs& a) {
    seg += d_seg;
    int carry = 0;
    if (seg >= a.nseg) {
      seg -= a.nseg;
      carry = 1;
    }
    slot += d_slot + carry;
    carry = 0;
    if (slot >= a.slots) {
      slot -= a.slots;
      carry = 1;
    }
    b += d_b + carry;
  }
};

// The statistics pass: warp w0 of W walks the (request, row, segment) items
// w0, w0 + W, w0 + 2W, ... in request-major order, so that at any moment the
// device streams one contiguous stretch of the logits.  Rows the rule does not
// read are skipped (parameter errors are reported by the scan).
template <int DT, bool WITH_TOP>
__device__ __forceinline__ void stats_pass(const VerifyArgs& a, unsigned w0, unsigned W) {
  const unsigned total = (unsigned)a.B * (unsigned)a.slots * (unsigned)a.nseg;
  if (w0 >= total) return;
  ItemWalker it;
  it.init(a, w0, W);
  for (unsigned i = w0; i < total; i += W, it.advance(a)) {
    const ReqParams rp = load_req(a, it.b);
    if (!row_needed(a, it.b, it.slot, rp)) continue;
    stats_item<DT, WITH_TOP>(a, it.b, it.slot, it.seg, rp);
  }
}

}  // namespace sv
