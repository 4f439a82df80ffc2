// row_stats.cu -- per-row statistics, the bandwidth-bound pass of the step.
//
// For every row the rule reads (target rows 0..D_b, draft rows 0..D_b-1 of
// non-greedy requests) this computes, per 32 KiB chunk, the partial
// log-sum-exp state of softmax(z / T), the lowest-index argmax (target rows)
// and the k largest logits (saguaro draft rows).  The accept scan merges the
// chunks of a row in chunk order in double precision.
//
// Sources: "Accélérer Sonar par la Spéculation", section "Cible-Brouillon"
// (the sampler compares the full draft and target distributions, so both
// normalisers are needed); "Speculative Speculative Decoding – асинхронизируй
// это.", saguaro recipe item 1 (the draft's top tokens).
//
// Design: one CTA of 256 threads per (row, chunk); each thread issues its eight
// 16-byte loads at once (32 KiB in flight per CTA), takes its maximum on packed
// bf16 pairs, the CTA agrees on the chunk maximum, and then every element costs
// one FFMA and one ex2 relative to that maximum -- no per-element rescaling.
#include "sv_common.cuh"

#include <float.h>
#include <limits.h>

namespace sv {

namespace {

constexpr uint32_t kNegInfBf2 = 0xFF80FF80u;  // two bf16 -inf
constexpr uint32_t kNegInfF32 = 0xFF800000u;

template <int DT>
__device__ __forceinline__ uint4 load_vec(const char* row, int v, int V, int nvec, int nfull,
                                          bool aligned) {
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

template <int DT, bool LSE, bool ARGMAX, bool TOP>
__device__ __forceinline__ void stats_chunk(const VerifyArgs& a, const char* row, int chunk,
                                            float k2, int topk, ChunkStat* out) {
  constexpr int VEC = DT == kF32 ? 4 : 8;
  __shared__ float s_max[kThreads / 32];
  __shared__ uint32_t s_bad[kThreads / 32];
  __shared__ float s_sum[kThreads / 32];
  __shared__ int s_idx[kThreads / 32];
  __shared__ unsigned long long s_key[kThreads / 32];
  __shared__ unsigned long long s_win;

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int V = a.V, nvec = a.nvec, nfull = V / VEC;
  const bool aligned = ((uintptr_t)row & 15u) == 0;
  const int v0 = chunk * kChunkVecs + t;

  uint4 raw[kVecsPerThread];
#pragma unroll
  for (int j = 0; j < kVecsPerThread; ++j)
    raw[j] = load_vec<DT>(row, v0 + j * kThreads, V, nvec, nfull, aligned);

  // ---- thread maximum, with NaN / +inf detection
  float m_t;
  uint32_t bad = 0;
  if (DT == kBF16) {
    __nv_bfloat162 mx = as_bf2(raw[0].x);
#pragma unroll
    for (int j = 0; j < kVecsPerThread; ++j) {
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
    for (int j = 0; j < kVecsPerThread; ++j)
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        const float z = elem<DT>(raw[j], e);
        bad |= (z != z) | (z == INFINITY);
        m_t = fmaxf(m_t, z);
      }
  }

  // ---- chunk maximum (every thread computes it from the warp maxima in a fixed order)
  {
    const float wm = warp_max(m_t);
    const uint32_t wb = __any_sync(0xFFFFFFFFu, bad) ? 1u : 0u;
    if (lane == 0) {
      s_max[warp] = wm;
      s_bad[warp] = wb;
    }
  }
  __syncthreads();
  float m_c = s_max[0];
  uint32_t bad_c = s_bad[0];
#pragma unroll
  for (int w = 1; w < kThreads / 32; ++w) {
    m_c = fmaxf(m_c, s_max[w]);
    bad_c |= s_bad[w];
  }

  // ---- sum of 2^(z*k2 - mk): one FFMA and one ex2 per element
  float S_t = 0.0f;
  const float mk = m_c * k2;
  if (LSE && m_c > -INFINITY) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
    for (int j = 0; j < kVecsPerThread; ++j)
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        const float z = elem<DT>(raw[j], e);
        acc[(j * VEC + e) & 7] += ex2_approx(fmaf(z, k2, -mk));
      }
    S_t = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
  }

  // ---- lowest index of the chunk maximum (only threads holding it search)
  int idx_t = INT_MAX;
  if (ARGMAX && m_t == m_c) {
#pragma unroll
    for (int j = kVecsPerThread - 1; j >= 0; --j)
#pragma unroll
      for (int e = VEC - 1; e >= 0; --e)
        if (elem<DT>(raw[j], e) == m_c) idx_t = (v0 + j * kThreads) * VEC + e;
  }

  if (LSE || ARGMAX) {
    const float ws = LSE ? warp_sum(S_t) : 0.0f;
    const int wi = ARGMAX ? warp_min_int(idx_t) : INT_MAX;
    if (lane == 0) {
      s_sum[warp] = ws;
      s_idx[warp] = wi;
    }
  }

  // ---- the k largest logits (value desc, index asc), saguaro draft rows
  float tv[kMaxTopK];
  int ti[kMaxTopK];
  if (TOP) {
#pragma unroll
    for (int s = 0; s < kMaxTopK; ++s) {
      tv[s] = -INFINITY;
      ti[s] = INT_MAX;
    }
#pragma unroll
    for (int j = 0; j < kVecsPerThread; ++j)
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        const float z = elem<DT>(raw[j], e);
        if (z > tv[kMaxTopK - 1]) {
          // elements arrive in increasing index order, so an equal value stays
          // below the earlier (lower-index) one: strict comparisons throughout
          tv[kMaxTopK - 1] = z;
          ti[kMaxTopK - 1] = (v0 + j * kThreads) * VEC + e;
#pragma unroll
          for (int s = kMaxTopK - 1; s > 0; --s) {
            if (tv[s] > tv[s - 1]) {
              const float fv = tv[s];
              tv[s] = tv[s - 1];
              tv[s - 1] = fv;
              const int fi = ti[s];
              ti[s] = ti[s - 1];
              ti[s - 1] = fi;
            }
          }
        }
      }
  }
  __syncthreads();

  if (TOP) {
    int h = 0;
    for (int r = 0; r < topk; ++r) {
      float hv = -INFINITY;
      int hi = INT_MAX;
#pragma unroll
      for (int s = 0; s < kMaxTopK; ++s)
        if (s == h) {
          hv = tv[s];
          hi = ti[s];
        }
      const unsigned long long key = hi == INT_MAX ? 0ull : value_index_key(hv, hi);
      const unsigned long long wk = warp_max_u64(key);
      if (lane == 0) s_key[warp] = wk;
      __syncthreads();
      if (t == 0) {
        unsigned long long best = s_key[0];
        for (int w = 1; w < kThreads / 32; ++w) best = s_key[w] > best ? s_key[w] : best;
        s_win = best;
      }
      __syncthreads();
      const unsigned long long win = s_win;
      if (win != 0ull && key == win) ++h;
      if (t == 0) {
        out->topv[r] = win ? key_value(win) : -INFINITY;
        out->topi[r] = win ? key_index(win) : INT_MAX;
      }
      __syncthreads();
    }
  }

  if (t == 0) {
    float S = 0.0f;
    int am = INT_MAX;
    if (LSE)
      S = ((s_sum[0] + s_sum[1]) + (s_sum[2] + s_sum[3])) +
          ((s_sum[4] + s_sum[5]) + (s_sum[6] + s_sum[7]));
    if (ARGMAX) {
      am = s_idx[0];
      for (int w = 1; w < kThreads / 32; ++w) am = min(am, s_idx[w]);
    }
    out->m = m_c;
    out->mk = LSE ? mk : -INFINITY;
    out->S = S;
    out->argmax = am;
    out->bad = bad_c;
    out->ntop = TOP ? topk : 0;
  }
}

template <int DT>
__global__ void __launch_bounds__(kThreads) row_stats_kernel(VerifyArgs a) {
  const int chunk = blockIdx.x % a.nch;
  const int rest = blockIdx.x / a.nch;
  const int slot = rest % a.slots;
  const int b = rest / a.slots;
  const ReqParams rp = load_req(a, b);
  if (rp.err) return;  // reported by the accept scan
  const bool is_target = slot <= a.D_max;
  const int d = is_target ? slot : slot - a.D_max - 1;
  if (is_target ? d > rp.Db : (d >= rp.Db || rp.mode == kGreedy)) return;  // row not read
  const char* row = row_base(a, b, slot);
  ChunkStat* out = a.cstat + ((size_t)b * a.slots + slot) * a.nch + chunk;
  const float k2 = rp.mode == kGreedy ? 0.0f : (float)(1.4426950408889634 / (double)rp.T);
  if (is_target) {
    if (rp.mode == kGreedy)
      stats_chunk<DT, false, true, false>(a, row, chunk, k2, 0, out);
    else
      stats_chunk<DT, true, true, false>(a, row, chunk, k2, 0, out);
  } else if (rp.mode == kSaguaro) {
    stats_chunk<DT, true, false, true>(a, row, chunk, k2, a.saguaro_k, out);
  } else {
    stats_chunk<DT, true, false, false>(a, row, chunk, k2, 0, out);
  }
}

}  // namespace

cudaError_t launch_row_stats(const VerifyArgs& a, cudaStream_t s) {
  const long long grid = (long long)a.B * a.slots * a.nch;
  if (grid == 0) return cudaSuccess;
  if (a.dtype == kF32)
    row_stats_kernel<kF32><<<(unsigned)grid, kThreads, 0, s>>>(a);
  else
    row_stats_kernel<kBF16><<<(unsigned)grid, kThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace sv
