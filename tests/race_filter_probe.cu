// Test helper: for every token of one target row (and draft row), the race's
// word-filter decision for a given reference key K0, the token's Philox race
// word, the single-precision upper bound of its key (key2_upper, log2 units)
// and its exact double-precision key (exact_key_of), so that a test can check
// that the filter keeps every token whose key reaches K0 - 1e-6 and drops the
// rest up to its documented slack, and that the bound is one.
#include "race_device.cuh"

using namespace sv;

template <int DT>
__device__ void probe_segment(const VerifyArgs& a, const RaceDesc& rd, const char* trow,
                              const char* qrow, bool residual, int seg, float cup,
                              unsigned char* keep_out, unsigned* words, double* exact,
                              float* upper) {
  constexpr int VEC = Lanes<DT>::VEC, QV = 32 / VEC, NG = kLaneVecs / QV;
  const int v0 = seg * kSegVecs + (threadIdx.x & 31);
  const RaceStream R = race_stream(a.seed, rd.g);
  for (int gi = 0; gi < NG; ++gi) {
    uint4 raw[QV];
    load_part<DT>(a, trow, seg, gi * QV, raw);
    const uint32_t drop = word_filter<DT>(raw, gi * QV, R, v0, rd.k2, cup);
    for (int t = 0; t < 32; ++t) {
      const int x = (v0 + 32 * (gi * QV + t / VEC)) * VEC + t % VEC;
      if (x >= a.V) continue;
      keep_out[x] = ((drop >> (31 - t)) & 1u) ? 0 : 1;
      words[x] = race_word(a.seed, rd.g, x);
      exact[x] = exact_key_of(a, rd, trow, qrow, residual, x);
      upper[x] = key2_upper(row_ctx(a), rd, trow, qrow, residual, x);
    }
  }
}

__global__ void probe_kernel(VerifyArgs a, RaceDesc rd, const char* trow, const char* qrow,
                             int residual, float cup, unsigned char* keep, unsigned* words,
                             double* exact, float* upper) {
  const int warp = threadIdx.x >> 5;
  const int seg = blockIdx.x * (blockDim.x >> 5) + warp;
  if (seg >= a.nseg) return;
  if (a.dtype == kF32)
    probe_segment<kF32>(a, rd, trow, qrow, residual != 0, seg, cup, keep, words, exact, upper);
  else
    probe_segment<kBF16>(a, rd, trow, qrow, residual != 0, seg, cup, keep, words, exact, upper);
}

__global__ void offset_kernel(double K0, double lse_t, float T, float* out) {
  out[0] = filter_offset(K0, lse_t);
  out[1] = log2e_over_T(T);
}

// All pointers but top and cup_out are device pointers; lse values are
// natural-log LSEs at T.  cup_out (host) receives the filter offset used.
extern "C" int race_filter_probe(const void* trow, const void* qrow, int V, int dtype, float T,
                                 double lse_t, double lse_q, int ntop, const int* top,
                                 double ln_c, double ln_Z, unsigned long long seed, unsigned g,
                                 int residual, double K0, unsigned char* keep, unsigned* words,
                                 double* exact, float* upper, float* cup_out) {
  VerifyArgs a;
  memset(&a, 0, sizeof a);
  a.V = V;
  a.dtype = dtype;
  row_geometry(V, dtype, &a.nvec, &a.nseg);
  a.seed = seed;
  RaceDesc rd;
  memset(&rd, 0, sizeof rd);
  rd.kind = residual ? kRaceResidual : kRaceBonus;
  rd.g = g;
  rd.T = (double)T;
  rd.lse_t = lse_t;
  rd.lse_q = lse_q;
  rd.ln_c = ln_c;
  rd.ln_Z = ln_Z;
  rd.ntop = ntop;
  for (int i = 0; i < ntop; ++i) rd.top[i] = top[i];
  // the filter offset and k2 exactly as the library computes them
  float* d_out = nullptr;
  if (cudaMalloc(&d_out, 2 * sizeof(float)) != cudaSuccess) return 1;
  offset_kernel<<<1, 1>>>(K0, lse_t, T, d_out);
  float h[2] = {0.0f, 0.0f};
  if (cudaMemcpy(h, d_out, sizeof h, cudaMemcpyDeviceToHost) != cudaSuccess) return 1;
  cudaFree(d_out);
  const float cup = h[0];
  rd.k2 = h[1];
  *cup_out = cup;
  probe_kernel<<<(a.nseg + 7) / 8, 256>>>(a, rd, (const char*)trow, (const char*)qrow, residual,
                                          cup, keep, words, exact, upper);
  return cudaDeviceSynchronize() == cudaSuccess ? 0 : 1;
}
