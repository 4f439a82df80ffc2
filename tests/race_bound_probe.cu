// Test helper: for every token of one target row (and draft row), the race's
// single-precision key bound (race_bounds) and its exact double-precision key
// (exact_key_of), so that a test can check bound >= exact * log2(e) everywhere.
#include "race_device.cuh"

using namespace sv;

template <int DT, bool RES, bool SAG>
__device__ void probe_segment(const VerifyArgs& a, const RaceDesc& rd, const char* trow,
                              const char* qrow, int seg, float* bounds, double* exact) {
  const RaceStream R = race_stream(a.seed, rd.g);
  race_bounds<DT>(a, rd, R, trow, qrow, RES, seg, [&](float b, int x) {
    if (x < a.V) {
      bounds[x] = b;
      exact[x] = exact_key_of(a, rd, trow, qrow, RES, x);
    }
  });
}

template <int DT>
__device__ void probe_dispatch(const VerifyArgs& a, const RaceDesc& rd, const char* trow,
                               const char* qrow, int residual, int seg, float* bounds,
                               double* exact) {
  if (!residual)
    probe_segment<DT, false, false>(a, rd, trow, qrow, seg, bounds, exact);
  else if (rd.ntop > 0)
    probe_segment<DT, true, true>(a, rd, trow, qrow, seg, bounds, exact);
  else
    probe_segment<DT, true, false>(a, rd, trow, qrow, seg, bounds, exact);
}

__global__ void probe_kernel(VerifyArgs a, RaceDesc rd, const char* trow, const char* qrow,
                             int residual, float* bounds, double* exact) {
  const int warp = threadIdx.x >> 5;
  const int seg = blockIdx.x * (blockDim.x >> 5) + warp;
  if (seg >= a.nseg) return;
  if (a.dtype == kF32)
    probe_dispatch<kF32>(a, rd, trow, qrow, residual, seg, bounds, exact);
  else
    probe_dispatch<kBF16>(a, rd, trow, qrow, residual, seg, bounds, exact);
}

// All pointers are device pointers; lse values are natural-log LSEs at T.
extern "C" int race_bound_probe(const void* trow, const void* qrow, int V, int dtype, float T,
                                double lse_t, double lse_q, int ntop, const int* top,
                                double ln_c, double ln_Z, unsigned long long seed, unsigned g,
                                int residual, float* bounds, double* exact) {
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
  rd.k2 = (float)(1.4426950408889634 / (double)T);  // any k2 near log2(e)/T keeps the bound valid
  rd.l2_t = (float)(lse_t * 1.4426950408889634);
  rd.l2_q = (float)((lse_q + ln_Z) * 1.4426950408889634);
  rd.kmin = INFINITY;
  if (ntop) {
    // the smallest logit of K, read from the draft row on the device
    float v = 0.0f;
    if (dtype == kF32) {
      cudaMemcpy(&v, (const float*)qrow + top[ntop - 1], 4, cudaMemcpyDeviceToHost);
    } else {
      unsigned short h = 0;
      cudaMemcpy(&h, (const unsigned short*)qrow + top[ntop - 1], 2, cudaMemcpyDeviceToHost);
      unsigned int bits = (unsigned int)h << 16;
      memcpy(&v, &bits, 4);
    }
    rd.kmin = v;
  }
  probe_kernel<<<(a.nseg + 7) / 8, 256>>>(a, rd, (const char*)trow, (const char*)qrow, residual,
                                          bounds, exact);
  return cudaDeviceSynchronize() == cudaSuccess ? 0 : 1;
}
