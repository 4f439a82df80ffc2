// ssd_lookup.cu -- the outcome lookup of speculative speculative decoding, on
// the device.
//
// "Speculative Speculative Decoding – асинхронизируй это.": while the target
// verifies, the draft predicts the likely verification outcomes and prepares a
// speculation for each; if the actual outcome is among them, its speculation
// is returned at once (the page's restaurant: a dish already on the shelf),
// else it is a miss and the next speculation starts from scratch.  Saguaro
// sampling (same page, recipe items 1-3) makes the outcomes concentrate on the
// draft's top tokens, which is what the keys usually are (sv_params.out_draft_top).
//
// Per request b (one warp): the outcome is (AL, out_tokens[b][AL - 1]); the hit
// is the lowest key index k with keys_al[b][k] == AL and keys_token[b][k] == that
// token (-1 if none, or if AL lies outside [1, D_max + 1]); on a hit the
// prepared speculation spec[b][k][0..S-1] is copied to out_spec[b], else
// out_spec[b] is -1.
#include <climits>
#include <cstring>

#include "specverify.h"
#include "sv_common.cuh"

namespace sv {

namespace {

struct LookupArgs {
  const int32_t* out_tokens;
  const int32_t* out_al;
  const int32_t* keys_al;
  const int32_t* keys_token;
  const int32_t* spec;
  int32_t* out_hit;
  int32_t* out_spec;
  int B, W, K, S;
};

constexpr int kLookupWarps = 8;

__global__ void __launch_bounds__(kLookupWarps * 32) lookup_kernel(LookupArgs e) {
  wait_for_previous_kernel();
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.x * kLookupWarps + (threadIdx.x >> 5);
  if (b >= e.B) return;
  const int AL = e.out_al[b];
  int best = INT_MAX;
  if (AL >= 1 && AL <= e.W) {
    const int tok = e.out_tokens[(size_t)b * e.W + AL - 1];
    for (int k = lane; k < e.K; k += 32) {
      const size_t i = (size_t)b * e.K + k;
      if (e.keys_al[i] == AL && e.keys_token[i] == tok) {
        best = k;
        break;  // the lane's keys ascend
      }
    }
  }
  best = __reduce_min_sync(0xFFFFFFFFu, best);
  const int hit = best == INT_MAX ? -1 : best;
  if (lane == 0) e.out_hit[b] = hit;
  if (e.out_spec)
    for (int j = lane; j < e.S; j += 32)
      e.out_spec[(size_t)b * e.S + j] = hit >= 0 ? e.spec[((size_t)b * e.K + hit) * e.S + j] : -1;
}

}  // namespace

int ssd_lookup_check(const int32_t* out_tokens, const int32_t* out_accept_len, int B, int D_max,
                     const int32_t* keys_al, const int32_t* keys_token, int K,
                     const int32_t* spec, int S, const int32_t* out_hit, const int32_t* out_spec,
                     const char** why) {
  if (B < 0) return *why = "B must be >= 0", SV_ERR_INVALID_ARG;
  if (D_max < 0 || D_max > SV_MAX_DRAFT) return *why = "D_max must be in [0, SV_MAX_DRAFT]", SV_ERR_INVALID_ARG;
  if (K < 0 || S < 0) return *why = "K and S must be >= 0", SV_ERR_INVALID_ARG;
  if (B == 0) return SV_OK;
  if (!out_tokens || !out_accept_len || !out_hit)
    return *why = "out_tokens, out_accept_len and out_hit must be non-NULL", SV_ERR_INVALID_ARG;
  if (K > 0 && (!keys_al || !keys_token)) return *why = "keys are NULL", SV_ERR_INVALID_ARG;
  if (out_spec && S > 0 && !spec) return *why = "out_spec needs spec", SV_ERR_INVALID_ARG;
  return SV_OK;
}

cudaError_t launch_ssd_lookup(const int32_t* out_tokens, const int32_t* out_accept_len, int B,
                              int D_max, const int32_t* keys_al, const int32_t* keys_token, int K,
                              const int32_t* spec, int S, int32_t* out_hit, int32_t* out_spec,
                              cudaStream_t s) {
  if (B == 0) return cudaSuccess;
  LookupArgs e;
  memset(&e, 0, sizeof e);
  e.out_tokens = out_tokens;
  e.out_al = out_accept_len;
  e.keys_al = keys_al;
  e.keys_token = keys_token;
  e.spec = spec;
  e.out_hit = out_hit;
  e.out_spec = out_spec;
  e.B = B;
  e.W = D_max + 1;
  e.K = K;
  e.S = S;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3((B + kLookupWarps - 1) / kLookupWarps);
  cfg.blockDim = dim3(kLookupWarps * 32);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, lookup_kernel, e);
}

}  // namespace sv
