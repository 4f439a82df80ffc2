// epilogue.cu -- the step after verification, on the device: the next run's
// shifted input window and the append of the emitted tokens to each request's
// sequence, so that the caller needs no GPU-to-CPU sync between steps.
//
// "Accélérer Sonar par la Spéculation", section "Calendrier MTP pour un jeton
// unique": once the target's input tokens are shifted, a kernel inserts the
// next target tokens at their slots, and the draft re-runs on that window
// (doing a little redundant work on the tokens that were not accepted) while
// the next sequence lengths, set by the accepted lengths, need no wait on the
// CPU.  Section "Inférence avec décodage spéculatif": the accepted length
// decides the next sequence length, the sync point this avoids.
//
// Per request b (one warp), with AL = out_accept_len[b] and n = AL - 1:
//   next_window[b][j] = window[b][j + 1] (j < D_max), next_window[b][D_max] = -1,
//   next_window[b][n] = out_tokens[b][n]                 (the inserted target token)
//   seq[b][seq_len[b] + j] = out_tokens[b][j] (j < AL), seq_len[b] += AL
// AL outside [1, D_max + 1] (a request the verification flagged): a row of -1
// and no append.  An append past seq_cap: no append, SV_FLAG_SEQ_FULL in the
// request's flags (if given) and in the device status word.
#include <cstring>

#include "specverify.h"
#include "sv_common.cuh"

namespace sv {

namespace {

struct EpilogueArgs {
  const int32_t* window;
  const int32_t* out_tokens;
  const int32_t* out_al;
  int32_t* next_window;
  int32_t* seq;
  int32_t* seq_len;
  uint32_t* flags;
  unsigned* status;
  int B, W, seq_cap;
};

constexpr int kEpiWarps = 8;  // requests per CTA

__global__ void __launch_bounds__(kEpiWarps * 32) epilogue_kernel(EpilogueArgs e) {
  wait_for_previous_kernel();  // launched as a dependent of the verification's last kernel
  const int lane = threadIdx.x & 31;
  const int b = blockIdx.x * kEpiWarps + (threadIdx.x >> 5);
  if (b >= e.B) return;
  const int W = e.W;  // D_max + 1 <= SV_MAX_DRAFT + 1 = 33: two slots per lane
  const int AL = e.out_al[b];
  const bool valid = AL >= 1 && AL <= W;
  const size_t row = (size_t)b * W;
  // read everything first: next_window may be window itself
  int32_t sh[2], ot[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int j = lane + 32 * k;
    sh[k] = (e.window && j + 1 < W) ? e.window[row + j + 1] : -1;
    ot[k] = j < W ? e.out_tokens[row + j] : -1;
  }
  int32_t L = 0;
  if (e.seq && lane == 0) L = e.seq_len[b];
  L = __shfl_sync(0xFFFFFFFFu, L, 0);
  __syncwarp();
  if (e.next_window) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int j = lane + 32 * k;
      if (j < W) e.next_window[row + j] = !valid ? -1 : (j == AL - 1 ? ot[k] : sh[k]);
    }
  }
  if (e.seq && valid) {
    if (L < 0 || (long long)L + AL > e.seq_cap) {
      if (lane == 0) {
        if (e.flags) e.flags[b] |= kFlagSeqFull;
        atomicOr(e.status, kFlagSeqFull);
      }
    } else {
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int j = lane + 32 * k;
        if (j < AL) e.seq[(size_t)b * e.seq_cap + L + j] = ot[k];
      }
      if (lane == 0) e.seq_len[b] = L + AL;
    }
  }
}

}  // namespace

int epilogue_check(const int32_t* window, const int32_t* out_tokens, const int32_t* out_accept_len,
                   int B, int D_max, const int32_t* next_window, const int32_t* seq, int seq_cap,
                   const int32_t* seq_len, const char** why) {
  if (B < 0) return *why = "B must be >= 0", SV_ERR_INVALID_ARG;
  if (D_max < 0 || D_max > SV_MAX_DRAFT) return *why = "D_max must be in [0, SV_MAX_DRAFT]", SV_ERR_INVALID_ARG;
  if (B == 0) return SV_OK;
  if (!out_tokens || !out_accept_len)
    return *why = "out_tokens and out_accept_len must be non-NULL", SV_ERR_INVALID_ARG;
  if (next_window && !window) return *why = "next_window needs window", SV_ERR_INVALID_ARG;
  if (seq && (!seq_len || seq_cap < 0))
    return *why = "seq needs seq_len and seq_cap >= 0", SV_ERR_INVALID_ARG;
  return SV_OK;
}

cudaError_t launch_epilogue(const int32_t* window, const int32_t* out_tokens,
                            const int32_t* out_accept_len, int B, int D_max, int32_t* next_window,
                            int32_t* seq, int seq_cap, int32_t* seq_len, uint32_t* flags,
                            unsigned* status, cudaStream_t s) {
  if (B == 0 || (!next_window && !seq)) return cudaSuccess;
  EpilogueArgs e;
  memset(&e, 0, sizeof e);
  e.window = window;
  e.out_tokens = out_tokens;
  e.out_al = out_accept_len;
  e.next_window = next_window;
  e.seq = seq;
  e.seq_len = seq_len;
  e.flags = flags;
  e.status = status;
  e.B = B;
  e.W = D_max + 1;
  e.seq_cap = seq_cap;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof cfg);
  cfg.gridDim = dim3((B + kEpiWarps - 1) / kEpiWarps);
  cfg.blockDim = dim3(kEpiWarps * 32);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, epilogue_kernel, e);
}

namespace {

__global__ void advance_seed_kernel(uint64_t* seed, uint64_t by) { *seed += by; }

}  // namespace

// *seed += by on stream s (sv_advance_seed).
cudaError_t launch_advance_seed(uint64_t* seed, uint64_t by, cudaStream_t s) {
  advance_seed_kernel<<<1, 1, 0, s>>>(seed, by);
  return cudaGetLastError();
}

}  // namespace sv
