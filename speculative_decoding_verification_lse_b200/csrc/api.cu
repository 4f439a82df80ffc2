// api.cu -- the C ABI of libspecverify (declared in include/specverify.h):
// argument checks, the per-device workspace cache, the device status word and
// the launch sequence.  Every step of the computation runs in the kernels.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "specverify.h"
#include "sv_common.cuh"

namespace sv {

// The device status word: one per device, in the library's own device memory.
__device__ unsigned int g_status_word;

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(SV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

struct DeviceCache {
  void* ws = nullptr;
  size_t ws_bytes = 0;
  unsigned int* status = nullptr;  // device address of g_status_word
  int sms = 0;                     // multiprocessor count
  int fused_per_sm[2][2 * SV_MAX_DRAFT + 2] = {};  // resident fused CTAs per SM, by dtype and slots
  int stats_per_sm[2] = {0, 0};    // resident statistics CTAs per SM, by dtype
};

std::mutex g_mu;
std::vector<DeviceCache> g_dev;

DeviceCache* device_cache(int dev) {
  if ((int)g_dev.size() <= dev) g_dev.resize(dev + 1);
  return &g_dev[dev];
}

// Device address of the status word on the current device (looked up once).
int status_word(int dev, unsigned int** out) {
  DeviceCache* c = device_cache(dev);
  if (!c->status) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_status_word);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status word)");
    c->status = (unsigned int*)p;
  }
  *out = c->status;
  return SV_OK;
}

// Resident grids of the persistent kernels on the current device.
int persistent_grid(int dev, int dtype, bool fused, int slots, int* grid) {
  DeviceCache* c = device_cache(dev);
  if (!c->sms) {
    cudaError_t e = cudaDeviceGetAttribute(&c->sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  }
  int* per_sm = fused ? &c->fused_per_sm[dtype][slots] : &c->stats_per_sm[dtype];
  if (!*per_sm) {
    *per_sm = fused ? fused_blocks_per_sm(dtype, slots) : row_stats_blocks_per_sm(dtype);
    if (*per_sm < 1) return fail(SV_ERR_CUDA, "kernel cannot be resident on this device");
  }
  *grid = c->sms * *per_sm;
  return SV_OK;
}

// The cached workspace of the current device, grown to at least `bytes`.
int cached_workspace(int dev, size_t bytes, void** out) {
  DeviceCache* c = device_cache(dev);
  if (c->ws_bytes < bytes) {
    if (c->ws) {
      // the old buffer may still be in use by work queued earlier on any stream
      cudaError_t e = cudaDeviceSynchronize();
      if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
      cudaFree(c->ws);
      c->ws = nullptr;
      c->ws_bytes = 0;
    }
    size_t want = bytes < (1u << 20) ? (1u << 20) : bytes;
    cudaError_t e = cudaMalloc(&c->ws, want);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(workspace)");
    c->ws_bytes = want;
  }
  *out = c->ws;
  return SV_OK;
}

// The epilogue sv_params asks for, after the verification on stream s.
int run_epilogue(const sv_params& prm, const int32_t* out_tokens, const int32_t* out_accept_len,
                 int B, int D_max, unsigned int* status, cudaStream_t s) {
  if (!prm.epilogue) return SV_OK;
  const sv_epilogue_args& ep = *prm.epilogue;
  const cudaError_t e = launch_epilogue(ep.window, out_tokens, out_accept_len, B, D_max,
                                        ep.next_window, ep.seq, ep.seq_cap, ep.seq_len,
                                        prm.out_flags, status, s);
  return e == cudaSuccess ? SV_OK : cuda_fail(e, "epilogue launch");
}

}  // namespace

// Every host-side argument check of sv_verify_ex (B == 0 passes them all);
// also run by sv_verify_static before its size test.
int check_args(const void* target_logits, const void* draft_logits, const int32_t* draft_tokens,
               int B, int D_max, int V, int dtype, float temperature, int mode,
               const int32_t* out_tokens, const int32_t* out_accept_len, const sv_params& prm) {
  if (B < 0) return fail(SV_ERR_INVALID_ARG, "B must be >= 0 (got %d)", B);
  if (D_max < 0 || D_max > SV_MAX_DRAFT)
    return fail(SV_ERR_INVALID_ARG, "D_max must be in [0, %d] (got %d)", SV_MAX_DRAFT, D_max);
  if (V < 1) return fail(SV_ERR_INVALID_ARG, "V must be >= 1 (got %d)", V);
  if (dtype != SV_F32 && dtype != SV_BF16)
    return fail(SV_ERR_INVALID_ARG, "dtype must be SV_F32 or SV_BF16 (got %d)", dtype);
  if (mode != SV_STOCHASTIC && mode != SV_GREEDY && mode != SV_SAGUARO)
    return fail(SV_ERR_INVALID_ARG, "mode must be SV_STOCHASTIC, SV_GREEDY or SV_SAGUARO (got %d)",
                mode);
  if (!prm.temperature_per_req && mode != SV_GREEDY && !(temperature > 0.0f && std::isfinite(temperature)))
    return fail(SV_ERR_INVALID_ARG, "temperature must be > 0 and finite (got %g)", (double)temperature);
  int k = prm.saguaro_k <= 0 ? 5 : prm.saguaro_k;
  if (k > SV_MAX_SAGUARO_K)
    return fail(SV_ERR_INVALID_ARG, "saguaro_k must be <= %d (got %d)", SV_MAX_SAGUARO_K, k);
  if (k > V) k = V;
  const float c = prm.saguaro_c <= 0.0f ? 0.5f : prm.saguaro_c;
  if (!(c > 0.0f && c <= 1.0f))
    return fail(SV_ERR_INVALID_ARG, "saguaro_c must be in (0, 1] (got %g)", (double)c);
  const int tail_bits = prm.variant & (SV_TAIL_PER_REQUEST | SV_TAIL_ITEMS);
  const int base_variant = prm.variant & ~(SV_TAIL_PER_REQUEST | SV_TAIL_ITEMS);
  if (base_variant < SV_VARIANT_AUTO || base_variant > SV_VARIANT_EARLY_EXIT ||
      tail_bits == (SV_TAIL_PER_REQUEST | SV_TAIL_ITEMS))
    return fail(SV_ERR_INVALID_ARG, "unknown variant %d", prm.variant);
  if (B == 0) return SV_OK;
  if (!target_logits || !out_tokens || !out_accept_len)
    return fail(SV_ERR_INVALID_ARG, "target_logits, out_tokens and out_accept_len must be non-NULL");
  if (D_max > 0 && !draft_tokens) return fail(SV_ERR_INVALID_ARG, "draft_tokens is NULL");
  if (!draft_logits && D_max > 0 && !prm.mode_per_req && mode != SV_GREEDY)
    return fail(SV_ERR_INVALID_ARG, "draft_logits is NULL but the mode reads it");
  const size_t es = dtype == SV_F32 ? 4 : 2;
  if (((uintptr_t)target_logits % es) || (draft_logits && ((uintptr_t)draft_logits % es)))
    return fail(SV_ERR_INVALID_ARG, "logit pointers must be aligned to the element size");

  int nvec, nseg;
  row_geometry(V, dtype, &nvec, &nseg);
  if (nseg > kMaxSegs)
    return fail(SV_ERR_UNSUPPORTED, "V larger than %d is not supported for this dtype",
                kMaxSegs * kSegVecs * vec_elems(dtype));
  if ((long long)B * (2LL * D_max + 2) * nseg > 0x7FFFFFFFLL)
    return fail(SV_ERR_UNSUPPORTED, "B * (2*D_max+2) * segments exceeds 2^31");
  return SV_OK;
}

int set_last_error(int code, const char* msg) { return fail(code, "%s", msg); }

// The state of one call between its checks and its launches.
struct Call {
  VerifyArgs a;
  WsLayout L;
  void* ws;
  unsigned int* status;
  int grid, base_variant;
  bool fused;
  int sms = 0;  // the device's multiprocessors
};

// Everything sv_verify_ex does before its launches: the argument checks, the
// workspace, the device queries and the kernels' argument block.  V is the row
// length (a shard's columns when the vocabulary is split, V_global = n_shards V,
// offset = the shard's first column); B == 0 returns SV_OK with *empty set.
int prepare_call(const void* target_logits, const void* draft_logits,
                 const int32_t* draft_tokens, const int32_t* row_D, int B, int D_max, int V,
                 int dtype, float temperature, int mode, uint64_t seed, int32_t* out_tokens,
                 int32_t* out_accept_len, const sv_params& prm, int V_global, int offset,
                 Call* call, bool* empty) {
  *empty = false;

  {
    const int rc = check_args(target_logits, draft_logits, draft_tokens, B, D_max, V, dtype,
                              temperature, mode, out_tokens, out_accept_len, prm);
    if (rc != SV_OK) return rc;
  }
  if (B == 0) {
    *empty = true;
    return SV_OK;
  }
  int k = prm.saguaro_k <= 0 ? 5 : prm.saguaro_k;
  if (k > V) k = V;
  const float c = prm.saguaro_c <= 0.0f ? 0.5f : prm.saguaro_c;
  const int tail_bits = prm.variant & (SV_TAIL_PER_REQUEST | SV_TAIL_ITEMS);
  const int base_variant = prm.variant & ~(SV_TAIL_PER_REQUEST | SV_TAIL_ITEMS);
  int nvec, nseg;
  row_geometry(V, dtype, &nvec, &nseg);
  const long long slots = 2LL * D_max + 1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");

  // the same layout sv_workspace_bytes reports, whatever the modes
  const WsLayout L = ws_layout(B, D_max, V, dtype, true);
  void* ws = prm.workspace;
  unsigned int* status = nullptr;
  const bool fused = base_variant == SV_VARIANT_FUSED;
  int grid = 0, sms = 0;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    int rc = status_word(dev, &status);
    if (rc) return rc;
    if ((rc = persistent_grid(dev, dtype, fused, (int)slots, &grid))) return rc;
    sms = device_cache(dev)->sms;
    if (ws) {
      if (prm.workspace_bytes < L.total)
        return fail(SV_ERR_INVALID_ARG, "workspace too small: %zu < %zu bytes",
                    prm.workspace_bytes, L.total);
      if ((uintptr_t)ws % 256)
        return fail(SV_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    } else {
      rc = cached_workspace(dev, L.total, &ws);
      if (rc) return rc;
    }
  }

  VerifyArgs& a = call->a;
  memset(&a, 0, sizeof a);
  a.target = target_logits;
  a.draft = draft_logits;
  a.tokens = draft_tokens;
  a.row_D = row_D;
  a.temp_per_req = prm.temperature_per_req;
  a.mode_per_req = prm.mode_per_req;
  a.out_tokens = out_tokens;
  a.out_al = out_accept_len;
  a.out_row_lse = prm.out_row_lse;
  a.out_flags = prm.out_flags;
  a.out_draft_top = prm.out_draft_top;
  a.status = status;
  a.pstat = (PartStat*)((char*)ws + L.pstat);
  a.tpart = (TopPart*)((char*)ws + L.tpart);
  a.rdesc = (RaceDesc*)((char*)ws + L.rdesc);
  a.rpart = (RacePart*)((char*)ws + L.rpart);
  a.rcount = (unsigned int*)((char*)ws + L.rcount);
  a.best_key = (unsigned long long*)((char*)ws + L.best_key);
  a.rorder = (unsigned short*)((char*)ws + L.rorder);
  a.ticket = (unsigned int*)((char*)ws + L.ticket);
  a.rowres = (RowRes*)((char*)ws + L.rowres);
  a.rowcnt = (unsigned int*)((char*)ws + L.rowcnt);
  a.reqcnt = (unsigned int*)((char*)ws + L.reqcnt);
  a.pubq = (unsigned int*)((char*)ws + L.pubq);
  a.ctl = (unsigned int*)((char*)ws + L.ctl);
  a.seed = seed;
  a.seed_ptr = prm.seed_device;
  a.B = B;
  a.D_max = D_max;
  a.V = V;
  a.V_global = V_global;
  a.vocab_offset = offset;
  a.dtype = dtype;
  a.nvec = nvec;
  a.nseg = nseg;
  a.slots = (int)slots;
  a.mode = mode;
  // one CTA per request once the requests fill four fifths of the multiprocessors (each
  // request's race then has a multiprocessor to itself, and one launch less beats spreading
  // the races over the rest), or when there are too few race segments to spread; else the
  // scan, then race items over the whole GPU
  const bool spread = 5LL * B < 4LL * sms && (long long)B * nseg > sms;
  a.per_request = tail_bits == SV_TAIL_PER_REQUEST ? 1 : tail_bits == SV_TAIL_ITEMS ? 0 : (spread ? 0 : 1);
  // the fused kernel races half segments; the split path cuts them while one wave holds them
  a.rsplit = fused ? kMaxRaceSplit : a.per_request ? 1 : race_split(B, nseg, dtype, sms);
  a.race_sm_every = fused ? fused_race_sm_every(a, grid) : 0;
  a.temperature = temperature;
  a.saguaro_k = k;
  a.saguaro_c = c;
  a.request_offset = prm.request_offset;
  call->L = L;
  call->ws = ws;
  call->status = status;
  call->grid = grid;
  call->base_variant = base_variant;
  call->fused = fused;
  call->sms = sms;
  return SV_OK;
}

}  // namespace sv

using namespace sv;

extern "C" {

int sv_version(void) { return 10000; }

const char* sv_last_error(void) { return g_last_error.c_str(); }

int sv_advance_seed(uint64_t* seed_device, uint64_t by, void* stream) {
  g_last_error.clear();
  if (seed_device == nullptr || (uintptr_t)seed_device % 8 != 0)
    return fail(SV_ERR_INVALID_ARG, "sv_advance_seed: seed_device must be an 8-byte aligned device pointer");
  cudaError_t e = launch_advance_seed(seed_device, by, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "sv_advance_seed launch");
  return SV_OK;
}

size_t sv_workspace_bytes(int B, int D_max, int V, int dtype) {
  if (B < 0 || D_max < 0 || V < 1 || (dtype != SV_F32 && dtype != SV_BF16)) return 0;
  return ws_layout(B, D_max, V, dtype, true).total;
}

int sv_verify_ex(const void* target_logits, const void* draft_logits,
                 const int32_t* draft_tokens, const int32_t* row_D, int B, int D_max, int V,
                 int dtype, float temperature, int mode, uint64_t seed, int32_t* out_tokens,
                 int32_t* out_accept_len, const sv_params* p) {
  sv_params prm;
  memset(&prm, 0, sizeof prm);
  if (p) prm = *p;
  g_last_error.clear();
  Call call;
  bool empty = false;
  {
    const int rc = prepare_call(target_logits, draft_logits, draft_tokens, row_D, B, D_max, V,
                                dtype, temperature, mode, seed, out_tokens, out_accept_len, prm, V,
                                0, &call, &empty);
    if (rc != SV_OK || empty) return rc;
  }
  VerifyArgs& a = call.a;
  const WsLayout& L = call.L;
  void* ws = call.ws;
  unsigned int* status = call.status;
  const int grid = call.grid, base_variant = call.base_variant;
  const bool fused = call.fused;
  cudaError_t e;
  cudaStream_t s = (cudaStream_t)prm.stream;
  cudaEvent_t* ev = (cudaEvent_t*)prm.timing_events;
  if (prm.epilogue) {
    const sv_epilogue_args& ep = *prm.epilogue;
    const char* why = nullptr;
    if (epilogue_check(ep.window, out_tokens, out_accept_len, B, D_max, ep.next_window, ep.seq,
                       ep.seq_cap, ep.seq_len, &why) != SV_OK)
      return fail(SV_ERR_INVALID_ARG, "sv_params.epilogue: %s", why);
  }
  if (base_variant == SV_VARIANT_CLUSTER) {
    if (ev && (e = cudaEventRecord(ev[0], s)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    if ((e = launch_cluster(a, s)) != cudaSuccess) return cuda_fail(e, "cluster launch");
    if (ev && (e = cudaEventRecord(ev[1], s)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    return run_epilogue(prm, out_tokens, out_accept_len, B, D_max, status, s);
  }
  if (fused) {
    // the fused kernel's counters, queue and tickets start at zero
    if ((e = cudaMemsetAsync((char*)ws + L.zero, 0, L.total - L.zero, s)) != cudaSuccess)
      return cuda_fail(e, "cudaMemsetAsync(fused bookkeeping)");
    if (ev && (e = cudaEventRecord(ev[0], s)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    if ((e = launch_fused(a, s, grid)) != cudaSuccess) return cuda_fail(e, "fused launch");
    if (ev && (e = cudaEventRecord(ev[1], s)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    return run_epilogue(prm, out_tokens, out_accept_len, B, D_max, status, s);
  }
  if (base_variant == SV_VARIANT_EARLY_EXIT) {
    // the rows position by position, then the usual finish from the merged rows
    a.ee_n = (int*)((char*)ws + L.ee);
    a.ee_alive = a.ee_n + B;
    a.ee_count = (unsigned int*)((char*)ws + align_up(L.ee + (size_t)3 * B * sizeof(int), 128));
    if ((e = cudaMemsetAsync(a.ticket, 0, 8 * 128, s)) != cudaSuccess)
      return cuda_fail(e, "cudaMemsetAsync(ticket)");
    if (ev && (e = cudaEventRecord(ev[0], s)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    if ((e = launch_early_exit_rounds(a, s, grid)) != cudaSuccess)
      return cuda_fail(e, "early-exit rounds launch");
    if (ev && (e = cudaEventRecord(ev[1], s)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  } else {
    const bool tickets = row_stats_tickets(a, grid);
    if (tickets && (e = cudaMemsetAsync(a.ticket, 0, 8 * 128, s)) != cudaSuccess)
      return cuda_fail(e, "cudaMemsetAsync(ticket)");
    if (ev && (e = cudaEventRecord(ev[0], s)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    if ((e = launch_row_stats(a, s, grid, tickets)) != cudaSuccess)
      return cuda_fail(e, "row statistics launch");
    if (ev && (e = cudaEventRecord(ev[1], s)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  }
  if (a.per_request) {
    if ((e = launch_requests(a, s, call.sms)) != cudaSuccess) return cuda_fail(e, "scan and race launch");
  } else {
    if ((e = launch_scan(a, s)) != cudaSuccess) return cuda_fail(e, "accept scan launch");
    if ((e = launch_race(a, s)) != cudaSuccess) return cuda_fail(e, "race launch");
  }
  return run_epilogue(prm, out_tokens, out_accept_len, B, D_max, status, s);
}

size_t sv_shard_exchange_bytes(int B, int D_max, int V_local, int dtype, int stage) {
  if (B < 0 || D_max < 0 || D_max > SV_MAX_DRAFT || V_local < 1 ||
      (dtype != SV_F32 && dtype != SV_BF16) || (stage != 1 && stage != 2))
    return 0;
  const ShardLayout L = shard_layout(B, D_max, V_local, dtype);
  return stage == 1 ? L.x1 : L.x2;
}

}  // extern "C"

namespace {

// The shard geometry: n_shards ranks of V_local columns each.
int shard_check(int n_shards, int shard, int V_local, int dtype) {
  if (n_shards < 1 || shard < 0 || shard >= n_shards)
    return fail(SV_ERR_INVALID_ARG, "shard %d of %d is out of range", shard, n_shards);
  if (V_local < 1 || V_local % 4)
    return fail(SV_ERR_INVALID_ARG, "V_local must be a positive multiple of 4 (got %d)", V_local);
  if ((long long)n_shards * V_local > 0x7FFFFFFFLL)
    return fail(SV_ERR_UNSUPPORTED, "n_shards * V_local exceeds 2^31");
  int nvec, nseg;
  row_geometry(V_local, dtype == SV_F32 ? SV_F32 : SV_BF16, &nvec, &nseg);
  if ((long long)nseg * n_shards > kMaxSegs)
    return fail(SV_ERR_UNSUPPORTED, "n_shards * segments per shard exceeds %d", kMaxSegs);
  return SV_OK;
}

}  // namespace

extern "C" {

int sv_shard_stats(const void* target_local, const void* draft_local, const int32_t* draft_tokens,
                   const int32_t* row_D, int B, int D_max, int V_local, int dtype,
                   float temperature, int mode, uint64_t seed, int n_shards, int shard,
                   const sv_params* p, void* exchange1) {
  sv_params prm;
  memset(&prm, 0, sizeof prm);
  if (p) prm = *p;
  prm.variant = SV_VARIANT_SPLIT;
  prm.epilogue = nullptr;
  g_last_error.clear();
  int rc = shard_check(n_shards, shard, V_local, dtype);
  if (rc != SV_OK) return rc;
  if (B > 0 && !exchange1) return fail(SV_ERR_INVALID_ARG, "exchange1 is NULL");
  // this stage writes no outputs; the exchange buffer stands in for them in the checks
  Call call;
  bool empty = false;
  rc = prepare_call(target_local, draft_local, draft_tokens, row_D, B, D_max, V_local, dtype,
                    temperature, mode, seed, (int32_t*)exchange1, (int32_t*)exchange1, prm,
                    n_shards * V_local, shard * V_local, &call, &empty);
  if (rc != SV_OK || empty) return rc;
  VerifyArgs& a = call.a;
  const ShardLayout X = shard_layout(B, D_max, V_local, dtype);
  a.pstat = (PartStat*)((char*)exchange1 + X.parts);
  a.tpart = (TopPart*)((char*)exchange1 + X.tops);
  cudaStream_t s = (cudaStream_t)prm.stream;
  cudaError_t e;
  const bool tickets = row_stats_tickets(a, call.grid);
  if (tickets && (e = cudaMemsetAsync(a.ticket, 0, 8 * 128, s)) != cudaSuccess)
    return cuda_fail(e, "cudaMemsetAsync(ticket)");
  if ((e = launch_row_stats(a, s, call.grid, tickets)) != cudaSuccess)
    return cuda_fail(e, "row statistics launch");
  if ((e = launch_shard_z(a, (char*)exchange1 + X.zx, s)) != cudaSuccess)
    return cuda_fail(e, "owned logits launch");
  return SV_OK;
}

int sv_shard_race(const void* target_local, const void* draft_local, const int32_t* draft_tokens,
                  const int32_t* row_D, int B, int D_max, int V_local, int dtype,
                  float temperature, int mode, uint64_t seed, int n_shards, int shard,
                  const sv_params* p, const void* gathered1, int32_t* out_tokens,
                  int32_t* out_accept_len, void* exchange2) {
  sv_params prm;
  memset(&prm, 0, sizeof prm);
  if (p) prm = *p;
  prm.variant = SV_VARIANT_SPLIT;
  prm.epilogue = nullptr;
  g_last_error.clear();
  int rc = shard_check(n_shards, shard, V_local, dtype);
  if (rc != SV_OK) return rc;
  if (B > 0 && (!gathered1 || !exchange2))
    return fail(SV_ERR_INVALID_ARG, "gathered1 and exchange2 must be non-NULL");
  Call call;
  bool empty = false;
  rc = prepare_call(target_local, draft_local, draft_tokens, row_D, B, D_max, V_local, dtype,
                    temperature, mode, seed, out_tokens, out_accept_len, prm, n_shards * V_local,
                    shard * V_local, &call, &empty);
  if (rc != SV_OK || empty) return rc;
  const cudaError_t e =
      launch_shard_tail(call.a, gathered1, n_shards, exchange2, (cudaStream_t)prm.stream);
  return e == cudaSuccess ? SV_OK : cuda_fail(e, "shard scan and race launch");
}

int sv_shard_finish(int B, int D_max, int n_shards, const void* gathered2, int32_t* out_tokens,
                    const sv_params* p) {
  sv_params prm;
  memset(&prm, 0, sizeof prm);
  if (p) prm = *p;
  g_last_error.clear();
  if (B < 0) return fail(SV_ERR_INVALID_ARG, "B must be >= 0 (got %d)", B);
  if (D_max < 0 || D_max > SV_MAX_DRAFT)
    return fail(SV_ERR_INVALID_ARG, "D_max must be in [0, %d] (got %d)", SV_MAX_DRAFT, D_max);
  if (n_shards < 1) return fail(SV_ERR_INVALID_ARG, "n_shards must be >= 1 (got %d)", n_shards);
  if (B == 0) return SV_OK;
  if (!gathered2 || !out_tokens)
    return fail(SV_ERR_INVALID_ARG, "gathered2 and out_tokens must be non-NULL");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  unsigned int* status = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    const int rc = status_word(dev, &status);
    if (rc) return rc;
  }
  e = launch_shard_finish(gathered2, B, D_max, n_shards, out_tokens, prm.out_flags, status,
                          (cudaStream_t)prm.stream);
  return e == cudaSuccess ? SV_OK : cuda_fail(e, "shard finish launch");
}

int sv_verify_tree(const void* target_logits, const void* draft_logits,
                   const int32_t* node_tokens, const int32_t* parents, const int32_t* n_nodes,
                   int B, int N_max, int V, int dtype, float temperature, int mode, uint64_t seed,
                   int32_t* out_tokens, int32_t* out_accept_len, int32_t* out_nodes,
                   const sv_params* p) {
  sv_params prm;
  memset(&prm, 0, sizeof prm);
  if (p) prm = *p;
  prm.variant = SV_VARIANT_SPLIT;
  prm.epilogue = nullptr;
  prm.out_draft_top = nullptr;
  g_last_error.clear();
  if (mode != SV_STOCHASTIC && mode != SV_GREEDY)
    return fail(SV_ERR_INVALID_ARG, "tree verification takes SV_STOCHASTIC or SV_GREEDY (got %d)",
                mode);
  if (B > 0 && N_max > 0 && !parents) return fail(SV_ERR_INVALID_ARG, "parents is NULL");
  Call call;
  bool empty = false;
  int rc = prepare_call(target_logits, draft_logits, node_tokens, n_nodes, B, N_max, V, dtype,
                        temperature, mode, seed, out_tokens, out_accept_len, prm, V, 0, &call,
                        &empty);
  if (rc != SV_OK || empty) return rc;
  VerifyArgs& a = call.a;
  a.parents = parents;
  a.out_nodes = out_nodes;
  cudaStream_t s = (cudaStream_t)prm.stream;
  cudaEvent_t* ev = (cudaEvent_t*)prm.timing_events;
  cudaError_t e;
  const bool tickets = row_stats_tickets(a, call.grid);
  if (tickets && (e = cudaMemsetAsync(a.ticket, 0, 8 * 128, s)) != cudaSuccess)
    return cuda_fail(e, "cudaMemsetAsync(ticket)");
  if (ev && (e = cudaEventRecord(ev[0], s)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  if ((e = launch_row_stats(a, s, call.grid, tickets)) != cudaSuccess)
    return cuda_fail(e, "row statistics launch");
  if (ev && (e = cudaEventRecord(ev[1], s)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  if ((e = launch_tree(a, s, call.sms)) != cudaSuccess) return cuda_fail(e, "tree walk launch");
  return SV_OK;
}

int sv_verify(const void* target_logits, const void* draft_logits, const int32_t* draft_tokens,
              const int32_t* row_D, int B, int D_max, int V, int dtype, float temperature,
              int mode, uint64_t seed, int32_t* out_tokens, int32_t* out_accept_len) {
  return sv_verify_ex(target_logits, draft_logits, draft_tokens, row_D, B, D_max, V, dtype,
                      temperature, mode, seed, out_tokens, out_accept_len, nullptr);
}

int sv_verify_greedy(const void* target_logits, const int32_t* draft_tokens,
                     const int32_t* row_D, int B, int D_max, int V, int dtype,
                     int32_t* out_tokens, int32_t* out_accept_len) {
  return sv_verify_ex(target_logits, nullptr, draft_tokens, row_D, B, D_max, V, dtype, 1.0f,
                      SV_GREEDY, 0, out_tokens, out_accept_len, nullptr);
}

int sv_epilogue(const int32_t* window, const int32_t* out_tokens, const int32_t* out_accept_len,
                int B, int D_max, int32_t* next_window, int32_t* seq, int seq_cap,
                int32_t* seq_len, uint32_t* flags, void* stream) {
  g_last_error.clear();
  const char* why = nullptr;
  if (epilogue_check(window, out_tokens, out_accept_len, B, D_max, next_window, seq, seq_cap,
                     seq_len, &why) != SV_OK)
    return fail(SV_ERR_INVALID_ARG, "sv_epilogue: %s", why);
  if (B == 0) return SV_OK;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  unsigned int* status = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    const int rc = status_word(dev, &status);
    if (rc) return rc;
  }
  e = launch_epilogue(window, out_tokens, out_accept_len, B, D_max, next_window, seq, seq_cap,
                      seq_len, flags, status, (cudaStream_t)stream);
  return e == cudaSuccess ? SV_OK : cuda_fail(e, "epilogue launch");
}

int sv_ssd_lookup(const int32_t* out_tokens, const int32_t* out_accept_len, int B, int D_max,
                  const int32_t* keys_al, const int32_t* keys_token, int K, const int32_t* spec,
                  int S, int32_t* out_hit, int32_t* out_spec, void* stream) {
  g_last_error.clear();
  const char* why = nullptr;
  if (ssd_lookup_check(out_tokens, out_accept_len, B, D_max, keys_al, keys_token, K, spec, S,
                       out_hit, out_spec, &why) != SV_OK)
    return fail(SV_ERR_INVALID_ARG, "sv_ssd_lookup: %s", why);
  const cudaError_t e = launch_ssd_lookup(out_tokens, out_accept_len, B, D_max, keys_al,
                                          keys_token, K, spec, S, out_hit, out_spec,
                                          (cudaStream_t)stream);
  return e == cudaSuccess ? SV_OK : cuda_fail(e, "ssd lookup launch");
}

int sv_get_device_status(void* stream, uint32_t* status_bits) {
  g_last_error.clear();
  if (!status_bits) return fail(SV_ERR_INVALID_ARG, "status_bits is NULL");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  unsigned int* status = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    int rc = status_word(dev, &status);
    if (rc) return rc;
  }
  cudaStream_t s = (cudaStream_t)stream;
  unsigned int host = 0;
  if ((e = cudaMemcpyAsync(&host, status, sizeof host, cudaMemcpyDeviceToHost, s)) != cudaSuccess)
    return cuda_fail(e, "cudaMemcpyAsync(status)");
  if ((e = cudaMemsetAsync(status, 0, sizeof host, s)) != cudaSuccess)
    return cuda_fail(e, "cudaMemsetAsync(status)");
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  *status_bits = host;
  return SV_OK;
}

void sv_shutdown(void) {
  std::lock_guard<std::mutex> lock(g_mu);
  int cur = 0;
  cudaGetDevice(&cur);
  for (size_t d = 0; d < g_dev.size(); ++d) {
    if (g_dev[d].ws) {
      cudaSetDevice((int)d);
      cudaFree(g_dev[d].ws);
    }
    g_dev[d].ws = nullptr;
    g_dev[d].ws_bytes = 0;
  }
  cudaSetDevice(cur);
}

}  // extern "C"
