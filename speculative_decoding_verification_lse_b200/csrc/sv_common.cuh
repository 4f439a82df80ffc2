// sv_common.cuh -- layouts and device helpers shared by the libspecverify kernels.
//
// Row decomposition (fixed by V and dtype only, so that identical rows always
// reduce in the same order and give bit-identical statistics, whatever the
// batch around them):
//   a row of V logits is read as 16-byte vectors of VEC elements (8 bf16 or 4 fp32);
//   a segment is kSegVecs = 32 * kLaneVecs consecutive vectors (8 KiB), handled by
//   one warp: lane l owns vectors seg*kSegVecs + l + 32*j, j = 0..kLaneVecs-1, so
//   the warp reads 512 contiguous bytes per j.
//   Each segment yields one partial (its maximum, the sum of 2^(z*k2 - max*k2),
//   the lowest index of its maximum); a row's partials are merged in segment
//   order by one warp in double precision.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sv {

constexpr int kThreads = 256;        // threads per CTA (8 independent warps)
constexpr int kWarps = kThreads / 32;
constexpr int kLaneVecs = 16;        // 16-byte vectors per lane per segment
constexpr int kSegVecs = 32 * kLaneVecs;  // 512 vectors = 8 KiB per segment
constexpr int kMaxDraft = 32;
constexpr int kMaxTopK = 8;
constexpr int kMaxRaceSplit = 2;    // race items per segment, at most
constexpr int kMaxSegs = 1024;       // segments per row (V up to 2^21 bf16 / 2^20 fp32)
constexpr int kScanWarps = 4;        // requests per accept-scan CTA
constexpr int kClusterMax = 8;       // CTAs per request in the cluster variant (portable limit)
constexpr int kClusterParts = kClusterMax * kThreads / 32;  // race results per request there

enum : int { kF32 = 0, kBF16 = 1 };
enum : int { kStochastic = 0, kGreedy = 1, kSaguaro = 2 };
enum : int { kRaceNone = 0, kRaceBonus = 1, kRaceResidual = 2 };

enum : uint32_t {
  kFlagAcceptNearTie = 1u << 0,
  kFlagRaceNearTie = 1u << 1,
  kFlagResidualEmpty = 1u << 2,
  kFlagBadToken = 1u << 8,
  kFlagBadRowD = 1u << 9,
  kFlagNonfinite = 1u << 10,
  kFlagBadParam = 1u << 11,
  kFlagErrors = kFlagBadToken | kFlagBadRowD | kFlagNonfinite | kFlagBadParam,
  kStatusTimeout = 1u << 12,  // a bounded wait of the fused kernel expired
  kFlagSeqFull = 1u << 13     // the epilogue's append would pass the sequence capacity
};

// Partial statistics of one segment of one row (16 bytes).
//   m     : largest logit in the segment (raw, as float); -inf if all are -inf
//   S     : sum over the segment of 2^(fl(z*k2 - mk)), mk = fl(m*k2),
//           k2 = fl(log2(e) / T); so S * 2^mk = sum 2^(z*k2)
//   argmax: lowest index of m inside the segment
//   bad   : nonzero if a NaN or +inf was seen
struct __align__(16) PartStat {
  float m;
  float S;
  int argmax;
  uint32_t bad;
};

// The k largest logits of one segment (value desc, index asc), saguaro draft rows.
struct __align__(16) TopPart {
  float v[kMaxTopK];
  int i[kMaxTopK];
};

// One row's merged statistics (written by the warp that merges the row).
struct __align__(16) RowRes {
  double lse;   // natural-log LSE at T (stochastic rows)
  double lnZ;   // saguaro draft rows: ln Z
  int argmax;   // greedy target rows
  uint32_t bad;
  int ntop;
  int mseg;     // the segment holding the row's largest logit (lowest such segment)
  int top[kMaxTopK];
  float topv[kMaxTopK];
};

// What the race of one request needs; written by the accept scan.
struct __align__(16) RaceDesc {
  int kind;          // kRaceNone / kRaceBonus / kRaceResidual
  int n;             // the position sampled (target row n; draft row n for residual)
  uint32_t g;        // global request index (Philox counter word 1)
  uint32_t flags;    // flags gathered so far (accept near-tie)
  double T;          // temperature (double of the float given)
  double lse_t;      // natural-log LSE of target row n
  double lse_q;      // natural-log LSE of draft row n (residual)
  double ln_c;       // saguaro: ln c
  double ln_Z;       // saguaro: ln Z of draft row n
  double K0;         // the exact key of one real candidate of this race (-inf: none known)
  float k2;          // fl(log2(e) / T)
  float cup;         // the word filter's offset for K0 (race_device.cuh); +inf keeps every token
  int ntop;          // saguaro: size of K (0 otherwise)
  int top[kMaxTopK]; // saguaro: K of draft row n
  int ref_seg;       // the segment of target row n holding its largest logit
};

// One race segment's result: the best and second-best exact keys and the winner.
struct __align__(16) RacePart {
  double best;
  double second;
  int idx;           // -1 if the segment had no survivor
  int pad;
};

// Vocabulary-sharded verification: one rank's race result for one request
// (exchanged between ranks; shard_verify.cu).
struct __align__(16) ShardRace {
  double best, second;    // the race of the request's kind on this rank's columns
  double bbest, bsecond;  // the bonus race there, when no column here was a residual candidate
  int idx, bidx;          // global token indices (-1: none)
  int kind, n;            // from the accept scan (identical on every rank)
  uint32_t flags;
  int pad;
};

// Byte offsets of one rank's exchange 1 (partials, top lists, owned logits of
// the draft tokens) and the sizes of both exchanges.
struct ShardLayout {
  size_t parts, tops, zx, x1, x2;
};

// Everything a kernel needs, passed by value.
struct VerifyArgs {
  const void* target;
  const void* draft;
  const int32_t* tokens;
  const int32_t* row_D;
  const float* temp_per_req;
  const int8_t* mode_per_req;
  int32_t* out_tokens;
  int32_t* out_al;
  float* out_row_lse;
  uint32_t* out_flags;
  int32_t* out_draft_top;  // [B, D_max, saguaro_k] optional: K of each saguaro draft row
  unsigned int* status;    // the device status word
  PartStat* pstat;         // [B, slots, nseg]
  TopPart* tpart;          // [B, D_max, nseg] (saguaro draft rows)
  RaceDesc* rdesc;         // [B] race descriptions (written by the scan)
  RacePart* rpart;         // [B, nseg * rsplit] race item results
  unsigned int* rcount;    // [B] race segments finished (zeroed by the scan)
  unsigned long long* best_key;  // [B] best exact race key so far, ordered bits (set by the scan)
  unsigned short* rorder;  // [B, nseg] race segments by descending largest logit (set by the scan)
  unsigned int* ticket;    // statistics tickets: 8 counters, 32 words apart (zero at launch)
  // the fused kernel's bookkeeping (zero at launch, except rowres)
  RowRes* rowres;          // [B, slots] merged rows
  unsigned int* rowcnt;    // [B, slots] statistics items finished per row
  unsigned int* reqcnt;    // [B] rows finished per request
  unsigned int* pubq;      // [B] published races in order, as request index + 1
  unsigned int* ctl;       // control words, one per 128-byte line (fused_verify.cu)
  uint64_t seed;
  int B, D_max, V, dtype;   // V: the row length (this shard's columns when sharded)
  int V_global;             // the vocabulary (V unless sharded)
  int vocab_offset;         // global index of column 0 (0 unless sharded; a multiple of 4)
  int nvec, nseg, slots;
  int mode;
  int per_request;         // after the statistics: 1 = one CTA per request, 0 = scan then race items
  int rsplit;              // race items per segment (1 or kMaxRaceSplit) in the race-items layout
  int race_sm_every;       // fused kernel: while statistics remain, only multiprocessors whose
                           // index is a multiple of this take race parts (0: every one)
  float temperature;
  int saguaro_k;
  float saguaro_c;
  uint32_t request_offset;
  const int32_t* parents;  // tree verification: [B, D_max] parent position of each node; NULL: linear
  int32_t* out_nodes;      // tree verification: [B, D_max] accepted nodes (optional)
  // early exit (early_exit.cu): rows are read position by position, only for
  // requests that accepted every earlier draft
  const uint64_t* seed_ptr;  // the seed in device memory, read by the kernels instead of `seed`; or NULL
  int* ee_n;               // [B] the decided position n (-1: parameter error); NULL: not used
  int* ee_alive;           // [2, B] the requests still accepting, by round parity
  unsigned int* ee_count;  // two counters 32 words apart: the lists' lengths
};

// Workspace layout (offsets in bytes from the workspace base, 256-aligned).
// [zero, total) must read zero when a fused launch starts.
struct WsLayout {
  size_t pstat, tpart, rdesc, rpart, rorder, rowres, ee, zero, rcount, best_key, rowcnt, reqcnt,
      pubq, ctl, ticket, total;
};

constexpr int kCtlWords = 8 * 32;  // the fused kernel's control words, 32 words (128 B) apart

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline int vec_elems(int dtype) { return dtype == kF32 ? 4 : 8; }

inline void row_geometry(int V, int dtype, int* nvec, int* nseg) {
  const int ve = vec_elems(dtype);
  *nvec = (V + ve - 1) / ve;
  *nseg = (*nvec + kSegVecs - 1) / kSegVecs;
}

inline WsLayout ws_layout(int B, int D_max, int V, int dtype, bool saguaro) {
  int nvec, nseg;
  row_geometry(V, dtype, &nvec, &nseg);
  const size_t slots = 2 * (size_t)D_max + 1;
  WsLayout L;
  size_t off = 0;
  L.pstat = off;
  off = align_up(off + (size_t)B * slots * nseg * sizeof(PartStat), 256);
  L.tpart = off;
  off = align_up(off + (saguaro ? (size_t)B * D_max * nseg * sizeof(TopPart) : 0), 256);
  L.rdesc = off;
  off = align_up(off + (size_t)B * sizeof(RaceDesc), 256);
  L.rpart = off;
  const size_t parts = (size_t)nseg * kMaxRaceSplit > (size_t)kClusterParts
                           ? (size_t)nseg * kMaxRaceSplit : (size_t)kClusterParts;
  off = align_up(off + (size_t)B * parts * sizeof(RacePart), 256);
  L.rorder = off;
  off = align_up(off + (size_t)B * nseg * sizeof(unsigned short), 256);
  L.rowres = off;
  off = align_up(off + (size_t)B * slots * sizeof(RowRes), 256);
  L.ee = off;  // early exit: decided positions [B], two alive lists [2, B], two counters
  off = align_up(off + (size_t)3 * B * sizeof(int) + 3 * 128, 256);  // counters on 128 B lines
  // everything from here on reads zero when a fused launch starts
  L.zero = off;
  L.rcount = off;
  off = align_up(off + (size_t)B * sizeof(unsigned int), 256);
  L.best_key = off;
  off = align_up(off + (size_t)B * sizeof(unsigned long long), 256);
  L.rowcnt = off;
  off = align_up(off + (size_t)B * slots * sizeof(unsigned int), 256);
  L.reqcnt = off;
  off = align_up(off + (size_t)B * sizeof(unsigned int), 256);
  L.pubq = off;
  off = align_up(off + (size_t)B * sizeof(unsigned int), 256);
  L.ctl = off;
  off = align_up(off + kCtlWords * sizeof(unsigned int), 256);
  L.ticket = off;
  off = align_up(off + 8 * 128, 256);  // eight counters, one 128-byte line each
  L.total = off;
  return L;
}

// ---------------------------------------------------------------- device helpers

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Streaming 16-byte load: read once, do not keep in L1.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation waits here until the kernel before it on the stream has
// completed and its writes are visible (it may be resident and set up before).
__device__ __forceinline__ void wait_for_previous_kernel() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Lets the next kernel on the stream (if launched for it) get resident now.
__device__ __forceinline__ void allow_next_kernel() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// bf16 halves of a 32-bit word as floats (exact widening).
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Float -> unsigned key whose unsigned order is the float order.
__device__ __forceinline__ uint32_t ordered_bits(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Key for "largest value, then lowest index": compare as unsigned 64-bit, max wins.
__device__ __forceinline__ unsigned long long value_index_key(float v, int idx) {
  return ((unsigned long long)ordered_bits(v) << 32) | (0xFFFFFFFFu - (uint32_t)idx);
}

__device__ __forceinline__ float key_value(unsigned long long k) {
  const uint32_t o = (uint32_t)(k >> 32);
  const uint32_t b = (o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o;
  return __uint_as_float(b);
}

__device__ __forceinline__ int key_index(unsigned long long k) {
  return (int)(0xFFFFFFFFu - (uint32_t)k);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

__device__ __forceinline__ int warp_min_int(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long w = __shfl_xor_sync(0xFFFFFFFFu, v, o);
    v = w > v ? w : v;
  }
  return v;
}

// Request parameters as the kernels read them.
struct ReqParams {
  int Db;
  int mode;
  float T;
  uint32_t err;  // kFlagBadRowD / kFlagBadParam found in the parameters
};

// The call's seed: from device memory when the caller keeps it there (so that
// a captured graph draws new numbers each replay), else the argument.
__device__ __forceinline__ uint64_t seed_of(const VerifyArgs& a) {
  return a.seed_ptr != nullptr ? *a.seed_ptr : a.seed;
}

__device__ __forceinline__ ReqParams load_req(const VerifyArgs& a, int b) {
  ReqParams r;
  r.Db = a.row_D ? __ldg(&a.row_D[b]) : a.D_max;
  r.mode = a.mode_per_req ? (int)__ldg(&a.mode_per_req[b]) : a.mode;
  r.T = a.temp_per_req ? __ldg(&a.temp_per_req[b]) : a.temperature;
  r.err = 0;
  if (r.Db < 0 || r.Db > a.D_max) r.err |= kFlagBadRowD;
  if (r.mode != kStochastic && r.mode != kGreedy && r.mode != kSaguaro) r.err |= kFlagBadParam;
  if (r.mode != kGreedy && !(r.T > 0.0f && r.T <= 3.0e38f)) r.err |= kFlagBadParam;
  if (r.mode != kGreedy && a.draft == nullptr && r.Db > 0) r.err |= kFlagBadParam;
  return r;
}

// Whether draft row d (position d) of request b is read: for a tree, only a
// position with a child (a node i < D_b hanging under it) has candidates to
// test; a linear batch tests every d < D_b.
__device__ __forceinline__ bool draft_row_read(const VerifyArgs& a, int b, int d, int Db) {
  if (d >= Db) return false;
  if (!a.parents) return true;
  const int32_t* par = a.parents + (size_t)b * a.D_max;
  for (int i = d; i < Db; ++i)
    if (__ldg(&par[i]) == d) return true;
  return false;
}

// Whether row `slot` of request b with parameters rp is read by the rule
// (target slots 0..D_max, draft slots D_max+1 ..).
__device__ __forceinline__ bool row_read(const VerifyArgs& a, int b, int slot, const ReqParams& rp) {
  if (rp.err) return false;
  if (slot <= a.D_max) return slot <= rp.Db;
  return rp.mode != kGreedy && draft_row_read(a, b, slot - a.D_max - 1, rp.Db);
}

// k2 = fl(log2(e) / T): the one scale every kernel applies to logits.
__device__ __forceinline__ float log2e_over_T(float T) { return __fdiv_rn(1.44269504088896341f, T); }

__device__ __forceinline__ const char* row_base(const VerifyArgs& a, int b, int slot) {
  const size_t es = a.dtype == kF32 ? 4 : 2;
  if (slot <= a.D_max)
    return (const char*)a.target + ((size_t)b * (a.D_max + 1) + slot) * (size_t)a.V * es;
  return (const char*)a.draft + ((size_t)b * a.D_max + (slot - a.D_max - 1)) * (size_t)a.V * es;
}

__device__ __forceinline__ float load_logit(const VerifyArgs& a, const char* row, int x) {
  if (a.dtype == kF32) return ((const float*)row)[x];
  return __uint_as_float((uint32_t)((const uint16_t*)row)[x] << 16);
}

}  // namespace sv

// Host-side launchers (one per kernel file), called from the C ABI.
namespace sv {
cudaError_t launch_row_stats(const VerifyArgs& a, cudaStream_t s, int grid, bool tickets);
bool row_stats_tickets(const VerifyArgs& a, int grid);
int row_stats_blocks_per_sm(int dtype);
cudaError_t launch_scan(const VerifyArgs& a, cudaStream_t s);
cudaError_t launch_race(const VerifyArgs& a, cudaStream_t s);
int race_split(int B, int nseg, int dtype, int sms);
// *seed += by on stream s (epilogue.cu; sv_advance_seed).
cudaError_t launch_advance_seed(uint64_t* seed, uint64_t by, cudaStream_t s);

// The early-exit rounds (early_exit.cu), before the usual finish with a.ee_n set.
cudaError_t launch_early_exit_rounds(const VerifyArgs& a, cudaStream_t s, int grid);
int ee_rounds(int D_max, int* bounds);

// One CTA per request, or a cluster of 2 or 4 while B times that fits two CTAs
// on each of the sms multiprocessors and the row has a segment for each of
// the cluster's warps.
cudaError_t launch_requests(const VerifyArgs& a, cudaStream_t s, int sms);
int request_cluster_size(int B, int nseg, int sms);
cudaError_t launch_fused(const VerifyArgs& a, cudaStream_t s, int grid);
int fused_blocks_per_sm(int dtype, int slots);
int fused_race_sm_every(const VerifyArgs& a, int grid);
cudaError_t launch_cluster(const VerifyArgs& a, cudaStream_t s);
// One cluster of up to 4 CTAs per request (as many as fit two CTAs per
// multiprocessor: sms of them).
cudaError_t launch_tree(const VerifyArgs& a, cudaStream_t s, int sms);
ShardLayout shard_layout(int B, int D_max, int V_local, int dtype);
cudaError_t launch_shard_z(const VerifyArgs& a, void* zx, cudaStream_t s);
cudaError_t launch_shard_tail(const VerifyArgs& a, const void* gathered1, int n_shards,
                              void* exchange2, cudaStream_t s);
cudaError_t launch_shard_finish(const void* gathered2, int B, int D_max, int n_shards,
                                int32_t* out_tokens, uint32_t* out_flags, unsigned* status,
                                cudaStream_t s);
int ssd_lookup_check(const int32_t* out_tokens, const int32_t* out_accept_len, int B, int D_max,
                     const int32_t* keys_al, const int32_t* keys_token, int K,
                     const int32_t* spec, int S, const int32_t* out_hit, const int32_t* out_spec,
                     const char** why);
cudaError_t launch_ssd_lookup(const int32_t* out_tokens, const int32_t* out_accept_len, int B,
                              int D_max, const int32_t* keys_al, const int32_t* keys_token, int K,
                              const int32_t* spec, int S, int32_t* out_hit, int32_t* out_spec,
                              cudaStream_t s);
int cluster_size(const VerifyArgs& a);
int epilogue_check(const int32_t* window, const int32_t* out_tokens, const int32_t* out_accept_len,
                   int B, int D_max, const int32_t* next_window, const int32_t* seq, int seq_cap,
                   const int32_t* seq_len, const char** why);
cudaError_t launch_epilogue(const int32_t* window, const int32_t* out_tokens,
                            const int32_t* out_accept_len, int B, int D_max, int32_t* next_window,
                            int32_t* seq, int seq_cap, int32_t* seq_len, uint32_t* flags,
                            unsigned* status, cudaStream_t s);
}  // namespace sv
