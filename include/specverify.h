/*
 * specverify.h -- libspecverify: the speculative-decoding verification step on
 * NVIDIA B200 (sm_100a), as a C ABI.
 *
 * What the step computes (sources cited by page title and section):
 *   [Sonar] "Accélérer Sonar par la Spéculation" (Perplexity):
 *           section "Décodage spéculatif" -- the target scores every drafted
 *           prefix in one pass (row d of the target logits is its distribution
 *           for draft token d) and gives one extra token (n drafts -> up to n+1
 *           tokens); section "Cible-Brouillon" -- the sampler finds the accepted
 *           length by comparing the full draft and target distributions, and the
 *           target's next logits are sampled for the extra token.
 *   [SSD]   "Speculative Speculative Decoding – асинхронизируй это." (x0ct.com):
 *           the numbered rule -- accept when q(x) <= p(x); otherwise accept with
 *           probability p(x)/q(x) (the page's "reject with probability p/q" is
 *           read as the acceptance probability, the only reading under which the
 *           output is distributed like p, as the page's closing remark states);
 *           on rejection draw from norm(max(0, p - q)).  The saguaro recipe:
 *           take the draft's five most likely tokens and lower their
 *           probabilities (read: multiply by c, renormalise) for drafting and
 *           for the residual.
 *   [NV5]   "NVIDIA: öt irányelv gyorsíthatja az LLM-ek spekulatív dekódolását",
 *           section "Mit csinál a spekulatív dekódolás?" -- accept the drafts in
 *           order until the first mismatch; the accepted length AL lies in
 *           [1, 1 + D]; greedy verification reproduces ordinary decoding.
 *
 * The rule, per request b with D_b drafts x_0..x_{D_b-1} and temperature T:
 *   p_d = softmax(target[b, d, :] / T),  q_d = softmax(draft[b, d, :] / T)
 *   (saguaro: q'_d(x) = q_d(x) c^[x in K_d] / Z_d, K_d the k largest draft
 *    logits, Z_d = 1 - (1 - c) sum_{x in K_d} q_d(x); q' replaces q below)
 *   a_d = min(1, p_d(x_d) / q_d(x_d));  u_d = Philox uniform (below)
 *   n = first d with u_d >= a_d, else D_b;  AL = n + 1
 *   token n = residual race on (p_n, q_n) if n < D_b, else bonus race on p_{D_b}
 *   race: argmax over candidates x of r(x) / E_x, E_x unit exponentials
 *     residual: r = p - q over {p > q};  bonus: r = p over {p > 0}
 *     (if {p > q} is empty through rounding, the bonus race runs on p_n)
 *   greedy: accept while x_d == argmax target[b, d, :]; token n = that argmax
 *
 * Random numbers (a convention of this library; the pages fix none):
 *   Philox4x32-10 (Salmon et al., SC'11) with key (seed mod 2^32, seed >> 32).
 *   u_d: word 0 at counter (d, g, 0, 0), top 24 bits times 2^-24.
 *   E_x: word (x mod 4) at counter (x / 4, g, 1, 0) = o, W = (o + 1/2) 2^-32,
 *        E_x = -ln(1 - W).
 *   g = request_offset + b is the request's global index, so a batch split
 *   across devices gives the same results as one call.  The caller changes
 *   `seed` between decoding steps.
 *
 * Ties: argmax, top-k and the race keep the lowest token index.
 *
 * Conventions for every entry point:
 *   - All array arguments are DEVICE pointers on the current CUDA device,
 *     row-major and contiguous; the caller owns every buffer.
 *   - Calls are asynchronous on the stream (sv_params.stream, default: the
 *     legacy default stream) and never synchronise.  Calls without their own
 *     workspace share the library's cached one on their device, so they must
 *     not overlap on the GPU: run them on one stream, or pass each its own
 *     workspace (sv_params.workspace).
 *   - Host-detectable argument errors return a negative code, launch nothing
 *     and leave the outputs untouched; sv_last_error() describes the error.
 *   - Errors found on the device (a draft token outside [0, V), row_D[b]
 *     outside [0, D_max], NaN or +inf in a row the rule reads, a row that is
 *     all -inf, a per-request temperature <= 0 or mode out of range) set bits
 *     in the library's device status word and in that request's flags, and
 *     that request's outputs are all -1.  No kernel traps or asserts.
 *   - A logit of -inf masks its token (p = 0).
 *   - Rows beyond a request's D_b (and draft rows of greedy requests) are
 *     never read; they may hold anything, NaN included.
 */
#ifndef SPECVERIFY_H
#define SPECVERIFY_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SV_API __attribute__((visibility("default")))
#else
#define SV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* dtype of the logits */
enum { SV_F32 = 0, SV_BF16 = 1 };

/* verification mode */
enum { SV_STOCHASTIC = 0, SV_GREEDY = 1, SV_SAGUARO = 2 };

/* return codes */
enum { SV_OK = 0, SV_ERR_INVALID_ARG = -1, SV_ERR_UNSUPPORTED = -2, SV_ERR_CUDA = -3 };

/* sv_params.variant: the launch structure, optionally OR-ed
 * with one layout of the work after the statistics pass (both layouts give the
 * same results; without one, the library takes ITEMS when B is below four
 * fifths of the device's multiprocessor count and B times the row's 8 KiB
 * segments is above that count, and PER_REQUEST otherwise):
 *   SV_TAIL_PER_REQUEST: one CTA per request merges, scans and races it;
 *   SV_TAIL_ITEMS: one CTA per request merges and scans, then one warp per
 *     (request, segment of the sampled row) races -- per half segment while
 *     those items fit in one wave of the device's resident warps.
 * The structures (all give the same results):
 *   SV_VARIANT_SPLIT: a persistent statistics kernel, then the layout above;
 *   SV_VARIANT_FUSED: one persistent launch in which each request's merge,
 *     scan and race run beside the statistics of later requests;
 *   SV_VARIANT_CLUSTER: one launch, one thread-block cluster (up to 8 CTAs) per
 *     request doing its statistics, merges, scan and race between cluster
 *     barriers;
 *   SV_VARIANT_EARLY_EXIT: the rows read position by position, in rounds
 *     (position 0, then 1-2, then 3 to D_max), each round only for the requests
 *     that accepted every earlier draft, then the layout above; the rule's
 *     rows after the first rejection are never read.  Same tokens, accepted
 *     lengths and flags as SPLIT, except that the rows of the positions past
 *     the outcome get no LSE (out_row_lse NaN), and those never read no
 *     SV_FLAG_NONFINITE check.  Source: the rule
 *     stops at the first rejection ("Speculative Speculative Decoding –
 *     асинхронизируй это.", rule items 1-2);
 *   SV_VARIANT_AUTO: the library's choice for the shape (never EARLY_EXIT,
 *     whose outputs differ in out_row_lse). */
enum {
  SV_VARIANT_AUTO = 0,
  SV_VARIANT_SPLIT = 1,
  SV_VARIANT_FUSED = 2,
  SV_VARIANT_CLUSTER = 3,
  SV_VARIANT_EARLY_EXIT = 4
};
enum { SV_TAIL_PER_REQUEST = 1 << 4, SV_TAIL_ITEMS = 1 << 5 };

/* per-request flag bits (sv_params.out_flags) */
enum {
  SV_FLAG_ACCEPT_NEAR_TIE = 1u << 0, /* a tested position had |u - a| < 1e-5 */
  SV_FLAG_RACE_NEAR_TIE = 1u << 1,   /* top-2 race keys ln r - ln E within 1e-6 */
  SV_FLAG_RESIDUAL_EMPTY = 1u << 2,  /* {p > q} empty: the token came from p */
  SV_FLAG_BAD_TOKEN = 1u << 8,
  SV_FLAG_BAD_ROW_D = 1u << 9,
  SV_FLAG_NONFINITE = 1u << 10,
  SV_FLAG_BAD_PARAM = 1u << 11,
  SV_FLAG_SEQ_FULL = 1u << 13        /* sv_epilogue: the append would pass seq_cap (skipped) */
};

/* device status word bits (sv_get_device_status): the union of the error
 * flags of every request since the word was last cleared, and
 * SV_STATUS_TIMEOUT: a bounded wait of the fused kernel expired (about two
 * seconds; the warps that gave up left, and that call's outputs are
 * undefined); the context stays usable. */
enum {
  SV_STATUS_BAD_TOKEN = SV_FLAG_BAD_TOKEN,
  SV_STATUS_BAD_ROW_D = SV_FLAG_BAD_ROW_D,
  SV_STATUS_NONFINITE = SV_FLAG_NONFINITE,
  SV_STATUS_BAD_PARAM = SV_FLAG_BAD_PARAM,
  SV_STATUS_RESIDUAL_EMPTY = SV_FLAG_RESIDUAL_EMPTY,
  SV_STATUS_TIMEOUT = 1u << 12,
  SV_STATUS_SEQ_FULL = SV_FLAG_SEQ_FULL
};

/* Limits checked on the host. */
#define SV_MAX_DRAFT 32  /* D_max <= 32 */
#define SV_MAX_SAGUARO_K 8

/* The step after verification, run on the device by sv_epilogue or by
 * sv_verify_ex when sv_params.epilogue is set (see sv_epilogue). */
typedef struct sv_epilogue_args {
  const int32_t* window;   /* [B, D_max+1] device: the verified input window of each request
                              (its last committed token, then its draft slots); may be NULL
                              when next_window is NULL */
  int32_t* next_window;    /* [B, D_max+1] device, optional: the shifted window with the
                              emitted target token inserted; may be `window` itself */
  int32_t* seq;            /* [B, seq_cap] device, optional: each request's token sequence */
  int seq_cap;             /* tokens per row of seq */
  int32_t* seq_len;        /* [B] device, in/out: each request's sequence length (with seq) */
} sv_epilogue_args;

/*
 * Optional parameters.  Zero-initialise, then set what you need.
 */
typedef struct sv_params {
  void* stream;                      /* cudaStream_t; NULL = legacy default stream */
  const float* temperature_per_req;  /* [B] device; NULL: every request uses `temperature` */
  const int8_t* mode_per_req;        /* [B] device; NULL: every request uses `mode` */
  int saguaro_k;                     /* size of K; <= 0 means 5; at most SV_MAX_SAGUARO_K */
  float saguaro_c;                   /* down-weighting factor in (0, 1]; <= 0 means 0.5 */
  int variant;                       /* SV_VARIANT_* [| SV_TAIL_*]; AUTO picks per shape */
  uint32_t request_offset;           /* global index of request 0 (sharded batches) */
  float* out_row_lse;                /* [B, 2*D_max+1] device, optional: natural-log LSE of
                                        target rows (slots 0..D_max) and draft rows (slots
                                        D_max+1..2*D_max) at temperature T; NaN where the row
                                        is not used (greedy requests, rows beyond D_b) */
  uint32_t* out_flags;               /* [B] device, optional: SV_FLAG_* per request */
  void* workspace;                   /* optional caller scratch (device, 256-byte aligned);
                                        NULL: a per-device cache grown on demand with
                                        cudaMalloc and freed by sv_shutdown */
  size_t workspace_bytes;            /* size of `workspace`; >= sv_workspace_bytes(...) */
  void* timing_events;               /* optional cudaEvent_t[2]: recorded on the stream
                                        immediately before and after the row-statistics
                                        kernel (split) or the fused kernel (fused) */
  int32_t* out_draft_top;            /* [B, D_max, k] device, optional (k = min(saguaro_k, V)):
                                        for each saguaro request, the k largest logits of each
                                        draft row it tested (logit desc, index asc), the keys
                                        of sv_ssd_lookup; -1 elsewhere */
  const sv_epilogue_args* epilogue;  /* optional: after the verification, on the same stream,
                                        the step sv_epilogue describes, on this call's
                                        out_tokens / out_accept_len (and out_flags, which get
                                        SV_FLAG_SEQ_FULL); host struct, read during the call */
  const uint64_t* seed_device;       /* optional device pointer: the seed is read from here when
                                        the kernels run (the `seed` argument is then unused), so
                                        that a captured graph draws new numbers on each replay
                                        once the value is advanced (sv_advance_seed) */
} sv_params;

/*
 * sv_verify: the whole verification step for B requests.
 *   target_logits  [B, D_max+1, V] of dtype; row d scores draft token d, row D_b is
 *                  the bonus row                       ([Sonar] "Décodage spéculatif")
 *   draft_logits   [B, D_max, V] of dtype; may be NULL only if every request is greedy
 *   draft_tokens   [B, D_max] int32; entries at d >= D_b are ignored
 *   row_D          [B] int32, D_b in [0, D_max]; NULL means D_max for every request
 *   B >= 0, 0 <= D_max <= SV_MAX_DRAFT, V >= 1, dtype SV_F32 or SV_BF16
 *   temperature    > 0 and finite unless every request is greedy
 *   mode           SV_STOCHASTIC, SV_GREEDY or SV_SAGUARO
 *   seed           Philox key for this step
 *   out_tokens     [B, D_max+1] int32: the accepted drafts x_0..x_{n-1}, then the
 *                  sampled token at slot n, then -1
 *   out_accept_len [B] int32: AL = n + 1 in [1, 1 + D_b]   ([NV5] "Mit csinál...")
 * Returns SV_OK or a negative code.
 */
SV_API int sv_verify(const void* target_logits, const void* draft_logits, const int32_t* draft_tokens,
              const int32_t* row_D, int B, int D_max, int V, int dtype, float temperature,
              int mode, uint64_t seed, int32_t* out_tokens, int32_t* out_accept_len);

/* Greedy verification ([NV5]: same output as ordinary argmax decoding).  Draft
 * logits are never read; T is not used.  Same layout as sv_verify. */
SV_API int sv_verify_greedy(const void* target_logits, const int32_t* draft_tokens,
                     const int32_t* row_D, int B, int D_max, int V, int dtype,
                     int32_t* out_tokens, int32_t* out_accept_len);

/* sv_verify with optional parameters (p may be NULL).
 * CUDA graphs: every call only enqueues work on sv_params.stream, so a decode
 * loop can capture its calls (with their epilogues) by stream capture and
 * replay them; the pointers are fixed at capture, and so is the seed unless
 * it is read from sv_params.seed_device, which a captured sv_advance_seed can
 * advance between the calls so that each replay draws new numbers.  Make one call
 * on the device before capturing (the first call does one-time device
 * queries), and pass sv_params.workspace, or capture only after a call of at
 * least the same sizes (the cached workspace grows with cudaMalloc, which a
 * capture does not allow).  sv_get_device_status synchronises: call it
 * outside the graph. */
SV_API int sv_verify_ex(const void* target_logits, const void* draft_logits,
                 const int32_t* draft_tokens, const int32_t* row_D, int B, int D_max, int V,
                 int dtype, float temperature, int mode, uint64_t seed, int32_t* out_tokens,
                 int32_t* out_accept_len, const sv_params* p);

/*
 * sv_verify_tree: tree (multi-candidate) verification ("Accélérer Sonar par la
 * Spéculation", section "EAGLE": the draft proposes a tree whose nodes hold
 * several candidate tokens).  Request b has n = n_nodes[b] (NULL: N_max) nodes;
 * node i holds node_tokens[b][i] and hangs under position parents[b][i] in
 * [0, i]: position 0 is the root (the last committed token), position i + 1 is
 * node i.  target_logits [B, N_max+1, V]: row p is the target's distribution
 * after position p's path; draft_logits [B, N_max, V]: row p is the
 * distribution position p's candidates were drawn from (read only for
 * positions with candidates; NULL allowed when greedy).
 * From the root, at position p the candidates under p are tried in node
 * order: candidate j is accepted with probability min(1, P_j(x)/q_p(x)) (u_j
 * from Philox at counter (node, g, 0, 0)), P_0 = p_p and a rejection replaces
 * P_j by norm(max(0, P_j - q_p)) ("Speculative Speculative Decoding", rule
 * items 1-3, applied recursively); an accepted candidate's token is emitted and
 * the walk moves to its position; after the last candidate the token is drawn
 * from the residual by the exponential race, and at a position with no
 * candidate the bonus token is drawn from p_p.  Greedy (mode SV_GREEDY): the
 * first candidate holding the argmax of target row p is accepted, otherwise
 * that argmax is emitted.  A chain (parents[b][i] == i) is sv_verify's rule.
 * Outputs: out_tokens [B, N_max+1] (the accepted path's tokens, then the drawn
 * token, then -1), out_accept_len [B] (AL = path length + 1), out_nodes
 * [B, N_max] (optional: the accepted nodes, then -1), and sv_params'
 * out_flags / out_row_lse.  mode: SV_STOCHASTIC or SV_GREEDY (per-request
 * modes likewise; saguaro requests are flagged SV_FLAG_BAD_PARAM, as are
 * parents outside [0, i]).  sv_params.variant, .epilogue and .out_draft_top
 * are ignored.  Otherwise as sv_verify_ex.
 */
SV_API int sv_verify_tree(const void* target_logits, const void* draft_logits,
                          const int32_t* node_tokens, const int32_t* parents,
                          const int32_t* n_nodes, int B, int N_max, int V, int dtype,
                          float temperature, int mode, uint64_t seed, int32_t* out_tokens,
                          int32_t* out_accept_len, int32_t* out_nodes, const sv_params* p);

/*
 * sv_verify_static: sv_verify_ex that allocates nothing.  (The pages have no
 * counterpart; this is a service for callers.)
 *
 * For callers that must not allocate device memory, e.g. because the process's
 * memory already belongs to a caching allocator that the library must not
 * bypass, or because cudaMalloc/cudaFree can synchronise the device in a
 * latency-critical decode loop.  The caller still passes every input and
 * output; the scratch is a fixed array of SV_STATIC_WORKSPACE_BYTES in the
 * library's own device memory, which every GPU that loads the library keeps
 * until the process exits.  sv_params.workspace and workspace_bytes are ignored.
 *   - Sizes whose sv_workspace_bytes(B, D_max, V, dtype) exceeds
 *     SV_STATIC_WORKSPACE_BYTES are rejected with SV_ERR_UNSUPPORTED (nothing
 *     launched; sv_last_error says why).  8 MiB covers B=256, D=7, V=128256.
 *   - The first call on a device looks up the array's device address (and does
 *     the same one-time device queries as sv_verify_ex); make that first call
 *     before any stream capture.
 *   - Every call shares the one array and it keeps the last call's contents;
 *     each call clears what must start at zero itself.  Calls that overlap on
 *     the GPU (other streams, other host threads) race on it: run them on one
 *     stream, or give each its own workspace through sv_verify_ex.
 * Otherwise identical to sv_verify_ex (same arguments, results and errors).
 */
#define SV_STATIC_WORKSPACE_BYTES (8u << 20)
SV_API int sv_verify_static(const void* target_logits, const void* draft_logits,
                            const int32_t* draft_tokens, const int32_t* row_D, int B, int D_max,
                            int V, int dtype, float temperature, int mode, uint64_t seed,
                            int32_t* out_tokens, int32_t* out_accept_len, const sv_params* p);

/*
 * sv_epilogue: the step after verification, on the device, so that the next
 * decoding step needs no GPU-to-CPU sync ("Accélérer Sonar par la
 * Spéculation", section "Calendrier MTP pour un jeton unique": the target's
 * input tokens are shifted and a kernel inserts the next target tokens at
 * their slots; section "Inférence avec décodage spéculatif": the accepted
 * length sets the next sequence length).  Per request b with
 * AL = out_accept_len[b] and n = AL - 1:
 *   next_window[b][j] = window[b][j + 1] for j < D_max; next_window[b][D_max] = -1;
 *   then next_window[b][n] = out_tokens[b][n] (the correction or bonus token).
 *   So next_window[b][0..n] are the AL emitted tokens, and the slots after n
 *   keep the drafts that were not accepted (the draft model may re-run on the
 *   whole window; their results are simply not used).
 *   seq[b][seq_len[b] + j] = out_tokens[b][j] for j < AL; seq_len[b] += AL.
 * A request whose AL lies outside [1, D_max + 1] (the verification flagged an
 * error for it) gets a next-window row of -1 and no append.  An append that
 * would pass seq_cap (or a negative seq_len) is skipped and sets
 * SV_FLAG_SEQ_FULL in flags[b] (when flags is not NULL) and in the device
 * status word.  All arrays are device arrays the caller owns; next_window and
 * seq may each be NULL (that part is skipped).  Asynchronous on `stream`
 * (cudaStream_t, NULL = legacy default); host-detectable errors return a
 * negative code and launch nothing.
 */
SV_API int sv_epilogue(const int32_t* window, const int32_t* out_tokens,
                       const int32_t* out_accept_len, int B, int D_max, int32_t* next_window,
                       int32_t* seq, int seq_cap, int32_t* seq_len, uint32_t* flags, void* stream);

/*
 * sv_ssd_lookup: the outcome lookup of speculative speculative decoding
 * ("Speculative Speculative Decoding – асинхронизируй это.": while the target
 * verifies, the draft predicts likely verification outcomes and prepares a
 * speculation for each; an outcome found among them returns its speculation at
 * once -- the page's cache hit -- and any other is a miss).  The outcome of
 * request b is (AL, token) = (out_accept_len[b], out_tokens[b][AL - 1]); its
 * prepared set is keys_al[b][0..K-1], keys_token[b][0..K-1] (typically AL = d+1
 * with the draft's top tokens at position d, sv_params.out_draft_top, on which
 * saguaro sampling concentrates the correction).
 *   out_hit[b]  = the lowest k with keys_al[b][k] == AL and keys_token[b][k] ==
 *                 token; -1 if none, or if AL lies outside [1, D_max + 1].
 *   out_spec[b] = spec[b][out_hit[b]][0..S-1] on a hit, else S values of -1
 *                 (optional: out_spec and spec may be NULL).
 * Arrays (device, caller-owned): out_tokens [B, D_max+1], out_accept_len,
 * out_hit [B], keys_al, keys_token [B, K], spec [B, K, S], out_spec [B, S].
 * Asynchronous on `stream`; host-detectable errors return a negative code. */
SV_API int sv_ssd_lookup(const int32_t* out_tokens, const int32_t* out_accept_len, int B,
                         int D_max, const int32_t* keys_al, const int32_t* keys_token, int K,
                         const int32_t* spec, int S, int32_t* out_hit, int32_t* out_spec,
                         void* stream);

/*
 * Verification with the vocabulary split across ranks (tensor-parallel logits):
 * rank r of n_shards holds columns [r V_local, (r + 1) V_local) of every target
 * and draft row, as [B, D_max+1, V_local] and [B, D_max, V_local] arrays; draft
 * tokens and every token the calls write are global indices in
 * [0, n_shards V_local).  ("Accélérer Sonar par la Spéculation", section
 * "Calendrier Brouillon-Cible": the verification batch is synchronised with
 * the tensor-parallel workers.)  Three calls per rank, with two all-gathers of
 * byte buffers in rank order between them (the caller's collectives, e.g.
 * NCCL over NVLink):
 *   sv_shard_stats   -> exchange1 (sv_shard_exchange_bytes(.., 1) bytes per rank):
 *                       the statistics of this rank's columns and the logits of
 *                       the draft tokens it owns;
 *   all-gather exchange1 of every rank -> gathered1 (n_shards x those bytes);
 *   sv_shard_race    -> out_tokens (accepted prefix), out_accept_len, and
 *                       sv_params' out_flags / out_row_lse / out_draft_top, the
 *                       same on every rank; exchange2 (.., 2 bytes): this rank's
 *                       race result per request;
 *   all-gather exchange2 -> gathered2;
 *   sv_shard_finish  -> the token at slot AL-1 of out_tokens (and out_flags).
 * The accept decisions and the tokens follow the same rule, the same random
 * numbers (the race's Philox words are those of the global token indices) and
 * the same tie rules as sv_verify_ex on the whole rows; the statistics are
 * merged over every rank's segments in global order, so they differ from an
 * unsharded call only in rounding.  V_local must be a multiple of 4; every rank
 * passes the same B, D_max, V_local, dtype, mode, seed and per-request arrays.
 * sv_params.variant and .epilogue are ignored (run sv_epilogue afterwards).
 * The calls use the library's workspace like sv_verify_ex; none synchronises. */
SV_API size_t sv_shard_exchange_bytes(int B, int D_max, int V_local, int dtype, int stage);
SV_API int sv_shard_stats(const void* target_local, const void* draft_local,
                          const int32_t* draft_tokens, const int32_t* row_D, int B, int D_max,
                          int V_local, int dtype, float temperature, int mode, uint64_t seed,
                          int n_shards, int shard, const sv_params* p, void* exchange1);
SV_API int sv_shard_race(const void* target_local, const void* draft_local,
                         const int32_t* draft_tokens, const int32_t* row_D, int B, int D_max,
                         int V_local, int dtype, float temperature, int mode, uint64_t seed,
                         int n_shards, int shard, const sv_params* p, const void* gathered1,
                         int32_t* out_tokens, int32_t* out_accept_len, void* exchange2);
SV_API int sv_shard_finish(int B, int D_max, int n_shards, const void* gathered2,
                           int32_t* out_tokens, const sv_params* p);

/* Enqueues *seed_device += by on `stream` (cudaStream_t, NULL = legacy
 * default): between captured verification calls that read their seed from
 * sv_params.seed_device, so that each replay of a graph draws new numbers.
 * seed_device: device pointer, 8-byte aligned, owned by the caller.
 * SV_ERR_INVALID_ARG for NULL or a misaligned pointer; SV_ERR_CUDA if the
 * launch fails.  No passage of the pages defines this call: it serves decode
 * loops that replay the verification step of "Accélérer Sonar par la
 * Spéculation" (section "Inférence avec décodage spéculatif": the step runs
 * once per generated window) from a captured graph. */
SV_API int sv_advance_seed(uint64_t* seed_device, uint64_t by, void* stream);

/* Bytes of scratch one call with these sizes needs (for sv_params.workspace). */
SV_API size_t sv_workspace_bytes(int B, int D_max, int V, int dtype);

/* Synchronises `stream` (cudaStream_t, NULL = legacy default), copies the device
 * status word of the current device into *status_bits and clears it.
 * Returns SV_OK or SV_ERR_CUDA. */
SV_API int sv_get_device_status(void* stream, uint32_t* status_bits);

/* Message for the last error returned on this host thread ("" if none). */
SV_API const char* sv_last_error(void);

/* Frees the cached per-device workspaces.  Call with no call in flight. */
SV_API void sv_shutdown(void);

/* Library version, major*10000 + minor*100 + patch. */
SV_API int sv_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SPECVERIFY_H */
