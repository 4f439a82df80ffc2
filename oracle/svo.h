/*
 * svo.h -- the ORACLE for speculative-decoding verification.
 *
 * TEST INFRASTRUCTURE ONLY.  This is a plain, slow, single-threaded (optionally
 * OpenMP-over-requests) CPU restatement of the verification rule in double
 * precision.  Only the test suite, the smoke check and the benchmark's CPU
 * baseline leg may load it.  It shares no code, header, table or constant
 * generator with the CUDA library, and it never calls it.
 *
 * Sources (cited by page title and section):
 *   [Sonar]  "Accélérer Sonar par la Spéculation" (Perplexity), sections
 *            "Décodage spéculatif", "Cible-Brouillon".
 *   [SSD]    "Speculative Speculative Decoding – асинхронизируй это." (x0ct.com),
 *            the numbered speculative-decoding rule (items 1-3 and the closing
 *            remark that the output is distributed like p) and the numbered
 *            saguaro recipe (items 1-3).
 *   [NV5]    "NVIDIA: öt irányelv gyorsíthatja az LLM-ek spekulatív
 *            dekódolását", section "Mit csinál a spekulatív dekódolás?"
 *            (accept in order until the first mismatch; AL in [1, 1+D]).
 *   Philox4x32-10: Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As
 *            Easy as 1, 2, 3", SC'11 (the published round function, multipliers
 *            and Weyl key schedule).
 *
 * Readings taken where the pages are silent or garbled are listed in the
 * project's design notes and repeated at the function that applies them.
 */
#ifndef SVO_H
#define SVO_H
#include <stdint.h>
#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { SVO_F32 = 0, SVO_BF16 = 1 };
enum { SVO_STOCHASTIC = 0, SVO_GREEDY = 1, SVO_SAGUARO = 2 };

/* per-request flag bits written to out_flags[b] */
enum {
  SVO_FLAG_ACCEPT_NEAR_TIE = 1u << 0, /* some tested position had |u - a| < 1e-5 */
  SVO_FLAG_RACE_NEAR_TIE = 1u << 1,   /* top-2 race keys closer than 1e-6 (log space) */
  SVO_FLAG_RESIDUAL_EMPTY = 1u << 2,  /* {p > q} was empty; sampled from p instead */
  SVO_FLAG_BAD_TOKEN = 1u << 8,       /* a tested draft token outside [0, V) */
  SVO_FLAG_BAD_ROW_D = 1u << 9,       /* row_D[b] outside [0, D_max] */
  SVO_FLAG_NONFINITE = 1u << 10       /* NaN or +inf in a needed row, or a row all -inf */
};

/* Published Philox4x32-10 bijection: counter ctr[4], key key[2] -> out[4]. */
void svo_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);

/* Accept uniform u for (seed, global request g, position d): word 0 of
 * Philox(key = seed, counter = (d, g, 0, 0)), top 24 bits, times 2^-24. */
double svo_accept_uniform(uint64_t seed, uint32_t g, uint32_t d);

/* Race exponential E for (seed, global request g, token x):
 * word (x mod 4) of Philox(key = seed, counter = (x / 4, g, 1, 0)) = o,
 * W = (o + 1/2) 2^-32, E = -ln(1 - W). */
double svo_race_exponential(uint64_t seed, uint32_t g, uint32_t x);

/* Log-sum-exp of one row at temperature T: ln sum_x exp(z_x / T), double.
 * Returns -inf for a row whose every entry is -inf. */
double svo_row_lse(const void* row, int V, int dtype, double T);

/* Lowest index of the largest raw logit. */
int svo_row_argmax(const void* row, int V, int dtype);

typedef struct {
  const float* temperature_per_req; /* [B] or NULL */
  const int8_t* mode_per_req;       /* [B] or NULL: per-request mode overrides */
  int saguaro_k;                    /* <= 0 -> 5 */
  double saguaro_c;                 /* <= 0 -> 0.5 */
  uint32_t request_offset;          /* global index of request 0 (sharding) */
} svo_params;

/*
 * The whole verification step for B requests.
 *   target  [B, D_max+1, V] dtype;  draft [B, D_max, V] dtype (may be NULL only
 *   if every request is greedy);  tokens [B, D_max];  row_D [B] or NULL (= D_max).
 * Outputs (all caller-owned, host):
 *   out_tokens [B, D_max+1], out_accept_len [B], out_flags [B] (may be NULL),
 *   out_row_lse [B, 2*D_max+1] (may be NULL): slots 0..D_max are target rows,
 *   slots D_max+1 .. 2*D_max draft rows; NaN where a row is not used.
 * nthreads: 1 = plain single-threaded loop; > 1 = the same loop split over
 * requests with OpenMP when the library was built with it.
 * Returns 0, or -1 for invalid arguments.
 */
int svo_verify(const void* target, const void* draft, const int32_t* tokens,
               const int32_t* row_D, int B, int D_max, int V, int dtype,
               float temperature, int mode, uint64_t seed, const svo_params* params,
               int32_t* out_tokens, int32_t* out_accept_len, uint32_t* out_flags,
               double* out_row_lse, int nthreads);

/*
 * The step after verification, on the host ("Accélérer Sonar par la
 * Spéculation", section "Calendrier MTP pour un jeton unique": the target's
 * input tokens are shifted and the next target token is inserted at its slot,
 * so the next run needs no CPU sync; the accepted length sets the next
 * sequence length).  For request b with AL = accept_len[b] and n = AL - 1:
 *   next_window[b][j] = window[b][j + 1] for j < D_max, next_window[b][D_max] = -1,
 *   then next_window[b][n] = out_tokens[b][n]          (when next_window != NULL)
 *   seq[b][seq_len[b] + j] = out_tokens[b][j] for j < AL, seq_len[b] += AL
 *                                                      (when seq != NULL)
 * A request with AL outside [1, D_max + 1] (an error flagged by the
 * verification) gets a next-window row of -1 and no append; one whose append would pass seq_cap
 * gets its next-window row but no append, and its bit in *full (when full is
 * not NULL) is set: full[b / 32] |= 1 << (b % 32).
 * Arrays: window, next_window [B, D_max+1]; out_tokens [B, D_max+1];
 * accept_len, seq_len [B]; seq [B, seq_cap].  Returns 0, or -1 for invalid
 * arguments.
 */
int svo_epilogue(const int32_t* window, const int32_t* out_tokens, const int32_t* accept_len,
                 int B, int D_max, int32_t* next_window, int32_t* seq, int seq_cap,
                 int32_t* seq_len, uint32_t* full);

/*
 * The k largest logits of a row, by (logit descending, index ascending):
 * idx[0..k-1].  ("Speculative Speculative Decoding – асинхронизируй это.",
 * saguaro recipe item 1: the draft's most likely tokens.)  k <= V.
 */
void svo_row_topk(const void* row, int V, int dtype, int k, int* idx);

/*
 * Outcome lookup of speculative speculative decoding ("Speculative Speculative
 * Decoding – асинхронизируй это.": while the target verifies, the draft
 * predicts likely verification outcomes and prepares speculations for them; if
 * the actual outcome is in the prepared set, its speculation is returned at
 * once -- the cache hit of the page's restaurant analogy -- else it is a miss).
 * The outcome of request b is (AL, token) = (accept_len[b], out_tokens[b][AL-1]);
 * the prepared set is keys_al[b][0..K-1], keys_token[b][0..K-1].
 *   out_hit[b] = the lowest k with keys_al[b][k] == AL and keys_token[b][k] ==
 *                token, else -1 (also -1 when AL lies outside [1, D_max + 1]);
 *   out_spec[b][0..S-1] = spec[b][out_hit[b]][0..S-1] on a hit, else -1
 *                (when out_spec and spec are not NULL).
 * Returns 0, or -1 for invalid arguments.
 */
int svo_ssd_lookup(const int32_t* out_tokens, const int32_t* accept_len, int B, int D_max,
                   const int32_t* keys_al, const int32_t* keys_token, int K, const int32_t* spec,
                   int S, int32_t* out_hit, int32_t* out_spec);

/*
 * Tree (multi-candidate) verification ("Accélérer Sonar par la Spéculation",
 * section "EAGLE": draft trees whose nodes hold several candidate tokens, the
 * top candidates at each node).  Request b has n = n_nodes[b] (or N_max) draft
 * nodes; node i holds token tokens[b][i] and hangs under position
 * parents[b][i] in [0, i] (position 0 is the root -- the last committed token --
 * and position i + 1 is node i).  Target row p of [B, N_max+1, V] is the
 * target's distribution after position p's path; draft row p of
 * [B, N_max, V] is the distribution position p's children were drawn from
 * (only rows of positions with children are read).
 * The walk from the root: at position p with children c_1 < c_2 < ... (node
 * order), with P = p_p (softmax of target row p at T) and q = q_p:
 *   candidate c_j is accepted with probability min(1, P(x)/q(x)), x its token,
 *   u from Philox at counter (c_j, g, 0, 0); accepted -> its token is emitted
 *   and the walk moves to position c_j + 1; rejected -> P = norm(max(0, P - q))
 *   and the next candidate is tried;
 *   every candidate rejected -> a token is drawn from P by the race and the
 *   walk ends; no candidate at all -> the bonus token is drawn from p_p.
 * Greedy: the first child whose token is the argmax of target row p is
 * accepted; otherwise that argmax is emitted and the walk ends.
 * Outputs: out_tokens [B, N_max+1] (the accepted tokens, then the drawn one,
 * then -1), out_accept_len [B] (AL), out_nodes [B, N_max] (the accepted nodes,
 * then -1; may be NULL), out_flags [B] (may be NULL).  A parent outside
 * [0, i] sets SVO_FLAG_BAD_PARAM (1 << 11); other errors as svo_verify.
 * Returns 0, or -1 for invalid arguments.
 */
int svo_verify_tree(const void* target, const void* draft, const int32_t* tokens,
                    const int32_t* parents, const int32_t* n_nodes, int B, int N_max, int V,
                    int dtype, float temperature, int mode, uint64_t seed,
                    uint32_t request_offset, int32_t* out_tokens, int32_t* out_accept_len,
                    int32_t* out_nodes, uint32_t* out_flags, int nthreads);

/* 1 when built with OpenMP, else 0. */
int svo_has_openmp(void);

#ifdef __cplusplus
}
#endif
#endif
