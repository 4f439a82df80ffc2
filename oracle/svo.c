/*
 * svo.c -- the ORACLE for speculative-decoding verification (test
 * infrastructure only; see svo.h for who may use it and for the sources).
 *
 * Everything here is the plain definition, written out in double precision
 * with no blocking, fusion or reordering: one request at a time, one row at a
 * time, one token at a time.  Where the pages leave a step open, the reading
 * taken is stated at that step.
 */
#include "svo.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- logits */

/* Widen one logit to double.  A bf16 value is the top half of an IEEE single,
 * so the widening is exact. */
static double logit_at(const void* base, size_t i, int dtype) {
  if (dtype == SVO_F32) return (double)((const float*)base)[i];
  uint32_t bits = (uint32_t)((const uint16_t*)base)[i] << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

static size_t dtype_size(int dtype) { return dtype == SVO_F32 ? 4 : 2; }

static const void* row_ptr(const void* base, size_t row, int V, int dtype) {
  return (const char*)base + row * (size_t)V * dtype_size(dtype);
}

/* A needed row is valid when it holds no NaN and no +inf, and not every
 * entry is -inf (reading: -inf masks a token, p = 0; a row with no unmasked
 * token defines no distribution). */
static int row_is_valid(const void* row, int V, int dtype) {
  int any_finite = 0;
  for (int x = 0; x < V; ++x) {
    double z = logit_at(row, (size_t)x, dtype);
    if (isnan(z) || z == INFINITY) return 0;
    if (z != -INFINITY) any_finite = 1;
  }
  return any_finite;
}

/* ---------------------------------------------------------------- Philox */

/* Philox4x32-10 as published by Salmon et al. (SC'11): ten rounds of the
 * multiply-xor S-box with multipliers 0xD2511F53 / 0xCD9E8D57 and a Weyl key
 * schedule with increments 0x9E3779B9 / 0xBB67AE85; round r uses key + r*W. */
void svo_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
  uint32_t k0 = key[0], k1 = key[1];
  for (int round = 0; round < 10; ++round) {
    uint64_t prod0 = (uint64_t)0xD2511F53u * (uint64_t)c0;
    uint64_t prod1 = (uint64_t)0xCD9E8D57u * (uint64_t)c2;
    uint32_t hi0 = (uint32_t)(prod0 >> 32), lo0 = (uint32_t)prod0;
    uint32_t hi1 = (uint32_t)(prod1 >> 32), lo1 = (uint32_t)prod1;
    uint32_t n0 = hi1 ^ c1 ^ k0;
    uint32_t n1 = lo1;
    uint32_t n2 = hi0 ^ c3 ^ k1;
    uint32_t n3 = lo0;
    c0 = n0;
    c1 = n1;
    c2 = n2;
    c3 = n3;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  out[0] = c0;
  out[1] = c1;
  out[2] = c2;
  out[3] = c3;
}

static void seed_key(uint64_t seed, uint32_t key[2]) {
  key[0] = (uint32_t)(seed & 0xffffffffu);
  key[1] = (uint32_t)(seed >> 32);
}

/* Reading: the pages fix no generator or stream layout.  The accept draw for
 * position d of request g is word 0 of Philox at counter (d, g, 0, 0); its top
 * 24 bits give u in [0, 1 - 2^-24], exactly representable in single precision. */
double svo_accept_uniform(uint64_t seed, uint32_t g, uint32_t d) {
  uint32_t key[2], ctr[4] = {d, g, 0u, 0u}, out[4];
  seed_key(seed, key);
  svo_philox4x32_10(ctr, key, out);
  return ldexp((double)(out[0] >> 8), -24);
}

/* The race draw for token x of request g: word x mod 4 of Philox at counter
 * (x / 4, g, 1, 0); W = (o + 1/2) 2^-32 lies strictly inside (0, 1) and
 * E = -ln(1 - W) is a unit exponential. */
double svo_race_exponential(uint64_t seed, uint32_t g, uint32_t x) {
  uint32_t key[2], ctr[4] = {x >> 2, g, 1u, 0u}, out[4];
  seed_key(seed, key);
  svo_philox4x32_10(ctr, key, out);
  double W = ldexp((double)out[x & 3u] + 0.5, -32);
  return -log1p(-W);
}

/* ---------------------------------------------------------------- rows */

/* p = softmax(z / T): its normaliser ln sum exp(z/T), as the max of z/T plus
 * the log of the sum of exp(z/T - max/T).  [Sonar] "Cible-Brouillon": the
 * sampler compares the full probability distributions of draft and target. */
double svo_row_lse(const void* row, int V, int dtype, double T) {
  double m = -INFINITY;
  for (int x = 0; x < V; ++x) {
    double z = logit_at(row, (size_t)x, dtype);
    if (z > m) m = z;
  }
  if (m == -INFINITY) return -INFINITY;
  double mT = m / T;
  double s = 0.0;
  for (int x = 0; x < V; ++x) {
    double z = logit_at(row, (size_t)x, dtype);
    s += exp(z / T - mT);
  }
  return mT + log(s);
}

/* Greedy target token: the largest raw logit, lowest index on ties (reading:
 * the pages give no tie rule; the lowest index makes the choice unique). */
int svo_row_argmax(const void* row, int V, int dtype) {
  int best = 0;
  double bz = logit_at(row, 0, dtype);
  for (int x = 1; x < V; ++x) {
    double z = logit_at(row, (size_t)x, dtype);
    if (z > bz) {
      bz = z;
      best = x;
    }
  }
  return best;
}

/* The k largest draft logits, by (logit descending, index ascending), by k
 * plain scans.  [SSD] saguaro recipe item 1: the draft's five most likely
 * tokens.  The choice is made on raw logits, so it does not depend on T. */
static void row_topk(const void* row, int V, int dtype, int k, int* idx) {
  for (int j = 0; j < k; ++j) {
    int best = -1;
    double bz = 0.0;
    for (int x = 0; x < V; ++x) {
      int taken = 0;
      for (int i = 0; i < j; ++i)
        if (idx[i] == x) taken = 1;
      if (taken) continue;
      double z = logit_at(row, (size_t)x, dtype);
      if (best < 0 || z > bz) {
        best = x;
        bz = z;
      }
    }
    idx[j] = best;
  }
}

/* ---------------------------------------------------------------- request */

typedef struct {
  /* log-probabilities of the draft row used in the ratio and the residual:
   * plain q, or saguaro's q' */
  const void* qrow;
  double lse_q;
  int saguaro;
  const int* topk;
  int k;
  double ln_c;
  double ln_Z;
} draft_dist;

/* ln q(x), or ln q'(x) = ln q(x) + [x in K] ln c - ln Z for saguaro.
 * [SSD] saguaro recipe item 2: lower the probabilities of the top tokens.
 * Reading: lower them by the factor c and renormalise, so that q' is again a
 * distribution; Z = 1 - (1 - c) * sum_{x in K} q(x). */
static double draft_logprob(const draft_dist* q, int x, int dtype, int V, double T) {
  double zq = logit_at(q->qrow, (size_t)x, dtype);
  (void)V;
  double lq = zq / T - q->lse_q;
  if (!q->saguaro || lq == -INFINITY) return lq;
  int in_k = 0;
  for (int i = 0; i < q->k; ++i)
    if (q->topk[i] == x) in_k = 1;
  return lq + (in_k ? q->ln_c : 0.0) - q->ln_Z;
}

/* Exponential race over the target row, optionally against a draft row.
 *   residual (q given): candidates are the tokens with p(x) > q(x); the key is
 *     ln(p(x) - q(x)) - ln E_x, with ln(p - q) = ln p + ln(-expm1(ln q - ln p)).
 *     [SSD] rule item 3: on rejection draw from norm(max(0, p - q)).
 *   bonus (q NULL): candidates are the tokens with p(x) > 0; the key is
 *     ln p(x) - ln E_x.  [Sonar] "Décodage spéculatif": the target gives one
 *     more token for free.
 * argmax over x of r(x) / E_x with E_x i.i.d. unit exponentials picks x with
 * probability r(x) / sum r, and the choice does not depend on any sum.
 * Ties keep the lowest index.  Returns -1 when no token is a candidate. */
static int race(const void* trow, double lse_t, const draft_dist* q, int V, int dtype,
                double T, uint64_t seed, uint32_t g, double* gap) {
  int best_x = -1;
  double best = -INFINITY, second = -INFINITY;
  for (int x = 0; x < V; ++x) {
    double lp = logit_at(trow, (size_t)x, dtype) / T - lse_t;
    if (lp == -INFINITY) continue;
    double lr = lp;
    if (q) {
      double lq = draft_logprob(q, x, dtype, V, T);
      if (!(lp > lq)) continue;
      if (lq != -INFINITY) lr = lp + log(-expm1(lq - lp));
    }
    double key = lr - log(svo_race_exponential(seed, g, (uint32_t)x));
    if (key > best) {
      second = best;
      best = key;
      best_x = x;
    } else if (key > second) {
      second = key;
    }
  }
  *gap = best - second;
  return best_x;
}

typedef struct {
  const void* target;
  const void* draft;
  const int32_t* tokens;
  const int32_t* row_D;
  int B, D_max, V, dtype;
  float temperature;
  int mode;
  uint64_t seed;
  svo_params p;
  int32_t* out_tokens;
  int32_t* out_accept_len;
  uint32_t* out_flags;
  double* out_row_lse;
} run_args;

static void verify_one(const run_args* a, int b) {
  const int Dm = a->D_max, V = a->V, dt = a->dtype;
  const uint32_t g = a->p.request_offset + (uint32_t)b;
  int32_t* ot = a->out_tokens + (size_t)b * (size_t)(Dm + 1);
  const int32_t* tok = a->tokens + (size_t)b * (size_t)Dm;
  double* lse_out = a->out_row_lse ? a->out_row_lse + (size_t)b * (size_t)(2 * Dm + 1) : NULL;
  uint32_t flags = 0;

  for (int j = 0; j <= Dm; ++j) ot[j] = -1;
  a->out_accept_len[b] = -1;
  if (lse_out)
    for (int j = 0; j < 2 * Dm + 1; ++j) lse_out[j] = NAN;

  const int Db = a->row_D ? a->row_D[b] : Dm;
  const int mode = a->p.mode_per_req ? (int)a->p.mode_per_req[b] : a->mode;
  const double T = a->p.temperature_per_req ? (double)a->p.temperature_per_req[b]
                                            : (double)a->temperature;
  if (Db < 0 || Db > Dm) {
    flags |= SVO_FLAG_BAD_ROW_D;
    goto done;
  }
  if (mode != SVO_STOCHASTIC && mode != SVO_GREEDY && mode != SVO_SAGUARO) {
    flags |= 1u << 11;
    goto done;
  }
  if (mode != SVO_GREEDY && !(T > 0.0 && isfinite(T))) {
    flags |= 1u << 11;
    goto done;
  }
  for (int d = 0; d < Db; ++d)
    if (tok[d] < 0 || tok[d] >= V) {
      flags |= SVO_FLAG_BAD_TOKEN;
      goto done;
    }

  {
    const size_t trow0 = (size_t)b * (size_t)(Dm + 1);
    const size_t qrow0 = (size_t)b * (size_t)Dm;
    for (int d = 0; d <= Db; ++d)
      if (!row_is_valid(row_ptr(a->target, trow0 + d, V, dt), V, dt)) {
        flags |= SVO_FLAG_NONFINITE;
        goto done;
      }
    if (mode != SVO_GREEDY)
      for (int d = 0; d < Db; ++d)
        if (!row_is_valid(row_ptr(a->draft, qrow0 + d, V, dt), V, dt)) {
          flags |= SVO_FLAG_NONFINITE;
          goto done;
        }

    if (mode == SVO_GREEDY) {
      /* Greedy verification: accept x_d while it is the target's top token;
       * emit the target's top token at the first mismatch, or at position D
       * when all match.  [NV5] "Mit csinál...": accept in order until the
       * first mismatch; the output equals ordinary (argmax) decoding. */
      int n = Db;
      for (int d = 0; d < Db; ++d) {
        int am = svo_row_argmax(row_ptr(a->target, trow0 + d, V, dt), V, dt);
        if (tok[d] != am) {
          n = d;
          break;
        }
      }
      for (int d = 0; d < n; ++d) ot[d] = tok[d];
      ot[n] = svo_row_argmax(row_ptr(a->target, trow0 + n, V, dt), V, dt);
      a->out_accept_len[b] = n + 1;
      goto done;
    }

    /* Stochastic (plain or saguaro). */
    double lse_t[Dm + 1], lse_q[Dm > 0 ? Dm : 1];
    for (int d = 0; d <= Db; ++d) {
      lse_t[d] = svo_row_lse(row_ptr(a->target, trow0 + d, V, dt), V, dt, T);
      if (lse_out) lse_out[d] = lse_t[d];
    }
    for (int d = 0; d < Db; ++d) {
      lse_q[d] = svo_row_lse(row_ptr(a->draft, qrow0 + d, V, dt), V, dt, T);
      if (lse_out) lse_out[Dm + 1 + d] = lse_q[d];
    }

    const int saguaro = (mode == SVO_SAGUARO);
    const int kreq = a->p.saguaro_k > 0 ? a->p.saguaro_k : 5;
    const int k = kreq < V ? kreq : V;
    const double c = a->p.saguaro_c > 0.0 ? a->p.saguaro_c : 0.5;
    int topk[Dm > 0 ? Dm : 1][k > 0 ? k : 1];
    draft_dist qd[Dm > 0 ? Dm : 1];
    for (int d = 0; d < Db; ++d) {
      qd[d].qrow = row_ptr(a->draft, qrow0 + d, V, dt);
      qd[d].lse_q = lse_q[d];
      qd[d].saguaro = saguaro;
      qd[d].topk = topk[d];
      qd[d].k = k;
      qd[d].ln_c = log(c);
      qd[d].ln_Z = 0.0;
      if (saguaro) {
        row_topk(qd[d].qrow, V, dt, k, topk[d]);
        double mass = 0.0;
        for (int i = 0; i < k; ++i)
          mass += exp(logit_at(qd[d].qrow, (size_t)topk[d][i], dt) / T - lse_q[d]);
        qd[d].ln_Z = log1p(-(1.0 - c) * mass);
      }
    }

    /* Accept scan.  [SSD] rule items 1-2: accept when q(x) <= p(x); otherwise
     * the printed "reject with probability p/q" is read as accept with
     * probability p/q (the only reading under which item 1 holds and the
     * output is distributed like p).  So a = min(1, p/q), accept iff u < a.
     * [NV5]: stop at the first rejection; AL = n + 1 lies in [1, 1 + D]. */
    int n = Db;
    for (int d = 0; d < Db; ++d) {
      const int x = tok[d];
      const double lp =
          logit_at(row_ptr(a->target, trow0 + d, V, dt), (size_t)x, dt) / T - lse_t[d];
      const double lq = draft_logprob(&qd[d], x, dt, V, T);
      double acc;
      if (lp == -INFINITY)
        acc = 0.0; /* p(x) = 0: never accept a token the target cannot emit */
      else if (lq == -INFINITY)
        acc = 1.0;
      else
        acc = fmin(1.0, exp(lp - lq));
      const double u = svo_accept_uniform(a->seed, g, (uint32_t)d);
      if (fabs(u - acc) < 1e-5) flags |= SVO_FLAG_ACCEPT_NEAR_TIE;
      if (!(u < acc)) {
        n = d;
        break;
      }
    }

    double gap = INFINITY;
    int x_out;
    const void* trow_n = row_ptr(a->target, trow0 + n, V, dt);
    if (n < Db) {
      x_out = race(trow_n, lse_t[n], &qd[n], V, dt, T, a->seed, g, &gap);
      if (x_out < 0) {
        /* Reading: the pages are silent when {p > q} is empty (possible only
         * through rounding); sample from p on the same row instead. */
        flags |= SVO_FLAG_RESIDUAL_EMPTY;
        x_out = race(trow_n, lse_t[n], NULL, V, dt, T, a->seed, g, &gap);
      }
    } else {
      x_out = race(trow_n, lse_t[n], NULL, V, dt, T, a->seed, g, &gap);
    }
    if (gap < 1e-6) flags |= SVO_FLAG_RACE_NEAR_TIE;
    for (int d = 0; d < n; ++d) ot[d] = tok[d];
    ot[n] = x_out;
    a->out_accept_len[b] = n + 1;
  }

done:
  if (a->out_flags) a->out_flags[b] = flags;
}

int svo_verify(const void* target, const void* draft, const int32_t* tokens,
               const int32_t* row_D, int B, int D_max, int V, int dtype,
               float temperature, int mode, uint64_t seed, const svo_params* params,
               int32_t* out_tokens, int32_t* out_accept_len, uint32_t* out_flags,
               double* out_row_lse, int nthreads) {
  if (B < 0 || D_max < 0 || V <= 0 || (dtype != SVO_F32 && dtype != SVO_BF16)) return -1;
  if (B > 0 && (!target || !out_tokens || !out_accept_len)) return -1;
  if (B > 0 && D_max > 0 && !tokens) return -1;
  if (mode != SVO_STOCHASTIC && mode != SVO_GREEDY && mode != SVO_SAGUARO) return -1;
  run_args a;
  memset(&a, 0, sizeof a);
  a.target = target;
  a.draft = draft;
  a.tokens = tokens;
  a.row_D = row_D;
  a.B = B;
  a.D_max = D_max;
  a.V = V;
  a.dtype = dtype;
  a.temperature = temperature;
  a.mode = mode;
  a.seed = seed;
  if (params) a.p = *params;
  a.out_tokens = out_tokens;
  a.out_accept_len = out_accept_len;
  a.out_flags = out_flags;
  a.out_row_lse = out_row_lse;
  /* every request that reads draft rows needs a draft pointer */
  if (!draft && B > 0) {
    if (a.p.mode_per_req) {
      for (int b = 0; b < B; ++b)
        if (a.p.mode_per_req[b] != SVO_GREEDY) return -1;
    } else if (mode != SVO_GREEDY) {
      return -1;
    }
  }
  if (!a.p.mode_per_req && !a.p.temperature_per_req && mode != SVO_GREEDY &&
      !(temperature > 0.0f && isfinite(temperature)))
    return -1;
#ifdef _OPENMP
  if (nthreads > 1) {
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (int b = 0; b < B; ++b) verify_one(&a, b);
    return 0;
  }
#endif
  (void)nthreads;
  for (int b = 0; b < B; ++b) verify_one(&a, b);
  return 0;
}

/* ---------------------------------------------------------------- trees */

/* The exponential race over an explicit distribution P (the candidates are the
 * tokens with P(x) > 0): argmax of ln P(x) - ln E_x, ties to the lowest index. */
static int race_vec(const double* P, int V, uint64_t seed, uint32_t g, double* gap) {
  int best_x = -1;
  double best = -INFINITY, second = -INFINITY;
  for (int x = 0; x < V; ++x) {
    if (!(P[x] > 0.0)) continue;
    double key = log(P[x]) - log(svo_race_exponential(seed, g, (uint32_t)x));
    if (key > best) {
      second = best;
      best = key;
      best_x = x;
    } else if (key > second) {
      second = key;
    }
  }
  *gap = best - second;
  return best_x;
}

/* Softmax of one row at temperature T into P (0 for masked entries). */
static void row_probs(const void* row, int V, int dtype, double T, double* P) {
  const double lse = svo_row_lse(row, V, dtype, T);
  for (int x = 0; x < V; ++x) P[x] = exp(logit_at(row, (size_t)x, dtype) / T - lse);
}

typedef struct {
  const void* target;
  const void* draft;
  const int32_t* tokens;
  const int32_t* parents;
  const int32_t* n_nodes;
  int B, N_max, V, dtype;
  double T;
  int mode;
  uint64_t seed;
  uint32_t request_offset;
  int32_t* out_tokens;
  int32_t* out_accept_len;
  int32_t* out_nodes;
  uint32_t* out_flags;
} tree_args;

/* One request's tree walk ("Accélérer Sonar par la Spéculation", section
 * "EAGLE": several candidates per node).  Reading: the candidates at a node are
 * tried in node order with the rule of "Speculative Speculative Decoding –
 * асинхронизируй это." (items 1-3) applied recursively -- accept with
 * probability min(1, P/q); on rejection the next candidate is tested against
 * the normalised residual P = norm(max(0, P - q)), and after the last one the
 * token is drawn from that residual -- which keeps the output distributed like
 * p when the candidates are independent draws from q.  A chain (one child per
 * node) is the linear rule. */
static void verify_tree_one(const tree_args* a, int b) {
  const int Nm = a->N_max, V = a->V, dt = a->dtype;
  const uint32_t g = a->request_offset + (uint32_t)b;
  int32_t* ot = a->out_tokens + (size_t)b * (size_t)(Nm + 1);
  int32_t* on = a->out_nodes ? a->out_nodes + (size_t)b * (size_t)Nm : NULL;
  const int32_t* tok = a->tokens + (size_t)b * (size_t)Nm;
  const int32_t* par = a->parents + (size_t)b * (size_t)Nm;
  uint32_t flags = 0;
  for (int j = 0; j <= Nm; ++j) ot[j] = -1;
  if (on)
    for (int j = 0; j < Nm; ++j) on[j] = -1;
  a->out_accept_len[b] = -1;

  const int n = a->n_nodes ? a->n_nodes[b] : Nm;
  if (n < 0 || n > Nm) {
    flags |= SVO_FLAG_BAD_ROW_D;
    goto done;
  }
  if (a->mode != SVO_STOCHASTIC && a->mode != SVO_GREEDY) {
    flags |= 1u << 11;
    goto done;
  }
  if (a->mode != SVO_GREEDY && !(a->T > 0.0 && isfinite(a->T))) {
    flags |= 1u << 11;
    goto done;
  }
  for (int i = 0; i < n; ++i) {
    if (par[i] < 0 || par[i] > i) {
      flags |= 1u << 11;
      goto done;
    }
    if (tok[i] < 0 || tok[i] >= V) {
      flags |= SVO_FLAG_BAD_TOKEN;
      goto done;
    }
  }
  {
    const size_t trow0 = (size_t)b * (size_t)(Nm + 1);
    const size_t qrow0 = (size_t)b * (size_t)Nm;
    int has_child[Nm + 1];
    for (int p = 0; p <= n; ++p) has_child[p] = 0;
    for (int i = 0; i < n; ++i) has_child[par[i]] = 1;
    for (int p = 0; p <= n; ++p)
      if (!row_is_valid(row_ptr(a->target, trow0 + p, V, dt), V, dt)) {
        flags |= SVO_FLAG_NONFINITE;
        goto done;
      }
    if (a->mode != SVO_GREEDY)
      for (int p = 0; p < n; ++p)
        if (has_child[p] && !row_is_valid(row_ptr(a->draft, qrow0 + p, V, dt), V, dt)) {
          flags |= SVO_FLAG_NONFINITE;
          goto done;
        }

    int path[Nm > 0 ? Nm : 1];
    int len = 0, pos = 0, emitted = -1;
    double* P = (double*)malloc(sizeof(double) * (size_t)V);
    double* q = (double*)malloc(sizeof(double) * (size_t)V);
    for (;;) {
      const void* trow = row_ptr(a->target, trow0 + pos, V, dt);
      if (a->mode == SVO_GREEDY) {
        /* accept the first child holding the target's top token */
        const int am = svo_row_argmax(trow, V, dt);
        int found = -1;
        for (int i = 0; i < n && found < 0; ++i)
          if (par[i] == pos && tok[i] == am) found = i;
        if (found < 0) {
          emitted = am;
          break;
        }
        path[len++] = found;
        pos = found + 1;
        continue;
      }
      row_probs(trow, V, dt, a->T, P);
      if (!has_child[pos]) {
        /* no candidate: the bonus token from p */
        double gap;
        emitted = race_vec(P, V, a->seed, g, &gap);
        if (gap < 1e-6) flags |= SVO_FLAG_RACE_NEAR_TIE;
        break;
      }
      row_probs(row_ptr(a->draft, qrow0 + pos, V, dt), V, dt, a->T, q);
      int accepted = -1;
      for (int i = 0; i < n && accepted < 0; ++i) {
        if (par[i] != pos) continue;
        const int x = tok[i];
        double acc;
        if (q[x] > 0.0)
          acc = fmin(1.0, P[x] / q[x]);
        else
          acc = P[x] > 0.0 ? 1.0 : 0.0;
        const double u = svo_accept_uniform(a->seed, g, (uint32_t)i);
        if (fabs(u - acc) < 1e-5) flags |= SVO_FLAG_ACCEPT_NEAR_TIE;
        if (u < acc) {
          accepted = i;
          break;
        }
        /* rejected: the next candidate faces the normalised residual */
        double Z = 0.0;
        for (int y = 0; y < V; ++y) Z += fmax(0.0, P[y] - q[y]);
        if (Z > 0.0) {
          for (int y = 0; y < V; ++y) P[y] = fmax(0.0, P[y] - q[y]) / Z;
        } else {
          /* reading: an empty residual (only through rounding) keeps P */
          flags |= SVO_FLAG_RESIDUAL_EMPTY;
        }
      }
      if (accepted >= 0) {
        path[len++] = accepted;
        pos = accepted + 1;
        continue;
      }
      double gap;
      emitted = race_vec(P, V, a->seed, g, &gap);
      if (gap < 1e-6) flags |= SVO_FLAG_RACE_NEAR_TIE;
      break;
    }
    free(P);
    free(q);
    for (int j = 0; j < len; ++j) {
      ot[j] = tok[path[j]];
      if (on) on[j] = path[j];
    }
    ot[len] = emitted;
    a->out_accept_len[b] = len + 1;
  }
done:
  if (a->out_flags) a->out_flags[b] = flags;
}

int svo_verify_tree(const void* target, const void* draft, const int32_t* tokens,
                    const int32_t* parents, const int32_t* n_nodes, int B, int N_max, int V,
                    int dtype, float temperature, int mode, uint64_t seed,
                    uint32_t request_offset, int32_t* out_tokens, int32_t* out_accept_len,
                    int32_t* out_nodes, uint32_t* out_flags, int nthreads) {
  if (B < 0 || N_max < 0 || V <= 0 || (dtype != SVO_F32 && dtype != SVO_BF16)) return -1;
  if (B > 0 && (!target || !out_tokens || !out_accept_len)) return -1;
  if (B > 0 && N_max > 0 && (!tokens || !parents)) return -1;
  if (B > 0 && N_max > 0 && mode != SVO_GREEDY && !draft) return -1;
  tree_args a;
  memset(&a, 0, sizeof a);
  a.target = target;
  a.draft = draft;
  a.tokens = tokens;
  a.parents = parents;
  a.n_nodes = n_nodes;
  a.B = B;
  a.N_max = N_max;
  a.V = V;
  a.dtype = dtype;
  a.T = (double)temperature;
  a.mode = mode;
  a.seed = seed;
  a.request_offset = request_offset;
  a.out_tokens = out_tokens;
  a.out_accept_len = out_accept_len;
  a.out_nodes = out_nodes;
  a.out_flags = out_flags;
#ifdef _OPENMP
  if (nthreads > 1) {
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
    for (int b = 0; b < B; ++b) verify_tree_one(&a, b);
    return 0;
  }
#endif
  (void)nthreads;
  for (int b = 0; b < B; ++b) verify_tree_one(&a, b);
  return 0;
}

/* ---------------------------------------------------------------- epilogue */

/* "Accélérer Sonar par la Spéculation", section "Calendrier MTP pour un jeton
 * unique": after verification the target's input tokens are shifted by one and
 * the next target token is inserted at its slot; the accepted length decides
 * the next sequence length.  Reading: the verification window of request b is
 * its last committed token followed by its D_max draft slots, so the shifted
 * window starts with the drafts, and the token the verifier emitted at slot n
 * (the correction or the bonus) goes to slot n of the shifted window; the slots
 * after n keep the shifted drafts (the page's "redundant work on tokens that
 * were not accepted") and the last slot, which nothing shifts into, is -1.  The
 * AL emitted tokens are appended to the request's sequence at its current
 * length. */
int svo_epilogue(const int32_t* window, const int32_t* out_tokens, const int32_t* accept_len,
                 int B, int D_max, int32_t* next_window, int32_t* seq, int seq_cap,
                 int32_t* seq_len, uint32_t* full) {
  if (B < 0 || D_max < 0) return -1;
  if (B > 0 && (!out_tokens || !accept_len)) return -1;
  if (next_window && !window) return -1;
  if (seq && (!seq_len || seq_cap < 0)) return -1;
  const size_t W = (size_t)D_max + 1;
  for (int b = 0; b < B; ++b) {
    /* an accepted length outside [1, D_max + 1] is an error the verification flagged */
    const int32_t AL = accept_len[b] >= 1 && (size_t)accept_len[b] <= W ? accept_len[b] : 0;
    const int32_t* ot = out_tokens + (size_t)b * W;
    if (next_window) {
      /* read the whole row first: next_window may be window itself */
      int32_t row[W];
      for (size_t j = 0; j < W; ++j) row[j] = -1;
      if (AL >= 1) {
        for (size_t j = 0; j + 1 < W; ++j) row[j] = window[(size_t)b * W + j + 1];
        row[AL - 1] = ot[AL - 1];
      }
      for (size_t j = 0; j < W; ++j) next_window[(size_t)b * W + j] = row[j];
    }
    if (seq && AL >= 1) {
      if ((long long)seq_len[b] + AL > seq_cap || seq_len[b] < 0) {
        if (full) full[b / 32] |= 1u << (b % 32);
      } else {
        for (int j = 0; j < AL; ++j) seq[(size_t)b * (size_t)seq_cap + seq_len[b] + j] = ot[j];
        seq_len[b] += AL;
      }
    }
  }
  return 0;
}

/* ---------------------------------------------------------------- SSD lookup */

void svo_row_topk(const void* row, int V, int dtype, int k, int* idx) {
  row_topk(row, V, dtype, k, idx);
}

/* "Speculative Speculative Decoding – асинхронизируй это.": the speculations
 * prepared during verification are keyed by the verification outcome; a hit
 * returns the prepared speculation, a miss returns nothing (the page's
 * fallbacks -- a random token, n-grams -- are left to the caller).  Reading:
 * the outcome is the accepted length with the token the verifier emitted
 * after the accepted drafts; the first matching key wins. */
int svo_ssd_lookup(const int32_t* out_tokens, const int32_t* accept_len, int B, int D_max,
                   const int32_t* keys_al, const int32_t* keys_token, int K, const int32_t* spec,
                   int S, int32_t* out_hit, int32_t* out_spec) {
  if (B < 0 || D_max < 0 || K < 0 || S < 0) return -1;
  if (B > 0 && (!out_tokens || !accept_len || !out_hit)) return -1;
  if (B > 0 && K > 0 && (!keys_al || !keys_token)) return -1;
  if (out_spec && S > 0 && !spec) return -1;
  for (int b = 0; b < B; ++b) {
    const int32_t AL = accept_len[b];
    int hit = -1;
    if (AL >= 1 && AL <= D_max + 1) {
      const int32_t tok = out_tokens[(size_t)b * (size_t)(D_max + 1) + (size_t)(AL - 1)];
      for (int k = 0; k < K && hit < 0; ++k)
        if (keys_al[(size_t)b * K + k] == AL && keys_token[(size_t)b * K + k] == tok) hit = k;
    }
    out_hit[b] = hit;
    if (out_spec)
      for (int j = 0; j < S; ++j)
        out_spec[(size_t)b * S + j] = hit >= 0 ? spec[((size_t)b * K + hit) * S + j] : -1;
  }
  return 0;
}

int svo_has_openmp(void) {
#ifdef _OPENMP
  return 1;
#else
  return 0;
#endif
}
