/*
 * oracle.c -- plain, slow, fp64 CPU oracle for the batched verify +
 * speculation-cache step of Speculative Speculative Decoding (Saguaro).
 *
 * TEST INFRASTRUCTURE.  Only the test-suite, the package smoke check and the
 * benchmark's CPU-baseline leg load this library.  It shares no source, header,
 * table or helper with the CUDA library; neither one calls the other.
 *
 * Every step is the plain definition written out, one row at a time, in
 * double precision, with no blocking, fusion or reordering.  Sources:
 *   [ZH] "Speculative Speculative Decoding", gist.science, Chinese edition,
 *        technical summary, section 2 (Methodology: basic flow, challenges 1-3).
 *   [NL] "Speculative Speculative Decoding", gist.science, Dutch edition,
 *        technical summary, sections 2 and 3A/3B/3C.
 *   [PHX] Salmon, Moraes, Dror and Shaw, "Parallel Random Numbers: As Easy
 *        as 1, 2, 3", SC'11, section 4 (the Philox bijection).
 * The pages state the verification rule only in words ("lossless", reject and
 * resample from the residual).  The rule written here is the standard lossless
 * speculative-sampling rule; each other reading is named at the function.
 *
 * Parity pins: tests/test_oracle_pins.py.  Nothing in here is "parity
 * unpinned" except the reading choices that the pages leave open (fan-out
 * probability model, largest-remainder rounding, the guesses for full
 * acceptance, the uniform and fallback-token encodings); those are pinned only
 * by their own definitions.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define SSDO_DTYPE_FP32 0
#define SSDO_DTYPE_BF16 1

/* Row status bits (same meaning as the product's, defined here independently). */
#define SSDO_ROW_NONFINITE 1     /* NaN or +inf logit, or a vocab row that is all -inf */
#define SSDO_ROW_BAD_TOKEN 2     /* draft token outside [0, V) */
#define SSDO_ROW_BAD_UNIFORM 4   /* uniform outside [0, 1) or NaN */
#define SSDO_ROW_ZERO_Q 8        /* q'(d_j) == 0 at some draft position */
#define SSDO_ROW_ZERO_RESIDUAL 16/* residual mass 0 at the rejected position */
#define SSDO_ROW_NEAR_TIE 32     /* a decision margin below 1e-5 */
#define SSDO_ROW_BAD_PLAN 64     /* fan-out plan entries negative, > V, or not summing to budget */
#define SSDO_ROW_INVALID (SSDO_ROW_NONFINITE | SSDO_ROW_BAD_TOKEN | SSDO_ROW_BAD_UNIFORM | SSDO_ROW_BAD_PLAN)

#define SSDO_NEAR_TIE 1e-5

/* ------------------------------------------------------------------------- */
/* Philox4x32-10 [PHX]: ten rounds of the 4x32 bijection, key bumped by the   */
/* Weyl constants after every round.                                          */
/* ------------------------------------------------------------------------- */
void ssdo_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  uint32_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
  uint32_t k0 = key[0], k1 = key[1];
  for (int round = 0; round < 10; ++round) {
    uint64_t m0 = (uint64_t)0xD2511F53u * (uint64_t)x0;
    uint64_t m1 = (uint64_t)0xCD9E8D57u * (uint64_t)x2;
    uint32_t hi0 = (uint32_t)(m0 >> 32), lo0 = (uint32_t)m0;
    uint32_t hi1 = (uint32_t)(m1 >> 32), lo1 = (uint32_t)m1;
    uint32_t y0 = hi1 ^ x1 ^ k0;
    uint32_t y1 = lo1;
    uint32_t y2 = hi0 ^ x3 ^ k1;
    uint32_t y3 = lo0;
    x0 = y0; x1 = y1; x2 = y2; x3 = y3;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

/* n independent evaluations: ctr [n,4], key [n,2], out [n,4]. */
void ssdo_philox_batch(long n, const uint32_t* ctr, const uint32_t* key, uint32_t* out) {
  for (long i = 0; i < n; ++i) ssdo_philox4x32_10(ctr + 4 * i, key + 2 * i, out + 4 * i);
}

/* First output word of Philox4x32-10 at counter (c0, c1, c2, 0), key = seed. */
static uint32_t philox_word(uint64_t seed, uint32_t c0, uint32_t c1, uint32_t c2) {
  uint32_t ctr[4] = {c0, c1, c2, 0u};
  uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  uint32_t out[4];
  ssdo_philox4x32_10(ctr, key, out);
  return out[0];
}

/* Fallback speculator for a cache miss ([ZH] section 2, challenge 3; [NL]
 * section 3C: random tokens for large batches).  Reading: token i of row b is
 * floor(x * V / 2^32), x = first Philox word at counter (b, i, 2, 0). */
int32_t ssdo_fallback_token(uint64_t seed, int b, int i, int V) {
  uint32_t x = philox_word(seed, (uint32_t)b, (uint32_t)i, 2u);
  return (int32_t)(((uint64_t)x * (uint64_t)(uint32_t)V) >> 32);
}

/* ------------------------------------------------------------------------- */
/* Logit loading: bf16 and fp32 bits convert exactly to double.              */
/* ------------------------------------------------------------------------- */
static double load_logit(const void* base, int dtype, size_t idx) {
  float f;
  if (dtype == SSDO_DTYPE_FP32) {
    memcpy(&f, (const char*)base + 4 * idx, 4);
  } else {
    uint16_t h;
    memcpy(&h, (const char*)base + 2 * idx, 2);
    uint32_t u = (uint32_t)h << 16;
    memcpy(&f, &u, 4);
  }
  return (double)f;
}

static void load_row(const void* base, int dtype, size_t row, int V, double* out) {
  for (int v = 0; v < V; ++v) out[v] = load_logit(base, dtype, row * (size_t)V + (size_t)v);
}

/* A vocab row is usable when it holds no NaN, no +inf and at least one value
 * above -inf (otherwise no distribution is defined). */
static int row_finite(const double* l, int V) {
  int any = 0;
  for (int v = 0; v < V; ++v) {
    if (isnan(l[v]) || l[v] == INFINITY) return 0;
    if (l[v] != -INFINITY) any = 1;
  }
  return any;
}

/* ------------------------------------------------------------------------- */
/* Fan-out plan ([ZH] section 2, challenge 1; [NL] section 3A).               */
/* The pages say the optimal split of the bonus-guess budget over accepted    */
/* lengths k is a geometric series that favours the more probable outcomes.  */
/* Reading: with a per-token acceptance alpha, P(k) = alpha^k (1 - alpha) for */
/* k < K and P(K) = alpha^K; the quotas budget * P(k) are rounded by the      */
/* largest-remainder rule, ties to the smaller k.  mode 1 is the uniform      */
/* control ([ZH] section 2: "compared with uniform allocation"):              */
/* floor(budget / (K+1)) each, the remainder to the smallest k.              */
/* ------------------------------------------------------------------------- */
int ssdo_fanout_plan(double alpha, int K, int budget, int mode, int32_t* F) {
  if (K < 1 || budget < 0) return -1;
  if (mode == 1) {
    for (int k = 0; k <= K; ++k) F[k] = budget / (K + 1) + (k < budget % (K + 1) ? 1 : 0);
    return 0;
  }
  if (mode != 0 || !(alpha >= 0.0 && alpha <= 1.0)) return -1;
  double* P = malloc(sizeof(double) * (size_t)(K + 1));
  double* frac = malloc(sizeof(double) * (size_t)(K + 1));
  int* taken = calloc((size_t)(K + 1), sizeof(int));
  double run = 1.0; /* alpha^k by repeated multiplication */
  for (int k = 0; k < K; ++k) {
    P[k] = run * (1.0 - alpha);
    run = run * alpha;
  }
  P[K] = run;
  long assigned = 0;
  for (int k = 0; k <= K; ++k) {
    double quota = (double)budget * P[k];
    double fl = floor(quota);
    F[k] = (int32_t)fl;
    frac[k] = quota - fl;
    assigned += F[k];
  }
  long rem = (long)budget - assigned;
  while (rem > 0) {
    int best = -1;
    for (int k = 0; k <= K; ++k)
      if (!taken[k] && (best < 0 || frac[k] > frac[best])) best = k;
    if (best < 0) { /* every k already topped up once: start over */
      memset(taken, 0, sizeof(int) * (size_t)(K + 1));
      continue;
    }
    taken[best] = 1;
    F[best] += 1;
    --rem;
  }
  free(P); free(frac); free(taken);
  return 0;
}

/* Power-law fan-out ([ZH] section 2, challenge 1: the acceptance follows a
 * power law and the split is a constrained optimisation; [NL] section 3A: the
 * optimal split is a geometric series).  Reading: if the hit rate of an
 * outcome given F guesses follows a power-law curve 1 - c F^-beta, the
 * budget-constrained optimum of sum_k P(k) h(F_k) puts F_k proportional to
 * P(k)^gamma with gamma = 1 / (1 + beta) -- still a geometric series in k,
 * of ratio alpha^gamma.  gamma = q / 8, q = 1..8.  alpha^gamma and
 * (1 - alpha)^gamma are formed from three square roots (the eighth root) and
 * q - 1 products, so every evaluation of the plan gives the same numbers.
 * Weights w_k = a^k c (k < K), w_K = a^K with a = alpha^gamma, c =
 * (1 - alpha)^gamma; quotas budget * w_k / W, W = w_0 + ... + w_K in that
 * order; largest remainder as for the geometric plan.  q = 8 is the
 * geometric plan itself. */
static double eighth_power(double x, int q) {
  double r = sqrt(sqrt(sqrt(x)));
  double y = r;
  for (int i = 1; i < q; ++i) y = y * r;
  return y;
}

int ssdo_fanout_plan_power(double alpha, int K, int budget, int q, int32_t* F) {
  if (K < 1 || budget < 0 || q < 1 || q > 8 || !(alpha >= 0.0 && alpha <= 1.0)) return -1;
  if (q == 8) return ssdo_fanout_plan(alpha, K, budget, 0, F);
  double a = eighth_power(alpha, q), c = eighth_power(1.0 - alpha, q);
  double* w = malloc(sizeof(double) * (size_t)(K + 1));
  double* frac = malloc(sizeof(double) * (size_t)(K + 1));
  int* taken = calloc((size_t)(K + 1), sizeof(int));
  double run = 1.0, W = 0.0;
  for (int k = 0; k < K; ++k) {
    w[k] = run * c;
    run = run * a;
  }
  w[K] = run;
  for (int k = 0; k <= K; ++k) W = W + w[k];
  long assigned = 0;
  for (int k = 0; k <= K; ++k) {
    double quota = (double)budget * w[k] / W;
    double fl = floor(quota);
    F[k] = (int32_t)fl;
    frac[k] = quota - fl;
    assigned += F[k];
  }
  long rem = (long)budget - assigned;
  while (rem > 0) {
    int best = -1;
    for (int k = 0; k <= K; ++k)
      if (!taken[k] && (best < 0 || frac[k] > frac[best])) best = k;
    if (best < 0) {
      memset(taken, 0, sizeof(int) * (size_t)(K + 1));
      continue;
    }
    taken[best] = 1;
    F[best] += 1;
    --rem;
  }
  free(w); free(frac); free(taken);
  return 0;
}

/* Per-row acceptance estimate from history ([ZH] section 2, challenge 1:
 * the fan-out follows the acceptance, which differs between requests).
 * Reading: the expected acceptance of position j given the drafts is a_j,
 * so the step's estimate of the per-token acceptance is the mean of a_j over
 * the K positions, and the row's alpha follows it by exponential smoothing:
 * alpha' = (1 - lambda) alpha + lambda mean_j a_j, in double, rounded to
 * float.  Rows flagged invalid, or with a NaN a_j, keep their alpha. */
void ssdo_alpha_update(int B, int K, const float* alpha, const float* accept_prob, const int32_t* status,
                       double lambda, float* alpha_out) {
  for (int b = 0; b < B; ++b) {
    int ok = !(status[b] & SSDO_ROW_INVALID);
    double s = 0.0;
    for (int j = 0; j < K; ++j) {
      double a = (double)accept_prob[(size_t)b * K + j];
      if (isnan(a)) ok = 0;
      s = s + a;
    }
    if (!ok) { alpha_out[b] = alpha[b]; continue; }
    double mean = s / (double)K;
    alpha_out[b] = (float)((1.0 - lambda) * (double)alpha[b] + lambda * mean);
  }
}

/* Fallback speculator by batch size ([ZH] section 2, challenge 3; [NL]
 * section 3C: a slow high-quality fallback for small batches, a fast
 * low-quality one (random tokens) for large ones, switching at a critical
 * batch size b*).  Reading: a row hits the cache with probability h,
 * independently; on any miss in the batch the whole batch waits for the
 * fallback.  A round takes L_target plus, with probability 1 - h^b, the
 * fallback's latency.  A hit, or a miss with the primary fallback, yields
 * E_p = sum_{i=0..K} alpha^i tokens (expected accepted drafts plus the
 * bonus); a miss with the fast fallback yields E_f.  The fast fallback is
 * chosen when its expected tokens per unit time are strictly higher.
 * Returns b* = the smallest b in [1, b_max] that chooses the fast fallback,
 * b_max + 1 when none does; choice[b-1] = 1 for the fast one, 0 otherwise
 * (choice may be NULL). */
int ssdo_fallback_bstar(double h, double alpha, int K, double L_target, double L_primary, double L_fast,
                        double E_fast, int b_max, uint8_t* choice) {
  double Ep = 0.0, ak = 1.0;
  for (int i = 0; i <= K; ++i) { Ep = Ep + ak; ak = ak * alpha; }
  int bstar = b_max + 1;
  double hb = 1.0;
  for (int b = 1; b <= b_max; ++b) {
    hb = hb * h;
    double miss_any = 1.0 - hb;
    double thr_primary = Ep / (L_target + miss_any * L_primary);
    double thr_fast = (h * Ep + (1.0 - h) * E_fast) / (L_target + miss_any * L_fast);
    int fast = thr_fast > thr_primary;
    if (choice) choice[b - 1] = (uint8_t)fast;
    if (fast && bstar > b_max) bstar = b;
  }
  return bstar;
}

/* ------------------------------------------------------------------------- */
/* Top-F of a logit row: the first F entries of the row sorted by (logit      */
/* descending, index ascending).  Softmax is monotone for T > 0, so this is   */
/* the top-F of the distribution; -0 and +0 compare equal, so they tie and    */
/* the lower index wins.  ([ZH] section 2, challenge 2: "top-F tokens".)      */
/* ------------------------------------------------------------------------- */
typedef struct { double key; int32_t idx; } kv_t;

static int cmp_desc(const void* a, const void* b) {
  const kv_t* x = (const kv_t*)a;
  const kv_t* y = (const kv_t*)b;
  if (x->key > y->key) return -1;
  if (x->key < y->key) return 1;
  return (x->idx < y->idx) ? -1 : (x->idx > y->idx ? 1 : 0);
}

static void topf_row(const double* l, int V, int F, int32_t* out) {
  kv_t* a = malloc(sizeof(kv_t) * (size_t)V);
  for (int v = 0; v < V; ++v) { a[v].key = l[v]; a[v].idx = v; }
  qsort(a, (size_t)V, sizeof(kv_t), cmp_desc);
  for (int i = 0; i < F; ++i) out[i] = a[i].idx;
  free(a);
}

int ssdo_topf(const double* logits, int V, int F, int32_t* out) {
  if (F < 0 || F > V) return -1;
  topf_row(logits, V, F, out);
  return 0;
}

/* Lowest index of the maximum (greedy decoding, temperature 0). */
static int argmax_row(const double* l, int V) {
  int best = 0;
  for (int v = 1; v < V; ++v)
    if (l[v] > l[best]) best = v;
  return best;
}

/* ------------------------------------------------------------------------- */
/* Temperature softmax: p(v) = exp(l(v)/T - m) / S, m = max_v l(v)/T,         */
/* S = sum_v exp(l(v)/T - m).  Returns the natural log-sum-exp m + log S.     */
/* ------------------------------------------------------------------------- */
static double softmax_row(const double* l, int V, double T, double* p) {
  double m = -INFINITY;
  for (int v = 0; v < V; ++v) {
    double x = l[v] / T;
    if (x > m) m = x;
  }
  double S = 0.0;
  for (int v = 0; v < V; ++v) {
    p[v] = exp(l[v] / T - m);
    S += p[v];
  }
  for (int v = 0; v < V; ++v) p[v] = p[v] / S;
  return m + log(S);
}

/* Saguaro sampling ([ZH] section 2, challenge 2; [NL] section 3B): the draft's
 * top-F tokens are down-weighted by C and the distribution renormalised.
 * Reading: q'(v) = w(v) q(v) / Z with w = C on the top-F set S of the
 * original q, w = 1 elsewhere, and Z = 1 - (1 - C) Q_S, Q_S = sum_{S} q.
 * Returns Z; writes Q_S and q'. */
static double saguaro_row(const double* q, int V, const int32_t* S, int F, double C,
                          double* QS_out, double* qp) {
  double QS = 0.0;
  for (int i = 0; i < F; ++i) QS += q[S[i]];
  double Z = 1.0 - (1.0 - C) * QS;
  for (int v = 0; v < V; ++v) qp[v] = q[v] / Z;
  for (int i = 0; i < F; ++i) qp[S[i]] = C * q[S[i]] / Z;
  *QS_out = QS;
  return Z;
}

/* Inverse-CDF draw: the smallest v whose running sum of r exceeds u * R, in
 * vocabulary-index order (reading).  If rounding leaves no such v, the last v
 * with r(v) > 0.  *margin = distance of u*R to the nearer CDF step, over R.
 * Near-tie window (reading of the 1e-5 decision tolerance): a draw made in
 * another precision may land anywhere whose CDF interval [c(v-1), c(v)) meets
 * [u R - 1e-5 R, u R + 1e-5 R]; *wlo and *whi are the lowest and highest
 * such v among the tokens with r(v) > 0. */
static int inverse_cdf(const double* r, int V, double R, double u, double* margin, int32_t* wlo,
                       int32_t* whi) {
  double t = u * R, c = 0.0, prev = 0.0;
  int last_pos = -1, drawn = -1;
  *margin = 0.0;
  for (int v = 0; v < V; ++v) {
    prev = c;
    c += r[v];
    if (r[v] > 0.0) last_pos = v;
    if (c > t) {
      double m1 = t - prev, m2 = c - t;
      *margin = (m1 < m2 ? m1 : m2) / R;
      drawn = v;
      break;
    }
  }
  if (drawn < 0) drawn = last_pos < 0 ? V - 1 : last_pos;
  const double lo_t = t - SSDO_NEAR_TIE * R, hi_t = t + SSDO_NEAR_TIE * R;
  int lo = -1, hi = -1;
  c = 0.0;
  for (int v = 0; v < V; ++v) {
    prev = c;
    c += r[v];
    if (!(r[v] > 0.0)) continue;
    if (lo < 0 && c > lo_t) lo = v;
    if (prev <= hi_t) hi = v;
  }
  if (lo < 0 || hi < 0) lo = hi = drawn;
  if (drawn < lo) lo = drawn;
  if (drawn > hi) hi = drawn;
  *wlo = lo;
  *whi = hi;
  return drawn;
}

/* ------------------------------------------------------------------------- */
/* One row of the verify + cache step.                                        */
/* ------------------------------------------------------------------------- */
typedef struct {
  int dtype, B, K, V, budget;
  const void* target;      /* [B, K+1, V] */
  const void* draft;       /* [B, K, V] */
  const void* draft_next;  /* [B, V] or NULL */
  const int32_t* tokens;   /* [B, K] */
  const float* uniforms;   /* [B, K+1] */
  double T, C;
  const int32_t* F;        /* [B, K+1] or NULL */
  const int32_t* payload;  /* [B, budget, K] or NULL */
  uint64_t fallback_seed;
  const int32_t* rows; int n_rows; int n_threads;
  /* outputs (row i of the subset) */
  int32_t* n_accepted; int32_t* bonus; int32_t* out_tokens;
  double* accept_prob; double* residual_mass;
  double* Z; double* QS; double* q_lse; double* p_lse;
  int32_t* offsets; int32_t* cache_tokens;
  uint8_t* hit; int32_t* slot; int32_t* next_tokens;
  int32_t* status; double* accept_margin; double* bonus_margin; double* p_hit;
  int32_t* bonus_lo; int32_t* bonus_hi;
  int early_exit;  /* read p_j only for j <= k* and j = K */
} verify_job;

/* The outputs of an invalid row. */
static void write_invalid_row(const verify_job* J, int i, int b, int32_t st, int32_t* outt, int32_t* ctok,
                              int32_t* nxt) {
  const int K = J->K, V = J->V;
  J->n_accepted[i] = -1;
  J->bonus[i] = -1;
  for (int j = 0; j <= K; ++j) outt[j] = -1;
  for (int j = 0; j < K; ++j) J->accept_prob[(size_t)i * K + j] = NAN;
  J->residual_mass[i] = NAN;
  for (int j = 0; j < K; ++j) {
    if (J->Z) J->Z[(size_t)i * K + j] = NAN;
    if (J->QS) J->QS[(size_t)i * K + j] = NAN;
    if (J->q_lse) J->q_lse[(size_t)i * K + j] = NAN;
  }
  if (J->p_lse) for (int j = 0; j <= K; ++j) J->p_lse[(size_t)i * (K + 1) + j] = NAN;
  if (ctok) for (int s = 0; s < J->budget; ++s) ctok[s] = -1;
  if (J->hit) J->hit[i] = 0;
  if (J->slot) J->slot[i] = -1;
  if (nxt) for (int t = 0; t < K; ++t) nxt[t] = ssdo_fallback_token(J->fallback_seed, b, t, V);
  J->status[i] = st;
  if (J->accept_margin) J->accept_margin[i] = INFINITY;
  if (J->bonus_margin) J->bonus_margin[i] = INFINITY;
  if (J->p_hit) J->p_hit[i] = NAN;
  if (J->bonus_lo) J->bonus_lo[i] = -1;
  if (J->bonus_hi) J->bonus_hi[i] = -1;
}

static void verify_row(const verify_job* J, int i) {
  const int K = J->K, V = J->V, budget = J->budget;
  const int b = J->rows ? J->rows[i] : i;
  int32_t st = 0;

  double** lp = malloc(sizeof(double*) * (size_t)(K + 1));
  double** lq = malloc(sizeof(double*) * (size_t)K);
  /* A non-finite target row makes the row invalid; with the early-exit read
   * schedule only the target rows the outcome depends on count: p_j for
   * j <= k* (decided below) and p_K. */
  int* pnf = malloc(sizeof(int) * (size_t)(K + 1));
  for (int j = 0; j <= K; ++j) {
    lp[j] = malloc(sizeof(double) * (size_t)V);
    load_row(J->target, J->dtype, (size_t)b * (size_t)(K + 1) + (size_t)j, V, lp[j]);
    pnf[j] = !row_finite(lp[j], V);
    if (pnf[j] && (!J->early_exit || j == K)) st |= SSDO_ROW_NONFINITE;
  }
  for (int j = 0; j < K; ++j) {
    lq[j] = malloc(sizeof(double) * (size_t)V);
    load_row(J->draft, J->dtype, (size_t)b * (size_t)K + (size_t)j, V, lq[j]);
    if (!row_finite(lq[j], V)) st |= SSDO_ROW_NONFINITE;
  }
  double* ln = NULL;
  if (J->draft_next) {
    ln = malloc(sizeof(double) * (size_t)V);
    load_row(J->draft_next, J->dtype, (size_t)b, V, ln);
    if (!row_finite(ln, V)) st |= SSDO_ROW_NONFINITE;
  }
  const int32_t* d = J->tokens + (size_t)b * (size_t)K;
  for (int j = 0; j < K; ++j)
    if (d[j] < 0 || d[j] >= V) st |= SSDO_ROW_BAD_TOKEN;
  const float* u = J->uniforms + (size_t)b * (size_t)(K + 1);
  for (int j = 0; j <= K; ++j)
    if (!(u[j] >= 0.0f && u[j] < 1.0f)) st |= SSDO_ROW_BAD_UNIFORM;
  const int32_t* F = J->F ? J->F + (size_t)b * (size_t)(K + 1) : NULL;
  if (F) {
    long sum = 0;
    for (int k = 0; k <= K; ++k) {
      if (F[k] < 0 || F[k] > V) st |= SSDO_ROW_BAD_PLAN;
      sum += F[k];
    }
    if (sum != budget) st |= SSDO_ROW_BAD_PLAN;
  }

  /* Cache segment offsets are the prefix sums of the plan (valid rows or not). */
  int32_t* offs = J->offsets ? J->offsets + (size_t)i * (size_t)(K + 2) : NULL;
  if (offs && F) {
    offs[0] = 0;
    for (int k = 0; k <= K; ++k) offs[k + 1] = offs[k] + ((st & SSDO_ROW_BAD_PLAN) ? 0 : F[k]);
  }
  int32_t* ctok = (J->cache_tokens && F) ? J->cache_tokens + (size_t)i * (size_t)budget : NULL;
  int32_t* nxt = J->next_tokens ? J->next_tokens + (size_t)i * (size_t)K : NULL;
  int32_t* outt = J->out_tokens + (size_t)i * (size_t)(K + 1);

  if (st & SSDO_ROW_INVALID) {
    write_invalid_row(J, i, b, st, outt, ctok, nxt);
    goto done;
  }

  {
    /* Top-F sets S_k of q_k (k < K) and the full-acceptance guesses G_K:
     * the top-F_K of draft_next when given, else of the target row p_K
     * (reading: the draft logits carry no distribution for that bonus). */
    int32_t** S = malloc(sizeof(int32_t*) * (size_t)(K + 1));
    for (int k = 0; k <= K; ++k) {
      int f = F ? F[k] : 0;
      S[k] = malloc(sizeof(int32_t) * (size_t)(f > 0 ? f : 1));
      if (f > 0) topf_row(k < K ? lq[k] : (ln ? ln : lp[K]), V, f, S[k]);
    }
    double* a = malloc(sizeof(double) * (size_t)K);
    int* zq = calloc((size_t)K, sizeof(int));
    int ee_bad = 0;
    int kstar = K, bon = -1;
    int32_t blo = -1, bhi = -1;
    double R = 1.0, amarg = INFINITY, bmarg = INFINITY, phit = NAN;

    if (J->T == 0.0) {
      /* Greedy verification (reading of temperature 0): p and q are one-hot at
       * the lowest-index argmax of the raw logits; accept iff d_j is the
       * target argmax; the bonus is the target argmax at k*; Saguaro sampling
       * is the identity. */
      for (int j = 0; j < K; ++j) {
        int am = argmax_row(lp[j], V);
        a[j] = (d[j] == am) ? 1.0 : 0.0;
        if (kstar == K && J->early_exit && pnf[j]) ee_bad = 1;  /* a target row read before k* */
        if (kstar == K && d[j] != am) kstar = j;
        int amq = argmax_row(lq[j], V);
        double qs = 0.0;
        for (int s = 0; s < (F ? F[j] : 0); ++s) if (S[j][s] == amq) qs = 1.0;
        if (J->Z) J->Z[(size_t)i * K + j] = 1.0;
        if (J->QS) J->QS[(size_t)i * K + j] = qs;
        if (J->q_lse) J->q_lse[(size_t)i * K + j] = lq[j][amq];
      }
      if (J->p_lse)
        for (int j = 0; j <= K; ++j) J->p_lse[(size_t)i * (K + 1) + j] = lp[j][argmax_row(lp[j], V)];
      bon = argmax_row(lp[kstar], V);
      blo = bhi = bon;
      R = 1.0;
    } else {
      double** p = malloc(sizeof(double*) * (size_t)(K + 1));
      double** qp = malloc(sizeof(double*) * (size_t)K);
      for (int j = 0; j <= K; ++j) {
        p[j] = malloc(sizeof(double) * (size_t)V);
        double lse = softmax_row(lp[j], V, J->T, p[j]);
        if (J->p_lse) J->p_lse[(size_t)i * (K + 1) + j] = lse;
      }
      double* q = malloc(sizeof(double) * (size_t)V);
      for (int j = 0; j < K; ++j) {
        qp[j] = malloc(sizeof(double) * (size_t)V);
        double lse = softmax_row(lq[j], V, J->T, q);
        double QSj = 0.0, Zj = 1.0;
        if (F) {
          Zj = saguaro_row(q, V, S[j], F[j], J->C, &QSj, qp[j]);
        } else {
          for (int v = 0; v < V; ++v) qp[j][v] = q[v];
        }
        if (J->Z) J->Z[(size_t)i * K + j] = Zj;
        if (J->QS) J->QS[(size_t)i * K + j] = QSj;
        if (J->q_lse) J->q_lse[(size_t)i * K + j] = lse;
      }
      free(q);
      /* Accept test: a_j = min(1, p_j(d_j) / q'_j(d_j)); position j is
       * accepted iff u_j < a_j; k* = first rejected position, else K.
       * A draft token with q'(d) = 0 is accepted iff p(d) > 0. */
      for (int j = 0; j < K; ++j) {
        double pd = p[j][d[j]], qd = qp[j][d[j]];
        if (qd > 0.0) {
          double ratio = pd / qd;
          a[j] = ratio < 1.0 ? ratio : 1.0;
        } else {
          a[j] = pd > 0.0 ? 1.0 : 0.0;
          zq[j] = 1;
        }
      }
      for (int j = 0; j < K; ++j) {
        if (J->early_exit && pnf[j]) { ee_bad = 1; break; }  /* a target row read before k* */
        double mg = fabs((double)u[j] - a[j]);
        if (mg < amarg) amarg = mg;
        if (!((double)u[j] < a[j])) { kstar = j; break; }
      }
      /* q'(d_j) = 0 is reported for every position, or with the early-exit
       * schedule for the positions up to k* */
      for (int j = 0; j < K; ++j)
        if (zq[j] && (!J->early_exit || j <= kstar)) st |= SSDO_ROW_ZERO_Q;
      /* Bonus token: at a rejection k* < K draw from r = max(0, p - q') / R,
       * R = sum r; if R is 0 draw from p instead (reading); after full
       * acceptance draw from p_K.  One uniform u_K serves every case. */
      double* r = malloc(sizeof(double) * (size_t)V);
      double uK = (double)u[K];
      if (kstar < K) {
        R = 0.0;
        for (int v = 0; v < V; ++v) {
          double x = p[kstar][v] - qp[kstar][v];
          r[v] = x > 0.0 ? x : 0.0;
          R += r[v];
        }
        if (R == 0.0) {
          st |= SSDO_ROW_ZERO_RESIDUAL;
          for (int v = 0; v < V; ++v) { r[v] = p[kstar][v]; R += r[v]; }
        }
      } else {
        R = 0.0;
        for (int v = 0; v < V; ++v) { r[v] = p[K][v]; R += r[v]; }
      }
      bon = inverse_cdf(r, V, R, uK, &bmarg, &blo, &bhi);

      if (J->p_hit && F) {
        /* Diagnostic: probability that the outcome (k*, bonus) lands in the
         * cache, given the drafts: sum_k P(k* = k | d) * mass of S_k under the
         * bonus distribution of outcome k. */
        double reach = 1.0, tot = 0.0;
        for (int k = 0; k <= K; ++k) {
          double pk = (k < K) ? reach * (1.0 - a[k]) : reach;
          double Rk = 0.0, in = 0.0;
          for (int v = 0; v < V; ++v) {
            double x = (k < K) ? p[k][v] - qp[k][v] : p[K][v];
            r[v] = x > 0.0 ? x : 0.0;
            Rk += r[v];
          }
          if (Rk == 0.0) for (int v = 0; v < V; ++v) { r[v] = p[k][v]; Rk += r[v]; }
          for (int s = 0; s < F[k]; ++s) in += r[S[k][s]];
          tot += pk * in / Rk;
          if (k < K) reach *= a[k];
        }
        phit = tot;
      }
      free(r);
      for (int j = 0; j <= K; ++j) free(p[j]);
      for (int j = 0; j < K; ++j) free(qp[j]);
      free(p); free(qp);
    }

    if (ee_bad) {
      write_invalid_row(J, i, b, st | SSDO_ROW_NONFINITE, outt, ctok, nxt);
      for (int k = 0; k <= K; ++k) free(S[k]);
      free(S); free(a); free(zq);
      goto done;
    }
    J->n_accepted[i] = kstar;
    J->bonus[i] = bon;
    for (int j = 0; j <= K; ++j) outt[j] = j < kstar ? d[j] : (j == kstar ? bon : -1);
    /* the early-exit schedule reports no a_j past k* (p_j was not read) */
    for (int j = 0; j < K; ++j) J->accept_prob[(size_t)i * K + j] = (J->early_exit && j > kstar) ? NAN : a[j];
    J->residual_mass[i] = R;

    /* Cache build and lookup ([ZH] section 2, basic flow steps 3-4; [NL]
     * section 2): keys are (k, bonus guess); a hit returns the row's
     * pre-speculated tokens, a miss falls back to random tokens. */
    int32_t sl = -1;
    if (F) {
      for (int k = 0; k <= K; ++k)
        for (int s = 0; s < F[k]; ++s) ctok[offs[k] + s] = S[k][s];
      for (int s = 0; s < F[kstar]; ++s)
        if (S[kstar][s] == bon) { sl = offs[kstar] + s; break; }
    }
    if (J->hit) J->hit[i] = sl >= 0 ? 1 : 0;
    if (J->slot) J->slot[i] = sl;
    if (nxt) {
      for (int t = 0; t < K; ++t) {
        if (sl >= 0)
          nxt[t] = J->payload ? J->payload[((size_t)b * (size_t)budget + (size_t)sl) * (size_t)K + (size_t)t] : -1;
        else
          nxt[t] = ssdo_fallback_token(J->fallback_seed, b, t, V);
      }
    }
    if (amarg < SSDO_NEAR_TIE || bmarg < SSDO_NEAR_TIE) st |= SSDO_ROW_NEAR_TIE;
    J->status[i] = st;
    if (J->accept_margin) J->accept_margin[i] = amarg;
    if (J->bonus_margin) J->bonus_margin[i] = bmarg;
    if (J->p_hit) J->p_hit[i] = phit;
    if (J->bonus_lo) J->bonus_lo[i] = blo;
    if (J->bonus_hi) J->bonus_hi[i] = bhi;
    for (int k = 0; k <= K; ++k) free(S[k]);
    free(S); free(a); free(zq);
  }

done:
  free(pnf);
  for (int j = 0; j <= K; ++j) free(lp[j]);
  for (int j = 0; j < K; ++j) free(lq[j]);
  free(lp); free(lq); free(ln);
}

typedef struct { const void* job; int tid; int nth; int n; void (*fn)(const void*, int); } worker_arg;

static void* worker(void* p) {
  worker_arg* w = (worker_arg*)p;
  for (int i = w->tid; i < w->n; i += w->nth) w->fn(w->job, i);
  return NULL;
}

/* Rows are independent; they are spread over plain threads, row i to thread
 * i mod n_threads.  No result depends on the thread count. */
static void run_rows(const void* job, int n, int n_threads, void (*fn)(const void*, int)) {
  if (n_threads < 1) n_threads = 1;
  if (n_threads > n) n_threads = n > 0 ? n : 1;
  pthread_t* th = malloc(sizeof(pthread_t) * (size_t)n_threads);
  worker_arg* args = malloc(sizeof(worker_arg) * (size_t)n_threads);
  for (int t = 0; t < n_threads; ++t) {
    args[t].job = job; args[t].tid = t; args[t].nth = n_threads; args[t].n = n; args[t].fn = fn;
    if (t > 0) pthread_create(&th[t], NULL, worker, &args[t]);
  }
  worker(&args[0]);
  for (int t = 1; t < n_threads; ++t) pthread_join(th[t], NULL);
  free(th); free(args);
}

static void verify_row_thunk(const void* job, int i) { verify_row((const verify_job*)job, i); }

int ssdo_verify_batch(int dtype, int B, int K, int V, int budget,
                      const void* target, const void* draft, const void* draft_next,
                      const int32_t* tokens, const float* uniforms, double T,
                      const int32_t* F, double C, const int32_t* payload, uint64_t fallback_seed,
                      const int32_t* rows, int n_rows, int n_threads,
                      int32_t* n_accepted, int32_t* bonus, int32_t* out_tokens,
                      double* accept_prob, double* residual_mass,
                      double* Z, double* QS, double* q_lse, double* p_lse,
                      int32_t* offsets, int32_t* cache_tokens,
                      uint8_t* hit, int32_t* slot, int32_t* next_tokens,
                      int32_t* status, double* accept_margin, double* bonus_margin, double* p_hit,
                      int32_t* bonus_lo, int32_t* bonus_hi, int early_exit) {
  if (B < 0 || K < 1 || V < 1 || !(T >= 0.0) || (F && !(C > 0.0 && C <= 1.0))) return -1;
  if (dtype != SSDO_DTYPE_FP32 && dtype != SSDO_DTYPE_BF16) return -1;
  if (F && (budget < 0 || budget > V)) return -1;
  verify_job J = {dtype, B, K, V, budget, target, draft, draft_next, tokens, uniforms, T, C, F,
                  payload, fallback_seed, rows, rows ? n_rows : B, n_threads,
                  n_accepted, bonus, out_tokens, accept_prob, residual_mass, Z, QS, q_lse, p_lse,
                  offsets, cache_tokens, hit, slot, next_tokens, status, accept_margin,
                  bonus_margin, p_hit, bonus_lo, bonus_hi, early_exit};
  run_rows(&J, J.n_rows, n_threads, verify_row_thunk);
  return 0;
}

/* ------------------------------------------------------------------------- */
/* Draft side: Saguaro reweighting of q_j (j < K) and, optionally, drawing   */
/* the draft token d_j ~ q'_j by the same inverse-CDF convention with the    */
/* caller's uniform.  ([ZH] section 2, challenge 2; [NL] section 3B.)        */
/* ------------------------------------------------------------------------- */
typedef struct {
  int dtype, B, K, V, budget;
  const void* draft; double T; const int32_t* F; double C; const float* u_draft;
  const int32_t* rows; int n_rows;
  int32_t* topf_tokens; int32_t* offsets; double* Z; double* QS; double* q_lse;
  int32_t* tokens_out; double* margin; int32_t* status;
  int32_t* tok_lo; int32_t* tok_hi;  /* [n, K] near-tie windows of the draws, or NULL */
} reweight_job;

static void reweight_row(const void* jp, int i) {
  const reweight_job* J = (const reweight_job*)jp;
  const int K = J->K, V = J->V;
  const int b = J->rows ? J->rows[i] : i;
  const int32_t* F = J->F + (size_t)b * (size_t)(K + 1);
  int32_t st = 0;
  long sum = 0;
  for (int k = 0; k <= K; ++k) {
    if (F[k] < 0 || F[k] > V) st |= SSDO_ROW_BAD_PLAN;
    sum += F[k];
  }
  if (sum != J->budget) st |= SSDO_ROW_BAD_PLAN;
  int32_t* offs = J->offsets + (size_t)i * (size_t)(K + 2);
  offs[0] = 0;
  for (int k = 0; k <= K; ++k) offs[k + 1] = offs[k] + ((st & SSDO_ROW_BAD_PLAN) ? 0 : F[k]);
  double* l = malloc(sizeof(double) * (size_t)V);
  double* q = malloc(sizeof(double) * (size_t)V);
  double* qp = malloc(sizeof(double) * (size_t)V);
  double worst = INFINITY;
  for (int j = 0; j < K; ++j) {
    load_row(J->draft, J->dtype, (size_t)b * (size_t)K + (size_t)j, V, l);
    int32_t* seg = J->topf_tokens + (size_t)i * (size_t)J->budget + offs[j];
    size_t o = (size_t)i * (size_t)K + (size_t)j;
    int bad = (st & SSDO_ROW_BAD_PLAN) || !row_finite(l, V);
    if (!row_finite(l, V)) st |= SSDO_ROW_NONFINITE;
    if (J->u_draft) {
      float uu = J->u_draft[(size_t)b * (size_t)K + (size_t)j];
      if (!(uu >= 0.0f && uu < 1.0f)) { st |= SSDO_ROW_BAD_UNIFORM; bad = 1; }
    }
    if (bad) {
      J->Z[o] = NAN; J->QS[o] = NAN; J->q_lse[o] = NAN;
      if (!(st & SSDO_ROW_BAD_PLAN)) for (int s = 0; s < F[j]; ++s) seg[s] = -1;
      if (J->tokens_out) J->tokens_out[o] = -1;
      if (J->tok_lo) { J->tok_lo[o] = -1; J->tok_hi[o] = -1; }
      continue;
    }
    topf_row(l, V, F[j], seg);
    if (J->T == 0.0) {
      int am = argmax_row(l, V);
      double qs = 0.0;
      for (int s = 0; s < F[j]; ++s) if (seg[s] == am) qs = 1.0;
      J->Z[o] = 1.0; J->QS[o] = qs; J->q_lse[o] = l[am];
      if (J->tokens_out) J->tokens_out[o] = am;
      if (J->tok_lo) { J->tok_lo[o] = am; J->tok_hi[o] = am; }
      continue;
    }
    J->q_lse[o] = softmax_row(l, V, J->T, q);
    double QSj;
    J->Z[o] = saguaro_row(q, V, seg, F[j], J->C, &QSj, qp);
    J->QS[o] = QSj;
    if (J->tokens_out) {
      double tot = 0.0, mg;
      int32_t wl, wh;
      for (int v = 0; v < V; ++v) tot += qp[v];
      J->tokens_out[o] = inverse_cdf(qp, V, tot, (double)J->u_draft[(size_t)b * (size_t)K + (size_t)j], &mg,
                                     &wl, &wh);
      if (J->tok_lo) { J->tok_lo[o] = wl; J->tok_hi[o] = wh; }
      if (mg < worst) worst = mg;
    }
  }
  if (worst < SSDO_NEAR_TIE) st |= SSDO_ROW_NEAR_TIE;
  if (J->margin) J->margin[i] = worst;
  J->status[i] = st;
  free(l); free(q); free(qp);
}

int ssdo_reweight_batch(int dtype, int B, int K, int V, int budget, const void* draft, double T,
                        const int32_t* F, double C, const float* u_draft,
                        const int32_t* rows, int n_rows, int n_threads,
                        int32_t* topf_tokens, int32_t* offsets, double* Z, double* QS, double* q_lse,
                        int32_t* tokens_out, double* margin, int32_t* status, int32_t* tok_lo,
                        int32_t* tok_hi) {
  if (B < 0 || K < 1 || V < 1 || !(T >= 0.0) || !(C > 0.0 && C <= 1.0) || !F) return -1;
  if (budget < 0 || budget > V) return -1;
  if (dtype != SSDO_DTYPE_FP32 && dtype != SSDO_DTYPE_BF16) return -1;
  if (tokens_out && !u_draft) return -1;
  reweight_job J = {dtype, B, K, V, budget, draft, T, F, C, u_draft, rows, rows ? n_rows : B,
                    topf_tokens, offsets, Z, QS, q_lse, tokens_out, margin, status, tok_lo, tok_hi};
  run_rows(&J, J.n_rows, n_threads, reweight_row);
  return 0;
}

/* Overlap sum_v min(p(v), q(v)) of two temperature softmaxes: the expected
 * acceptance of plain speculative sampling, used to state the fan-out's
 * alpha for a synthetic workload. */
double ssdo_overlap(int dtype, const void* lp, const void* lq, int V, double T) {
  double* a = calloc((size_t)V, sizeof(double));
  double* b = calloc((size_t)V, sizeof(double));
  double* pa = malloc(sizeof(double) * (size_t)V);
  double* pb = malloc(sizeof(double) * (size_t)V);
  load_row(lp, dtype, 0, V, a);
  load_row(lq, dtype, 0, V, b);
  softmax_row(a, V, T, pa);
  softmax_row(b, V, T, pb);
  double s = 0.0;
  for (int v = 0; v < V; ++v) s += pa[v] < pb[v] ? pa[v] : pb[v];
  free(a); free(b); free(pa); free(pb);
  return s;
}

/* Cache lookup on its own ([ZH] section 2, basic flow step 4): segment k of
 * row b is tokens[b, offsets[b,k] : offsets[b,k+1]]; hit iff the bonus is in
 * segment k.  slot = its index in the row's token list, -1 on a miss. */
int ssdo_cache_lookup(int B, int K, int budget, const int32_t* offsets, const int32_t* tokens,
                      const int32_t* k, const int32_t* bonus, const int32_t* payload,
                      uint64_t fallback_seed, int V, uint8_t* hit, int32_t* slot, int32_t* next_tokens) {
  for (int b = 0; b < B; ++b) {
    int32_t sl = -1;
    int kk = k[b];
    if (kk >= 0 && kk <= K) {
      const int32_t* o = offsets + (size_t)b * (size_t)(K + 2);
      for (int s = o[kk]; s < o[kk + 1] && s < budget; ++s)
        if (s >= 0 && tokens[(size_t)b * (size_t)budget + (size_t)s] == bonus[b]) { sl = s; break; }
    }
    hit[b] = sl >= 0;
    slot[b] = sl;
    for (int t = 0; t < K; ++t) {
      if (sl >= 0)
        next_tokens[(size_t)b * K + t] = payload ? payload[((size_t)b * (size_t)budget + (size_t)sl) * (size_t)K + (size_t)t] : -1;
      else
        next_tokens[(size_t)b * K + t] = ssdo_fallback_token(fallback_seed, b, t, V);
    }
  }
  return 0;
}
