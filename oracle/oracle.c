/*
 * Plain CPU fp64 oracle for block-draft speculative verification.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by the tests, the smoke check and the
 * benchmark's CPU-baseline leg, never by the product library. It shares no
 * code, header, table or constant with the CUDA path.
 *
 * Style: one loop per definition, in the order the method states its steps,
 * fp64 throughout, libm exp/log, sums taken in ascending index order. No
 * blocking, fusion or reordering; threads only split independent requests.
 * Build: gcc -std=c11 -O2 -ffp-contract=off -fPIC -shared (no fast-math).
 */
#include "oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- inputs */

static int esize(int dtype) { return dtype == ORC_F32 ? 4 : 2; }

/* Exact widening of one stored logit: fp32 as is, bf16 as its top 16 bits. */
static double load_x(const void* base, int dtype, int64_t idx) {
  float f;
  if (dtype == ORC_F32) {
    f = ((const float*)base)[idx];
  } else {
    uint32_t bits = (uint32_t)((const uint16_t*)base)[idx] << 16;
    memcpy(&f, &bits, sizeof f);
  }
  return (double)f;
}

static const void* row_at(const void* base, int dtype, int64_t row, int64_t stride) {
  return (const char*)base + row * stride * esize(dtype);
}

/* ------------------------------------------------------ temperature softmax */

/* z_v = x_v / T;  m = max_v z_v;  lse = m + log sum_v exp(z_v - m).
 * The same temperature scales target and draft logits: both are sampled
 * with one sampling filter (DBLAST review, "Assumptions", and "What would
 * settle it": target sampling at T = 1.5). */
static void row_softmax_stats(const void* row, int dtype, int64_t V, double T,
                              double* m_out, double* lse_out) {
  double m = -INFINITY;
  for (int64_t v = 0; v < V; ++v) {
    double z = load_x(row, dtype, v) / T;
    if (z > m) m = z;
  }
  double s = 0.0;
  for (int64_t v = 0; v < V; ++v) s += exp(load_x(row, dtype, v) / T - m);
  *m_out = m;
  *lse_out = m + log(s);
}

int oracle_softmax_T(const void* x, int dtype, int64_t rows, int64_t V, int64_t row_stride,
                     double T, double* row_max, double* row_lse, double* probs) {
  if (!x || rows < 0 || V < 1 || row_stride < V || !(T > 0.0) || !row_max || !row_lse ||
      (dtype != ORC_F32 && dtype != ORC_BF16))
    return ORC_ERR_ARG;
  for (int64_t r = 0; r < rows; ++r) {
    const void* row = row_at(x, dtype, r, row_stride);
    row_softmax_stats(row, dtype, V, T, &row_max[r], &row_lse[r]);
    if (probs)
      for (int64_t v = 0; v < V; ++v)
        probs[r * V + v] = exp(load_x(row, dtype, v) / T - row_lse[r]);
  }
  return ORC_OK;
}

/* ---------------------------------------------------------- verification */

/* log sum_k exp(a_k), with the maximum factored out; -inf if every a_k is -inf. */
static double logsumexp(const double* a, int n) {
  double m = -INFINITY;
  for (int k = 0; k < n; ++k)
    if (a[k] > m) m = a[k];
  if (m == -INFINITY) return -INFINITY;
  double s = 0.0;
  for (int k = 0; k < n; ++k) s += exp(a[k] - m);
  return m + log(s);
}

/* Top-p (nucleus) filtering of one temperature-softmax row: the sampling
 * filter of target sampling (DBLAST review, "What would settle it":
 * temperature 1.5 with top-p 0.95; "Assumptions": target probabilities are
 * taken under the same sampling filter). The nucleus is the shortest prefix
 * of the tokens ordered by probability (descending, ties to the lower index)
 * whose mass reaches top_p; filtered log-probabilities are log p(v) minus the
 * log of that mass inside it and -inf outside. A nucleus is kept as its last
 * member (log-probability, token) and the log of its mass. */
typedef struct {
  int all;          /* top_p >= 1: no filtering */
  double lp_cut;    /* log-probability of the last member */
  int64_t v_cut;    /* its token; equal log-probabilities are members up to it */
  double log_mass;  /* log of the nucleus mass */
  double margin;    /* min(mass with the last member - top_p, top_p - mass without it) */
} nucleus;

typedef struct { double lp; int64_t v; } ranked;

static int ranked_order(const void* pa, const void* pb) {
  const ranked* a = (const ranked*)pa;
  const ranked* b = (const ranked*)pb;
  if (a->lp > b->lp) return -1;
  if (a->lp < b->lp) return 1;
  return (a->v > b->v) - (a->v < b->v);
}

static void row_nucleus(const void* row, int dtype, int64_t V, double T, double lse, double top_p, nucleus* n) {
  n->all = top_p >= 1.0;
  n->lp_cut = -INFINITY;
  n->v_cut = V - 1;
  n->log_mass = 0.0;
  n->margin = INFINITY;
  if (n->all) return;
  ranked* r = malloc((size_t)V * sizeof(ranked));
  for (int64_t v = 0; v < V; ++v) {
    r[v].lp = load_x(row, dtype, v) / T - lse;
    r[v].v = v;
  }
  qsort(r, (size_t)V, sizeof(ranked), ranked_order);
  double mass = 0.0, before = 0.0;
  int64_t k = 0;
  for (; k < V; ++k) {
    before = mass;
    mass += exp(r[k].lp);
    if (mass >= top_p) break;
  }
  if (k == V) { /* rounding kept the total just below top_p: the whole row */
    k = V - 1;
    n->margin = top_p - mass;
  } else {
    n->margin = fmin(mass - top_p, top_p - before);
  }
  n->lp_cut = r[k].lp;
  n->v_cut = r[k].v;
  n->log_mass = log(mass);
  free(r);
}

/* Filtered log-probability of token v whose unfiltered one is lpv. */
static double nucleus_lp(const nucleus* n, double lpv, int64_t v) {
  if (n->all) return lpv;
  const int in = lpv > n->lp_cut || (lpv == n->lp_cut && v <= n->v_cut);
  return in ? lpv - n->log_mass : -INFINITY;
}

typedef struct {
  const void* target;
  const int32_t* target_row_off;
  const void* draft;
  int dtype;
  const int32_t* tokens;
  const int32_t* verify_len;
  const float* u;
  const float* g;
  const float* mix_w;
  int K, B, L;
  int64_t V;
  double T;
  double top_p;
  int32_t* accept_len;
  int32_t* out_tokens;
  const oracle_diag* diag;
} verify_args;

/* Category posterior after the accepted prefix x_0..x_{i-1}:
 *   log pi_i(z) = log q(z|y) + sum_{k<i} log q_k(x_k|y,z)  - normaliser over z.
 * This is Bayes' rule on the latent-mixture proposal
 *   q_dep(x_{1:b}|y) = sum_z q(z|y) prod_i q_i(x_i|y,z)
 * (DBLAST review, "What carries the argument", Eq. 5: verification conditions
 * on the accepted prefix through the category posterior). */
static int category_posterior(const double* logw, const double* lqz, int K, int L, int i,
                              double* logpi, double* scratch) {
  for (int z = 0; z < K; ++z) {
    double a = logw[z];
    for (int k = 0; k < i; ++k) a += lqz[z * L + k];
    scratch[z] = a;
  }
  double norm = logsumexp(scratch, K);
  if (!isfinite(norm)) return ORC_FLAG_NONFINITE;
  for (int z = 0; z < K; ++z) logpi[z] = scratch[z] - norm;
  return 0;
}

/* log q_i(v | x_<i) = log sum_z pi_i(z) q_i(v|y,z): the position-i proposal,
 * the mixture marginal under the posterior. For K = 1 it is log q_i(v|y). */
static double proposal_logprob(const double* logpi, const double* lq_v, int K, double* scratch) {
  for (int z = 0; z < K; ++z) scratch[z] = logpi[z] + lq_v[z];
  return logsumexp(scratch, K);
}

static int verify_one(const verify_args* a, int b) {
  const int K = a->K, L = a->L;
  const int64_t V = a->V;
  const double T = a->T;
  const oracle_diag* d = a->diag;
  int32_t* out = a->out_tokens + (int64_t)b * (L + 1);
  for (int i = 0; i <= L; ++i) out[i] = -1;
  a->accept_len[b] = -1;
  if (d) {
    for (int i = 0; i < L; ++i) {
      if (d->lp) d->lp[(int64_t)b * L + i] = NAN;
      if (d->lq) d->lq[(int64_t)b * L + i] = NAN;
      if (d->rho) d->rho[(int64_t)b * L + i] = NAN;
      if (d->accept_margin) d->accept_margin[(int64_t)b * L + i] = NAN;
    }
    if (d->terminal_row) d->terminal_row[b] = -1;
    if (d->terminal_kind) d->terminal_kind[b] = -1;
    if (d->argmax_gap) d->argmax_gap[b] = NAN;
    if (d->argmax_kappa) d->argmax_kappa[b] = NAN;
    if (d->terminal_dist)
      for (int64_t v = 0; v < V; ++v) d->terminal_dist[(int64_t)b * V + v] = 0.0;
    if (d->nucleus_margin) d->nucleus_margin[b] = NAN;
  }

  const int ell = a->verify_len ? a->verify_len[b] : L;
  if (ell < 0 || ell > L) return ORC_FLAG_VERIFY_LEN;
  const int32_t* x = a->tokens + (int64_t)b * L;
  for (int i = 0; i < ell; ++i)
    if (x[i] < 0 || (int64_t)x[i] >= V) return ORC_FLAG_TOKEN_RANGE;

  const int64_t trow0 = a->target_row_off ? (int64_t)a->target_row_off[b] : (int64_t)b * (L + 1);
  const void* trow[65];
  for (int i = 0; i <= ell; ++i) trow[i] = row_at(a->target, a->dtype, trow0 + i, V);
#define DROW(z, i) row_at(a->draft, a->dtype, ((int64_t)b * K + (z)) * L + (i), V)

  int flags = 0;
  double* lse_t = calloc((size_t)L + 1, sizeof(double));
  double* lse_d = calloc((size_t)K * L, sizeof(double));
  double* lqz = calloc((size_t)K * L, sizeof(double)); /* log q_k(x_k|y,z) */
  double* lp = calloc((size_t)L + 1, sizeof(double));  /* log p_k(x_k)     */
  double* logw = calloc((size_t)K, sizeof(double));
  double* logpi = calloc((size_t)K, sizeof(double));
  double* s1 = calloc((size_t)K, sizeof(double));
  double* s2 = calloc((size_t)K, sizeof(double));
  double* lqv = calloc((size_t)K, sizeof(double));
  nucleus* nt = calloc((size_t)L + 1, sizeof(nucleus));       /* target rows 0..ell */
  nucleus* nd = calloc((size_t)K * L + 1, sizeof(nucleus));   /* draft rows (z, i) */
  double* dist = d && d->terminal_dist ? d->terminal_dist + (int64_t)b * V : NULL;
  double m_unused;

  /* Step 1: temperature softmax normalisers (and, below top_p = 1, nuclei) of
   * every tested row. */
  for (int i = 0; i < ell; ++i) {
    row_softmax_stats(trow[i], a->dtype, V, T, &m_unused, &lse_t[i]);
    if (!isfinite(lse_t[i]) || !isfinite(m_unused)) flags |= ORC_FLAG_NONFINITE;
    for (int z = 0; z < K; ++z) {
      row_softmax_stats(DROW(z, i), a->dtype, V, T, &m_unused, &lse_d[z * L + i]);
      if (!isfinite(lse_d[z * L + i]) || !isfinite(m_unused)) flags |= ORC_FLAG_NONFINITE;
    }
  }
  if (flags) goto done;
  for (int i = 0; i < ell; ++i) {
    row_nucleus(trow[i], a->dtype, V, T, lse_t[i], a->top_p, &nt[i]);
    for (int z = 0; z < K; ++z) row_nucleus(DROW(z, i), a->dtype, V, T, lse_d[z * L + i], a->top_p, &nd[z * L + i]);
  }

  /* Step 2: (filtered) log-probabilities of the drafted tokens under target and branches. */
  for (int i = 0; i < ell; ++i) {
    lp[i] = nucleus_lp(&nt[i], load_x(trow[i], a->dtype, x[i]) / T - lse_t[i], x[i]);
    for (int z = 0; z < K; ++z)
      lqz[z * L + i] = nucleus_lp(&nd[z * L + i], load_x(DROW(z, i), a->dtype, x[i]) / T - lse_d[z * L + i], x[i]);
  }
  for (int z = 0; z < K; ++z) logw[z] = a->mix_w ? log((double)a->mix_w[(int64_t)b * K + z]) : 0.0;

  /* Step 3: sequential accept tests. Position i is accepted iff
   * u_i < min(1, p_i(x_i) / q_i(x_i)); the first failure stops the block
   * (speculative sampling with rejection correction, DBLAST review,
   * "Assumptions"; the verifier accepts tokens sequentially, "The reading"). */
  int j = ell;
  for (int i = 0; i < ell; ++i) {
    if ((flags |= category_posterior(logw, lqz, K, L, i, logpi, s1))) goto done;
    for (int z = 0; z < K; ++z) lqv[z] = lqz[z * L + i];
    const double lq = proposal_logprob(logpi, lqv, K, s2);
    /* A token outside the filtered target has p = 0, so rho = 0 (even when the
     * filtered proposal gives it 0 as well). */
    const double rho = (lp[i] == -INFINITY && a->top_p < 1.0) ? 0.0 : exp(lp[i] - lq);
    if (isnan(rho)) { flags |= ORC_FLAG_NONFINITE; goto done; }
    const double thr = rho < 1.0 ? rho : 1.0;
    const double ui = (double)a->u[(int64_t)b * L + i];
    if (d) {
      if (d->lp) d->lp[(int64_t)b * L + i] = lp[i];
      if (d->lq) d->lq[(int64_t)b * L + i] = lq;
      if (d->rho) d->rho[(int64_t)b * L + i] = rho;
      if (d->accept_margin) d->accept_margin[(int64_t)b * L + i] = fabs(ui - thr);
    }
    if (!(ui < thr)) { j = i; break; }
  }

  /* Step 4: the terminal token. After a rejection at j it is drawn from the
   * residual norm(max(0, p_j - q_j)); when all ell positions pass it is the
   * bonus draw from target row ell. Both draws are Gumbel-max over the
   * caller's noise row g[b, j, :]; ties go to the lowest index. */
  const float* gj = a->g + ((int64_t)b * (L + 1) + j) * V;
  int kind;
  double best1 = -INFINITY, best2 = -INFINITY, kap1 = 1.0, kap2 = 1.0;
  int64_t t = -1;
  if (j < ell) {
    kind = 0;
    if ((flags |= category_posterior(logw, lqz, K, L, j, logpi, s1))) goto done;
    double rsum = 0.0;
    for (int64_t v = 0; v < V; ++v) {
      const double lpv = nucleus_lp(&nt[j], load_x(trow[j], a->dtype, v) / T - lse_t[j], v);
      for (int z = 0; z < K; ++z)
        lqv[z] = nucleus_lp(&nd[z * L + j], load_x(DROW(z, j), a->dtype, v) / T - lse_d[z * L + j], v);
      const double lqv_mix = proposal_logprob(logpi, lqv, K, s2);
      const double pv = exp(lpv), qv = exp(lqv_mix);
      const double r = pv - qv;
      if (!(r > 0.0)) continue;
      if (dist) { dist[v] = r; rsum += r; }
      const double score = log(r) + (double)gj[v];
      const double kap = pv / r;
      if (score > best1) {
        best2 = best1; kap2 = kap1; best1 = score; kap1 = kap; t = v;
      } else if (score > best2) {
        best2 = score; kap2 = kap;
      }
    }
    if (dist && rsum > 0.0)
      for (int64_t v = 0; v < V; ++v) dist[v] /= rsum;
  }
  if (j == ell || t < 0) {
    /* Bonus draw (or, if no residual mass survived rounding, the same rule on
     * row j): score_v = log p(v) + g_v. */
    kind = (j == ell) ? 1 : 2;
    double lse;
    if (j == ell) {
      row_softmax_stats(trow[ell], a->dtype, V, T, &m_unused, &lse);
      if (!isfinite(lse) || !isfinite(m_unused)) { flags |= ORC_FLAG_NONFINITE; goto done; }
      row_nucleus(trow[ell], a->dtype, V, T, lse, a->top_p, &nt[ell]);
    } else {
      lse = lse_t[j];
    }
    best1 = best2 = -INFINITY; kap1 = kap2 = 1.0; t = -1;
    for (int64_t v = 0; v < V; ++v) {
      const double lpv = nucleus_lp(&nt[j], load_x(trow[j], a->dtype, v) / T - lse, v);
      if (dist) dist[v] = exp(lpv);
      const double score = lpv + (double)gj[v];
      if (score > best1) {
        best2 = best1; best1 = score; t = v;
      } else if (score > best2) {
        best2 = score;
      }
    }
  }
  if (t < 0) { flags |= ORC_FLAG_NONFINITE; goto done; }

  for (int i = 0; i < j; ++i) out[i] = x[i];
  out[j] = (int32_t)t;
  a->accept_len[b] = j;
  if (d) {
    if (d->nucleus_margin) { /* rows 0..j of target and drafts (their tests and the residual), or the bonus row */
      double mg = INFINITY;
      const int last = j < ell ? j : ell - 1;
      for (int i = 0; i <= last; ++i) {
        mg = fmin(mg, nt[i].margin);
        for (int z = 0; z < K; ++z) mg = fmin(mg, nd[z * L + i].margin);
      }
      if (j == ell) mg = fmin(mg, nt[ell].margin);
      d->nucleus_margin[b] = mg;
    }
    if (d->terminal_row) d->terminal_row[b] = j;
    if (d->terminal_kind) d->terminal_kind[b] = kind;
    if (d->argmax_gap) d->argmax_gap[b] = best1 - best2; /* +inf with a single candidate */
    if (d->argmax_kappa) {
      double k = kap1 > kap2 ? kap1 : kap2;
      d->argmax_kappa[b] = k > 1.0 ? k : 1.0;
    }
  }

done:
#undef DROW
  if (flags) {
    for (int i = 0; i <= L; ++i) out[i] = -1;
    a->accept_len[b] = -1;
  }
  free(lse_t); free(lse_d); free(lqz); free(lp); free(logw); free(logpi);
  free(s1); free(s2); free(lqv); free(nt); free(nd);
  return flags;
}

typedef struct {
  const verify_args* a;
  int first, step;
  int flags;
} verify_job;

static void* verify_worker(void* p) {
  verify_job* job = (verify_job*)p;
  for (int b = job->first; b < job->a->B; b += job->step) job->flags |= verify_one(job->a, b);
  return NULL;
}

int oracle_verify(const void* target, const int32_t* target_row_off, const void* draft, int dtype,
                  const int32_t* tokens, const int32_t* verify_len, const float* u, const float* g,
                  const float* mix_w, int K, int B, int L, int64_t V, double T, double top_p, int n_threads,
                  int32_t* accept_len, int32_t* out_tokens, const oracle_diag* diag) {
  if (!target || !draft || !tokens || !u || !g || !accept_len || !out_tokens) return ORC_ERR_ARG;
  if (dtype != ORC_F32 && dtype != ORC_BF16) return ORC_ERR_ARG;
  if (B < 0 || L < 0 || L > 64 || V < 1 || K < 1 || !(T > 0.0)) return ORC_ERR_ARG;
  if (!(top_p > 0.0 && top_p <= 1.0)) return ORC_ERR_ARG;
  if (!mix_w && K != 1) return ORC_ERR_ARG;
  verify_args a = {target, target_row_off, draft, dtype, tokens, verify_len, u, g, mix_w,
                   K, B, L, V, T, top_p, accept_len, out_tokens, diag};
  if (n_threads < 1) n_threads = 1;
  if (n_threads > B) n_threads = B > 0 ? B : 1;
  verify_job* jobs = calloc((size_t)n_threads, sizeof(verify_job));
  pthread_t* th = calloc((size_t)n_threads, sizeof(pthread_t));
  for (int k = 0; k < n_threads; ++k) {
    jobs[k].a = &a; jobs[k].first = k; jobs[k].step = n_threads; jobs[k].flags = 0;
  }
  for (int k = 1; k < n_threads; ++k) pthread_create(&th[k], NULL, verify_worker, &jobs[k]);
  verify_worker(&jobs[0]);
  int flags = jobs[0].flags;
  for (int k = 1; k < n_threads; ++k) {
    pthread_join(th[k], NULL);
    flags |= jobs[k].flags;
  }
  free(jobs); free(th);
  return flags;
}

/* -------------------------------------------------------- DVL allocation */

typedef struct { double P; int b, i; } dvl_entry;

/* (P desc, b asc, i asc) */
static int dvl_order(const void* pa, const void* pb) {
  const dvl_entry* x = pa;
  const dvl_entry* y = pb;
  if (x->P > y->P) return -1;
  if (x->P < y->P) return 1;
  if (x->b != y->b) return x->b < y->b ? -1 : 1;
  if (x->i != y->i) return x->i < y->i ? -1 : 1;
  return 0;
}

/* DScale, Abstract: dynamic verify-length allocation packs scored prefixes
 * into half the native verification capacity. Position i of request b is
 * worth its prefix-survival probability P[b,i] = prod_{k<=i} s[b,k] (the
 * block-diffusion failure-mode Q&A: verify length from prefix survival
 * probabilities). Every request keeps its root slot; the remaining
 * budget' - B slots go to the largest P overall. */
int oracle_dvl_allocate(const float* scores, int B, int L, int budget,
                        int32_t* verify_len, int32_t* offsets, int32_t* slot_map, double* prefix) {
  if (!scores || !verify_len || !offsets || B < 1 || L < 0 || budget < B) return ORC_ERR_ARG;
  int flags = 0;
  for (int64_t k = 0; k < (int64_t)B * L; ++k)
    if (!(scores[k] >= 0.0f && scores[k] <= 1.0f)) flags |= ORC_FLAG_SCORES;
  const int64_t cap = (int64_t)B * (L + 1);
  const int64_t used = budget < cap ? budget : cap;
  const int64_t take = used - B;

  dvl_entry* e = calloc((size_t)B * L + 1, sizeof(dvl_entry));
  for (int b = 0; b < B; ++b) {
    double P = 1.0;
    for (int i = 0; i < L; ++i) {
      P = P * (double)scores[(int64_t)b * L + i];
      e[(int64_t)b * L + i] = (dvl_entry){P, b, i};
      if (prefix) prefix[(int64_t)b * L + i] = P;
    }
  }
  qsort(e, (size_t)B * L, sizeof(dvl_entry), dvl_order);
  for (int b = 0; b < B; ++b) verify_len[b] = 0;
  for (int64_t k = 0; k < take; ++k) verify_len[e[k].b] += 1;
  free(e);

  offsets[0] = 0;
  for (int b = 0; b < B; ++b) offsets[b + 1] = offsets[b] + verify_len[b] + 1;
  if (slot_map) {
    for (int s = 0; s < budget; ++s) slot_map[s] = -1;
    for (int b = 0; b < B; ++b)
      for (int i = 0; i <= verify_len[b]; ++i) slot_map[offsets[b] + i] = b * (L + 1) + i;
  }
  return flags;
}

int oracle_pack(const void* dense, int dtype, int B, int L, int64_t V,
                const int32_t* verify_len, const int32_t* offsets, void* packed) {
  if (!dense || !verify_len || !offsets || !packed || B < 0 || L < 0 || V < 1) return ORC_ERR_ARG;
  const size_t row_bytes = (size_t)V * esize(dtype);
  for (int b = 0; b < B; ++b)
    for (int i = 0; i <= verify_len[b]; ++i)
      memcpy((char*)packed + (size_t)(offsets[b] + i) * row_bytes,
             (const char*)dense + ((size_t)b * (L + 1) + i) * row_bytes, row_bytes);
  return ORC_OK;
}
