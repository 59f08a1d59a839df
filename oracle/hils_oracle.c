/*
 * hils_oracle.c -- fp64 CPU oracle of the HiLS attention forward pass (test infrastructure).
 * The header states the steps, the sources and the readings R1-R11; this file takes the steps
 * in that order for one (query token, KV head) at a time, with no blocking or fusion.
 */
#define _GNU_SOURCE
#include "hils_oracle.h"

#include <math.h>
#include <pthread.h>
#include <sched.h>
#include <stdatomic.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* Rule R1 (eligibility). */
int64_t hils_oracle_n_eligible(int64_t pos, int32_t S, int32_t W) {
  int64_t first_window_token = pos - (int64_t)W + 1;
  if (first_window_token <= 0) return 0;
  return first_window_token / S;
}

int hils_oracle_default_threads(void) {
  cpu_set_t set;
  CPU_ZERO(&set);
  if (sched_getaffinity(0, sizeof(set), &set) == 0) {
    int n = CPU_COUNT(&set);
    if (n > 0) return n;
  }
  long n = sysconf(_SC_NPROCESSORS_ONLN);
  return n > 0 ? (int)n : 1;
}

static double dot(const double* a, const double* b, int d) {
  double acc = 0.0;
  for (int k = 0; k < d; ++k) acc += a[k] * b[k];
  return acc;
}

static const double* token_row(const hils_oracle_rows* r, int64_t j, int d) {
  if (j < 0 || j >= r->n_tokens) return NULL;
  int64_t row = r->row_map ? r->row_map[j] : j;
  if (row < 0) return NULL;
  return r->base + row * (int64_t)d;
}

typedef struct {
  double sigma;
  int64_t c;
} candidate;

/* Rule R5: larger sigma first; equal sigma -> lower chunk index first. */
static int by_sigma_desc_then_index(const void* pa, const void* pb) {
  const candidate* a = (const candidate*)pa;
  const candidate* b = (const candidate*)pb;
  if (a->sigma > b->sigma) return -1;
  if (a->sigma < b->sigma) return 1;
  return (a->c < b->c) ? -1 : (a->c > b->c ? 1 : 0);
}

/* Step 3 for one unit: exact softmax attention of query q over tokens [t0, t1).
 * Writes lse and o (d values).  Returns 0 or HILS_ORACLE_EROW. */
static int attend_unit(const double* q, const hils_oracle_rows* K, const hils_oracle_rows* V,
                       int64_t t0, int64_t t1, int d, double scale, double* x_buf,
                       double* lse, double* o) {
  double m = -INFINITY;
  for (int64_t j = t0; j < t1; ++j) {
    const double* kj = token_row(K, j, d);
    if (!kj) return HILS_ORACLE_EROW;
    double x = dot(q, kj, d) * scale;
    x_buf[j - t0] = x;
    if (x > m) m = x;
  }
  double sum = 0.0;
  for (int64_t j = t0; j < t1; ++j) sum += exp(x_buf[j - t0] - m);
  double l = m + log(sum);
  for (int k = 0; k < d; ++k) o[k] = 0.0;
  for (int64_t j = t0; j < t1; ++j) {
    const double* vj = token_row(V, j, d);
    if (!vj) return HILS_ORACLE_EROW;
    double p = exp(x_buf[j - t0] - l);
    for (int k = 0; k < d; ++k) o[k] += p * vj[k];
  }
  *lse = l;
  return HILS_ORACLE_OK;
}

static int run_job(const hils_oracle_cfg* cfg, hils_oracle_job* jb) {
  const int d = cfg->d, G = cfg->G, S = cfg->S, Kt = cfg->K_top;
  const double scale = cfg->scale > 0.0 ? cfg->scale : 1.0 / sqrt((double)d);
  const int64_t p = jb->pos;
  if (d <= 0 || G <= 0 || S <= 0 || Kt < 0 || cfg->W < 1 || p < 0) return HILS_ORACLE_EINVAL;

  /* R1: eligible distant chunks and the local window [ell, p]. */
  const int64_t n = hils_oracle_n_eligible(p, S, cfg->W);
  if (n > cfg->n_chunks) return HILS_ORACLE_EINVAL;
  const int64_t ell = (int64_t)S * n;

  int rc = HILS_ORACLE_OK;
  candidate* cand = (candidate*)malloc((size_t)(n > 0 ? n : 1) * sizeof(candidate));
  int64_t* sel = (int64_t*)malloc((size_t)(Kt > 0 ? Kt : 1) * sizeof(int64_t));
  double* sel_sigma = (double*)malloc((size_t)(Kt > 0 ? Kt : 1) * sizeof(double));
  int64_t max_unit = (p - ell + 1) > S ? (p - ell + 1) : S;
  double* x_buf = (double*)malloc((size_t)max_unit * sizeof(double));
  double* unit_lse = (double*)malloc((size_t)(Kt + 1) * sizeof(double));
  double* unit_o = (double*)malloc((size_t)(Kt + 1) * (size_t)d * sizeof(double));
  double* score = (double*)malloc((size_t)(Kt + 1) * sizeof(double));
  if (!cand || !sel || !sel_sigma || !x_buf || !unit_lse || !unit_o || !score) {
    rc = HILS_ORACLE_ENOMEM;
    goto done;
  }

  /* Step 1: per-head surrogate scores, group score sigma = max over heads (R4). */
  for (int64_t c = 0; c < n; ++c) {
    const double* kc = jb->klm + c * (int64_t)d;
    double sig = -INFINITY;
    for (int h = 0; h < G; ++h) {
      double s = dot(jb->qc + h * jb->qc_hs, kc, d) * scale + jb->blm[c];
      if (s > sig) sig = s;
    }
    cand[c].sigma = sig;
    cand[c].c = c;
  }

  /* Step 2: order all candidates (R5) and keep the first min(K, n) (R7). */
  int64_t k_sel = 0;
  double gap = INFINITY;
  if (jb->idx_in == NULL) {
    qsort(cand, (size_t)n, sizeof(candidate), by_sigma_desc_then_index);
    k_sel = n < Kt ? n : Kt;
    for (int64_t r = 0; r < k_sel; ++r) {
      sel[r] = cand[r].c;
      sel_sigma[r] = cand[r].sigma;
    }
    if (n > Kt && Kt > 0) {
      double a = cand[Kt - 1].sigma, b = cand[Kt].sigma;
      gap = (a == b) ? 0.0 : a - b;
    } else if (n > Kt) {
      gap = INFINITY;
    }
  } else {
    /* Forced selection (used where near-ties make several selections valid). */
    for (int r = 0; r < Kt; ++r) {
      int64_t c = jb->idx_in[r];
      if (c < 0) continue;
      if (c >= n) { rc = HILS_ORACLE_EINVAL; goto done; }
      for (int64_t t = 0; t < k_sel; ++t)
        if (sel[t] == c) { rc = HILS_ORACLE_EINVAL; goto done; }
      sel[k_sel] = c;
      sel_sigma[k_sel] = cand[c].sigma;
      ++k_sel;
    }
    gap = NAN;
  }
  if (jb->idx_out)
    for (int r = 0; r < Kt; ++r) jb->idx_out[r] = r < k_sel ? (int32_t)sel[r] : -1;
  if (jb->sigma_out)
    for (int r = 0; r < Kt; ++r) jb->sigma_out[r] = r < k_sel ? sel_sigma[r] : -INFINITY;
  if (jb->gap_out) *jb->gap_out = gap;

  /* Steps 3 and 4 for each head of the group (skipped when none of their outputs is wanted,
   * so a selection-only job needs no K/V rows). */
  const int want_attend = jb->out || jb->lse_out || jb->unit_o_out || jb->unit_lse_out;
  for (int h = 0; h < G; ++h) {
    const double* qh = jb->q + h * jb->q_hs;
    const double* qch = jb->qc + h * jb->qc_hs;
    /* this head's own surrogate score of each selected chunk (R4) */
    for (int64_t r = 0; r < k_sel; ++r) {
      int64_t c = sel[r];
      score[r] = dot(qch, jb->klm + c * (int64_t)d, d) * scale + jb->blm[c];
    }
    if (!want_attend) {
      if (jb->s_sel_out)
        for (int r = 0; r < Kt; ++r)
          jb->s_sel_out[h * jb->s_sel_hs + r] = r < k_sel ? score[r] : -INFINITY;
      continue;
    }
    /* step 3: one unit per selected chunk, then the local window as unit Kt */
    for (int64_t r = 0; r < k_sel; ++r) {
      int64_t c = sel[r];
      rc = attend_unit(qh, &jb->K, &jb->V, c * S, c * S + S, d, scale, x_buf, &unit_lse[r],
                       unit_o + r * d);
      if (rc) goto done;
    }
    for (int64_t r = k_sel; r < Kt; ++r) {
      unit_lse[r] = -INFINITY;
      score[r] = -INFINITY;
      for (int k = 0; k < d; ++k) unit_o[r * d + k] = 0.0;
    }
    rc = attend_unit(qh, &jb->K, &jb->V, ell, p + 1, d, scale, x_buf, &unit_lse[Kt],
                     unit_o + (int64_t)Kt * d);
    if (rc) goto done;
    score[Kt] = unit_lse[Kt]; /* R2 */

    /* step 4: softmax over the unit scores (R3), fused output and its logsumexp */
    double m = -INFINITY;
    for (int u = 0; u <= Kt; ++u)
      if (score[u] > m) m = score[u];
    double z = 0.0;
    for (int u = 0; u <= Kt; ++u) z += exp(score[u] - m);
    if (jb->out) {
      double* oh = jb->out + h * jb->out_hs;
      for (int k = 0; k < d; ++k) oh[k] = 0.0;
      for (int u = 0; u <= Kt; ++u) {
        double w = exp(score[u] - m) / z;
        if (w == 0.0) continue;
        for (int k = 0; k < d; ++k) oh[k] += w * unit_o[u * d + k];
      }
    }
    if (jb->lse_out) jb->lse_out[h * jb->lse_hs] = m + log(z);
    if (jb->s_sel_out)
      for (int r = 0; r < Kt; ++r) jb->s_sel_out[h * jb->s_sel_hs + r] = score[r];
    if (jb->unit_o_out)
      memcpy(jb->unit_o_out + h * jb->unit_o_hs, unit_o,
             (size_t)(Kt + 1) * (size_t)d * sizeof(double));
    if (jb->unit_lse_out)
      for (int u = 0; u <= Kt; ++u) jb->unit_lse_out[h * jb->unit_lse_hs + u] = unit_lse[u];
  }

done:
  free(cand);
  free(sel);
  free(sel_sigma);
  free(x_buf);
  free(unit_lse);
  free(unit_o);
  free(score);
  return rc;
}

typedef struct {
  const hils_oracle_cfg* cfg;
  hils_oracle_job* jobs;
  int64_t n_jobs;
  atomic_llong next;
} pool_ctx;

static void* pool_worker(void* arg) {
  pool_ctx* ctx = (pool_ctx*)arg;
  for (;;) {
    long long j = atomic_fetch_add(&ctx->next, 1);
    if (j >= ctx->n_jobs) break;
    ctx->jobs[j].status = run_job(ctx->cfg, &ctx->jobs[j]);
  }
  return NULL;
}

int hils_oracle_run(const hils_oracle_cfg* cfg, int64_t n_jobs, hils_oracle_job* jobs,
                    int n_threads) {
  if (!cfg || (n_jobs > 0 && !jobs) || n_jobs < 0) return HILS_ORACLE_EINVAL;
  if (n_threads <= 0) n_threads = hils_oracle_default_threads();
  if (n_threads > n_jobs) n_threads = (int)(n_jobs > 0 ? n_jobs : 1);
  pool_ctx ctx;
  ctx.cfg = cfg;
  ctx.jobs = jobs;
  ctx.n_jobs = n_jobs;
  atomic_init(&ctx.next, 0);
  if (n_threads <= 1) {
    pool_worker(&ctx);
  } else {
    pthread_t* th = (pthread_t*)malloc((size_t)n_threads * sizeof(pthread_t));
    if (!th) return HILS_ORACLE_ENOMEM;
    int started = 0;
    for (; started < n_threads; ++started)
      if (pthread_create(&th[started], NULL, pool_worker, &ctx) != 0) break;
    if (started == 0) pool_worker(&ctx);
    for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
    free(th);
  }
  for (int64_t j = 0; j < n_jobs; ++j)
    if (jobs[j].status != HILS_ORACLE_OK) return jobs[j].status;
  return HILS_ORACLE_OK;
}

int hils_oracle_forward(const hils_oracle_problem* pr, const double* q, const double* qc,
                        const double* K, const double* V, const double* klm, const double* blm,
                        const int32_t* idx_in, int32_t* idx_out, double* sigma_out,
                        double* gap_out, double* s_sel_out, double* out, double* lse_out,
                        double* unit_o_out, double* unit_lse_out, int n_threads) {
  if (!pr || pr->B < 0 || pr->Hkv <= 0 || pr->Hq <= 0 || pr->Hq % pr->Hkv != 0 ||
      pr->d <= 0 || pr->S <= 0 || pr->K_top < 0 || pr->W < 1 || pr->N_q < 0 ||
      pr->q_pos0 < 0 || pr->q_pos0 + pr->N_q > pr->N_kv)
    return HILS_ORACLE_EINVAL;
  const int64_t G = pr->Hq / pr->Hkv, d = pr->d, Nq = pr->N_q, Nkv = pr->N_kv;
  const int64_t C = Nkv / pr->S, Kt = pr->K_top;
  hils_oracle_cfg cfg;
  cfg.d = (int32_t)d;
  cfg.G = (int32_t)G;
  cfg.S = pr->S;
  cfg.K_top = pr->K_top;
  cfg.W = pr->W;
  cfg.n_chunks = C;
  cfg.scale = pr->scale;
  const int64_t n_jobs = pr->B * pr->Hkv * Nq;
  hils_oracle_job* jobs = (hils_oracle_job*)calloc((size_t)(n_jobs > 0 ? n_jobs : 1),
                                                   sizeof(hils_oracle_job));
  if (!jobs) return HILS_ORACLE_ENOMEM;
  int64_t jn = 0;
  for (int64_t b = 0; b < pr->B; ++b)
    for (int64_t g = 0; g < pr->Hkv; ++g)
      for (int64_t i = 0; i < Nq; ++i, ++jn) {
        hils_oracle_job* jb = &jobs[jn];
        const int64_t h0 = g * G;
        const int64_t qrow = ((b * pr->Hq + h0) * Nq + i);   /* first head's row */
        const int64_t bg = b * pr->Hkv + g;
        jb->pos = pr->q_pos0 + i;
        jb->q = q + qrow * d;
        jb->q_hs = Nq * d;
        jb->qc = qc + qrow * d;
        jb->qc_hs = Nq * d;
        jb->klm = klm + bg * C * d;
        jb->blm = blm + bg * C;
        jb->K.base = K + bg * Nkv * d;
        jb->K.row_map = NULL;
        jb->K.n_tokens = Nkv;
        jb->V.base = V + bg * Nkv * d;
        jb->V.row_map = NULL;
        jb->V.n_tokens = Nkv;
        const int64_t sel_row = (bg * Nq + i) * Kt;
        jb->idx_in = idx_in ? idx_in + sel_row : NULL;
        jb->idx_out = idx_out ? idx_out + sel_row : NULL;
        jb->sigma_out = sigma_out ? sigma_out + sel_row : NULL;
        jb->gap_out = gap_out ? gap_out + (bg * Nq + i) : NULL;
        jb->s_sel_out = s_sel_out ? s_sel_out + qrow * Kt : NULL;
        jb->s_sel_hs = Nq * Kt;
        jb->out = out ? out + qrow * d : NULL;
        jb->out_hs = Nq * d;
        jb->lse_out = lse_out ? lse_out + qrow : NULL;
        jb->lse_hs = Nq;
        jb->unit_o_out = unit_o_out ? unit_o_out + qrow * (Kt + 1) * d : NULL;
        jb->unit_o_hs = Nq * (Kt + 1) * d;
        jb->unit_lse_out = unit_lse_out ? unit_lse_out + qrow * (Kt + 1) : NULL;
        jb->unit_lse_hs = Nq * (Kt + 1);
      }
  int rc = hils_oracle_run(&cfg, n_jobs, jobs, n_threads);
  free(jobs);
  return rc;
}

int hils_oracle_landmarks(int64_t B, int64_t Hkv, int64_t N_kv, int64_t d, int32_t S,
                          double scale, const double* qlm, const double* K, double* klm,
                          double* blm) {
  if (B < 0 || Hkv <= 0 || N_kv < 0 || d <= 0 || S <= 0) return HILS_ORACLE_EINVAL;
  const int64_t C = N_kv / S;
  const double sc = scale > 0.0 ? scale : 1.0 / sqrt((double)d);
  double* x = (double*)malloc((size_t)S * sizeof(double));
  if (!x) return HILS_ORACLE_ENOMEM;
  for (int64_t bg = 0; bg < B * Hkv; ++bg)
    for (int64_t c = 0; c < C; ++c) {
      const double* qv = qlm + (bg * C + c) * d;
      const double* Kc = K + (bg * N_kv + c * S) * d;   /* the chunk's S keys */
      double* kout = klm + (bg * C + c) * d;
      /* the landmark query's logits and their softmax */
      double m = -INFINITY;
      for (int32_t j = 0; j < S; ++j) {
        x[j] = sc * dot(qv, Kc + (int64_t)j * d, (int)d);
        if (x[j] > m) m = x[j];
      }
      double z = 0.0;
      for (int32_t j = 0; j < S; ++j) z += exp(x[j] - m);
      /* summary key and entropy bias */
      for (int64_t e = 0; e < d; ++e) kout[e] = 0.0;
      double h = 0.0;
      for (int32_t j = 0; j < S; ++j) {
        const double pj = exp(x[j] - m) / z;
        for (int64_t e = 0; e < d; ++e) kout[e] += pj * Kc[(int64_t)j * d + e];
        if (pj > 0.0) h -= pj * log(pj);
      }
      blm[bg * C + c] = h;
    }
  free(x);
  return HILS_ORACLE_OK;
}
