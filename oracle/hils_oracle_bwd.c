/*
 * hils_oracle_bwd.c -- fp64 CPU oracle of the HiLS attention backward pass (test
 * infrastructure).  Reverse-mode differentiation of the forward defined in hils_oracle.h, with
 * the selection held fixed: the top-K is piecewise constant in its inputs, so it passes no
 * gradient, and the gradient reaches the landmark keys and biases through the fusion weights
 * only ([Reader] Fig. 3 caption: the loss gradient flows back to the compressed key through the
 * chunk weights; [Reader] "The HiLS-Attention Mechanism": the surrogate score is differentiable
 * where the exact chunk mass is not).
 *
 * For the scalar L = sum dO . O + sum dlse . LSE, per (query token, head), taking the forward's
 * steps in reverse order, each one by the plain chain rule:
 *   step 4  w = softmax(score), O = sum_u w_u o_u, LSE = logsumexp(score):
 *             do_u = w_u dO;  dw_u = dO . o_u;
 *             dscore_u = w_u (dw_u - sum_v w_v dw_v) + dlse w_u.
 *   step 1  a chunk's score s = scale qc . klm_c + blm_c:
 *             dqc += scale dscore klm_c;  dklm_c += scale dscore qc;  dblm_c += dscore.
 *           the window's score is its own log-sum-exp (R2): it passes dscore_local on to that
 *           unit's lse.
 *   step 3  per unit, p_j = exp(x_j - lse_u), o_u = sum_j p_j V_j, lse_u = log sum_j exp(x_j):
 *             dV_j += p_j do_u;  dp_j = do_u . V_j;
 *             dx_j = p_j (dp_j - sum_k p_k dp_k) + p_j dlse_u;
 *           and x_j = scale q . K_j:  dq += scale dx_j K_j;  dK_j += scale dx_j q.
 * No step is merged with another or simplified.
 */
#define _GNU_SOURCE
#include <math.h>
#include <pthread.h>
#include <stdatomic.h>
#include <stdlib.h>
#include <string.h>

#include "hils_oracle.h"

static double bdot(const double* a, const double* b, int64_t d) {
  double acc = 0.0;
  for (int64_t k = 0; k < d; ++k) acc += a[k] * b[k];
  return acc;
}

static void baxpy(double alpha, const double* x, double* y, int64_t d) {
  for (int64_t k = 0; k < d; ++k) y[k] += alpha * x[k];
}

typedef struct {
  const hils_oracle_problem* pr;
  const double *q, *qc, *K, *V, *klm, *blm, *dO, *dlse;
  const int32_t* idx;
  double *dq, *dqc, *dK, *dV, *dklm, *dblm;
  atomic_llong next;
  atomic_int status;
} bwd_ctx;

/* One unit's tokens [t0, t1) for query q: logits x, lse, probabilities p (in x), output o. */
static void unit_forward(const double* q, const double* Kb, const double* Vb, int64_t t0,
                         int64_t t1, int64_t d, double scale, double* x, double* lse,
                         double* o) {
  double m = -INFINITY;
  for (int64_t j = t0; j < t1; ++j) {
    x[j - t0] = bdot(q, Kb + j * d, d) * scale;
    if (x[j - t0] > m) m = x[j - t0];
  }
  double z = 0.0;
  for (int64_t j = t0; j < t1; ++j) z += exp(x[j - t0] - m);
  *lse = m + log(z);
  for (int64_t k = 0; k < d; ++k) o[k] = 0.0;
  for (int64_t j = t0; j < t1; ++j) {
    x[j - t0] = exp(x[j - t0] - *lse);   /* now p_j */
    baxpy(x[j - t0], Vb + j * d, o, d);
  }
}

/* Step 3 in reverse for one unit: p holds its probabilities, do_u the output gradient,
 * dlse_u the gradient reaching its lse directly. */
static void unit_backward(const double* q, const double* Kb, const double* Vb, int64_t t0,
                          int64_t t1, int64_t d, double scale, const double* p,
                          const double* do_u, double dlse_u, double* dp, double* dq,
                          double* dKb, double* dVb) {
  double pdp = 0.0;
  for (int64_t j = t0; j < t1; ++j) {
    baxpy(p[j - t0], do_u, dVb + j * d, d);
    dp[j - t0] = bdot(do_u, Vb + j * d, d);
    pdp += p[j - t0] * dp[j - t0];
  }
  for (int64_t j = t0; j < t1; ++j) {
    const double dx = p[j - t0] * (dp[j - t0] - pdp) + p[j - t0] * dlse_u;
    baxpy(scale * dx, Kb + j * d, dq, d);
    baxpy(scale * dx, q, dKb + j * d, d);
  }
}

/* All queries of one (b, g): the only writer of that pair's dK, dV, dklm, dblm and of its
 * heads' dq, dqc rows. */
static int run_pair(bwd_ctx* cx, int64_t bg) {
  const hils_oracle_problem* pr = cx->pr;
  const int64_t d = pr->d, Nq = pr->N_q, Nkv = pr->N_kv, S = pr->S, Kt = pr->K_top;
  const int64_t G = pr->Hq / pr->Hkv, C = Nkv / S;
  const int64_t b = bg / pr->Hkv, g = bg % pr->Hkv;
  const double scale = pr->scale > 0.0 ? pr->scale : 1.0 / sqrt((double)d);
  const double* Kb = cx->K + bg * Nkv * d;
  const double* Vb = cx->V + bg * Nkv * d;
  double* dKb = cx->dK + bg * Nkv * d;
  double* dVb = cx->dV + bg * Nkv * d;
  const double* klm = cx->klm + bg * C * d;
  const double* blm = cx->blm + bg * C;
  double* dklm = cx->dklm + bg * C * d;
  double* dblm = cx->dblm + bg * C;
  const int64_t max_unit = (S > pr->W + S ? S : pr->W + S);
  double* x = (double*)malloc((size_t)(Kt + 1) * (size_t)max_unit * sizeof(double));
  double* dp = (double*)malloc((size_t)max_unit * sizeof(double));
  double* o = (double*)malloc((size_t)(Kt + 1) * (size_t)d * sizeof(double));
  double* do_u = (double*)malloc((size_t)d * sizeof(double));
  double* score = (double*)malloc((size_t)(Kt + 1) * sizeof(double));
  double* lse = (double*)malloc((size_t)(Kt + 1) * sizeof(double));
  double* w = (double*)malloc((size_t)(Kt + 1) * sizeof(double));
  double* dscore = (double*)malloc((size_t)(Kt + 1) * sizeof(double));
  int64_t* t0 = (int64_t*)malloc((size_t)(Kt + 1) * sizeof(int64_t));
  int64_t* t1 = (int64_t*)malloc((size_t)(Kt + 1) * sizeof(int64_t));
  int64_t* chunk = (int64_t*)malloc((size_t)(Kt + 1) * sizeof(int64_t));
  int rc = HILS_ORACLE_OK;
  if (!x || !dp || !o || !do_u || !score || !lse || !w || !dscore || !t0 || !t1 || !chunk) {
    rc = HILS_ORACLE_ENOMEM;
    goto done;
  }
  for (int64_t i = 0; i < Nq; ++i) {
    const int64_t p = pr->q_pos0 + i;
    const int64_t n = hils_oracle_n_eligible(p, pr->S, pr->W);
    if (n > C) { rc = HILS_ORACLE_EINVAL; goto done; }
    /* the units: the selected chunks (as given), then the window [S n, p] (R1) */
    const int32_t* sel = cx->idx + (bg * Nq + i) * Kt;
    int64_t nu = 0;
    for (int64_t r = 0; r < Kt; ++r) {
      if (sel[r] < 0) continue;
      if (sel[r] >= n) { rc = HILS_ORACLE_EINVAL; goto done; }
      for (int64_t u = 0; u < nu; ++u)
        if (chunk[u] == sel[r]) { rc = HILS_ORACLE_EINVAL; goto done; }
      chunk[nu] = sel[r];
      t0[nu] = sel[r] * S;
      t1[nu] = sel[r] * S + S;
      ++nu;
    }
    chunk[nu] = -1;
    t0[nu] = S * n;
    t1[nu] = p + 1;
    const int64_t L = nu;   /* index of the window unit */
    for (int64_t h = g * G; h < (g + 1) * G; ++h) {
      const int64_t row = (b * pr->Hq + h) * Nq + i;
      const double* qh = cx->q + row * d;
      const double* qch = cx->qc + row * d;
      const double* dOh = cx->dO + row * d;
      const double dl = cx->dlse ? cx->dlse[row] : 0.0;
      double* dqh = cx->dq + row * d;
      double* dqch = cx->dqc + row * d;
      /* forward again: units, scores, weights */
      for (int64_t u = 0; u <= L; ++u)
        unit_forward(qh, Kb, Vb, t0[u], t1[u], d, scale, x + u * max_unit, &lse[u], o + u * d);
      for (int64_t u = 0; u < L; ++u)
        score[u] = bdot(qch, klm + chunk[u] * d, d) * scale + blm[chunk[u]];
      score[L] = lse[L];
      double m = -INFINITY;
      for (int64_t u = 0; u <= L; ++u)
        if (score[u] > m) m = score[u];
      double z = 0.0;
      for (int64_t u = 0; u <= L; ++u) z += exp(score[u] - m);
      for (int64_t u = 0; u <= L; ++u) w[u] = exp(score[u] - m) / z;
      /* step 4 in reverse */
      double wdw = 0.0;
      for (int64_t u = 0; u <= L; ++u) wdw += w[u] * bdot(dOh, o + u * d, d);
      for (int64_t u = 0; u <= L; ++u)
        dscore[u] = w[u] * (bdot(dOh, o + u * d, d) - wdw) + dl * w[u];
      /* step 1 in reverse (the chunks' scores) */
      for (int64_t u = 0; u < L; ++u) {
        baxpy(scale * dscore[u], klm + chunk[u] * d, dqch, d);
        baxpy(scale * dscore[u], qch, dklm + chunk[u] * d, d);
        dblm[chunk[u]] += dscore[u];
      }
      /* step 3 in reverse, each unit; the window's lse also carries its score's gradient */
      for (int64_t u = 0; u <= L; ++u) {
        for (int64_t k = 0; k < d; ++k) do_u[k] = w[u] * dOh[k];
        unit_backward(qh, Kb, Vb, t0[u], t1[u], d, scale, x + u * max_unit, do_u,
                      u == L ? dscore[L] : 0.0, dp, dqh, dKb, dVb);
      }
    }
  }
done:
  free(x);
  free(dp);
  free(o);
  free(do_u);
  free(score);
  free(lse);
  free(w);
  free(dscore);
  free(t0);
  free(t1);
  free(chunk);
  return rc;
}

static void* bwd_worker(void* arg) {
  bwd_ctx* cx = (bwd_ctx*)arg;
  const int64_t pairs = cx->pr->B * cx->pr->Hkv;
  for (;;) {
    long long bg = atomic_fetch_add(&cx->next, 1);
    if (bg >= pairs) break;
    int rc = run_pair(cx, bg);
    if (rc != HILS_ORACLE_OK) atomic_store(&cx->status, rc);
  }
  return NULL;
}

int hils_oracle_backward(const hils_oracle_problem* pr, const double* q, const double* qc,
                         const double* K, const double* V, const double* klm, const double* blm,
                         const int32_t* idx, const double* dO, const double* dlse, double* dq,
                         double* dqc, double* dK, double* dV, double* dklm, double* dblm,
                         int n_threads) {
  if (!pr || pr->B < 0 || pr->Hkv <= 0 || pr->Hq <= 0 || pr->Hq % pr->Hkv != 0 ||
      pr->d <= 0 || pr->S <= 0 || pr->K_top < 0 || pr->W < 1 || pr->N_q < 0 ||
      pr->q_pos0 < 0 || pr->q_pos0 + pr->N_q > pr->N_kv || !idx || !dO)
    return HILS_ORACLE_EINVAL;
  const int64_t d = pr->d, C = pr->N_kv / pr->S;
  const size_t nq = (size_t)(pr->B * pr->Hq * pr->N_q * d);
  const size_t nk = (size_t)(pr->B * pr->Hkv * pr->N_kv * d);
  memset(dq, 0, nq * sizeof(double));
  memset(dqc, 0, nq * sizeof(double));
  memset(dK, 0, nk * sizeof(double));
  memset(dV, 0, nk * sizeof(double));
  memset(dklm, 0, (size_t)(pr->B * pr->Hkv * C * d) * sizeof(double));
  memset(dblm, 0, (size_t)(pr->B * pr->Hkv * C) * sizeof(double));
  bwd_ctx cx;
  cx.pr = pr;
  cx.q = q; cx.qc = qc; cx.K = K; cx.V = V; cx.klm = klm; cx.blm = blm;
  cx.dO = dO; cx.dlse = dlse; cx.idx = idx;
  cx.dq = dq; cx.dqc = dqc; cx.dK = dK; cx.dV = dV; cx.dklm = dklm; cx.dblm = dblm;
  atomic_init(&cx.next, 0);
  atomic_init(&cx.status, HILS_ORACLE_OK);
  const int64_t pairs = pr->B * pr->Hkv;
  if (n_threads <= 0) n_threads = hils_oracle_default_threads();
  if (n_threads > pairs) n_threads = (int)(pairs > 0 ? pairs : 1);
  if (n_threads <= 1) {
    bwd_worker(&cx);
  } else {
    pthread_t* th = (pthread_t*)malloc((size_t)n_threads * sizeof(pthread_t));
    if (!th) return HILS_ORACLE_ENOMEM;
    int started = 0;
    for (; started < n_threads; ++started)
      if (pthread_create(&th[started], NULL, bwd_worker, &cx) != 0) break;
    if (started == 0) bwd_worker(&cx);
    for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
    free(th);
  }
  return atomic_load(&cx.status);
}
