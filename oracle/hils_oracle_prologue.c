/*
 * hils_oracle_prologue.c -- fp64 CPU oracle of the query prologue (test infrastructure):
 * Q-Cal and HoPE, the two producers of step 1's calibrated query and step 3's token query.
 *
 * Q-Cal ([Reader] "Implementation and Training Recipes", Q-Cal worked example and the low-rank
 * question): per query head h a low-rank correction of the token query from the token's hidden
 * state, dq = W_up[h] (W_down[h] hidden), W_down[h] of shape r x d_model and W_up[h] of shape
 * d x r; the calibrated query is q + dq.
 *
 * HoPE ([Reader] same section, "How does HoPE differ from the standard RoPE"; [Essay]
 * "Hierarchical Positional Encoding"): rotary position encoding on the dimension pairs whose
 * rotation period fits the training length, no rotation (NoPE) on the others.  Readings fixed
 * here (R17): the pairs are (m, m + d/2) for m < d/2 with angular frequency
 * theta_m = base^(-2m/d) and period 2 pi / theta_m; a pair rotates iff its period is at most
 * train_len; a token at position p turns pair m by the angle p theta_m:
 *   x'_m = x_m cos(a) - x_{m+d/2} sin(a),  x'_{m+d/2} = x_m sin(a) + x_{m+d/2} cos(a).
 * The token query and the calibrated query are both turned at the query's position (the keys,
 * and through them the landmark keys, at their own positions), so that their products with the
 * keys depend on the relative position only along the rotating pairs.
 */
#define _GNU_SOURCE
#include <math.h>
#include <stdlib.h>

#include "hils_oracle.h"

/* Whether pair m of a d-dim head rotates under HoPE (R17). */
int hils_oracle_hope_rotates(int64_t m, int64_t d, double base, double train_len) {
  const double theta = pow(base, -2.0 * (double)m / (double)d);
  return 2.0 * M_PI / theta <= train_len;
}

static void rotate(double* x, int64_t d, int64_t pos, double base, double train_len) {
  const int64_t half = d / 2;
  for (int64_t m = 0; m < half; ++m) {
    if (!hils_oracle_hope_rotates(m, d, base, train_len)) continue;
    const double a = (double)pos * pow(base, -2.0 * (double)m / (double)d);
    const double c = cos(a), s = sin(a);
    const double x0 = x[m], x1 = x[m + half];
    x[m] = x0 * c - x1 * s;
    x[m + half] = x0 * s + x1 * c;
  }
}

int hils_oracle_hope_rotate(int64_t B, int64_t H, int64_t N, int64_t d, int64_t pos0,
                            double base, double train_len, const double* x, double* out) {
  if (B < 0 || H < 0 || N < 0 || d <= 0 || d % 2 != 0 || pos0 < 0 || !(base > 1.0))
    return HILS_ORACLE_EINVAL;
  for (int64_t bh = 0; bh < B * H; ++bh)
    for (int64_t n = 0; n < N; ++n) {
      const double* src = x + (bh * N + n) * d;
      double* dst = out + (bh * N + n) * d;
      for (int64_t e = 0; e < d; ++e) dst[e] = src[e];
      rotate(dst, d, pos0 + n, base, train_len);
    }
  return HILS_ORACLE_OK;
}

int hils_oracle_qcal_hope(int64_t B, int64_t Hq, int64_t N_q, int64_t d, int64_t d_model,
                          int64_t r, int64_t pos0, double base, double train_len,
                          const double* q, const double* hidden, const double* W_down,
                          const double* W_up, double* q_out, double* qc_out) {
  if (B < 0 || Hq < 0 || N_q < 0 || d <= 0 || d % 2 != 0 || d_model <= 0 || r < 0 ||
      pos0 < 0 || !(base > 1.0))
    return HILS_ORACLE_EINVAL;
  double* u = (double*)malloc((size_t)(r > 0 ? r : 1) * sizeof(double));
  if (!u) return HILS_ORACLE_ENOMEM;
  for (int64_t b = 0; b < B; ++b)
    for (int64_t h = 0; h < Hq; ++h)
      for (int64_t i = 0; i < N_q; ++i) {
        const int64_t row = (b * Hq + h) * N_q + i;
        const double* hid = hidden + (b * N_q + i) * d_model;
        /* the low-rank correction: u = W_down[h] hid, dq = W_up[h] u */
        for (int64_t j = 0; j < r; ++j) {
          const double* wd = W_down + (h * r + j) * d_model;
          double acc = 0.0;
          for (int64_t k = 0; k < d_model; ++k) acc += wd[k] * hid[k];
          u[j] = acc;
        }
        double* qo = q_out + row * d;
        double* qc = qc_out + row * d;
        for (int64_t e = 0; e < d; ++e) {
          const double* wu = W_up + (h * d + e) * r;
          double dq = 0.0;
          for (int64_t j = 0; j < r; ++j) dq += wu[j] * u[j];
          qo[e] = q[row * d + e];
          qc[e] = q[row * d + e] + dq;
        }
        /* both turned at the query's position */
        rotate(qo, d, pos0 + i, base, train_len);
        rotate(qc, d, pos0 + i, base, train_len);
      }
  free(u);
  return HILS_ORACLE_OK;
}
