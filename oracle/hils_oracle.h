/*
 * hils_oracle.h -- plain, slow, fp64 CPU definition of the HiLS attention forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke entry point and the
 * benchmark's CPU-baseline leg may load this library.  The CUDA product path shares no code,
 * header, table or constant with it, and neither side includes or links the other.
 *
 * Sources (web pages about the paper "Hierarchical Sparse Attention Done Right: Toward
 * Infinite Context Modeling", arXiv 2607.02980).  Short names used in citations below:
 *   [Reader]  paperglide.net simplified reader of the paper
 *   [Abstract] engineersofai.com paper breakdown, section "Abstract"
 *   [DevTo]   dev.to, "HiLS Attention: How Tencent Built a Sparse Attention Mechanism That
 *             Extrapolates to 4 Million Tokens"
 *   [Essay]   nestfrontier.com, "Long context just stopped being a memory problem"
 *
 * What is computed, per query token i at absolute position p, per KV head g with its G query
 * heads h (head h belongs to KV head floor(h/G), [Reader] "Implementation and Training
 * Recipes", GQA paragraph):
 *   step 1  s_{h,c} = qc_h . klm_c * scale + blm_c for every eligible distant chunk c
 *           ([Reader] "The HiLS-Attention Mechanism", surrogate-score step; Q-Cal worked
 *           example in "Implementation and Training Recipes"), and the group score
 *           sigma_c = max_h s_{h,c} ([Reader] GQA paragraph: max across the group's heads).
 *   step 2  the K_top eligible chunks with largest sigma ([Reader] "Limitations of Naive
 *           Sparse Attention": local window plus top-K distant chunks; [Essay] "The routing
 *           problem hiding inside sparse attention": score -> top K distant -> token attention).
 *   step 3  exact softmax attention of q_h inside every selected chunk and inside the local
 *           window, each unit u giving (o_u, lse_u) ([Reader] Fig. 3 caption: intra-chunk
 *           softmax; [Abstract]: each query attends independently with each retrieved chunk).
 *   step 4  fusion: w_u = softmax_u(score_u) with score = s_{h,c} for a chunk and lse_local for
 *           the window, O = sum_u w_u o_u, LSE = logsumexp_u score_u ([Reader] Fig. 3 caption:
 *           inter-chunk softmax assigns each chunk's mass; [Abstract]: outputs fused according
 *           to chunk retrieval scores; [Essay]: "hierarchical softmax").
 *
 * Readings fixed where the pages are silent or garbled (the CUDA path applies the same ones):
 *   R1  eligibility: n = floor(max(0, p - W + 1) / S) distant chunks {0..n-1}; the local window
 *       is tokens [S*n, p] (the W-token window [p-W+1, p] extended back to a chunk boundary).
 *       Every token <= p is then covered exactly once.
 *   R2  the local window is one fusion unit whose score is its exact log-sum-exp.
 *   R3  fusion weights are normalised over selected chunks plus the window (they sum to 1).
 *   R4  selection uses sigma = max over the group's heads; each head fuses with its own s_{h,c}.
 *   R5  ties in sigma go to the lower chunk index; idx is ordered by (sigma desc, c asc).
 *   R6  qc (the calibrated query) scores chunks; q scores tokens; both use `scale`
 *       (default 1/sqrt(d); [Reader] Fig. 3 omits it "for simplicity", the Q-Cal example
 *       applies it).
 *   R7  if n <= K_top every eligible chunk is selected; n == 0 leaves plain windowed attention.
 *   R8  K/V hold only ordinary tokens; klm/blm are separate, one row per completed chunk.
 *   R9  (packing) every query attends only its own selected chunks.
 *   R10 a bias of -inf is allowed (that chunk gets weight 0); NaN inputs are undefined.
 *   R11 decode: the query sits at p = N_kv - 1 and the cache already holds its token.
 *   R15 landmark construction: one landmark query per completed chunk; its logits against the
 *       chunk's keys use the same `scale` as step 1, so that the surrogate score at the
 *       expansion point equals the chunk's log-mass exactly.
 *
 * Upstream of step 1, the producer of klm/blm (landmark construction):
 *   p = softmax_j(scale * qlm_c . K_j) over the chunk's S keys; klm_c = sum_j p_j K_j;
 *   blm_c = H(p) = -sum_j p_j log p_j ([Reader] "The HiLS-Attention Mechanism": the chunk
 *   summary is the p-weighted sum of the chunk's keys and its bias the entropy of p; [Reader]
 *   "Paper Primer": the surrogate is a first-order Taylor expansion of the full-attention chunk
 *   mass, calibrated by an entropy term; [DevTo] "The Core Idea: Landmark Tokens and
 *   Hierarchical Factorization").
 *
 * Backward (hils_oracle_bwd.c): reverse-mode differentiation of steps 4, 1 and 3 above with
 * the selection held fixed (R18: the top-K passes no gradient; the landmark keys and biases
 * receive theirs through the fusion weights, [Reader] Fig. 3 caption).
 *
 * Query prologue (hils_oracle_prologue.c): Q-Cal's low-rank correction of the query from the
 * hidden state and HoPE's partial rotary encoding (R17), the producers of q_cal and q.
 *
 * Every function here is pinned by CPU tests against values the pages print, closed forms
 * and brute force (no function is "parity unpinned").
 */
#ifndef HILS_ORACLE_H
#define HILS_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  HILS_ORACLE_OK = 0,
  HILS_ORACLE_EINVAL = 1,   /* bad sizes, idx outside [0, n) or repeated, n > n_chunks */
  HILS_ORACLE_EROW = 2,     /* a K/V token the computation needs was not provided */
  HILS_ORACLE_ENOMEM = 3
};

typedef struct {
  int32_t d;         /* head dimension */
  int32_t G;         /* query heads per KV head */
  int32_t S;         /* chunk size (tokens) */
  int32_t K_top;     /* chunks selected per query */
  int32_t W;         /* local window (tokens), >= 1 */
  int64_t n_chunks;  /* rows available in klm / blm */
  double scale;      /* logit scale; <= 0 means 1/sqrt(d) */
} hils_oracle_cfg;

/* Token rows of one KV head: token j lives at base + r*d with r = j (row_map NULL) or
 * r = row_map[j]; a negative row_map entry means the caller did not provide that token. */
typedef struct {
  const double* base;
  const int64_t* row_map;
  int64_t n_tokens;
} hils_oracle_rows;

/* One (query token, KV head) problem: all G heads of the group.  Head h of an input or output
 * array starts at ptr + h*stride (strides in doubles / int32s).  Outputs may be NULL. */
typedef struct {
  int64_t pos;                 /* absolute position p of the query token */
  const double* q;  int64_t q_hs;   /* [G][d] token queries */
  const double* qc; int64_t qc_hs;  /* [G][d] calibrated queries */
  const double* klm;           /* [n_chunks][d] landmark keys of this KV head */
  const double* blm;           /* [n_chunks] landmark biases */
  hils_oracle_rows K, V;
  const int32_t* idx_in;       /* NULL: select; else [K_top] forced chunk ids, -1 = empty */
  int32_t* idx_out;            /* [K_top] (sigma desc, c asc), -1 padded */
  double* sigma_out;           /* [K_top] group score of each selected chunk, -inf padded */
  double* gap_out;             /* [1] sigma_(K) - sigma_(K+1); +inf when n <= K_top */
  double* s_sel_out;  int64_t s_sel_hs;    /* [G][K_top] per-head score of each selected chunk */
  double* out;        int64_t out_hs;      /* [G][d] fused output */
  double* lse_out;    int64_t lse_hs;      /* [G] logsumexp of the fusion scores */
  double* unit_o_out; int64_t unit_o_hs;   /* [G][K_top+1][d]; slot K_top = local window */
  double* unit_lse_out; int64_t unit_lse_hs; /* [G][K_top+1] */
  int32_t status;              /* written by the oracle */
} hils_oracle_job;

/* Runs every job (independently; threads over jobs).  n_threads <= 0: one per usable core.
 * Returns the first non-zero job status, else HILS_ORACLE_OK. */
int hils_oracle_run(const hils_oracle_cfg* cfg, int64_t n_jobs, hils_oracle_job* jobs,
                    int n_threads);

/* Whole problem over contiguous row-major arrays:
 *   q, qc, out [B,Hq,N_q,d]; K, V [B,Hkv,N_kv,d]; klm [B,Hkv,C,d] and blm [B,Hkv,C] with
 *   C = floor(N_kv/S); idx, sigma [B,Hkv,N_q,K_top]; gap [B,Hkv,N_q]; s_sel [B,Hq,N_q,K_top];
 *   lse [B,Hq,N_q]; unit_o [B,Hq,N_q,K_top+1,d]; unit_lse [B,Hq,N_q,K_top+1].
 * Query i sits at position q_pos0 + i. */
typedef struct {
  int64_t B, Hq, Hkv, N_q, N_kv, d, q_pos0;
  int32_t S, K_top, W;
  double scale;
} hils_oracle_problem;

int hils_oracle_forward(const hils_oracle_problem* pr, const double* q, const double* qc,
                        const double* K, const double* V, const double* klm, const double* blm,
                        const int32_t* idx_in, int32_t* idx_out, double* sigma_out,
                        double* gap_out, double* s_sel_out, double* out, double* lse_out,
                        double* unit_o_out, double* unit_lse_out, int n_threads);

/* Landmark construction (R15): for every (b, g) and completed chunk c < C = floor(N_kv / S),
 *   x_j = scale * qlm[b,g,c] . K[b,g,c*S+j] (j < S), p = softmax(x),
 *   klm[b,g,c] = sum_j p_j K[b,g,c*S+j],  blm[b,g,c] = -sum_{j: p_j > 0} p_j log p_j.
 * qlm, klm [B,Hkv,C,d]; K [B,Hkv,N_kv,d]; blm [B,Hkv,C].  scale <= 0 means 1/sqrt(d).  The
 * tokens of a partial last chunk get no landmark (R8). */
int hils_oracle_landmarks(int64_t B, int64_t Hkv, int64_t N_kv, int64_t d, int32_t S,
                          double scale, const double* qlm, const double* K, double* klm,
                          double* blm);

/* Backward pass (hils_oracle_bwd.c): the gradient of L = sum dO . out + sum dlse . lse with
 * respect to q, qc, K, V, klm and blm, the selection idx [B,Hkv,N_q,K_top] (-1 padded, as
 * idx_in) held fixed.  dO [B,Hq,N_q,d]; dlse [B,Hq,N_q] or NULL (zero); dq, dqc like q; dK, dV
 * like K; dklm, dblm like klm, blm (all overwritten).  Threads over (b, g) pairs. */
int hils_oracle_backward(const hils_oracle_problem* pr, const double* q, const double* qc,
                         const double* K, const double* V, const double* klm, const double* blm,
                         const int32_t* idx, const double* dO, const double* dlse, double* dq,
                         double* dqc, double* dK, double* dV, double* dklm, double* dblm,
                         int n_threads);

/* Query prologue (hils_oracle_prologue.c), reading R17.  HoPE: pair (m, m + d/2), m < d/2,
 * turns by pos * base^(-2m/d) iff its period 2 pi base^(2m/d) <= train_len.
 * hils_oracle_hope_rotate: x, out [B, H, N, d]; token n at position pos0 + n.
 * hils_oracle_qcal_hope: q [B,Hq,N_q,d], hidden [B,N_q,d_model], W_down [Hq,r,d_model],
 * W_up [Hq,d,r]; q_out = HoPE(q), qc_out = HoPE(q + W_up (W_down hidden)) at position
 * pos0 + i. */
int hils_oracle_hope_rotates(int64_t m, int64_t d, double base, double train_len);
int hils_oracle_hope_rotate(int64_t B, int64_t H, int64_t N, int64_t d, int64_t pos0,
                            double base, double train_len, const double* x, double* out);
int hils_oracle_qcal_hope(int64_t B, int64_t Hq, int64_t N_q, int64_t d, int64_t d_model,
                          int64_t r, int64_t pos0, double base, double train_len,
                          const double* q, const double* hidden, const double* W_down,
                          const double* W_up, double* q_out, double* qc_out);

/* Rule R1: number of eligible distant chunks of the query at position pos. */
int64_t hils_oracle_n_eligible(int64_t pos, int32_t S, int32_t W);

/* Threads the oracle uses when asked for n_threads <= 0. */
int hils_oracle_default_threads(void);

#ifdef __cplusplus
}
#endif
#endif
