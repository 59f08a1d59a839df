/*
 * hils.h -- C ABI of the B200 (sm_100a) HiLS attention forward pass.
 *
 * HiLS = Hierarchical Landmark Sparse attention, from the paper "Hierarchical Sparse Attention
 * Done Right: Toward Infinite Context Modeling" (arXiv 2607.02980).  Citations name the page
 * and its section or figure:
 *   [Reader]   paperglide.net simplified reader of the paper
 *   [Abstract] engineersofai.com paper breakdown, "Abstract"
 *   [Essay]    nestfrontier.com, "Long context just stopped being a memory problem"
 *
 * Notation.  B batch; Hq query heads; Hkv KV heads; G = Hq/Hkv; query head h reads KV head
 * floor(h/G) ([Reader] "Implementation and Training Recipes", GQA paragraph: heads sharing a KV
 * head).  d head dim; S chunk size; C = floor(N_kv/S) completed chunks, each with one landmark
 * key k_lm[c] and bias b_lm[c]; K = K_top; W local window.  Query i sits at position
 * p = q_pos0 + i.  Eligible distant chunks: n = floor(max(0, p-W+1)/S), chunks 0..n-1; the
 * local window is tokens [S*n, p] (covers every token <= p exactly once with the chunks).
 *
 * Layouts (row-major, contiguous, base pointers 16-byte aligned, all device memory):
 *   q, q_cal, out       [B, Hq,  N_q,  d]   dtype
 *   K, V                [B, Hkv, N_kv, d]   dtype
 *   k_lm                [B, Hkv, C,    d]   dtype
 *   b_lm                [B, Hkv, C]         fp32
 *   idx                 [B, Hkv, N_q, K]    int32, ordered (sigma desc, c asc), -1 padded
 *   s_sel               [B, Hq,  N_q, K]    fp32 per-head score of each selected chunk
 *                                           (-inf where idx is -1)
 *   unit_o              [B, Hq,  N_q, K+1, d] fp32; slot k < K = chunk idx[k], slot K = window
 *   unit_lse, lse       [B, Hq,  N_q, K+1] / [B, Hq, N_q] fp32
 *
 * Ownership and errors.  The caller owns every buffer, including the workspace; the library
 * allocates no device memory and keeps no state between calls.  Arguments are checked on the
 * host before anything is launched: a bad argument returns an error with nothing written.
 * Otherwise the call is asynchronous on `stream` and returns HILS_ERR_CUDA if a launch fails.
 * Kernels that wait on on-chip barriers give up after a bounded number of polls and record
 * HILS_ERR_TIMEOUT in the workspace's status word (read it with hils_device_status after the
 * stream is synchronised).  No exception crosses this interface.
 *
 * Supported: sm_100a device; dtype fp32 (CUDA-core FFMA, no TF32) or bf16 (fp32 accumulate);
 * 4 <= d <= 128 with d % 4 == 0; 1 <= S <= 4096; 0 <= K <= 32; W >= 1; 1 <= G <= 16;
 * q_pos0 + N_q <= N_kv; B or N_q may be 0 (nothing is launched).  Anything else returns HILS_ERR_UNSUPPORTED or
 * HILS_ERR_INVALID_ARG; there is no fallback path.
 */
#ifndef HILS_H
#define HILS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* hils_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  HILS_OK = 0,
  HILS_ERR_INVALID_ARG = 1,  /* null / misaligned pointer, inconsistent sizes */
  HILS_ERR_UNSUPPORTED = 2,  /* valid but outside the supported set above */
  HILS_ERR_WORKSPACE = 3,    /* workspace missing or smaller than hils_workspace_size() */
  HILS_ERR_CUDA = 4,         /* a CUDA call or kernel launch failed */
  HILS_ERR_DEVICE_CHECK = 5, /* a kernel's own bounds check fired (status word) */
  HILS_ERR_TIMEOUT = 6       /* a bounded on-chip wait gave up (status word) */
} hils_status;

typedef enum { HILS_F32 = 0, HILS_BF16 = 1 } hils_dtype;

typedef struct {
  int64_t B, Hq, Hkv;
  int64_t N_q, N_kv, d;
  int64_t q_pos0;   /* position of query 0: prefill 0 (N_q == N_kv); decode N_kv - 1 (N_q == 1) */
  int32_t S, K_top, W;
  int32_t dtype;    /* hils_dtype of q, q_cal, K, V, k_lm and out */
  float scale;      /* logit scale for chunk and token scores; <= 0 means 1/sqrt(d) */
} hils_params;

/* Bytes of scratch the calls below need for these parameters (>= 256). */
size_t hils_workspace_size(const hils_params* p);

/*
 * The whole forward pass, steps 1-4 ([Essay] "The routing problem hiding inside sparse
 * attention": score the chunk summaries, keep the top K distant chunks, token attention inside
 * them and the local window, hierarchical softmax; [Reader] Fig. 3 caption):
 *   out[b,h,i]  = sum_u w_u o_u, w = softmax_u(score_u), score = s_{h,c} for each selected chunk
 *                 and the window's exact log-sum-exp for the window ([Abstract]: per-chunk
 *                 outputs fused according to chunk retrieval scores);
 *   lse_out     = logsumexp_u score_u (nullable);
 *   topk_idx_out = the selection (nullable).
 * q scores tokens, q_cal scores chunks ([Reader] "Implementation and Training Recipes", Q-Cal).
 */
hils_status hils_forward(const hils_params* p, const void* q, const void* q_cal, const void* K,
                         const void* V, const void* k_lm, const float* b_lm, void* out,
                         float* lse_out, int32_t* topk_idx_out, void* workspace,
                         size_t workspace_bytes, hils_stream_t stream);

/*
 * hils_forward with phase timing: `events` holds n_events cudaEvent_t handles created by the
 * caller; events[0] is recorded on `stream` before the first kernel and events[k] right after
 * the k-th kernel (k >= 1), as far as n_events reaches.  Everything else is hils_forward.
 */
hils_status hils_forward_timed(const hils_params* p, const void* q, const void* q_cal,
                               const void* K, const void* V, const void* k_lm, const float* b_lm,
                               void* out, float* lse_out, int32_t* topk_idx_out, void* workspace,
                               size_t workspace_bytes, hils_stream_t stream, void* const* events,
                               int n_events);

/* Number of kernels hils_forward launches for these parameters (-1 if they are invalid); the
 * first max_names of their names are stored in names (static strings; names may be NULL). */
int hils_forward_phases(const hils_params* p, const char** names, int max_names);

/*
 * Steps 1-2: s_{h,i,c} = q_cal[b,h,i] . k_lm[b,g,c] * scale + b_lm[b,g,c] for every eligible c
 * ([Reader] "The HiLS-Attention Mechanism", surrogate score; Q-Cal worked example), group score
 * sigma = max over the G heads of KV head g ([Reader] GQA paragraph), and the K largest sigma
 * with ties to the lower chunk index ([Reader] "Limitations of Naive Sparse Attention": top-K
 * distant chunks).  Writes idx and, if non-NULL, s_sel (the per-head scores of those chunks).
 */
hils_status hils_select(const hils_params* p, const void* q_cal, const void* k_lm,
                        const float* b_lm, int32_t* idx, float* s_sel, void* workspace,
                        size_t workspace_bytes, hils_stream_t stream);

/*
 * Step 3: exact softmax attention of q[b,h,i] inside each selected chunk (idx as produced by
 * hils_select; -1 entries, and ids that are not eligible chunks of that query, give
 * unit_o = 0, unit_lse = -inf) and inside the local window
 * ([Reader] Fig. 3 caption: intra-chunk softmax; [Abstract]: each query attends independently
 * with each retrieved chunk).  Writes unit_o and unit_lse (layouts above).
 */
hils_status hils_chunk_attn(const hils_params* p, const void* q, const void* K, const void* V,
                            const int32_t* idx, float* unit_o, float* unit_lse,
                            hils_stream_t stream);

/*
 * Step 4: w_u = softmax over {s_sel[k] : idx[k] >= 0} and the window's unit_lse[K];
 * out = sum_u w_u unit_o[u]; lse_out = logsumexp (nullable).  ([Reader] Fig. 3 caption:
 * inter-chunk softmax; [Abstract]: fusion by chunk retrieval scores.)
 */
hils_status hils_fuse(const hils_params* p, const float* s_sel, const float* unit_o,
                      const float* unit_lse, void* out, float* lse_out, hils_stream_t stream);

/*
 * Landmark construction, upstream of step 1 (the producer of k_lm and b_lm): for every (b, g)
 * and completed chunk c (tokens c*S .. c*S+S-1; a partial last chunk has none),
 *   p = softmax_j(scale * q_lm[b,g,c] . K[b,g,c*S+j]),
 *   k_lm[b,g,c] = sum_j p_j K[b,g,c*S+j],   b_lm[b,g,c] = -sum_j p_j ln p_j
 * ([Reader] "The HiLS-Attention Mechanism": the chunk summary is the landmark query's
 * attention-weighted sum of the chunk's keys and its bias the entropy of those weights; with the
 * same scale as step 1 the surrogate score at q_lm equals the chunk's exact log-mass).
 * q_lm: [B, Hkv, C, d] dtype, one landmark query per completed chunk and KV head; K as for
 * hils_forward; k_lm: [B, Hkv, C, d] dtype and b_lm: [B, Hkv, C] fp32 are written.  Reads only
 * B, Hkv, N_kv, d, S, dtype and scale of `p` (the other fields must still be valid); d must be
 * 16, 32, 64 or 128.  Asynchronous on `stream`; allocates nothing and needs no workspace.
 */
hils_status hils_landmarks(const hils_params* p, const void* q_lm, const void* K, void* k_lm,
                           float* b_lm, hils_stream_t stream);

/*
 * One decode step over a KV cache that grows by one token per call ([Reader] Fig. 6 caption:
 * decode latency per token, timed with CUDA graphs; [Essay] "What the numbers actually say": the
 * cache is paged by chunk, a chunk's landmark exists once the chunk is complete).  `p` describes
 * the cache: N_kv is its capacity (rows per (b, g) plane of K, V; C = N_kv / S landmark rows per
 * plane of k_lm, b_lm), q_pos0 = pos is the new token's position (pos < N_kv) and N_q = 1.  The
 * call
 *   1. appends the new token: K[b,g,pos] = k_new[b,g], V[b,g,pos] = v_new[b,g];
 *   2. if the token completes chunk c = pos / S (that is, (pos + 1) % S == 0), builds that
 *      chunk's landmark k_lm[b,g,c], b_lm[b,g,c] from its landmark query q_lm_new[b,g] as
 *      hils_landmarks does (q_lm_new may be NULL otherwise);
 *   3. runs hils_forward for the query at pos (q, q_cal [B, Hq, 1, d]; out, lse_out,
 *      topk_idx_out as there).  Only tokens 0..pos and landmarks of chunks before the query's
 *      window are read, so the cache beyond pos may hold anything.
 * k_new, v_new, q_lm_new: [B, Hkv, d] in dtype.  Workspace: hils_workspace_size(p).  Supported:
 * the decode shapes of hils_forward (d = 64 or 128).  Asynchronous on `stream`; the launches are
 * fixed for given arguments, so a step can be captured in a CUDA graph and replayed.
 */
hils_status hils_decode_step(const hils_params* p, const void* q, const void* q_cal,
                             const void* k_new, const void* v_new, const void* q_lm_new,
                             void* K, void* V, void* k_lm, float* b_lm, void* out,
                             float* lse_out, int32_t* topk_idx_out, void* workspace,
                             size_t workspace_bytes, hils_stream_t stream);

/*
 * Query prologue: Q-Cal and HoPE, the producers of step 1's calibrated query and step 3's token
 * query.  Q-Cal ([Reader] "Implementation and Training Recipes", Q-Cal worked example and the
 * low-rank question): per query head h, dq = W_up[h] (W_down[h] hidden) with W_down[h] r x
 * d_model and W_up[h] d x r, and q_cal = q + dq.  HoPE ([Reader] same section, HoPE vs RoPE;
 * [Essay] "Hierarchical Positional Encoding"): the dimension pairs (m, m + d/2), m < d/2, whose
 * rotation period 2 pi rope_base^(2m/d) is at most train_len turn by pos rope_base^(-2m/d)
 * radians; the other pairs are left as they are (NoPE).  Queries are turned at their position,
 * keys at theirs (hils_hope_rotate), so a query's products with the keys, and with the landmark
 * keys built from them, see relative positions only along the turning pairs.
 */
typedef struct {
  int64_t d_model;    /* width of the hidden state and of W_down's rows (a multiple of 64) */
  int32_t r;          /* Q-Cal rank: 0 (no correction) or 1..64 with Hq * r a multiple of 64 */
  double rope_base;   /* > 1 */
  double train_len;   /* pairs with a longer period do not turn (<= 0: none turns) */
} hils_prologue_params;

/* Workspace of hils_qcal_hope: a 256-byte status word, then B N_q Hq r fp32 values of
 * W_down hidden. */
size_t hils_qcal_workspace_size(const hils_params* p, const hils_prologue_params* c);

/*
 * q_out = HoPE(q), q_cal_out = HoPE(q + W_up (W_down hidden)) for query i at position
 * q_pos0 + i.  Reads B, Hq, N_q, d (64 or 128), q_pos0 and dtype of `p`.  q, q_out, q_cal_out
 * [B, Hq, N_q, d] and W_up [Hq, d, r] in dtype; hidden [B, N_q, d_model] and W_down
 * [Hq, r, d_model] bf16 (the down-projection, a dense GEMM, runs on the tcgen05 tensor cores with
 * fp32 accumulation; unused when r = 0).  q_out may equal q (in place); q_cal_out must not
 * overlap q.  Workspace: hils_qcal_workspace_size bytes, status word zeroed once
 * (hils_workspace_init; read with hils_device_status).  Asynchronous on `stream`.
 */
hils_status hils_qcal_hope(const hils_params* p, const hils_prologue_params* c, const void* q,
                           const void* hidden, const void* W_down, const void* W_up,
                           void* q_out, void* q_cal_out, void* workspace,
                           size_t workspace_bytes, hils_stream_t stream);

/*
 * x_out = HoPE(x) for x [B, H, N, d] (dtype of `p`, d = 64 or 128), token n at position
 * pos0 + n: the keys' side of the encoding (turn K before hils_forward and before building
 * landmarks).  Reads only d and dtype of `p` besides the arguments; x_out may equal x.
 */
hils_status hils_hope_rotate(const hils_params* p, const hils_prologue_params* c, int64_t B,
                             int64_t H, int64_t N, int64_t pos0, const void* x, void* x_out,
                             hils_stream_t stream);

/*
 * Backward pass: the gradients of L = sum dout . out + sum dlse . lse (out, lse as hils_forward
 * computes them) with respect to q, q_cal, K, V, k_lm and b_lm, with the selection topk_idx held
 * fixed.  The top-K is piecewise constant in its inputs and passes no gradient; the landmark keys
 * and biases receive theirs through the fusion weights ([Reader] Fig. 3 caption: the loss
 * gradient flows back to the compressed key; "The HiLS-Attention Mechanism": the surrogate is
 * differentiable where the exact chunk mass is not).  By the chain rule through steps 4, 1 and
 * 3, per query-head row with units u (the selected chunks, then the window) and fused weights w:
 *   d score_u = w_u (dout . o_u - dout . out + dlse);  a chunk's score passes it to q_cal, k_lm
 *   and b_lm; the window's score is its own lse and passes it to the window's token logits;
 *   dV_j += a_j dout, d x_j = a_j (dout . V_j - dout . o_u) (+ a_j d score_window for window
 *   tokens), a_j = w_u exp(x_j - lse_u) the token's fused weight.
 * Inputs as for hils_forward (p, q, q_cal, K, V, k_lm, b_lm, same dtype); topk_idx [B, Hkv, N_q,
 * K_top] int32 the forward's selection (ids outside a query's eligible chunks count as empty
 * slots and a repeated id is attended once; the forward never writes either); dout [B, Hq, N_q,
 * d] in dtype; dlse [B, Hq, N_q] fp32 or NULL (zero).  Outputs, all fp32 and every element
 * written: dq, dq_cal [B, Hq, N_q, d]; dK, dV [B, Hkv, N_kv, d]; dk_lm [B, Hkv, C, d]; db_lm
 * [B, Hkv, C].  Workspace: hils_backward_workspace_size(p) bytes, 16-byte aligned (per-row
 * fusion terms, 4 (2 K_top + 3) bytes per query-head, and a chunk -> selecting-query index,
 * 4 K_top bytes per query and KV head).  Supported: d = 64 or 128, S in {16, 32, 64, 128},
 * G = Hq / Hkv dividing 64, K_top <= 32; else HILS_ERR_UNSUPPORTED.  Every gradient is a sum
 * formed in one thread's registers (no atomics), but the order in which the rows that selected a
 * chunk reach the K, V, k_lm and b_lm gradients follows the index build and may differ between
 * runs, so those four can differ between runs in the last bits.  Asynchronous on `stream`.
 */
size_t hils_backward_workspace_size(const hils_params* p);
hils_status hils_backward(const hils_params* p, const void* q, const void* q_cal, const void* K,
                          const void* V, const void* k_lm, const float* b_lm,
                          const int32_t* topk_idx, const void* dout, const float* dlse,
                          float* dq, float* dq_cal, float* dK, float* dV, float* dk_lm,
                          float* db_lm, void* workspace, size_t workspace_bytes,
                          hils_stream_t stream);

/*
 * hils_select without a caller-provided workspace.  The paper has no counterpart: this entry
 * point exists for callers that cannot allocate device memory or pass a scratch buffer, e.g. a
 * plugin host that hands a kernel only its input and output tensors, or a serving loop whose
 * device memory is planned up front so that cudaMalloc (which may synchronise the device) is
 * not allowed on the request path.  It computes exactly what hils_select computes.
 *
 * Scratch: a fixed array of hils_select_noalloc_max_bytes() bytes (8 MiB) inside the library,
 * one per device, held by every device that loads the library until the process exits.  The
 * first call on a device (this one or hils_select_noalloc_status) looks up that device's copy
 * (cudaGetSymbolAddress, with the device current), keeps the address for the life of the
 * process and zeroes the array's status word on `stream`; make that first call before any
 * stream capture.  The kept address does not survive cudaDeviceReset: resetting a device after
 * the first call is not supported.  Calls whose scratch would exceed the maximum (decode shapes
 * with B*Hkv*N_q * ceil(n/512) * K * 8 bytes beyond ~8 MiB) return HILS_ERR_WORKSPACE before
 * launching anything.  Every call on a device shares the same scratch, so calls that overlap on
 * the GPU (different streams, or concurrent host threads) race and give undefined results:
 * order them on one stream.  Kernels record a failed bounded wait in the array's status word,
 * which keeps the first failure until hils_select_noalloc_status reads and clears it.
 * Allocates nothing.
 */
hils_status hils_select_noalloc(const hils_params* p, const void* q_cal, const void* k_lm,
                                const float* b_lm, int32_t* idx, float* s_sel,
                                hils_stream_t stream);

/* Size in bytes of the fixed scratch array hils_select_noalloc uses. */
size_t hils_select_noalloc_max_bytes(void);

/* Copies this device's hils_select_noalloc status word to *status (HILS_OK, or the first
 * failure a kernel recorded since the word was last read) and clears it.  Synchronous on
 * `stream`; order it after the calls it reports on.  The paper has no counterpart. */
hils_status hils_select_noalloc_status(hils_stream_t stream, int32_t* status);

/* Zeroes the workspace's status word; call once on a newly allocated workspace. */
hils_status hils_workspace_init(void* workspace, size_t workspace_bytes, hils_stream_t stream);

/* Copies the workspace's status word to *status (HILS_OK or the first failure a kernel
 * recorded) and clears it.  Synchronous on `stream`. */
hils_status hils_device_status(void* workspace, hils_stream_t stream, int32_t* status);

/*
 * Check of the bounded on-chip waits (the paper has no counterpart).  Every tensor-core kernel
 * waits on mbarriers for its TMA copies and MMAs; each wait gives up after a bounded number of
 * polls, records HILS_ERR_TIMEOUT in the workspace's status word and lets the kernel return, so
 * a wait that can never finish cannot hang the GPU.  This launches one CTA that performs such a
 * wait with a limit of `polls` polls: with `complete` nonzero the barrier phase is completed
 * first (the wait succeeds, nothing is recorded); with `complete` zero nothing ever arrives and
 * the wait must give up.  Read the outcome with hils_device_status.  Asynchronous on `stream`.
 */
hils_status hils_wait_check(uint32_t polls, int complete, void* workspace,
                            size_t workspace_bytes, hils_stream_t stream);

const char* hils_status_string(hils_status s);

/* Library build identification: "hils-b200 <git-describe> sm_100a". */
const char* hils_version(void);

#ifdef __cplusplus
}
#endif
#endif
