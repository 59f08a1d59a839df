// Launchers of the HiLS kernels (internal to the library; the public interface is hils.h).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace hils {

struct Dims;

cudaError_t launch_select_rows(const Dims& D, bool bf16, const void* qc, const void* klm,
                               const float* blm, int32_t* idx, float* s_sel, cudaStream_t st);

cudaError_t launch_select_scores(const Dims& D, bool bf16, const void* qc, const void* klm,
                                 const float* blm, const int32_t* idx, float* s_sel,
                                 cudaStream_t st);

bool score_tc_supported(const Dims& D, bool bf16);
// s_out (nullable): the winners' scores sigma, laid out like idx (-inf where idx is -1)
cudaError_t launch_score_topk_tc(const Dims& D, const void* qc, const void* klm,
                                 const float* blm, int32_t* idx, float* s_out, int32_t* status,
                                 cudaStream_t st);

// landmark-major variant (landmark rows as the MMA's M, all G heads of a block as its N);
// s_head (nullable): every head's score of each selected chunk, [B, Hq, N_q, K]
bool score_t_tc_supported(const Dims& D, bool bf16);
cudaError_t launch_score_topk_t_tc(const Dims& D, const void* qc, const void* klm,
                                   const float* blm, int32_t* idx, float* s_out,
                                   float* s_head, int32_t* status, cudaStream_t st);

bool attn_tc_supported(const Dims& D, bool bf16);
// d = 128 with K <= 16 where two attention CTAs fit one SM: the kernel then takes every head's
// scores of the selected chunks from s_sig instead of scoring them itself
bool attn_tc_two_cta(const Dims& D);
// whether the attention kernel for D reads the per-head selected-chunk scores from s_sig
bool attn_tc_external_scores(const Dims& D);
// s_sig: per-head scores of the selected chunks [B, Hq, N_q, K], required when
// attn_tc_external_scores(D) (with G == 1 the scoring kernel's sigma of the winners); otherwise
// the kernel scores the selected chunks per head itself
cudaError_t launch_attn_tc(const Dims& D, const void* q, const void* qc, const void* K,
                           const void* V, const int32_t* idx, const float* s_sig,
                           const void* klm, const float* blm, void* out, float* lse,
                           int32_t* status, cudaStream_t st);

size_t split_smem_bytes(int cps);
cudaError_t launch_select_split(const Dims& D, bool bf16, int cps, int n_split, const void* qc,
                                const void* klm, const float* blm, float* part_v,
                                int32_t* part_c, cudaStream_t st);
cudaError_t launch_select_stream(const Dims& D, bool bf16, int cps, int n_split,
                                 int64_t n_stride, const void* qc, const void* klm,
                                 const float* blm, float* sigma, int32_t* status,
                                 cudaStream_t st);
bool stream_tc_supported(const Dims& D, bool bf16);
// gmax (nullable): [rows][g_stride] maxima of 32 consecutive sigmas, g_stride >= 4 per
// 128-landmark tile of the longest row.
cudaError_t launch_select_stream_tc(const Dims& D, const void* qc, const void* klm,
                                    const float* blm, float* sigma, int64_t n_stride,
                                    int32_t* status, cudaStream_t st, float* gmax = nullptr,
                                    int64_t g_stride = 0);
bool units_tc_supported(const Dims& D, bool bf16);
cudaError_t launch_attn_units_tc(const Dims& D, int n_pieces, const void* q, const void* K,
                                 const void* V, const int32_t* idx, float* part_o,
                                 float* part_lse, int32_t* status, cudaStream_t st);
cudaError_t launch_select_topk_row(const Dims& D, bool bf16, int64_t n_stride,
                                   const float* sigma, const void* qc, const void* klm,
                                   const float* blm, int32_t* idx, float* s_sel, cudaStream_t st,
                                   const float* gmax = nullptr, int64_t g_stride = 0);
cudaError_t launch_select_merge(const Dims& D, bool bf16, int n_split, const float* part_v,
                                const int32_t* part_c, const void* qc, const void* klm,
                                const float* blm, int32_t* idx, float* s_sel, cudaStream_t st);

cudaError_t launch_attn_rows(const Dims& D, bool bf16, const void* q, const void* K,
                             const void* V, const int32_t* idx, const float* s_sel, void* out,
                             float* lse, float* unit_o, float* unit_lse, cudaStream_t st);

cudaError_t launch_attn_units(const Dims& D, bool bf16, int n_pieces, const void* q,
                              const void* K, const void* V, const int32_t* idx, float* part_o,
                              float* part_lse, int32_t* status, cudaStream_t st);

cudaError_t launch_fuse_units(const Dims& D, bool bf16, int n_pieces, const float* s_sel,
                              const float* part_o, const float* part_lse, void* out, float* lse,
                              cudaStream_t st);

// Landmark construction: k_lm = softmax(scale q_lm . K_chunk) K_chunk, b_lm = its entropy, for
// chunks c0 .. c0+nc-1 of every (b, g); chunk c0 + cc's landmark query is row bg*qlm_rows + cc.
cudaError_t launch_landmarks(const Dims& D, bool bf16, int64_t c0, int64_t nc,
                             int64_t qlm_rows, const void* qlm, const void* K, void* klm,
                             float* blm, cudaStream_t st);
// K[b, g, pos] = k_new[b, g], V[b, g, pos] = v_new[b, g] (row stride of the cache: D.N_kv).
cudaError_t launch_append_kv(const Dims& D, bool bf16, int64_t pos, const void* k_new,
                             const void* v_new, void* K, void* V, cudaStream_t st);

// Backward pass (csrc/bwd.cu).  Inputs in the forward's dtype except b_lm / dlse (fp32); every
// gradient fp32, overwritten.
struct BwdArgs {
  const void *q, *q_cal, *K, *V, *k_lm;
  const float* b_lm;
  const int32_t* idx;
  const void* dout;
  const float* dlse;   // nullable
  float *dq, *dq_cal, *dK, *dV, *dk_lm, *db_lm;
};
struct BwdWs {
  float *lam, *gam, *ds;              // per (row, unit): lambda * log2(e), gamma; dscore
  int32_t *inv_cnt, *inv_cur, *inv_off, *inv_list;   // chunk -> selecting (query, slot)
};
bool backward_supported(const Dims& D);
// Bytes of the backward's workspace; with base != nullptr also carves it into *w.
size_t backward_ws_layout(const Dims& D, BwdWs* w, char* base);
cudaError_t launch_backward(const Dims& D, bool bf16, const BwdArgs& a, const BwdWs& w,
                            cudaStream_t st);

// Query prologue (csrc/prologue.cu).  u [M, N] fp32 = hidden [M, d_model] x W_down [N,
// d_model]^T (bf16 operands, tcgen05); q_cal = R(q + W_up u), q = R(q) per head; R = HoPE.
bool qdown_supported(int64_t N, int64_t d_model);
cudaError_t launch_qdown(int64_t M, int64_t N, int64_t d_model, const void* hidden,
                         const void* W_down, float* u, int32_t* status, cudaStream_t st);
cudaError_t launch_qcal_hope(int64_t B, int64_t Hq, int64_t N_q, int64_t d, int64_t q_pos0,
                             int r, double base, double train_len, bool bf16, const void* q,
                             const float* u, const void* W_up, void* q_out, void* qc_out,
                             cudaStream_t st);
cudaError_t launch_hope_rotate(int64_t BH, int64_t N, int64_t d, int64_t pos0, double base,
                               double train_len, bool bf16, const void* x, void* out,
                               cudaStream_t st);

// One CTA waits on an mbarrier phase for at most `polls` polls (completed first if `complete`);
// a wait that gives up records HILS_ERR_TIMEOUT in *status.
cudaError_t launch_wait_check(uint32_t polls, int complete, int32_t* status, cudaStream_t st);

}  // namespace hils
