// Host side of the C ABI declared in include/hils.h: argument checks, workspace layout and the
// choice of kernels.  Every step of the computation runs in the kernels; nothing here touches
// tensor data.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "hils.h"
#include "kernels.h"

#ifndef HILS_GIT_DESCRIBE
#define HILS_GIT_DESCRIBE "unknown"
#endif

namespace hils {
namespace {

constexpr size_t kAlign = 256;
constexpr size_t kStatusBytes = 256;
constexpr int kChunksPerSplit = 512;
constexpr int64_t kDecodeMaxQueries = 16;
constexpr int kStreamRows = 1024;  // landmark rows per streaming CTA (a ring of bulk copies)
// decode rows from this many eligible chunks take the two-level top-K (group maxima)
constexpr int64_t kTopkGroupMinChunks = 1024;


size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Plan {
  Dims D;
  bool bf16 = false;
  bool decode = false;
  bool tc_select = false;
  bool tc_select_t = false;   // the landmark-major scoring kernel (G = 2, 4, 8)
  bool attn_ext = false;      // the tensor-core attention reads per-head scores from s_sel
  bool tc_attn = false;
  bool tc_stream = false;
  bool tc_units = false;
  int cps = 0, n_split = 0, n_pieces = 0;
  size_t off_idx = 0, off_ssel = 0, off_po = 0, off_pl = 0;
  size_t off_sig = 0;
  size_t off_gmax = 0;        // decode on the tensor-core stream: maxima of 32 sigmas per row
  int64_t n_stride = 0, g_stride = 0;
  size_t total = 0;
};

hils_status check_params(const hils_params* p) {
  if (!p) return HILS_ERR_INVALID_ARG;
  if (p->B < 0 || p->N_q < 0 || p->Hq < 1 || p->Hkv < 1 || p->N_kv < 1 || p->d < 1 ||
      p->q_pos0 < 0 || p->S < 1 || p->K_top < 0 || p->W < 1)
    return HILS_ERR_INVALID_ARG;
  if (p->Hq % p->Hkv != 0) return HILS_ERR_INVALID_ARG;
  if (p->q_pos0 + p->N_q > p->N_kv) return HILS_ERR_INVALID_ARG;
  if (p->dtype != HILS_F32 && p->dtype != HILS_BF16) return HILS_ERR_INVALID_ARG;
  if (std::isnan(p->scale) || std::isinf(p->scale)) return HILS_ERR_INVALID_ARG;
  if (p->d > kMaxD || p->d % 4 != 0) return HILS_ERR_UNSUPPORTED;
  if (p->K_top > kMaxK) return HILS_ERR_UNSUPPORTED;
  if (p->Hq / p->Hkv > 16) return HILS_ERR_UNSUPPORTED;
  if (p->S > 4096) return HILS_ERR_UNSUPPORTED;
  if (p->N_kv / p->S > (int64_t)INT32_MAX - 1) return HILS_ERR_UNSUPPORTED;
  return HILS_OK;
}

Plan make_plan(const hils_params* p) {
  Plan P;
  Dims& D = P.D;
  D.B = p->B; D.Hq = p->Hq; D.Hkv = p->Hkv; D.N_q = p->N_q; D.N_kv = p->N_kv; D.d = p->d;
  D.q_pos0 = p->q_pos0;
  D.S = p->S; D.K = p->K_top; D.W = p->W;
  D.G = (int32_t)(p->Hq / p->Hkv);
  D.C = p->N_kv / p->S;
  D.scale = p->scale > 0.f ? p->scale : (float)(1.0 / std::sqrt((double)p->d));
  P.bf16 = p->dtype == HILS_BF16;
  // decode kernels put (b, g, query) rows on grid.y (<= 65535)
  P.decode = p->N_q <= kDecodeMaxQueries && (p->d == 64 || p->d == 128) &&
             p->B * p->Hkv * p->N_q <= 65535;
  // the prefill tensor-core kernels address q/q_cal, K/V and landmark rows by 32-bit TMA
  // coordinates; beyond that the CUDA-core kernels (64-bit offsets) run
  const bool rows32 = D.B * D.Hq * D.N_q < (int64_t)INT32_MAX &&
                      D.B * D.Hkv * D.N_kv < (int64_t)INT32_MAX &&
                      D.B * D.Hkv * D.C < (int64_t)INT32_MAX;
  P.tc_select = !P.decode && rows32 && score_tc_supported(D, P.bf16);
  P.tc_attn = !P.decode && rows32 && attn_tc_supported(D, P.bf16);
  P.attn_ext = P.tc_attn && attn_tc_external_scores(D);
  // the landmark-major scoring kernel: always for eight heads; for four, on long sequences
  // (8192 chunks and more) or when its per-head scores of the winners feed the two-CTA
  // attention.  Short four-head blocks alone favour the query-major kernel, whose blocks of 128
  // queries amortise the per-block start-up better (7B-like prefill scoring: 2.29 ms against
  // 2.91 ms), but that kernel leaves the per-head scores to a separate launch (2.5 ms there).
  P.tc_select_t = P.tc_select && score_t_tc_supported(D, P.bf16) &&
                  (D.G == 8 || D.C >= 8192 || (P.tc_attn && attn_tc_two_cta(D)));
  P.tc_stream = P.decode && stream_tc_supported(D, P.bf16);
  P.tc_units = P.decode && units_tc_supported(D, P.bf16);

  const size_t sel_rows = (size_t)(p->B * p->Hkv * p->N_q);
  const size_t head_rows = (size_t)(p->B * p->Hq * p->N_q);
  size_t off = kStatusBytes;
  P.off_idx = off;   off = align_up(off + sel_rows * (size_t)D.K * sizeof(int32_t));
  // per-head scores of the selected chunks: the tensor-core attention takes them from the
  // scoring kernel when a KV group has one head (sel_rows = head_rows) and otherwise scores the
  // selected chunks itself
  if (!P.tc_attn || !P.tc_select || P.attn_ext) {
    P.off_ssel = off;
    off = align_up(off + head_rows * (size_t)D.K * sizeof(float));
  }
  if (P.decode) {
    int64_t n_max = 0, win_max = 1;
    for (int64_t i = 0; i < p->N_q; ++i) {
      const int64_t pos = p->q_pos0 + i;
      const int64_t n = n_eligible(pos, D.S, D.W);
      n_max = n > n_max ? n : n_max;
      const int64_t win = pos - (int64_t)D.S * n + 1;
      win_max = win > win_max ? win : win_max;
    }
    P.cps = kChunksPerSplit;
    P.n_split = (int)((n_max + P.cps - 1) / P.cps);
    if (P.n_split < 1) P.n_split = 1;
    P.n_pieces = (int)((win_max + D.S - 1) / D.S);
    const int NU = D.K + P.n_pieces;
    P.off_po = off; off = align_up(off + head_rows * NU * (size_t)D.d * sizeof(float));
    P.off_pl = off; off = align_up(off + head_rows * NU * sizeof(float));
    P.n_stride = (n_max + 3) / 4 * 4;
    P.off_sig = off; off = align_up(off + sel_rows * (size_t)P.n_stride * sizeof(float));
    if (P.tc_stream && n_max >= kTopkGroupMinChunks) {   // four groups of 32 per 128-row tile
      P.g_stride = (P.n_stride + 127) / 128 * 4;
      P.off_gmax = off;
      off = align_up(off + sel_rows * (size_t)P.g_stride * sizeof(float));
    }
  }
  P.total = off;
  return P;
}

int n_stream_split(const Plan& P) {
  const int64_t n_max = P.n_stride;
  const int64_t s = (n_max + kStreamRows - 1) / kStreamRows;
  return (int)(s < 1 ? 1 : s);
}

hils_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HILS_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return HILS_ERR_CUDA;
  if (major != 10 || minor != 0) return HILS_ERR_UNSUPPORTED;
  return HILS_OK;
}

bool ok_ptr(const void* ptr, bool needed) { return !needed || (ptr && aligned16(ptr)); }

}  // namespace
}  // namespace hils

using namespace hils;

extern "C" size_t hils_workspace_size(const hils_params* p) {
  if (check_params(p) != HILS_OK) return 0;
  return make_plan(p).total;
}

namespace hils {
namespace {

// Records the caller's timing events between kernel launches (no-op without events).
struct PhaseMarks {
  void* const* ev;
  int n;
  int k;
  cudaStream_t st;
  void mark() {
    if (ev && k < n && ev[k]) cudaEventRecord(reinterpret_cast<cudaEvent_t>(ev[k]), st);
    ++k;
  }
};

int phase_names(const Plan& P, const char** names, int max_names) {
  const char* pre[4];
  int n = 0;
  if (P.decode) {
    pre[0] = P.tc_stream ? "select_stream_tc" : "select_stream";
    pre[1] = "select_topk";
    pre[2] = P.tc_units ? "attn_units_tc" : "attn_units";
    pre[3] = "fuse_units";
    for (int i = 0; i < 4 && i < max_names; ++i) names[i] = pre[i];
    return 4;
  }
  if (P.tc_select) {
    pre[n++] = P.tc_select_t ? "score_topk_t_tc" : "score_topk_tc";
    if (!P.tc_attn || (P.attn_ext && P.D.G > 1 && !P.tc_select_t)) pre[n++] = "select_scores";
  } else {
    pre[n++] = "select_rows";
  }
  pre[n++] = P.tc_attn ? "attn_tc" : "attn_rows";
  for (int i = 0; i < n && i < max_names; ++i) names[i] = pre[i];
  return n;
}

// Steps 1-2 of a prefill plan on the tensor cores: the landmark-major kernel where it applies,
// else the query-major one.
// s_head (nullable): every head's score of each selected chunk, written by the landmark-major
// kernel itself; returns in *s_head_done whether it was.
cudaError_t launch_prefill_select_tc(const Plan& P, const void* q_cal, const void* k_lm,
                                     const float* b_lm, int32_t* idx, float* s_out,
                                     float* s_head, int32_t* status, cudaStream_t st,
                                     bool* s_head_done) {
  *s_head_done = P.tc_select_t && s_head;
  return P.tc_select_t
             ? launch_score_topk_t_tc(P.D, q_cal, k_lm, b_lm, idx, s_out, s_head, status, st)
             : launch_score_topk_tc(P.D, q_cal, k_lm, b_lm, idx, s_out, status, st);
}

// Steps 1-2 of a decode plan: the streaming scorer (sigma rows in the workspace) and one top-K
// CTA per row.  Marks the caller's phase events after each kernel.
cudaError_t launch_decode_select(const Plan& P, const void* q_cal, const void* k_lm,
                                 const float* b_lm, int32_t* idx, float* s_sel, char* ws,
                                 cudaStream_t st, PhaseMarks& pm) {
  cudaError_t e;
  float* sig = reinterpret_cast<float*>(ws + P.off_sig);
  float* gmax = P.g_stride > 0 ? reinterpret_cast<float*>(ws + P.off_gmax) : nullptr;
  e = P.tc_stream ? launch_select_stream_tc(P.D, q_cal, k_lm, b_lm, sig, P.n_stride,
                                            reinterpret_cast<int32_t*>(ws), st, gmax, P.g_stride)
                  : launch_select_stream(P.D, P.bf16, kStreamRows, n_stream_split(P), P.n_stride,
                                         q_cal, k_lm, b_lm, sig, reinterpret_cast<int32_t*>(ws), st);
  pm.mark();
  if (e == cudaSuccess)
    e = launch_select_topk_row(P.D, P.bf16, P.n_stride, sig, q_cal, k_lm, b_lm, idx, s_sel, st,
                               gmax, P.g_stride);
  pm.mark();
  return e;
}

hils_status forward_impl(const hils_params* p, const void* q, const void* q_cal, const void* K,
                         const void* V, const void* k_lm, const float* b_lm, void* out,
                         float* lse_out, int32_t* topk_idx_out, void* workspace,
                         size_t workspace_bytes, hils_stream_t stream, void* const* events,
                         int n_events) {
  hils_status s = check_params(p);
  if (s != HILS_OK) return s;
  const Plan P = make_plan(p);
  const bool any = p->B > 0 && p->N_q > 0;
  const bool any_lm = any && P.D.C > 0;
  if (!ok_ptr(q, any) || !ok_ptr(q_cal, any) || !ok_ptr(K, any) || !ok_ptr(V, any) ||
      !ok_ptr(k_lm, any_lm) || !ok_ptr(b_lm, any_lm) || !ok_ptr(out, any) ||
      (lse_out && !aligned16(lse_out)) || (topk_idx_out && !aligned16(topk_idx_out)))
    return HILS_ERR_INVALID_ARG;
  if (!workspace || !aligned16(workspace) || workspace_bytes < P.total) return HILS_ERR_WORKSPACE;
  if (!any) return HILS_OK;
  if ((s = check_device()) != HILS_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  PhaseMarks pm{events, n_events, 0, st};
  char* ws = static_cast<char*>(workspace);
  int32_t* idx = topk_idx_out ? topk_idx_out : reinterpret_cast<int32_t*>(ws + P.off_idx);
  float* s_sel = reinterpret_cast<float*>(ws + P.off_ssel);
  cudaError_t e;
  pm.mark();
  if (P.decode) {
    float* po = reinterpret_cast<float*>(ws + P.off_po);
    float* pl = reinterpret_cast<float*>(ws + P.off_pl);
    e = launch_decode_select(P, q_cal, k_lm, b_lm, idx, s_sel, ws, st, pm);
    if (e == cudaSuccess)
      e = P.tc_units ? launch_attn_units_tc(P.D, P.n_pieces, q, K, V, idx, po, pl,
                                            reinterpret_cast<int32_t*>(ws), st)
                     : launch_attn_units(P.D, P.bf16, P.n_pieces, q, K, V, idx, po, pl,
                                         reinterpret_cast<int32_t*>(ws), st);
    pm.mark();
    if (e == cudaSuccess)
      e = launch_fuse_units(P.D, P.bf16, P.n_pieces, s_sel, po, pl, out, lse_out, st);
    pm.mark();
  } else {
    if (P.tc_select) {
      bool heads_done = false;
      e = launch_prefill_select_tc(P, q_cal, k_lm, b_lm, idx,
                                   P.tc_attn && P.D.G == 1 ? s_sel : nullptr,
                                   P.attn_ext && P.D.G > 1 ? s_sel : nullptr,
                                   reinterpret_cast<int32_t*>(ws), st, &heads_done);
      // the tensor-core attention takes the scores from there (one head per group), from the
      // per-head scores of the winners (two attention CTAs per SM: the landmark-major scoring
      // kernel writes them, else select_scores), or scores per head itself
      if (e == cudaSuccess && !heads_done && (!P.tc_attn || (P.attn_ext && P.D.G > 1))) {
        pm.mark();
        e = launch_select_scores(P.D, P.bf16, q_cal, k_lm, b_lm, idx, s_sel, st);
      }
    } else {
      e = launch_select_rows(P.D, P.bf16, q_cal, k_lm, b_lm, idx, s_sel, st);
    }
    pm.mark();
    if (e == cudaSuccess)
      e = P.tc_attn ? launch_attn_tc(P.D, q, q_cal, K, V, idx, s_sel, k_lm, b_lm, out, lse_out,
                                     reinterpret_cast<int32_t*>(ws), st)
                    : launch_attn_rows(P.D, P.bf16, q, K, V, idx, s_sel, out, lse_out, nullptr,
                                       nullptr, st);
    pm.mark();
  }
  return e == cudaSuccess ? HILS_OK : HILS_ERR_CUDA;
}

}  // namespace
}  // namespace hils

extern "C" hils_status hils_forward(const hils_params* p, const void* q, const void* q_cal,
                                    const void* K, const void* V, const void* k_lm,
                                    const float* b_lm, void* out, float* lse_out,
                                    int32_t* topk_idx_out, void* workspace,
                                    size_t workspace_bytes, hils_stream_t stream) {
  return forward_impl(p, q, q_cal, K, V, k_lm, b_lm, out, lse_out, topk_idx_out, workspace,
                      workspace_bytes, stream, nullptr, 0);
}

extern "C" hils_status hils_forward_timed(const hils_params* p, const void* q, const void* q_cal,
                                          const void* K, const void* V, const void* k_lm,
                                          const float* b_lm, void* out, float* lse_out,
                                          int32_t* topk_idx_out, void* workspace,
                                          size_t workspace_bytes, hils_stream_t stream,
                                          void* const* events, int n_events) {
  return forward_impl(p, q, q_cal, K, V, k_lm, b_lm, out, lse_out, topk_idx_out, workspace,
                      workspace_bytes, stream, events, n_events);
}

extern "C" int hils_forward_phases(const hils_params* p, const char** names, int max_names) {
  if (check_params(p) != HILS_OK) return -1;
  return phase_names(make_plan(p), names, names ? max_names : 0);
}

extern "C" hils_status hils_select(const hils_params* p, const void* q_cal, const void* k_lm,
                                   const float* b_lm, int32_t* idx, float* s_sel,
                                   void* workspace, size_t workspace_bytes,
                                   hils_stream_t stream) {
  hils_status s = check_params(p);
  if (s != HILS_OK) return s;
  const Plan P = make_plan(p);
  const bool any = p->B > 0 && p->N_q > 0;
  const bool any_lm = any && P.D.C > 0;
  if (!ok_ptr(q_cal, any) || !ok_ptr(k_lm, any_lm) || !ok_ptr(b_lm, any_lm) ||
      !ok_ptr(idx, any && p->K_top > 0) || (s_sel && !aligned16(s_sel)))
    return HILS_ERR_INVALID_ARG;
  if (!workspace || !aligned16(workspace) || workspace_bytes < P.total) return HILS_ERR_WORKSPACE;
  if (!any) return HILS_OK;
  if ((s = check_device()) != HILS_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  cudaError_t e;
  if (P.decode) {
    PhaseMarks none{nullptr, 0, 0, st};
    e = launch_decode_select(P, q_cal, k_lm, b_lm, idx, s_sel, ws, st, none);
  } else if (P.tc_select) {
    // with one head per KV group the scores the selection ranked by are the per-head scores
    bool heads_done = false;
    e = launch_prefill_select_tc(P, q_cal, k_lm, b_lm, idx, P.D.G == 1 ? s_sel : nullptr,
                                 P.D.G != 1 ? s_sel : nullptr, reinterpret_cast<int32_t*>(ws),
                                 st, &heads_done);
    if (e == cudaSuccess && s_sel && P.D.G != 1 && !heads_done)
      e = launch_select_scores(P.D, P.bf16, q_cal, k_lm, b_lm, idx, s_sel, st);
  } else {
    e = launch_select_rows(P.D, P.bf16, q_cal, k_lm, b_lm, idx, s_sel, st);
  }
  return e == cudaSuccess ? HILS_OK : HILS_ERR_CUDA;
}

extern "C" hils_status hils_chunk_attn(const hils_params* p, const void* q, const void* K,
                                       const void* V, const int32_t* idx, float* unit_o,
                                       float* unit_lse, hils_stream_t stream) {
  hils_status s = check_params(p);
  if (s != HILS_OK) return s;
  const Plan P = make_plan(p);
  const bool any = p->B > 0 && p->N_q > 0;
  if (!ok_ptr(q, any) || !ok_ptr(K, any) || !ok_ptr(V, any) ||
      !ok_ptr(idx, any && p->K_top > 0) || !ok_ptr(unit_o, any) || !ok_ptr(unit_lse, any))
    return HILS_ERR_INVALID_ARG;
  if (!any) return HILS_OK;
  if ((s = check_device()) != HILS_OK) return s;
  cudaError_t e = launch_attn_rows(P.D, P.bf16, q, K, V, idx, nullptr, nullptr, nullptr, unit_o,
                                   unit_lse, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HILS_OK : HILS_ERR_CUDA;
}

extern "C" hils_status hils_fuse(const hils_params* p, const float* s_sel, const float* unit_o,
                                 const float* unit_lse, void* out, float* lse_out,
                                 hils_stream_t stream) {
  hils_status s = check_params(p);
  if (s != HILS_OK) return s;
  const Plan P = make_plan(p);
  const bool any = p->B > 0 && p->N_q > 0;
  if (!ok_ptr(s_sel, any && p->K_top > 0) || !ok_ptr(unit_o, any) || !ok_ptr(unit_lse, any) ||
      !ok_ptr(out, any) || (lse_out && !aligned16(lse_out)))
    return HILS_ERR_INVALID_ARG;
  if (!any) return HILS_OK;
  if ((s = check_device()) != HILS_OK) return s;
  cudaError_t e = launch_fuse_units(P.D, P.bf16, 1, s_sel, unit_o, unit_lse, out, lse_out,
                                    reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HILS_OK : HILS_ERR_CUDA;
}

extern "C" hils_status hils_landmarks(const hils_params* p, const void* q_lm, const void* K,
                                      void* k_lm, float* b_lm, hils_stream_t stream) {
  hils_status s = check_params(p);
  if (s != HILS_OK) return s;
  if (p->d != 16 && p->d != 32 && p->d != 64 && p->d != 128) return HILS_ERR_UNSUPPORTED;
  const Plan P = make_plan(p);
  const bool any = P.D.B > 0 && P.D.C > 0;
  if (!ok_ptr(q_lm, any) || !ok_ptr(K, any) || !ok_ptr(k_lm, any) || !ok_ptr(b_lm, any))
    return HILS_ERR_INVALID_ARG;
  if (!any) return HILS_OK;
  if ((s = check_device()) != HILS_OK) return s;
  return launch_landmarks(P.D, P.bf16, 0, P.D.C, P.D.C, q_lm, K, k_lm, b_lm,
                          reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? HILS_OK
             : HILS_ERR_CUDA;
}

extern "C" hils_status hils_decode_step(const hils_params* p, const void* q, const void* q_cal,
                                        const void* k_new, const void* v_new,
                                        const void* q_lm_new, void* K, void* V, void* k_lm,
                                        float* b_lm, void* out, float* lse_out,
                                        int32_t* topk_idx_out, void* workspace,
                                        size_t workspace_bytes, hils_stream_t stream) {
  hils_status s = check_params(p);
  if (s != HILS_OK) return s;
  if (p->N_q != 1) return HILS_ERR_INVALID_ARG;
  const Plan P = make_plan(p);
  if (!P.decode || p->d % (p->dtype == HILS_BF16 ? 8 : 4) != 0) return HILS_ERR_UNSUPPORTED;
  const int64_t pos = p->q_pos0;
  // the new token completes chunk c_done when it is the chunk's last one
  const bool completes = (pos + 1) % p->S == 0;
  const bool any = p->B > 0;
  if (!ok_ptr(k_new, any) || !ok_ptr(v_new, any) || !ok_ptr(K, any) || !ok_ptr(V, any) ||
      !ok_ptr(q_lm_new, any && completes) || !ok_ptr(k_lm, any && completes) ||
      !ok_ptr(b_lm, any && completes))
    return HILS_ERR_INVALID_ARG;
  if (!any) return HILS_OK;
  // the forward's own checks come first, so a bad call writes nothing
  if (!ok_ptr(q, true) || !ok_ptr(q_cal, true) || !ok_ptr(out, true) ||
      (lse_out && !aligned16(lse_out)) || (topk_idx_out && !aligned16(topk_idx_out)) ||
      (P.D.C > 0 && (!ok_ptr(k_lm, true) || !ok_ptr(b_lm, true))))
    return HILS_ERR_INVALID_ARG;
  if (!workspace || !aligned16(workspace) || workspace_bytes < P.total) return HILS_ERR_WORKSPACE;
  if ((s = check_device()) != HILS_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (launch_append_kv(P.D, P.bf16, pos, k_new, v_new, K, V, st) != cudaSuccess)
    return HILS_ERR_CUDA;
  if (completes && launch_landmarks(P.D, P.bf16, pos / p->S, 1, 1, q_lm_new, K, k_lm, b_lm, st) !=
                       cudaSuccess)
    return HILS_ERR_CUDA;
  return forward_impl(p, q, q_cal, K, V, k_lm, b_lm, out, lse_out, topk_idx_out, workspace,
                      workspace_bytes, stream, nullptr, 0);
}

namespace hils {
namespace {
hils_status check_prologue(const hils_params* p, const hils_prologue_params* c) {
  hils_status s = check_params(p);
  if (s != HILS_OK) return s;
  if (!c || !(c->rope_base > 1.0) || std::isnan(c->train_len) || c->r < 0 || c->d_model < 0)
    return HILS_ERR_INVALID_ARG;
  if (p->d != 64 && p->d != 128) return HILS_ERR_UNSUPPORTED;
  if (c->r > 64) return HILS_ERR_UNSUPPORTED;
  if (c->r > 0 && !qdown_supported(p->Hq * c->r, c->d_model)) return HILS_ERR_UNSUPPORTED;
  if (p->B * p->N_q >= (int64_t)INT32_MAX || p->Hq > 65535 || p->B > 65535)
    return HILS_ERR_UNSUPPORTED;
  return HILS_OK;
}
}  // namespace
}  // namespace hils

extern "C" size_t hils_qcal_workspace_size(const hils_params* p, const hils_prologue_params* c) {
  if (check_prologue(p, c) != HILS_OK) return 0;
  return kStatusBytes + align_up((size_t)(p->B * p->N_q * p->Hq) * (size_t)c->r * 4);
}

extern "C" hils_status hils_qcal_hope(const hils_params* p, const hils_prologue_params* c,
                                      const void* q, const void* hidden, const void* W_down,
                                      const void* W_up, void* q_out, void* q_cal_out,
                                      void* workspace, size_t workspace_bytes,
                                      hils_stream_t stream) {
  hils_status s = check_prologue(p, c);
  if (s != HILS_OK) return s;
  const bool any = p->B > 0 && p->N_q > 0;
  const bool qcal = any && c->r > 0;
  if (!ok_ptr(q, any) || !ok_ptr(q_out, any) || !ok_ptr(q_cal_out, any) ||
      !ok_ptr(hidden, qcal) || !ok_ptr(W_down, qcal) || !ok_ptr(W_up, qcal))
    return HILS_ERR_INVALID_ARG;
  if (q_cal_out == q) return HILS_ERR_INVALID_ARG;
  const size_t need = hils_qcal_workspace_size(p, c);
  if (!workspace || !aligned16(workspace) || workspace_bytes < need) return HILS_ERR_WORKSPACE;
  if (!any) return HILS_OK;
  if ((s = check_device()) != HILS_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  float* u = reinterpret_cast<float*>(ws + kStatusBytes);
  cudaError_t e = cudaSuccess;
  if (qcal)
    e = launch_qdown(p->B * p->N_q, p->Hq * c->r, c->d_model, hidden, W_down, u,
                     reinterpret_cast<int32_t*>(ws), st);
  if (e == cudaSuccess)
    e = launch_qcal_hope(p->B, p->Hq, p->N_q, p->d, p->q_pos0, c->r, c->rope_base,
                         c->train_len, p->dtype == HILS_BF16, q, u, W_up, q_out, q_cal_out, st);
  return e == cudaSuccess ? HILS_OK : HILS_ERR_CUDA;
}

extern "C" hils_status hils_hope_rotate(const hils_params* p, const hils_prologue_params* c,
                                        int64_t B, int64_t H, int64_t N, int64_t pos0,
                                        const void* x, void* x_out, hils_stream_t stream) {
  hils_status s = check_params(p);
  if (s != HILS_OK) return s;
  if (!c || !(c->rope_base > 1.0) || std::isnan(c->train_len) || B < 0 || H < 0 || N < 0 ||
      pos0 < 0)
    return HILS_ERR_INVALID_ARG;
  if (p->d != 64 && p->d != 128) return HILS_ERR_UNSUPPORTED;
  if (B * H > 65535) return HILS_ERR_UNSUPPORTED;
  const bool any = B > 0 && H > 0 && N > 0;
  if (!ok_ptr(x, any) || !ok_ptr(x_out, any)) return HILS_ERR_INVALID_ARG;
  if (!any) return HILS_OK;
  if ((s = check_device()) != HILS_OK) return s;
  return launch_hope_rotate(B * H, N, p->d, pos0, c->rope_base, c->train_len,
                            p->dtype == HILS_BF16, x, x_out,
                            reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? HILS_OK
             : HILS_ERR_CUDA;
}

extern "C" size_t hils_backward_workspace_size(const hils_params* p) {
  if (check_params(p) != HILS_OK) return 0;
  const Plan P = make_plan(p);
  if (!backward_supported(P.D)) return 0;
  return backward_ws_layout(P.D, nullptr, nullptr);
}

extern "C" hils_status hils_backward(const hils_params* p, const void* q, const void* q_cal,
                                     const void* K, const void* V, const void* k_lm,
                                     const float* b_lm, const int32_t* topk_idx,
                                     const void* dout, const float* dlse, float* dq,
                                     float* dq_cal, float* dK, float* dV, float* dk_lm,
                                     float* db_lm, void* workspace, size_t workspace_bytes,
                                     hils_stream_t stream) {
  hils_status s = check_params(p);
  if (s != HILS_OK) return s;
  const Plan P = make_plan(p);
  if (!backward_supported(P.D)) return HILS_ERR_UNSUPPORTED;
  const bool rows = p->B > 0 && p->N_q > 0;
  const bool keys = p->B > 0;
  const bool lm = keys && P.D.C > 0;
  if (!ok_ptr(q, rows) || !ok_ptr(q_cal, rows) || !ok_ptr(dout, rows) || !ok_ptr(dq, rows) ||
      !ok_ptr(dq_cal, rows) || !ok_ptr(topk_idx, rows && p->K_top > 0) || !ok_ptr(K, keys) ||
      !ok_ptr(V, keys) || !ok_ptr(dK, keys) || !ok_ptr(dV, keys) || !ok_ptr(k_lm, lm) ||
      !ok_ptr(b_lm, lm) || !ok_ptr(dk_lm, lm) || !ok_ptr(db_lm, lm) ||
      (dlse && !aligned16(dlse)))
    return HILS_ERR_INVALID_ARG;
  const size_t need = backward_ws_layout(P.D, nullptr, nullptr);
  if (!workspace || !aligned16(workspace) || workspace_bytes < need) return HILS_ERR_WORKSPACE;
  if (!keys) return HILS_OK;
  if ((s = check_device()) != HILS_OK) return s;
  BwdWs w;
  backward_ws_layout(P.D, &w, static_cast<char*>(workspace));
  BwdArgs a{q, q_cal, K, V, k_lm, b_lm, topk_idx, dout, dlse, dq, dq_cal, dK, dV, dk_lm, db_lm};
  return launch_backward(P.D, P.bf16, a, w, reinterpret_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? HILS_OK
             : HILS_ERR_CUDA;
}

extern "C" hils_status hils_workspace_init(void* workspace, size_t workspace_bytes,
                                           hils_stream_t stream) {
  if (!workspace || !aligned16(workspace) || workspace_bytes < kStatusBytes)
    return HILS_ERR_WORKSPACE;
  return cudaMemsetAsync(workspace, 0, kStatusBytes, reinterpret_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? HILS_OK
             : HILS_ERR_CUDA;
}

extern "C" hils_status hils_device_status(void* workspace, hils_stream_t stream,
                                          int32_t* status) {
  if (!workspace || !status) return HILS_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemsetAsync(workspace, 0, sizeof(word), st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return HILS_ERR_CUDA;
  *status = word;
  return HILS_OK;
}

extern "C" hils_status hils_wait_check(uint32_t polls, int complete, void* workspace,
                                       size_t workspace_bytes, hils_stream_t stream) {
  if (!workspace || !aligned16(workspace) || workspace_bytes < kStatusBytes)
    return HILS_ERR_WORKSPACE;
  if (polls == 0) return HILS_ERR_INVALID_ARG;
  hils_status s = check_device();
  if (s != HILS_OK) return s;
  return launch_wait_check(polls, complete, static_cast<int32_t*>(workspace),
                           reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? HILS_OK
             : HILS_ERR_CUDA;
}

extern "C" const char* hils_status_string(hils_status s) {
  switch (s) {
    case HILS_OK: return "ok";
    case HILS_ERR_INVALID_ARG: return "invalid argument";
    case HILS_ERR_UNSUPPORTED: return "unsupported configuration";
    case HILS_ERR_WORKSPACE: return "workspace missing or too small";
    case HILS_ERR_CUDA: return "CUDA error";
    case HILS_ERR_DEVICE_CHECK: return "device-side check failed";
    case HILS_ERR_TIMEOUT: return "bounded on-chip wait timed out";
  }
  return "unknown status";
}

extern "C" const char* hils_version(void) { return "hils-b200 " HILS_GIT_DESCRIBE " sm_100a"; }

// ---------------------------------------------------------------------------------------------
// Steps 1-2 with the library's own scratch memory, for callers that cannot hand the library a
// workspace buffer.  The scratch (the status word and the decode path's per-split candidate
// lists) lives in one file-scope device array of fixed size; every device that loads the
// library holds its own copy until the process exits.
namespace hils {
namespace {

constexpr size_t kStaticScratchBytes = 8u << 20;   // 8 MiB per device
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of this device's scratch array.  In host code `g_static_scratch` names a host
// stand-in, not device memory, so the address is looked up once per device (with that device
// current) and cached; that first lookup also zeroes the array's status word on `st`.
hils_status static_scratch(cudaStream_t st, void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HILS_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return HILS_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return HILS_ERR_CUDA;
    if (cudaMemsetAsync(p, 0, kStatusBytes, st) != cudaSuccess) return HILS_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return HILS_OK;
}

}  // namespace
}  // namespace hils

extern "C" size_t hils_select_noalloc_max_bytes(void) { return hils::kStaticScratchBytes; }

extern "C" hils_status hils_select_noalloc(const hils_params* p, const void* q_cal,
                                           const void* k_lm, const float* b_lm, int32_t* idx,
                                           float* s_sel, hils_stream_t stream) {
  hils_status s = check_params(p);
  if (s != HILS_OK) return s;
  const Plan P = make_plan(p);
  const bool any = p->B > 0 && p->N_q > 0;
  const bool any_lm = any && P.D.C > 0;
  if (!ok_ptr(q_cal, any) || !ok_ptr(k_lm, any_lm) || !ok_ptr(b_lm, any_lm) ||
      !ok_ptr(idx, any && p->K_top > 0) || (s_sel && !aligned16(s_sel)))
    return HILS_ERR_INVALID_ARG;
  // scratch layout: [status word | decode split lists (values) | decode split lists (ids)]
  const size_t sel_rows = (size_t)(p->B * p->Hkv * p->N_q);
  const size_t list_bytes =
      P.decode ? align_up(sel_rows * (size_t)P.n_split * (size_t)P.D.K * sizeof(float)) : 0;
  const size_t need = kStatusBytes + 2 * list_bytes;
  if (need > kStaticScratchBytes) return HILS_ERR_WORKSPACE;
  if (!any) return HILS_OK;
  if ((s = check_device()) != HILS_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  void* scratch = nullptr;
  if ((s = static_scratch(st, &scratch)) != HILS_OK) return s;
  char* ws = static_cast<char*>(scratch);
  // the status word keeps the first failure since it was last read (hils_select_noalloc_status)
  cudaError_t e;
  if (P.decode) {
    float* pv = reinterpret_cast<float*>(ws + kStatusBytes);
    int32_t* pc = reinterpret_cast<int32_t*>(ws + kStatusBytes + list_bytes);
    e = launch_select_split(P.D, P.bf16, P.cps, P.n_split, q_cal, k_lm, b_lm, pv, pc, st);
    if (e == cudaSuccess)
      e = launch_select_merge(P.D, P.bf16, P.n_split, pv, pc, q_cal, k_lm, b_lm, idx, s_sel, st);
  } else if (P.tc_select) {
    // with one head per KV group the scores the selection ranked by are the per-head scores
    bool heads_done = false;
    e = launch_prefill_select_tc(P, q_cal, k_lm, b_lm, idx, P.D.G == 1 ? s_sel : nullptr,
                                 P.D.G != 1 ? s_sel : nullptr, reinterpret_cast<int32_t*>(ws),
                                 st, &heads_done);
    if (e == cudaSuccess && s_sel && P.D.G != 1 && !heads_done)
      e = launch_select_scores(P.D, P.bf16, q_cal, k_lm, b_lm, idx, s_sel, st);
  } else {
    e = launch_select_rows(P.D, P.bf16, q_cal, k_lm, b_lm, idx, s_sel, st);
  }
  return e == cudaSuccess ? HILS_OK : HILS_ERR_CUDA;
}

extern "C" hils_status hils_select_noalloc_status(hils_stream_t stream, int32_t* status) {
  if (!status) return HILS_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  void* scratch = nullptr;
  hils_status s = static_scratch(st, &scratch);
  if (s != HILS_OK) return s;
  int32_t word = 0;
  if (cudaMemcpyAsync(&word, scratch, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemsetAsync(scratch, 0, sizeof(word), st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return HILS_ERR_CUDA;
  *status = word;
  return HILS_OK;
}
