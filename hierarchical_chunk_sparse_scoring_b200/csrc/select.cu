// Steps 1-2 on CUDA cores: landmark scores, group max, top-K with ties to the lower chunk.
//
// Surrogate chunk score s_{h,c} = q_cal[h] . k_lm[c] * scale + b_lm[c] ([Reader] "The
// HiLS-Attention Mechanism" surrogate step and the Q-Cal worked example in "Implementation and
// Training Recipes"); the group keeps a chunk by the max over its heads ([Reader] GQA
// paragraph); the K best distant chunks are kept ([Reader] "Limitations of Naive Sparse
// Attention").  [Reader] = paperglide.net reader of "Hierarchical Sparse Attention Done Right".
//
// Two layouts of the same computation:
//   select_rows_kernel   one warp per (b, g, query): lanes stride over chunks; used where there
//                        are many queries (prefill) and for any d.
//   select_split_kernel  many CTAs per (b, g, query) over disjoint chunk ranges, each writing
//                        its own top-K; select_merge_kernel merges them.  Used for decode,
//                        where one query's landmark stream (n x d) must be spread over the GPU.
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace hils {

// s_sel for the winners held by lanes 0..K-1 (lane r: chunk c_r); per-head dot on CUDA cores.
template <typename T, int GM>
__device__ __forceinline__ void write_selection(const Dims& D, int64_t b, int64_t g, int64_t i,
                                                const float* qs /* [G][d] smem or null */,
                                                const T* qc, const T* kb, const float* bb,
                                                int lane, int c, int32_t* idx, float* s_sel) {
  const int K = D.K, G = D.G, d = (int)D.d;
  const int64_t sel_row = ((b * D.Hkv + g) * D.N_q + i) * K;
  if (lane < K) {
    const bool valid = c != INT_MAX;
    idx[sel_row + lane] = valid ? c : -1;
    if (s_sel) {
      float acc[GM];
#pragma unroll
      for (int h = 0; h < GM; ++h) acc[h] = 0.f;
      if (valid) {
        const T* kr = kb + (int64_t)c * d;
        for (int k = 0; k < d; k += 4) {
          float kv[4];
          Elem<T>::load4(kr + k, kv);
#pragma unroll
          for (int h = 0; h < GM; ++h) {
            if (h < G) {
              float qv[4];
              if (qs) {
                float4 t = *reinterpret_cast<const float4*>(qs + h * d + k);
                qv[0] = t.x; qv[1] = t.y; qv[2] = t.z; qv[3] = t.w;
              } else {
                Elem<T>::load4(qc + (((b * D.Hq) + g * G + h) * D.N_q + i) * D.d + k, qv);
              }
              acc[h] = fmaf(qv[0], kv[0], acc[h]);
              acc[h] = fmaf(qv[1], kv[1], acc[h]);
              acc[h] = fmaf(qv[2], kv[2], acc[h]);
              acc[h] = fmaf(qv[3], kv[3], acc[h]);
            }
          }
        }
      }
      const float bc = valid ? bb[c] : 0.f;
#pragma unroll
      for (int h = 0; h < GM; ++h) {
        if (h < G) {
          const int64_t hrow = ((b * D.Hq) + g * G + h) * D.N_q + i;
          s_sel[hrow * K + lane] = valid ? fmaf(acc[h], D.scale, bc) : -INFINITY;
        }
      }
    }
  }
}

// Same result for bf16 inputs with the winners' landmark rows read by wide loads that are all in
// flight at once, and the group's calibrated queries staged once per warp in shared memory
// (qsh: [GM][D_] bf16; already filled, and visible to this warp, when q_staged); lane r < K
// handles winner c_r.
template <int D_, int GM>
__device__ __forceinline__ void write_selection_wide(const Dims& D, int64_t b, int64_t g,
                                                     int64_t i, __nv_bfloat16* qsh,
                                                     const __nv_bfloat16* qc,
                                                     const __nv_bfloat16* kb, const float* bb,
                                                     int lane, int c, int32_t* idx,
                                                     float* s_sel, bool q_staged = false) {
  constexpr int NV = D_ / 8;   // 16-byte vectors per row
  const int K = D.K, G = D.G;
  uint4* q4 = reinterpret_cast<uint4*>(qsh);
  for (int e = lane; !q_staged && e < G * NV; e += 32) {
    const int h = e / NV, j = e - h * NV;
    const int64_t hrow = ((b * D.Hq) + g * G + h) * D.N_q + i;
    q4[h * NV + j] = __ldg(reinterpret_cast<const uint4*>(qc + hrow * D_) + j);
  }
  __syncwarp();
  const int64_t sel_row = ((b * D.Hkv + g) * D.N_q + i) * K;
  if (lane >= K) return;
  const bool valid = c != INT_MAX;
  idx[sel_row + lane] = valid ? c : -1;
  if (!s_sel) return;
  uint4 kv[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j)
    kv[j] = valid ? __ldg(reinterpret_cast<const uint4*>(kb + (int64_t)c * D_) + j)
                  : make_uint4(0u, 0u, 0u, 0u);
  const float bc = valid ? __ldg(bb + c) : 0.f;
  // (loops kept rolled: this runs once per row, and straight-line code this long would be
  // fetched from L2 instruction by instruction)
#pragma unroll 1
  for (int h = 0; h < GM; ++h) {
    if (h >= G) break;
    float a4[4] = {0.f, 0.f, 0.f, 0.f};   // four short dependency chains
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const uint4 qv = q4[h * NV + j];
      float& a = a4[j & 3];
      a = fmaf(bf16_lo(qv.x), bf16_lo(kv[j].x), a);
      a = fmaf(bf16_hi(qv.x), bf16_hi(kv[j].x), a);
      a = fmaf(bf16_lo(qv.y), bf16_lo(kv[j].y), a);
      a = fmaf(bf16_hi(qv.y), bf16_hi(kv[j].y), a);
      a = fmaf(bf16_lo(qv.z), bf16_lo(kv[j].z), a);
      a = fmaf(bf16_hi(qv.z), bf16_hi(kv[j].z), a);
      a = fmaf(bf16_lo(qv.w), bf16_lo(kv[j].w), a);
      a = fmaf(bf16_hi(qv.w), bf16_hi(kv[j].w), a);
    }
    const float a = (a4[0] + a4[1]) + (a4[2] + a4[3]);
    const int64_t hrow = ((b * D.Hq) + g * G + h) * D.N_q + i;
    s_sel[hrow * K + lane] = valid ? fmaf(a, D.scale, bc) : -INFINITY;
  }
}

template <typename T, int GM, int KM>
__global__ void __launch_bounds__(256) select_rows_kernel(Dims D, const T* __restrict__ qc,
                                                          const T* __restrict__ klm,
                                                          const float* __restrict__ blm,
                                                          int32_t* __restrict__ idx,
                                                          float* __restrict__ s_sel) {
  extern __shared__ __align__(16) float smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t rows = D.B * D.Hkv * D.N_q;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= rows) return;
  const int64_t i = row % D.N_q, bg = row / D.N_q, g = bg % D.Hkv, b = bg / D.Hkv;
  const int d = (int)D.d, G = D.G;
  float* qs = smem + (size_t)warp * G * d;
  for (int e = lane; e < G * d; e += 32) {
    const int h = e / d, k = e - h * d;
    qs[e] = Elem<T>::to_f(qc[(((b * D.Hq) + g * G + h) * D.N_q + i) * D.d + k]);
  }
  __syncwarp();
  const int64_t n = n_eligible(D.q_pos0 + i, D.S, D.W);
  const T* kb = klm + bg * D.C * D.d;
  const float* bb = blm + bg * D.C;
  TopList<KM> L;
  L.clear();
  for (int64_t c = lane; c < n; c += 32) {
    const T* kr = kb + c * d;
    float acc[GM];
#pragma unroll
    for (int h = 0; h < GM; ++h) acc[h] = 0.f;
    for (int k = 0; k < d; k += 4) {
      float kv[4];
      Elem<T>::load4(kr + k, kv);
#pragma unroll
      for (int h = 0; h < GM; ++h) {
        if (h < G) {
          float4 qv = *reinterpret_cast<const float4*>(qs + h * d + k);
          acc[h] = fmaf(qv.x, kv[0], acc[h]);
          acc[h] = fmaf(qv.y, kv[1], acc[h]);
          acc[h] = fmaf(qv.z, kv[2], acc[h]);
          acc[h] = fmaf(qv.w, kv[3], acc[h]);
        }
      }
    }
    const float bc = bb[c];
    float sig = -INFINITY;
#pragma unroll
    for (int h = 0; h < GM; ++h)
      if (h < G) sig = fmaxf(sig, fmaf(acc[h], D.scale, bc));
    L.insert(sig, (int)c, D.K);
  }
  float wv;
  int wc;
  warp_merge_topk<KM>(L, D.K, lane, wv, wc);
  write_selection<T, GM>(D, b, g, i, qs, qc, kb, bb, lane, wc, idx, s_sel);
}

// Per-head scores of already selected chunks (used after the tensor-core selection, which
// keeps only the group score): one warp per (b, g, query); the group's calibrated queries are
// staged in shared memory and lane r handles idx[r].
template <typename T, int GM>
__global__ void __launch_bounds__(128) select_scores_kernel(Dims D, const T* __restrict__ qc,
                                                            const T* __restrict__ klm,
                                                            const float* __restrict__ blm,
                                                            const int32_t* __restrict__ idx,
                                                            float* __restrict__ s_sel) {
  __shared__ __align__(16) float qs[4][GM * kMaxD];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t rows = D.B * D.Hkv * D.N_q;
  const int64_t row = (int64_t)blockIdx.x * 4 + warp;
  if (row >= rows) return;
  const int64_t i = row % D.N_q, bg = row / D.N_q, g = bg % D.Hkv, b = bg / D.Hkv;
  const int K = D.K, G = D.G, d = (int)D.d;
  for (int e = lane * 4; e < G * d; e += 128) {
    const int h = e / d, k = e - h * d;
    float v[4];
    Elem<T>::load4(qc + (((b * D.Hq) + g * G + h) * D.N_q + i) * D.d + k, v);
    Elem<float>::store4(&qs[warp][e], v);
  }
  __syncwarp();
  if (lane >= K) return;
  const int c = idx[row * K + lane];
  const bool valid = c >= 0 && c < D.C;
  float acc[GM];
#pragma unroll
  for (int h = 0; h < GM; ++h) acc[h] = 0.f;
  if (valid) {
    const T* kr = klm + (bg * D.C + c) * d;
    for (int k = 0; k < d; k += 4) {
      float kv[4];
      Elem<T>::load4(kr + k, kv);
#pragma unroll
      for (int h = 0; h < GM; ++h) {
        if (h < G) {
          const float4 qv = *reinterpret_cast<const float4*>(&qs[warp][h * d + k]);
          acc[h] = fmaf(qv.x, kv[0], acc[h]);
          acc[h] = fmaf(qv.y, kv[1], acc[h]);
          acc[h] = fmaf(qv.z, kv[2], acc[h]);
          acc[h] = fmaf(qv.w, kv[3], acc[h]);
        }
      }
    }
  }
  const float bc = valid ? blm[bg * D.C + c] : 0.f;
#pragma unroll
  for (int h = 0; h < GM; ++h) {
    if (h < G) {
      const int64_t hrow = ((b * D.Hq) + g * G + h) * D.N_q + i;
      s_sel[hrow * K + lane] = valid ? fmaf(acc[h], D.scale, bc) : -INFINITY;
    }
  }
}

// bf16 variant: one warp per (b, g, query); LPC lanes share a selected chunk, each holding
// D_/LPC of its landmark dimensions in registers (16-byte loads, all issued before use); the
// group's calibrated queries are staged in shared memory as fp32.
template <int D_, int GM, int LPC>
__global__ void __launch_bounds__(128) select_scores_bf16_kernel(
    Dims D, const __nv_bfloat16* __restrict__ qc, const __nv_bfloat16* __restrict__ klm,
    const float* __restrict__ blm, const int32_t* __restrict__ idx, float* __restrict__ s_sel) {
  constexpr int DPL = D_ / LPC;          // dims per lane
  constexpr int NV = DPL / 8;            // 16-byte vectors per lane
  __shared__ __align__(16) float qs[4][GM * D_];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t rows = D.B * D.Hkv * D.N_q;
  const int64_t row = (int64_t)blockIdx.x * 4 + warp;
  if (row >= rows) return;
  const int64_t i = row % D.N_q, bg = row / D.N_q, g = bg % D.Hkv, b = bg / D.Hkv;
  const int K = D.K, G = D.G;
  const int slot = lane / LPC, part = lane % LPC;
  // independent loads first (the selection and this row's calibrated queries), then the
  // selected landmark rows and biases, which depend on the selection
  const int c = slot < K ? idx[row * K + slot] : -1;
  constexpr int QV = (GM * D_ + 255) / 256;   // 16-byte query vectors per lane
  float qv[QV][8];
#pragma unroll
  for (int x = 0; x < QV; ++x) {
    const int e = x * 256 + lane * 8;
    if (e < G * D_) {
      const int h = e / D_, k = e - h * D_;
      load_vec<__nv_bfloat16, 8>(qc + (((b * D.Hq) + g * G + h) * D.N_q + i) * D_ + k, qv[x]);
    }
  }
  const bool valid = c >= 0 && c < D.C;
  float kv[DPL];
  if (valid) {
    const __nv_bfloat16* kr = klm + (bg * D.C + c) * D_ + part * DPL;
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      float t[8];
      load_vec<__nv_bfloat16, 8>(kr + v * 8, t);
#pragma unroll
      for (int e = 0; e < 8; ++e) kv[v * 8 + e] = t[e];
    }
  } else {
#pragma unroll
    for (int e = 0; e < DPL; ++e) kv[e] = 0.f;
  }
  const float bc = valid ? __ldg(blm + bg * D.C + c) : 0.f;
#pragma unroll
  for (int x = 0; x < QV; ++x) {
    const int e = x * 256 + lane * 8;
    if (e < G * D_) {
      *reinterpret_cast<float4*>(&qs[warp][e]) =
          make_float4(qv[x][0], qv[x][1], qv[x][2], qv[x][3]);
      *reinterpret_cast<float4*>(&qs[warp][e + 4]) =
          make_float4(qv[x][4], qv[x][5], qv[x][6], qv[x][7]);
    }
  }
  __syncwarp();
#pragma unroll
  for (int h = 0; h < GM; ++h) {
    if (h >= G) break;
    float a = 0.f;
#pragma unroll
    for (int e4 = 0; e4 < DPL; e4 += 4) {
      const float4 q4 = *reinterpret_cast<const float4*>(&qs[warp][h * D_ + part * DPL + e4]);
      a = fmaf(q4.x, kv[e4 + 0], a);
      a = fmaf(q4.y, kv[e4 + 1], a);
      a = fmaf(q4.z, kv[e4 + 2], a);
      a = fmaf(q4.w, kv[e4 + 3], a);
    }
#pragma unroll
    for (int o = LPC / 2; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if (part == 0 && slot < K) {
      const int64_t hrow = ((b * D.Hq) + g * G + h) * D.N_q + i;
      s_sel[hrow * K + slot] = valid ? fmaf(a, D.scale, bc) : -INFINITY;
    }
  }
}

template <int D_, int GM>
static cudaError_t launch_scores_bf16_g(const Dims& D, const void* qc, const void* klm,
                                        const float* blm, const int32_t* idx, float* s_sel,
                                        cudaStream_t st) {
  const int64_t rows = D.B * D.Hkv * D.N_q;
  const unsigned blocks = (unsigned)((rows + 3) / 4);
  const auto* q = (const __nv_bfloat16*)qc;
  const auto* k = (const __nv_bfloat16*)klm;
  if (D.K <= 8)
    select_scores_bf16_kernel<D_, GM, 4><<<blocks, 128, 0, st>>>(D, q, k, blm, idx, s_sel);
  else if (D.K <= 16)
    select_scores_bf16_kernel<D_, GM, 2><<<blocks, 128, 0, st>>>(D, q, k, blm, idx, s_sel);
  else
    select_scores_bf16_kernel<D_, GM, 1><<<blocks, 128, 0, st>>>(D, q, k, blm, idx, s_sel);
  return cudaGetLastError();
}

template <int D_>
static cudaError_t launch_scores_bf16_d(const Dims& D, const void* qc, const void* klm,
                                        const float* blm, const int32_t* idx, float* s_sel,
                                        cudaStream_t st) {
  if (D.G <= 1) return launch_scores_bf16_g<D_, 1>(D, qc, klm, blm, idx, s_sel, st);
  if (D.G <= 2) return launch_scores_bf16_g<D_, 2>(D, qc, klm, blm, idx, s_sel, st);
  if (D.G <= 4) return launch_scores_bf16_g<D_, 4>(D, qc, klm, blm, idx, s_sel, st);
  return launch_scores_bf16_g<D_, 8>(D, qc, klm, blm, idx, s_sel, st);
}

template <typename T>
static cudaError_t launch_scores_g(const Dims& D, const void* qc, const void* klm,
                                   const float* blm, const int32_t* idx, float* s_sel,
                                   cudaStream_t st) {
  const int64_t rows = D.B * D.Hkv * D.N_q;
  const unsigned blocks = (unsigned)((rows + 3) / 4);
#define HILS_SC(GM) select_scores_kernel<T, GM><<<blocks, 128, 0, st>>>(D, (const T*)qc, \
                        (const T*)klm, blm, idx, s_sel)
  if (D.G <= 1) HILS_SC(1);
  else if (D.G <= 2) HILS_SC(2);
  else if (D.G <= 4) HILS_SC(4);
  else if (D.G <= 8) HILS_SC(8);
  else HILS_SC(16);
#undef HILS_SC
  return cudaGetLastError();
}

cudaError_t launch_select_scores(const Dims& D, bool bf16, const void* qc, const void* klm,
                                 const float* blm, const int32_t* idx, float* s_sel,
                                 cudaStream_t st) {
  if (D.B * D.Hkv * D.N_q == 0 || D.K == 0) return cudaSuccess;
  if (bf16 && D.G <= 8 && (D.d == 64 || D.d == 128))
    return D.d == 128 ? launch_scores_bf16_d<128>(D, qc, klm, blm, idx, s_sel, st)
                      : launch_scores_bf16_d<64>(D, qc, klm, blm, idx, s_sel, st);
  return bf16 ? launch_scores_g<__nv_bfloat16>(D, qc, klm, blm, idx, s_sel, st)
              : launch_scores_g<float>(D, qc, klm, blm, idx, s_sel, st);
}

constexpr int kSplitThreads = 256;
constexpr int kSplitWarps = kSplitThreads / 32;

template <typename T, int D_, int GM, int KM>
__global__ void __launch_bounds__(kSplitThreads) select_split_kernel(
    Dims D, int cps, int n_split, const T* __restrict__ qc, const T* __restrict__ klm,
    const float* __restrict__ blm, float* __restrict__ part_v, int32_t* __restrict__ part_c) {
  using SS = SplitShape<T, D_, GM>;
  extern __shared__ __align__(16) float sig_buf[];   // [cps] scores, then [warps][K] lists
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int split = blockIdx.x;
  const int64_t row = blockIdx.y;
  const int64_t i = row % D.N_q, bg = row / D.N_q, g = bg % D.Hkv, b = bg / D.Hkv;
  const int G = D.G, K = D.K;
  const int64_t n = n_eligible(D.q_pos0 + i, D.S, D.W);
  const int64_t c0 = (int64_t)split * cps;
  const int64_t c1 = c0 + cps < n ? c0 + cps : n;
  const int cnt = c1 > c0 ? (int)(c1 - c0) : 0;

  // this lane's slice of every head's calibrated query, in registers
  const int grp = lane / SS::L, gl = lane % SS::L;
  float qreg[GM][SS::DPL];
#pragma unroll
  for (int h = 0; h < GM; ++h) {
#pragma unroll
    for (int v = 0; v < SS::NV; ++v) {
      float t[SS::VEC];
      if (h < G) {
        load_vec<T, SS::VEC>(qc + (((b * D.Hq) + g * G + h) * D.N_q + i) * D_ +
                                 (v * SS::L + gl) * SS::VEC, t);
      } else {
#pragma unroll
        for (int e = 0; e < SS::VEC; ++e) t[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < SS::VEC; ++e) qreg[h][v * SS::VEC + e] = t[e];
    }
  }

  const T* kb = klm + bg * D.C * D_;
  const float* bb = blm + bg * D.C;
  constexpr int U = 2;   // warp steps in flight per iteration
  for (int base = warp * SS::RPW; base < cnt; base += kSplitWarps * SS::RPW * U) {
    float kv[U][SS::DPL];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int r = base + u * kSplitWarps * SS::RPW + grp;
      if (r < cnt) {
        const T* kr = kb + (c0 + r) * D_;
#pragma unroll
        for (int v = 0; v < SS::NV; ++v) {
          float t[SS::VEC];
          load_vec<T, SS::VEC>(kr + (v * SS::L + gl) * SS::VEC, t);
#pragma unroll
          for (int e = 0; e < SS::VEC; ++e) kv[u][v * SS::VEC + e] = t[e];
        }
      } else {
#pragma unroll
        for (int e = 0; e < SS::DPL; ++e) kv[u][e] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int r = base + u * kSplitWarps * SS::RPW + grp;
      float acc[GM];
#pragma unroll
      for (int h = 0; h < GM; ++h) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < SS::DPL; ++e) a = fmaf(qreg[h][e], kv[u][e], a);
        acc[h] = a;
      }
#pragma unroll
      for (int o = SS::L / 2; o > 0; o >>= 1) {
#pragma unroll
        for (int h = 0; h < GM; ++h) acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], o);
      }
      if (gl == 0 && r < cnt) {
        const float bc = bb[c0 + r];
        float sig = -INFINITY;
#pragma unroll
        for (int h = 0; h < GM; ++h)
          if (h < G) sig = fmaxf(sig, fmaf(acc[h], D.scale, bc));
        sig_buf[r] = sig;
      }
    }
  }
  __syncthreads();

  // top-K of this split: per-lane lists, warp merge, then one warp merges the warps' lists
  TopList<KM> Ls;
  Ls.clear();
  for (int r = threadIdx.x; r < cnt; r += kSplitThreads) Ls.insert(sig_buf[r], (int)(c0 + r), K);
  float wv;
  int wc;
  warp_merge_topk<KM>(Ls, K, lane, wv, wc);
  __syncthreads();   // sig_buf is reused below
  float* lv = sig_buf;                                           // [warps][K]
  int* lc = reinterpret_cast<int*>(sig_buf + kSplitWarps * kMaxK);
  if (lane < K) { lv[warp * K + lane] = wv; lc[warp * K + lane] = wc; }
  __syncthreads();
  if (warp == 0) {
    int ptr = 0;
    float* outv = part_v + (row * n_split + split) * K;
    int32_t* outc = part_c + (row * n_split + split) * K;
    for (int r = 0; r < K; ++r) {
      float v = -INFINITY;
      int c = INT_MAX;
      if (lane < kSplitWarps && ptr < K) { v = lv[lane * K + ptr]; c = lc[lane * K + ptr]; }
      float bv = v;
      int bc = c;
      warp_best(bv, bc);
      if (lane < kSplitWarps && c == bc && bc != INT_MAX) ++ptr;
      if (lane == 0) { outv[r] = bv; outc[r] = bc; }
    }
  }
}

template <typename T, int GM, int KM>
__global__ void __launch_bounds__(128) select_merge_kernel(Dims D, int n_split,
                                                           const float* __restrict__ part_v,
                                                           const int32_t* __restrict__ part_c,
                                                           const T* __restrict__ qc,
                                                           const T* __restrict__ klm,
                                                           const float* __restrict__ blm,
                                                           int32_t* __restrict__ idx,
                                                           float* __restrict__ s_sel) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t rows = D.B * D.Hkv * D.N_q;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= rows) return;
  const int64_t i = row % D.N_q, bg = row / D.N_q, g = bg % D.Hkv, b = bg / D.Hkv;
  const int K = D.K;
  TopList<KM> L;
  L.clear();
  const int total = n_split * K;
  for (int e = lane; e < total; e += 32)
    L.insert(part_v[row * total + e], part_c[row * total + e], K);
  float wv;
  int wc;
  warp_merge_topk<KM>(L, K, lane, wv, wc);
  write_selection<T, GM>(D, b, g, i, nullptr, qc, klm + bg * D.C * D.d, blm + bg * D.C, lane,
                         wc, idx, s_sel);
}

// ---------------------------------------------------------------------------------------------
// Decode, streaming form.  select_stream_kernel reads every eligible landmark row of a query
// exactly once (coalesced 16-byte loads, several rows in flight per lane group) and writes the
// group score sigma_c = max_h s_{h,c} to a scratch row; select_topk_row_kernel then selects the K
// best of each row and computes the per-head scores of the winners.  The scratch write is
// 4 bytes per landmark row read (d * 2 bytes), under 2% extra traffic for d = 128.
constexpr int kStreamWarps = 4;                          // consumer warps
constexpr int kStreamThreads = (kStreamWarps + 1) * 32;  // + one producer warp
constexpr int kStreamStages = 4;
constexpr int kStreamStageRows = 64;

template <typename T, int D_, int GM>
__global__ void __launch_bounds__(kStreamThreads) select_stream_kernel(
    Dims D, int cps, int64_t n_stride, const T* __restrict__ qc, const T* __restrict__ klm,
    const float* __restrict__ blm, float* __restrict__ sigma, int32_t* __restrict__ status) {
  using SS = SplitShape<T, D_, GM>;
  extern __shared__ __align__(128) uint8_t sm_stream[];
  T* ring = reinterpret_cast<T*>(sm_stream);   // [kStreamStages][kStreamStageRows][D_]
  __shared__ uint64_t full[kStreamStages], empty[kStreamStages];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int split = blockIdx.x;
  const int64_t row = blockIdx.y;
  const int64_t i = row % D.N_q, bg = row / D.N_q, g = bg % D.Hkv, b = bg / D.Hkv;
  const int G = D.G;
  const int64_t n = n_eligible(D.q_pos0 + i, D.S, D.W);
  const int64_t c0 = (int64_t)split * cps;
  const int64_t c1 = c0 + cps < n ? c0 + cps : n;
  const int cnt = c1 > c0 ? (int)(c1 - c0) : 0;
  if (cnt == 0) return;
  const int n_stages = (cnt + kStreamStageRows - 1) / kStreamStageRows;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStreamStages; ++s) {
      sm100::mbar_init(&full[s], 1);
      sm100::mbar_init(&empty[s], kStreamWarps);
    }
    sm100::fence_barrier_init();
  }
  __syncthreads();
  const T* src = klm + (bg * D.C + c0) * D_;
  if (warp == kStreamWarps) {
    // producer warp: keeps up to kStreamStages bulk copies of landmark rows in flight
    if (lane == 0) {
      for (int t = 0; t < n_stages; ++t) {
        const int s = t % kStreamStages;
        const uint32_t u = (uint32_t)(t / kStreamStages);
        if (!sm100::mbar_wait(&empty[s], (u & 1u) ^ 1u, 1u << 24)) {
          record_status(status, kStatusTimeout);
          break;
        }
        const int r0 = t * kStreamStageRows;
        const int rows_here = cnt - r0 < kStreamStageRows ? cnt - r0 : kStreamStageRows;
        const uint32_t bytes = (uint32_t)rows_here * D_ * sizeof(T);
        sm100::mbar_expect_tx(&full[s], bytes);
        sm100::bulk_load(ring + (size_t)s * kStreamStageRows * D_, src + (int64_t)r0 * D_, bytes,
                         &full[s]);
      }
    }
    return;
  }
  // consumer warps: this lane's slice of every head's calibrated query stays in registers
  const int grp = lane / SS::L, gl = lane % SS::L;
  float qreg[GM][SS::DPL];
#pragma unroll
  for (int h = 0; h < GM; ++h) {
#pragma unroll
    for (int v = 0; v < SS::NV; ++v) {
      float t[SS::VEC];
      if (h < G) {
        load_vec<T, SS::VEC>(qc + (((b * D.Hq) + g * G + h) * D.N_q + i) * D_ +
                                 (v * SS::L + gl) * SS::VEC, t);
      } else {
#pragma unroll
        for (int e = 0; e < SS::VEC; ++e) t[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < SS::VEC; ++e) qreg[h][v * SS::VEC + e] = t[e];
    }
  }
  const float* bb = blm + bg * D.C + c0;
  float* out = sigma + row * n_stride + c0;
  constexpr int STEP = kStreamWarps * SS::RPW;
  constexpr int PER_STAGE = (kStreamStageRows + STEP - 1) / STEP;   // row-steps per warp
  for (int t = 0; t < n_stages; ++t) {
    const int s = t % kStreamStages;
    const uint32_t u = (uint32_t)(t / kStreamStages);
    const int r0 = t * kStreamStageRows;
    const int rows_here = cnt - r0 < kStreamStageRows ? cnt - r0 : kStreamStageRows;
    // landmark biases of this warp's rows, requested before waiting for the rows themselves
    float bias[PER_STAGE];
#pragma unroll
    for (int k = 0; k < PER_STAGE; ++k) {
      const int r = warp * SS::RPW + k * STEP + grp;
      bias[k] = r < rows_here ? __ldg(bb + r0 + r) : 0.f;
    }
    if (!sm100::mbar_wait(&full[s], u & 1u, 1u << 24)) {
      record_status(status, kStatusTimeout);
      break;
    }
    const T* stage = ring + (size_t)s * kStreamStageRows * D_;
#pragma unroll
    for (int k = 0; k < PER_STAGE; ++k) {
      const int base = warp * SS::RPW + k * STEP;
      if (base >= rows_here) break;
      const int r = base + grp;
      float kv[SS::DPL];
      if (r < rows_here) {
        const T* kr = stage + (size_t)r * D_;
#pragma unroll
        for (int v = 0; v < SS::NV; ++v) {
          float tv[SS::VEC];
          load_vec_shared<T, SS::VEC>(kr + (v * SS::L + gl) * SS::VEC, tv);
#pragma unroll
          for (int e = 0; e < SS::VEC; ++e) kv[v * SS::VEC + e] = tv[e];
        }
      } else {
#pragma unroll
        for (int e = 0; e < SS::DPL; ++e) kv[e] = 0.f;
      }
      float acc[GM];
#pragma unroll
      for (int h = 0; h < GM; ++h) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < SS::DPL; ++e) a = fmaf(qreg[h][e], kv[e], a);
        acc[h] = a;
      }
#pragma unroll
      for (int o = SS::L / 2; o > 0; o >>= 1)
#pragma unroll
        for (int h = 0; h < GM; ++h) acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], o);
      if (gl == 0 && r < rows_here) {
        const float bc = bias[k];
        float sig = -INFINITY;
#pragma unroll
        for (int h = 0; h < GM; ++h)
          if (h < G) sig = fmaxf(sig, fmaf(acc[h], D.scale, bc));
        out[r0 + r] = sig;
      }
    }
    __syncwarp();
    if (lane == 0) sm100::mbar_arrive(&empty[s]);
  }
}

// Decode top-K of one query row's group scores, one 128-thread CTA per (b, g, query); warp w
// takes the w-th quarter of the row.
//   1. every lane takes the best (value, chunk) of its share: 32 lane maxima per warp;
//   2. each warp sorts its maxima (bitonic network over shuffles); the K-th of them is a lower
//      bound of its quarter's K-th best, so the largest of the four, theta, is a lower bound of
//      the row's K-th best;
//   3. every candidate >= theta is appended to a shared list (ballot compaction; typically a
//      few dozen);
//   4. warp 0 takes the exact top-K of that list -- one bitonic sort when it holds at most 64,
//      register lists and a warp merge otherwise -- and writes idx and the per-head scores.  If
//      a warp has more candidates than its quarter of kSurvivorCap (many ties at theta), step 4
//      runs over the whole row instead (slower, same result).
// With the streaming scorer's group maxima (gmax: the max of each 32 consecutive chunks), steps
// 1 and 3 read far less: the lane maxima are taken over group maxima (each group max is a
// chunk's score, so theta stays a lower bound of the row's K-th best, now as a value, every tie
// passing; a row of at most 256 groups is read whole by every warp, for a tighter theta), and
// step 3 reads only the groups whose maximum reaches theta, which hold every candidate.
constexpr int kTopkWarps = 4;
constexpr int kTopkThreads = 32 * kTopkWarps;
constexpr int kSurvivorCap = 1024;
constexpr int kTopkBatch = 8;

// ascending-by-`better` position: true if (v, c) should come before (ov, oc)
__device__ __forceinline__ void cmpx(float& v, int& c, int partner_lane_xor, bool keep_better) {
  const float ov = __shfl_xor_sync(0xffffffffu, v, partner_lane_xor);
  const int oc = __shfl_xor_sync(0xffffffffu, c, partner_lane_xor);
  const bool other_better = better(ov, oc, v, c);
  if (keep_better == other_better) { v = ov; c = oc; }
}

// Sorts one (value, chunk) per lane, best first (lane 0 = best).
__device__ __forceinline__ void warp_sort_best_first(float& v, int& c, int lane) {
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const bool up = ((lane & size) == 0);          // this 'size' block sorts best-first
      const bool lower = ((lane & stride) == 0);     // lower index of the compared pair
      cmpx(v, c, stride, up == lower);
    }
  }
}

template <typename T, int D_, int GM, int KM>
__global__ void __launch_bounds__(kTopkThreads) select_topk_row_kernel(
    Dims D, int64_t n_stride, const float* __restrict__ sigma, const T* __restrict__ qc,
    const T* __restrict__ klm, const float* __restrict__ blm, int32_t* __restrict__ idx,
    float* __restrict__ s_sel, const float* __restrict__ gmax, int64_t g_stride) {
  __shared__ float sv[kSurvivorCap];
  __shared__ int scn[kSurvivorCap];
  __shared__ float th_v[kTopkWarps];
  __shared__ int th_c[kTopkWarps];
  __shared__ int wcnt[kTopkWarps];   // survivors per warp
  __shared__ __align__(16) __nv_bfloat16 qsh[GM * D_];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t row = blockIdx.x;
  const int64_t i = row % D.N_q, bg = row / D.N_q, g = bg % D.Hkv, b = bg / D.Hkv;
  const int K = D.K;
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    // the group's calibrated queries for the winners' per-head scores, staged now so that their
    // loads overlap the selection (visible to warp 0 after the barrier below)
    constexpr int NV = D_ / 8;
    for (int e = threadIdx.x; e < D.G * NV; e += kTopkThreads) {
      const int h = e / NV, j = e - h * NV;
      const int64_t hrow = ((b * D.Hq) + g * D.G + h) * D.N_q + i;
      reinterpret_cast<uint4*>(qsh)[h * NV + j] =
          __ldg(reinterpret_cast<const uint4*>(qc + hrow * D_) + j);
    }
  }
  const int64_t n = n_eligible(D.q_pos0 + i, D.S, D.W);
  const float* sr = sigma + row * n_stride;             // 16-byte aligned (n_stride % 4 == 0)
  const int64_t n4 = n >> 2;
  // this warp's quarter of the row's float4 vectors (the scalar tail goes to the last warp)
  const int64_t w0 = n4 * warp / kTopkWarps, w1 = n4 * (warp + 1) / kTopkWarps;
  // with group maxima: this warp's quarter of the row's groups of 32 chunks
  const float* gr = gmax ? gmax + row * g_stride : nullptr;
  const int64_t n_g = (n + 31) >> 5;
  const int64_t g0 = n_g * warp / kTopkWarps, g1 = n_g * (warp + 1) / kTopkWarps;
  // 1. lane maxima (a lane's chunks come in increasing order: a strict compare keeps the lower
  //    index on ties; over group maxima the chunk stays unknown, INT_MAX)
  float mv = -INFINITY;
  int mc = INT_MAX;
  // (a row of at most 32 * kTopkBatch groups is read whole by every warp, one round per lane:
  // each lane's maximum then covers four times as many chunks, and theta, the same in every
  // warp, is that much tighter)
  const bool whole = n_g <= 32 * kTopkBatch;
  const int64_t p0 = whole ? 0 : g0, p1 = whole ? n_g : g1;
  for (int64_t q0 = p0; gr && q0 < p1; q0 += 32 * kTopkBatch) {
    float t[kTopkBatch];
#pragma unroll
    for (int u = 0; u < kTopkBatch; ++u) {
      const int64_t gi = q0 + u * 32 + lane;
      t[u] = gi < p1 ? __ldg(gr + gi) : -INFINITY;
    }
#pragma unroll
    for (int u = 0; u < kTopkBatch; ++u) mv = fmaxf(mv, t[u]);
  }
  for (int64_t q0 = w0; !gr && q0 < w1; q0 += 32 * kTopkBatch) {
    float4 t[kTopkBatch];
#pragma unroll
    for (int u = 0; u < kTopkBatch; ++u) {
      const int64_t q4 = q0 + u * 32 + lane;
      t[u] = q4 < w1 ? __ldg(reinterpret_cast<const float4*>(sr) + q4)
                     : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    }
#pragma unroll
    for (int u = 0; u < kTopkBatch; ++u) {
      const int c = (int)((q0 + u * 32 + lane) * 4);
      if (t[u].x > mv) { mv = t[u].x; mc = c; }
      if (t[u].y > mv) { mv = t[u].y; mc = c + 1; }
      if (t[u].z > mv) { mv = t[u].z; mc = c + 2; }
      if (t[u].w > mv) { mv = t[u].w; mc = c + 3; }
    }
  }
  if (!gr && warp == kTopkWarps - 1) {
    for (int64_t c = n4 * 4 + lane; c < n; c += 32) {
      const float v = __ldg(sr + c);
      if (better(v, (int)c, mv, mc)) { mv = v; mc = (int)c; }
    }
  }
  // 2. theta = the best of the warps' K-th lane maxima
  {
    float v = mv;
    int c = mc;
    warp_sort_best_first(v, c, lane);
    const int kk = K < 32 ? K : 32;
    const float tv = __shfl_sync(0xffffffffu, v, kk - 1);
    const int tcc = __shfl_sync(0xffffffffu, c, kk - 1);
    if (lane == 0) { th_v[warp] = tv; th_c[warp] = tcc; }
  }
  __syncthreads();
  float tv = th_v[0];
  int tcc = th_c[0];
#pragma unroll
  for (int w = 1; w < kTopkWarps; ++w)
    if (better(th_v[w], th_c[w], tv, tcc)) { tv = th_v[w]; tcc = th_c[w]; }
  // 3. survivors: candidates not worse than theta, compacted in ballot order per warp batch
  const unsigned lt = (1u << lane) - 1u;
  // each warp appends to its own region of the list: a ballot and a prefix count, no atomics
  constexpr int kCapW = kSurvivorCap / kTopkWarps;
  float* svw = sv + warp * kCapW;
  int* scw = scn + warp * kCapW;
  int ns_w = 0;   // warp-uniform
  auto append = [&](bool keep, float v, int c) {
    const unsigned m = __ballot_sync(0xffffffffu, keep);
    const int pos = ns_w + __popc(m & lt);
    if (keep && pos < kCapW) { svw[pos] = v; scw[pos] = c; }
    ns_w += __popc(m);
  };
  // over group maxima: 32 groups per round; the chunks of up to 8 groups that reach theta are
  // loaded together (one per lane each, in chunk order), then appended
  for (int64_t gb = g0; gr && gb < g1; gb += 32) {
    // (lanes past the warp's groups never flag: with theta = -inf they would pass the compare
    // and pull in another warp's groups)
    const bool in = gb + lane < g1;
    const float gm = in ? __ldg(gr + gb + lane) : -INFINITY;
    unsigned m = __ballot_sync(0xffffffffu, in && gm >= tv);
    while (m) {
      int gs[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        gs[k] = m ? __ffs(m) - 1 : -1;
        m &= m - 1u;
      }
      float v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int64_t c = (gb + gs[k]) * 32 + lane;
        v[k] = gs[k] >= 0 && c < n ? __ldg(sr + c) : -INFINITY;
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if (gs[k] < 0) break;   // (warp-uniform)
        const int64_t c = (gb + gs[k]) * 32 + lane;
        append(c < n && !better(tv, tcc, v[k], (int)c), v[k], (int)c);
      }
    }
  }
  for (int64_t q0 = w0; !gr && q0 < w1; q0 += 32 * kTopkBatch) {
    float4 t[kTopkBatch];
#pragma unroll
    for (int u = 0; u < kTopkBatch; ++u) {
      const int64_t q4 = q0 + u * 32 + lane;
      t[u] = q4 < w1 ? __ldg(reinterpret_cast<const float4*>(sr) + q4)
                     : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    }
#pragma unroll
    for (int u = 0; u < kTopkBatch; ++u) {
      const int64_t q4 = q0 + u * 32 + lane;
      const bool in = q4 < w1;
      const int c = (int)(q4 * 4);
      const bool k0 = in && !better(tv, tcc, t[u].x, c);
      const bool k1 = in && !better(tv, tcc, t[u].y, c + 1);
      const bool k2 = in && !better(tv, tcc, t[u].z, c + 2);
      const bool k3 = in && !better(tv, tcc, t[u].w, c + 3);
      // most of a row is below theta: skip the compaction when no lane keeps anything
      if (!__any_sync(0xffffffffu, k0 || k1 || k2 || k3)) continue;
      append(k0, t[u].x, c);
      append(k1, t[u].y, c + 1);
      append(k2, t[u].z, c + 2);
      append(k3, t[u].w, c + 3);
    }
  }
  if (!gr && warp == kTopkWarps - 1) {
    for (int64_t c0 = n4 * 4; c0 < n; c0 += 32) {
      const int64_t c = c0 + lane;
      const float v = c < n ? __ldg(sr + c) : -INFINITY;
      append(c < n && !better(tv, tcc, v, (int)c), v, (int)c);
    }
  }
  if (lane == 0) wcnt[warp] = ns_w;
  __syncthreads();
  if (warp != 0) return;
  int cnt[kTopkWarps], ns = 0;
  bool overflow = false;
#pragma unroll
  for (int w = 0; w < kTopkWarps; ++w) {
    cnt[w] = wcnt[w];
    overflow |= cnt[w] > kCapW;
    ns += cnt[w];
  }
  // survivor e of the concatenated warp regions
  auto survivor = [&](int e, float& v, int& c) {
    v = -INFINITY;
    c = INT_MAX;
#pragma unroll
    for (int w = 0; w < kTopkWarps; ++w) {
      if (e >= 0 && e < cnt[w]) { v = sv[w * kCapW + e]; c = scn[w * kCapW + e]; }
      e -= cnt[w];
    }
  };
  // 4. exact top-K of the survivors (or of every candidate if too many tied at theta)
  float wv;
  int wc;
  if (!overflow && ns <= 64) {
    // one bitonic sort of up to 64 survivors, two per lane (elements lane and lane + 32)
    float va, vb;
    int ca, cb;
    survivor(lane, va, ca);
    survivor(lane + 32, vb, cb);
#pragma unroll
    for (int size = 2; size <= 64; size <<= 1) {
#pragma unroll
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        if (stride == 32) {
          // elements lane and lane + 32, both in blocks sorted best first
          if (better(vb, cb, va, ca)) {
            const float tv2 = va; va = vb; vb = tv2;
            const int tc2 = ca; ca = cb; cb = tc2;
          }
        } else {
          const bool lower = (lane & stride) == 0;
          cmpx(va, ca, stride, ((lane & size) == 0) == lower);
          cmpx(vb, cb, stride, (((lane + 32) & size) == 0) == lower);
        }
      }
    }
    wv = lane < K ? va : -INFINITY;
    wc = lane < K ? ca : INT_MAX;
  } else {
    TopList<KM> L;
    L.clear();
    if (!overflow) {
      for (int e = lane; e < ns; e += 32) {
        float v;
        int c;
        survivor(e, v, c);
        L.insert(v, c, K);
      }
    } else {
      for (int64_t c = lane; c < n; c += 32) L.insert(__ldg(sr + c), (int)c, K);
    }
    warp_merge_topk<KM>(L, K, lane, wv, wc);
  }
  if constexpr (std::is_same<T, __nv_bfloat16>::value)
    write_selection_wide<D_, GM>(D, b, g, i, qsh, qc, klm + bg * D.C * D_, blm + bg * D.C, lane,
                                 wc, idx, s_sel, /*q_staged=*/true);
  else
    write_selection<T, GM>(D, b, g, i, nullptr, qc, klm + bg * D.C * D.d, blm + bg * D.C, lane,
                           wc, idx, s_sel);
}

template <typename T, int D_, int GM, int KM>
struct TopkRowRun {
  static cudaError_t run(const Dims* D, int64_t n_stride, const float* sigma, const void* qc,
                         const void* klm, const float* blm, int32_t* idx, float* s_sel,
                         const float* gmax, int64_t g_stride, cudaStream_t st) {
    const int64_t rows = D->B * D->Hkv * D->N_q;
    select_topk_row_kernel<T, D_, GM, KM><<<(unsigned)rows, kTopkThreads, 0, st>>>(
        *D, n_stride, sigma, (const T*)qc, (const T*)klm, blm, idx, s_sel, gmax, g_stride);
    return cudaGetLastError();
  }
};

// ---------------------------------------------------------------------------------------------
// Host-side launchers.

template <typename T, int GM, int KM>
static cudaError_t launch_rows_t(const Dims& D, const void* qc, const void* klm, const float* blm,
                                 int32_t* idx, float* s_sel, cudaStream_t st) {
  const int per_warp = D.G * (int)D.d * (int)sizeof(float);
  int warps = 49152 / per_warp;
  if (warps > 8) warps = 8;
  if (warps < 1) warps = 1;
  const int64_t rows = D.B * D.Hkv * D.N_q;
  const int64_t blocks = (rows + warps - 1) / warps;
  select_rows_kernel<T, GM, KM><<<(unsigned)blocks, warps * 32, (size_t)warps * per_warp, st>>>(
      D, (const T*)qc, (const T*)klm, blm, idx, s_sel);
  return cudaGetLastError();
}

template <typename T, int GM>
static cudaError_t launch_rows_k(const Dims& D, const void* qc, const void* klm, const float* blm,
                                 int32_t* idx, float* s_sel, cudaStream_t st) {
  if (D.K <= 8) return launch_rows_t<T, GM, 8>(D, qc, klm, blm, idx, s_sel, st);
  if (D.K <= 16) return launch_rows_t<T, GM, 16>(D, qc, klm, blm, idx, s_sel, st);
  return launch_rows_t<T, GM, 32>(D, qc, klm, blm, idx, s_sel, st);
}

template <typename T>
static cudaError_t launch_rows_g(const Dims& D, const void* qc, const void* klm, const float* blm,
                                 int32_t* idx, float* s_sel, cudaStream_t st) {
  if (D.G <= 1) return launch_rows_k<T, 1>(D, qc, klm, blm, idx, s_sel, st);
  if (D.G <= 2) return launch_rows_k<T, 2>(D, qc, klm, blm, idx, s_sel, st);
  if (D.G <= 4) return launch_rows_k<T, 4>(D, qc, klm, blm, idx, s_sel, st);
  if (D.G <= 8) return launch_rows_k<T, 8>(D, qc, klm, blm, idx, s_sel, st);
  return launch_rows_k<T, 16>(D, qc, klm, blm, idx, s_sel, st);
}

cudaError_t launch_select_rows(const Dims& D, bool bf16, const void* qc, const void* klm,
                               const float* blm, int32_t* idx, float* s_sel, cudaStream_t st) {
  if (D.B * D.Hkv * D.N_q == 0) return cudaSuccess;
  return bf16 ? launch_rows_g<__nv_bfloat16>(D, qc, klm, blm, idx, s_sel, st)
              : launch_rows_g<float>(D, qc, klm, blm, idx, s_sel, st);
}

size_t split_smem_bytes(int cps) {
  size_t a = (size_t)cps * sizeof(float);
  size_t b = (size_t)kSplitWarps * kMaxK * (sizeof(float) + sizeof(int));
  return a > b ? a : b;
}

template <typename T, int D_, int GM, int KM>
static cudaError_t launch_split_t(const Dims& D, int cps, int n_split, const void* qc,
                                  const void* klm, const float* blm, float* pv, int32_t* pc,
                                  cudaStream_t st) {
  const int64_t rows = D.B * D.Hkv * D.N_q;
  const size_t smem = split_smem_bytes(cps);
  auto kern = select_split_kernel<T, D_, GM, KM>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid((unsigned)n_split, (unsigned)rows);
  kern<<<grid, kSplitThreads, smem, st>>>(D, cps, n_split, (const T*)qc, (const T*)klm, blm, pv,
                                          pc);
  return cudaGetLastError();
}

template <typename T, int GM, int KM>
static cudaError_t launch_merge_t(const Dims& D, int n_split, const float* pv, const int32_t* pc,
                                  const void* qc, const void* klm, const float* blm, int32_t* idx,
                                  float* s_sel, cudaStream_t st) {
  const int64_t rows = D.B * D.Hkv * D.N_q;
  select_merge_kernel<T, GM, KM><<<(unsigned)((rows + 3) / 4), 128, 0, st>>>(
      D, n_split, pv, pc, (const T*)qc, (const T*)klm, blm, idx, s_sel);
  return cudaGetLastError();
}

// Dispatch on (dtype, d, group size, list length) for a callable templated on them.
template <template <typename, int, int, int> class F, typename... A>
static cudaError_t dispatch_tdgk(bool bf16, int64_t d, int G, int K, A... a) {
#define HILS_K(T, D_, GM)                                         \
  if (K <= 8) return F<T, D_, GM, 8>::run(a...);                  \
  if (K <= 16) return F<T, D_, GM, 16>::run(a...);                \
  return F<T, D_, GM, 32>::run(a...);
#define HILS_G(T, D_)                                             \
  if (G <= 4) { HILS_K(T, D_, 4) }                                \
  if (G <= 8) { HILS_K(T, D_, 8) }                                \
  HILS_K(T, D_, 16)
  if (bf16) {
    if (d == 128) { HILS_G(__nv_bfloat16, 128) }
    HILS_G(__nv_bfloat16, 64)
  }
  if (d == 128) { HILS_G(float, 128) }
  HILS_G(float, 64)
#undef HILS_G
#undef HILS_K
}

template <typename T, int D_, int GM, int KM>
struct SplitRun {
  static cudaError_t run(const Dims* D, int cps, int n_split, const void* qc, const void* klm,
                         const float* blm, float* pv, int32_t* pc, cudaStream_t st) {
    return launch_split_t<T, D_, GM, KM>(*D, cps, n_split, qc, klm, blm, pv, pc, st);
  }
};

template <typename T, int D_, int GM, int KM>
struct MergeRun {
  static cudaError_t run(const Dims* D, int n_split, const float* pv, const int32_t* pc,
                         const void* qc, const void* klm, const float* blm, int32_t* idx,
                         float* s_sel, cudaStream_t st) {
    return launch_merge_t<T, GM, KM>(*D, n_split, pv, pc, qc, klm, blm, idx, s_sel, st);
  }
};

cudaError_t launch_select_split(const Dims& D, bool bf16, int cps, int n_split, const void* qc,
                                const void* klm, const float* blm, float* part_v,
                                int32_t* part_c, cudaStream_t st) {
  if (D.B * D.Hkv * D.N_q == 0) return cudaSuccess;
  return dispatch_tdgk<SplitRun>(bf16, D.d, D.G, D.K, &D, cps, n_split, qc, klm, blm, part_v,
                                 part_c, st);
}

cudaError_t launch_select_merge(const Dims& D, bool bf16, int n_split, const float* part_v,
                                const int32_t* part_c, const void* qc, const void* klm,
                                const float* blm, int32_t* idx, float* s_sel, cudaStream_t st) {
  if (D.B * D.Hkv * D.N_q == 0) return cudaSuccess;
  return dispatch_tdgk<MergeRun>(bf16, D.d, D.G, D.K, &D, n_split, part_v, part_c, qc, klm, blm,
                                 idx, s_sel, st);
}

template <typename T, int D_, int GM, int KM>
struct StreamOnly {
  static cudaError_t run(const Dims* D, int cps, int n_split, int64_t n_stride, const void* qc,
                         const void* klm, const float* blm, float* sigma, int32_t* status,
                         cudaStream_t st) {
    const int64_t rows = D->B * D->Hkv * D->N_q;
    dim3 grid((unsigned)n_split, (unsigned)rows);
    const size_t smem = (size_t)kStreamStages * kStreamStageRows * D_ * sizeof(T);
    cudaError_t e = cudaFuncSetAttribute(select_stream_kernel<T, D_, GM>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // many small CTAs per SM keep many bulk copies in flight: ask for the largest carveout
    e = cudaFuncSetAttribute(select_stream_kernel<T, D_, GM>,
                             cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    select_stream_kernel<T, D_, GM><<<grid, kStreamThreads, smem, st>>>(
        *D, cps, n_stride, (const T*)qc, (const T*)klm, blm, sigma, status);
    return cudaGetLastError();
  }
};

cudaError_t launch_select_stream(const Dims& D, bool bf16, int cps, int n_split,
                                 int64_t n_stride, const void* qc, const void* klm,
                                 const float* blm, float* sigma, int32_t* status,
                                 cudaStream_t st) {
  if (D.B * D.Hkv * D.N_q == 0) return cudaSuccess;
  return dispatch_tdgk<StreamOnly>(bf16, D.d, D.G, D.K, &D, cps, n_split, n_stride, qc, klm,
                                   blm, sigma, status, st);
}

cudaError_t launch_select_topk_row(const Dims& D, bool bf16, int64_t n_stride,
                                   const float* sigma, const void* qc, const void* klm,
                                   const float* blm, int32_t* idx, float* s_sel, cudaStream_t st,
                                   const float* gmax, int64_t g_stride) {
  if (D.B * D.Hkv * D.N_q == 0) return cudaSuccess;
  return dispatch_tdgk<TopkRowRun>(bf16, D.d, D.G, D.K, &D, n_stride, sigma, qc, klm, blm, idx,
                                   s_sel, gmax, g_stride, st);
}

}  // namespace hils
