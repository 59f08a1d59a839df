// Landmark construction, the producer of step 1's inputs: for every (b, g) and completed chunk c
// (tokens cS .. cS+S-1),
//   x_j = scale * q_lm[b,g,c] . K[b,g,cS+j],   p = softmax_j(x),
//   k_lm[b,g,c] = sum_j p_j K[b,g,cS+j],        b_lm[b,g,c] = H(p) = -sum_j p_j ln p_j
// ([Reader] "The HiLS-Attention Mechanism": the chunk summary is the landmark query's
// attention-weighted sum of the chunk's keys and its bias the entropy of those weights; [Reader]
// "Paper Primer": the surrogate is a first-order expansion of the chunk's log-mass, so with the
// same scale as step 1 the surrogate score at q_lm equals the chunk's exact log-mass).
//
// HBM-bound: every key is read once (S*d elements per chunk) and one row is written.  One warp
// per chunk; the lanes split a key row into 4-element pieces (d/4 lanes per key, so d = 64 runs
// two keys per warp step), each lane keeps its dims of the weighted sum.  Keys are read straight
// from global memory, NB per batch so that every lane has NB loads in flight; the softmax is
// taken online (running max, rescale once per batch) so the chunk is read a single time, and the
// entropy follows from the same pass as ln Z - sum_j p_j x_j.
#include "common.cuh"
#include "kernels.h"

namespace hils {
namespace {

constexpr int kLmWarps = 8;       // chunks per CTA
constexpr int kLmBatch = 8;       // keys per lane group in flight
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <typename T>
__device__ __forceinline__ void load4(const T* p, float (&v)[4]) {
  Elem<T>::load4(p, v);
}

// Chunks c0 .. c0+nc-1 of every (b, g); the landmark query of chunk c0 + cc of plane bg is row
// bg * qlm_rows + cc of qlm.
template <typename T, int DD>
__global__ void __launch_bounds__(32 * kLmWarps)
    landmarks_kernel(Dims D, int64_t c0, int64_t nc, int64_t qlm_rows,
                     const T* __restrict__ qlm, const T* __restrict__ K, T* __restrict__ klm,
                     float* __restrict__ blm) {
  constexpr int LPK = DD / 4;     // lanes per key row (4 elements each)
  constexpr int PAR = 32 / LPK;   // keys per warp step
  static_assert(DD >= 16 && DD <= 128 && (DD & (DD - 1)) == 0, "head dims 16, 32, 64, 128");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * kLmWarps + warp;   // over B * Hkv * nc
  if (item >= D.B * D.Hkv * nc) return;   // (no block-wide barrier below)
  const int64_t bg = item / nc, cc = item - bg * nc;
  const int64_t c = c0 + cc;
  const int64_t chunk = bg * D.C + c;   // the landmark's row
  const int grp = lane / LPK, sl = lane % LPK;   // key group, 4-element slice of the row
  const int dim = sl * 4;
  float q[4];
  load4(qlm + (bg * qlm_rows + cc) * DD + dim, q);
  // logits in base 2: y = x * log2(e)
  const float qs = D.scale * kLog2e;
#pragma unroll
  for (int e = 0; e < 4; ++e) q[e] *= qs;
  const T* kb = K + (bg * D.N_kv + c * (int64_t)D.S) * DD;
  float m = -INFINITY, z = 0.f, sx = 0.f;   // running max (base 2), sum of 2^(y-m), sum of 2^(y-m) y
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int j0 = 0; j0 < D.S; j0 += PAR * kLmBatch) {
    float kv[kLmBatch][4];
    float y[kLmBatch];
#pragma unroll
    for (int u = 0; u < kLmBatch; ++u) {
      const int j = j0 + u * PAR + grp;
      if (j < D.S) {
        load4(kb + (int64_t)j * DD + dim, kv[u]);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) kv[u][e] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < kLmBatch; ++u) {
      float s = q[0] * kv[u][0];
      s = fmaf(q[1], kv[u][1], s);
      s = fmaf(q[2], kv[u][2], s);
      s = fmaf(q[3], kv[u][3], s);
#pragma unroll
      for (int o = LPK / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      y[u] = (j0 + u * PAR + grp) < D.S ? s : -INFINITY;
    }
    float bm = y[0];
#pragma unroll
    for (int u = 1; u < kLmBatch; ++u) bm = fmaxf(bm, y[u]);
    if (bm > m) {   // (uniform within a key group) new running max: rescale once per batch
      const float f = exp2f(m - bm);
      z *= f;
      sx *= f;
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[e] *= f;
      m = bm;
    }
#pragma unroll
    for (int u = 0; u < kLmBatch; ++u) {
      // a key past the chunk (y = -inf) weighs 0, also while the group has seen no key
      const bool in = y[u] != -INFINITY;
      const float w = in ? exp2f(y[u] - m) : 0.f;
      z += w;
      sx = fmaf(w, in ? y[u] : 0.f, sx);
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[e] = fmaf(w, kv[u][e], acc[e]);
    }
  }
  // merge the PAR key groups' states (d = 64: two groups of 16 lanes)
#pragma unroll
  for (int o = LPK; o < 32; o <<= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float z2 = __shfl_xor_sync(0xffffffffu, z, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, sx, o);
    float a2[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) a2[e] = __shfl_xor_sync(0xffffffffu, acc[e], o);
    const float mm = fmaxf(m, m2);
    const float f1 = m == -INFINITY ? 0.f : exp2f(m - mm);
    const float f2 = m2 == -INFINITY ? 0.f : exp2f(m2 - mm);
    z = z * f1 + z2 * f2;
    sx = sx * f1 + s2 * f2;
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] = acc[e] * f1 + a2[e] * f2;
    m = mm;
  }
  // k_lm = sum_j p_j K_j; H(p) = ln Z - sum_j p_j x_j with ln Z = (m + log2 z) ln 2
  const float inv = 1.f / z;
  if (grp == 0) {
    float o4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) o4[e] = acc[e] * inv;
    Elem<T>::store4(klm + chunk * DD + dim, o4);
  }
  if (lane == 0) blm[chunk] = fmaxf((m + log2f(z) - sx * inv) * kLn2, 0.f);
}

}  // namespace

cudaError_t launch_landmarks(const Dims& D, bool bf16, int64_t c0, int64_t nc,
                             int64_t qlm_rows, const void* qlm, const void* K, void* klm,
                             float* blm, cudaStream_t st) {
  const int64_t n = D.B * D.Hkv * nc;
  if (n == 0) return cudaSuccess;
  const dim3 grid((unsigned)((n + kLmWarps - 1) / kLmWarps));
#define HILS_LM(TT, DDV)                                                                      \
  landmarks_kernel<TT, DDV><<<grid, 32 * kLmWarps, 0, st>>>(                                  \
      D, c0, nc, qlm_rows, static_cast<const TT*>(qlm), static_cast<const TT*>(K),            \
      static_cast<TT*>(klm), blm)
  if (bf16) {
    if (D.d == 128) HILS_LM(__nv_bfloat16, 128);
    else if (D.d == 64) HILS_LM(__nv_bfloat16, 64);
    else if (D.d == 32) HILS_LM(__nv_bfloat16, 32);
    else if (D.d == 16) HILS_LM(__nv_bfloat16, 16);
    else return cudaErrorInvalidValue;
  } else {
    if (D.d == 128) HILS_LM(float, 128);
    else if (D.d == 64) HILS_LM(float, 64);
    else if (D.d == 32) HILS_LM(float, 32);
    else if (D.d == 16) HILS_LM(float, 16);
    else return cudaErrorInvalidValue;
  }
#undef HILS_LM
  return cudaGetLastError();
}

}  // namespace hils

namespace hils {
namespace {

// K[b, g, pos] = k_new[b, g] and V[b, g, pos] = v_new[b, g]: one 16-byte piece per thread.
template <typename T>
__global__ void __launch_bounds__(256)
    append_kv_kernel(Dims D, int64_t pos, const T* __restrict__ k_new,
                     const T* __restrict__ v_new, T* __restrict__ K, T* __restrict__ V) {
  constexpr int U = 16 / (int)sizeof(T);          // elements per 16-byte piece
  const int64_t pieces = D.d / U;                 // per row
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= 2 * D.B * D.Hkv * pieces) return;
  const int64_t kv = e / (D.B * D.Hkv * pieces), r = e - kv * D.B * D.Hkv * pieces;
  const int64_t bg = r / pieces, u = r - bg * pieces;
  const T* src = (kv == 0 ? k_new : v_new) + bg * D.d + u * U;
  T* dst = (kv == 0 ? K : V) + (bg * D.N_kv + pos) * D.d + u * U;
  *reinterpret_cast<uint4*>(dst) = __ldg(reinterpret_cast<const uint4*>(src));
}

}  // namespace

cudaError_t launch_append_kv(const Dims& D, bool bf16, int64_t pos, const void* k_new,
                             const void* v_new, void* K, void* V, cudaStream_t st) {
  const int64_t n = 2 * D.B * D.Hkv * D.d / (bf16 ? 8 : 4);
  if (n == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((n + 255) / 256);
  if (bf16)
    append_kv_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
        D, pos, static_cast<const __nv_bfloat16*>(k_new), static_cast<const __nv_bfloat16*>(v_new),
        static_cast<__nv_bfloat16*>(K), static_cast<__nv_bfloat16*>(V));
  else
    append_kv_kernel<float><<<grid, 256, 0, st>>>(D, pos, static_cast<const float*>(k_new),
                                                  static_cast<const float*>(v_new),
                                                  static_cast<float*>(K), static_cast<float*>(V));
  return cudaGetLastError();
}

}  // namespace hils
