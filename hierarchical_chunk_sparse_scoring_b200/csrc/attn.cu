// Steps 3-4 on CUDA cores.
//
// Step 3: exact softmax attention of the token query inside each selected chunk and inside the
// local window, one (o_u, lse_u) per unit ([Reader] Fig. 3 caption: the intra-chunk softmax
// spreads a chunk's mass over its tokens; [Abstract]: each query attends independently with
// each retrieved chunk).  Step 4: the units are fused with softmax weights over their scores,
// the chunk's surrogate s_{h,c} for a chunk and the exact log-sum-exp for the window ([Reader]
// Fig. 3 caption: inter-chunk softmax; [Abstract]: fused according to chunk retrieval scores).
//
//   attn_rows_kernel   one warp per (b, h, query): all units in turn, fused online; can also
//                      emit the per-unit (o, lse).  Any d <= 128, fp32 or bf16.
//   attn_units_kernel  one CTA per (b, g, query, unit) for all G heads of the group, so a chunk's
//                      K/V rows are read once per group; the window is cut into pieces of S
//                      tokens.  Used for decode.
//   fuse_units_kernel  one warp per (b, h, query): combines chunk units and window pieces.
#include "common.cuh"
#include "kernels.h"

namespace hils {

template <typename T>
__global__ void __launch_bounds__(128) attn_rows_kernel(Dims D, const T* __restrict__ q,
                                                        const T* __restrict__ Kc,
                                                        const T* __restrict__ Vc,
                                                        const int32_t* __restrict__ idx,
                                                        const float* __restrict__ s_sel,
                                                        T* __restrict__ out,
                                                        float* __restrict__ lse_out,
                                                        float* __restrict__ unit_o,
                                                        float* __restrict__ unit_lse) {
  __shared__ __align__(16) float qsm[4][kMaxD];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t rows = D.B * D.Hq * D.N_q;
  const int64_t row = (int64_t)blockIdx.x * 4 + warp;
  if (row >= rows) return;
  const int64_t i = row % D.N_q, bh = row / D.N_q, h = bh % D.Hq, b = bh / D.Hq;
  const int64_t g = h / D.G;
  const int d = (int)D.d, K = D.K;
  for (int k = lane; k < d; k += 32) qsm[warp][k] = Elem<T>::to_f(q[row * d + k]);
  __syncwarp();
  const int64_t pos = D.q_pos0 + i;
  const int64_t n = n_eligible(pos, D.S, D.W);
  const int64_t ell = (int64_t)D.S * n;
  const T* Kb = Kc + (b * D.Hkv + g) * D.N_kv * d;
  const T* Vb = Vc + (b * D.Hkv + g) * D.N_kv * d;
  const int32_t* ib = idx + ((b * D.Hkv + g) * D.N_q + i) * K;
  const bool has_dims = lane * 4 < d;
  const bool fuse = out != nullptr;

  float M = -INFINITY, Z = 0.f, Oa[4] = {0.f, 0.f, 0.f, 0.f};
  for (int u = 0; u <= K; ++u) {
    int64_t t0, t1;
    float score = 0.f;
    if (u < K) {
      const int c = ib[u];
      if (c < 0 || c >= n) {   // empty slot, or an id that is not an eligible chunk
        if (unit_o && has_dims) {
          const float z[4] = {0.f, 0.f, 0.f, 0.f};
          Elem<float>::store4(unit_o + (row * (K + 1) + u) * d + lane * 4, z);
        }
        if (unit_lse && lane == 0) unit_lse[row * (K + 1) + u] = -INFINITY;
        continue;
      }
      t0 = (int64_t)c * D.S;
      t1 = t0 + D.S;
      score = s_sel ? s_sel[row * K + u] : 0.f;
    } else {
      t0 = ell;
      t1 = pos + 1;
    }
    float m = -INFINITY, l = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
    for (int64_t j0 = t0; j0 < t1; j0 += 32) {
      const int64_t j = j0 + lane;
      float x = -INFINITY;
      if (j < t1) {
        const T* kr = Kb + j * d;
        float acc = 0.f;
        for (int k = 0; k < d; k += 4) {
          float kv[4];
          Elem<T>::load4(kr + k, kv);
          const float4 qv = *reinterpret_cast<const float4*>(&qsm[warp][k]);
          acc = fmaf(qv.x, kv[0], acc);
          acc = fmaf(qv.y, kv[1], acc);
          acc = fmaf(qv.z, kv[2], acc);
          acc = fmaf(qv.w, kv[3], acc);
        }
        x = acc * D.scale;
      }
      const float mn = fmaxf(m, warp_max(x));
      const float corr = (m == -INFINITY) ? 0.f : expf(m - mn);
      const float p = (j < t1) ? expf(x - mn) : 0.f;
      l = l * corr + warp_sum(p);
#pragma unroll
      for (int e = 0; e < 4; ++e) o[e] *= corr;
      const int cnt = (int)((t1 - j0) < 32 ? (t1 - j0) : 32);
      for (int t = 0; t < cnt; ++t) {
        const float pt = __shfl_sync(0xffffffffu, p, t);
        if (has_dims) {
          float vv[4];
          Elem<T>::load4(Vb + (j0 + t) * d + lane * 4, vv);
#pragma unroll
          for (int e = 0; e < 4; ++e) o[e] = fmaf(pt, vv[e], o[e]);
        }
      }
      m = mn;
    }
    const float lse_u = m + logf(l);
    const float inv = 1.f / l;
#pragma unroll
    for (int e = 0; e < 4; ++e) o[e] *= inv;
    if (unit_o && has_dims) Elem<float>::store4(unit_o + (row * (K + 1) + u) * d + lane * 4, o);
    if (unit_lse && lane == 0) unit_lse[row * (K + 1) + u] = lse_u;
    if (fuse) {
      const float sc = (u < K) ? score : lse_u;
      if (sc != -INFINITY) {
        const float Mn = fmaxf(M, sc);
        const float a = (M == -INFINITY) ? 0.f : expf(M - Mn);
        const float w = expf(sc - Mn);
#pragma unroll
        for (int e = 0; e < 4; ++e) Oa[e] = Oa[e] * a + w * o[e];
        Z = Z * a + w;
        M = Mn;
      }
    }
  }
  if (fuse) {
    const float inv = 1.f / Z;
    float r[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) r[e] = Oa[e] * inv;
    if (has_dims) Elem<T>::store4(out + row * d + lane * 4, r);
    if (lse_out && lane == 0) lse_out[row] = M + logf(Z);
  }
}

// ---------------------------------------------------------------------------------------------
constexpr int kUnitThreads = 128;
constexpr int kUnitTile = 32;   // tokens per smem tile

template <typename T>
__global__ void __launch_bounds__(kUnitThreads) attn_units_kernel(
    Dims D, int n_pieces, const T* __restrict__ q, const T* __restrict__ Kc,
    const T* __restrict__ Vc, const int32_t* __restrict__ idx, float* __restrict__ part_o,
    float* __restrict__ part_lse) {
  extern __shared__ __align__(16) float sm[];
  const int d = (int)D.d, G = D.G, K = D.K;
  const int dp = d + 4;                                  // padded row (floats)
  float* qf = sm;                                        // [G][d]
  float* Ks = qf + G * d;                                // [tile][dp]
  float* Vs = Ks + kUnitTile * dp;                       // [tile][dp]
  float* xs = Vs + kUnitTile * dp;                       // [G][tile]
  float* mst = xs + G * kUnitTile;                       // [G] running max
  float* lst = mst + G;                                  // [G] running sum
  float* cst = lst + G;                                  // [G] rescale of this tile

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int unit = blockIdx.x;
  const int64_t row = blockIdx.y;                        // (b, g, i)
  const int64_t i = row % D.N_q, bg = row / D.N_q, g = bg % D.Hkv, b = bg / D.Hkv;
  const int NU = K + n_pieces;
  const int64_t pos = D.q_pos0 + i;
  const int64_t n = n_eligible(pos, D.S, D.W);
  const int64_t ell = (int64_t)D.S * n;
  int64_t t0 = 0, t1 = 0;
  if (unit < K) {
    const int c = idx[row * K + unit];
    if (c >= 0 && c < n) { t0 = (int64_t)c * D.S; t1 = t0 + D.S; }
  } else {
    t0 = ell + (int64_t)(unit - K) * D.S;
    t1 = t0 + D.S < pos + 1 ? t0 + D.S : pos + 1;
    if (t1 < t0) t1 = t0;
  }
  const int64_t hrow0 = (b * D.Hq + g * G) * D.N_q + i;   // head g*G, stride N_q per head

  for (int e = tid; e < G * d; e += kUnitThreads) {
    const int hh = e / d, k = e - hh * d;
    qf[e] = Elem<T>::to_f(q[(hrow0 + (int64_t)hh * D.N_q) * d + k]);
  }
  if (tid < G) { mst[tid] = -INFINITY; lst[tid] = 0.f; }
  const T* Kb = Kc + bg * D.N_kv * d;
  const T* Vb = Vc + bg * D.N_kv * d;

  // this thread's (head, dim) outputs: pairs tid, tid + 128, ...
  constexpr int kMaxPairs = 16 * kMaxD / kUnitThreads;
  float acc[kMaxPairs];
#pragma unroll
  for (int r = 0; r < kMaxPairs; ++r) acc[r] = 0.f;
  const int n_pairs = G * d;

  for (int64_t j0 = t0; j0 < t1; j0 += kUnitTile) {
    const int cnt = (int)(t1 - j0 < kUnitTile ? t1 - j0 : kUnitTile);
    __syncthreads();   // previous tile fully consumed; qf / stats initialised
    for (int e = tid * 4; e < kUnitTile * d; e += kUnitThreads * 4) {
      const int t = e / d, k = e - t * d;
      float kv[4] = {0.f, 0.f, 0.f, 0.f}, vv[4] = {0.f, 0.f, 0.f, 0.f};
      if (t < cnt) {
        Elem<T>::load4(Kb + (j0 + t) * d + k, kv);
        Elem<T>::load4(Vb + (j0 + t) * d + k, vv);
      }
      Elem<float>::store4(Ks + t * dp + k, kv);
      Elem<float>::store4(Vs + t * dp + k, vv);
    }
    __syncthreads();
    for (int pr = tid; pr < G * kUnitTile; pr += kUnitThreads) {
      const int hh = pr / kUnitTile, t = pr - hh * kUnitTile;
      float x = -INFINITY;
      if (t < cnt) {
        const float* kr = Ks + t * dp;
        const float* qr = qf + hh * d;
        float a = 0.f;
        for (int k = 0; k < d; k += 4) {
          const float4 kv = *reinterpret_cast<const float4*>(kr + k);
          const float4 qv = *reinterpret_cast<const float4*>(qr + k);
          a = fmaf(qv.x, kv.x, a);
          a = fmaf(qv.y, kv.y, a);
          a = fmaf(qv.z, kv.z, a);
          a = fmaf(qv.w, kv.w, a);
        }
        x = a * D.scale;
      }
      xs[pr] = x;
    }
    __syncthreads();
    // online softmax statistics, one warp per head (kUnitTile == 32)
    for (int hh = warp; hh < G; hh += kUnitThreads / 32) {
      const float x = xs[hh * kUnitTile + lane];
      const float m_old = mst[hh];
      const float mn = fmaxf(m_old, warp_max(x));
      const float p = (x == -INFINITY) ? 0.f : expf(x - mn);
      const float s = warp_sum(p);
      xs[hh * kUnitTile + lane] = p;
      if (lane == 0) {
        const float corr = (m_old == -INFINITY) ? 0.f : expf(m_old - mn);
        cst[hh] = corr;
        lst[hh] = lst[hh] * corr + s;
        mst[hh] = mn;
      }
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kMaxPairs; ++r) {
      const int pr = tid + r * kUnitThreads;
      if (pr < n_pairs) {
        const int hh = pr / d, k = pr - hh * d;
        float a = acc[r] * cst[hh];
        const float* pp = xs + hh * kUnitTile;
        for (int t = 0; t < cnt; ++t) a = fmaf(pp[t], Vs[t * dp + k], a);
        acc[r] = a;
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kMaxPairs; ++r) {
    const int pr = tid + r * kUnitThreads;
    if (pr < n_pairs) {
      const int hh = pr / d, k = pr - hh * d;
      const float l = lst[hh];
      const float v = l > 0.f ? acc[r] / l : 0.f;
      part_o[((hrow0 + (int64_t)hh * D.N_q) * NU + unit) * d + k] = v;
    }
  }
  if (tid < G) {
    const float l = lst[tid];
    part_lse[(hrow0 + (int64_t)tid * D.N_q) * NU + unit] = l > 0.f ? mst[tid] + logf(l) : -INFINITY;
  }
}

// Fusion of K chunk units (scores s_sel) and n_pieces window pieces (scores = their lse, whose
// log-sum-exp is the window's lse).  Units with score -inf get weight 0.
template <typename T>
__global__ void __launch_bounds__(128) fuse_units_kernel(Dims D, int n_pieces,
                                                         const float* __restrict__ s_sel,
                                                         const float* __restrict__ part_o,
                                                         const float* __restrict__ part_lse,
                                                         T* __restrict__ out,
                                                         float* __restrict__ lse_out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t rows = D.B * D.Hq * D.N_q;
  const int64_t row = (int64_t)blockIdx.x * 4 + warp;
  if (row >= rows) return;
  const int K = D.K, NU = K + n_pieces, d = (int)D.d;
  auto score_of = [&](int u) -> float {
    return u < K ? s_sel[row * K + u] : part_lse[row * NU + u];
  };
  float M = -INFINITY;
  for (int u = lane; u < NU; u += 32) M = fmaxf(M, score_of(u));
  M = warp_max(M);
  float Z = 0.f;
  for (int u = lane; u < NU; u += 32) {
    const float s = score_of(u);
    Z += (s == -INFINITY) ? 0.f : expf(s - M);
  }
  Z = warp_sum(Z);
  const float invZ = 1.f / Z;
  for (int k0 = lane * 4; k0 < d; k0 += 128) {
    float o[4] = {0.f, 0.f, 0.f, 0.f};
    for (int u = 0; u < NU; ++u) {
      const float s = score_of(u);
      if (s == -INFINITY) continue;
      const float w = expf(s - M) * invZ;
      float v[4];
      Elem<float>::load4(part_o + (row * NU + u) * d + k0, v);
#pragma unroll
      for (int e = 0; e < 4; ++e) o[e] = fmaf(w, v[e], o[e]);
    }
    Elem<T>::store4(out + row * d + k0, o);
  }
  if (lse_out && lane == 0) lse_out[row] = M + logf(Z);
}

// ---------------------------------------------------------------------------------------------
cudaError_t launch_attn_rows(const Dims& D, bool bf16, const void* q, const void* K,
                             const void* V, const int32_t* idx, const float* s_sel, void* out,
                             float* lse, float* unit_o, float* unit_lse, cudaStream_t st) {
  const int64_t rows = D.B * D.Hq * D.N_q;
  if (rows == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((rows + 3) / 4);
  if (bf16)
    attn_rows_kernel<__nv_bfloat16><<<blocks, 128, 0, st>>>(
        D, (const __nv_bfloat16*)q, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, idx, s_sel,
        (__nv_bfloat16*)out, lse, unit_o, unit_lse);
  else
    attn_rows_kernel<float><<<blocks, 128, 0, st>>>(D, (const float*)q, (const float*)K,
                                                     (const float*)V, idx, s_sel, (float*)out,
                                                     lse, unit_o, unit_lse);
  return cudaGetLastError();
}

size_t units_smem_bytes(const Dims& D) {
  const size_t dp = (size_t)D.d + 4;
  return sizeof(float) * ((size_t)D.G * D.d + 2 * kUnitTile * dp + (size_t)D.G * kUnitTile +
                          3 * (size_t)D.G);
}

cudaError_t launch_attn_units(const Dims& D, bool bf16, int n_pieces, const void* q,
                              const void* K, const void* V, const int32_t* idx, float* part_o,
                              float* part_lse, cudaStream_t st) {
  const int64_t rows = D.B * D.Hkv * D.N_q;
  if (rows == 0) return cudaSuccess;
  const size_t smem = units_smem_bytes(D);
  dim3 grid((unsigned)(D.K + n_pieces), (unsigned)rows);
  if (bf16) {
    auto k = attn_units_kernel<__nv_bfloat16>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, kUnitThreads, smem, st>>>(D, n_pieces, (const __nv_bfloat16*)q,
                                        (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, idx,
                                        part_o, part_lse);
  } else {
    auto k = attn_units_kernel<float>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    k<<<grid, kUnitThreads, smem, st>>>(D, n_pieces, (const float*)q, (const float*)K,
                                        (const float*)V, idx, part_o, part_lse);
  }
  return cudaGetLastError();
}

cudaError_t launch_fuse_units(const Dims& D, bool bf16, int n_pieces, const float* s_sel,
                              const float* part_o, const float* part_lse, void* out, float* lse,
                              cudaStream_t st) {
  const int64_t rows = D.B * D.Hq * D.N_q;
  if (rows == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((rows + 3) / 4);
  if (bf16)
    fuse_units_kernel<__nv_bfloat16><<<blocks, 128, 0, st>>>(D, n_pieces, s_sel, part_o, part_lse,
                                                             (__nv_bfloat16*)out, lse);
  else
    fuse_units_kernel<float><<<blocks, 128, 0, st>>>(D, n_pieces, s_sel, part_o, part_lse,
                                                     (float*)out, lse);
  return cudaGetLastError();
}

}  // namespace hils
