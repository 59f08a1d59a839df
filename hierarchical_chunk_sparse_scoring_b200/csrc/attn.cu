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
#include "sm100.cuh"

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
// Decode units.  One CTA per (b, g, query, unit) serves all G heads of the group, so each K/V row
// of the unit is read from memory once.  Per tile of up to 64 tokens the K and V rows (contiguous
// in memory) arrive by two bulk copies into shared memory; then L lanes share a token row, lane
// l holding d/L of its dimensions (the grouping of the decode selection): pass 1 computes the
// G x 64 logits, the tile's softmax statistics update the running (m, l) per head, pass 2
// accumulates p * V into per-lane partial outputs, reduced across lane groups and warps at the
// end.
constexpr int kUnitThreads = 128;
constexpr int kUnitWarps = kUnitThreads / 32;
constexpr int kUnitTile = 64;   // tokens per tile

// Lane grouping of the unit kernel: 8 dims per lane (4 for 16 heads), so that both the group's
// query slice and its output accumulators stay in registers.
template <typename T, int D_, int GM>
struct UnitShape {
  static constexpr int DPL = GM <= 8 ? 8 : 4;
  static constexpr int L = D_ / DPL;
  static constexpr int VEC = (16 / (int)sizeof(T)) < DPL ? (16 / (int)sizeof(T)) : DPL;
  static constexpr int NV = DPL / VEC;
  static constexpr int RPW = 32 / L;
  static_assert(L >= 1 && L <= 32 && (32 % L) == 0, "lane grouping");
};

// Fusion of K chunk units (scores s_sel) and n_pieces window pieces (scores = their lse, whose
// log-sum-exp is the window's lse).  Units with score -inf get weight 0.  One warp per
// (b, h, query) row: the lanes first hold the units' weights, then sweep d with the weights
// broadcast, loading several units' vectors before accumulating them.
template <typename T>
__device__ __forceinline__ void fuse_row(const Dims& D, int n_pieces, int64_t row, int lane,
                                         const float* __restrict__ s_sel,
                                         const float* __restrict__ part_o,
                                         const float* __restrict__ part_lse, T* __restrict__ out,
                                         float* __restrict__ lse_out) {
  const int K = D.K, NU = K + n_pieces, d = (int)D.d;
  // L2-coherent loads: inside the units kernel the partials come from other CTAs of the same
  // launch, which the read-only path does not promise to see
  auto score_of = [&](int u) -> float {
    return u < K ? __ldcg(s_sel + row * K + u) : __ldcg(part_lse + row * NU + u);
  };
  auto load4cg = [](const float* p, float (&v)[4]) {
    const float4 t = __ldcg(reinterpret_cast<const float4*>(p));
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
  };
  const float* pr = part_o + row * NU * d;
  if (NU <= 64 && d == 128) {
    // lanes hold the weights of units lane and lane + 32 (scores read once); every lane reads its
    // 4 output columns of all units, 32 loads in flight per batch (two rounds for up to 64
    // units), the first batch issued before the score loads so that both are in flight together
    float v[32][4];
    auto load_batch = [&](int u0) {
#pragma unroll
      for (int e2 = 0; e2 < 32; ++e2) {
        if (u0 + e2 < NU) {
          load4cg(pr + (int64_t)(u0 + e2) * 128 + lane * 4, v[e2]);
        } else {
          v[e2][0] = v[e2][1] = v[e2][2] = v[e2][3] = 0.f;
        }
      }
    };
    load_batch(0);
    const float s0 = lane < NU ? score_of(lane) : -INFINITY;
    const float s1 = lane + 32 < NU ? score_of(lane + 32) : -INFINITY;
    const float M = warp_max(fmaxf(s0, s1));
    const float e0 = s0 == -INFINITY ? 0.f : __expf(s0 - M);
    const float e1 = s1 == -INFINITY ? 0.f : __expf(s1 - M);
    const float Z = warp_sum(e0 + e1);
    const float w0 = e0 / Z, w1 = e1 / Z;
    float o[4] = {0.f, 0.f, 0.f, 0.f};
    for (int u0 = 0; u0 < NU; u0 += 32) {
      if (u0 > 0) load_batch(u0);
      const float wsrc = u0 < 32 ? w0 : w1;   // batch 0: units 0-31, batch 1: units 32-63
#pragma unroll
      for (int e2 = 0; e2 < 32; ++e2) {
        const float w = __shfl_sync(0xffffffffu, wsrc, e2);
#pragma unroll
        for (int x = 0; x < 4; ++x) o[x] = fmaf(w, v[e2][x], o[x]);
      }
    }
    Elem<T>::store4(out + row * 128 + lane * 4, o);
    if (lse_out && lane == 0) lse_out[row] = M + logf(Z);
    return;
  }
  float M = -INFINITY;
  for (int u = lane; u < NU; u += 32) M = fmaxf(M, score_of(u));
  M = warp_max(M);
  float Z = 0.f;
  for (int u = lane; u < NU; u += 32) {
    const float s = score_of(u);
    Z += (s == -INFINITY) ? 0.f : __expf(s - M);
  }
  Z = warp_sum(Z);
  const float invZ = 1.f / Z;
  // every lane runs every iteration (the loop body shuffles); lanes past d only skip memory
  for (int kb = 0; kb < d; kb += 128) {
    const int k0 = kb + lane * 4;
    const bool act = k0 < d;
    float o[4] = {0.f, 0.f, 0.f, 0.f};
    for (int ub = 0; ub < NU; ub += 32) {
      const int um = ub + lane;
      const float su = um < NU ? score_of(um) : -INFINITY;
      const float wl = su == -INFINITY ? 0.f : __expf(su - M) * invZ;   // lane's unit weight
      const int cnt = NU - ub < 32 ? NU - ub : 32;
      for (int u8 = 0; u8 < cnt; u8 += 8) {
        float v[8][4];
        float w[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          w[e] = __shfl_sync(0xffffffffu, wl, (u8 + e) & 31);
          if (u8 + e < cnt && act) {
            load4cg(pr + (int64_t)(ub + u8 + e) * d + k0, v[e]);
          } else {
            w[e] = 0.f;
            v[e][0] = v[e][1] = v[e][2] = v[e][3] = 0.f;
          }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e)
#pragma unroll
          for (int x = 0; x < 4; ++x) o[x] = fmaf(w[e], v[e][x], o[x]);
      }
    }
    if (act) Elem<T>::store4(out + row * d + k0, o);
  }
  if (lse_out && lane == 0) lse_out[row] = M + logf(Z);
}

template <typename T, int D_, int GM>
__global__ void __launch_bounds__(kUnitThreads) attn_units_kernel(
    Dims D, int n_pieces, const T* __restrict__ q, const T* __restrict__ Kc,
    const T* __restrict__ Vc, const int32_t* __restrict__ idx, float* __restrict__ part_o,
    float* __restrict__ part_lse, int32_t* __restrict__ status) {
  using SS = UnitShape<T, D_, GM>;
  extern __shared__ __align__(128) uint8_t sm_units[];
  T* Ks = reinterpret_cast<T*>(sm_units);                       // [64][D_]
  T* Vs = Ks + kUnitTile * D_;                                   // [64][D_]
  float* red = reinterpret_cast<float*>(Vs + kUnitTile * D_);    // [warps][GM*D_/4]
  __shared__ float xs[GM][kUnitTile];
  __shared__ float mst[GM], lst[GM], cst[GM];
  __shared__ uint64_t full;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int unit = blockIdx.x;
  const int64_t row = blockIdx.y;                        // (b, g, i)
  const int64_t i = row % D.N_q, bg = row / D.N_q, g = bg % D.Hkv, b = bg / D.Hkv;
  const int G = D.G, K = D.K;
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
  const int64_t hrow0 = (b * D.Hq + g * G) * D.N_q + i;   // head g*G; stride N_q per head
  if (tid == 0) {
    sm100::mbar_init(&full, 1);
    sm100::fence_barrier_init();
  }
  if (tid < GM) { mst[tid] = -INFINITY; lst[tid] = 0.f; cst[tid] = 1.f; }
  __syncthreads();
  const int grp = lane / SS::L, gl = lane % SS::L;
  float qreg[GM][SS::DPL];
#pragma unroll
  for (int h = 0; h < GM; ++h) {
#pragma unroll
    for (int v = 0; v < SS::NV; ++v) {
      float t[SS::VEC];
      if (h < G) {
        load_vec<T, SS::VEC>(q + (hrow0 + (int64_t)h * D.N_q) * D_ + (v * SS::L + gl) * SS::VEC, t);
      } else {
#pragma unroll
        for (int e = 0; e < SS::VEC; ++e) t[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < SS::VEC; ++e) qreg[h][v * SS::VEC + e] = t[e];
    }
  }
  const T* Kb = Kc + bg * D.N_kv * D_;
  const T* Vb = Vc + bg * D.N_kv * D_;
  constexpr int TPW = kUnitTile / kUnitWarps;            // tokens per warp per tile (16)
  constexpr int STEPS = TPW / SS::RPW;
  float oacc[GM][SS::DPL];
#pragma unroll
  for (int h = 0; h < GM; ++h)
#pragma unroll
    for (int e = 0; e < SS::DPL; ++e) oacc[h][e] = 0.f;

  uint32_t phase = 0;
  bool ok = true;
  for (int64_t j0 = t0; j0 < t1; j0 += kUnitTile) {
    const int cnt = (int)(t1 - j0 < kUnitTile ? t1 - j0 : kUnitTile);
    if (tid == 0) {
      const uint32_t bytes = (uint32_t)cnt * D_ * sizeof(T);
      sm100::mbar_expect_tx(&full, 2 * bytes);
      sm100::bulk_load(Ks, Kb + j0 * D_, bytes, &full);
      sm100::bulk_load(Vs, Vb + j0 * D_, bytes, &full);
    }
    const bool landed = sm100::mbar_wait(&full, phase, 1u << 24);
    phase ^= 1u;
    if (!__syncthreads_and(landed)) { ok = false; break; }
    // pass 1: logits of this warp's tokens
#pragma unroll
    for (int st = 0; st < STEPS; ++st) {
      const int tk = warp * TPW + st * SS::RPW + grp;
      float kv[SS::DPL];
      if (tk < cnt) {
#pragma unroll
        for (int v = 0; v < SS::NV; ++v) {
          float t[SS::VEC];
          load_vec_shared<T, SS::VEC>(Ks + tk * D_ + (v * SS::L + gl) * SS::VEC, t);
#pragma unroll
          for (int e = 0; e < SS::VEC; ++e) kv[v * SS::VEC + e] = t[e];
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
      if (gl == 0) {
#pragma unroll
        for (int h = 0; h < GM; ++h) xs[h][tk] = tk < cnt ? acc[h] * D.scale : -INFINITY;
      }
    }
    __syncthreads();
    // softmax statistics of the tile, one warp per head
    for (int h = warp; h < G; h += kUnitWarps) {
      const float x0 = xs[h][lane], x1 = xs[h][lane + 32];
      const float m_old = mst[h];
      const float mn = fmaxf(m_old, warp_max(fmaxf(x0, x1)));
      const float p0 = x0 == -INFINITY ? 0.f : __expf(x0 - mn);
      const float p1 = x1 == -INFINITY ? 0.f : __expf(x1 - mn);
      const float sum = warp_sum(p0 + p1);
      xs[h][lane] = p0;
      xs[h][lane + 32] = p1;
      if (lane == 0) {
        const float corr = m_old == -INFINITY ? 0.f : __expf(m_old - mn);
        cst[h] = corr;
        lst[h] = lst[h] * corr + sum;
        mst[h] = mn;
      }
    }
    __syncthreads();
    // pass 2: p * V for this warp's tokens
#pragma unroll
    for (int h = 0; h < GM; ++h) {
      const float cr = h < G ? cst[h] : 1.f;
#pragma unroll
      for (int e = 0; e < SS::DPL; ++e) oacc[h][e] *= cr;
    }
#pragma unroll
    for (int st = 0; st < STEPS; ++st) {
      const int tk = warp * TPW + st * SS::RPW + grp;
      if (tk < cnt) {
        float vv[SS::DPL];
#pragma unroll
        for (int v = 0; v < SS::NV; ++v) {
          float t[SS::VEC];
          load_vec_shared<T, SS::VEC>(Vs + tk * D_ + (v * SS::L + gl) * SS::VEC, t);
#pragma unroll
          for (int e = 0; e < SS::VEC; ++e) vv[v * SS::VEC + e] = t[e];
        }
#pragma unroll
        for (int h = 0; h < GM; ++h) {
          const float pv = h < G ? xs[h][tk] : 0.f;
#pragma unroll
          for (int e = 0; e < SS::DPL; ++e) oacc[h][e] = fmaf(pv, vv[e], oacc[h][e]);
        }
      }
    }
    __syncthreads();   // Ks / Vs / xs / cst are rewritten by the next tile
  }
  if (!ok && tid == 0) record_status(status, kStatusTimeout);
  // reduce partial outputs: across the lane groups of a warp, then across warps
#pragma unroll
  for (int o = SS::L; o < 32; o <<= 1)
#pragma unroll
    for (int h = 0; h < GM; ++h)
#pragma unroll
      for (int e = 0; e < SS::DPL; ++e) oacc[h][e] += __shfl_xor_sync(0xffffffffu, oacc[h][e], o);
  constexpr int QUARTER = GM * D_ / 4;
#pragma unroll
  for (int qq = 0; qq < 4; ++qq) {
    if (grp == 0) {
#pragma unroll
      for (int h = 0; h < GM; ++h)
#pragma unroll
        for (int v = 0; v < SS::NV; ++v)
#pragma unroll
          for (int e = 0; e < SS::VEC; ++e) {
            const int flat = h * D_ + (v * SS::L + gl) * SS::VEC + e;
            if (flat / QUARTER == qq)
              red[warp * QUARTER + flat - qq * QUARTER] = oacc[h][v * SS::VEC + e];
          }
    }
    __syncthreads();
    for (int f = tid; f < QUARTER; f += kUnitThreads) {
      const int flat = qq * QUARTER + f;
      const int h = flat / D_, k = flat - h * D_;
      if (h < G) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < kUnitWarps; ++w) sum += red[w * QUARTER + f];
        const float l = lst[h];
        part_o[((hrow0 + (int64_t)h * D.N_q) * NU + unit) * D_ + k] = l > 0.f ? sum / l : 0.f;
      }
    }
    __syncthreads();
  }
  if (tid < G) {
    const float l = lst[tid];
    part_lse[(hrow0 + (int64_t)tid * D.N_q) * NU + unit] =
        l > 0.f ? mst[tid] + logf(l) : -INFINITY;
  }
}

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
  fuse_row<T>(D, n_pieces, row, lane, s_sel, part_o, part_lse, out, lse_out);
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


template <typename T, int D_>
static cudaError_t launch_units_d(const Dims& D, int n_pieces, const void* q, const void* K,
                                  const void* V, const int32_t* idx, float* part_o,
                                  float* part_lse, int32_t* status, cudaStream_t st) {
  dim3 grid((unsigned)(D.K + n_pieces), (unsigned)(D.B * D.Hkv * D.N_q));
#define HILS_UNITS(GM)                                                                        \
  do {                                                                                        \
    const size_t smem = 2 * kUnitTile * D_ * sizeof(T) +                                     \
                        (size_t)kUnitWarps * GM * D_ / 4 * sizeof(float);                    \
    cudaError_t e = cudaFuncSetAttribute(attn_units_kernel<T, D_, GM>,                        \
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,         \
                                         (int)smem);                                          \
    if (e != cudaSuccess) return e;                                                           \
    e = cudaFuncSetAttribute(attn_units_kernel<T, D_, GM>,                                    \
                             cudaFuncAttributePreferredSharedMemoryCarveout,                  \
                             cudaSharedmemCarveoutMaxShared);                                 \
    if (e != cudaSuccess) return e;                                                           \
    attn_units_kernel<T, D_, GM><<<grid, kUnitThreads, smem, st>>>(                           \
        D, n_pieces, (const T*)q, (const T*)K, (const T*)V, idx, part_o, part_lse, status);   \
  } while (0)
  if (D.G <= 4) HILS_UNITS(4);
  else if (D.G <= 8) HILS_UNITS(8);
  else HILS_UNITS(16);
#undef HILS_UNITS
  return cudaGetLastError();
}

cudaError_t launch_attn_units(const Dims& D, bool bf16, int n_pieces, const void* q,
                              const void* K, const void* V, const int32_t* idx, float* part_o,
                              float* part_lse, int32_t* status, cudaStream_t st) {
  if (D.B * D.Hkv * D.N_q == 0) return cudaSuccess;
  if (D.d == 128)
    return bf16 ? launch_units_d<__nv_bfloat16, 128>(D, n_pieces, q, K, V, idx, part_o,
                                                     part_lse, status, st)
                : launch_units_d<float, 128>(D, n_pieces, q, K, V, idx, part_o, part_lse,
                                             status, st);
  return bf16 ? launch_units_d<__nv_bfloat16, 64>(D, n_pieces, q, K, V, idx, part_o, part_lse,
                                                 status, st)
              : launch_units_d<float, 64>(D, n_pieces, q, K, V, idx, part_o, part_lse, status,
                                          st);
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
