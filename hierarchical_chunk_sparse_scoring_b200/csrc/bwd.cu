// Backward pass: gradients of L = sum dO . O + sum dlse . LSE with respect to q, q_cal, K, V,
// k_lm and b_lm, the forward's selection held fixed (the top-K is piecewise constant and passes
// no gradient; the landmark keys and biases receive theirs through the fusion weights, [Reader]
// Fig. 3 caption: the loss gradient flows back to the compressed key).
//
// Per row (query i, head h) with units u (its selected chunks, then the local window) and fused
// weights w_u = exp(score_u - LSE), a token j of unit u has the fused weight a_j =
// exp(x_j + lambda_u) with lambda_u = score_u - LSE - lse_u, and by the chain rule through
// steps 4, 1 and 3 (the window's score is its own lse, so it adds its score gradient to its
// tokens' logits):
//   dV_j += a_j dO,  dx_j = a_j (dO . V_j - gamma_u),  dq += scale dx_j K_j,  dK_j += scale dx_j q
//   gamma_c = delta_c = dO . o_c for a chunk, gamma_local = D - dlse with D = sum_u w_u delta_u,
//   dscore_c = w_c (delta_c - D + dlse):  dq_cal += scale dscore_c k_lm_c,
//   dk_lm_c += scale dscore_c q_cal,  db_lm_c += dscore_c.
// delta_u needs a pass over the unit's tokens before any gradient can be formed, so:
//   bwd_rows_kernel  (query-major; CTA = 64 rows of one KV group: 64/G queries x G heads over the
//                    union of their chunks) pass 1: lse_u and delta_u by an online reduction of
//                    the logits x = q K^T and dP = dO V^T; then the fusion terms per row, d q_cal,
//                    and lambda, gamma, dscore to the workspace; pass 2: dq.
//   inverse index    (count, scan, fill) chunk -> the (query, slot) entries that selected it.
//   bwd_keys_kernel  (key-major; CTA = one tile of up to 64 keys of one chunk) over the rows whose
//                    window covers the tile and the rows that selected its chunk: dK and dV held
//                    in registers, then d k_lm and d b_lm from the selecting rows' dscore.
// No gradient is accumulated with atomics.  fp32 inputs: the products are CUDA-core tiles, 4 x
// (T/16) outputs per thread, operands staged in shared memory as fp32 (rows padded by 4 floats so
// the 16-byte loads of consecutive rows fall in different banks).  bf16 inputs: warp-level
// m16n8k16 tensor-core products (see the tensor-core tiles below).
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace hils {
namespace {

constexpr int kBwdRows = 64;      // rows per batch
constexpr int kBwdThreads = 256;
constexpr int kBwdMaxK = 32;

__host__ __device__ constexpr int pow2_at_least(int n) {
  int p = 1;
  while (p < n) p <<= 1;
  return p;
}
constexpr float kB2 = 1.4426950408889634f;          // log2(e)
constexpr float kLn2b = 0.6931471805599453f;

template <int DD, int T>
struct BwdShape {
  static constexpr int LD = DD + 4;            // fp32 row stride of staged q / dO / K / V rows
  static constexpr int LDA = T + 1;            // stride of the a / dx tiles
  static constexpr int KPT = T / 16;           // keys per thread in the logit tiles
  static constexpr int DG = DD / 64;           // float4 groups of dims per thread (dims td*4+64e)
  static constexpr int ROWS_F = kBwdRows * LD;
  static constexpr int KEYS_F = T * LD;
  static constexpr int TILE_F = kBwdRows * LDA;
  static_assert(DD == 64 || DD == 128, "head dims 64 and 128");
  static_assert(T == 16 || T == 32 || T == 64, "key tiles of 16, 32 or 64");
};

template <typename TI>
__device__ __forceinline__ void load_piece(const TI* src, float* dst);
template <>
__device__ __forceinline__ void load_piece<float>(const float* src, float* dst) {
  *reinterpret_cast<float4*>(dst) = __ldg(reinterpret_cast<const float4*>(src));
}
// Rows r < n of dst (stride LD floats) from rowp[r] (nullptr: zeros), fp32.
template <typename TI, int DD, int LD>
__device__ __forceinline__ void stage_rows(float* dst, const TI* const* rowp, int n) {
  constexpr int EPP = 16 / (int)sizeof(TI);   // elements per 16-byte piece
  constexpr int PPR = DD / EPP;
  for (int e = threadIdx.x; e < n * PPR; e += kBwdThreads) {
    const int r = e / PPR, u = e - r * PPR;
    const TI* src = rowp[r];
    float* d = dst + r * LD + u * EPP;
    if (src) {
      load_piece<TI>(src + u * EPP, d);
    } else {
      *reinterpret_cast<float4*>(d) = make_float4(0.f, 0.f, 0.f, 0.f);
      if (EPP == 8) *reinterpret_cast<float4*>(d + 4) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}

// Keys k0 .. k0 + T - 1 of one (b, g) plane (zeros past N_kv), fp32.
template <typename TI, int DD, int LD, int T>
__device__ __forceinline__ void stage_keys(float* dst, const TI* base, int64_t k0, int64_t nkv) {
  constexpr int EPP = 16 / (int)sizeof(TI);
  constexpr int PPR = DD / EPP;
  for (int e = threadIdx.x; e < T * PPR; e += kBwdThreads) {
    const int r = e / PPR, u = e - r * PPR;
    float* d = dst + r * LD + u * EPP;
    if (k0 + r < nkv) {
      load_piece<TI>(base + (k0 + r) * DD + u * EPP, d);
    } else {
      *reinterpret_cast<float4*>(d) = make_float4(0.f, 0.f, 0.f, 0.f);
      if (EPP == 8) *reinterpret_cast<float4*>(d + 4) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}

__device__ __forceinline__ float dot4(const float4 a, const float4 b, float acc) {
  acc = fmaf(a.x, b.x, acc);
  acc = fmaf(a.y, b.y, acc);
  acc = fmaf(a.z, b.z, acc);
  return fmaf(a.w, b.w, acc);
}

// X = Q K^T and P = dO V^T for rows tr*4 + i and keys tc + 16 e of the staged tiles.
template <int DD, int T>
__device__ __forceinline__ void logits_tile(const float* sQ, const float* sdO, const float* sK,
                                            const float* sV, int tr, int tc,
                                            float (&X)[4][T / 16], float (&P)[4][T / 16]) {
  using SH = BwdShape<DD, T>;
  constexpr int KPT = SH::KPT, LD = SH::LD;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int e = 0; e < KPT; ++e) X[i][e] = P[i][e] = 0.f;
#pragma unroll 2
  for (int k = 0; k < DD; k += 4) {
    float4 kk[KPT], vv[KPT];
#pragma unroll
    for (int e = 0; e < KPT; ++e) {
      kk[e] = *reinterpret_cast<const float4*>(sK + (tc + 16 * e) * LD + k);
      vv[e] = *reinterpret_cast<const float4*>(sV + (tc + 16 * e) * LD + k);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 q = *reinterpret_cast<const float4*>(sQ + (tr * 4 + i) * LD + k);
      const float4 o = *reinterpret_cast<const float4*>(sdO + (tr * 4 + i) * LD + k);
#pragma unroll
      for (int e = 0; e < KPT; ++e) {
        X[i][e] = dot4(q, kk[e], X[i][e]);
        P[i][e] = dot4(o, vv[e], P[i][e]);
      }
    }
  }
}

// ------------------------------------------------------------------ tensor-core (bf16) tiles
// With bf16 inputs the products run as warp-level m16n8k16 bf16 MMAs with fp32 accumulation:
// operands staged in shared memory as bf16 (rows padded by 8 elements, so the eight 16-byte rows
// an ldmatrix reads fall in different banks), fragments loaded with ldmatrix (.trans where the
// stored layout is the operand's transpose).  The logits and dO . V products take the bf16 inputs
// exactly; the fused weights a and logit gradients dx enter the dq, dK and dV products rounded to
// bf16, as the intermediate probabilities of a flash-attention backward do.
constexpr int kPadB = 8;   // bf16 elements of row padding
// Staging buffers of the tensor-core kernels' streamed operands (K/V tiles, gathered row
// batches): 1 keeps a CTA within half an SM's shared memory (two CTAs, 16 warps per SM, which
// hides the MMA chains' latency), 2 prefetches the next tile within one CTA per SM instead.
constexpr int kBwdBufs = 1;

__device__ __forceinline__ uint32_t su32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void ldsm4(uint32_t a, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                      uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(a));
}
__device__ __forceinline__ void ldsm4t(uint32_t a, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                       uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(a));
}
__device__ __forceinline__ void ldsm2(uint32_t a, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];\n"
               : "=r"(r0), "=r"(r1) : "r"(a));
}
__device__ __forceinline__ void ldsm2t(uint32_t a, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];\n"
               : "=r"(r0), "=r"(r1) : "r"(a));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// 16-byte asynchronous global -> shared copies (zero-filled when src_bytes is 0), in groups.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(su32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Rows r < n of a bf16 [n][DD + kPadB] tile from rowp[r] (nullptr: zeros), asynchronously (one
// commit group per call).
template <int DD>
__device__ __forceinline__ void fetch_rows_b(__nv_bfloat16* dst, const __nv_bfloat16* const* rowp,
                                             int n, const __nv_bfloat16* any) {
  constexpr int PPR = DD / 8, LDB = DD + kPadB;
  for (int e = threadIdx.x; e < n * PPR; e += kBwdThreads) {
    const int r = e / PPR, u = e - r * PPR;
    const __nv_bfloat16* src = rowp[r];
    cp_async16(dst + r * LDB + u * 8, src ? src + u * 8 : any, src ? 16u : 0u);
  }
  cp_async_commit();
}

// Keys k0 .. k0 + T - 1 of one (b, g) plane, bf16 [T][DD + kPadB], asynchronously (zeros past
// N_kv; no commit).
template <int DD, int T>
__device__ __forceinline__ void fetch_keys_b(__nv_bfloat16* dst, const __nv_bfloat16* base,
                                             int64_t k0, int64_t nkv) {
  constexpr int PPR = DD / 8, LDB = DD + kPadB;
  for (int e = threadIdx.x; e < T * PPR; e += kBwdThreads) {
    const int r = e / PPR, u = e - r * PPR;
    const bool in = k0 + r < nkv;
    cp_async16(dst + r * LDB + u * 8, in ? base + (k0 + r) * DD + u * 8 : base, in ? 16u : 0u);
  }
}

// Rows r < n of a bf16 [n][DD + kPadB] tile from rowp[r] (nullptr: zeros).
template <int DD>
__device__ __forceinline__ void stage_rows_b(__nv_bfloat16* dst,
                                             const __nv_bfloat16* const* rowp, int n) {
  constexpr int PPR = DD / 8, LDB = DD + kPadB;
  for (int e = threadIdx.x; e < n * PPR; e += kBwdThreads) {
    const int r = e / PPR, u = e - r * PPR;
    const __nv_bfloat16* src = rowp[r];
    *reinterpret_cast<uint4*>(dst + r * LDB + u * 8) =
        src ? __ldg(reinterpret_cast<const uint4*>(src + u * 8)) : make_uint4(0u, 0u, 0u, 0u);
  }
}

// Keys k0 .. k0 + T - 1 of one (b, g) plane as bf16 [T][DD + kPadB] (zeros past N_kv).
template <int DD, int T>
__device__ __forceinline__ void stage_keys_b(__nv_bfloat16* dst, const __nv_bfloat16* base,
                                             int64_t k0, int64_t nkv) {
  constexpr int PPR = DD / 8, LDB = DD + kPadB;
  for (int e = threadIdx.x; e < T * PPR; e += kBwdThreads) {
    const int r = e / PPR, u = e - r * PPR;
    *reinterpret_cast<uint4*>(dst + r * LDB + u * 8) =
        k0 + r < nkv ? __ldg(reinterpret_cast<const uint4*>(base + (k0 + r) * DD + u * 8))
                     : make_uint4(0u, 0u, 0u, 0u);
  }
}

// X = Q K^T and P = dO V^T for rows 16 rb .. 16 rb + 15 and keys kh T/2 .. (kh + 1) T/2 - 1:
// NT = T/16 accumulator tiles of m16n8 each; element v of tile j is (row 16 rb + lane/4 + 8 (v/2),
// key kh T/2 + 8 j + 2 (lane%4) + v%2).
template <int DD, int T>
__device__ __forceinline__ void logits_frag(const __nv_bfloat16* sQ, const __nv_bfloat16* sdO,
                                            const __nv_bfloat16* sK, const __nv_bfloat16* sV,
                                            int rb, int kh, float (&X)[T / 16][4],
                                            float (&P)[T / 16][4]) {
  constexpr int NT = T / 16, LDB = DD + kPadB;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int v = 0; v < 4; ++v) X[j][v] = P[j][v] = 0.f;
  const int arow = 16 * rb + (lane & 15), acol = (lane >> 4) * 8;
  const int i8 = lane >> 3, r8 = lane & 7;
#pragma unroll
  for (int ks = 0; ks < DD / 16; ++ks) {
    uint32_t aq[4], ao[4];
    ldsm4(su32(sQ + arow * LDB + 16 * ks + acol), aq[0], aq[1], aq[2], aq[3]);
    ldsm4(su32(sdO + arow * LDB + 16 * ks + acol), ao[0], ao[1], ao[2], ao[3]);
    if constexpr (NT == 1) {
      const int key = kh * (T / 2) + r8, dim = 16 * ks + (i8 & 1) * 8;
      uint32_t k0, k1, v0, v1;
      ldsm2(su32(sK + key * LDB + dim), k0, k1);
      ldsm2(su32(sV + key * LDB + dim), v0, v1);
      mma16816(X[0], aq, k0, k1);
      mma16816(P[0], ao, v0, v1);
    } else {
#pragma unroll
      for (int j = 0; j < NT; j += 2) {
        const int key = kh * (T / 2) + 8 * j + r8 + (i8 >> 1) * 8, dim = 16 * ks + (i8 & 1) * 8;
        uint32_t k0, k1, k2, k3, v0, v1, v2, v3;
        ldsm4(su32(sK + key * LDB + dim), k0, k1, k2, k3);
        ldsm4(su32(sV + key * LDB + dim), v0, v1, v2, v3);
        mma16816(X[j], aq, k0, k1);
        mma16816(X[j + 1], aq, k2, k3);
        mma16816(P[j], ao, v0, v1);
        mma16816(P[j + 1], ao, v2, v3);
      }
    }
  }
}

// Bytes of a kernel's product operands at the start of its shared memory (the bookkeeping
// follows): fp32 tiles for the CUDA cores, bf16 tiles for the tensor cores.
template <int DD, int T, bool TC>
constexpr int rows_prod_bytes() {
  using SH = BwdShape<DD, T>;
  return TC ? ((2 * kBwdRows + 2 * kBwdBufs * T) * (DD + kPadB) + kBwdRows * (T + kPadB)) * 2 +
                  2 * kBwdRows * 3 * 4
            : (2 * SH::ROWS_F + 2 * SH::KEYS_F + SH::TILE_F) * 4;
}
template <int DD, int T, bool TC>
constexpr int keys_prod_bytes() {
  using SH = BwdShape<DD, T>;
  return TC ? ((2 * kBwdBufs * kBwdRows + 2 * T) * (DD + kPadB) + 2 * kBwdRows * (T + kPadB)) * 2
            : (2 * SH::ROWS_F + 2 * SH::KEYS_F + 2 * SH::TILE_F) * 4;
}

}  // namespace

// ---------------------------------------------------------------------------------------------
// Query-major kernel: CTA = (b, g, 64/G queries); row r = query r / G, head g G + r % G.
// TC: the products on the tensor cores (bf16 inputs), else on the CUDA cores.
template <typename TI, int DD, int T, bool TC>
__global__ void __launch_bounds__(kBwdThreads, TC && kBwdBufs == 1 ? 2 : 1)
    bwd_rows_kernel(Dims D, const TI* __restrict__ q, const TI* __restrict__ qc,
                    const TI* __restrict__ K, const TI* __restrict__ V,
                    const TI* __restrict__ klm, const float* __restrict__ blm,
                    const int32_t* __restrict__ idx, const TI* __restrict__ dO,
                    const float* __restrict__ dlse, float* __restrict__ dq,
                    float* __restrict__ dqc, float* __restrict__ lam_ws,
                    float* __restrict__ gam_ws, float* __restrict__ ds_ws) {
  using SH = BwdShape<DD, T>;
  constexpr int LD = SH::LD, LDA = SH::LDA, KPT = SH::KPT, DG = SH::DG;
  const int SU = D.K + 1;   // stats row stride (units)
  using BF = __nv_bfloat16;
  constexpr int LDB = DD + kPadB, LDX = T + kPadB;
  extern __shared__ float4 smem_f4[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(smem_f4);
  // the products' operands: fp32 tiles (CUDA cores) or bf16 tiles (tensor cores)
  float* sQ = reinterpret_cast<float*>(smem);
  float* sdO = sQ + SH::ROWS_F;
  float* sK = sdO + SH::ROWS_F;
  float* sV = sK + SH::KEYS_F;
  float* sdX = sV + SH::KEYS_F;
  BF* bQ = reinterpret_cast<BF*>(smem);
  BF* bdO = bQ + kBwdRows * LDB;
  BF* bK = bdO + kBwdRows * LDB;   // [kBwdBufs][T][LDB]
  BF* bV = bK + kBwdBufs * T * LDB;   // [kBwdBufs][T][LDB]
  BF* bdX = bV + kBwdBufs * T * LDB;
  float* sPart = reinterpret_cast<float*>(bdX + kBwdRows * LDX);   // [2 key halves][64][3]
  float* sM = reinterpret_cast<float*>(smem + rows_prod_bytes<DD, T, TC>());   // [64][SU] running
                                                                           // max (base 2), then lambda2
  float* sL = sM + kBwdRows * SU;            // running sum, then gamma
  float* sT = sL + kBwdRows * SU;            // running sum of p dP, then dscore
  float* sS = sT + kBwdRows * SU;            // [64][SU] chunk scores
  // bookkeeping sized for this launch's K and G (see rows_smem)
  const int n_ids = (kBwdRows / D.G) * D.K;
  int* sel = reinterpret_cast<int*>(sS + kBwdRows * SU);   // [QT][K]
  int* sU = sel + ((n_ids + 1) & ~1);        // selected chunks below the window range, sorted
  int64_t* sPos = reinterpret_cast<int64_t*>(
      sU + ((pow2_at_least(n_ids) + 1) & ~1));   // [64] (8-byte aligned: even int counts)
  float* sDl = reinterpret_cast<float*>(sPos + kBwdRows);          // [64] dlse
  int* sUnit = reinterpret_cast<int*>(sDl + kBwdRows);             // [64]
  const TI** rowp = reinterpret_cast<const TI**>(sUnit + kBwdRows + 2);   // [64]
  int* sCount = reinterpret_cast<int*>(rowp + kBwdRows);                  // [1]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tr = tid >> 4, tc = tid & 15;
  const int G = D.G, QT = kBwdRows / G, Kt = D.K;
  const int64_t bg = blockIdx.y, b = bg / D.Hkv, g = bg - b * D.Hkv;
  const int64_t i0 = (int64_t)blockIdx.x * QT;
  const int nq = (int)(D.N_q - i0 < QT ? D.N_q - i0 : QT);
  const float sc2 = D.scale * kB2;
  const TI* Kb = K + bg * D.N_kv * DD;
  const TI* Vb = V + bg * D.N_kv * DD;
  auto grow_of = [&](int r) {   // global row of batch row r (valid rows only)
    return (b * D.Hq + g * G + r % G) * D.N_q + i0 + r / G;
  };

  // ---- rows, selections, union of the selected chunks below the window range
  if (tid < kBwdRows) {
    const int qq = tid / G;
    const bool valid = qq < nq;
    sPos[tid] = valid ? D.q_pos0 + i0 + qq : INT64_MIN;
    sDl[tid] = (valid && dlse) ? dlse[grow_of(tid)] : 0.f;
    rowp[tid] = valid ? q + grow_of(tid) * DD : nullptr;
  }
  const int64_t c_lo = n_eligible(D.q_pos0 + i0, D.S, D.W);
  const int64_t c_hi = (D.q_pos0 + i0 + nq - 1) / D.S;
  const int np = pow2_at_least(QT * Kt);
  for (int e = tid; e < np; e += kBwdThreads) {
    int c = INT_MAX;
    if (e < QT * Kt) {
      const int qq = e / Kt;
      int v = qq < nq ? idx[(bg * D.N_q + i0 + qq) * Kt + (e - qq * Kt)] : -1;
      // an id outside the query's eligible chunks is an empty slot (no memory outside k_lm is
      // read for it); a repeated id is attended once, in its first slot
      if (v >= 0 && v >= n_eligible(D.q_pos0 + i0 + qq, D.S, D.W)) v = -1;
      sel[e] = v;
      if (v >= 0 && v < c_lo) c = v;
    }
    sU[e] = c;
  }
  __syncthreads();
  if constexpr (TC) stage_rows_b<DD>(bQ, reinterpret_cast<const BF* const*>(rowp), kBwdRows);
  else stage_rows<TI, DD, LD>(sQ, rowp, kBwdRows);
  __syncthreads();
  if (tid < kBwdRows) rowp[tid] = sPos[tid] != INT64_MIN ? dO + grow_of(tid) * DD : nullptr;
  __syncthreads();
  // bitonic sort of the union candidates
  for (int k2 = 2; k2 <= np; k2 <<= 1)
    for (int j2 = k2 >> 1; j2 > 0; j2 >>= 1) {
      for (int e = tid; e < np; e += kBwdThreads) {
        const int f = e ^ j2;
        if (f > e) {
          const int a = sU[e], c = sU[f];
          const bool up = (e & k2) == 0;
          if ((a > c) == up) {
            sU[e] = c;
            sU[f] = a;
          }
        }
      }
      __syncthreads();
    }
  if constexpr (TC) stage_rows_b<DD>(bdO, reinterpret_cast<const BF* const*>(rowp), kBwdRows);
  else stage_rows<TI, DD, LD>(sdO, rowp, kBwdRows);
  if (warp == 0) {   // compact the distinct ids to the front (sorted: a repeat follows its twin)
    int n = 0, last = INT_MIN;
    for (int e0 = 0; e0 < np; e0 += 32) {
      const int e = e0 + lane;
      const int v = e < np ? sU[e] : INT_MAX;
      int prev = __shfl_up_sync(0xffffffffu, v, 1);
      if (lane == 0) prev = last;
      last = __shfl_sync(0xffffffffu, v, 31);
      const bool keep = v != INT_MAX && v != prev;
      const uint32_t bal = __ballot_sync(0xffffffffu, keep);
      __syncwarp();
      if (keep) sU[n + __popc(bal & ((1u << lane) - 1u))] = v;
      n += __popc(bal);
      __syncwarp();
    }
    if (lane == 0) *sCount = n;
  }
  for (int e = tid; e < kBwdRows * SU; e += kBwdThreads) {
    sM[e] = -INFINITY;
    sL[e] = 0.f;
    sT[e] = 0.f;
  }
  __syncthreads();
  const int n_sel = *sCount;
  const int SPT = D.S / T;   // key tiles per chunk
  const int n_tiles = (n_sel + (int)(c_hi - c_lo + 1)) * SPT;

  auto tile_k0 = [&](int t) -> int64_t {
    const int ci = t / SPT;
    const int64_t c = ci < n_sel ? (int64_t)sU[ci] : c_lo + (ci - n_sel);
    return c * D.S + (int64_t)(t - ci * SPT) * T;
  };
  // unit of each row for the tile starting at k0 (-1: not attended)
  auto set_units = [&](int64_t k0) {
    if (tid < kBwdRows) {
      const int64_t pos = sPos[tid];
      int u = -1;
      if (pos != INT64_MIN) {
        const int64_t c = k0 / D.S;
        if (c >= n_eligible(pos, D.S, D.W)) {
          u = k0 <= pos ? Kt : -1;
        } else {
          const int* sr = sel + (tid / G) * Kt;
          for (int k = Kt - 1; k >= 0; --k)
            if (sr[k] == (int)c) u = k;
        }
      }
      sUnit[tid] = u;
    }
  };

  // tensor cores: tile t's keys and values into buffer t % kBwdBufs, one commit group
  auto fetch_kv = [&](int t) {
    const int64_t k0 = tile_k0(t);
    const int o = (t % kBwdBufs) * T * LDB;
    fetch_keys_b<DD, T>(bK + o, reinterpret_cast<const BF*>(Kb), k0, D.N_kv);
    fetch_keys_b<DD, T>(bV + o, reinterpret_cast<const BF*>(Vb), k0, D.N_kv);
    cp_async_commit();
  };
  // tile t in its buffer: the next tile prefetched (two buffers) or this one fetched now (one;
  // the caller's barrier has retired the previous tile's readers)
  auto land_kv = [&](int t) {
    if constexpr (kBwdBufs == 2) {
      if (t + 1 < n_tiles) fetch_kv(t + 1);
      else cp_async_commit();
      cp_async_wait<1>();
    } else {
      if (t > 0) fetch_kv(t);
      cp_async_wait<0>();
    }
  };
  // merges a tile's (max, sum, sum p dP) of row r's unit u into the running state
  auto merge_stats = [&](int r, int u, float m, float l, float tt) {
    if (u < 0 || m == -INFINITY) return;
    float* pm = sM + r * SU + u;
    float* pl = sL + r * SU + u;
    float* pt = sT + r * SU + u;
    const float M = *pm;
    if (m > M) {
      const float f = M == -INFINITY ? 0.f : exp2f(M - m);
      *pl = *pl * f + l;
      *pt = *pt * f + tt;
      *pm = m;
    } else {
      const float f = exp2f(m - M);
      *pl += l * f;
      *pt += tt * f;
    }
  };

  // ---- pass 1: per (row, unit) lse and delta = dO . o_u by online reduction
  if constexpr (TC) {
    if (n_tiles > 0) fetch_kv(0);
  }
  for (int t = 0; t < n_tiles; ++t) {
    const int64_t k0 = tile_k0(t);
    if constexpr (TC) {
      land_kv(t);   // tile t has landed (this thread's copies; the barrier below: all)
    } else {
      stage_keys<TI, DD, LD, T>(sK, Kb, k0, D.N_kv);
      stage_keys<TI, DD, LD, T>(sV, Vb, k0, D.N_kv);
    }
    set_units(k0);
    __syncthreads();
    if constexpr (TC) {
      // warp: rows 16 rb .., keys kh T/2 ..; a row's values sit in the 4 lanes of its quad
      const int rb = warp & 3, kh = warp >> 2, g8 = lane >> 2, t4 = lane & 3;
      float X[T / 16][4], P[T / 16][4];
      logits_frag<DD, T>(bQ, bdO, bK + (t % kBwdBufs) * T * LDB, bV + (t % kBwdBufs) * T * LDB,
                         rb, kh, X, P);
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int r = 16 * rb + g8 + 8 * hr;
        const int u = sUnit[r];
        const int64_t pos = sPos[r];
        float m = -INFINITY;
#pragma unroll
        for (int j = 0; j < T / 16; ++j)
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            const int64_t key = k0 + kh * (T / 2) + 8 * j + 2 * t4 + v;
            const bool ok = u >= 0 && key <= pos && key < D.N_kv;
            X[j][2 * hr + v] = ok ? X[j][2 * hr + v] * sc2 : -INFINITY;
            m = fmaxf(m, X[j][2 * hr + v]);
          }
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        float l = 0.f, tt = 0.f;
#pragma unroll
        for (int j = 0; j < T / 16; ++j)
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            const float x = X[j][2 * hr + v];
            const float w = x == -INFINITY ? 0.f : exp2f(x - m);
            l += w;
            tt = fmaf(w, P[j][2 * hr + v], tt);
          }
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) {
          l += __shfl_xor_sync(0xffffffffu, l, o);
          tt += __shfl_xor_sync(0xffffffffu, tt, o);
        }
        if (t4 == 0) {
          float* pp = sPart + (kh * kBwdRows + r) * 3;
          pp[0] = m;
          pp[1] = l;
          pp[2] = tt;
        }
      }
      __syncthreads();
      if (tid < kBwdRows) {   // the two key halves of row tid, then its unit's running state
        const float* p0 = sPart + tid * 3;
        const float* p1 = sPart + (kBwdRows + tid) * 3;
        const float m = fmaxf(p0[0], p1[0]);
        float l = 0.f, tt = 0.f;
        if (m != -INFINITY) {
          const float f0 = p0[0] == -INFINITY ? 0.f : exp2f(p0[0] - m);
          const float f1 = p1[0] == -INFINITY ? 0.f : exp2f(p1[0] - m);
          l = p0[1] * f0 + p1[1] * f1;
          tt = p0[2] * f0 + p1[2] * f1;
        }
        merge_stats(tid, sUnit[tid], m, l, tt);
      }
    } else {
      float X[4][KPT], P[4][KPT];
      logits_tile<DD, T>(sQ, sdO, sK, sV, tr, tc, X, P);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = tr * 4 + i;
        const int u = sUnit[r];
        const int64_t pos = sPos[r];
        float m = -INFINITY;
#pragma unroll
        for (int e = 0; e < KPT; ++e) {
          const int64_t j = k0 + tc + 16 * e;
          const bool ok = u >= 0 && j <= pos && j < D.N_kv;
          X[i][e] = ok ? X[i][e] * sc2 : -INFINITY;
          m = fmaxf(m, X[i][e]);
        }
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float l = 0.f, tt = 0.f;
#pragma unroll
        for (int e = 0; e < KPT; ++e) {
          const float w = X[i][e] == -INFINITY ? 0.f : exp2f(X[i][e] - m);
          l += w;
          tt = fmaf(w, P[i][e], tt);
        }
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) {
          l += __shfl_xor_sync(0xffffffffu, l, o);
          tt += __shfl_xor_sync(0xffffffffu, tt, o);
        }
        if (tc == 0) merge_stats(r, u, m, l, tt);
      }
    }
    __syncthreads();
  }

  // ---- fusion terms per row
  for (int r = warp; r < kBwdRows; r += kBwdThreads / 32) {   // chunk scores s = scale qc.klm + b
    if (sPos[r] == INT64_MIN) continue;
    constexpr int DL = DD / 32, U = 8;
    float qv[DL];
    const TI* qr = qc + grow_of(r) * DD + lane * DL;
#pragma unroll
    for (int e = 0; e < DL; ++e) qv[e] = Elem<TI>::to_f(qr[e]);
    for (int k0 = 0; k0 < Kt; k0 += U) {   // eight landmark rows' loads in flight together
      int cs[U];
      float kv[U][DL], bias[U];
#pragma unroll
      for (int j = 0; j < U; ++j) {
        cs[j] = k0 + j < Kt ? sel[(r / G) * Kt + k0 + j] : -1;
        const TI* kr = klm + (bg * D.C + (cs[j] < 0 ? 0 : cs[j])) * DD + lane * DL;
#pragma unroll
        for (int e = 0; e < DL; ++e) kv[j][e] = cs[j] >= 0 ? Elem<TI>::to_f(kr[e]) : 0.f;
        bias[j] = cs[j] >= 0 ? blm[bg * D.C + cs[j]] : 0.f;
      }
#pragma unroll
      for (int j = 0; j < U; ++j) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < DL; ++e) a = fmaf(qv[e], kv[j][e], a);
        a = warp_sum(a);
        if (lane == 0 && cs[j] >= 0) sS[r * SU + k0 + j] = fmaf(a, D.scale, bias[j]);
      }
    }
  }
  __syncthreads();
  if (tid < kBwdRows && sPos[tid] != INT64_MIN) {
    const int r = tid;
    const int* sr = sel + (r / G) * Kt;
    float* M = sM + r * SU;
    float* Ls = sL + r * SU;
    float* Ts = sT + r * SU;
    // lse_u (natural log) to M, delta_u to Ts, score_u to Ls; the window's score is its lse
    float mx = -INFINITY;
    for (int u = 0; u <= Kt; ++u) {
      const bool present = u == Kt || (sr[u] >= 0 && Ls[u] > 0.f);
      const float lse = present ? (M[u] + log2f(Ls[u])) * kLn2b : -INFINITY;
      const float dlt = present ? Ts[u] / Ls[u] : 0.f;
      const float score = u == Kt ? lse : (present ? sS[r * SU + u] : -INFINITY);
      M[u] = lse;
      Ts[u] = dlt;
      Ls[u] = score;
      mx = fmaxf(mx, score);
    }
    float z = 0.f;
    for (int u = 0; u <= Kt; ++u) z += Ls[u] == -INFINITY ? 0.f : expf(Ls[u] - mx);
    const float LSE = mx + logf(z);
    float Dsum = 0.f;
    for (int u = 0; u <= Kt; ++u)
      if (Ls[u] != -INFINITY) Dsum = fmaf(expf(Ls[u] - LSE), Ts[u], Dsum);
    const float dl = sDl[r];
    const int64_t grow = grow_of(r);
    for (int u = 0; u <= Kt; ++u) {
      const float score = Ls[u];
      const bool live = score != -INFINITY;
      const float w = live ? expf(score - LSE) : 0.f;
      const float lam2 = live ? (score - LSE - M[u]) * kB2 : -INFINITY;
      const float gam = u == Kt ? Dsum - dl : Ts[u];
      const float dsc = u == Kt ? 0.f : w * (Ts[u] - Dsum + dl);
      M[u] = lam2;
      Ls[u] = gam;
      Ts[u] = dsc;
      lam_ws[grow * (Kt + 1) + u] = lam2;
      gam_ws[grow * (Kt + 1) + u] = gam;
      if (u < Kt) ds_ws[grow * Kt + u] = dsc;
    }
  }
  __syncthreads();
  for (int r = warp; r < kBwdRows; r += kBwdThreads / 32) {   // d q_cal = scale sum ds k_lm
    if (sPos[r] == INT64_MIN) continue;
    constexpr int DL = DD / 32, U = 8;
    float acc[DL];
#pragma unroll
    for (int e = 0; e < DL; ++e) acc[e] = 0.f;
    for (int k0 = 0; k0 < Kt; k0 += U) {   // eight landmark rows' loads in flight together
      float kv[U][DL], dsv[U];
#pragma unroll
      for (int j = 0; j < U; ++j) {
        const int c = k0 + j < Kt ? sel[(r / G) * Kt + k0 + j] : -1;
        dsv[j] = c >= 0 ? sT[r * SU + k0 + j] : 0.f;
        const TI* kr = klm + (bg * D.C + (c < 0 ? 0 : c)) * DD + lane * DL;
#pragma unroll
        for (int e = 0; e < DL; ++e) kv[j][e] = c >= 0 ? Elem<TI>::to_f(kr[e]) : 0.f;
      }
#pragma unroll
      for (int j = 0; j < U; ++j)
#pragma unroll
        for (int e = 0; e < DL; ++e) acc[e] = fmaf(dsv[j], kv[j][e], acc[e]);
    }
    float* out = dqc + grow_of(r) * DD + lane * DL;
#pragma unroll
    for (int e = 0; e < DL; ++e) out[e] = acc[e] * D.scale;
  }

  // ---- pass 2: dq = scale sum_j dx_j K_j
  if constexpr (TC) {
    // dx tile to shared memory as bf16, then dq += dx K on the tensor cores: warp = rows 16 rb ..
    // and dims dh d/2 .. (NTD = d/16 accumulator tiles)
    constexpr int NTD = DD / 16;
    const int rb = warp & 3, kh = warp >> 2, g8 = lane >> 2, t4 = lane & 3;
    const int dh = kh;
    float acc[NTD][4];
#pragma unroll
    for (int j = 0; j < NTD; ++j)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[j][v] = 0.f;
    __syncthreads();   // (pass 1's tiles are consumed)
    if (n_tiles > 0) fetch_kv(0);
    for (int t = 0; t < n_tiles; ++t) {
      const int64_t k0 = tile_k0(t);
      __syncthreads();   // the previous tile is consumed: its buffer takes the next one
      land_kv(t);
      set_units(k0);
      __syncthreads();
      const BF* bKt = bK + (t % kBwdBufs) * T * LDB;
      float X[T / 16][4], P[T / 16][4];
      logits_frag<DD, T>(bQ, bdO, bKt, bV + (t % kBwdBufs) * T * LDB, rb, kh, X, P);
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int r = 16 * rb + g8 + 8 * hr;
        const int u = sUnit[r];
        const int64_t pos = sPos[r];
        const float lam2 = u >= 0 ? sM[r * SU + u] : -INFINITY;
        const float gam = u >= 0 ? sL[r * SU + u] : 0.f;
#pragma unroll
        for (int j = 0; j < T / 16; ++j) {
          float dx[2];
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            const int64_t key = k0 + kh * (T / 2) + 8 * j + 2 * t4 + v;
            const bool ok = u >= 0 && key <= pos && key < D.N_kv && lam2 != -INFINITY;
            const float aw = ok ? exp2f(fmaf(X[j][2 * hr + v], sc2, lam2)) : 0.f;
            dx[v] = aw * (P[j][2 * hr + v] - gam);
          }
          *reinterpret_cast<uint32_t*>(bdX + r * LDX + kh * (T / 2) + 8 * j + 2 * t4) =
              pack_bf16(dx[0], dx[1]);
        }
      }
      __syncthreads();
      const int i8 = lane >> 3, r8 = lane & 7;
#pragma unroll
      for (int ks = 0; ks < T / 16; ++ks) {
        uint32_t af[4];
        ldsm4(su32(bdX + (16 * rb + (lane & 15)) * LDX + 16 * ks + (lane >> 4) * 8), af[0], af[1],
              af[2], af[3]);
#pragma unroll
        for (int j = 0; j < NTD / 2; ++j) {   // two dim tiles per ldmatrix
          const int key = 16 * ks + r8 + (i8 & 1) * 8;
          const int dim = dh * (DD / 2) + 16 * j + (i8 >> 1) * 8;
          uint32_t b0, b1, b2, b3;
          ldsm4t(su32(bKt + key * LDB + dim), b0, b1, b2, b3);
          mma16816(acc[2 * j], af, b0, b1);
          mma16816(acc[2 * j + 1], af, b2, b3);
        }
      }
    }
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int r = 16 * rb + g8 + 8 * hr;
      if (sPos[r] == INT64_MIN) continue;
      float* out = dq + grow_of(r) * DD + dh * (DD / 2);
#pragma unroll
      for (int j = 0; j < NTD; ++j)
        *reinterpret_cast<float2*>(out + 8 * j + 2 * t4) =
            make_float2(acc[j][2 * hr] * D.scale, acc[j][2 * hr + 1] * D.scale);
    }
  } else {
    float acc[4][DG][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int e = 0; e < DG; ++e)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[i][e][v] = 0.f;
    for (int t = 0; t < n_tiles; ++t) {
      const int64_t k0 = tile_k0(t);
      __syncthreads();
      stage_keys<TI, DD, LD, T>(sK, Kb, k0, D.N_kv);
      stage_keys<TI, DD, LD, T>(sV, Vb, k0, D.N_kv);
      set_units(k0);
      __syncthreads();
      float X[4][KPT], P[4][KPT];
      logits_tile<DD, T>(sQ, sdO, sK, sV, tr, tc, X, P);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = tr * 4 + i;
        const int u = sUnit[r];
        const int64_t pos = sPos[r];
        const float lam2 = u >= 0 ? sM[r * SU + u] : -INFINITY;
        const float gam = u >= 0 ? sL[r * SU + u] : 0.f;
#pragma unroll
        for (int e = 0; e < KPT; ++e) {
          const int64_t j = k0 + tc + 16 * e;
          const bool ok = u >= 0 && j <= pos && j < D.N_kv && lam2 != -INFINITY;
          const float aw = ok ? exp2f(fmaf(X[i][e], sc2, lam2)) : 0.f;
          sdX[r * LDA + tc + 16 * e] = aw * (P[i][e] - gam);
        }
      }
      __syncthreads();
#pragma unroll 4
      for (int j = 0; j < T; ++j) {
        float w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) w[i] = sdX[(tr * 4 + i) * LDA + j];
#pragma unroll
        for (int e = 0; e < DG; ++e) {
          const float4 kv = *reinterpret_cast<const float4*>(sK + j * LD + tc * 4 + 64 * e);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            acc[i][e][0] = fmaf(w[i], kv.x, acc[i][e][0]);
            acc[i][e][1] = fmaf(w[i], kv.y, acc[i][e][1]);
            acc[i][e][2] = fmaf(w[i], kv.z, acc[i][e][2]);
            acc[i][e][3] = fmaf(w[i], kv.w, acc[i][e][3]);
          }
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = tr * 4 + i;
      if (sPos[r] == INT64_MIN) continue;
      float* out = dq + grow_of(r) * DD;
#pragma unroll
      for (int e = 0; e < DG; ++e)
        *reinterpret_cast<float4*>(out + tc * 4 + 64 * e) =
            make_float4(acc[i][e][0] * D.scale, acc[i][e][1] * D.scale, acc[i][e][2] * D.scale,
                        acc[i][e][3] * D.scale);
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Key-major kernel: CTA = (b, g, keys k0 .. k0 + T - 1 of chunk c = k0 / S).  Its rows are the
// window rows (queries whose local window [S n, p] reaches the tile: n <= c and p >= k0, all G
// heads) and the selecting rows (the inverse index of chunk c, all G heads), in batches of 64.
// TC: the products on the tensor cores (bf16 inputs), else on the CUDA cores.
template <typename TI, int DD, int T, bool TC>
__global__ void __launch_bounds__(kBwdThreads, TC && kBwdBufs == 1 ? 2 : 1)
    bwd_keys_kernel(Dims D, const TI* __restrict__ q, const TI* __restrict__ qc,
                    const TI* __restrict__ K, const TI* __restrict__ V,
                    const TI* __restrict__ dO, const float* __restrict__ lam_ws,
                    const float* __restrict__ gam_ws, const float* __restrict__ ds_ws,
                    const int32_t* __restrict__ inv_off, const int32_t* __restrict__ inv_list,
                    float* __restrict__ dK, float* __restrict__ dV, float* __restrict__ dklm,
                    float* __restrict__ dblm) {
  using SH = BwdShape<DD, T>;
  using BF = __nv_bfloat16;
  constexpr int LD = SH::LD, LDA = SH::LDA, KPT = SH::KPT, DG = SH::DG;
  constexpr int LDB = DD + kPadB, LDX = T + kPadB;
  // tensor-core split of the [T keys x DD] outputs: KB key blocks of 16 x DGW dim groups
  constexpr int KB = T / 16, DGW = (kBwdThreads / 32) / KB, DPG = DD / DGW, NTK = DPG / 8;
  extern __shared__ float4 smem_f4[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(smem_f4);
  float* sQ = reinterpret_cast<float*>(smem);
  float* sdO = sQ + SH::ROWS_F;
  float* sK = sdO + SH::ROWS_F;
  float* sV = sK + SH::KEYS_F;
  float* sA = sV + SH::KEYS_F;
  float* sdX = sA + SH::TILE_F;
  BF* bQ = reinterpret_cast<BF*>(smem);   // [kBwdBufs][64][LDB] gathered q rows
  BF* bdO = bQ + kBwdBufs * kBwdRows * LDB;      // [kBwdBufs][64][LDB]
  BF* bK = bdO + kBwdBufs * kBwdRows * LDB;
  BF* bV = bK + T * LDB;
  BF* bA = bV + T * LDB;
  BF* bdX = bA + kBwdRows * LDX;
  // row bookkeeping of a batch, [3] buffers (the CUDA-core path uses the first)
  int64_t* sPos = reinterpret_cast<int64_t*>(smem + keys_prod_bytes<DD, T, TC>());   // [3][64]
  float* sLam = reinterpret_cast<float*>(sPos + 3 * kBwdRows);     // [3][64]
  float* sGam = sLam + 3 * kBwdRows;                               // [3][64]
  const TI** rowq = reinterpret_cast<const TI**>(sGam + 3 * kBwdRows);   // [3][64]
  const TI** rowo = rowq + 3 * kBwdRows;                                 // [3][64]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tr = tid >> 4, tc = tid & 15;
  const int G = D.G, Kt = D.K;
  const int64_t bg = blockIdx.y, b = bg / D.Hkv, g = bg - b * D.Hkv;
  const int64_t k0 = (int64_t)blockIdx.x * T;
  const int64_t c = k0 / D.S;
  const float sc2 = D.scale * kB2;
  // window rows: positions [max(k0, q_pos0), min((c + 1) S + W - 2, last query)]
  const int64_t p_lo = k0 > D.q_pos0 ? k0 : D.q_pos0;
  const int64_t p_last = D.q_pos0 + D.N_q - 1;
  const int64_t p_cap = (c + 1) * D.S + D.W - 2;
  const int64_t p_hi = p_cap < p_last ? p_cap : p_last;
  const int64_t n_win = p_hi >= p_lo ? p_hi - p_lo + 1 : 0;
  int64_t e_lo = 0, n_inv = 0;
  if (c < D.C && Kt > 0) {
    e_lo = inv_off[bg * (D.C + 1) + c];
    n_inv = inv_off[bg * (D.C + 1) + c + 1] - e_lo;
  }
  const int32_t* ents = inv_list + bg * D.N_q * Kt + e_lo;
  const int64_t total = (n_win + n_inv) * G;

  if constexpr (TC) {
    stage_keys_b<DD, T>(bK, reinterpret_cast<const BF*>(K) + bg * D.N_kv * DD, k0, D.N_kv);
    stage_keys_b<DD, T>(bV, reinterpret_cast<const BF*>(V) + bg * D.N_kv * DD, k0, D.N_kv);
  } else {
    stage_keys<TI, DD, LD, T>(sK, K + bg * D.N_kv * DD, k0, D.N_kv);
    stage_keys<TI, DD, LD, T>(sV, V + bg * D.N_kv * DD, k0, D.N_kv);
  }
  float aK[KPT][DG][4], aV[KPT][DG][4];      // CUDA-core accumulators
  float tK[NTK][4], tV[NTK][4];              // tensor-core accumulators
#pragma unroll
  for (int i = 0; i < KPT; ++i)
#pragma unroll
    for (int e = 0; e < DG; ++e)
#pragma unroll
      for (int v = 0; v < 4; ++v) aK[i][e][v] = aV[i][e][v] = 0.f;
#pragma unroll
  for (int j = 0; j < NTK; ++j)
#pragma unroll
    for (int v = 0; v < 4; ++v) tK[j][v] = tV[j][v] = 0.f;

  // the rows f0 .. f0 + 63 of the tile's row list: one row per thread < 64, loaded into registers
  // (prep_load) and later stored into a bookkeeping buffer (prep_store)
  struct RowMeta {
    int64_t pos;   // INT64_MIN: no row
    float lam, gam;
    const TI* rq;
    const TI* ro;
  };
  auto prep_load = [&](int64_t f0) -> RowMeta {
    RowMeta m{INT64_MIN, -INFINITY, 0.f, nullptr, nullptr};
    const int64_t f = f0 + tid;
    if (tid < kBwdRows && f < total) {
      int64_t qi;
      int u, h;
      if (f < n_win * G) {
        qi = p_lo - D.q_pos0 + f / G;
        h = (int)(f % G);
        u = Kt;
      } else {
        const int64_t fe = f - n_win * G;
        const int32_t ent = ents[fe / G];
        qi = ent / Kt;
        u = ent - (int)qi * Kt;
        h = (int)(fe % G);
      }
      const int64_t grow = (b * D.Hq + g * G + h) * D.N_q + qi;
      m.pos = D.q_pos0 + qi;
      m.lam = lam_ws[grow * (Kt + 1) + u];
      m.gam = gam_ws[grow * (Kt + 1) + u];
      m.rq = q + grow * DD;
      m.ro = dO + grow * DD;
    }
    return m;
  };
  auto prep_store = [&](const RowMeta& m, int buf) {
    if (tid < kBwdRows) {
      const int o = buf * kBwdRows + tid;
      sPos[o] = m.pos;
      sLam[o] = m.lam;
      sGam[o] = m.gam;
      rowq[o] = m.rq;
      rowo[o] = m.ro;
    }
  };
  auto prep = [&](int64_t f0, int buf) { prep_store(prep_load(f0), buf); };
  if constexpr (TC) {
    // batch i computes from row buffer i % kBwdBufs and bookkeeping buffer i % 3; with two row
    // buffers batch i + 1's rows load into the other meanwhile; batch i + 2's bookkeeping loads
    // into registers (stored after batch i's products, so its dependent loads overlap them)
    auto fetch = [&](int buf, int mb) {
      fetch_rows_b<DD>(bQ + buf * kBwdRows * LDB,
                       reinterpret_cast<const BF* const*>(rowq + mb * kBwdRows), kBwdRows,
                       reinterpret_cast<const BF*>(q));
      fetch_rows_b<DD>(bdO + buf * kBwdRows * LDB,
                       reinterpret_cast<const BF* const*>(rowo + mb * kBwdRows), kBwdRows,
                       reinterpret_cast<const BF*>(dO));
    };
    if (total > 0) {
      prep(0, 0);
      prep(kBwdRows, 1);
      __syncthreads();
      fetch(0, 0);
    }
    int bi = 0;
    for (int64_t f0 = 0; f0 < total; f0 += kBwdRows, ++bi) {
      const int buf = bi % kBwdBufs, mb = bi % 3;
      const RowMeta ahead = prep_load(f0 + 2 * kBwdRows);
      if constexpr (kBwdBufs == 2) {
        if (f0 + kBwdRows < total) {
          fetch(buf ^ 1, (bi + 1) % 3);
          cp_async_wait<2>();   // this batch's two groups have landed
        } else {
          cp_async_wait<0>();
        }
      } else {
        if (bi > 0) fetch(0, mb);   // (the previous batch's readers retired at its barrier)
        cp_async_wait<0>();
      }
      __syncthreads();
      const BF* cQ = bQ + buf * kBwdRows * LDB;
      const BF* cdO = bdO + buf * kBwdRows * LDB;
      const int64_t* cPos = sPos + mb * kBwdRows;
      const float* cLam = sLam + mb * kBwdRows;
      const float* cGam = sGam + mb * kBwdRows;
      const int rb = warp & 3, kh = warp >> 2, g8 = lane >> 2, t4 = lane & 3;
      float X[T / 16][4], P[T / 16][4];
      logits_frag<DD, T>(cQ, cdO, bK, bV, rb, kh, X, P);
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int r = 16 * rb + g8 + 8 * hr;
        const int64_t pos = cPos[r];
        const float lam2 = cLam[r], gam = cGam[r];
#pragma unroll
        for (int j = 0; j < T / 16; ++j) {
          float aw[2], dx[2];
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            const int64_t key = k0 + kh * (T / 2) + 8 * j + 2 * t4 + v;
            const bool ok = pos != INT64_MIN && key <= pos && key < D.N_kv && lam2 != -INFINITY;
            aw[v] = ok ? exp2f(fmaf(X[j][2 * hr + v], sc2, lam2)) : 0.f;
            dx[v] = aw[v] * (P[j][2 * hr + v] - gam);
          }
          const int col = kh * (T / 2) + 8 * j + 2 * t4;
          *reinterpret_cast<uint32_t*>(bA + r * LDX + col) = pack_bf16(aw[0], aw[1]);
          *reinterpret_cast<uint32_t*>(bdX + r * LDX + col) = pack_bf16(dx[0], dx[1]);
        }
      }
      __syncthreads();
      // dK += dx^T q, dV += a^T dO over the batch's 64 rows: warp = keys 16 kb .., dims dg DPG ..
      const int kb = warp % KB, dg = warp / KB;
      const int i8 = lane >> 3, r8 = lane & 7;
#pragma unroll
      for (int ks = 0; ks < kBwdRows / 16; ++ks) {
        const int srow = 16 * ks + r8 + (i8 >> 1) * 8, skey = 16 * kb + (i8 & 1) * 8;
        uint32_t ax[4], aa[4];
        ldsm4t(su32(bdX + srow * LDX + skey), ax[0], ax[1], ax[2], ax[3]);
        ldsm4t(su32(bA + srow * LDX + skey), aa[0], aa[1], aa[2], aa[3]);
        if constexpr (NTK == 1) {
          const int row = 16 * ks + r8 + (i8 & 1) * 8, dim = dg * DPG;
          uint32_t q0, q1, o0, o1;
          ldsm2t(su32(cQ + row * LDB + dim), q0, q1);
          ldsm2t(su32(cdO + row * LDB + dim), o0, o1);
          mma16816(tK[0], ax, q0, q1);
          mma16816(tV[0], aa, o0, o1);
        } else {
#pragma unroll
          for (int j = 0; j < NTK / 2; ++j) {
            const int row = 16 * ks + r8 + (i8 & 1) * 8;
            const int dim = dg * DPG + 16 * j + (i8 >> 1) * 8;
            uint32_t q0, q1, q2, q3, o0, o1, o2, o3;
            ldsm4t(su32(cQ + row * LDB + dim), q0, q1, q2, q3);
            ldsm4t(su32(cdO + row * LDB + dim), o0, o1, o2, o3);
            mma16816(tK[2 * j], ax, q0, q1);
            mma16816(tK[2 * j + 1], ax, q2, q3);
            mma16816(tV[2 * j], aa, o0, o1);
            mma16816(tV[2 * j + 1], aa, o2, o3);
          }
        }
      }
      prep_store(ahead, (bi + 2) % 3);
      __syncthreads();   // the batch's buffers are consumed (the next prep and fetch reuse them)
    }
  } else {
  for (int64_t f0 = 0; f0 < total; f0 += kBwdRows) {
    __syncthreads();   // the previous batch's tiles are consumed
    prep(f0, 0);
    __syncthreads();
    {
      stage_rows<TI, DD, LD>(sQ, rowq, kBwdRows);
      stage_rows<TI, DD, LD>(sdO, rowo, kBwdRows);
      __syncthreads();
      float X[4][KPT], P[4][KPT];
      logits_tile<DD, T>(sQ, sdO, sK, sV, tr, tc, X, P);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = tr * 4 + i;
        const int64_t pos = sPos[r];
        const float lam2 = sLam[r], gam = sGam[r];
#pragma unroll
        for (int e = 0; e < KPT; ++e) {
          const int64_t j = k0 + tc + 16 * e;
          const bool ok = pos != INT64_MIN && j <= pos && j < D.N_kv && lam2 != -INFINITY;
          const float aw = ok ? exp2f(fmaf(X[i][e], sc2, lam2)) : 0.f;
          sA[r * LDA + tc + 16 * e] = aw;
          sdX[r * LDA + tc + 16 * e] = aw * (P[i][e] - gam);
        }
      }
      __syncthreads();
#pragma unroll 2
      for (int r = 0; r < kBwdRows; ++r) {
        float xs[KPT], as[KPT];
#pragma unroll
        for (int i = 0; i < KPT; ++i) {
          xs[i] = sdX[r * LDA + tr * KPT + i];
          as[i] = sA[r * LDA + tr * KPT + i];
        }
#pragma unroll
        for (int e = 0; e < DG; ++e) {
          const float4 qv = *reinterpret_cast<const float4*>(sQ + r * LD + tc * 4 + 64 * e);
          const float4 ov = *reinterpret_cast<const float4*>(sdO + r * LD + tc * 4 + 64 * e);
#pragma unroll
          for (int i = 0; i < KPT; ++i) {
            aK[i][e][0] = fmaf(xs[i], qv.x, aK[i][e][0]);
            aK[i][e][1] = fmaf(xs[i], qv.y, aK[i][e][1]);
            aK[i][e][2] = fmaf(xs[i], qv.z, aK[i][e][2]);
            aK[i][e][3] = fmaf(xs[i], qv.w, aK[i][e][3]);
            aV[i][e][0] = fmaf(as[i], ov.x, aV[i][e][0]);
            aV[i][e][1] = fmaf(as[i], ov.y, aV[i][e][1]);
            aV[i][e][2] = fmaf(as[i], ov.z, aV[i][e][2]);
            aV[i][e][3] = fmaf(as[i], ov.w, aV[i][e][3]);
          }
        }
      }
    }
  }
  }
  if constexpr (TC) {
    const int kb = warp % KB, dg = warp / KB, g8 = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int64_t j = k0 + 16 * kb + g8 + 8 * hr;
      if (j >= D.N_kv) continue;
#pragma unroll
      for (int jt = 0; jt < NTK; ++jt) {
        const int64_t o = (bg * D.N_kv + j) * DD + dg * DPG + 8 * jt + 2 * t4;
        *reinterpret_cast<float2*>(dK + o) =
            make_float2(tK[jt][2 * hr] * D.scale, tK[jt][2 * hr + 1] * D.scale);
        *reinterpret_cast<float2*>(dV + o) = make_float2(tV[jt][2 * hr], tV[jt][2 * hr + 1]);
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < KPT; ++i) {
      const int64_t j = k0 + tr * KPT + i;
      if (j >= D.N_kv) continue;
#pragma unroll
      for (int e = 0; e < DG; ++e) {
        const int64_t o = (bg * D.N_kv + j) * DD + tc * 4 + 64 * e;
        *reinterpret_cast<float4*>(dK + o) =
            make_float4(aK[i][e][0] * D.scale, aK[i][e][1] * D.scale, aK[i][e][2] * D.scale,
                        aK[i][e][3] * D.scale);
        *reinterpret_cast<float4*>(dV + o) =
            make_float4(aV[i][e][0], aV[i][e][1], aV[i][e][2], aV[i][e][3]);
      }
    }
  }

  // d k_lm and d b_lm of chunk c: scale sum dscore q_cal and sum dscore over its selecting rows.
  // A warp per row, lanes over dims; eight rows per warp have their loads in flight together
  // (each row's loads depend on its index entry).
  if (c < D.C && k0 == c * D.S) {
    constexpr int EPL = DD / 32, NW = kBwdThreads / 32, U = 8;
    float acc[EPL], dsum = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
    const int64_t nr = n_inv * G;
    for (int64_t f0 = warp; f0 < nr; f0 += NW * U) {
      int64_t grow[U];
      int slot[U];
#pragma unroll
      for (int j = 0; j < U; ++j) {
        const int64_t f = f0 + (int64_t)NW * j;
        grow[j] = -1;
        slot[j] = 0;
        if (f < nr) {
          const int32_t ent = ents[f / G];
          const int64_t qi = ent / Kt;
          slot[j] = ent - (int)qi * Kt;
          grow[j] = (b * D.Hq + g * G + f % G) * D.N_q + qi;
        }
      }
      float dsv[U], qv[U][EPL];
#pragma unroll
      for (int j = 0; j < U; ++j) {
        dsv[j] = grow[j] >= 0 ? ds_ws[grow[j] * Kt + slot[j]] : 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e)
          qv[j][e] = grow[j] >= 0 ? Elem<TI>::to_f(qc[grow[j] * DD + lane * EPL + e]) : 0.f;
      }
#pragma unroll
      for (int j = 0; j < U; ++j) {
        dsum += dsv[j];
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = fmaf(dsv[j], qv[j][e], acc[e]);
      }
    }
    __syncthreads();
    float* red = reinterpret_cast<float*>(smem);   // [NW][DD + 1] (the products' area)
#pragma unroll
    for (int e = 0; e < EPL; ++e) red[warp * (DD + 1) + lane * EPL + e] = acc[e];
    if (lane == 0) red[warp * (DD + 1) + DD] = dsum;
    __syncthreads();
    if (tid < DD) {
      float a2 = 0.f;
      for (int w = 0; w < NW; ++w) a2 += red[w * (DD + 1) + tid];
      dklm[(bg * D.C + c) * DD + tid] = a2 * D.scale;
    } else if (tid == DD) {
      float t = 0.f;
      for (int w = 0; w < NW; ++w) t += red[w * (DD + 1) + DD];
      dblm[bg * D.C + c] = t;
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Inverse index: per (b, g) and chunk c the entries i * K + slot of the queries that selected c.
__global__ void __launch_bounds__(256)
    inv_count_kernel(Dims D, const int32_t* __restrict__ idx, int32_t* __restrict__ cnt) {
  const int64_t per = D.N_q * D.K;
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= D.B * D.Hkv * per) return;
  const int32_t c = idx[e];
  if (c >= 0 && c < D.C) atomicAdd(&cnt[(e / per) * D.C + c], 1);
}

__global__ void __launch_bounds__(1024)
    inv_scan_kernel(Dims D, const int32_t* __restrict__ cnt, int32_t* __restrict__ off) {
  __shared__ int32_t wsum[32];
  const int64_t bg = blockIdx.x;
  const int64_t C = D.C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t seg = (C + 1023) / 1024;
  const int64_t lo = tid * seg < C ? tid * seg : C;
  const int64_t hi = lo + seg < C ? lo + seg : C;
  const int32_t* cb = cnt + bg * C;
  int32_t s = 0;
  for (int64_t x = lo; x < hi; ++x) s += cb[x];
  // exclusive scan of the per-thread sums
  int32_t inc = s;
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int32_t w = wsum[lane];
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    wsum[lane] = w;
  }
  __syncthreads();
  int32_t run = inc - s + (warp > 0 ? wsum[warp - 1] : 0);
  int32_t* ob = off + bg * (C + 1);
  for (int64_t x = lo; x < hi; ++x) {
    ob[x] = run;
    run += cb[x];
  }
  if (tid == 1023) ob[C] = run;
}

__global__ void __launch_bounds__(256)
    inv_fill_kernel(Dims D, const int32_t* __restrict__ idx, const int32_t* __restrict__ off,
                    int32_t* __restrict__ cur, int32_t* __restrict__ list) {
  const int64_t per = D.N_q * D.K;
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= D.B * D.Hkv * per) return;
  const int32_t c = idx[e];
  if (c < 0 || c >= D.C) return;
  const int64_t bg = e / per;
  const int32_t slot = atomicAdd(&cur[bg * D.C + c], 1);
  list[bg * per + off[bg * (D.C + 1) + c] + slot] = (int32_t)(e - bg * per);
}


// ---------------------------------------------------------------------------------------------
namespace {

// Shared memory of the query-major kernel for this launch: the product operands, then the
// per-(row, unit) state, the chunk scores, the selections of the block's queries, the sorted
// union and the row bookkeeping.
template <int DD, int T, bool TC>
size_t rows_smem(const Dims& D) {
  const int SU = D.K + 1, n_ids = (kBwdRows / D.G) * D.K;
  return (size_t)rows_prod_bytes<DD, T, TC>() + (size_t)(4 * kBwdRows * SU) * 4 +
         (size_t)(((n_ids + 1) & ~1) + ((pow2_at_least(n_ids) + 1) & ~1)) * 4 + kBwdRows * 8 +
         kBwdRows * 4 + kBwdRows * 4 + 8 + kBwdRows * 8 + 16;
}

template <int DD, int T, bool TC>
constexpr size_t keys_smem() {
  return (size_t)keys_prod_bytes<DD, T, TC>() + 3 * (kBwdRows * 8 + 2 * kBwdRows * 4 +
                                                    2 * kBwdRows * 8);
}

template <typename TI, int DD, int T>
cudaError_t launch_bwd_t(const Dims& D, const BwdArgs& a, const BwdWs& w, cudaStream_t st) {
  constexpr bool TC = std::is_same<TI, __nv_bfloat16>::value;
  const size_t RS = rows_smem<DD, T, TC>(D);
  constexpr size_t KS = keys_smem<DD, T, TC>();
  static_assert(KS <= 227 * 1024, "shared memory");
  if (RS > 227 * 1024) return cudaErrorInvalidValue;
  auto kr = bwd_rows_kernel<TI, DD, T, TC>;
  auto kk = bwd_keys_kernel<TI, DD, T, TC>;
  cudaError_t e = cudaFuncSetAttribute(kr, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)RS);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)KS);
  if (e != cudaSuccess) return e;
  const TI* q = static_cast<const TI*>(a.q);
  const TI* qc = static_cast<const TI*>(a.q_cal);
  const TI* K = static_cast<const TI*>(a.K);
  const TI* V = static_cast<const TI*>(a.V);
  const TI* klm = static_cast<const TI*>(a.k_lm);
  const TI* dO = static_cast<const TI*>(a.dout);
  const int QT = kBwdRows / D.G;
  if (D.N_q > 0) {
    const dim3 gr((unsigned)((D.N_q + QT - 1) / QT), (unsigned)(D.B * D.Hkv));
    kr<<<gr, kBwdThreads, RS, st>>>(D, q, qc, K, V, klm, a.b_lm, a.idx, dO, a.dlse, a.dq, a.dq_cal,
                                    w.lam, w.gam, w.ds);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const dim3 gk((unsigned)((D.N_kv + T - 1) / T), (unsigned)(D.B * D.Hkv));
  kk<<<gk, kBwdThreads, KS, st>>>(D, q, qc, K, V, dO, w.lam, w.gam, w.ds, w.inv_off, w.inv_list,
                                  a.dK, a.dV, a.dk_lm, a.db_lm);
  return cudaGetLastError();
}

template <typename TI>
cudaError_t launch_bwd_d(const Dims& D, const BwdArgs& a, const BwdWs& w, cudaStream_t st) {
  const int T = D.S < 64 ? D.S : 64;
  if (D.d == 128) {
    if (T == 64) return launch_bwd_t<TI, 128, 64>(D, a, w, st);
    if (T == 32) return launch_bwd_t<TI, 128, 32>(D, a, w, st);
    return launch_bwd_t<TI, 128, 16>(D, a, w, st);
  }
  if (T == 64) return launch_bwd_t<TI, 64, 64>(D, a, w, st);
  if (T == 32) return launch_bwd_t<TI, 64, 32>(D, a, w, st);
  return launch_bwd_t<TI, 64, 16>(D, a, w, st);
}

}  // namespace

bool backward_supported(const Dims& D) {
  if (D.d != 64 && D.d != 128) return false;
  if (D.S != 16 && D.S != 32 && D.S != 64 && D.S != 128) return false;
  if (D.G < 1 || D.G > kBwdRows || kBwdRows % D.G != 0) return false;
  if (D.K < 0 || D.K > kBwdMaxK) return false;
  if (D.B * D.Hkv > 65535) return false;
  if (D.N_q * (int64_t)(D.K > 0 ? D.K : 1) >= (int64_t)INT32_MAX) return false;
  if ((D.N_kv + 15) / 16 >= (int64_t)INT32_MAX) return false;
  return true;
}

size_t backward_ws_layout(const Dims& D, BwdWs* w, char* base) {
  const int64_t R = D.B * D.Hq * D.N_q;
  const int64_t BG = D.B * D.Hkv;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) & ~size_t(255);
    return base ? base + o : nullptr;
  };
  char* lam = take((size_t)R * (D.K + 1) * 4);
  char* gam = take((size_t)R * (D.K + 1) * 4);
  char* ds = take((size_t)R * (D.K > 0 ? D.K : 1) * 4);
  char* cnt = take((size_t)BG * (D.C > 0 ? D.C : 1) * 4);
  char* cur = take((size_t)BG * (D.C > 0 ? D.C : 1) * 4);
  char* ioff = take((size_t)BG * (D.C + 1) * 4);
  char* list = take((size_t)BG * D.N_q * (D.K > 0 ? D.K : 1) * 4);
  if (w) {
    w->lam = reinterpret_cast<float*>(lam);
    w->gam = reinterpret_cast<float*>(gam);
    w->ds = reinterpret_cast<float*>(ds);
    w->inv_cnt = reinterpret_cast<int32_t*>(cnt);
    w->inv_cur = reinterpret_cast<int32_t*>(cur);
    w->inv_off = reinterpret_cast<int32_t*>(ioff);
    w->inv_list = reinterpret_cast<int32_t*>(list);
  }
  return off;
}

cudaError_t launch_backward(const Dims& D, bool bf16, const BwdArgs& a, const BwdWs& w,
                            cudaStream_t st) {
  const int64_t BG = D.B * D.Hkv;
  cudaError_t e = cudaSuccess;
  if (D.K > 0 && D.C > 0 && D.N_q > 0) {
    e = cudaMemsetAsync(w.inv_cnt, 0, (size_t)BG * D.C * 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(w.inv_cur, 0, (size_t)BG * D.C * 4, st);
    if (e != cudaSuccess) return e;
    const int64_t n = BG * D.N_q * D.K;
    const unsigned grid = (unsigned)((n + 255) / 256);
    inv_count_kernel<<<grid, 256, 0, st>>>(D, a.idx, w.inv_cnt);
    inv_scan_kernel<<<(unsigned)BG, 1024, 0, st>>>(D, w.inv_cnt, w.inv_off);
    inv_fill_kernel<<<grid, 256, 0, st>>>(D, a.idx, w.inv_off, w.inv_cur, w.inv_list);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  } else if (D.C > 0) {
    // no selections: every chunk's list is empty
    e = cudaMemsetAsync(w.inv_off, 0, (size_t)BG * (D.C + 1) * 4, st);
    if (e != cudaSuccess) return e;
  }
  return bf16 ? launch_bwd_d<__nv_bfloat16>(D, a, w, st) : launch_bwd_d<float>(D, a, w, st);
}

}  // namespace hils
