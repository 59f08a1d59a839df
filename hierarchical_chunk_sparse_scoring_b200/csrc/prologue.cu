// Query prologue, upstream of steps 1 and 3: Q-Cal and HoPE.
//
// Q-Cal ([Reader] "Implementation and Training Recipes", Q-Cal worked example): per query head h
// the calibrated query adds a low-rank correction computed from the token's hidden state,
// q_cal = q + W_up[h] (W_down[h] hidden), W_down[h]: r x d_model, W_up[h]: d x r.
// HoPE ([Reader] same section, HoPE vs RoPE; [Essay] "Hierarchical Positional Encoding"): the
// dimension pairs (m, m + d/2) whose rotation period 2 pi base^(2m/d) fits the training length
// turn by pos * base^(-2m/d); the others are left as they are (NoPE).  q and q_cal are turned at
// the query's position, keys at their own (hope_rotate).
//
// Kernels:
//   qdown_kernel   u = hidden W_down^T for all heads at once: [B N_q, d_model] x [Hq r, d_model]^T,
//                  a dense contraction on the tcgen05 tensor cores (bf16 operands by TMA with the
//                  128-byte swizzle, fp32 accumulator in TMEM, 128 x BN tiles, a 4-stage ring).
//   qcal_hope_kernel  per (b, 32 tokens), every head in turn: q_cal = R(q + W_up u), q = R(q);
//                  q read, both written, u read; W_up[h] read through L1; four tokens per warp
//                  in flight together, each lane d/64 whole rotation pairs (dims m and m + d/2,
//                  so the rotation stays in the lane); the block's (token, pair) angles
//                  p theta_m reduced modulo 2 pi in fp64 once (p up to 2^22 makes an fp32
//                  product lose whole radians), then sincosf, kept in shared memory for all
//                  heads.  hope_rotate_kernel turns keys the same way.
//   qcal_hope_mma_kernel  the same pass for bf16, d = 128 and r a multiple of 16, with W_up u on
//                  m16n8k16 tensor-core tiles and the q / output tiles staged in shared memory.
#include <cudaTypedefs.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace hils {
using namespace sm100;

namespace {

constexpr uint32_t kPrPollLimit = 1u << 24;
constexpr int kQdBM = 128;        // token rows per tile (M)
constexpr int kQdThreads = 192;   // TMA warp, MMA warp, 4 epilogue warps
constexpr double kTwoPi = 6.283185307179586476925286766559;

template <int BN>
struct QdShape {
  static constexpr int A_BYTES = kQdBM * 128;   // 128 rows x 64 bf16
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int STAGES = 4;
  static constexpr int SMEM = STAGES * STAGE + 1024 + 256;
  static constexpr uint32_t TMEM_COLS = BN;
  static_assert(BN == 64 || BN == 128 || BN == 256, "N tiles of 64, 128 or 256");
};

template <int BN>
__global__ void __launch_bounds__(kQdThreads, 1)
    qdown_kernel(const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmW,
                 int64_t M, int64_t N, int64_t Kdim, float* __restrict__ u,
                 int32_t* __restrict__ status) {
  using SH = QdShape<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SH::STAGES * SH::STAGE);
  uint64_t* full = bars;
  uint64_t* empty = bars + SH::STAGES;
  uint64_t* acc_full = bars + 2 * SH::STAGES;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_full + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t m0 = (int64_t)blockIdx.x * kQdBM, n0 = (int64_t)blockIdx.y * BN;
  const int nk = (int)(Kdim / 64);
  if (threadIdx.x == 0) {
    for (int s = 0; s < SH::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_holder, SH::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&tmH);
      prefetch_tensormap(&tmW);
      int last_s = -1;
      uint32_t last_par = 0;
      for (int kt = 0; kt < nk; ++kt) {
        const int s = kt % SH::STAGES;
        const uint32_t v = (uint32_t)(kt / SH::STAGES);
        if (!mbar_wait(&empty[s], (v & 1u) ^ 1u, kPrPollLimit)) {
          record_status(status, kStatusTimeout);
          break;
        }
        uint8_t* st = smem + s * SH::STAGE;
        mbar_expect_tx(&full[s], SH::STAGE);
        tma_load_2d(st, &tmH, kt * 64, (int32_t)m0, &full[s]);
        tma_load_2d(st + SH::A_BYTES, &tmW, kt * 64, (int32_t)n0, &full[s]);
        last_s = s;
        last_par = v & 1u;
      }
      if (last_s >= 0) mbar_wait(&full[last_s], last_par, kPrPollLimit);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(kQdBM, BN);
      bool ok = true;
      for (int kt = 0; ok && kt < nk; ++kt) {
        const int s = kt % SH::STAGES;
        const uint32_t v = (uint32_t)(kt / SH::STAGES);
        ok = mbar_wait(&full[s], v & 1u, kPrPollLimit);
        if (!ok) break;
        tc_fence_after();
        const uint8_t* st = smem + s * SH::STAGE;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t ad = desc_kmajor_sw128(smem_u32(st) + ks * 32);
          const uint64_t bd = desc_kmajor_sw128(smem_u32(st + SH::A_BYTES) + ks * 32);
          mma_bf16_ss(tmem, ad, bd, IDESC, (kt | ks) > 0 ? 1u : 0u);
        }
        mma_commit(&empty[s]);
      }
      if (!ok) record_status(status, kStatusTimeout);
      mma_commit(acc_full);   // (also after a timeout: the epilogue's wait then ends)
    }
  } else {
    // epilogue: warp w reads TMEM lanes 32 (w % 4) ..: one token row per thread
    const int qd = warp & 3;
    const int64_t row = m0 + qd * 32 + lane;
    const bool ok = mbar_wait_warp(acc_full, 0, kPrPollLimit);
    if (!ok) record_status(status, kStatusTimeout);
    tc_fence_after();
    if (ok) {
      for (int c0 = 0; c0 < BN; c0 += 16) {
        float v[16];
        tmem_ld16(tmem + ((uint32_t)(qd * 32) << 16) + (uint32_t)c0, v);
        tmem_wait_ld();
        if (row < M) {
          float4* dst = reinterpret_cast<float4*>(u + row * N + n0 + c0);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, SH::TMEM_COLS);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// [rows, cols] bf16 row-major, boxes of [box_rows, 64] with the 128-byte swizzle.
bool map_rows(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
              uint32_t box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN>
cudaError_t launch_qdown_t(int64_t M, int64_t N, int64_t Kdim, const void* hidden,
                           const void* W_down, float* u, int32_t* status, cudaStream_t st) {
  using SH = QdShape<BN>;
  CUtensorMap tmH, tmW;
  if (!map_rows(&tmH, hidden, (uint64_t)M, (uint64_t)Kdim, kQdBM) ||
      !map_rows(&tmW, W_down, (uint64_t)N, (uint64_t)Kdim, BN))
    return cudaErrorInvalidValue;
  auto kern = qdown_kernel<BN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SH::SMEM);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)((M + kQdBM - 1) / kQdBM), (unsigned)(N / BN));
  kern<<<grid, kQdThreads, SH::SMEM, st>>>(tmH, tmW, M, N, Kdim, u, status);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------------
constexpr int kQhTokens = 32;     // tokens per CTA
constexpr int kQhThreads = 256;

// Two consecutive dims of a row as floats, and back (EPL = 2).
template <typename T, int EPL>
__device__ __forceinline__ void load_dims(const T* p, float (&v)[EPL]);
template <>
__device__ __forceinline__ void load_dims<__nv_bfloat16, 2>(const __nv_bfloat16* p, float (&v)[2]) {
  const uint32_t t = *reinterpret_cast<const uint32_t*>(p);
  v[0] = bf16_lo(t); v[1] = bf16_hi(t);
}
template <>
__device__ __forceinline__ void load_dims<float, 2>(const float* p, float (&v)[2]) {
  const float2 t = *reinterpret_cast<const float2*>(p);
  v[0] = t.x; v[1] = t.y;
}
template <typename T, int EPL>
__device__ __forceinline__ void store_dims(T* p, const float (&v)[EPL]) {
  static_assert(EPL == 2, "two dims");
  if constexpr (std::is_same<T, float>::value) {
    *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
  } else {
    const __nv_bfloat162 h = __floats2bfloat162_rn(v[0], v[1]);
    *reinterpret_cast<uint32_t*>(p) = *reinterpret_cast<const uint32_t*>(&h);
  }
}

// Cosine and sine of every (token, pair) angle of a CTA's token block, fp64 reduction modulo
// 2 pi (the angle p theta_m reaches 2^22 rad), once per CTA for all its heads; pairs that do not
// turn get (1, 0).
template <int DD>
__device__ __forceinline__ void angle_table(float2* sCS, int64_t pos0, double base,
                                            double train_len) {
  for (int e = threadIdx.x; e < kQhTokens * (DD / 2); e += kQhThreads) {
    const int t = e / (DD / 2), m = e - t * (DD / 2);
    const double th = pow(base, -2.0 * (double)m / (double)DD);
    float2 cs = make_float2(1.f, 0.f);
    if (kTwoPi / th <= train_len) {
      double a = (double)(pos0 + t) * th;
      a -= kTwoPi * floor(a * (1.0 / kTwoPi));
      sincosf((float)a, &cs.y, &cs.x);
    }
    sCS[e] = cs;
  }
}

// Eight consecutive elements (16 or 32 bytes, 16-byte aligned) as floats, through L1.
template <typename T>
__device__ __forceinline__ void load_piece8(const T* p, float (&v)[8]);
template <>
__device__ __forceinline__ void load_piece8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 t = __ldg(reinterpret_cast<const uint4*>(p));
  v[0] = bf16_lo(t.x); v[1] = bf16_hi(t.x); v[2] = bf16_lo(t.y); v[3] = bf16_hi(t.y);
  v[4] = bf16_lo(t.z); v[5] = bf16_hi(t.z); v[6] = bf16_lo(t.w); v[7] = bf16_hi(t.w);
}
template <>
__device__ __forceinline__ void load_piece8<float>(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// HP consecutive elements (HP = 1 or 2) of a row as floats, and back.
template <typename T, int HP>
__device__ __forceinline__ void load_n(const T* p, float (&v)[HP]) {
  if constexpr (HP == 2) {
    load_dims<T, 2>(p, v);
  } else {
    v[0] = Elem<T>::to_f(p[0]);
  }
}
template <typename T, int HP>
__device__ __forceinline__ void store_n(T* p, const float (&v)[HP]) {
  if constexpr (HP == 2) {
    store_dims<T, 2>(p, v);
  } else if constexpr (std::is_same<T, float>::value) {
    p[0] = v[0];
  } else {
    p[0] = __float2bfloat16_rn(v[0]);
  }
}

// grid (token blocks, B); every head of the block in turn.  r = 0 leaves q_cal = R(q).  Each
// warp takes kQhTpw tokens together (their loads in flight at once).  A lane holds HP = d/64
// whole rotation pairs, dims m0 .. m0 + HP - 1 and their partners m + d/2, so the rotation
// needs no exchange between lanes; the rows of W_up[h] for the lane's dims are read through L1
// (every warp of every CTA reads the same d x r block), 8 columns at a time, and applied to all
// of the warp's tokens.  The pass is bound by instruction issue, not memory: three CTAs per SM
// (no spills) issue faster than two; four spill.
constexpr int kQhTpw = kQhTokens / (kQhThreads / 32);
template <typename T, int DD>
__global__ void __launch_bounds__(kQhThreads, 3)
    qcal_hope_kernel(int64_t N_q, int64_t Hq, int64_t q_pos0, int r, double base,
                     double train_len, const T* __restrict__ q, const float* __restrict__ u,
                     const T* __restrict__ W_up, T* __restrict__ q_out, T* __restrict__ qc_out) {
  constexpr int EPL = DD / 32;   // dims per lane
  constexpr int HP = EPL / 2;    // pairs per lane
  constexpr int HALF = DD / 2;
  __shared__ float2 sCS[kQhTokens * HALF];
  const int64_t b = blockIdx.y;
  const int64_t i0 = (int64_t)blockIdx.x * kQhTokens;
  angle_table<DD>(sCS, q_pos0 + i0, base, train_len);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = lane * HP;      // element e < HP: dim m0 + e; e >= HP: dim HALF + m0 + e - HP
  const int t0 = warp * kQhTpw;
  const bool vec_w = r % (sizeof(T) == 2 ? 8 : 4) == 0;
  for (int64_t h = 0; h < Hq; ++h) {
    float x[kQhTpw][EPL], c[kQhTpw][EPL], ua[kQhTpw], ub[kQhTpw];
#pragma unroll
    for (int tt = 0; tt < kQhTpw; ++tt) {
      const int64_t i = i0 + t0 + tt;
      if (i < N_q) {
        const T* qr = q + ((b * Hq + h) * N_q + i) * DD;
        float lo[HP], hi[HP];
        load_n<T, HP>(qr + m0, lo);
        load_n<T, HP>(qr + HALF + m0, hi);
#pragma unroll
        for (int k = 0; k < HP; ++k) { x[tt][k] = lo[k]; x[tt][HP + k] = hi[k]; }
        const float* ur = u + (b * N_q + i) * (Hq * r) + h * r;
        ua[tt] = lane < r ? ur[lane] : 0.f;
        ub[tt] = lane + 32 < r ? ur[lane + 32] : 0.f;
      } else {
#pragma unroll
        for (int e = 0; e < EPL; ++e) x[tt][e] = 0.f;
        ua[tt] = ub[tt] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < EPL; ++e) c[tt][e] = x[tt][e];
    }
    // the rows of W_up[h] (d x r) of this lane's dims: element e's row at wrow(e)
    const T* wlo = W_up + (h * DD + m0) * r;
    const T* whi = wlo + HALF * r;
    auto wrow = [&](int e) { return e < HP ? wlo + e * r : whi + (e - HP) * r; };
    for (int j0 = 0; j0 < r; j0 += 8) {
      float w[EPL][8];
      if (vec_w && j0 + 8 <= r) {   // 16-byte pieces of the rows (r a multiple of 8 / 4)
#pragma unroll
        for (int e = 0; e < EPL; ++e) load_piece8<T>(wrow(e) + j0, w[e]);
      } else {
#pragma unroll
        for (int e = 0; e < EPL; ++e)
#pragma unroll
          for (int jj = 0; jj < 8; ++jj)
            w[e][jj] = j0 + jj < r ? Elem<T>::to_f(__ldg(wrow(e) + j0 + jj)) : 0.f;
      }
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const int j = j0 + jj;   // (warp-uniform)
        if (j >= r) break;
#pragma unroll
        for (int tt = 0; tt < kQhTpw; ++tt) {
          const float uj = __shfl_sync(0xffffffffu, j < 32 ? ua[tt] : ub[tt], j & 31);
#pragma unroll
          for (int e = 0; e < EPL; ++e) c[tt][e] = fmaf(w[e][jj], uj, c[tt][e]);
        }
      }
    }
#pragma unroll
    for (int tt = 0; tt < kQhTpw; ++tt) {
      const int64_t i = i0 + t0 + tt;
      const float2* cs_row = sCS + (t0 + tt) * HALF + m0;
#pragma unroll
      for (int k = 0; k < HP; ++k) {   // pair m0 + k: (m, m + d/2) turned by its angle
        const float2 cs = cs_row[k];
        const float xa = x[tt][k], xb = x[tt][HP + k];
        x[tt][k] = xa * cs.x - xb * cs.y;
        x[tt][HP + k] = xa * cs.y + xb * cs.x;
        const float ca = c[tt][k], cb = c[tt][HP + k];
        c[tt][k] = ca * cs.x - cb * cs.y;
        c[tt][HP + k] = ca * cs.y + cb * cs.x;
      }
      if (i < N_q) {
        const int64_t row = (b * Hq + h) * N_q + i;
        float lo[HP], hi[HP];
#pragma unroll
        for (int k = 0; k < HP; ++k) { lo[k] = x[tt][k]; hi[k] = x[tt][HP + k]; }
        store_n<T, HP>(q_out + row * DD + m0, lo);
        store_n<T, HP>(q_out + row * DD + HALF + m0, hi);
#pragma unroll
        for (int k = 0; k < HP; ++k) { lo[k] = c[tt][k]; hi[k] = c[tt][HP + k]; }
        store_n<T, HP>(qc_out + row * DD + m0, lo);
        store_n<T, HP>(qc_out + row * DD + HALF + m0, hi);
      }
    }
  }
}

// bf16, d = 128, r a multiple of 16: the correction of a block's 32 tokens, one head at a time,
// as a product on the tensor cores, dq[128 dims x 32 tokens] = W_up[h] [128 x r] . u^T [r x 32],
// with m16n8k16 tiles (bf16 operands, fp32 accumulators).  W_up[h] is bf16 already; u (fp32,
// from the down-projection) enters as two bf16 parts, hi = bf16(u) and lo = bf16(u - hi), each
// multiplied in turn, so the product keeps u to about 2^-17 of itself.  Warp w takes the dim
// tiles mp = w % 4 and mp + 4 (so a lane holds dims m and m + 64, whole rotation pairs) and the
// token tiles 2 (w / 4) and 2 (w / 4) + 1.  The head's q tile [32 tokens x 128] is staged in
// shared memory by 16-byte loads, the turned q and q_cal tiles are written there in the
// accumulator's order and stored by 16-byte writes (rows padded to 136 elements so the
// fragment-order accesses spread over the banks).  Two barriers per head order the reuse.
constexpr int kQmLd = 136;   // staged row stride (elements)
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void split_bf16x2(float x, float y, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x - __low2float(h), y - __high2float(h));
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

__global__ void __launch_bounds__(kQhThreads, 3)
    qcal_hope_mma_kernel(int64_t N_q, int64_t Hq, int64_t q_pos0, int r, double base,
                         double train_len, const __nv_bfloat16* __restrict__ q,
                         const float* __restrict__ u, const __nv_bfloat16* __restrict__ W_up,
                         __nv_bfloat16* __restrict__ q_out, __nv_bfloat16* __restrict__ qc_out) {
  constexpr int DD = 128, HALF = 64;
  static_assert(kQhTokens == 32 && kQhThreads == 256, "8 warps x (2 dim tiles, 2 token tiles)");
  __shared__ float2 sCS[kQhTokens * HALF];
  __shared__ __align__(16) __nv_bfloat16 sQ[kQhTokens * kQmLd];
  __shared__ __align__(16) __nv_bfloat16 sX[kQhTokens * kQmLd];
  __shared__ __align__(16) __nv_bfloat16 sC[kQhTokens * kQmLd];
  const int64_t b = blockIdx.y;
  const int64_t i0 = (int64_t)blockIdx.x * kQhTokens;
  angle_table<DD>(sCS, q_pos0 + i0, base, train_len);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tq = lane & 3;   // fragment row group and thread in group
  const int mp = warp & 3;                  // dim tiles mp and mp + 4
  const int nt0 = 2 * (warp >> 2);          // token tiles nt0 and nt0 + 1
  // 16-byte pieces of the 32 x 128 tile: two per thread (piece p: token p / 16, dims 8 (p % 16))
  constexpr int kPieces = kQhTokens * DD / 8;
  for (int64_t h = 0; h < Hq; ++h) {
    const int64_t row0 = ((b * Hq + h) * N_q + i0) * DD;   // the block's first token row
#pragma unroll
    for (int p = threadIdx.x; p < kPieces; p += kQhThreads) {
      const int t = p >> 4, c8 = (p & 15) * 8;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (i0 + t < N_q) v = __ldg(reinterpret_cast<const uint4*>(q + row0 + t * DD + c8));
      *reinterpret_cast<uint4*>(sQ + t * kQmLd + c8) = v;
    }
    float acc[2][2][4];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[a][n][e] = 0.f;
    for (int kc = 0; kc < r; kc += 16) {
      uint32_t af[2][4];
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        const __nv_bfloat16* w0 = W_up + (h * DD + 16 * (mp + 4 * a) + g) * r + kc + 2 * tq;
        const __nv_bfloat16* w1 = w0 + 8 * r;
        af[a][0] = __ldg(reinterpret_cast<const uint32_t*>(w0));
        af[a][1] = __ldg(reinterpret_cast<const uint32_t*>(w1));
        af[a][2] = __ldg(reinterpret_cast<const uint32_t*>(w0 + 8));
        af[a][3] = __ldg(reinterpret_cast<const uint32_t*>(w1 + 8));
      }
#pragma unroll
      for (int n = 0; n < 2; ++n) {
        const int64_t i = i0 + 8 * (nt0 + n) + g;   // this lane's token of the B fragment
        float2 u0 = make_float2(0.f, 0.f), u1 = make_float2(0.f, 0.f);
        if (i < N_q) {
          const float* ur = u + (b * N_q + i) * (Hq * r) + h * r + kc + 2 * tq;
          u0 = __ldg(reinterpret_cast<const float2*>(ur));
          u1 = __ldg(reinterpret_cast<const float2*>(ur + 8));
        }
        uint32_t b0h, b0l, b1h, b1l;
        split_bf16x2(u0.x, u0.y, b0h, b0l);
        split_bf16x2(u1.x, u1.y, b1h, b1l);
#pragma unroll
        for (int a = 0; a < 2; ++a) {
          mma_bf16_16816(acc[a][n], af[a], b0h, b1h);
          mma_bf16_16816(acc[a][n], af[a], b0l, b1l);
        }
      }
    }
    __syncthreads();   // the q tile (and, for h = 0, the angle table) is in place; the previous
                       // head's output tiles have been stored
    // accumulator element e of token tile n: dim 16 * tile + g + 8 * (e >> 1), token
    // 8 * (nt0 + n) + 2 * tq + (e & 1); tiles mp and mp + 4 hold the two dims of a pair
#pragma unroll
    for (int n = 0; n < 2; ++n) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int t = 8 * (nt0 + n) + 2 * tq + (e & 1);   // token in the block
        const int m = 16 * mp + g + 8 * (e >> 1);          // pair (m, m + 64)
        const float xa = __bfloat162float(sQ[t * kQmLd + m]);
        const float xb = __bfloat162float(sQ[t * kQmLd + HALF + m]);
        const float ca = xa + acc[0][n][e], cb = xb + acc[1][n][e];
        const float2 cs = sCS[t * HALF + m];
        sX[t * kQmLd + m] = __float2bfloat16_rn(xa * cs.x - xb * cs.y);
        sX[t * kQmLd + HALF + m] = __float2bfloat16_rn(xa * cs.y + xb * cs.x);
        sC[t * kQmLd + m] = __float2bfloat16_rn(ca * cs.x - cb * cs.y);
        sC[t * kQmLd + HALF + m] = __float2bfloat16_rn(ca * cs.y + cb * cs.x);
      }
    }
    __syncthreads();   // both output tiles complete; sQ free for the next head
#pragma unroll
    for (int p = threadIdx.x; p < kPieces; p += kQhThreads) {
      const int t = p >> 4, c8 = (p & 15) * 8;
      if (i0 + t < N_q) {
        *reinterpret_cast<uint4*>(q_out + row0 + t * DD + c8) =
            *reinterpret_cast<const uint4*>(sX + t * kQmLd + c8);
        *reinterpret_cast<uint4*>(qc_out + row0 + t * DD + c8) =
            *reinterpret_cast<const uint4*>(sC + t * kQmLd + c8);
      }
    }
  }
}

// x [B H, N, d] -> R(x), token n at position pos0 + n; grid (token blocks), every (b, h) in turn.
template <typename T, int DD>
__global__ void __launch_bounds__(kQhThreads)
    hope_rotate_kernel(int64_t BH, int64_t N, int64_t pos0, double base, double train_len,
                       const T* __restrict__ x, T* __restrict__ out) {
  constexpr int HP = DD / 64;   // whole pairs per lane
  constexpr int HALF = DD / 2;
  __shared__ float2 sCS[kQhTokens * HALF];
  const int64_t n0 = (int64_t)blockIdx.x * kQhTokens;
  angle_table<DD>(sCS, pos0 + n0, base, train_len);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = lane * HP;
  for (int64_t bh = 0; bh < BH; ++bh) {
    for (int t = warp; t < kQhTokens; t += kQhThreads / 32) {
      const int64_t n = n0 + t;
      if (n >= N) break;
      const int64_t row = bh * N + n;
      // this lane's pairs m0 .. m0 + HP - 1 with their partners m + d/2 (in place is safe: a
      // lane writes back exactly the elements it read)
      float lo[HP], hi[HP];
      load_n<T, HP>(x + row * DD + m0, lo);
      load_n<T, HP>(x + row * DD + HALF + m0, hi);
#pragma unroll
      for (int k = 0; k < HP; ++k) {
        const float2 cs = sCS[t * HALF + m0 + k];
        const float a = lo[k], bb = hi[k];
        lo[k] = a * cs.x - bb * cs.y;
        hi[k] = a * cs.y + bb * cs.x;
      }
      store_n<T, HP>(out + row * DD + m0, lo);
      store_n<T, HP>(out + row * DD + HALF + m0, hi);
    }
  }
}

}  // namespace

bool qdown_supported(int64_t N, int64_t d_model) {
  return d_model >= 64 && d_model % 64 == 0 && N >= 64 && N % 64 == 0;
}

cudaError_t launch_qdown(int64_t M, int64_t N, int64_t d_model, const void* hidden,
                         const void* W_down, float* u, int32_t* status, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  if (N % 256 == 0) return launch_qdown_t<256>(M, N, d_model, hidden, W_down, u, status, st);
  if (N % 128 == 0) return launch_qdown_t<128>(M, N, d_model, hidden, W_down, u, status, st);
  return launch_qdown_t<64>(M, N, d_model, hidden, W_down, u, status, st);
}

cudaError_t launch_qcal_hope(int64_t B, int64_t Hq, int64_t N_q, int64_t d, int64_t q_pos0,
                             int r, double base, double train_len, bool bf16, const void* q,
                             const float* u, const void* W_up, void* q_out, void* qc_out,
                             cudaStream_t st) {
  if (B == 0 || N_q == 0) return cudaSuccess;
  const dim3 grid((unsigned)((N_q + kQhTokens - 1) / kQhTokens), (unsigned)B);
#define HILS_QH(TT, DDV)                                                                      \
  qcal_hope_kernel<TT, DDV><<<grid, kQhThreads, 0, st>>>(                                      \
      N_q, Hq, q_pos0, r, base, train_len, static_cast<const TT*>(q), u,                       \
      static_cast<const TT*>(W_up), static_cast<TT*>(q_out), static_cast<TT*>(qc_out))
  if (bf16) {
    if (d == 128 && r > 0 && r % 16 == 0)
      qcal_hope_mma_kernel<<<grid, kQhThreads, 0, st>>>(
          N_q, Hq, q_pos0, r, base, train_len, static_cast<const __nv_bfloat16*>(q), u,
          static_cast<const __nv_bfloat16*>(W_up), static_cast<__nv_bfloat16*>(q_out),
          static_cast<__nv_bfloat16*>(qc_out));
    else if (d == 128) HILS_QH(__nv_bfloat16, 128);
    else HILS_QH(__nv_bfloat16, 64);
  } else {
    if (d == 128) HILS_QH(float, 128);
    else HILS_QH(float, 64);
  }
#undef HILS_QH
  return cudaGetLastError();
}

cudaError_t launch_hope_rotate(int64_t BH, int64_t N, int64_t d, int64_t pos0, double base,
                               double train_len, bool bf16, const void* x, void* out,
                               cudaStream_t st) {
  if (BH == 0 || N == 0) return cudaSuccess;
  const dim3 grid((unsigned)((N + kQhTokens - 1) / kQhTokens));
#define HILS_HR(TT, DDV)                                                                      \
  hope_rotate_kernel<TT, DDV><<<grid, kQhThreads, 0, st>>>(                                   \
      BH, N, pos0, base, train_len, static_cast<const TT*>(x), static_cast<TT*>(out))
  if (bf16) {
    if (d == 128) HILS_HR(__nv_bfloat16, 128);
    else HILS_HR(__nv_bfloat16, 64);
  } else {
    if (d == 128) HILS_HR(float, 128);
    else HILS_HR(float, 64);
  }
#undef HILS_HR
  return cudaGetLastError();
}

}  // namespace hils
