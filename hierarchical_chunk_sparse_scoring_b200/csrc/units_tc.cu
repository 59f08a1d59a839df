// Step 3 for decode on the tcgen05 tensor cores: per-unit exact attention (o_u, lse_u) of the
// G heads of a (b, g, query) row over each selected chunk and each window piece of S tokens
// (S = 64 or 128).
//
// [Reader] Fig. 3 caption and [Abstract]: each retrieved chunk is attended on its own, with its
// own softmax, and the per-chunk outputs are fused later by the retrieval scores; the local
// window is one more unit (here cut into pieces of 64 tokens, recombined by their lse in the
// fusion).  In decode the step streams the selected K/V chunks from HBM; the arithmetic is put on
// the tensor core so the SMs only move data:
//   * a tile is 128 tokens of one row: two units when S = 64, one unit when S = 128 (its two
//     64-token halves); their K rows form the 128-row A operand, the row's G query heads
//     (N = 16 rows; rows past G are never read) the B operand: S = K_tile . Q^T (M = 128 tokens,
//     N = 16, K = d);
//   * the softmax warps (one token per thread) take each unit's max and sum over its tokens per
//     head and write P (bf16) as a K-major [16 heads x 128 tokens] operand;
//   * O_u^T = V_u^T . P_u (M = d = 128, N = 16, K = 64 tokens per half; V read as an MN-major
//     operand): per half into its own accumulator when the halves are two units, both halves
//     into one when they are one; the epilogue (one d-row per thread) divides by the unit's sum.
// Persistent CTAs, three per SM, each with one stage whose K and V halves are released
// separately: the next tile's K (and queries) load once this tile's Q.K^T has read K, its V once
// the P.V products have read V, so both copies overlap this tile's softmax and output phases.
// Every mbarrier wait gives up after a bounded number of polls and records HILS_ERR_TIMEOUT.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace hils {
using namespace sm100;

namespace {

constexpr int kUtThreads = 192;
constexpr int kUtTok = 64;          // tokens per tile half (S = 64: one unit; S = 128: half of one)
constexpr int kUtRows = 128;        // tokens per tile
constexpr int kUtCols = 16;         // query heads per tile (MMA N)
constexpr int kUtD = 128;           // head dim (MMA M of the P.V product)
constexpr int kUtCtasPerSm = 3;
constexpr uint32_t kUtPoll = 1u << 24;
constexpr uint32_t kUtTmemCols = 64;   // S (16) | pad | O of unit A (16) | O of unit B (16)
constexpr uint32_t kColS = 0, kColOA = 32, kColOB = 48;

struct UtShape {
  static constexpr int KB = kUtD / 64;
  static constexpr int UNIT_BOX = kUtTok * 128;          // [64 tokens x 64] bf16, 8 KB
  static constexpr int BLK = kUtRows * 128;              // [128 tokens x 64], 16 KB
  static constexpr int KT = KB * BLK;                    // K (or V) tile
  static constexpr int Q_BOX = kUtCols * 128;            // [16 heads x 64], 2 KB
  static constexpr int QT = KB * Q_BOX;
  static constexpr int STAGE = 2 * KT + QT;
  static constexpr int P_BLK = kUtCols * 128;            // [16 heads x 64 tokens] bf16
  static constexpr int P_BYTES = 2 * P_BLK;
  // barriers and the TMEM address, then two reduction arrays [2 parities][4 warps][16 heads]
  static constexpr int TAIL = 64 + 2 * 2 * 4 * kUtCols * 4;
  static constexpr int SMEM = 1024 /*align*/ + STAGE + P_BYTES + TAIL;
  static_assert(SMEM * kUtCtasPerSm <= 227 * 1024, "three CTAs per SM");
  static_assert(kUtCtasPerSm * kUtTmemCols <= 512, "TMEM columns");
};

// Unit x of a row: token range start and length (0: empty unit); units are S tokens long.
__device__ __forceinline__ void unit_span(const Dims& D, const int32_t* __restrict__ idx,
                                          int64_t row, int64_t n, int64_t pos, int n_units, int x,
                                          int64_t& t0, int& len) {
  t0 = 0;
  len = 0;
  if (x < D.K) {
    const int c = __ldg(idx + row * D.K + x);
    if (c >= 0 && c < n) { t0 = (int64_t)c * D.S; len = D.S; }
  } else if (x < n_units) {
    const int64_t s = (int64_t)D.S * n + (int64_t)(x - D.K) * D.S;
    const int64_t l = pos + 1 - s;
    t0 = s;
    len = l <= 0 ? 0 : (l >= D.S ? D.S : (int)l);
  }
}

}  // namespace

// GM: a bound on the group's heads (4, 8 or 16), so the per-head loops unroll to G's size.
template <int GM>
__global__ void __launch_bounds__(kUtThreads, kUtCtasPerSm)
    attn_units_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, Dims D, int n_pieces,
                         int64_t tiles_per_row, int64_t n_tiles_total,
                         const int32_t* __restrict__ idx, float* __restrict__ part_o,
                         float* __restrict__ part_lse, int32_t* __restrict__ status) {
  using SH = UtShape;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sK = smem;
  uint8_t* sV = sK + SH::KT;
  uint8_t* sQ = sV + SH::KT;
  uint8_t* sP = sQ + SH::QT;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + SH::P_BYTES);
  uint64_t* k_full = bars;        // K and Q of the tile landed
  uint64_t* v_full = bars + 1;    // V landed
  uint64_t* k_empty = bars + 2;   // Q.K^T has read K and Q
  uint64_t* v_empty = bars + 3;   // P.V has read V
  uint64_t* s_full = bars + 4;
  uint64_t* p_full = bars + 5;
  uint64_t* o_full = bars + 6;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 7);
  float* red_m = reinterpret_cast<float*>(bars + 8);   // [2 parities][4 warps][16 heads]
  float* red_l = red_m + 2 * 4 * kUtCols;              // [2][4][16]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_units = D.K + n_pieces;
  const bool wide = D.S == kUtRows;   // one unit per tile (S = 128), else two (S = 64)
  const int64_t t_begin = n_tiles_total * blockIdx.x / gridDim.x;
  const int64_t t_end = n_tiles_total * (blockIdx.x + 1) / gridDim.x;
  const int n_local = (int)(t_end - t_begin);

  if (threadIdx.x == 0) {
    mbar_init(k_full, 1);
    mbar_init(v_full, 1);
    mbar_init(k_empty, 1);
    mbar_init(v_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, 4);
    mbar_init(o_full, 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_holder, kUtTmemCols);
  // P rows of heads >= GM are never written in the loop: zero them once (they only feed output
  // columns nobody reads, but stay finite)
  for (int e = threadIdx.x; e < SH::P_BYTES / 16; e += kUtThreads)
    reinterpret_cast<uint4*>(sP)[e] = make_uint4(0u, 0u, 0u, 0u);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0 && n_local > 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      // token rows of a tile's two halves (the idx reads of the next tile are issued before
      // the waits for the current stage, so their latency hides behind them)
      auto spans = [&](int u, int32_t (&y)[2], int32_t& qi, int32_t& qh) {
        const int64_t t = t_begin + u;
        const int64_t row = t / tiles_per_row, pr = t - row * tiles_per_row;
        const int64_t i = row % D.N_q, bg = row / D.N_q;
        const int64_t g = bg % D.Hkv, b = bg / D.Hkv;
        const int64_t pos = D.q_pos0 + i, n = n_eligible(pos, D.S, D.W);
        // an empty unit, or a unit's missing second half, still loads (from token 0 of the row,
        // or past the unit's end); the softmax masks those tokens
        if (wide) {
          int64_t t0;
          int len;
          unit_span(D, idx, row, n, pos, n_units, (int)pr, t0, len);
          y[0] = (int32_t)(bg * D.N_kv + t0);
          y[1] = y[0] + kUtTok;
        } else {
          for (int half = 0; half < 2; ++half) {
            int64_t t0;
            int len;
            unit_span(D, idx, row, n, pos, n_units, (int)(2 * pr + half), t0, len);
            y[half] = (int32_t)(bg * D.N_kv + t0);
          }
        }
        qi = (int32_t)i;
        qh = (int32_t)(b * D.Hq + g * D.G);
      };
      int32_t y[2], qi, qh;
      spans(0, y, qi, qh);
      bool ok = true;
      for (int u = 0; u < n_local; ++u) {
        const uint32_t ph = (uint32_t)u & 1u;
        if (!mbar_wait(k_empty, ph ^ 1u, kUtPoll)) { ok = false; break; }
        mbar_expect_tx(k_full, 2 * SH::KB * SH::UNIT_BOX + SH::QT);
        for (int half = 0; half < 2; ++half)
          for (int kb = 0; kb < SH::KB; ++kb)
            tma_load_2d(sK + kb * SH::BLK + half * SH::UNIT_BOX, &tmK, kb * 64, y[half], k_full);
        for (int kb = 0; kb < SH::KB; ++kb)
          asm volatile(
              "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
              " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(sQ + kb * SH::Q_BOX)),
              "l"(reinterpret_cast<uint64_t>(&tmQ)), "r"(kb * 64), "r"(qi), "r"(qh),
              "r"(smem_u32(k_full))
              : "memory");
        if (!mbar_wait(v_empty, ph ^ 1u, kUtPoll)) { ok = false; break; }
        mbar_expect_tx(v_full, 2 * SH::KB * SH::UNIT_BOX);
        for (int half = 0; half < 2; ++half)
          for (int kb = 0; kb < SH::KB; ++kb)
            tma_load_2d(sV + kb * SH::BLK + half * SH::UNIT_BOX, &tmV, kb * 64, y[half], v_full);
        if (u + 1 < n_local) spans(u + 1, y, qi, qh);
      }
      if (!ok) record_status(status, kStatusTimeout);
      // this thread's copies have landed before it leaves (bounded)
      if (ok) {
        mbar_wait(k_full, (uint32_t)(n_local - 1) & 1u, kUtPoll);
        mbar_wait(v_full, (uint32_t)(n_local - 1) & 1u, kUtPoll);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0 && n_local > 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(kUtRows, kUtCols);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(kUtD, kUtCols) | (1u << 15);   // A MN-major
      bool ok = true;
      for (int u = 0; ok && u < n_local; ++u) {
        const uint32_t ph = (uint32_t)u & 1u;
        if (!mbar_wait(k_full, ph, kUtPoll)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kUtD / 16; ++ks) {
          const int kb = ks >> 2, kin = ks & 3;
          mma_bf16_ss(tmem + kColS, desc_kmajor_sw128(smem_u32(sK + kb * SH::BLK) + kin * 32),
                      desc_kmajor_sw128(smem_u32(sQ + kb * SH::Q_BOX) + kin * 32), IDESC_S,
                      ks > 0 ? 1u : 0u);
        }
        mma_commit(s_full);
        mma_commit(k_empty);
        if (!mbar_wait(p_full, ph, kUtPoll) || !mbar_wait(v_full, ph, kUtPoll)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int half = 0; half < 2; ++half) {
#pragma unroll
          for (int ks = 0; ks < kUtTok / 16; ++ks) {
            // A = V^T: d is the contiguous (MN) dimension, 16 tokens per K step
            const uint64_t ad = desc_mnmajor_sw128(
                smem_u32(sV + half * SH::UNIT_BOX + ks * 16 * 128), SH::BLK);
            const uint64_t bd = desc_kmajor_sw128(smem_u32(sP + half * SH::P_BLK) + ks * 32);
            // two units: one accumulator each; one unit: both halves into the first.  (One MMA
            // statement with the column and the accumulate flag as values: the same choice
            // written as two MMA statements under a branch gave wrong S = 64 results.)
            const uint32_t col = (wide || half == 0) ? kColOA : kColOB;
            const uint32_t acc = (ks > 0 || (wide && half > 0)) ? 1u : 0u;
            mma_bf16_ss(tmem + col, ad, bd, IDESC_O, acc);
          }
        }
        mma_commit(o_full);
        mma_commit(v_empty);
      }
      if (!ok) record_status(status, kStatusTimeout);
    }
  } else {
    // ---------------------------------------------------------------- softmax and outputs
    const int qd = warp & 3;                      // TMEM lane quadrant
    const int tk = qd * 32 + lane;                // token of the tile (S phase) / d-row (O phase)
    const int half = qd >> 1;                     // which unit this thread's token belongs to
    const uint32_t lane_base = tmem + ((uint32_t)(qd * 32) << 16);
    const int G = D.G;
    bool ok = true;
    for (int u = 0; u < n_local; ++u) {
      const uint32_t ph = (uint32_t)u & 1u;
      const int64_t t = t_begin + u;
      const int64_t row = t / tiles_per_row, pr = t - row * tiles_per_row;
      const int64_t i = row % D.N_q, bg = row / D.N_q;
      const int64_t g = bg % D.Hkv, b = bg / D.Hkv;
      const int64_t pos = D.q_pos0 + i, n = n_eligible(pos, D.S, D.W);
      int64_t t0a, t0b;
      int lena, lenb;
      bool tok_ok;
      if (wide) {
        unit_span(D, idx, row, n, pos, n_units, (int)pr, t0a, lena);
        tok_ok = tk < lena;
      } else {
        unit_span(D, idx, row, n, pos, n_units, (int)(2 * pr), t0a, lena);
        unit_span(D, idx, row, n, pos, n_units, (int)(2 * pr + 1), t0b, lenb);
        tok_ok = (tk & 63) < (half ? lenb : lena);
      }
      float* rm = red_m + ph * 4 * kUtCols;
      float* rl = red_l + ph * 4 * kUtCols;
      // ---- logits of this thread's token for the 16 head columns.  A failed (timed-out) wait
      // does not leave the loop: the four warps meet at named barriers on every tile, so after
      // a failure a warp only skips its waits and TMEM accesses (ok is warp-uniform).
      if (ok) ok = mbar_wait_warp(s_full, ph, kUtPoll);
      float x[kUtCols];
      if (ok) {
        tc_fence_after();
        tmem_ld16(lane_base + kColS, x);
        tmem_wait_ld();
      }
#pragma unroll
      for (int h = 0; h < GM; ++h) x[h] = (ok && tok_ok && h < G) ? x[h] * D.scale : -INFINITY;
      // ---- unit max per head over the unit's warps (two, or all four when the tile is one unit)
#pragma unroll
      for (int h = 0; h < GM; ++h) {
        if (h >= G) break;
        const float wm = warp_max(x[h]);
        if (lane == 0) rm[qd * kUtCols + h] = wm;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      float p[GM];
#pragma unroll
      for (int h = 0; h < GM; ++h) {
        p[h] = 0.f;
        if (h >= G) continue;
        float m = fmaxf(rm[qd * kUtCols + h], rm[(qd ^ 1) * kUtCols + h]);
        if (wide) m = fmaxf(m, fmaxf(rm[(qd ^ 2) * kUtCols + h], rm[(qd ^ 3) * kUtCols + h]));
        p[h] = (x[h] == -INFINITY) ? 0.f : __expf(x[h] - m);
        const float ws = warp_sum(p[h]);
        if (lane == 0) rl[qd * kUtCols + h] = ws;
      }
      // ---- P (bf16) as the K-major [16 heads x 128 tokens] operand, 128-byte swizzle
      {
        uint8_t* pb = sP + half * SH::P_BLK;
        const int tt = tk & 63;
#pragma unroll
        for (int h = 0; h < GM; ++h) {
          const int off = (h >> 3) * 1024 + (h & 7) * 128 + ((((tt >> 3) ^ (h & 7))) << 4) +
                          (tt & 7) * 2;
          *reinterpret_cast<__nv_bfloat16*>(pb + off) = __float2bfloat16_rn(p[h]);
        }
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(p_full);
      asm volatile("bar.sync 1, 128;" ::: "memory");   // unit sums complete
      // ---- O of both units: this thread is d-row tk
      if (ok) ok = mbar_wait_warp(o_full, ph, kUtPoll);
      if (!ok) continue;
      tc_fence_after();
      float oa[kUtCols], ob[kUtCols];
      tmem_ld16(lane_base + kColOA, oa);
      tmem_ld16(lane_base + kColOB, ob);
      tmem_wait_ld();
      if (wide) {
#pragma unroll
        for (int h = 0; h < GM; ++h) {
          if (h >= G) break;
          const int64_t hrow = (b * D.Hq + g * G + h) * D.N_q + i;
          const float l = (rl[0 * kUtCols + h] + rl[1 * kUtCols + h]) +
                          (rl[2 * kUtCols + h] + rl[3 * kUtCols + h]);
          part_o[(hrow * n_units + pr) * kUtD + tk] = l > 0.f ? oa[h] / l : 0.f;
          if (tk == 0) {
            const float m = fmaxf(fmaxf(rm[0 * kUtCols + h], rm[1 * kUtCols + h]),
                                  fmaxf(rm[2 * kUtCols + h], rm[3 * kUtCols + h]));
            part_lse[hrow * n_units + pr] = l > 0.f ? m + logf(l) : -INFINITY;
          }
        }
        continue;
      }
      const int ua = (int)(2 * pr), ub = ua + 1;
#pragma unroll
      for (int h = 0; h < GM; ++h) {
        if (h >= G) break;
        const int64_t hrow = (b * D.Hq + g * G + h) * D.N_q + i;
        const float la = rl[0 * kUtCols + h] + rl[1 * kUtCols + h];
        const float lb = rl[2 * kUtCols + h] + rl[3 * kUtCols + h];
        part_o[(hrow * n_units + ua) * kUtD + tk] = la > 0.f ? oa[h] / la : 0.f;
        if (ub < n_units) part_o[(hrow * n_units + ub) * kUtD + tk] = lb > 0.f ? ob[h] / lb : 0.f;
        if (tk == 0) {
          const float ma = fmaxf(rm[0 * kUtCols + h], rm[1 * kUtCols + h]);
          const float mb = fmaxf(rm[2 * kUtCols + h], rm[3 * kUtCols + h]);
          part_lse[hrow * n_units + ua] = la > 0.f ? ma + logf(la) : -INFINITY;
          if (ub < n_units) part_lse[hrow * n_units + ub] = lb > 0.f ? mb + logf(lb) : -INFINITY;
        }
      }
    }
    if (!ok) record_status(status, kStatusTimeout);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kUtTmemCols);
}

// ---------------------------------------------------------------------------------------------
namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode_ut() {
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

bool map_rows(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
  auto enc = get_encode_ut();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kUtD, rows};
  cuuint64_t strides[1] = {(cuuint64_t)kUtD * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool units_tc_supported(const Dims& D, bool bf16) {
  if (!bf16 || D.d != kUtD || (D.S != kUtTok && D.S != kUtRows) || D.G < 1 || D.G > kUtCols)
    return false;
  // token rows are int32 TMA coordinates, the second half of a unit up to 64 past its end
  if (D.B * D.Hkv * D.N_kv + kUtRows >= (int64_t)INT32_MAX) return false;
  if (D.B * D.Hq >= (int64_t)INT32_MAX || D.N_q >= (int64_t)INT32_MAX) return false;
  return true;
}

cudaError_t launch_attn_units_tc(const Dims& D, int n_pieces, const void* q, const void* K,
                                 const void* V, const int32_t* idx, float* part_o,
                                 float* part_lse, int32_t* status, cudaStream_t st) {
  const int64_t rows = D.B * D.Hkv * D.N_q;
  const int n_units = D.K + n_pieces;
  if (rows == 0 || n_units == 0) return cudaSuccess;
  auto enc = get_encode_ut();
  if (!enc) return cudaErrorInvalidValue;
  CUtensorMap tmQ, tmK, tmV;
  if (!map_rows(&tmK, K, (uint64_t)(D.B * D.Hkv * D.N_kv), kUtTok) ||
      !map_rows(&tmV, V, (uint64_t)(D.B * D.Hkv * D.N_kv), kUtTok))
    return cudaErrorInvalidValue;
  {
    // q as [B*Hq][N_q][d], boxes of [16 heads, 1 query, 64]
    cuuint64_t dims[3] = {(cuuint64_t)kUtD, (cuuint64_t)D.N_q, (cuuint64_t)(D.B * D.Hq)};
    cuuint64_t strides[2] = {(cuuint64_t)kUtD * 2, (cuuint64_t)(D.N_q * kUtD * 2)};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)kUtCols};
    cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const int64_t tiles_per_row = D.S == kUtRows ? n_units : (n_units + 1) / 2;
  const int64_t total = rows * tiles_per_row;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int64_t slots = (int64_t)kUtCtasPerSm * sms;
  const int64_t grid = total < slots ? total : slots;
  auto kern = D.G <= 4 ? attn_units_tc_kernel<4>
                        : D.G <= 8 ? attn_units_tc_kernel<8> : attn_units_tc_kernel<16>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, UtShape::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)grid, kUtThreads, UtShape::SMEM, st>>>(
      tmQ, tmK, tmV, D, n_pieces, tiles_per_row, total, idx, part_o, part_lse, status);
  return cudaGetLastError();
}

}  // namespace hils
