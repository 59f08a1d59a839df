// Steps 3-4 for prefill on the tcgen05 tensor cores (bf16 inputs, fp32 accumulation, S = 64 or
// 128).  The unit of work is a tile of 64 tokens; with S = 128 a chunk is two adjacent tiles of
// the list, and its intra-chunk softmax is taken over both at the first one (the second tile's
// logits are already in the other S buffer of TMEM): the first tile's P and the second's share
// one max and one normaliser.
//
// [Reader] "Implementation and Training Recipes", Figure 4: pack M adjacent queries and the G
// heads of their KV group into one tile of M*G rows and attend the union of the rows' chunks,
// so one (M*G, d) x (d, S) product serves every row that uses the chunk.  Here M*G = 128 rows
// (the tcgen05 tile height).  The union is taken over the queries' selected chunks plus the
// chunks their local windows cover; for each (row, tile) the row either
//   * selected this chunk: intra-chunk softmax with the chunk's own log-sum-exp, weighted by the
//     row's surrogate score s_{h,c} ([Reader] Fig. 3 caption: inter-chunk softmax gives a
//     chunk's mass, the intra-chunk softmax spreads it; [Abstract]: each query attends each
//     retrieved chunk independently and the outputs are fused by the retrieval scores);
//   * has the tile inside its causal local window: plain online softmax over those tokens
//     (the window is one fusion unit scored by its exact log-sum-exp);
//   * or does not use it: weight 0 (each row attends only its own chunks, so packing never
//     changes a row's result).
// Every weight is measured against one running reference m per row that starts at the row's
// largest selected-chunk score, so chunk units never rescale the accumulator; window tiles
// raise it only when a logit exceeds it by more than 8 (the O row in TMEM is then rescaled).
//
// CTA = (b, g, 128/G queries); 6 warps: warp 0 TMA (Q once, then K and V tiles of the union),
// warp 1 TMEM owner and MMA issuer (S = Q K^T into a double-buffered TMEM tile, O += P V into a
// TMEM accumulator, P read from TMEM as the A operand), warps 2-5 one row per thread
// (classification, softmax, the row's P as bf16 into its own TMEM lane).
#include <cudaTypedefs.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace hils {
using namespace sm100;

namespace {

constexpr int kAtThreads = 192;
constexpr int kAtRows = 128;
constexpr int kTile = 64;                    // tokens per tile (= chunk size S)
constexpr uint32_t kAtPollLimit = 1u << 24;
constexpr float kRescaleMargin = 8.0f;       // natural-log units
constexpr int kAtSmemLimit = 227 * 1024;

// TWO = 1: d = 128 with two CTAs per SM.  The per-head scores of the selected chunks come from
// the selection step (no calibrated-query tile, no landmark product here), P is written into its
// own S columns of TMEM (256 columns per CTA), the K/V ring has two stages and the tile bitmap is
// built in the second of them; a CTA then needs under half of the SM's shared memory, so two
// CTAs share each SM and one's softmax and prologue latencies hide behind the other's work.
template <int DD, int G, int TWO = 0>
struct AtShape {
  static constexpr int TQ = kAtRows / G;                 // queries per CTA
  static constexpr int KB = DD / 64;
  static constexpr int Q_BOX = kAtRows * 128;            // [128 rows x 64] per 64-col box
  static constexpr int Q_BYTES = KB * Q_BOX;
  static constexpr int KV_BOX = kTile * 128;             // [64 tokens x 64]
  static constexpr int KV_BYTES = KB * KV_BOX;           // one K (or V) tile
  // prologue scratch (two [128 x 128-byte] areas): the staged landmark rows, then each row's
  // parked landmark scores
  static constexpr int P_BYTES = kAtRows * 128;
  // K/V ring: STAGES_MAIN stage pairs of their own, plus one that reuses the calibrated-query
  // tile once the selected chunks' scores have been taken from it (same size: Q_BYTES = 2 KV)
  // d = 64: two CTAs per SM (each one's prologue and softmax latency hide behind the other's)
  static constexpr int STAGES_MAIN = TWO ? 2 : (DD == 128 ? 3 : 2);
  static constexpr int STAGES = TWO ? STAGES_MAIN : STAGES_MAIN + 1;
  static_assert(Q_BYTES == 2 * KV_BYTES, "the q_cal tile holds one K/V stage pair");
  static constexpr int KLM_ROWS = 64;                    // landmark rows staged in smem
  static constexpr int KLM_BYTES = KB * KLM_ROWS * 128;  // same swizzled layout as a K tile
  static constexpr int FIXED =
      TWO ? Q_BYTES + STAGES_MAIN * 2 * KV_BYTES + 256 /*bars*/ + 1024 /*align*/ + 64 /*scan*/
          : 2 * Q_BYTES /*q and q_cal*/ + STAGES_MAIN * 2 * KV_BYTES + 2 * P_BYTES +
                1024 /*bars*/ + 1024 /*align*/ + 1024 /*scan*/;
  static_assert(KLM_BYTES <= 2 * P_BYTES, "landmark rows fit the prologue scratch");
  // TMEM: S[2] (2 x 64 columns), O (DD), the landmark scores (64); a power of two.  Once the
  // landmark scores are read, their columns hold P[2]: 64 bf16 per row, two per column, the A
  // operand of the P V product.
  static constexpr uint32_t O_COL = 128;
  static constexpr uint32_t LM_COL = O_COL + DD;
  // P[x]: its own columns after the landmark scores, or (TWO) the first half of S[x]
  static constexpr uint32_t P_COL = TWO ? 0 : LM_COL;
  static constexpr uint32_t P_STRIDE = TWO ? kTile : kTile / 2;   // columns between P[0], P[1]
  static constexpr uint32_t TMEM_COLS = TWO ? 256 : (LM_COL + 64 <= 256 ? 256 : 512);
  static_assert(P_COL + P_STRIDE + kTile / 2 <= TMEM_COLS, "P buffers in TMEM");
  static_assert(!TWO || O_COL + DD <= TMEM_COLS, "S and O in 256 columns");
  // co-resident CTAs never exceed the SM's 512 TMEM columns: d = 64 and TWO run two CTAs per SM
  // on 256 columns each; otherwise d = 128 needs 512 and its shared memory footprint keeps a
  // second CTA away
  static_assert(DD == 64 || TWO ? TMEM_COLS == 256 : FIXED > 232448 / 2, "CTAs per SM");
  static_assert(DD == 64 ? FIXED < 232448 / 2 - 8192 : true, "d = 64: two CTAs per SM");
};

constexpr float kLog2e = 1.4426950408889634f;

// 2^x with the SFU's approximate base-2 exponential (ex2.approx; 2^-inf = 0).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed fp32 pairs (sm_100 f32x2 arithmetic): two lanes of work per instruction.
__device__ __forceinline__ void fma2(float& x0, float& x1, float b, float c) {   // x = x*b + c
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%0, %1};\n\tmov.b64 rb, {%2, %2};\n\tmov.b64 rd, {%3, %3};\n\t"
      "fma.rn.f32x2 ra, ra, rb, rd;\n\tmov.b64 {%0, %1}, ra;\n\t}"
      : "+f"(x0), "+f"(x1)
      : "f"(b), "f"(c));
}
__device__ __forceinline__ void add2(float& s0, float& s1, float x0, float x1) {   // s += x
  asm("{\n\t.reg .b64 ra, rb;\n\t"
      "mov.b64 ra, {%0, %1};\n\tmov.b64 rb, {%2, %3};\n\t"
      "add.rn.f32x2 ra, ra, rb;\n\tmov.b64 {%0, %1}, ra;\n\t}"
      : "+f"(s0), "+f"(s1)
      : "f"(x0), "f"(x1));
}
__device__ __forceinline__ void mul2(float& x0, float& x1, float b) {   // x *= b
  asm("{\n\t.reg .b64 ra, rb;\n\t"
      "mov.b64 ra, {%0, %1};\n\tmov.b64 rb, {%2, %2};\n\t"
      "mul.rn.f32x2 ra, ra, rb;\n\tmov.b64 {%0, %1}, ra;\n\t}"
      : "+f"(x0), "+f"(x1)
      : "f"(b));
}
__device__ __forceinline__ float fmax3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// q_cal row r (128-byte-swizzled tile) . k_lm row, for a selected chunk whose landmark row was
// not staged.  Out of line: it is rare, and one inlined copy per list slot would bloat the
// kernel.
template <int KB, int Q_BOX>
__device__ __noinline__ float lm_dot(const uint8_t* sQc, int r, const __nv_bfloat16* kr) {
  float a = 0.f;
  for (int kb = 0; kb < KB; ++kb) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint4 qv = *reinterpret_cast<const uint4*>(
          sQc + kb * Q_BOX + (r >> 3) * 1024 + (r & 7) * 128 + ((j ^ (r & 7)) << 4));
      const uint4 kv = __ldg(reinterpret_cast<const uint4*>(kr + kb * 64 + j * 8));
      a = fmaf(bf16_lo(qv.x), bf16_lo(kv.x), a);
      a = fmaf(bf16_hi(qv.x), bf16_hi(kv.x), a);
      a = fmaf(bf16_lo(qv.y), bf16_lo(kv.y), a);
      a = fmaf(bf16_hi(qv.y), bf16_hi(kv.y), a);
      a = fmaf(bf16_lo(qv.z), bf16_lo(kv.z), a);
      a = fmaf(bf16_hi(qv.z), bf16_hi(kv.z), a);
      a = fmaf(bf16_lo(qv.w), bf16_lo(kv.w), a);
      a = fmaf(bf16_hi(qv.w), bf16_hi(kv.w), a);
    }
  }
  return a;
}

// max of a row's 64 logits: eight independent three-input chains, then a short tree
__device__ __forceinline__ float max64(const float (&p)[64]) {
  float pm[8];
#pragma unroll
  for (int q8 = 0; q8 < 8; ++q8) {
    pm[q8] = fmax3f(p[q8], p[q8 + 8], p[q8 + 16]);
    pm[q8] = fmax3f(pm[q8], p[q8 + 24], p[q8 + 32]);
    pm[q8] = fmax3f(pm[q8], p[q8 + 40], p[q8 + 48]);
    pm[q8] = fmaxf(pm[q8], p[q8 + 56]);
  }
  return fmaxf(fmax3f(pm[0], pm[1], pm[2]), fmaxf(fmax3f(pm[3], pm[4], pm[5]),
                                                 fmaxf(pm[6], pm[7])));
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 t = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&t);
}

}  // namespace

template <int DD, int G, int KM, int RS, int TWO>
__global__ void __launch_bounds__(kAtThreads, ((DD == 64 && KM <= 16) || TWO) ? 2 : 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                   const __grid_constant__ CUtensorMap tmQc,
                   const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                   Dims D, const int32_t* __restrict__ idx, const float* __restrict__ s_sig,
                   const __nv_bfloat16* __restrict__ klm, const float* __restrict__ blm,
                   __nv_bfloat16* __restrict__ out, float* __restrict__ lse_out,
                   int list_cap, int bitmap_words, int32_t* __restrict__ status) {
  using SH = AtShape<DD, G, TWO>;
  constexpr int TQ = SH::TQ;
  static_assert(!TWO || (DD == 128 && KM <= 16), "two CTAs per SM: d = 128, K <= 16");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  // calibrated queries (G > 1: the per-head scores of the selection; with G = 1 this tile is
  // never loaded and serves only as a K/V stage; absent with TWO)
  uint8_t* sQc = sQ + SH::Q_BYTES;
  uint8_t* sK = TWO ? sQc : sQc + SH::Q_BYTES;
  uint8_t* sV = sK + SH::STAGES_MAIN * SH::KV_BYTES;
  uint8_t* sP = sV + SH::STAGES_MAIN * SH::KV_BYTES;   // (TWO: only the barriers follow)
  // stage s of the K/V ring (the last one lives in the q_cal tile)
  auto stage_k = [&](int s) -> uint8_t* {
    return s < SH::STAGES_MAIN ? sK + s * SH::KV_BYTES : sQc;
  };
  auto stage_v = [&](int s) -> uint8_t* {
    return s < SH::STAGES_MAIN ? sV + s * SH::KV_BYTES : sQc + SH::KV_BYTES;
  };
  // landmark rows of the first 64 tiles (K-tile layout) in the prologue scratch; dead once their
  // product has completed
  uint8_t* sKlm = sP;
  uint64_t* bars = reinterpret_cast<uint64_t*>(TWO ? sP : sP + 2 * SH::P_BYTES);
  uint64_t* kv_full = bars;                       // [STAGES]
  uint64_t* kv_empty = bars + SH::STAGES;         // [STAGES]
  uint64_t* q_full = bars + 2 * SH::STAGES;
  uint64_t* s_full = q_full + 1;                  // [2]
  uint64_t* s_empty = s_full + 2;                 // [2]
  uint64_t* p_full = s_empty + 2;                 // [2]
  uint64_t* p_empty = p_full + 2;                 // [2]
  uint64_t* o_done = p_empty + 2;
  uint64_t* o_final = o_done + 1;
  uint64_t* lm_done = o_final + 1;
  uint64_t* qc_free = lm_done + 1;   // every softmax warp is done reading the q_cal tile
  uint64_t* bm_free = qc_free + 1;   // (TWO) every row has read the bitmap in K/V stage 1
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bm_free + 1);
  int* n_tiles_sh = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(bars) + (TWO ? 256 : 1024));
  int* tiles = TWO ? n_tiles_sh + 16
                   : reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(bars) + 2048);  // [cap]
  // the tile bitmap of the union and the list position of each of its words live in the
  // prologue scratch (up to 2 x 16 KB; TWO: K/V stage 1): they are read for the last time by the
  // rows' ranking, before the landmark rows (or the stage's tiles) land there
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(TWO ? sK + SH::KV_BYTES : sP);   // [words]
  int* wpre = reinterpret_cast<int*>(TWO ? sV + SH::KV_BYTES : sP + SH::P_BYTES);
  // per row, its selected chunks in tile-list order: (tile index, surrogate score) [128][KM]
  // (TWO: tile indices as 16-bit integers)
  constexpr bool kSelSmem = KM <= 16;
  using SelT = typename std::conditional<TWO != 0, int16_t, int>::type;
  SelT* sel_t = reinterpret_cast<SelT*>(tiles + list_cap);
  float* sel_u = reinterpret_cast<float*>(sel_t + (kSelSmem ? kAtRows * KM : 0));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t bg = blockIdx.y;
  const int64_t g = bg % D.Hkv, b = bg / D.Hkv;
  const int64_t i0 = (int64_t)blockIdx.x * TQ;
  const int64_t i_last = (i0 + TQ - 1 < D.N_q - 1) ? i0 + TQ - 1 : D.N_q - 1;
  const int64_t p_first = D.q_pos0 + i0;
  const int64_t p_max = D.q_pos0 + i_last;
  const int64_t n_first = n_eligible(p_first, D.S, D.W);
  const int64_t last_chunk = p_max / kTile;   // last tile (64 tokens) any window reaches
  constexpr int rs = RS;                       // tiles per chunk = 1 << rs
  const int K = D.K;
  // warps 2-5 own one row each: row r = (query qi, head h), query-major, so a warp holds
  // 32 / G whole queries and skips the softmax of every selected-chunk tile none of them chose
  const bool is_row = warp >= 2;
  const int qd = warp & 3;
  const int r = qd * 32 + lane;
  const int qi = r / G, h = r - qi * G;
  const int64_t i = i0 + qi;
  const bool valid = i < D.N_q;
  // With one head per KV group the row's surrogate score of a selected chunk is the score the
  // selection ranked it by (s_sig); with several, each head's own score comes from a landmark
  // product below.
  constexpr bool kOwnScores = G > 1 && !TWO;
  // the row's selected chunks go out first: they feed both the tile list and the row's scores
  int sc[KM];
  float su[KM];
#pragma unroll
  for (int k = 0; k < KM; ++k) {
    const bool has = is_row && valid && k < K;
    sc[k] = has ? __ldg(idx + (bg * D.N_q + i) * K + k) : -1;
    if constexpr (!kOwnScores)
      su[k] = has ? __ldg(s_sig + (((b * D.Hq + g * G + h) * D.N_q + i) * K + k)) : -INFINITY;
  }

  // ---------------------------------------------------------------- barriers, TMEM, tile list
  if (threadIdx.x == 0) {
    for (int s = 0; s < SH::STAGES; ++s) { mbar_init(&kv_full[s], 1); mbar_init(&kv_empty[s], 1); }
    mbar_init(q_full, 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&s_empty[x], 4);
      mbar_init(&p_full[x], 4);
      mbar_init(&p_empty[x], 1);
    }
    mbar_init(o_done, 1);
    mbar_init(o_final, 1);
    mbar_init(lm_done, 1);
    mbar_init(qc_free, 4);
    mbar_init(bm_free, 4);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_holder, SH::TMEM_COLS);
  const int nbw = (int)(last_chunk / 32) + 1;
  for (int w = threadIdx.x; w < nbw; w += kAtThreads) bitmap[w] = 0u;
  __syncthreads();
  if (threadIdx.x == 0) {
    // the query and calibrated-query tiles load while the tile list is built
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmQc);
    mbar_expect_tx(q_full, (kOwnScores ? 2 : 1) * SH::Q_BYTES);
    // one box of [TQ queries][G heads][64 dims] per 64 columns: rows land query-major
    for (int kb = 0; kb < SH::KB; ++kb) {
      const int32_t y = (int32_t)(b * D.Hq + g * G), z = (int32_t)i0;
      tma_load_3d(sQ + kb * SH::Q_BOX, &tmQ, kb * 64, y, z, q_full);
      if constexpr (kOwnScores) tma_load_3d(sQc + kb * SH::Q_BOX, &tmQc, kb * 64, y, z, q_full);
    }
  }
  // selected chunks of every valid query of the tile (the G rows of a query hold the same
  // selection: row (h, qi) sets the bits of the entries k = h mod G), and the chunks of the
  // local windows
  if (is_row) {
#pragma unroll
    for (int k = 0; k < KM; ++k) {
      const int c = sc[k];
      if (k % G == h && c >= 0 && c < D.C && ((int64_t)c << rs) <= last_chunk) {
        for (int e2 = 0; e2 <= rs; ++e2) {
          const int tl = (c << rs) + e2;
          atomicOr(&bitmap[tl >> 5], 1u << (tl & 31));
        }
      }
    }
  }
  // the biases of the row's chunks load while the list is built
  float bsel[kOwnScores ? KM : 1];
  if constexpr (kOwnScores) {
#pragma unroll
    for (int k = 0; k < KM; ++k) {
      const int c = sc[k];
      bsel[k] = (c >= 0 && c < D.C) ? __ldg(blm + bg * D.C + c) : 0.f;
    }
  }
  for (int64_t c = (n_first << rs) + threadIdx.x; c <= last_chunk; c += kAtThreads)
    atomicOr(&bitmap[c >> 5], 1u << (c & 31));
  __syncthreads();
  {
    // list position of each bitmap word and the list itself (ascending tile order): every
    // thread owns a contiguous run of words, counts their bits, takes its offset from a
    // block-wide scan of those counts and places its own tiles; the work per thread grows with
    // the sequence only by one load per word of its run
    int* warp_tot = n_tiles_sh + 4;   // [6] bits per warp
    const int seg = (nbw + kAtThreads - 1) / kAtThreads;
    const int w_lo = threadIdx.x * seg;
    const int w_hi = w_lo + seg < nbw ? w_lo + seg : nbw;
    int mine = 0;
    for (int w = w_lo; w < w_hi; ++w) mine += __popc(bitmap[w]);
    int x = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    int off = x - mine, total = 0;
#pragma unroll
    for (int w2 = 0; w2 < kAtThreads / 32; ++w2) {
      const int t2 = warp_tot[w2];
      off += w2 < warp ? t2 : 0;
      total += t2;
    }
    if (threadIdx.x == 0) {
      if (total > list_cap) record_status(status, kStatusDeviceCheck);
      *n_tiles_sh = total < list_cap ? total : list_cap;
    }
    for (int w = w_lo; w < w_hi; ++w) {
      wpre[w] = off;
      uint32_t wb = bitmap[w];
      while (wb) {
        if (off < list_cap) tiles[off] = w * 32 + __ffs(wb) - 1;
        ++off;
        wb &= wb - 1u;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int n_tiles = *n_tiles_sh;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      int last_s = -1;
      uint32_t last_par = 0;
      // (TWO: K/V stage 1 holds the bitmap until every row has ranked its chunks)
      bool go = !TWO || mbar_wait(bm_free, 0, kAtPollLimit);
      if (!go) record_status(status, kStatusTimeout);
      for (int t = 0; go && t < n_tiles; ++t) {
        const int s = t % SH::STAGES;
        const uint32_t u = (uint32_t)(t / SH::STAGES);
        if (!mbar_wait(&kv_empty[s], (u & 1u) ^ 1u, kAtPollLimit) ||
            (!TWO && t == SH::STAGES_MAIN && !mbar_wait(qc_free, 0, kAtPollLimit))) {
          record_status(status, kStatusTimeout);
          break;
        }
        mbar_expect_tx(&kv_full[s], 2 * SH::KV_BYTES);
        const int32_t y = (int32_t)(bg * D.N_kv + (int64_t)tiles[t] * kTile);
        for (int kb = 0; kb < SH::KB; ++kb) {
          tma_load_2d(stage_k(s) + kb * SH::KV_BOX, &tmK, kb * 64, y, &kv_full[s]);
          tma_load_2d(stage_v(s) + kb * SH::KV_BOX, &tmV, kb * 64, y, &kv_full[s]);
        }
        last_s = s;
        last_par = u & 1u;
      }
      if (last_s >= 0) mbar_wait(&kv_full[last_s], last_par, kAtPollLimit);
      mbar_wait(q_full, 0, kAtPollLimit);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_QK = idesc_bf16_f32(kAtRows, kTile);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(kAtRows, DD) | (1u << 16);   // V is MN-major
      bool ok = mbar_wait(q_full, 0, kAtPollLimit);
      tc_fence_after();
      auto issue_qk = [&](int t) -> bool {
        const int s = t % SH::STAGES, x = t & 1;
        const uint32_t u = (uint32_t)(t / SH::STAGES), v = (uint32_t)(t >> 1);
        if (!mbar_wait(&kv_full[s], u & 1u, kAtPollLimit)) return false;
        if (!mbar_wait(&s_empty[x], (v & 1u) ^ 1u, kAtPollLimit)) return false;
        // (TWO: P[x] lives in S[x]; the P V product of tile t-2 must have read it)
        if (TWO && t >= 2 && !mbar_wait(&p_empty[x], (uint32_t)((t - 2) >> 1) & 1u, kAtPollLimit))
          return false;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < DD / 16; ++ks) {
          const int kb = ks >> 2, kin = ks & 3;
          const uint64_t ad = desc_kmajor_sw128(smem_u32(sQ + kb * SH::Q_BOX) + kin * 32);
          const uint64_t bd =
              desc_kmajor_sw128(smem_u32(stage_k(s) + kb * SH::KV_BOX) + kin * 32);
          mma_bf16_ss(tmem + (uint32_t)(x * kTile), ad, bd, IDESC_QK, ks > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[x]);
        return true;
      };
      if (ok && n_tiles > 0) ok = issue_qk(0);
      if (ok && n_tiles > 1) ok = issue_qk(1);
      for (int t = 0; ok && t < n_tiles; ++t) {
        const int s = t % SH::STAGES, x = t & 1;
        const uint32_t v = (uint32_t)(t >> 1);
        if (!mbar_wait(&p_full[x], v & 1u, kAtPollLimit)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kTile / 16; ++ks) {
          // 16 tokens of P = 8 TMEM columns
          const uint32_t at = tmem + SH::P_COL + (uint32_t)(x * SH::P_STRIDE + ks * 8);
          const uint64_t bd = desc_mnmajor_sw128(
              smem_u32(stage_v(s)) + ks * 16 * 128, SH::KV_BOX);
          mma_bf16_ts(tmem + SH::O_COL, at, bd, IDESC_PV, (t > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(&kv_empty[s]);
        mma_commit(&p_empty[x]);
        mma_commit(o_done);
        if (t == n_tiles - 1) mma_commit(o_final);
        if (t + 2 < n_tiles) ok = issue_qk(t + 2);
      }
      if (!ok) record_status(status, kStatusTimeout);
    }
  } else {
    // ---------------------------------------------------------------- softmax rows
    const int64_t pos = D.q_pos0 + (valid ? i : i_last);
    const int64_t n_i = n_eligible(pos, D.S, D.W);
    const int64_t hrow = (b * D.Hq + g * G + h) * D.N_q + i;
    float m_run = -INFINITY;
    int rk[KM];   // list position of each selected chunk's first tile (INT_MAX: none)
    int at[kSelSmem ? KM : 1];   // its place in the row's queue
    // each selected chunk's position in the (sorted) tile list, the rank of its first tile's
    // bit, and the chunk's place in the row's list-ordered queue (distinct chunks have distinct
    // ranks)
    auto rank_chunks = [&]() {
#pragma unroll
      for (int k = 0; k < KM; ++k) {
        const int c = sc[k];
        rk[k] = INT_MAX;
        if (c >= 0 && c < D.C && ((int64_t)c << rs) <= last_chunk) {
          const int tc = c << rs;
          rk[k] = wpre[tc >> 5] + __popc(bitmap[tc >> 5] & ((1u << (tc & 31)) - 1u));
        }
      }
      if constexpr (kSelSmem) {
#pragma unroll
        for (int k = 0; k < KM; ++k) {
          int a = 0;
#pragma unroll
          for (int k2 = 0; k2 < KM; ++k2) a += rk[k2] < rk[k] ? 1 : 0;
          at[k] = a;
        }
      }
    };
    bool lm_ok = true;
    if constexpr (kOwnScores) {
      // This head's surrogate score of each selected chunk, q_cal . k_lm[c] * scale + b_lm[c].
      // The landmark rows of the first 64 tiles of the (sorted) tile list are staged in shared
      // memory in the K-tile layout and one (128 x d) x (d x 64) product on the tensor core
      // scores every row of the tile against them; a chunk beyond those 64 is scored by a
      // plain dot.
      const int nk = n_tiles < SH::KLM_ROWS ? n_tiles : SH::KLM_ROWS;
      {
        constexpr int UPR = DD / 8;   // 16-byte units per landmark row
        const int tid = threadIdx.x - 64;
        uint4 u[SH::KLM_ROWS * UPR / 128];
#pragma unroll
        for (int e = 0; e < SH::KLM_ROWS * UPR / 128; ++e) {
          const int f = tid + e * 128, t = f / UPR, j = f - t * UPR;
          const int c = t < nk ? (tiles[t] >> rs) : D.C;   // the tile's chunk
          u[e] = c < D.C ? __ldg(reinterpret_cast<const uint4*>(klm + (bg * D.C + c) * DD) + j)
                         : make_uint4(0u, 0u, 0u, 0u);
        }
        rank_chunks();   // while those rows load
        // every row has read the bitmap before the landmark rows overwrite it
        asm volatile("bar.sync 1, 128;" ::: "memory");
#pragma unroll
        for (int e = 0; e < SH::KLM_ROWS * UPR / 128; ++e) {
          const int f = tid + e * 128, t = f / UPR, j = f - t * UPR;
          const int kb = j >> 3, jj = j & 7;
          *reinterpret_cast<uint4*>(sKlm + kb * SH::KV_BOX + (t >> 3) * 1024 + (t & 7) * 128 +
                                    ((jj ^ (t & 7)) << 4)) = u[e];
        }
        fence_async_smem();
        asm volatile("bar.sync 1, 128;" ::: "memory");   // the four softmax warps
      }
      const bool q_ok = mbar_wait_warp(q_full, 0, kAtPollLimit);
      if (warp == 2 && lane == 0 && q_ok) {
        tc_fence_after();
        constexpr uint32_t IDESC_LM = idesc_bf16_f32(kAtRows, SH::KLM_ROWS);
#pragma unroll
        for (int ks = 0; ks < DD / 16; ++ks) {
          const int kb = ks >> 2, kin = ks & 3;
          const uint64_t ad = desc_kmajor_sw128(smem_u32(sQc + kb * SH::Q_BOX) + kin * 32);
          const uint64_t bd = desc_kmajor_sw128(smem_u32(sKlm + kb * SH::KV_BOX) + kin * 32);
          mma_bf16_ss(tmem + SH::LM_COL, ad, bd, IDESC_LM, ks > 0 ? 1u : 0u);
        }
        mma_commit(lm_done);
      }
      lm_ok = q_ok && mbar_wait_warp(lm_done, 0, kAtPollLimit);
      // the row's 64 landmark scores, parked in this thread's own 128-byte rows of both scratch
      // areas (the staged landmark rows there are dead: their product completed), 16-byte slots
      // rotated
      uint8_t* park = sP + r * 128;
      if (lm_ok) {
        tc_fence_after();
#pragma unroll
        for (int part = 0; part < 4; ++part) {
          float vv[16];
          tmem_ld16(tmem + ((uint32_t)(qd * 32) << 16) + SH::LM_COL + part * 16, vv);
          tmem_wait_ld();
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int col4 = part * 4 + q4;   // 4-column group 0..15
            *reinterpret_cast<float4*>(park + (col4 >> 3) * SH::P_BYTES +
                                       (((col4 & 7) + r) & 7) * 16) =
                make_float4(vv[q4 * 4], vv[q4 * 4 + 1], vv[q4 * 4 + 2], vv[q4 * 4 + 3]);
          }
        }
      }
#pragma unroll
      for (int k = 0; k < KM; ++k) {
        su[k] = -INFINITY;
        const int c = sc[k];
        if (!lm_ok || rk[k] == INT_MAX) continue;
        const float bias = bsel[k];
        const int slot = rk[k] < nk ? rk[k] : -1;
        float a;
        if (slot >= 0) {
          const int col4 = slot >> 2;
          a = *reinterpret_cast<const float*>(park + (col4 >> 3) * SH::P_BYTES +
                                              (((col4 & 7) + r) & 7) * 16 + (slot & 3) * 4);
        } else {
          a = lm_dot<SH::KB, SH::Q_BOX>(sQc, r, klm + (bg * D.C + c) * DD);
        }
        su[k] = fmaf(a, D.scale, bias);
        m_run = fmaxf(m_run, su[k]);
      }
    } else {
      rank_chunks();
      if constexpr (TWO) {
        // the bitmap (in K/V stage 1) is read for the last time: the stage may fill
        __syncwarp();
        if (lane == 0) mbar_arrive(bm_free);
      }
#pragma unroll
      for (int k = 0; k < KM; ++k) {
        if (rk[k] == INT_MAX) su[k] = -INFINITY;
        m_run = fmaxf(m_run, su[k]);
      }
    }
    int n_sel = 0;   // selected chunks of this row (kSelSmem: their tile indices are in sel_t)
    if constexpr (kSelSmem) {
      // the row's selected chunks in list order (a chunk scored -inf carries weight 0)
#pragma unroll
      for (int k = 0; k < KM; ++k) {
        if (rk[k] == INT_MAX) continue;
        sel_t[r * KM + at[k]] = (SelT)rk[k];
        sel_u[r * KM + at[k]] = su[k];
        ++n_sel;
      }
    }
    // the q_cal tile (if loaded) is read for the last time above: it becomes a K/V stage
    __syncwarp();
    if (lane == 0) mbar_arrive(qc_free);
    if (!lm_ok) record_status(status, kStatusTimeout);
    float l = 0.f;
    bool sec_pending = false;   // S = 128: this row's next tile is the second half of its chunk
    float sec_off = 0.f, sec_f = 0.f;
    int sel_next = 0;
    int sel_tn = (kSelSmem && n_sel > 0) ? sel_t[r * KM] : -1;
    const uint32_t lane_base = tmem + ((uint32_t)(qd * 32) << 16);
    bool ok = true;
    for (int t = 0; t < n_tiles; ++t) {
      const int x = t & 1;
      const uint32_t v = (uint32_t)(t >> 1);
      if (!mbar_wait_warp(&s_full[x], v & 1u, kAtPollLimit)) { ok = false; break; }
      tc_fence_after();
      float p[kTile];
#pragma unroll
      for (int j = 0; j < kTile / 16; ++j) {
        float tmp[16];
        tmem_ld16(lane_base + (uint32_t)(x * kTile + 16 * j), tmp);
#pragma unroll
        for (int e = 0; e < 16; ++e) p[16 * j + e] = tmp[e];
      }
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[x]);

      const int c = tiles[t];   // tile index (64 tokens)
      float u = -INFINITY;
      bool is_sel = false;
      const bool is_second = sec_pending;
      sec_pending = false;
      if constexpr (kSelSmem) {
        // the next selected chunk of this row, in list order
        if (sel_next < n_sel && sel_tn == t) {
          is_sel = true;
          u = sel_u[r * KM + sel_next];
          ++sel_next;
          sel_tn = sel_next < n_sel ? sel_t[r * KM + sel_next] : -1;
        }
      } else {
#pragma unroll
        for (int k = 0; k < KM; ++k)
          if (sc[k] >= 0 && (sc[k] << rs) == c) { is_sel = true; u = su[k]; }
      }
      const int64_t t0 = (int64_t)c * kTile;
      const bool is_win = valid && !is_sel && !is_second && c >= (n_i << rs) && t0 <= pos;
      // S = 128: the first tile of a selected chunk also reads the second tile's logits
      const bool first2 = RS && is_sel && u != -INFINITY && t + 1 < n_tiles;
      // (TMEM loads are warp-collective: every lane runs these passes, a lane without a first
      // half of its own ignores the results)
      const float sc2 = D.scale * kLog2e;
      float mxc = 0.f;          // the chunk's max over both tiles (raw logits)
      float sum2_raw = 0.f;     // the second tile's exponentials' sum against that max
      const int x2 = x ^ 1;
      const bool need2 = RS && __any_sync(0xffffffffu, first2);
      if (need2) {
        if (!mbar_wait_warp(&s_full[x2], (uint32_t)((t + 1) >> 1) & 1u, kAtPollLimit)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float mx2 = -INFINITY;
#pragma unroll
        for (int j = 0; j < kTile / 16; ++j) {
          float tmp[16];
          tmem_ld16(lane_base + (uint32_t)(x2 * kTile + 16 * j), tmp);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) mx2 = fmaxf(mx2, tmp[e]);
        }
        mxc = fmaxf(max64(p), mx2);
        const float offc = -mxc * sc2;
#pragma unroll
        for (int j = 0; j < kTile / 16; ++j) {
          float tmp[16];
          tmem_ld16(lane_base + (uint32_t)(x2 * kTile + 16 * j), tmp);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            fma2(tmp[e], tmp[e + 1], sc2, offc);
            sum2_raw += fast_exp2(tmp[e]) + fast_exp2(tmp[e + 1]);
          }
        }
      }
      bool rescale = false;
      float factor = 1.f;
      // base-2 exponentials throughout: x * scale * log2(e) is the logit in log2 units
      if (is_second) {
        // second half of a selected chunk: the max and normaliser of its first half
#pragma unroll
        for (int j = 0; j < kTile; j += 2) {
          fma2(p[j], p[j + 1], sc2, sec_off);
          p[j] = fast_exp2(p[j]);
          p[j + 1] = fast_exp2(p[j + 1]);
          mul2(p[j], p[j + 1], sec_f);
        }
      } else if (is_sel && u != -INFINITY) {
        // intra-chunk softmax of this chunk, weighted by exp(u - m_run) (u <= m_run)
        // (three-input maxima, and fp32 pairs for the affine, sum and scale passes)
        const float mx = first2 ? mxc : max64(p);
        const float off = -mx * sc2;
        float ps[8];
#pragma unroll
        for (int q8 = 0; q8 < 8; ++q8) ps[q8] = 0.f;
#pragma unroll
        for (int j = 0; j < kTile; j += 2) {
          fma2(p[j], p[j + 1], sc2, off);
          p[j] = fast_exp2(p[j]);
          p[j + 1] = fast_exp2(p[j + 1]);
          add2(ps[j & 7], ps[(j & 7) + 1], p[j], p[j + 1]);
        }
        const float sum = ((ps[0] + ps[1]) + (ps[2] + ps[3])) +
                          ((ps[4] + ps[5]) + (ps[6] + ps[7])) +
                          (first2 ? sum2_raw : 0.f);
        const float w = fast_exp2((u - m_run) * kLog2e);
        const float f = w / sum;
#pragma unroll
        for (int j = 0; j < kTile; j += 2) mul2(p[j], p[j + 1], f);
        l += w;
        if (first2) { sec_pending = true; sec_off = off; sec_f = f; }
      } else if (is_win) {
        // raw logits; only the tile holding the query's own position needs the causal mask
        if (t0 + kTile - 1 > pos) {
#pragma unroll
          for (int j = 0; j < kTile; ++j)
            if (t0 + j > pos) p[j] = -INFINITY;
        }
        const float mt = max64(p) * D.scale;   // scale > 0
        if (mt > m_run + kRescaleMargin) {
          if (l > 0.f) {
            factor = fast_exp2((m_run - mt) * kLog2e);
            l *= factor;
            rescale = true;
          }
          m_run = mt;
        }
        // a masked logit (-inf) gives 2^-inf = 0, unless m_run is still -inf (no finite logit)
        const float off = m_run == -INFINITY ? -INFINITY : -m_run * kLog2e;
        float ps[8];
#pragma unroll
        for (int q8 = 0; q8 < 8; ++q8) ps[q8] = 0.f;
#pragma unroll
        for (int j = 0; j < kTile; j += 2) {
          fma2(p[j], p[j + 1], sc2, off);
          p[j] = fast_exp2(p[j]);
          p[j + 1] = fast_exp2(p[j + 1]);
          add2(ps[j & 7], ps[(j & 7) + 1], p[j], p[j + 1]);
        }
        l += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      } else {
#pragma unroll
        for (int j = 0; j < kTile; ++j) p[j] = 0.f;
      }
      // the P buffer is free once the P V product of tile t-2 has completed
      if (!mbar_wait_warp(&p_empty[x], (v & 1u) ^ 1u, kAtPollLimit)) { ok = false; break; }
      if (__any_sync(0xffffffffu, rescale)) {
        // O row *= factor, after the P V product of tile t-1 has landed
        if (!mbar_wait_warp(o_done, (uint32_t)((t - 1) & 1), kAtPollLimit)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int j = 0; j < DD / 16; ++j) {
          float o[16];
          tmem_ld16(lane_base + SH::O_COL + 16 * j, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] *= factor;
          tmem_st16(lane_base + SH::O_COL + 16 * j, o);
        }
        tmem_wait_st();
      }
      // the row's P into its TMEM lane: 64 bf16 in 32 columns
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[e] = pack_bf16(p[32 * hf + 2 * e], p[32 * hf + 2 * e + 1]);
        tmem_st16u(lane_base + SH::P_COL + (uint32_t)(x * SH::P_STRIDE + 16 * hf), pk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[x]);
    }
    // ---------------------------------------------------------------- output rows
    const bool fin = __all_sync(0xffffffffu, ok) && n_tiles > 0 &&
                     mbar_wait_warp(o_final, 0, kAtPollLimit);
    if (fin) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* orow = out + hrow * DD;
#pragma unroll
      for (int j = 0; j < DD / 16; ++j) {
        float o[16];
        tmem_ld16(lane_base + SH::O_COL + 16 * j, o);
        tmem_wait_ld();
        if (valid) {
          uint4 a, c4;
          a.x = pack_bf16(o[0] * inv, o[1] * inv);
          a.y = pack_bf16(o[2] * inv, o[3] * inv);
          a.z = pack_bf16(o[4] * inv, o[5] * inv);
          a.w = pack_bf16(o[6] * inv, o[7] * inv);
          c4.x = pack_bf16(o[8] * inv, o[9] * inv);
          c4.y = pack_bf16(o[10] * inv, o[11] * inv);
          c4.z = pack_bf16(o[12] * inv, o[13] * inv);
          c4.w = pack_bf16(o[14] * inv, o[15] * inv);
          *reinterpret_cast<uint4*>(orow + 16 * j) = a;
          *reinterpret_cast<uint4*>(orow + 16 * j + 8) = c4;
        }
      }
      if (valid && lse_out) lse_out[hrow] = m_run + logf(l);
    } else if (!ok || n_tiles > 0) {
      record_status(status, kStatusTimeout);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, SH::TMEM_COLS);
}

// ---------------------------------------------------------------------------------------------
namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode_at() {
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

bool make_map_at(CUtensorMap* map, const void* base, uint64_t rows, uint64_t d, uint32_t box_rows) {
  auto enc = get_encode_at();
  if (!enc) return false;
  cuuint64_t dims[2] = {d, rows};
  cuuint64_t strides[1] = {d * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [B Hq, N_q, d] bf16 viewed as 3-D (dims, heads, queries), boxes of [TQ queries][G heads][64
// dims] with the 128-byte swizzle: the G heads of a query are consecutive rows in shared memory.
bool make_map_q3(CUtensorMap* map, const void* base, uint64_t heads, uint64_t n_q, uint64_t d,
                 uint32_t G, uint32_t TQ) {
  auto enc = get_encode_at();
  if (!enc) return false;
  cuuint64_t dims[3] = {d, heads, n_q};
  cuuint64_t strides[2] = {n_q * d * 2, d * 2};
  cuuint32_t box[3] = {64, G, TQ};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int list_capacity(const Dims& D, int TQ) {
  // union of TQ queries' selections (S / 64 tiles each) plus the tiles their windows cover
  return TQ * D.K * (D.S / kTile) + (int)((D.W + D.S + TQ) / kTile) + 4;
}

// shared memory of a CTA when two share an SM (each also reserves 1 KB of the SM's 228 KB)
constexpr int kTwoCtaSmemLimit = (228 * 1024) / 2 - 1024;

int64_t two_cta_smem(const Dims& D) {
  const int TQ = kAtRows / D.G;
  const int64_t cap = (int64_t)TQ * D.K * (D.S / kTile) + (D.W + D.S + TQ) / kTile + 4;
  const int km = D.K <= 8 ? 8 : 16;
  return AtShape<128, 1, 1>::FIXED + cap * 4 + (int64_t)kAtRows * km * 6;
}

template <int DD, int G, int KM, int RS, int TWO>
cudaError_t launch_at_t(const Dims& D, const void* q, const void* qc, const void* K,
                        const void* V, const int32_t* idx, const float* s_sig, const void* klm,
                        const float* blm, void* out, float* lse, int32_t* status,
                        cudaStream_t st) {
  using SH = AtShape<DD, G, TWO>;
  CUtensorMap tmQ, tmQc, tmK, tmV;
  if (!make_map_q3(&tmQ, q, (uint64_t)(D.B * D.Hq), (uint64_t)D.N_q, DD, G, SH::TQ) ||
      !make_map_q3(&tmQc, qc, (uint64_t)(D.B * D.Hq), (uint64_t)D.N_q, DD, G, SH::TQ) ||
      !make_map_at(&tmK, K, (uint64_t)(D.B * D.Hkv * D.N_kv), DD, kTile) ||
      !make_map_at(&tmV, V, (uint64_t)(D.B * D.Hkv * D.N_kv), DD, kTile))
    return cudaErrorInvalidValue;
  const int cap = list_capacity(D, SH::TQ);
  const int words = (int)((D.N_kv / kTile) / 32) + 2;
  if (words * 4 > (TWO ? SH::KV_BYTES : SH::P_BYTES)) return cudaErrorInvalidConfiguration;
  const int smem = TWO ? SH::FIXED + cap * 4 + kAtRows * KM * 6
                       : SH::FIXED + 1024 + cap * 4 + (KM <= 16 ? kAtRows * KM * 8 : 0);
  if (smem > (TWO ? kTwoCtaSmemLimit : kAtSmemLimit)) return cudaErrorInvalidConfiguration;
  auto kern = attn_tc_kernel<DD, G, KM, RS, TWO>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((D.N_q + SH::TQ - 1) / SH::TQ), (unsigned)(D.B * D.Hkv));
  kern<<<grid, kAtThreads, smem, st>>>(tmQ, tmQc, tmK, tmV, D, idx, s_sig,
                                       (const __nv_bfloat16*)klm, blm, (__nv_bfloat16*)out, lse,
                                       cap, words, status);
  return cudaGetLastError();
}

template <int DD, int G>
cudaError_t launch_at_k(const Dims& D, const void* q, const void* qc, const void* K,
                        const void* V, const int32_t* idx, const float* s_sig, const void* klm,
                        const float* blm, void* out, float* lse, int32_t* status,
                        cudaStream_t st) {
  if constexpr (DD == 128) {
    if (attn_tc_two_cta(D)) {
      if (D.S == 2 * kTile) {
        if (D.K <= 8)
          return launch_at_t<DD, G, 8, 1, 1>(D, q, qc, K, V, idx, s_sig, klm, blm, out, lse,
                                             status, st);
        return launch_at_t<DD, G, 16, 1, 1>(D, q, qc, K, V, idx, s_sig, klm, blm, out, lse,
                                            status, st);
      }
      if (D.K <= 8)
        return launch_at_t<DD, G, 8, 0, 1>(D, q, qc, K, V, idx, s_sig, klm, blm, out, lse, status,
                                           st);
      return launch_at_t<DD, G, 16, 0, 1>(D, q, qc, K, V, idx, s_sig, klm, blm, out, lse, status,
                                          st);
    }
    // chunks of 128 tokens (two tiles per chunk) are built for d = 128 only
    if (D.S == 2 * kTile) {
      if (D.K <= 8)
        return launch_at_t<DD, G, 8, 1, 0>(D, q, qc, K, V, idx, s_sig, klm, blm, out, lse, status,
                                        st);
      if (D.K <= 16)
        return launch_at_t<DD, G, 16, 1, 0>(D, q, qc, K, V, idx, s_sig, klm, blm, out, lse, status,
                                         st);
      return launch_at_t<DD, G, 32, 1, 0>(D, q, qc, K, V, idx, s_sig, klm, blm, out, lse, status, st);
    }
  }
  if (D.K <= 8)
    return launch_at_t<DD, G, 8, 0, 0>(D, q, qc, K, V, idx, s_sig, klm, blm, out, lse, status, st);
  if (D.K <= 16)
    return launch_at_t<DD, G, 16, 0, 0>(D, q, qc, K, V, idx, s_sig, klm, blm, out, lse, status, st);
  return launch_at_t<DD, G, 32, 0, 0>(D, q, qc, K, V, idx, s_sig, klm, blm, out, lse, status, st);
}

}  // namespace

bool attn_tc_two_cta(const Dims& D) {
  if (D.d != 128 || D.K > 16) return false;
  if (D.S != kTile && D.S != 2 * kTile) return false;
  if (D.G != 1 && D.G != 2 && D.G != 4 && D.G != 8) return false;
  if ((D.N_kv / kTile) / 32 + 2 > AtShape<128, 1, 1>::KV_BYTES / 4) return false;
  return two_cta_smem(D) <= kTwoCtaSmemLimit;
}

bool attn_tc_external_scores(const Dims& D) { return D.G == 1 || attn_tc_two_cta(D); }

bool attn_tc_supported(const Dims& D, bool bf16) {
  if (!bf16 || D.K > kMaxK) return false;
  if (D.S != kTile && !(D.S == 2 * kTile && D.d == 128)) return false;
  if (D.d != 64 && D.d != 128) return false;
  if (D.G != 1 && D.G != 2 && D.G != 4 && D.G != 8) return false;
  if (D.B * D.Hkv > 65535) return false;
  const int TQ = kAtRows / D.G;
  const int64_t cap = (int64_t)TQ * D.K * (D.S / kTile) + (D.W + D.S + TQ) / kTile + 4;
  // the tile bitmap (one bit per 64-token tile of the sequence) fits one prologue scratch area
  // of 16 KB: sequences of up to about 8.3 M tokens
  const int64_t words = (D.N_kv / kTile) / 32 + 2;
  if (words * 4 > AtShape<64, 1>::P_BYTES) return false;
  const int fixed = D.d == 128 ? AtShape<128, 1>::FIXED : AtShape<64, 1>::FIXED;
  if (D.C >= (int64_t)INT32_MAX) return false;
  const int km = D.K <= 8 ? 8 : (D.K <= 16 ? 16 : 32);
  const int64_t sel_bytes = km <= 16 ? (int64_t)kAtRows * km * 8 : 0;
  return attn_tc_two_cta(D) || fixed + 1024 + cap * 4 + sel_bytes <= kAtSmemLimit;
}

cudaError_t launch_attn_tc(const Dims& D, const void* q, const void* qc, const void* K,
                           const void* V, const int32_t* idx, const float* s_sig,
                           const void* klm, const float* blm, void* out, float* lse,
                           int32_t* status, cudaStream_t st) {
  if (D.B * D.Hq * D.N_q == 0) return cudaSuccess;
#define HILS_AT(DD, GG) \
  return launch_at_k<DD, GG>(D, q, qc, K, V, idx, s_sig, klm, blm, out, lse, status, st)
  if (D.d == 128) {
    if (D.G == 1) HILS_AT(128, 1);
    if (D.G == 2) HILS_AT(128, 2);
    if (D.G == 4) HILS_AT(128, 4);
    HILS_AT(128, 8);
  }
  if (D.G == 1) HILS_AT(64, 1);
  if (D.G == 2) HILS_AT(64, 2);
  if (D.G == 4) HILS_AT(64, 4);
  HILS_AT(64, 8);
#undef HILS_AT
}

}  // namespace hils
