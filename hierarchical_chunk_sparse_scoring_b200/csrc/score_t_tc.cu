// Steps 1-2 for prefill on the tcgen05 tensor cores, landmark-major: the product is taken with the
// landmark rows as the MMA's M (128 per tile) and every (head, query) row of a block of
// MQ = 256/G queries as its N (256), so one 128 x 256 x 16 instruction serves all G heads of the
// KV group and each operand is read from shared memory once per 256 output columns
// ([Reader] "The HiLS-Attention Mechanism": surrogate score q_cal . k_lm / sqrt(d) + b; GQA
// paragraph of "Implementation and Training Recipes": the group's score is the max over its
// heads; "Limitations of Naive Sparse Attention": top-K distant chunks, ties to the lower index).
//
// TMEM lane = landmark of the tile, column = head * MQ + query.  Epilogue: one landmark per
// thread (its bias is one register); per query the max over the G head columns, scale and bias,
// the causal chunk mask (chunk c is eligible for query q iff c < n_q), then:
//   * tiles after the first: a compare with the query's current K-th best value theta_q (shared
//     memory).  Survivors (rare once the list is full) are appended to a per-query buffer and
//     merged into the query's sorted list once per tile by one thread per query.
//   * the first tile: the whole tile is written to shared memory query-major, TPQ threads per
//     query each keep the best R = ceil(K/TPQ) values of an interleaved stripe, and the smallest
//     of their R-th values is a lower bound theta0 of the query's K-th best (TPQ * R >= K values
//     reach it); the values >= theta0 are the first tile's candidates.
//   * a query with more candidates than its buffer holds is merged from the tile's full column
//     by one thread (exact for any input, slower).
// The list of a query holds (score, chunk) best first with ties to the lower chunk; no score is
// written to memory.
//
// CTA = (b, g, MQ queries); 10 warps: warp 0 TMA (the block's calibrated queries once, then the
// landmark tiles through a ring), warp 1 TMEM owner and MMA issuer (two 256-column
// accumulators), warps 2-9 epilogue (warp w reads TMEM lanes 32 * (w % 4).. and one half of the
// block's queries).  Every mbarrier wait gives up after a bounded number of polls and records
// HILS_ERR_TIMEOUT.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace hils {
using namespace sm100;

namespace {

constexpr uint32_t kTtPollLimit = 1u << 24;
constexpr int kTtSmemLimit = 227 * 1024;
constexpr int kTtThreads = 320;   // warp 0 TMA, warp 1 MMA, warps 2-9 epilogue
constexpr int kTtEpi = 256;
constexpr int kLm = 128;          // landmark rows per tile (M)
constexpr int kCols = 256;        // (head, query) columns per tile (N)

template <int DD, int G, int KM>
struct TtShape {
  static constexpr int MQ = kCols / G;             // queries per CTA
  static constexpr int QH = MQ / 2;                // queries of one epilogue half
  static constexpr int QP = 32;                    // queries per full-column pass
  static constexpr int NPASS = MQ / QP;
  static constexpr int TPQ = kTtEpi / QP;          // stripe threads per query (8)
  static constexpr int RM = (KM + TPQ - 1) / TPQ;  // stripe list slots
  static constexpr int SCR_LD = kLm + TPQ;         // scratch row stride: conflict-free stripes
  static constexpr int CAP = MQ >= 128 ? 32 : 64;  // buffered candidates per query per tile
  // row strides of the lists and buffers: odd, so the threads of consecutive queries hit
  // different banks
  static constexpr int LS = KM + 1;
  static constexpr int CS = CAP + 1;
  static constexpr int KB = DD / 64;
  static constexpr int B_BOX = kCols * 128;        // [256 (head, query) rows x 64 dims]
  static constexpr int B_BYTES = KB * B_BOX;
  static constexpr int A_BOX = kLm * 128;          // [128 landmark rows x 64 dims]
  static constexpr int A_STAGE = KB * A_BOX;
  static constexpr int LIST_BYTES = MQ * LS * 8;
  static constexpr int CAND_BYTES = MQ * CS * 8;
  static constexpr int SCR_BYTES = QP * SCR_LD * 4;
  static constexpr int MISC_BYTES = MQ * 12 + 64;  // theta, counts, eligible counts, flags
  static constexpr int FIXED = B_BYTES + LIST_BYTES + CAND_BYTES + SCR_BYTES + MISC_BYTES +
                               256 /*barriers*/ + 1024 /*alignment*/;
  static constexpr int STAGES_FIT = (kTtSmemLimit - FIXED) / A_STAGE;
  static constexpr int STAGES = STAGES_FIT > 4 ? 4 : STAGES_FIT;
  // more than half of the SM's shared memory, so no second CTA is co-resident and competes for
  // the 512 TMEM columns this CTA allocates
  static constexpr int SMEM_USED = FIXED + STAGES * A_STAGE;
  static constexpr int SMEM = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
  static constexpr uint32_t TMEM_COLS = 512;       // two 256-column accumulators
  static_assert(STAGES >= 2, "shared memory too small for this shape");
  static_assert(QH % 16 == 0, "queries in groups of 16");
  static_assert((MQ * 128) % 1024 == 0, "whole swizzle atoms per head");
  static_assert(32 % TPQ == 0 && QP * TPQ == kTtEpi, "stripe threads");
  static_assert(TPQ * RM >= KM, "witnesses");
};

}  // namespace

template <int DD, int G, int KM>
__global__ void __launch_bounds__(kTtThreads, 1)
    score_t_tc_kernel(const __grid_constant__ CUtensorMap tmQc,
                      const __grid_constant__ CUtensorMap tmKlm, Dims D,
                      const float* __restrict__ blm, int32_t* __restrict__ idx,
                      float* __restrict__ s_out, int32_t* __restrict__ status) {
  using SH = TtShape<DD, G, KM>;
  constexpr int MQ = SH::MQ, QH = SH::QH, QP = SH::QP, TPQ = SH::TPQ, CAP = SH::CAP;
  constexpr int RM = SH::RM, LD = SH::SCR_LD, LS = SH::LS, CS = SH::CS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sB = smem;                                                      // q_cal block (N)
  uint8_t* sA = sB + SH::B_BYTES;                                          // landmark ring (M)
  float* list_v = reinterpret_cast<float*>(sA + SH::STAGES * SH::A_STAGE);   // [MQ][LS]
  int* list_c = reinterpret_cast<int*>(list_v + MQ * LS);                    // [MQ][LS]
  float* cand_v = reinterpret_cast<float*>(list_c + MQ * LS);                // [MQ][CS]
  int* cand_c = reinterpret_cast<int*>(cand_v + MQ * CS);                    // [MQ][CS]
  float* scr = reinterpret_cast<float*>(cand_c + MQ * CS);                   // [QP][LD]
  float* theta = scr + QP * LD;                                              // [MQ]
  int* cnt = reinterpret_cast<int*>(theta + MQ);                             // [MQ]
  int* nq = cnt + MQ;                                                        // [MQ]
  int* flags = nq + MQ;                                                      // [4]
  uint64_t* bars = reinterpret_cast<uint64_t*>(
      (reinterpret_cast<uintptr_t>(flags + 16) + 7) & ~static_cast<uintptr_t>(7));
  uint64_t* full = bars;                     // [STAGES] landmark tile landed
  uint64_t* empty = bars + SH::STAGES;       // [STAGES] its MMAs completed
  uint64_t* b_full = bars + 2 * SH::STAGES;  // calibrated queries landed
  uint64_t* acc_full = b_full + 1;           // [2]
  uint64_t* acc_empty = acc_full + 2;        // [2]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t qt = (int64_t)gridDim.x - 1 - blockIdx.x;   // longest query blocks first
  const int64_t bg = blockIdx.y;
  const int64_t g = bg % D.Hkv, b = bg / D.Hkv;
  const int64_t i0 = qt * MQ;
  const int nqv = (int)(D.N_q - i0 < MQ ? D.N_q - i0 : MQ);   // valid queries of the block
  const int64_t n_max = n_eligible(D.q_pos0 + i0 + nqv - 1, D.S, D.W);
  const int n_tiles = (int)((n_max + kLm - 1) / kLm);
  const int K = D.K;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SH::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(b_full, 1);
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], kTtEpi / 32);
    }
    fence_barrier_init();
  }
  // lists start empty: K live slots (-inf, INT_MAX) at the end of KM, sentinels in front
  for (int e = threadIdx.x; e < MQ * LS; e += kTtThreads) {
    const bool sentinel = (e % LS) < KM - K;
    list_v[e] = sentinel ? INFINITY : -INFINITY;
    list_c[e] = sentinel ? -1 : INT_MAX;
  }
  for (int q = threadIdx.x; q < MQ; q += kTtThreads) {
    theta[q] = -INFINITY;
    cnt[q] = 0;
    nq[q] = q < nqv ? (int)n_eligible(D.q_pos0 + i0 + q, D.S, D.W) : 0;
  }
  if (threadIdx.x < 16) flags[threadIdx.x] = 0;
  if (warp == 1) tmem_alloc(tmem_holder, SH::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && n_tiles > 0) {
      prefetch_tensormap(&tmQc);
      prefetch_tensormap(&tmKlm);
      mbar_expect_tx(b_full, SH::B_BYTES);
      for (int h = 0; h < G; ++h)
        for (int kb = 0; kb < SH::KB; ++kb)
          tma_load_2d(sB + kb * SH::B_BOX + h * MQ * 128, &tmQc, kb * 64,
                      (int32_t)((b * D.Hq + g * G + h) * D.N_q + i0), b_full);
      int last_s = -1;
      uint32_t last_par = 0;
      for (int t = 0; t < n_tiles; ++t) {
        const int s = t % SH::STAGES;
        const uint32_t u = (uint32_t)(t / SH::STAGES);
        if (!mbar_wait(&empty[s], (u & 1u) ^ 1u, kTtPollLimit)) {
          record_status(status, kStatusTimeout);
          break;
        }
        mbar_expect_tx(&full[s], SH::A_STAGE);
        for (int kb = 0; kb < SH::KB; ++kb)
          tma_load_2d(sA + s * SH::A_STAGE + kb * SH::A_BOX, &tmKlm, kb * 64,
                      (int32_t)(bg * D.C + (int64_t)t * kLm), &full[s]);
        last_s = s;
        last_par = u & 1u;
      }
      // our last copies have landed before this warp leaves (bounded)
      if (last_s >= 0) mbar_wait(&full[last_s], last_par, kTtPollLimit);
      mbar_wait(b_full, 0, kTtPollLimit);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(kLm, kCols);
      bool ok = mbar_wait(b_full, 0, kTtPollLimit);
      tc_fence_after();
      for (int t = 0; ok && t < n_tiles; ++t) {
        const int s = t % SH::STAGES;
        const uint32_t u = (uint32_t)(t / SH::STAGES);
        const int a = t & 1;
        const uint32_t v = (uint32_t)(t >> 1);
        ok = mbar_wait(&acc_empty[a], (v & 1u) ^ 1u, kTtPollLimit) &&
             mbar_wait(&full[s], u & 1u, kTtPollLimit);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < DD / 16; ++ks) {
          const int kb = ks >> 2, kin = ks & 3;
          const uint64_t ad =
              desc_kmajor_sw128(smem_u32(sA + s * SH::A_STAGE + kb * SH::A_BOX) + kin * 32);
          const uint64_t bd = desc_kmajor_sw128(smem_u32(sB + kb * SH::B_BOX) + kin * 32);
          mma_bf16_ss(tmem + (uint32_t)(a * kCols), ad, bd, IDESC, ks > 0 ? 1u : 0u);
        }
        mma_commit(&empty[s]);
        mma_commit(&acc_full[a]);
      }
      if (!ok) record_status(status, kStatusTimeout);
    }
  } else {
    // ------------------------------------------------------------ epilogue (256 threads)
    const int ew = warp - 2;                  // 0..7
    const int qd = warp & 3;                  // TMEM lane quadrant of this warp
    const int half = ew >> 2;                 // which half of the block's queries
    const int r = qd * 32 + lane;             // landmark row of the tile (TMEM lane)
    const int tid = ew * 32 + lane;           // 0..255
    const uint32_t lane_base = tmem + ((uint32_t)(qd * 32) << 16);
    const float* bb = blm + bg * D.C;
    bool ok = true;
    float bias_next = r < D.C ? __ldg(bb + r) : 0.f;
    for (int t = 0; t < n_tiles; ++t) {
      const int a = t & 1;
      const uint32_t v = (uint32_t)(t >> 1);
      const int64_t cbase = (int64_t)t * kLm;
      const int64_t c = cbase + r;           // this thread's landmark
      const float bias = bias_next;
      {   // the next tile's bias loads while this one is processed
        const int64_t cn = c + kLm;
        bias_next = cn < D.C ? __ldg(bb + cn) : 0.f;
      }
      // first query of the block for which chunk c is eligible: c < n(p) <=> p >= (c+1)S + W - 1
      const int64_t qmin64 = (c + 1) * D.S + D.W - 1 - D.q_pos0 - i0;
      const int qmin = qmin64 < 0 ? 0 : (qmin64 > MQ ? MQ : (int)qmin64);
      const int qlo = qmin;                          // eligible queries: [qlo, nqv)
      if (threadIdx.x == 64) flags[(t + 1) & 1] = 0;   // the next tile's overflow flag
      // (every epilogue warp takes the same path through the named barriers; after a timeout
      // a warp stops waiting and touching TMEM)
      if (ok) ok = mbar_wait_warp(&acc_full[a], v & 1u, kTtPollLimit);
      if (ok) tc_fence_after();
      // scores of this thread's landmark for the 16 queries q0.. (group max, scale, bias)
      auto sig16 = [&](int q0, float (&sg)[16]) {
        constexpr int HG = G < 4 ? G : 4;   // heads whose loads are in flight together
#pragma unroll
        for (int h0 = 0; h0 < G; h0 += HG) {
          float tmp[HG][16];
#pragma unroll
          for (int hh = 0; hh < HG; ++hh)
            tmem_ld16(lane_base + (uint32_t)(a * kCols + (h0 + hh) * MQ + q0), tmp[hh]);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float m = h0 == 0 ? tmp[0][e] : fmaxf(sg[e], tmp[0][e]);
#pragma unroll
            for (int hh = 1; hh < HG; ++hh) m = fmaxf(m, tmp[hh][e]);
            sg[e] = m;
          }
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) sg[e] = fmaf(sg[e], D.scale, bias);
      };

      // the full column of the pass's queries, query-major in the scratch rows (a -inf score
      // is kept as the lowest finite value so that it can still fill an empty slot)
      auto dump_pass = [&](int p) {
        if (ok) {
#pragma unroll 1
          for (int q0 = half * QH; q0 < (half + 1) * QH; q0 += 16) {
            if (q0 < p * QP || q0 >= (p + 1) * QP) continue;
            float sg[16];
            sig16(q0, sg);
#pragma unroll
            for (int e = 0; e < 16; ++e)
              scr[(q0 - p * QP + e) * LD + r] = fmaxf(sg[e], -FLT_MAX);
          }
        }
      };
      // one thread merges the column of query q (pass p) into q's list: exact for any input
      auto serial_merge = [&](int q, int p) {
        TailList<KM> L;
#pragma unroll
        for (int k = 0; k < KM; ++k) { L.v[k] = list_v[q * LS + k]; L.c[k] = list_c[q * LS + k]; }
        const int ne = (int)(nq[q] - cbase < kLm ? nq[q] - cbase : kLm);
        const float* row = scr + (q - p * QP) * LD;
        for (int k0 = 0; k0 < kLm; ++k0) {
          const int k = (k0 + q) & (kLm - 1);    // rotated start: lanes hit different banks
          if (k >= ne) continue;
          const float x = row[k];
          const int cc = (int)(cbase + k);
          if (better(x, cc, L.kth_v(), L.kth_c())) L.insert(x, cc);
        }
#pragma unroll
        for (int k = 0; k < KM; ++k) { list_v[q * LS + k] = L.v[k]; list_c[q * LS + k] = L.c[k]; }
        theta[q] = L.kth_c() == INT_MAX ? -INFINITY : L.kth_v();
        cnt[q] = 0;
      };
      // merges the buffered candidates of query q into its list
      auto buffer_merge = [&](int q, int n) {
        TailList<KM> L;
#pragma unroll
        for (int k = 0; k < KM; ++k) { L.v[k] = list_v[q * LS + k]; L.c[k] = list_c[q * LS + k]; }
        for (int j = 0; j < n; ++j) L.insert(cand_v[q * CS + j], cand_c[q * CS + j]);
#pragma unroll
        for (int k = 0; k < KM; ++k) { list_v[q * LS + k] = L.v[k]; list_c[q * LS + k] = L.c[k]; }
        theta[q] = L.kth_c() == INT_MAX ? -INFINITY : L.kth_v();
        cnt[q] = 0;
      };

      if (t == 0) {
        // ---------------------------------------------------------- first tile
#pragma unroll 1
        for (int p = 0; p < SH::NPASS; ++p) {
          dump_pass(p);
          asm volatile("bar.sync 1, %0;" ::"n"(kTtEpi) : "memory");
          // stripe threads: query q, stripe j = landmarks j, j + TPQ, ...
          const int ql = tid / TPQ, j = tid % TPQ;
          const int q = p * QP + ql;
          const int ne = nq[q] < kLm ? nq[q] : kLm;
          const float* row = scr + ql * LD;
          const int R = (K + TPQ - 1) / TPQ;
          TailList<RM> w;
          w.clear(R);
          for (int k = j; k < ne; k += TPQ) {
            const float x = row[k];
            if (x > w.kth_v()) w.insert_stream(x, k);
          }
          // theta0: the smallest of the stripes' R-th values (TPQ * R >= K values reach it);
          // a stripe with fewer than R eligible values leaves -inf (every value is kept)
          float th = w.kth_c() == INT_MAX ? -INFINITY : w.kth_v();
#pragma unroll
          for (int o = 1; o < TPQ; o <<= 1) th = fminf(th, __shfl_xor_sync(0xffffffffu, th, o));
          int mine = 0;
          for (int k = j; k < ne; k += TPQ) mine += row[k] >= th ? 1 : 0;
          // offsets of the stripes' candidates: exclusive scan over the query's TPQ lanes
          int incl = mine;
#pragma unroll
          for (int o = 1; o < TPQ; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o, TPQ);
            if (j >= o) incl += y;
          }
          const int total = __shfl_sync(0xffffffffu, incl, TPQ - 1, TPQ);
          if (total <= CAP) {
            int off = incl - mine;
            for (int k = j; k < ne; k += TPQ) {
              const float x = row[k];
              if (x >= th) {
                cand_v[q * CS + off] = x;
                cand_c[q * CS + off] = k;   // (chunk = k, the first tile)
                ++off;
              }
            }
          }
          asm volatile("bar.sync 1, %0;" ::"n"(kTtEpi) : "memory");
          if (total > CAP) {
            // more candidates than the buffer holds: one thread merges the whole column
            if (j == 0) serial_merge(q, p);
          } else {
            // the list is empty: each candidate's rank among the query's candidates is its
            // place in the sorted list (ties to the lower chunk)
            for (int i = j; i < total; i += TPQ) {
              const float cv = cand_v[q * CS + i];
              const int cc = cand_c[q * CS + i];
              int rank = 0;
              for (int i2 = 0; i2 < total; ++i2)
                rank += better(cand_v[q * CS + i2], cand_c[q * CS + i2], cv, cc) ? 1 : 0;
              if (rank < K) {
                list_v[q * LS + KM - K + rank] = cv;
                list_c[q * LS + KM - K + rank] = cc;
                if (rank == K - 1) theta[q] = cv;
              }
            }
            if (j == 0) cnt[q] = 0;
          }
          asm volatile("bar.sync 1, %0;" ::"n"(kTtEpi) : "memory");
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[a]);
      } else {
        // ---------------------------------------------------------- later tiles
        if (ok) {
#pragma unroll 1
          for (int q0 = half * QH; q0 < (half + 1) * QH; q0 += 16) {
            // eligible queries of this group for this thread's landmark: [qlo, nqv); the group
            // is skipped only when no lane has one (the TMEM loads below are warp-collective)
            const int lo = qlo - q0, hi = nqv - q0;
            const uint32_t emask =
                (hi <= 0 || lo >= 16) ? 0u
                                      : ((lo <= 0 ? 0xFFFFu : (0xFFFFu << lo) & 0xFFFFu) &
                                         (hi >= 16 ? 0xFFFFu : (1u << hi) - 1u));
            if (__all_sync(0xffffffffu, emask == 0u)) continue;
            float sg[16];
            sig16(q0, sg);
            const float4* th4 = reinterpret_cast<const float4*>(theta + q0);
            uint32_t pass = 0;
#pragma unroll
            for (int e4 = 0; e4 < 4; ++e4) {
              const float4 th = th4[e4];
              pass |= (sg[4 * e4] > th.x ? 1u : 0u) << (4 * e4);
              pass |= (sg[4 * e4 + 1] > th.y ? 1u : 0u) << (4 * e4 + 1);
              pass |= (sg[4 * e4 + 2] > th.z ? 1u : 0u) << (4 * e4 + 2);
              pass |= (sg[4 * e4 + 3] > th.w ? 1u : 0u) << (4 * e4 + 3);
            }
            pass &= emask;
            while (pass) {
              const int e = __ffs(pass) - 1;
              pass &= pass - 1;
              float x = 0.f;
#pragma unroll
              for (int e2 = 0; e2 < 16; ++e2) x = e2 == e ? sg[e2] : x;
              const int q = q0 + e;
              const int slot = atomicAdd(&cnt[q], 1);
              if (slot < CAP) {
                cand_v[q * CS + slot] = x;
                cand_c[q * CS + slot] = (int)c;
              } else {
                flags[t & 1] = 1;
              }
            }
          }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kTtEpi) : "memory");
        const bool ovf = *reinterpret_cast<volatile int*>(&flags[t & 1]) != 0;
        if (!ovf) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[a]);
        }
        for (int q = tid; q < MQ; q += kTtEpi) {
          const int n = cnt[q];
          if (n > 0 && n <= CAP) buffer_merge(q, n);
        }
        if (ovf) {
          // a query had more candidates than its buffer: its full column, exactly
#pragma unroll 1
          for (int p = 0; p < SH::NPASS; ++p) {
            asm volatile("bar.sync 1, %0;" ::"n"(kTtEpi) : "memory");
            dump_pass(p);
            asm volatile("bar.sync 1, %0;" ::"n"(kTtEpi) : "memory");
            if (tid < QP) {
              const int qm = p * QP + tid;
              if (cnt[qm] > CAP) serial_merge(qm, p);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[a]);
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kTtEpi) : "memory");
      }
    }
    if (!ok) record_status(status, kStatusTimeout);
    // outputs: one thread per query, best first (sigma desc, c asc), -1 / -inf padded
    for (int q = tid; q < nqv; q += kTtEpi) {
      const int64_t i = i0 + q;
      int32_t* out = idx + (bg * D.N_q + i) * K - (KM - K);
      float* so = s_out ? s_out + (bg * D.N_q + i) * K - (KM - K) : nullptr;
      for (int k = KM - K; k < KM; ++k) {
        const int cc = list_c[q * LS + k];
        out[k] = cc == INT_MAX ? -1 : cc;
        if (so) {
          const float vv = list_v[q * LS + k];
          so[k] = (cc == INT_MAX || vv <= -FLT_MAX) ? -INFINITY : vv;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, SH::TMEM_COLS);
}

// ---------------------------------------------------------------------------------------------
namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode_t() {
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

// 2-D bf16 tensor map over a [rows, d] row-major matrix, boxes of [box_rows, 64], 128-byte
// swizzle (the layout the K-major UMMA descriptors expect).
bool make_map_t(CUtensorMap* map, const void* base, uint64_t rows, uint64_t d,
                uint32_t box_rows) {
  auto enc = get_encode_t();
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

template <int DD, int G, int KM>
cudaError_t launch_t(const Dims& D, const void* qc, const void* klm, const float* blm,
                     int32_t* idx, float* s_out, int32_t* status, cudaStream_t st) {
  using SH = TtShape<DD, G, KM>;
  CUtensorMap tmQc, tmKlm;
  if (!make_map_t(&tmQc, qc, (uint64_t)(D.B * D.Hq * D.N_q), DD, SH::MQ) ||
      !make_map_t(&tmKlm, klm, (uint64_t)(D.B * D.Hkv * (D.C > 0 ? D.C : 1)), DD, kLm))
    return cudaErrorInvalidValue;
  auto kern = score_t_tc_kernel<DD, G, KM>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SH::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((D.N_q + SH::MQ - 1) / SH::MQ), (unsigned)(D.B * D.Hkv));
  kern<<<grid, kTtThreads, SH::SMEM, st>>>(tmQc, tmKlm, D, blm, idx, s_out, status);
  return cudaGetLastError();
}

template <int DD, int G>
cudaError_t launch_t_k(const Dims& D, const void* qc, const void* klm, const float* blm,
                       int32_t* idx, float* s_out, int32_t* status, cudaStream_t st) {
  if (D.K <= 16) return launch_t<DD, G, 16>(D, qc, klm, blm, idx, s_out, status, st);
  if constexpr (DD == 128 && G == 2) return cudaErrorInvalidConfiguration;
  else return launch_t<DD, G, 32>(D, qc, klm, blm, idx, s_out, status, st);
}

}  // namespace

bool score_t_tc_supported(const Dims& D, bool bf16) {
  if (!bf16 || D.K < 1 || D.K > kMaxK || D.C < 1) return false;
  if (D.B * D.Hkv > 65535) return false;
  if (D.d != 64 && D.d != 128) return false;
  // (two heads of 128 dimensions with 32-slot lists do not fit shared memory with a landmark
  // ring of two stages)
  if (D.G == 2 && D.d == 128 && D.K > 16) return false;
  return D.G == 2 || D.G == 4 || D.G == 8;
}

cudaError_t launch_score_topk_t_tc(const Dims& D, const void* qc, const void* klm,
                                   const float* blm, int32_t* idx, float* s_out,
                                   int32_t* status, cudaStream_t st) {
  if (D.B * D.Hkv * D.N_q == 0) return cudaSuccess;
  if (D.d == 128) {
    if (D.G == 2) return launch_t_k<128, 2>(D, qc, klm, blm, idx, s_out, status, st);
    if (D.G == 4) return launch_t_k<128, 4>(D, qc, klm, blm, idx, s_out, status, st);
    return launch_t_k<128, 8>(D, qc, klm, blm, idx, s_out, status, st);
  }
  if (D.G == 2) return launch_t_k<64, 2>(D, qc, klm, blm, idx, s_out, status, st);
  if (D.G == 4) return launch_t_k<64, 4>(D, qc, klm, blm, idx, s_out, status, st);
  return launch_t_k<64, 8>(D, qc, klm, blm, idx, s_out, status, st);
}

}  // namespace hils
