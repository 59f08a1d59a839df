// Steps 1-2 for prefill on the tcgen05 tensor cores, landmark-major: the product is taken with the
// landmark rows as the MMA's M (128 per tile) and every (head, query) row of a block of
// MQ = 256/G queries as its N (256), so one 128 x 256 x 16 instruction serves all G heads of the
// KV group and each operand is read from shared memory once per 256 output columns
// ([Reader] "The HiLS-Attention Mechanism": surrogate score q_cal . k_lm / sqrt(d) + b; GQA
// paragraph of "Implementation and Training Recipes": the group's score is the max over its
// heads; "Limitations of Naive Sparse Attention": top-K distant chunks, ties to the lower index).
//
// TMEM lane = landmark of the tile, column = head * MQ + query.  Two roles work on the tiles as a
// pipeline:
//   * compare warps (8; one landmark per thread, warp w reads TMEM lanes 32 * (w % 4).. and one
//     half of the queries): per query the max over the G head columns, scale and bias, the causal
//     chunk mask (chunk c is eligible for query q iff c < n_q) and a compare with the query's
//     current K-th best value theta_q.  The tile's scores go to a shared-memory dump and the
//     survivors to one bit each (a warp ballot per query), double-buffered by tile parity.
//   * merge warps (MQ/32; one query per lane, its top-K list in registers): for tile t they take
//     the survivors in chunk order and insert those that beat the list's K-th entry, then
//     publish the new theta_q.  The compare warps work on tile t+1 meanwhile; they read theta
//     at most two tiles old, which only lets more candidates through (theta only grows).
// The first tile has no threshold yet: the compare warps write it to the dump, TPQ threads per
// query each keep the best R = ceil(K/TPQ) values of an interleaved stripe, the smallest of
// their R-th values bounds the query's K-th best from below (TPQ * R >= K values reach it), and
// the values at or above that bound are ranked into the query's sorted list.  A query with more
// of them than the rank buffer holds is merged from its full row by one thread.  Lists hold
// (score, chunk) best first with ties to the lower chunk; no score is written to memory.
//
// CTA = (b, g, MQ queries): warp 0 TMA (the block's calibrated queries once, then the landmark
// tiles through a ring), warp 1 TMEM owner and MMA issuer (two 256-column accumulators), warps
// 2-9 compare, warps 10.. merge.  Every mbarrier wait gives up after a bounded number of polls
// and records HILS_ERR_TIMEOUT.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace hils {
using namespace sm100;

namespace {

constexpr uint32_t kTtPollLimit = 1u << 24;
constexpr int kTtSmemLimit = 227 * 1024;
constexpr int kTtCmp = 256;       // compare threads (warps 2-9)
constexpr int kLm = 128;          // landmark rows per tile (M)
constexpr int kCols = 256;        // (head, query) columns per tile (N)

template <int DD, int G, int KM>
struct TtShape {
  static constexpr int MQ = kCols / G;             // queries per CTA
  static constexpr int QH = MQ / 2;                // queries of one compare half
  static constexpr int NMW = MQ / 32;              // merge warps
  static constexpr int THREADS = 64 + kTtCmp + 32 * NMW;
  static constexpr int TPQ = kTtCmp / MQ;          // first-tile stripe threads per query
  static constexpr int RM = (KM + TPQ - 1) / TPQ;  // stripe list slots
  // dump row stride: TPQ mod 32, so the first tile's stripes read conflict-free
  static constexpr int LD = kLm + TPQ;
  // first-tile rank buffer (values, then chunk ids) and list staging share the row of dump 1
  static constexpr int CAP0 = (LD - 2 * KM) / 2;
  static constexpr int LIST0 = 2 * CAP0;           // offset of the staged list in the row
  static constexpr int KB = DD / 64;
  static constexpr int B_BOX = kCols * 128;        // [256 (head, query) rows x 64 dims]
  static constexpr int B_BYTES = KB * B_BOX;
  static constexpr int A_BOX = kLm * 128;          // [128 landmark rows x 64 dims]
  static constexpr int A_STAGE = KB * A_BOX;
  static constexpr int DUMP_BYTES = 2 * MQ * LD * 4;
  static constexpr int MASK_BYTES = 2 * MQ * 4 * 4;
  static constexpr int MISC_BYTES = MQ * 8 + 64;   // theta, eligible counts
  static constexpr int FIXED = B_BYTES + DUMP_BYTES + MASK_BYTES + MISC_BYTES +
                               256 /*barriers*/ + 1024 /*alignment*/;
  static constexpr int STAGES_FIT = (kTtSmemLimit - FIXED) / A_STAGE;
  static constexpr int STAGES = STAGES_FIT > 4 ? 4 : STAGES_FIT;
  // more than half of the SM's shared memory, so no second CTA is co-resident and competes for
  // the 512 TMEM columns this CTA allocates
  static constexpr int SMEM_USED = FIXED + STAGES * A_STAGE;
  static constexpr int SMEM = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
  static constexpr uint32_t TMEM_COLS = 512;       // two 256-column accumulators
  static_assert(STAGES >= 2, "shared memory too small for this shape");
  static_assert(QH % 16 == 0 && MQ % 32 == 0, "queries in groups of 16, merge warps of 32");
  static_assert((MQ * 128) % 1024 == 0, "whole swizzle atoms per head");
  static_assert(32 % TPQ == 0 && MQ * TPQ == kTtCmp, "stripe threads");
  static_assert(TPQ * RM >= KM, "witnesses");
  static_assert(CAP0 >= KM, "rank buffer");
  static_assert(MQ * KM * 4 <= A_STAGE, "final chunk ids in one ring stage");
};

// Parity of the wait for the u-th completion of a barrier phase sequence.
__device__ __forceinline__ uint32_t par(int u) { return (uint32_t)u & 1u; }

}  // namespace

// m16n8k16 bf16 MMA with fp32 accumulation (the legacy warp-level form: the per-head scores of a
// block's winners are a few hundred such products, a gather per query, not a streamed GEMM).
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Every head's surrogate score of each selected chunk, q_cal[h] . k_lm[c] * scale + b_lm[c]
// (-inf for an empty slot), from the block's calibrated queries still in shared memory, so the
// attention step need not score the chunks again.  A job is one query and 16 of its list slots:
// one warp takes a 16 (slots) x 8 (heads) x d product on the tensor cores, A = the slots'
// landmark rows gathered from global memory, B = the query's G head rows of the q_cal tile
// (heads past G are zero).  A dot product does not depend on the order of its terms, so each
// lane loads whole 16-byte pieces and the fragment's k positions are assigned to dims in the
// order the pieces arrive: lane (r, c) = (lane / 4, lane % 4) holds dims 32m + 8c .. 32m + 8c + 7
// of rows r and r + 8 of A and of column r of B, the first half of them for the MMA of k step 2m
// and the second half for step 2m + 1, the same assignment on both operands.  The block waits
// for this at its end, so the gathers of JB jobs per warp are issued together (one memory
// latency per JB jobs rather than two per job).
template <int DD, int G, int KM>
__device__ __noinline__ void head_scores(const Dims& D, const int* __restrict__ fin,
                                         const uint8_t* sB, bool have_q, int64_t b, int64_t g,
                                         int64_t bg, int64_t i0, int nqv,
                                         const __nv_bfloat16* __restrict__ klm,
                                         const float* __restrict__ blm,
                                         float* __restrict__ s_head) {
  using SH = TtShape<DD, G, KM>;
  constexpr int MQ = SH::MQ, NW = SH::THREADS / 32;
  constexpr int MS = DD / 32;   // 32-dim segments of a row
  constexpr int JB = 3;         // jobs of a warp in flight together
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = lane >> 2, c = lane & 3;
  const int K = D.K;
  const int n_t16 = (K + 15) / 16;
  const int n_jobs = nqv * n_t16;
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  for (int base = warp; base < n_jobs; base += NW * JB) {
    uint4 A0[JB][MS], A1[JB][MS];
    int ca[JB], cb[JB];
    float ba[JB], bb[JB];
#pragma unroll
    for (int jj = 0; jj < JB; ++jj) {
      const int job = base + jj * NW;
      const int q = job / n_t16, k0 = (job - q * n_t16) * 16;
      const int ka = k0 + r, kb = ka + 8;
      ca[jj] = job < n_jobs && ka < K ? fin[q * K + ka] : -1;
      cb[jj] = job < n_jobs && kb < K ? fin[q * K + kb] : -1;
      const uint4* ra = reinterpret_cast<const uint4*>(klm + (bg * D.C + max(ca[jj], 0)) * DD);
      const uint4* rb = reinterpret_cast<const uint4*>(klm + (bg * D.C + max(cb[jj], 0)) * DD);
#pragma unroll
      for (int m = 0; m < MS; ++m) {
        A0[jj][m] = have_q && ca[jj] >= 0 ? __ldg(ra + m * 4 + c) : z;
        A1[jj][m] = have_q && cb[jj] >= 0 ? __ldg(rb + m * 4 + c) : z;
      }
      ba[jj] = ca[jj] >= 0 ? __ldg(blm + bg * D.C + ca[jj]) : 0.f;
      bb[jj] = cb[jj] >= 0 ? __ldg(blm + bg * D.C + cb[jj]) : 0.f;
    }
#pragma unroll
    for (int jj = 0; jj < JB; ++jj) {
      const int job = base + jj * NW;
      if (job >= n_jobs) break;   // (warp-uniform)
      const int q = job / n_t16, k0 = (job - q * n_t16) * 16;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      const int row = r * MQ + q;   // column r of B: head r's row of the q_cal tile
#pragma unroll
      for (int m = 0; m < MS; ++m) {
        const int u = m * 4 + c;    // 16-byte piece of the row
        const uint4 bq = have_q && r < G
                             ? *reinterpret_cast<const uint4*>(
                                   sB + (u >> 3) * SH::B_BOX + (row >> 3) * 1024 +
                                   (row & 7) * 128 + (((u & 7) ^ (row & 7)) << 4))
                             : z;
        mma_16816(acc, A0[jj][m].x, A1[jj][m].x, A0[jj][m].y, A1[jj][m].y, bq.x, bq.y);
        mma_16816(acc, A0[jj][m].z, A1[jj][m].z, A0[jj][m].w, A1[jj][m].w, bq.z, bq.w);
      }
      // acc: (slot ka, head 2c), (ka, 2c + 1), (kb, 2c), (kb, 2c + 1)
      const int64_t i = i0 + q;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int h = 2 * c + (e & 1);
        const int k = k0 + r + (e < 2 ? 0 : 8);
        const int ch = e < 2 ? ca[jj] : cb[jj];
        if (h < G && k < K)
          s_head[((b * D.Hq + g * G + h) * D.N_q + i) * K + k] =
              ch >= 0 ? fmaf(acc[e], D.scale, e < 2 ? ba[jj] : bb[jj]) : -INFINITY;
      }
    }
  }
}

template <int DD, int G, int KM>
__global__ void __launch_bounds__(TtShape<DD, G, KM>::THREADS, 1)
    score_t_tc_kernel(const __grid_constant__ CUtensorMap tmQc,
                      const __grid_constant__ CUtensorMap tmKlm, Dims D,
                      const float* __restrict__ blm, int32_t* __restrict__ idx,
                      float* __restrict__ s_out, float* __restrict__ s_head,
                      const __nv_bfloat16* __restrict__ klm, int32_t* __restrict__ status) {
  using SH = TtShape<DD, G, KM>;
  constexpr int MQ = SH::MQ, QH = SH::QH, TPQ = SH::TPQ, RM = SH::RM, LD = SH::LD;
  constexpr int CAP0 = SH::CAP0, LIST0 = SH::LIST0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sB = smem;                                                    // q_cal block (N)
  uint8_t* sA = sB + SH::B_BYTES;                                        // landmark ring (M)
  float* dump = reinterpret_cast<float*>(sA + SH::STAGES * SH::A_STAGE);   // [2][MQ][LD]
  uint32_t* mask = reinterpret_cast<uint32_t*>(dump + 2 * MQ * LD);      // [2][MQ][4]
  float* theta = reinterpret_cast<float*>(mask + 2 * MQ * 4);            // [MQ]
  int* nq = reinterpret_cast<int*>(theta + MQ);                          // [MQ]
  uint64_t* bars = reinterpret_cast<uint64_t*>(
      (reinterpret_cast<uintptr_t>(nq + MQ + 16) + 7) & ~static_cast<uintptr_t>(7));
  uint64_t* full = bars;                     // [STAGES] landmark tile landed
  uint64_t* empty = bars + SH::STAGES;       // [STAGES] its MMAs completed
  uint64_t* b_full = bars + 2 * SH::STAGES;  // calibrated queries landed
  uint64_t* acc_full = b_full + 1;           // [2]
  uint64_t* acc_empty = acc_full + 2;        // [2] compare warps read the accumulator
  uint64_t* cf = acc_empty + 2;              // [2] a tile's dump and survivor bits written
  uint64_t* df = cf + 2;                     // [2] the merge warps are done with that dump
  uint64_t* lists_ready = df + 2;            // the first tile's lists are staged
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(lists_ready + 1);

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
      mbar_init(&acc_empty[a], kTtCmp / 32);
      mbar_init(&cf[a], kTtCmp / 32);
      mbar_init(&df[a], SH::NMW);
    }
    mbar_init(lists_ready, kTtCmp / 32);
    fence_barrier_init();
  }
  for (int q = threadIdx.x; q < MQ; q += SH::THREADS) {
    theta[q] = -INFINITY;
    nq[q] = q < nqv ? (int)n_eligible(D.q_pos0 + i0 + q, D.S, D.W) : 0;
  }
  for (int e = threadIdx.x; e < 2 * MQ * 4; e += SH::THREADS) mask[e] = 0u;
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
  } else if (warp < 2 + kTtCmp / 32) {
    // ------------------------------------------------------------ compare warps
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
      const int a = t & 1, bsel = t & 1;
      const uint32_t v = (uint32_t)(t >> 1);
      const int64_t c = (int64_t)t * kLm + r;   // this thread's landmark
      const float bias = bias_next;
      {   // the next tile's bias loads while this one is processed
        const int64_t cn = c + kLm;
        bias_next = cn < D.C ? __ldg(bb + cn) : 0.f;
      }
      // first query of the block for which chunk c is eligible: c < n(p) <=> p >= (c+1)S + W - 1
      const int64_t qmin64 = (c + 1) * D.S + D.W - 1 - D.q_pos0 - i0;
      const int qlo = qmin64 < 0 ? 0 : (qmin64 > MQ ? MQ : (int)qmin64);
      float* dmp = dump + bsel * MQ * LD;
      // (waits are warp-uniform; after a timeout a warp stops waiting and touching TMEM)
      if (ok) ok = mbar_wait_warp(&acc_full[a], v & 1u, kTtPollLimit);
      if (t >= 1 && ok) {
        // the merge warps are done with this dump: its (t-1)/2-th release (tiles 1 and 2 wait
        // for the first one, given once the first tile's lists are loaded)
        ok = mbar_wait_warp(&df[bsel], par((t - 1) >> 1), kTtPollLimit);
      }
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
      if (t == 0) {
        // ---------------------------------------------------------- first tile
        // the whole tile, query-major (a -inf score is kept as the lowest finite value so that
        // it can still fill an empty slot; ineligible entries are never read)
        if (ok) {
#pragma unroll 1
          for (int q0 = half * QH; q0 < (half + 1) * QH; q0 += 16) {
            float sg[16];
            sig16(q0, sg);
#pragma unroll
            for (int e = 0; e < 16; ++e) dmp[(q0 + e) * LD + r] = fmaxf(sg[e], -FLT_MAX);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[a]);
        asm volatile("bar.sync 1, %0;" ::"n"(kTtCmp) : "memory");
        // stripe threads: query q, stripe j = landmarks j, j + TPQ, ...
        const int q = tid / TPQ, j = tid % TPQ;
        const int ne = nq[q] < kLm ? nq[q] : kLm;
        const float* row = dmp + q * LD;
        float* stage = dump + MQ * LD + q * LD;   // the row of dump 1 (rank buffer, list)
        const int R = (K + TPQ - 1) / TPQ;
        // the stripe's values, loaded at once (independent loads in flight), kept for the passes
        constexpr int NS = kLm / TPQ;
        float xs[NS];
#pragma unroll
        for (int u = 0; u < NS; ++u) xs[u] = row[j + u * TPQ];
        TailList<RM> w;
        w.clear(R);
#pragma unroll
        for (int u = 0; u < NS; ++u)
          if (j + u * TPQ < ne && xs[u] > w.kth_v()) w.insert_stream(xs[u], u);
        // theta0: the smallest of the stripes' R-th values (TPQ * R >= K values reach it);
        // a stripe with fewer than R eligible values leaves -inf (every value is kept)
        float th = w.kth_c() == INT_MAX ? -INFINITY : w.kth_v();
#pragma unroll
        for (int o = 1; o < TPQ; o <<= 1) th = fminf(th, __shfl_xor_sync(0xffffffffu, th, o));
        uint32_t keep = 0;   // bit u: value u of the stripe is a candidate
#pragma unroll
        for (int u = 0; u < NS; ++u)
          keep |= (j + u * TPQ < ne && xs[u] >= th ? 1u : 0u) << u;
        const int mine = __popc(keep);
        // offsets of the stripes' candidates: exclusive scan over the query's TPQ lanes
        int incl = mine;
#pragma unroll
        for (int o = 1; o < TPQ; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o, TPQ);
          if (j >= o) incl += y;
        }
        const int total = __shfl_sync(0xffffffffu, incl, TPQ - 1, TPQ);
        if (total <= CAP0) {
          int off = incl - mine;
#pragma unroll
          for (int u = 0; u < NS; ++u) {
            if ((keep >> u) & 1u) {
              stage[off] = xs[u];
              stage[CAP0 + off] = __int_as_float(j + u * TPQ);   // (chunk, the first tile)
              ++off;
            }
          }
        }
        // the staged list starts empty: K live slots (-inf, INT_MAX) at the end of KM
        for (int k = j; k < KM; k += TPQ) {
          const bool sentinel = k < KM - K;
          stage[LIST0 + k] = sentinel ? INFINITY : -INFINITY;
          stage[LIST0 + KM + k] = __int_as_float(sentinel ? -1 : INT_MAX);
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kTtCmp) : "memory");
        if (total > CAP0) {
          // more candidates than the rank buffer holds: one thread merges the whole row
          if (j == 0) {
            TailList<KM> L;
            L.clear(K);
            for (int k = 0; k < ne; ++k) {
              const float x = row[k];
              if (x > L.kth_v()) L.insert_stream(x, k);
            }
#pragma unroll
            for (int k = 0; k < KM; ++k) {
              stage[LIST0 + k] = L.v[k];
              stage[LIST0 + KM + k] = __int_as_float(L.c[k]);
            }
            theta[q] = L.kth_c() == INT_MAX ? -INFINITY : L.kth_v();
          }
        } else {
          // each candidate's rank among the query's candidates is its place in the sorted
          // list (ties to the lower chunk): this thread's candidates i = j, j + TPQ, ... are held
          // in registers and every candidate of the query is read once
          constexpr int NMC = (CAP0 + TPQ - 1) / TPQ;
          float mv[NMC];
          int mc[NMC], rk[NMC];
#pragma unroll
          for (int m = 0; m < NMC; ++m) {
            const int i = j + m * TPQ;
            mv[m] = i < total ? stage[i] : -INFINITY;
            mc[m] = i < total ? __float_as_int(stage[CAP0 + i]) : INT_MAX;
            rk[m] = 0;
          }
          int i2 = 0;
          for (; i2 + 4 <= total; i2 += 4) {
            float ov[4];
            int oc[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              ov[e] = stage[i2 + e];
              oc[e] = __float_as_int(stage[CAP0 + i2 + e]);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e)
#pragma unroll
              for (int m = 0; m < NMC; ++m) rk[m] += better(ov[e], oc[e], mv[m], mc[m]) ? 1 : 0;
          }
          for (; i2 < total; ++i2) {
            const float ov = stage[i2];
            const int oc = __float_as_int(stage[CAP0 + i2]);
#pragma unroll
            for (int m = 0; m < NMC; ++m) rk[m] += better(ov, oc, mv[m], mc[m]) ? 1 : 0;
          }
#pragma unroll
          for (int m = 0; m < NMC; ++m) {
            if (j + m * TPQ < total && rk[m] < K) {
              stage[LIST0 + KM - K + rk[m]] = mv[m];
              stage[LIST0 + KM + KM - K + rk[m]] = __int_as_float(mc[m]);
              if (rk[m] == K - 1) theta[q] = mv[m];
            }
          }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kTtCmp) : "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(lists_ready);
      } else {
        // ---------------------------------------------------------- later tiles
        uint32_t* msk = mask + bsel * MQ * 4;
        if (ok) {
#pragma unroll 1
          for (int q0 = half * QH; q0 < (half + 1) * QH; q0 += 16) {
            // eligible queries of this group for this thread's landmark: [qlo, nqv); the group
            // is skipped only when no lane has one (the TMEM loads below are warp-collective;
            // the merge warps left this tile's survivor words at 0)
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
            // (once the thresholds have settled most groups have no survivor in the warp)
            if (__any_sync(0xffffffffu, pass != 0u)) {
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                if ((pass >> e) & 1u) dmp[(q0 + e) * LD + r] = sg[e];
                const uint32_t bits = __ballot_sync(0xffffffffu, (pass >> e) & 1u);
                if (lane == 0 && bits) msk[(q0 + e) * 4 + qd] = bits;
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&acc_empty[a]);
          mbar_arrive(&cf[bsel]);
        }
      }
    }
    if (!ok) record_status(status, kStatusTimeout);
  } else {
    // ------------------------------------------------------------ merge warps
    const int q = (warp - 2 - kTtCmp / 32) * 32 + lane;   // this lane's query
    TailList<KM> L;
    L.clear(K);
    bool ok = true;
    if (n_tiles > 0) {
      ok = mbar_wait_warp(lists_ready, 0, kTtPollLimit);
      const float* stage = dump + MQ * LD + q * LD;
      if (ok) {
#pragma unroll
        for (int k = 0; k < KM; ++k) {
          L.v[k] = stage[LIST0 + k];
          L.c[k] = __float_as_int(stage[LIST0 + KM + k]);
        }
      }
      __syncwarp();
      if (lane == 0) {   // both dumps are free for tiles 1 and 2
        mbar_arrive(&df[0]);
        mbar_arrive(&df[1]);
      }
      for (int t = 1; ok && t < n_tiles; ++t) {
        const int bsel = t & 1;
        ok = mbar_wait_warp(&cf[bsel], par((t - 1) >> 1), kTtPollLimit);
        if (!ok) break;
        const float* row = dump + bsel * MQ * LD + q * LD;
        uint32_t* msk = mask + bsel * MQ * 4 + q * 4;
        const int64_t cb = (int64_t)t * kLm;
#pragma unroll
        for (int w4 = 0; w4 < 4; ++w4) {
          uint32_t bits = msk[w4];
          if (bits) msk[w4] = 0u;
          // survivors in chunk order: every list entry is from an earlier chunk, so a strict
          // value compare gives the (score desc, chunk asc) order
          while (bits) {
            const int rr = w4 * 32 + __ffs(bits) - 1;
            bits &= bits - 1u;
            const float x = row[rr];
            if (x > L.kth_v()) L.insert_stream(x, (int)(cb + rr));
          }
        }
        theta[q] = L.kth_c() == INT_MAX ? -INFINITY : L.kth_v();
        __syncwarp();
        if (lane == 0) mbar_arrive(&df[bsel]);
      }
    }
    if (!ok) record_status(status, kStatusTimeout);
    // outputs: best first (sigma desc, c asc), -1 / -inf padded; the chunk ids also go to
    // shared memory for the per-head scores below, into the landmark ring: every tile's MMAs
    // have completed once a merge warp is past the last tile (the dumps are not free yet: with
    // two merge warps the other may still be reading one)
    int* fin = reinterpret_cast<int*>(sA);   // [MQ][K]
#pragma unroll
    for (int k = 0; k < KM; ++k)
      if (k >= KM - K) fin[q * K + k - (KM - K)] = L.c[k] == INT_MAX ? -1 : L.c[k];
    if (q < nqv) {
      const int64_t i = i0 + q;
      int32_t* out = idx + (bg * D.N_q + i) * K - (KM - K);
      float* so = s_out ? s_out + (bg * D.N_q + i) * K - (KM - K) : nullptr;
#pragma unroll
      for (int k = 0; k < KM; ++k) {
        if (k >= KM - K) {
          out[k] = L.c[k] == INT_MAX ? -1 : L.c[k];
          if (so) so[k] = (L.c[k] == INT_MAX || L.v[k] <= -FLT_MAX) ? -INFINITY : L.v[k];
        }
      }
    }
  }
  if (s_head) {
    __syncthreads();   // fin complete
    const bool have_q = n_tiles > 0 && mbar_wait(b_full, 0, kTtPollLimit);
    head_scores<DD, G, KM>(D, reinterpret_cast<const int*>(sA), sB, have_q, b, g, bg, i0, nqv,
                           klm, blm, s_head);
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
                     int32_t* idx, float* s_out, float* s_head, int32_t* status,
                     cudaStream_t st) {
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
  kern<<<grid, SH::THREADS, SH::SMEM, st>>>(tmQc, tmKlm, D, blm, idx, s_out, s_head,
                                            (const __nv_bfloat16*)klm, status);
  return cudaGetLastError();
}

template <int DD, int G>
cudaError_t launch_t_k(const Dims& D, const void* qc, const void* klm, const float* blm,
                       int32_t* idx, float* s_out, float* s_head, int32_t* status,
                       cudaStream_t st) {
  if (D.K <= 16) return launch_t<DD, G, 16>(D, qc, klm, blm, idx, s_out, s_head, status, st);
  return launch_t<DD, G, 32>(D, qc, klm, blm, idx, s_out, s_head, status, st);
}

}  // namespace

bool score_t_tc_supported(const Dims& D, bool bf16) {
  if (!bf16 || D.K < 1 || D.K > kMaxK || D.C < 1) return false;
  if (D.B * D.Hkv > 65535) return false;
  if (D.d != 64 && D.d != 128) return false;
  return D.G == 4 || D.G == 8;
}

cudaError_t launch_score_topk_t_tc(const Dims& D, const void* qc, const void* klm,
                                   const float* blm, int32_t* idx, float* s_out,
                                   float* s_head, int32_t* status, cudaStream_t st) {
  if (D.B * D.Hkv * D.N_q == 0) return cudaSuccess;
  if (D.d == 128) {
    if (D.G == 4) return launch_t_k<128, 4>(D, qc, klm, blm, idx, s_out, s_head, status, st);
    return launch_t_k<128, 8>(D, qc, klm, blm, idx, s_out, s_head, status, st);
  }
  if (D.G == 4) return launch_t_k<64, 4>(D, qc, klm, blm, idx, s_out, s_head, status, st);
  return launch_t_k<64, 8>(D, qc, klm, blm, idx, s_out, s_head, status, st);
}

}  // namespace hils
