// Steps 1-2 for prefill on the tcgen05 tensor cores (bf16 inputs, fp32 accumulation).
//
// The landmark scores of a tile of 128 queries against a tile of NT chunks are a dense
// contraction S_h = Qcal_h (128 x d) . Klm (NT x d)^T for each head h of the KV group
// ([Reader] "The HiLS-Attention Mechanism", surrogate score; Q-Cal example in "Implementation
// and Training Recipes").  The epilogue fuses everything else of steps 1-2: scale and landmark
// bias, the causal chunk mask (chunk c is eligible for query i iff c < n_i), the group max over
// heads ([Reader] GQA paragraph) and a streaming top-K with ties to the lower chunk index
// ([Reader] "Limitations of Naive Sparse Attention").  No score is written to memory.
//
// CTA = one (b, g) and 128 consecutive queries; 2 + 4*NCG warps:
//   warp 0     TMA producer: the G calibrated-query tiles once, then the landmark tiles
//              through a ring of shared-memory stages;
//   warp 1     allocates 512 TMEM columns (two accumulator sets of G x NT columns) and issues
//              tcgen05.mma from one thread;
//   warps 2..  epilogue: warp w reads TMEM lanes 32*(w%4).. (its 32 queries) and one of NCG
//              column groups of each tile, so every query has NCG partial top-K lists, merged
//              pairwise at the end.  Candidates that reach the best of the NCG lists' current
//              K-th values are inserted into the thread's sorted register list.
//
// Head pairs (HP = 2, used for G = 8 at d = 128, where the G query tiles of 128 rows would not fit
// in shared memory): the 128 MMA rows are 64 queries x 2 heads, interleaved (row 2q + e is query
// q, head 2m + e of accumulator m), loaded by a 3-D TMA box; G/2 accumulators per tile.  Each
// query's score is the max over its two lanes (one shuffle) and the two lanes split the columns,
// so a query has four partial lists (two lanes x two column halves), merged at the end.
// Every mbarrier wait gives up after a bounded number of polls and records HILS_ERR_TIMEOUT.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace hils {
using namespace sm100;

namespace {

constexpr int kRows = 128;

// max of three floats in one instruction (sm_100 three-input max)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
constexpr uint32_t kPollLimit = 1u << 24;
constexpr int kSmemLimit = 227 * 1024;

template <int DD, int G, int KM, int NCG, int HP, int CPS>
struct TcShape {
  static constexpr int THREADS = 64 + 128 * NCG;
  static constexpr int EPI = 128 * NCG;                       // epilogue threads
  static constexpr int MQ = kRows / HP;                       // queries per CTA
  static constexpr int GV = G / HP;                           // accumulators per tile
  // CPS CTAs per SM share its 512 TMEM columns: two accumulator sets of GV x NT each
  static constexpr int NT = (256 / CPS) / GV < 256 ? (256 / CPS) / GV : 256;   // chunks per tile
  static constexpr int KB = DD / 64;                          // 128-byte boxes along d
  static constexpr int A_BOX = kRows * 128;
  static constexpr int A_BYTES = GV * KB * A_BOX;
  static constexpr int B_BOX = NT * 128;
  static constexpr int B_STAGE = KB * B_BOX;
  static constexpr int STASH_A = 16 * EPI * 4;                  // 16 scores per thread
  static constexpr int STASH_B = (NCG / 2) * kRows * KM * 8;     // lists in one merge round
  static constexpr int STASH_BYTES = STASH_A > STASH_B ? STASH_A : STASH_B;
  static constexpr int FIXED = A_BYTES + STASH_BYTES + 1024 /*barriers*/ + 1024 /*align*/ +
                               2048 /*shared thresholds*/ + 4 * NT * 4 /*bias tiles*/;
  static constexpr int STAGES_FIT = ((CPS == 1 ? kSmemLimit : kSmemLimit / CPS - 1024) - FIXED) /
                                    B_STAGE;
  static constexpr int STAGES = STAGES_FIT > 4 ? 4 : STAGES_FIT;
  // more than half of the SM's shared memory, so a second CTA can never be co-resident and
  // compete for the 512 TMEM columns this CTA allocates
  static constexpr int SMEM_USED = FIXED + STAGES * B_STAGE;
  static constexpr int SMEM =
      CPS == 1 ? (SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024) : SMEM_USED;
  static constexpr int CG = NT / NCG;                          // columns per epilogue warp
  static constexpr int HG = GV < 4 ? GV : 4;   // accumulators whose TMEM loads are in flight
  static constexpr uint32_t TMEM_COLS = 2 * GV * NT;
  static_assert(TMEM_COLS * CPS == 512, "the accumulator sets fill TMEM");
  static_assert(STAGES >= 2, "shared memory too small for this shape");
  static_assert(CG % 16 == 0, "sub-blocks of 16 columns");
  static_assert(NCG == 2 || NCG == 4, "two or four column groups");
  static_assert(HP == 1 || (HP == 2 && G % 2 == 0), "head pairs");
};

}  // namespace

template <int DD, int G, int KM, int NCG, int HP, int CPS>
__global__ void __launch_bounds__(64 + 128 * NCG, CPS)
    score_topk_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ CUtensorMap tmB, Dims D,
                         const float* __restrict__ blm, int32_t* __restrict__ idx,
                         float* __restrict__ s_out, int32_t* __restrict__ status) {
  using SH = TcShape<DD, G, KM, NCG, HP, CPS>;
  constexpr int NT = SH::NT;
  constexpr int GV = SH::GV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + SH::A_BYTES;
  float* stash = reinterpret_cast<float*>(sB + SH::STAGES * SH::B_STAGE);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(stash) +
                                               SH::STASH_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + SH::STAGES;
  uint64_t* bias_empty = bars + 2 * SH::STAGES;   // epilogue done with a stage's biases
  uint64_t* a_full = bars + 3 * SH::STAGES;
  uint64_t* acc_full = a_full + 1;      // [2]
  uint64_t* acc_empty = acc_full + 2;   // [2]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_empty + 2);
  // each epilogue thread's current K-th best value, read by the threads serving the same query
  // in the other column groups: [NCG groups][128 rows]
  float* th_v = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + 1024);
  // landmark biases of each stage's tile (bulk-copied with the landmark rows when aligned)
  float* sbias = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + 3072);
  const bool bias_bulk = (D.C % 4) == 0 && (reinterpret_cast<uintptr_t>(blm) & 15) == 0;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t qt = (int64_t)gridDim.x - 1 - blockIdx.x;   // longest query tiles first
  const int64_t bg = blockIdx.y;
  const int64_t g = bg % D.Hkv, b = bg / D.Hkv;
  const int64_t i0 = qt * SH::MQ;
  const int64_t i_last = (i0 + SH::MQ - 1 < D.N_q - 1) ? i0 + SH::MQ - 1 : D.N_q - 1;
  const int64_t n_max = n_eligible(D.q_pos0 + i_last, D.S, D.W);
  const int n_tiles = (int)((n_max + NT - 1) / NT);
  const int K = D.K;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SH::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&bias_empty[s], 4 * NCG);
    }
    mbar_init(a_full, 1);
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4 * NCG);
    }
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_holder, SH::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && n_tiles > 0) {
      prefetch_tensormap(&tmA);
      prefetch_tensormap(&tmB);
      mbar_expect_tx(a_full, SH::A_BYTES);
      for (int h = 0; h < GV; ++h)
        for (int kb = 0; kb < SH::KB; ++kb) {
          if constexpr (HP == 1) {
            tma_load_2d(sA + (h * SH::KB + kb) * SH::A_BOX, &tmA, kb * 64,
                        (int32_t)((b * D.Hq + g * G + h) * D.N_q + i0), a_full);
          } else {
            // [64 queries][2 heads][64] from the (d, head, query) view of q_cal
            asm volatile(
                "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
                " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
                    smem_u32(sA + (h * SH::KB + kb) * SH::A_BOX)),
                "l"(reinterpret_cast<uint64_t>(&tmA)), "r"(kb * 64),
                "r"((int32_t)(b * D.Hq + g * G + 2 * h)), "r"((int32_t)i0),
                "r"(smem_u32(a_full))
                : "memory");
          }
        }
      int last_s = -1;
      uint32_t last_par = 0;
      for (int t = 0; t < n_tiles; ++t) {
        const int s = t % SH::STAGES;
        const uint32_t u = (uint32_t)(t / SH::STAGES);
        if (!mbar_wait(&empty[s], (u & 1u) ^ 1u, kPollLimit) ||
            !mbar_wait(&bias_empty[s], (u & 1u) ^ 1u, kPollLimit)) {
          record_status(status, kStatusTimeout);
          break;
        }
        const int64_t cb0 = (int64_t)t * NT;
        const int brows = (int)(D.C - cb0 < NT ? D.C - cb0 : NT);
        const uint32_t bias_bytes = bias_bulk ? (uint32_t)((brows + 3) / 4 * 16) : 0u;
        mbar_expect_tx(&full[s], SH::B_STAGE + bias_bytes);
        for (int kb = 0; kb < SH::KB; ++kb)
          tma_load_2d(sB + s * SH::B_STAGE + kb * SH::B_BOX, &tmB, kb * 64,
                      (int32_t)(bg * D.C + cb0), &full[s]);
        if (bias_bulk) bulk_load(sbias + s * NT, blm + bg * D.C + cb0, bias_bytes, &full[s]);
        last_s = s;
        last_par = u & 1u;
      }
      // our last copies have landed before this warp leaves (bounded)
      if (last_s >= 0) mbar_wait(&full[last_s], last_par, kPollLimit);
      mbar_wait(a_full, 0, kPollLimit);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(kRows, NT);
      bool ok = mbar_wait(a_full, 0, kPollLimit);
      tc_fence_after();
      for (int t = 0; ok && t < n_tiles; ++t) {
        const int s = t % SH::STAGES;
        const uint32_t u = (uint32_t)(t / SH::STAGES);
        const int a = t & 1;
        const uint32_t v = (uint32_t)(t >> 1);
        ok = mbar_wait(&acc_empty[a], (v & 1u) ^ 1u, kPollLimit) &&
             mbar_wait(&full[s], u & 1u, kPollLimit);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < GV; ++h) {
          const uint32_t d_tmem = tmem + (uint32_t)((a * GV + h) * NT);
#pragma unroll
          for (int ks = 0; ks < DD / 16; ++ks) {
            const int kb = ks >> 2, kin = ks & 3;
            const uint64_t ad = desc_kmajor_sw128(smem_u32(sA + (h * SH::KB + kb) * SH::A_BOX) +
                                                  kin * 32);
            const uint64_t bd = desc_kmajor_sw128(
                smem_u32(sB + s * SH::B_STAGE + kb * SH::B_BOX) + kin * 32);
            mma_bf16_ss(d_tmem, ad, bd, IDESC, ks > 0 ? 1u : 0u);
          }
        }
        mma_commit(&empty[s]);
        mma_commit(&acc_full[a]);
      }
      if (!ok) record_status(status, kStatusTimeout);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int e = warp - 2;                 // 0 .. 4*NCG-1
    const int qd = warp & 3;                // TMEM lane quadrant this warp may access
    const int ch = e >> 2;                  // which column group of each tile
    const int r = qd * 32 + lane;           // MMA row (TMEM lane) of this thread
    const int64_t i = i0 + r / HP;          // its query
    const bool valid = i < D.N_q;
    const int64_t n_i = valid ? n_eligible(D.q_pos0 + i, D.S, D.W) : 0;
    const float* bb = blm + bg * D.C;
    float* st = stash + e * 32 + lane;      // stash[j * EPI + thread]
    TailList<KM> L;
    L.clear(K);
    float thv = -INFINITY;
    th_v[ch * kRows + r] = -INFINITY;
    float* my_tv = th_v + ch * kRows + r;
    asm volatile("bar.sync 1, %0;" ::"n"(SH::EPI) : "memory");   // thresholds initialised
    const uint32_t lane_base = tmem + ((uint32_t)(qd * 32) << 16);
    bool ok = true;
    for (int t = 0; t < n_tiles; ++t) {
      const int a = t & 1;
      const uint32_t v = (uint32_t)(t >> 1);
      const int bs = t % SH::STAGES;
      const uint32_t bu = (uint32_t)(t / SH::STAGES);
      // accumulators of tile t, and (for the biases) the stage's own completion
      if (!mbar_wait_warp(&acc_full[a], v & 1u, kPollLimit) ||
          !mbar_wait_warp(&full[bs], bu & 1u, kPollLimit)) { ok = false; break; }
      tc_fence_after();
#pragma unroll 1
      for (int sb = 0; sb < SH::CG / 16; ++sb) {
        const int col0 = ch * SH::CG + sb * 16;
        const int64_t c0 = (int64_t)t * NT + col0;
        // landmark biases of these 16 chunks
        float bl = 0.f;
        if (!bias_bulk) {
          const int64_t cb = c0 + (lane & 15);
          bl = cb < n_max ? __ldg(bb + cb) : 0.f;
        }
        float sig[16];
        constexpr int HG = SH::HG;
#pragma unroll
        for (int h0 = 0; h0 < GV; h0 += HG) {
          float tmp[HG][16];
#pragma unroll
          for (int hh = 0; hh < HG; ++hh)
            tmem_ld16(lane_base + (uint32_t)((a * GV + h0 + hh) * NT + col0), tmp[hh]);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            // group max over the heads, two new heads per three-input max
            int hh = 0;
            if (h0 == 0) { sig[j] = tmp[0][j]; hh = 1; }
#pragma unroll
            for (; hh + 1 < HG; hh += 2) sig[j] = fmax3(sig[j], tmp[hh][j], tmp[hh + 1][j]);
            if (hh < HG) sig[j] = fmaxf(sig[j], tmp[hh][j]);
          }
        }
        if constexpr (HP == 2) {
          // the other head of each pair sits in the neighbouring lane
#pragma unroll
          for (int j = 0; j < 16; ++j)
            sig[j] = fmaxf(sig[j], __shfl_xor_sync(0xffffffffu, sig[j], 1));
        }
        // a candidate must reach every group's current K-th best (each list already holds K
        // candidates at least that good); exact ties at the threshold are passed on and
        // resolved by the insertion itself
        float thr = thv;
#pragma unroll
        for (int o = 1; o < NCG; ++o)
          thr = fmaxf(thr, *reinterpret_cast<const volatile float*>(
                               th_v + ((ch + o) & (NCG - 1)) * kRows + r));
        if constexpr (HP == 2) {
          // the partner lane's lists serve the same query
#pragma unroll
          for (int o = 0; o < NCG; ++o)
            thr = fmaxf(thr, *reinterpret_cast<const volatile float*>(
                                 th_v + ((ch + o) & (NCG - 1)) * kRows + (r ^ 1)));
        }
        const int64_t left = n_i - c0;
        uint32_t vmask = left >= 16 ? 0xFFFFu : (left <= 0 ? 0u : (1u << left) - 1u);
        if constexpr (HP == 2) vmask &= (lane & 1) ? 0xFF00u : 0x00FFu;   // the pair splits columns
        const float4* sbt = reinterpret_cast<const float4*>(sbias + bs * NT + col0);
#pragma unroll
        for (int j4 = 0; j4 < 4; ++j4) {
          float4 b4;
          if (bias_bulk) {
            b4 = sbt[j4];
          } else {
            b4.x = __shfl_sync(0xffffffffu, bl, 4 * j4);
            b4.y = __shfl_sync(0xffffffffu, bl, 4 * j4 + 1);
            b4.z = __shfl_sync(0xffffffffu, bl, 4 * j4 + 2);
            b4.w = __shfl_sync(0xffffffffu, bl, 4 * j4 + 3);
          }
          sig[4 * j4] = fmaf(sig[4 * j4], D.scale, b4.x);
          sig[4 * j4 + 1] = fmaf(sig[4 * j4 + 1], D.scale, b4.y);
          sig[4 * j4 + 2] = fmaf(sig[4 * j4 + 2], D.scale, b4.z);
          sig[4 * j4 + 3] = fmaf(sig[4 * j4 + 3], D.scale, b4.w);
        }
        // the sub-block's best score decides whether any candidate can pass
        const float m01 = fmax3(sig[0], sig[1], sig[2]), m02 = fmax3(sig[3], sig[4], sig[5]);
        const float m03 = fmax3(sig[6], sig[7], sig[8]), m04 = fmax3(sig[9], sig[10], sig[11]);
        const float m05 = fmax3(sig[12], sig[13], sig[14]);
        const float mx = fmaxf(fmax3(m01, m02, m03), fmax3(m04, m05, sig[15]));
        if (__any_sync(0xffffffffu, mx >= thr && vmask != 0u)) {
          uint32_t pass = 0;
#pragma unroll
          for (int j = 0; j < 16; ++j) pass |= (sig[j] >= thr ? 1u : 0u) << j;
          pass &= vmask;
#pragma unroll
          for (int j = 0; j < 16; ++j) st[j * SH::EPI] = sig[j];
          if (pass) {
            while (pass) {
              const int j = __ffs(pass) - 1;
              pass &= pass - 1;
              L.insert_stream(st[j * SH::EPI], (int)(c0 + j));
            }
            thv = L.kth_v();
            *reinterpret_cast<volatile float*>(my_tv) = thv;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bias_empty[bs]);
        mbar_arrive(&acc_empty[a]);
      }
    }
    if (!ok) record_status(status, kStatusTimeout);
    // merge the column groups' lists of each query pairwise: in each round the upper half of
    // the remaining groups hands its lists to the lower half
    float* xv = stash;                                                   // [NCG/2][128][KM]
    int* xc = reinterpret_cast<int*>(stash + (NCG / 2) * kRows * KM);   // [NCG/2][128][KM]
#pragma unroll
    for (int half = NCG / 2; half >= 1; half >>= 1) {
      asm volatile("bar.sync 1, %0;" ::"n"(SH::EPI) : "memory");
      if (ch >= half && ch < 2 * half) {
        const int o = ((ch - half) * kRows + r) * KM;
#pragma unroll
        for (int k = 0; k < KM; ++k) { xv[o + k] = L.v[k]; xc[o + k] = L.c[k]; }
      }
      asm volatile("bar.sync 1, %0;" ::"n"(SH::EPI) : "memory");
      if (ch < half) {
        // the partner's live entries are its last K slots
        const int o = (ch * kRows + r) * KM;
        for (int k = KM - K; k < KM; ++k) {
          const int c = xc[o + k];
          if (c != INT_MAX) L.insert(xv[o + k], c);
        }
      }
    }
    if constexpr (HP == 2) {
      // then the odd lane of each pair hands its (merged) list to the even lane
      asm volatile("bar.sync 1, %0;" ::"n"(SH::EPI) : "memory");
      if (ch == 0 && (r & 1)) {
#pragma unroll
        for (int k = 0; k < KM; ++k) { xv[r * KM + k] = L.v[k]; xc[r * KM + k] = L.c[k]; }
      }
      asm volatile("bar.sync 1, %0;" ::"n"(SH::EPI) : "memory");
      if (ch == 0 && !(r & 1)) {
        const int o = (r + 1) * KM;
        for (int k = KM - K; k < KM; ++k) {
          const int c = xc[o + k];
          if (c != INT_MAX) L.insert(xv[o + k], c);
        }
      }
    }
    if (ch == 0 && valid && (HP == 1 || !(r & 1))) {
      int32_t* out = idx + (bg * D.N_q + i) * K - (KM - K);
#pragma unroll
      for (int k = 0; k < KM; ++k)
        if (k >= KM - K) out[k] = (L.c[k] == INT_MAX) ? -1 : L.c[k];
      if (s_out) {
        // the winners' scores sigma (with one head per group, that head's surrogate score)
        float* so = s_out + (bg * D.N_q + i) * K - (KM - K);
#pragma unroll
        for (int k = 0; k < KM; ++k)
          if (k >= KM - K)   // (a -inf score was kept as -FLT_MAX in the list)
            so[k] = (L.c[k] == INT_MAX || L.v[k] <= -FLT_MAX) ? -INFINITY : L.v[k];
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

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
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

// 2-D bf16 tensor map over a [rows, d] row-major matrix, boxes of [box_rows, 64] with the
// 128-byte swizzle the UMMA K-major descriptors expect.
bool make_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t d, uint32_t box_rows) {
  auto enc = get_encode();
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

template <int DD, int G, int KM, int NCG, int HP, int CPS>
cudaError_t launch_tc_t(const Dims& D, const void* qc, const void* klm, const float* blm,
                        int32_t* idx, float* s_out, int32_t* status, cudaStream_t st) {
  using SH = TcShape<DD, G, KM, NCG, HP, CPS>;
  CUtensorMap tmA, tmB;
  bool ok_a;
  if constexpr (HP == 1) {
    ok_a = make_map(&tmA, qc, (uint64_t)(D.B * D.Hq * D.N_q), DD, kRows);
  } else {
    // q_cal viewed as (d, head [stride N_q d], query [stride d]): a box of 64 queries x 2 heads
    // lands as 128 rows ordered (query, head)
    auto enc = get_encode();
    cuuint64_t dims[3] = {(cuuint64_t)DD, (cuuint64_t)(D.B * D.Hq), (cuuint64_t)D.N_q};
    cuuint64_t strides[2] = {(cuuint64_t)(D.N_q * DD * 2), (cuuint64_t)DD * 2};
    cuuint32_t box[3] = {64, 2, (cuuint32_t)SH::MQ};
    cuuint32_t estr[3] = {1, 1, 1};
    ok_a = enc && enc(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(qc), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  if (!ok_a || !make_map(&tmB, klm, (uint64_t)(D.B * D.Hkv * (D.C > 0 ? D.C : 1)), DD, SH::NT))
    return cudaErrorInvalidValue;
  auto kern = score_topk_tc_kernel<DD, G, KM, NCG, HP, CPS>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SH::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((D.N_q + SH::MQ - 1) / SH::MQ), (unsigned)(D.B * D.Hkv));
  kern<<<grid, SH::THREADS, SH::SMEM, st>>>(tmA, tmB, D, blm, idx, s_out, status);
  return cudaGetLastError();
}

template <int DD, int G>
cudaError_t launch_tc_k(const Dims& D, const void* qc, const void* klm, const float* blm,
                        int32_t* idx, float* s_out, int32_t* status, cudaStream_t st) {
  // Two column groups: with four, the 18 warps cap a thread at 96 registers and the slower
  // epilogue (spills, fewer TMEM loads in flight) outweighs the extra latency hiding.
  // the list length follows K: an insertion costs a compare and two selects per slot
  // eight heads of 128 dimensions: head pairs (the eight query tiles would not fit)
  constexpr int HP = (G == 8 && DD == 128) ? 2 : 1;
  if (D.K <= 8) {
    // small query tiles and short lists: two CTAs per SM (each one's epilogue latency hides
    // behind the other's)
    if constexpr (DD == 64 && G <= 2)
      return launch_tc_t<DD, G, 8, 2, HP, 2>(D, qc, klm, blm, idx, s_out, status, st);
    return launch_tc_t<DD, G, 8, 2, HP, 1>(D, qc, klm, blm, idx, s_out, status, st);
  }
  if (D.K <= 16) return launch_tc_t<DD, G, 16, 2, HP, 1>(D, qc, klm, blm, idx, s_out, status, st);
  return launch_tc_t<DD, G, 32, 2, HP, 1>(D, qc, klm, blm, idx, s_out, status, st);
}

}  // namespace

bool score_tc_supported(const Dims& D, bool bf16) {
  if (!bf16 || D.K < 1 || D.K > kMaxK || D.C < 1) return false;
  if (D.B * D.Hkv > 65535) return false;
  if (D.d == 128) return D.G == 1 || D.G == 2 || D.G == 4 || D.G == 8;
  if (D.d == 64) return D.G == 1 || D.G == 2 || D.G == 4 || D.G == 8;
  return false;
}

cudaError_t launch_score_topk_tc(const Dims& D, const void* qc, const void* klm,
                                 const float* blm, int32_t* idx, float* s_out, int32_t* status,
                                 cudaStream_t st) {
  if (D.B * D.Hkv * D.N_q == 0) return cudaSuccess;
  if (D.d == 128) {
    if (D.G == 1) return launch_tc_k<128, 1>(D, qc, klm, blm, idx, s_out, status, st);
    if (D.G == 2) return launch_tc_k<128, 2>(D, qc, klm, blm, idx, s_out, status, st);
    if (D.G == 4) return launch_tc_k<128, 4>(D, qc, klm, blm, idx, s_out, status, st);
    return launch_tc_k<128, 8>(D, qc, klm, blm, idx, s_out, status, st);
  }
  if (D.G == 1) return launch_tc_k<64, 1>(D, qc, klm, blm, idx, s_out, status, st);
  if (D.G == 2) return launch_tc_k<64, 2>(D, qc, klm, blm, idx, s_out, status, st);
  if (D.G == 4) return launch_tc_k<64, 4>(D, qc, klm, blm, idx, s_out, status, st);
  return launch_tc_k<64, 8>(D, qc, klm, blm, idx, s_out, status, st);
}

}  // namespace hils
