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
// CTA = one (b, g) and 128 consecutive queries; 10 warps:
//   warp 0     TMA producer: the G calibrated-query tiles once, then the landmark tiles
//              through a ring of shared-memory stages;
//   warp 1     allocates 512 TMEM columns (two accumulator sets of G x NT columns) and issues
//              tcgen05.mma from one thread;
//   warps 2-9  epilogue: warp w reads TMEM lanes 32*(w%4).. (its 32 queries) and one half of
//              each tile's columns, so every query has two partial top-K lists, merged at the
//              end.  Candidates that beat a thread's current K-th best are inserted into its
//              sorted register list.
// Every mbarrier wait gives up after a bounded number of polls and records HILS_ERR_TIMEOUT.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace hils {
using namespace sm100;

namespace {

constexpr int kTcThreads = 320;
constexpr int kRows = 128;
constexpr uint32_t kPollLimit = 1u << 24;
constexpr int kSmemLimit = 227 * 1024;

template <int DD, int G, int KM>
struct TcShape {
  static constexpr int NT = 256 / G < 256 ? 256 / G : 256;   // chunks per tile
  static constexpr int KB = DD / 64;                          // 128-byte boxes along d
  static constexpr int A_BOX = kRows * 128;
  static constexpr int A_BYTES = G * KB * A_BOX;
  static constexpr int B_BOX = NT * 128;
  static constexpr int B_STAGE = KB * B_BOX;
  static constexpr int STASH_BYTES = (16 * 256 * 4) > (kRows * KM * 8) ? (16 * 256 * 4)
                                                                       : (kRows * KM * 8);
  static constexpr int FIXED = A_BYTES + STASH_BYTES + 1024 /*barriers*/ + 1024 /*align*/ +
                               2048 /*shared thresholds*/ + 4 * NT * 4 /*bias tiles*/;
  static constexpr int STAGES_FIT = (kSmemLimit - FIXED) / B_STAGE;
  static constexpr int STAGES = STAGES_FIT > 4 ? 4 : STAGES_FIT;
  // more than half of the SM's shared memory, so a second CTA can never be co-resident and
  // compete for the 512 TMEM columns this CTA allocates
  static constexpr int SMEM_USED = FIXED + STAGES * B_STAGE;
  static constexpr int SMEM = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
  static constexpr int HALF = NT / 2;                          // columns per epilogue warp
  static constexpr uint32_t TMEM_COLS = 2 * G * NT;
  static_assert(TMEM_COLS == 512, "two accumulator sets fill TMEM");
  static_assert(STAGES >= 2, "shared memory too small for this shape");
  static_assert(HALF % 16 == 0, "sub-blocks of 16 columns");
};

}  // namespace

template <int DD, int G, int KM>
__global__ void __launch_bounds__(kTcThreads, 1)
    score_topk_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ CUtensorMap tmB, Dims D,
                         const float* __restrict__ blm, int32_t* __restrict__ idx,
                         int32_t* __restrict__ status) {
  using SH = TcShape<DD, G, KM>;
  constexpr int NT = SH::NT;
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
  // each epilogue thread's current K-th best (value, chunk), read by the thread serving the
  // same query in the other column half: [2 halves][128 rows]
  float* th_v = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + 1024);
  int* th_c = reinterpret_cast<int*>(th_v + 2 * kRows);
  // landmark biases of each stage's tile (bulk-copied with the landmark rows when aligned)
  float* sbias = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + 3072);
  const bool bias_bulk = (D.C % 4) == 0 && (reinterpret_cast<uintptr_t>(blm) & 15) == 0;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t qt = (int64_t)gridDim.x - 1 - blockIdx.x;   // longest query tiles first
  const int64_t bg = blockIdx.y;
  const int64_t g = bg % D.Hkv, b = bg / D.Hkv;
  const int64_t i0 = qt * kRows;
  const int64_t i_last = (i0 + kRows - 1 < D.N_q - 1) ? i0 + kRows - 1 : D.N_q - 1;
  const int64_t n_max = n_eligible(D.q_pos0 + i_last, D.S, D.W);
  const int n_tiles = (int)((n_max + NT - 1) / NT);
  const int K = D.K;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SH::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&bias_empty[s], 8);
    }
    mbar_init(a_full, 1);
    for (int a = 0; a < 2; ++a) { mbar_init(&acc_full[a], 1); mbar_init(&acc_empty[a], 8); }
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
      for (int h = 0; h < G; ++h)
        for (int kb = 0; kb < SH::KB; ++kb)
          tma_load_2d(sA + (h * SH::KB + kb) * SH::A_BOX, &tmA, kb * 64,
                      (int32_t)((b * D.Hq + g * G + h) * D.N_q + i0), a_full);
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
        for (int h = 0; h < G; ++h) {
          const uint32_t d_tmem = tmem + (uint32_t)((a * G + h) * NT);
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
    const int e = warp - 2;                 // 0..7
    const int qd = warp & 3;                // TMEM lane quadrant this warp may access
    const int ch = e >> 2;                  // which half of each tile's columns
    const int r = qd * 32 + lane;           // query row within the tile
    const int64_t i = i0 + r;
    const bool valid = i < D.N_q;
    const int64_t n_i = valid ? n_eligible(D.q_pos0 + i, D.S, D.W) : 0;
    const float* bb = blm + bg * D.C;
    float* st = stash + e * 32 + lane;      // stash[j * 256 + thread]
    TailList<KM> L;
    L.clear(K);
    float thv = -INFINITY;
    th_v[ch * kRows + r] = -INFINITY;
    float* my_tv = th_v + ch * kRows + r;
    const float* pa_tv = th_v + (1 - ch) * kRows + r;
    asm volatile("bar.sync 1, 256;" ::: "memory");   // thresholds initialised
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
      for (int sb = 0; sb < SH::HALF / 16; ++sb) {
        const int col0 = ch * SH::HALF + sb * 16;
        const int64_t c0 = (int64_t)t * NT + col0;
        // landmark biases of these 16 chunks
        float bl = 0.f;
        if (!bias_bulk) {
          const int64_t cb = c0 + (lane & 15);
          bl = cb < n_max ? __ldg(bb + cb) : 0.f;
        }
        float sig[16];
        constexpr int HG = G < 4 ? G : 4;     // heads whose TMEM loads are in flight together
#pragma unroll
        for (int h0 = 0; h0 < G; h0 += HG) {
          float tmp[HG][16];
#pragma unroll
          for (int hh = 0; hh < HG; ++hh)
            tmem_ld16(lane_base + (uint32_t)((a * G + h0 + hh) * NT + col0), tmp[hh]);
          tmem_wait_ld();
#pragma unroll
          for (int hh = 0; hh < HG; ++hh)
#pragma unroll
            for (int j = 0; j < 16; ++j)
              sig[j] = (h0 + hh == 0) ? tmp[hh][j] : fmaxf(sig[j], tmp[hh][j]);
        }
        // a candidate must reach both this list's K-th best and the other half's (either list
        // already holds K candidates at least that good); exact ties at the threshold are
        // passed on and resolved by the insertion itself
        const float pv = *reinterpret_cast<const volatile float*>(pa_tv);
        const float thr = fmaxf(thv, pv);
        const int64_t left = n_i - c0;
        const uint32_t vmask = left >= 16 ? 0xFFFFu : (left <= 0 ? 0u : (1u << left) - 1u);
        const float* sbt = sbias + bs * NT + col0;
        uint32_t pass = 0;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float bj = bias_bulk ? sbt[j] : __shfl_sync(0xffffffffu, bl, j);
          sig[j] = fmaf(sig[j], D.scale, bj);
          pass |= (sig[j] >= thr ? 1u : 0u) << j;
        }
        pass &= vmask;
        if (__any_sync(0xffffffffu, pass != 0)) {
#pragma unroll
          for (int j = 0; j < 16; ++j) st[j * 256] = sig[j];
          if (pass) {
            while (pass) {
              const int j = __ffs(pass) - 1;
              pass &= pass - 1;
              L.insert_stream(st[j * 256], (int)(c0 + j));
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
    // merge the two column halves' lists of each query
    asm volatile("bar.sync 1, 256;" ::: "memory");
    float* xv = stash;                                           // [128][KM]
    int* xc = reinterpret_cast<int*>(stash + kRows * KM);        // [128][KM]
    if (ch == 1) {
#pragma unroll
      for (int k = 0; k < KM; ++k) { xv[r * KM + k] = L.v[k]; xc[r * KM + k] = L.c[k]; }
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (ch == 0 && valid) {
      // the partner's live entries are its last K slots
      for (int k = KM - K; k < KM; ++k) {
        const int c = xc[r * KM + k];
        if (c != INT_MAX) L.insert(xv[r * KM + k], c);
      }
      int32_t* out = idx + (bg * D.N_q + i) * K - (KM - K);
#pragma unroll
      for (int k = 0; k < KM; ++k)
        if (k >= KM - K) out[k] = (L.c[k] == INT_MAX) ? -1 : L.c[k];
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

template <int DD, int G, int KM>
cudaError_t launch_tc_t(const Dims& D, const void* qc, const void* klm, const float* blm,
                        int32_t* idx, int32_t* status, cudaStream_t st) {
  using SH = TcShape<DD, G, KM>;
  CUtensorMap tmA, tmB;
  if (!make_map(&tmA, qc, (uint64_t)(D.B * D.Hq * D.N_q), DD, kRows) ||
      !make_map(&tmB, klm, (uint64_t)(D.B * D.Hkv * (D.C > 0 ? D.C : 1)), DD, SH::NT))
    return cudaErrorInvalidValue;
  auto kern = score_topk_tc_kernel<DD, G, KM>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SH::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((D.N_q + kRows - 1) / kRows), (unsigned)(D.B * D.Hkv));
  kern<<<grid, kTcThreads, SH::SMEM, st>>>(tmA, tmB, D, blm, idx, status);
  return cudaGetLastError();
}

template <int DD, int G>
cudaError_t launch_tc_k(const Dims& D, const void* qc, const void* klm, const float* blm,
                        int32_t* idx, int32_t* status, cudaStream_t st) {
  if (D.K <= 16) return launch_tc_t<DD, G, 16>(D, qc, klm, blm, idx, status, st);
  return launch_tc_t<DD, G, 32>(D, qc, klm, blm, idx, status, st);
}

}  // namespace

bool score_tc_supported(const Dims& D, bool bf16) {
  if (!bf16 || D.K < 1 || D.K > kMaxK || D.C < 1) return false;
  if (D.B * D.Hkv > 65535) return false;
  if (D.d == 128) return D.G == 1 || D.G == 2 || D.G == 4;
  if (D.d == 64) return D.G == 1 || D.G == 2 || D.G == 4 || D.G == 8;
  return false;
}

cudaError_t launch_score_topk_tc(const Dims& D, const void* qc, const void* klm,
                                 const float* blm, int32_t* idx, int32_t* status,
                                 cudaStream_t st) {
  if (D.B * D.Hkv * D.N_q == 0) return cudaSuccess;
  if (D.d == 128) {
    if (D.G == 1) return launch_tc_k<128, 1>(D, qc, klm, blm, idx, status, st);
    if (D.G == 2) return launch_tc_k<128, 2>(D, qc, klm, blm, idx, status, st);
    return launch_tc_k<128, 4>(D, qc, klm, blm, idx, status, st);
  }
  if (D.G == 1) return launch_tc_k<64, 1>(D, qc, klm, blm, idx, status, st);
  if (D.G == 2) return launch_tc_k<64, 2>(D, qc, klm, blm, idx, status, st);
  if (D.G == 4) return launch_tc_k<64, 4>(D, qc, klm, blm, idx, status, st);
  return launch_tc_k<64, 8>(D, qc, klm, blm, idx, status, st);
}

}  // namespace hils
