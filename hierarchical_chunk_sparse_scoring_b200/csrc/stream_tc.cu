// Step 1 for decode on the tcgen05 tensor cores: the group score sigma_c = max_h s_{h,c} of
// every eligible landmark of every (b, g, query) row, written as one fp32 row per query for the
// top-K kernel.
//
// [Reader] "The HiLS-Attention Mechanism": the surrogate score s_{h,c} = q_cal . k_lm_c / sqrt(d)
// + b_c; GQA paragraph of "Implementation and Training Recipes": the group selects on the max
// over its heads.  In decode every landmark row is read once per step, so this step is a stream
// of the whole k_lm array (HBM-bound).  The dot products are put on the tensor core so that the
// SMs only move data: a tile of 128 landmark rows (M) times the group's calibrated queries
// (N = 16 rows: the G heads and, above them, rows that are never read) is one tcgen05.mma chain
// of K = d, and each epilogue thread turns its TMEM lane (one landmark) into one sigma.
//
// Persistent CTAs, three per SM: three producers with two stages each kept more copies in flight
// than one CTA with a six-stage ring (measured 5.1 against 4.2 TB/s).  The tiles (row, 128-chunk
// block) are split into contiguous ranges, one per CTA, so a CTA's stream crosses few rows.
// Warp 0: TMA producer (a ring of stages, each one landmark tile plus the row's query tile);
// warp 1: TMEM owner and MMA issuer;
// warps 2-5: epilogue (tcgen05.ld of 16 columns, group max, scale, bias, mask c < n; with gmax,
// each warp also writes the max of its 32 consecutive sigmas, -inf past n, for the top-K
// kernel's two-level scan).
// g_stride: group maxima per row (at least 4 per tile).
// Every mbarrier wait gives up after a bounded number of polls and records HILS_ERR_TIMEOUT.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace hils {
using namespace sm100;

namespace {

constexpr int kStThreads = 192;
constexpr int kStRows = 128;            // landmark rows per tile (MMA M)
constexpr int kStCols = 16;             // query rows per tile (MMA N): the G <= 16 heads
constexpr uint32_t kStPoll = 1u << 24;
constexpr int kStSmemLimit = 227 * 1024;
constexpr int kStCtasPerSm = 3;

template <int DD>
struct StShape {
  static constexpr int KB = DD / 64;
  static constexpr int A_BOX = kStRows * 128;   // [128 rows x 64] bf16
  static constexpr int B_BOX = kStCols * 128;   // [16 rows x 64] bf16
  static constexpr int STAGE = KB * (A_BOX + B_BOX);
  static constexpr int FIXED = 1024 /*align*/ + 1024 /*barriers*/;
  static constexpr int STAGES_FIT = (kStSmemLimit / kStCtasPerSm - FIXED) / STAGE;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr int SMEM = FIXED + STAGES * STAGE;
  static_assert(STAGES >= 2, "shared memory too small");
  // 32 TMEM columns (two accumulators of 16) per CTA: co-resident CTAs never exhaust TMEM
  static_assert(kStCtasPerSm * 32 <= 512, "TMEM columns");
};

}  // namespace

template <int DD>
__global__ void __launch_bounds__(kStThreads, kStCtasPerSm)
    select_stream_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                            const __grid_constant__ CUtensorMap tmB, Dims D, int64_t tiles_per_row,
                            int64_t n_tiles_total, int64_t n_stride,
                            const float* __restrict__ blm, float* __restrict__ sigma,
                            int32_t* __restrict__ status, float* __restrict__ gmax,
                            int64_t g_stride) {
  using SH = StShape<DD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* ring = smem;   // [STAGES][KB A boxes, KB B boxes]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SH::STAGES * SH::STAGE);
  uint64_t* full = bars;                        // [STAGES]
  uint64_t* empty = bars + SH::STAGES;          // [STAGES]
  uint64_t* acc_full = bars + 2 * SH::STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;           // [2]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acc_empty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this CTA's contiguous range of tiles
  const int64_t t_begin = n_tiles_total * blockIdx.x / gridDim.x;
  const int64_t t_end = n_tiles_total * (blockIdx.x + 1) / gridDim.x;
  const int n_local = (int)(t_end - t_begin);

  if (threadIdx.x == 0) {
    for (int s = 0; s < SH::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&acc_full[a], 1); mbar_init(&acc_empty[a], 4); }
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_holder, 32);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0 && n_local > 0) {
      prefetch_tensormap(&tmA);
      prefetch_tensormap(&tmB);
      int last_s = -1;
      uint32_t last_par = 0;
      for (int u = 0; u < n_local; ++u) {
        const int s = u % SH::STAGES;
        const uint32_t ph = (uint32_t)(u / SH::STAGES) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, kStPoll)) {
          record_status(status, kStatusTimeout);
          break;
        }
        const int64_t t = t_begin + u;
        const int64_t row = t / tiles_per_row, tb = t - row * tiles_per_row;
        const int64_t i = row % D.N_q, bg = row / D.N_q;
        const int64_t g = bg % D.Hkv, b = bg / D.Hkv;
        uint8_t* st = ring + s * SH::STAGE;
        mbar_expect_tx(&full[s], SH::STAGE);
        for (int kb = 0; kb < SH::KB; ++kb) {
          tma_load_2d(st + kb * SH::A_BOX, &tmA, kb * 64,
                      (int32_t)(bg * D.C + tb * kStRows), &full[s]);
          // query rows (b, g*G + r, i) for r < 16: a 3-D box over [B*Hq][N_q][d]
          asm volatile(
              "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
              " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
                  smem_u32(st + SH::KB * SH::A_BOX + kb * SH::B_BOX)),
              "l"(reinterpret_cast<uint64_t>(&tmB)), "r"(kb * 64), "r"((int32_t)i),
              "r"((int32_t)(b * D.Hq + g * D.G)), "r"(smem_u32(&full[s]))
              : "memory");
        }
        last_s = s;
        last_par = ph;
      }
      if (last_s >= 0) mbar_wait(&full[last_s], last_par, kStPoll);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0 && n_local > 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(kStRows, kStCols);
      bool ok = true;
      for (int u = 0; ok && u < n_local; ++u) {
        const int s = u % SH::STAGES, a = u & 1;
        const uint32_t ph = (uint32_t)(u / SH::STAGES) & 1u, pa = (uint32_t)(u >> 1) & 1u;
        ok = mbar_wait(&acc_empty[a], pa ^ 1u, kStPoll) && mbar_wait(&full[s], ph, kStPoll);
        if (!ok) break;
        tc_fence_after();
        const uint8_t* st = ring + s * SH::STAGE;
#pragma unroll
        for (int ks = 0; ks < DD / 16; ++ks) {
          const int kb = ks >> 2, kin = ks & 3;
          const uint64_t ad = desc_kmajor_sw128(smem_u32(st + kb * SH::A_BOX) + kin * 32);
          const uint64_t bd =
              desc_kmajor_sw128(smem_u32(st + SH::KB * SH::A_BOX + kb * SH::B_BOX) + kin * 32);
          mma_bf16_ss(tmem + (uint32_t)(a * kStCols), ad, bd, IDESC, ks > 0 ? 1u : 0u);
        }
        mma_commit(&empty[s]);
        mma_commit(&acc_full[a]);
      }
      if (!ok) record_status(status, kStatusTimeout);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int qd = warp & 3;                  // TMEM lane quadrant of this warp
    const int rr = qd * 32 + lane;            // landmark row within the tile
    const uint32_t lane_base = tmem + ((uint32_t)(qd * 32) << 16);
    const int G = D.G;
    bool ok = true;
    for (int u = 0; u < n_local; ++u) {
      const int a = u & 1;
      const uint32_t pa = (uint32_t)(u >> 1) & 1u;
      const int64_t t = t_begin + u;
      const int64_t row = t / tiles_per_row, tb = t - row * tiles_per_row;
      const int64_t i = row % D.N_q, bg = row / D.N_q;
      const int64_t n = n_eligible(D.q_pos0 + i, D.S, D.W);
      const int64_t c = tb * kStRows + rr;
      const bool live = c < n;
      const float bias = live ? __ldg(blm + bg * D.C + c) : 0.f;   // in flight during the wait
      if (!mbar_wait_warp(&acc_full[a], pa, kStPoll)) { ok = false; break; }
      tc_fence_after();
      float v[16];
      tmem_ld16(lane_base + (uint32_t)(a * kStCols), v);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[a]);
      float m = v[0];
#pragma unroll
      for (int h = 1; h < kStCols; ++h)
        if (h < G) m = fmaxf(m, v[h]);
      const float s = fmaf(m, D.scale, bias);
      if (live) sigma[row * n_stride + c] = s;
      if (gmax) {
        const float gm = warp_max(live ? s : -INFINITY);   // chunks c - lane .. c - lane + 31
        if (lane == 0) gmax[row * g_stride + (c >> 5)] = gm;
      }
    }
    if (!ok) record_status(status, kStatusTimeout);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 32);
}

// ---------------------------------------------------------------------------------------------
namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode_st() {
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

template <int DD>
cudaError_t launch_st_t(const Dims& D, const void* qc, const void* klm, const float* blm,
                        float* sigma, int64_t n_stride, int32_t* status, cudaStream_t st,
                        float* gmax, int64_t g_stride) {
  using SH = StShape<DD>;
  auto enc = get_encode_st();
  if (!enc) return cudaErrorInvalidValue;
  CUtensorMap tmA, tmB;
  {
    // k_lm as [B*Hkv*C rows, d], boxes of [128 rows, 64]
    cuuint64_t dims[2] = {(cuuint64_t)DD, (cuuint64_t)(D.B * D.Hkv * D.C)};
    cuuint64_t strides[1] = {(cuuint64_t)DD * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)kStRows};
    cuuint32_t estr[2] = {1, 1};
    if (enc(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(klm), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    // q_cal as [B*Hq][N_q][d], boxes of [16 heads, 1 query, 64]
    cuuint64_t dims[3] = {(cuuint64_t)DD, (cuuint64_t)D.N_q, (cuuint64_t)(D.B * D.Hq)};
    cuuint64_t strides[2] = {(cuuint64_t)DD * 2, (cuuint64_t)(D.N_q * DD * 2)};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)kStCols};
    cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(qc), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  int64_t n_max = 0;
  for (int64_t i = 0; i < D.N_q; ++i) {
    const int64_t n = n_eligible(D.q_pos0 + i, D.S, D.W);
    n_max = n > n_max ? n : n_max;
  }
  if (n_max == 0) return cudaSuccess;
  const int64_t tiles_per_row = (n_max + kStRows - 1) / kStRows;
  const int64_t rows = D.B * D.Hkv * D.N_q;
  const int64_t total = rows * tiles_per_row;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int64_t slots = (int64_t)kStCtasPerSm * sms;
  const int64_t grid = total < slots ? total : slots;
  auto kern = select_stream_tc_kernel<DD>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SH::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)grid, kStThreads, SH::SMEM, st>>>(tmA, tmB, D, tiles_per_row, total, n_stride,
                                                     blm, sigma, status, gmax, g_stride);
  return cudaGetLastError();
}

}  // namespace

bool stream_tc_supported(const Dims& D, bool bf16) {
  if (!bf16 || (D.d != 64 && D.d != 128) || D.G < 1 || D.G > kStCols) return false;
  if (D.C >= (int64_t)INT32_MAX / 2 || D.B * D.Hkv * D.C >= (int64_t)INT32_MAX) return false;
  if (D.B * D.Hq >= (int64_t)INT32_MAX || D.N_q >= (int64_t)INT32_MAX) return false;
  return true;
}

cudaError_t launch_select_stream_tc(const Dims& D, const void* qc, const void* klm,
                                    const float* blm, float* sigma, int64_t n_stride,
                                    int32_t* status, cudaStream_t st, float* gmax,
                                    int64_t g_stride) {
  if (D.B * D.Hkv * D.N_q == 0 || D.C == 0) return cudaSuccess;
  if (D.d == 128)
    return launch_st_t<128>(D, qc, klm, blm, sigma, n_stride, status, st, gmax, g_stride);
  return launch_st_t<64>(D, qc, klm, blm, sigma, n_stride, status, st, gmax, g_stride);
}

}  // namespace hils
