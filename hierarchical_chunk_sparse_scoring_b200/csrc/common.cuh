// Device helpers shared by the HiLS kernels: element loads, warp reductions, the candidate
// ordering used by every top-K, and the eligibility rule.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cfloat>
#include <climits>

namespace hils {

constexpr int kMaxK = 32;        // largest K_top supported
constexpr int kMaxD = 128;       // largest head dim supported
constexpr int kStatusTimeout = 6;
constexpr int kStatusDeviceCheck = 5;

// Problem description handed to every kernel (plain values, no pointers).
struct Dims {
  int64_t B, Hq, Hkv, N_q, N_kv, d, q_pos0;
  int64_t C;       // completed chunks = floor(N_kv / S)
  int32_t S, K, W, G;
  float scale;
};

// Eligible distant chunks of the query at position pos: the chunks that end before the
// W-token window [pos-W+1, pos] starts; the local window then runs from S*n to pos.
__host__ __device__ __forceinline__ int64_t n_eligible(int64_t pos, int32_t S, int32_t W) {
  int64_t first = pos - (int64_t)W + 1;
  return first <= 0 ? 0 : first / S;
}

template <typename T>
struct Elem;

template <>
struct Elem<float> {
  static __device__ __forceinline__ float to_f(float x) { return x; }
  static __device__ __forceinline__ float from_f(float x) { return x; }
  // four consecutive elements, 16-byte aligned
  static __device__ __forceinline__ void load4(const float* p, float (&v)[4]) {
    float4 t = __ldg(reinterpret_cast<const float4*>(p));
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
  }
  static __device__ __forceinline__ void store4(float* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <>
struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
  // four consecutive elements, 8-byte aligned
  static __device__ __forceinline__ void load4(const __nv_bfloat16* p, float (&v)[4]) {
    uint2 t = __ldg(reinterpret_cast<const uint2*>(p));
    v[0] = bf16_lo(t.x); v[1] = bf16_hi(t.x); v[2] = bf16_lo(t.y); v[3] = bf16_hi(t.y);
  }
  static __device__ __forceinline__ void store4(__nv_bfloat16* p, const float (&v)[4]) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
    uint2 t;
    t.x = *reinterpret_cast<uint32_t*>(&a);
    t.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = t;
  }
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Candidate order of the selection: larger score first, equal scores -> lower chunk index.
// An empty slot is (-inf, INT_MAX), so a real -inf candidate still beats it.
__device__ __forceinline__ bool better(float v, int c, float ov, int oc) {
  return v > ov || (v == ov && c < oc);
}

// Sorted top-KM list held in registers (static indexing only).  Slots >= K stay empty.
template <int KM>
struct TopList {
  float v[KM];
  int c[KM];

  __device__ __forceinline__ void clear() {
#pragma unroll
    for (int k = 0; k < KM; ++k) { v[k] = -INFINITY; c[k] = INT_MAX; }
  }

  // Inserts (x, ci) if it beats slot K-1; keeps the list ordered by `better`.  Because the list
  // is sorted, "x beats slot k" holds exactly for the slots from x's position on, so every slot's
  // new content follows from the old list in parallel (no dependent chain through the slots):
  // slot k takes x if x beats it but not slot k-1, slot k-1's old entry if x beats both.
  __device__ __forceinline__ void insert(float x, int ci, int K) {
    bool m[KM];
#pragma unroll
    for (int k = 0; k < KM; ++k) m[k] = (k < K) && better(x, ci, v[k], c[k]);
#pragma unroll
    for (int k = KM - 1; k >= 0; --k) {
      if (m[k]) {
        const bool shift = k > 0 && m[k - 1];
        v[k] = shift ? v[k - 1] : x;
        c[k] = shift ? c[k - 1] : ci;
      }
    }
  }

  __device__ __forceinline__ void pop_front() {
#pragma unroll
    for (int k = 0; k < KM - 1; ++k) { v[k] = v[k + 1]; c[k] = c[k + 1]; }
    v[KM - 1] = -INFINITY;
    c[KM - 1] = INT_MAX;
  }
};

// Sorted list of the K best candidates kept in the LAST K of KM register slots; the first KM-K
// slots hold unbeatable sentinels (+inf), so the K-th best is always slot KM-1 and no access
// depends on the runtime K (dynamic indexing would move the list to local memory).
template <int KM>
struct TailList {
  float v[KM];
  int c[KM];

  __device__ __forceinline__ void clear(int K) {
#pragma unroll
    for (int k = 0; k < KM; ++k) {
      const bool sentinel = k < KM - K;
      v[k] = sentinel ? INFINITY : -INFINITY;
      c[k] = sentinel ? -1 : INT_MAX;
    }
  }

  // Parallel insertion as in TopList::insert (sentinels are never beaten).
  __device__ __forceinline__ void insert(float x, int ci) {
    bool m[KM];
#pragma unroll
    for (int k = 0; k < KM; ++k) m[k] = better(x, ci, v[k], c[k]);
#pragma unroll
    for (int k = KM - 1; k >= 0; --k) {
      if (m[k]) {
        const bool shift = k > 0 && m[k - 1];
        v[k] = shift ? v[k - 1] : x;
        c[k] = shift ? c[k - 1] : ci;
      }
    }
  }

  // Insertion for a candidate from the thread's own chunk stream: every entry already in the
  // list came earlier in that stream (lower chunk index), so an equal value never moves ahead of
  // one and a strict value compare gives the same order as `better`.  -inf is clamped to the
  // lowest finite value so it still fills an empty (-inf) slot.
  __device__ __forceinline__ void insert_stream(float x, int ci) {
    x = fmaxf(x, -FLT_MAX);
    bool m[KM];
#pragma unroll
    for (int k = 0; k < KM; ++k) m[k] = x > v[k];
#pragma unroll
    for (int k = KM - 1; k >= 0; --k) {
      if (m[k]) {
        const bool shift = k > 0 && m[k - 1];
        v[k] = shift ? v[k - 1] : x;
        c[k] = shift ? c[k - 1] : ci;
      }
    }
  }

  __device__ __forceinline__ float kth_v() const { return v[KM - 1]; }
  __device__ __forceinline__ int kth_c() const { return c[KM - 1]; }
};

// Warp-wide arg-best of one (value, index) per lane under `better`; every lane gets it.
__device__ __forceinline__ void warp_best(float& v, int& c) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float ov = __shfl_xor_sync(0xffffffffu, v, o);
    int oc = __shfl_xor_sync(0xffffffffu, c, o);
    if (better(ov, oc, v, c)) { v = ov; c = oc; }
  }
}

// Merges the 32 lanes' sorted lists into the warp's top-K.  Result slot r (r < K) is
// returned in lane r (value, index); other lanes get the empty slot.
template <int KM>
__device__ __forceinline__ void warp_merge_topk(TopList<KM>& L, int K, int lane, float& out_v,
                                                int& out_c) {
  out_v = -INFINITY;
  out_c = INT_MAX;
  for (int r = 0; r < K; ++r) {
    float v = L.v[0];
    int c = L.c[0];
    warp_best(v, c);
    if (c != INT_MAX && L.c[0] == c) L.pop_front();
    if (lane == r) { out_v = v; out_c = c; }
  }
}

// Decode layout.  Lanes are grouped L per landmark row; lane l of a group owns the row's
// 16-byte vectors l, l+L, l+2L, ... so one warp instruction reads 32/L whole rows contiguously.
template <typename T, int D_, int GM>
struct SplitShape {
  static constexpr int DPL = GM <= 4 ? 16 : (GM == 8 ? 8 : 4);   // dims per lane
  static constexpr int L = D_ / DPL;                              // lanes per row
  static constexpr int VEC = (16 / (int)sizeof(T)) < DPL ? (16 / (int)sizeof(T)) : DPL;
  static constexpr int NV = DPL / VEC;                            // vector loads per row
  static constexpr int RPW = 32 / L;                              // rows per warp step
  static_assert(L >= 1 && L <= 32 && (32 % L) == 0, "lane grouping");
};

template <typename T, int VEC>
__device__ __forceinline__ void load_vec(const T* p, float (&v)[VEC]);

template <>
__device__ __forceinline__ void load_vec<__nv_bfloat16, 8>(const __nv_bfloat16* p, float (&v)[8]) {
  uint4 t = __ldg(reinterpret_cast<const uint4*>(p));
  v[0] = bf16_lo(t.x); v[1] = bf16_hi(t.x); v[2] = bf16_lo(t.y); v[3] = bf16_hi(t.y);
  v[4] = bf16_lo(t.z); v[5] = bf16_hi(t.z); v[6] = bf16_lo(t.w); v[7] = bf16_hi(t.w);
}
template <>
__device__ __forceinline__ void load_vec<__nv_bfloat16, 4>(const __nv_bfloat16* p, float (&v)[4]) {
  Elem<__nv_bfloat16>::load4(p, v);
}
template <>
__device__ __forceinline__ void load_vec<float, 4>(const float* p, float (&v)[4]) {
  Elem<float>::load4(p, v);
}

// Same vectors from shared memory (no read-only cache path).
template <typename T, int VEC>
__device__ __forceinline__ void load_vec_shared(const T* p, float (&v)[VEC]);

template <>
__device__ __forceinline__ void load_vec_shared<__nv_bfloat16, 8>(const __nv_bfloat16* p,
                                                                  float (&v)[8]) {
  const uint4 t = *reinterpret_cast<const uint4*>(p);
  v[0] = bf16_lo(t.x); v[1] = bf16_hi(t.x); v[2] = bf16_lo(t.y); v[3] = bf16_hi(t.y);
  v[4] = bf16_lo(t.z); v[5] = bf16_hi(t.z); v[6] = bf16_lo(t.w); v[7] = bf16_hi(t.w);
}
template <>
__device__ __forceinline__ void load_vec_shared<__nv_bfloat16, 4>(const __nv_bfloat16* p,
                                                                  float (&v)[4]) {
  const uint2 t = *reinterpret_cast<const uint2*>(p);
  v[0] = bf16_lo(t.x); v[1] = bf16_hi(t.x); v[2] = bf16_lo(t.y); v[3] = bf16_hi(t.y);
}
template <>
__device__ __forceinline__ void load_vec_shared<float, 4>(const float* p, float (&v)[4]) {
  const float4 t = *reinterpret_cast<const float4*>(p);
  v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
}

__device__ __forceinline__ void record_status(int32_t* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

}  // namespace hils
