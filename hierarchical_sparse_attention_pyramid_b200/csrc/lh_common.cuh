// Shared device helpers and internal launch declarations of liblh.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "lh.h"

namespace lh {

// ---------------------------------------------------------------------------
// derived shape of one call, computed on the host from lh_config + lh_plan
// ---------------------------------------------------------------------------
struct Dims {
  int64_t BH, N, S;
  int d, L, p, log2p, chunk;
  int dtype;   // LH_BF16 / LH_FP32
  int scorer;  // lh_scorer
  int selection;  // lh_selection
  int64_t level_len[LH_MAX_LEVELS];
  int64_t level_off[LH_MAX_LEVELS];  // into slot_of rows
  int64_t upper_off[LH_MAX_LEVELS];  // into pyramid rows (levels >= 1)
  int64_t upper_entries, pyr_entries;
  int32_t kprime[LH_MAX_LEVELS];
  int64_t sel_off[LH_MAX_LEVELS];
  int64_t sel_per_head;
};

// error word bits (first int32 of ws)
// ERRW_RANGE: a value the backward keeps in fp16 (dOs, Vs) is outside fp16's
// finite range (|x| > 65504)
enum : int { ERRW_TIMEOUT = 1, ERRW_BOUNDS = 2, ERRW_RANGE = 4 };

__device__ __forceinline__ void report_error(int* errw, int bits) {
  if (errw) atomicOr(errw, bits);
}

// ---------------------------------------------------------------------------
// element conversion
// ---------------------------------------------------------------------------
template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f(float x) { return x; }
  static __device__ __forceinline__ float from_f(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

// raw vector of B bytes (4, 8 or 16)
template <int B> struct RawVec;
template <> struct RawVec<4> { using type = uint32_t; };
template <> struct RawVec<8> { using type = uint2; };
template <> struct RawVec<16> { using type = uint4; };

// load VE elements (VE * sizeof(T) bytes, naturally aligned) as floats
template <typename T, int VE>
__device__ __forceinline__ void load_vec(const T* src, float (&x)[VE]) {
  using V = typename RawVec<sizeof(T) * VE>::type;
  V u = __ldg(reinterpret_cast<const V*>(src));
  const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
  for (int i = 0; i < VE; ++i) x[i] = Elem<T>::to_f(e[i]);
}

// same, through L1/L2 with the default cache policy (data written earlier in the stream)
template <typename T, int VE>
__device__ __forceinline__ void load_vec_rw(const T* src, float (&x)[VE]) {
  using V = typename RawVec<sizeof(T) * VE>::type;
  V u = *reinterpret_cast<const V*>(src);
  const T* e = reinterpret_cast<const T*>(&u);
#pragma unroll
  for (int i = 0; i < VE; ++i) x[i] = Elem<T>::to_f(e[i]);
}

// store of VE elements with the streaming cache policy (st.global.cs)
template <typename T, int VE>
__device__ __forceinline__ void store_vec_stream(T* dst, const float (&x)[VE]) {
  using V = typename RawVec<sizeof(T) * VE>::type;
  V u;
  T* e = reinterpret_cast<T*>(&u);
#pragma unroll
  for (int i = 0; i < VE; ++i) e[i] = Elem<T>::from_f(x[i]);
  __stcs(reinterpret_cast<V*>(dst), u);
}

template <typename T, int VE>
__device__ __forceinline__ void store_vec(T* dst, const float (&x)[VE]) {
  using V = typename RawVec<sizeof(T) * VE>::type;
  V u;
  T* e = reinterpret_cast<T*>(&u);
#pragma unroll
  for (int i = 0; i < VE; ++i) e[i] = Elem<T>::from_f(x[i]);
  *reinterpret_cast<V*>(dst) = u;
}

// fp32 vector of VE floats (VE in {2, 4, 8}) from 16-byte-aligned-or-smaller chunks
template <int VE>
__device__ __forceinline__ void load_f32(const float* src, float (&x)[VE]) {
  if constexpr (VE == 8) {
    float4 a = *reinterpret_cast<const float4*>(src);
    float4 b = *reinterpret_cast<const float4*>(src + 4);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  } else if constexpr (VE == 4) {
    float4 a = *reinterpret_cast<const float4*>(src);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  } else {
    static_assert(VE == 2, "2, 4 or 8 floats");
    float2 a = *reinterpret_cast<const float2*>(src);
    x[0] = a.x; x[1] = a.y;
  }
}

// ---------------------------------------------------------------------------
// launchers (host side, one per stage); all return cudaGetLastError()
// ---------------------------------------------------------------------------
// levels below first_level are not written (their sums still carry upward)
// errw may be null (no error word): a bounded wait that runs out is then not reported
cudaError_t launch_pool(const Dims& D, const void* q, const void* k, const void* v, void* pq, void* pk, void* pv,
                        float* norms, int* errw, cudaStream_t st, int first_level = 1);
cudaError_t launch_score_topk(const Dims& D, const float* norms, float* spyr, int32_t* sel, int* errw,
                              cudaStream_t st);
// kept entries of levels 1 .. first_level-1 are averaged from level 0 here
// instead of being read from the pyramid
// shard (optional): the plan of a layer of the shard's tokens [t0, t0 + shard->N);
// only the entries whose key lies there are gathered, from the shard's rows,
// into per-head segments of seg_rows rows starting at slot seg_off[bh]
cudaError_t launch_gather(const Dims& D, const void* q, const void* k, const void* v, const void* pq,
                          const void* pk, const void* pv, const int32_t* sel, void* qs, void* ks, void* vs,
                          int32_t* seq_map, int32_t* slot_of, int* errw, cudaStream_t st, int first_level = 1,
                          const Dims* shard = nullptr, int64_t t0 = 0, const int64_t* seg_off = nullptr,
                          int64_t seg_rows = 0);

// first pyramid level lh_forward materialises: finer kept entries are cheaper
// to average from level 0 in the gather than to write whole levels
int materialized_level(const Dims& D);
// halo (optional, context parallelism; [BH][L-1][d] fp32): the previous
// shard's last entries' Os rows (scatter-back), the next shard's sums of dY
// over its first p^l - 1 rows (adjoint)
cudaError_t launch_scatter_back(const Dims& D, const float* os, const int32_t* slot_of, void* y, cudaStream_t st,
                                const float* halo = nullptr);
cudaError_t launch_scatter_adjoint(const Dims& D, const void* dy, const int32_t* seq_map, const float* os,
                                   void* dos, float* delta, int* errw, cudaStream_t st, const float* halo = nullptr);
// sums[bh][l-1] = sum of dY rows [0, p^l - 1) of head bh, l = 1 .. L-1 (fp32)
cudaError_t launch_head_sums(const Dims& D, const void* dy, float* sums, cudaStream_t st);
cudaError_t launch_pool_adjoint(const Dims& D, const float* dqs, const float* dks, const float* dvs,
                                const int32_t* slot_of, void* dq, void* dk, void* dv, cudaStream_t st);
// wait_cycles bounds every barrier wait of the kernel (SM clocks);
// issue_loads = 0 only for the timeout self-test (the producer loads nothing)
// query tiles [qt0, qt1) of 128 rows (qt1 < 0: to the last tile); O and LSE
// rows outside the window are not written
cudaError_t launch_attn_fwd(int64_t BH, int64_t S, int d, const void* qs, const void* ks, const void* vs, float* os,
                            float* lse, int* errw, cudaStream_t st, long long wait_cycles = 4000000000ll,
                            int issue_loads = 1, int64_t qt0 = 0, int64_t qt1 = -1);
// dQ of the query tiles [qt0, qt1), dK and dV of the key tiles [kt0, kt1)
// (a negative end: to the last tile)
cudaError_t launch_attn_bwd(int64_t BH, int64_t S, int d, const void* qs, const void* ks, const void* vs,
                            const float* lse, const void* dos, const float* delta, float* dqs, float* dks,
                            float* dvs, int* errw, cudaStream_t st, int64_t qt0 = 0, int64_t qt1 = -1,
                            int64_t kt0 = 0, int64_t kt1 = -1);

// message of the last failure on this thread (set by the API layer)
void set_error_message(const char* fmt, ...);

// validate cfg and fill the plan and the kernel-side shape (lh_plan's checks)
lh_status make_dims(const lh_config* cfg, lh_plan_info* info, Dims* D);

}  // namespace lh
