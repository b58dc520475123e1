// Stage 1 (pyramid pooling + level-0 norms) and its adjoint fused with the
// gather adjoint (stages 3 and 1 backward).
//
// Lighthouse Attention pools Q, K and V with one factor p over L levels
// (techllm post "Lighthouse Attention: long-context pretraining", How it
// works (1); aitrends.kr summary, Technical details (1)); level-0 scores are
// the l2 norms of Q_t and K_t (aitrends.kr summary, Technical details (2)).
//
// Both kernels are HBM streams: one warp walks a contiguous run of rows of
// one head and one of Q, K, V, so every load or store instruction of the warp
// touches whole rows.
#include "lh_common.cuh"

namespace lh {
namespace {

constexpr int kWarps = 8;   // warps per block
constexpr int kUnroll = 8;  // row groups loaded ahead per warp
constexpr unsigned kFull = 0xffffffffu;

// 16-byte lanes for bf16 d=128 (8 elements), 8- or 16-byte lanes otherwise;
// R rows per warp instruction, and R <= 2 <= p always.
template <typename T, int D>
struct PoolLayout {
  static constexpr int VE = (sizeof(T) == 2 && D == 128) ? 8 : 4;
  static constexpr int LPR = D / VE;  // lanes per row
  static constexpr int R = 32 / LPR;  // rows per warp instruction
  static_assert(R == 1 || R == 2, "layout");
};

struct PoolArgs {
  const void* x[3];
  void* pyr[3];
  float* norms;  // [2][BH][N]
  int64_t BH, N, upper_entries;
  int64_t upper_off[LH_MAX_LEVELS];
  int64_t tasks_per_head;
  int task_rows, log2p;
};

template <typename T, int D, int NL>
__global__ void __launch_bounds__(kWarps * 32) pool_kernel(PoolArgs a) {
  using Lay = PoolLayout<T, D>;
  constexpr int VE = Lay::VE, LPR = Lay::LPR, R = Lay::R;
  constexpr int GPW = 32 / R;  // row groups per 32-row window of norms
  const int lane = threadIdx.x & 31;
  const int64_t wid = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int tensor = (int)(wid % 3);
  const int64_t rest = wid / 3;
  const int64_t bh = rest / a.tasks_per_head;
  if (bh >= a.BH) return;
  const int64_t row0 = (rest % a.tasks_per_head) * a.task_rows;
  const int rows = (int)min((int64_t)a.task_rows, a.N - row0);
  const int lr = lane / LPR, cv = lane % LPR;
  const int log2p = a.log2p;
  const T* src = static_cast<const T*>(a.x[tensor]) + (bh * a.N + row0) * D + cv * VE;
  T* dst = static_cast<T*>(a.pyr[tensor]);
  const int n_rg = (rows + R - 1) / R;
  const bool want_norm = tensor < 2;
  float* norm_out = a.norms + ((int64_t)tensor * a.BH + bh) * a.N + row0;

  float acc[NL + 1][VE];
#pragma unroll
  for (int l = 0; l <= NL; ++l)
#pragma unroll
    for (int i = 0; i < VE; ++i) acc[l][i] = 0.f;
  float mynorm = 0.f;

  auto write_level = [&](int l, int64_t e_rel, const float (&v)[VE]) {
    if (lr != 0) return;
    float m[VE];
    const float inv = ldexpf(1.f, -l * log2p);  // exact power of two
#pragma unroll
    for (int i = 0; i < VE; ++i) m[i] = v[i] * inv;
    const int64_t e = (row0 >> (l * log2p)) + e_rel;
    store_vec<T, VE>(dst + (bh * a.upper_entries + a.upper_off[l] + e) * D + cv * VE, m);
  };

  for (int g0 = 0; g0 < n_rg; g0 += kUnroll) {
    float x[kUnroll][VE];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int row = (g0 + u) * R + lr;
      if (g0 + u < n_rg && row < rows) {
        load_vec<T, VE>(src + (int64_t)row * D, x[u]);
      } else {
#pragma unroll
        for (int i = 0; i < VE; ++i) x[u][i] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int g = g0 + u;
      if (g >= n_rg) break;
      if (want_norm) {
        float sq = 0.f;
#pragma unroll
        for (int i = 0; i < VE; ++i) sq = fmaf(x[u][i], x[u][i], sq);
#pragma unroll
        for (int o = LPR / 2; o >= 1; o >>= 1) sq += __shfl_xor_sync(kFull, sq, o);
        const float t = __shfl_sync(kFull, sq, (lane % R) * LPR);
        if (lane / R == g % GPW) mynorm = sqrtf(t);
        if (g % GPW == GPW - 1 || g == n_rg - 1) {
          const int r = (g / GPW) * 32 + lane;
          if (r < rows) norm_out[r] = mynorm;
        }
      }
      if constexpr (NL > 1) {
#pragma unroll
        for (int i = 0; i < VE; ++i) acc[1][i] += x[u][i];
        const int done = (g + 1) * R;  // rows of this task consumed so far
        if ((done & ((1 << log2p) - 1)) == 0) {
          // a level-1 entry is complete: add the R row lanes together
          float s1[VE];
#pragma unroll
          for (int i = 0; i < VE; ++i) {
            float v = acc[1][i];
#pragma unroll
            for (int o = LPR; o < 32; o <<= 1) v += __shfl_xor_sync(kFull, v, o);
            s1[i] = v;
            acc[1][i] = 0.f;
            acc[2][i] += v;
          }
          write_level(1, (done >> log2p) - 1, s1);
#pragma unroll
          for (int l = 2; l < NL; ++l) {
            if ((done & ((1 << (l * log2p)) - 1)) != 0) break;
            write_level(l, (done >> (l * log2p)) - 1, acc[l]);
#pragma unroll
            for (int i = 0; i < VE; ++i) {
              acc[l + 1][i] += acc[l][i];
              acc[l][i] = 0.f;
            }
          }
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// adjoint: dX_t = sum_l [kept(l, t >> l log2p)] p^-l dXs[slot]  (fp32, rounded once)
// one row per warp instruction; contributions of levels >= 1 are cached and
// refreshed only when t crosses a level-1 boundary.
// ---------------------------------------------------------------------------
struct PoolAdjArgs {
  const float* dxs[3];
  void* dx[3];
  const int32_t* slot_of;
  int64_t BH, N, S, pyr_entries;
  int64_t level_off[LH_MAX_LEVELS];
  int64_t tasks_per_head;
  int task_rows, log2p;
};

template <typename T, int D, int NL>
__global__ void __launch_bounds__(kWarps * 32) pool_adjoint_kernel(PoolAdjArgs a) {
  constexpr int VE = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t wid = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int tensor = (int)(wid % 3);
  const int64_t rest = wid / 3;
  const int64_t bh = rest / a.tasks_per_head;
  if (bh >= a.BH) return;
  const int64_t row0 = (rest % a.tasks_per_head) * a.task_rows;
  const int rows = (int)min((int64_t)a.task_rows, a.N - row0);
  const int log2p = a.log2p;
  const int32_t* so = a.slot_of + bh * a.pyr_entries;
  const float* xs = a.dxs[tensor] + bh * a.S * D + lane * VE;
  T* out = static_cast<T*>(a.dx[tensor]) + (bh * a.N + row0) * D + lane * VE;

  float up[NL + 1][VE];
  float upper[VE];
#pragma unroll
  for (int i = 0; i < VE; ++i) upper[i] = 0.f;
  int s0w = -1;
  for (int r = 0; r < rows; ++r) {
    const int64_t t = row0 + r;
    if ((r & 31) == 0) s0w = (r + lane < rows) ? so[a.level_off[0] + t + lane] : -1;
    if constexpr (NL > 1) {
      if ((t & ((1 << log2p) - 1)) == 0) {
#pragma unroll
        for (int l = 1; l < NL; ++l) {
          if ((t & ((1ll << (l * log2p)) - 1)) == 0) {
            const int s = so[a.level_off[l] + (t >> (l * log2p))];
            if (s >= 0) {
              float v[VE];
              load_f32<VE>(xs + (int64_t)s * D, v);
              const float inv = ldexpf(1.f, -l * log2p);
#pragma unroll
              for (int i = 0; i < VE; ++i) up[l][i] = v[i] * inv;
            } else {
#pragma unroll
              for (int i = 0; i < VE; ++i) up[l][i] = 0.f;
            }
          }
        }
#pragma unroll
        for (int i = 0; i < VE; ++i) {
          float s = 0.f;
#pragma unroll
          for (int l = NL - 1; l >= 1; --l) s += up[l][i];
          upper[i] = s;
        }
      }
    }
    const int s0 = __shfl_sync(kFull, s0w, r & 31);
    float y[VE];
#pragma unroll
    for (int i = 0; i < VE; ++i) y[i] = upper[i];
    if (s0 >= 0) {
      float v[VE];
      load_f32<VE>(xs + (int64_t)s0 * D, v);
#pragma unroll
      for (int i = 0; i < VE; ++i) y[i] += v[i];
    }
    store_vec<T, VE>(out + (int64_t)r * D, y);
  }
}

template <typename T, int D>
cudaError_t pool_dispatch_L(int L, const PoolArgs& a, int64_t blocks, cudaStream_t st) {
  switch (L) {
#define LH_CASE(n) \
  case n: pool_kernel<T, D, n><<<(unsigned)blocks, kWarps * 32, 0, st>>>(a); break;
    LH_CASE(1) LH_CASE(2) LH_CASE(3) LH_CASE(4) LH_CASE(5) LH_CASE(6) LH_CASE(7) LH_CASE(8)
#undef LH_CASE
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t pool_adj_dispatch_L(int L, const PoolAdjArgs& a, int64_t blocks, cudaStream_t st) {
  switch (L) {
#define LH_CASE(n) \
  case n: pool_adjoint_kernel<T, D, n><<<(unsigned)blocks, kWarps * 32, 0, st>>>(a); break;
    LH_CASE(1) LH_CASE(2) LH_CASE(3) LH_CASE(4) LH_CASE(5) LH_CASE(6) LH_CASE(7) LH_CASE(8)
#undef LH_CASE
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

int task_rows_for(const Dims& D) {
  const int64_t ptop = (int64_t)1 << ((D.L - 1) * D.log2p);
  return (int)(ptop > 32 ? ptop : 32);
}

}  // namespace

cudaError_t launch_pool(const Dims& D, const void* q, const void* k, const void* v, void* pq, void* pk, void* pv,
                        float* norms, cudaStream_t st) {
  PoolArgs a{};
  a.x[0] = q; a.x[1] = k; a.x[2] = v;
  a.pyr[0] = pq; a.pyr[1] = pk; a.pyr[2] = pv;
  a.norms = norms;
  a.BH = D.BH; a.N = D.N; a.upper_entries = D.upper_entries;
  for (int l = 0; l < LH_MAX_LEVELS; ++l) a.upper_off[l] = D.upper_off[l];
  a.task_rows = task_rows_for(D);
  a.tasks_per_head = (D.N + a.task_rows - 1) / a.task_rows;
  a.log2p = D.log2p;
  const int64_t warps = 3 * D.BH * a.tasks_per_head;
  const int64_t blocks = (warps + kWarps - 1) / kWarps;
  if (D.dtype == LH_BF16) {
    return D.d == 128 ? pool_dispatch_L<__nv_bfloat16, 128>(D.L, a, blocks, st)
                      : pool_dispatch_L<__nv_bfloat16, 64>(D.L, a, blocks, st);
  }
  return D.d == 128 ? pool_dispatch_L<float, 128>(D.L, a, blocks, st) : pool_dispatch_L<float, 64>(D.L, a, blocks, st);
}

cudaError_t launch_pool_adjoint(const Dims& D, const float* dqs, const float* dks, const float* dvs,
                                const int32_t* slot_of, void* dq, void* dk, void* dv, cudaStream_t st) {
  PoolAdjArgs a{};
  a.dxs[0] = dqs; a.dxs[1] = dks; a.dxs[2] = dvs;
  a.dx[0] = dq; a.dx[1] = dk; a.dx[2] = dv;
  a.slot_of = slot_of;
  a.BH = D.BH; a.N = D.N; a.S = D.S; a.pyr_entries = D.pyr_entries;
  for (int l = 0; l < LH_MAX_LEVELS; ++l) a.level_off[l] = D.level_off[l];
  a.task_rows = task_rows_for(D);
  a.tasks_per_head = (D.N + a.task_rows - 1) / a.task_rows;
  a.log2p = D.log2p;
  const int64_t warps = 3 * D.BH * a.tasks_per_head;
  const int64_t blocks = (warps + kWarps - 1) / kWarps;
  if (D.dtype == LH_BF16) {
    return D.d == 128 ? pool_adj_dispatch_L<__nv_bfloat16, 128>(D.L, a, blocks, st)
                      : pool_adj_dispatch_L<__nv_bfloat16, 64>(D.L, a, blocks, st);
  }
  return D.d == 128 ? pool_adj_dispatch_L<float, 128>(D.L, a, blocks, st)
                    : pool_adj_dispatch_L<float, 64>(D.L, a, blocks, st);
}

}  // namespace lh
