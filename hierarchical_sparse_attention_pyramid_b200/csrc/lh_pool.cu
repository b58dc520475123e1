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
#include <algorithm>
#include <type_traits>

#include "lh_common.cuh"
#include "sm100.cuh"

namespace lh {
namespace {
using namespace sm100;

constexpr int kWarps = 8;  // warps per block (pool adjoint)
constexpr unsigned kFull = 0xffffffffu;
// pooling: one CTA per SM of kPoolWarps warps, each with a ring of kStages
// shared-memory stages of kStageBytes (192 KB per CTA).  Measured on the
// 512K-token layer (16 heads, d = 128, bf16): the pass is bound by the warps'
// own summing work below 16 warps per SM (4 warps: 3.29 ms, 8: 1.83, 12: 1.46,
// 16: 1.133) and by DRAM above (24 warps with 2 stages: 1.122 ms)
constexpr int kPoolWarps = 24;
constexpr int kStages = 2;
constexpr int kStageBytes = 4096;

struct PoolArgs {
  const void* x[3];
  void* pyr[3];
  float* norms;  // [2][BH][N]
  int* errw;     // error word, or null
  int64_t BH, N, upper_entries;
  int64_t upper_off[LH_MAX_LEVELS];
  int64_t tasks_per_head, tasks;  // tasks = 3 * BH * tasks_per_head
  int task_rows, log2p, first_level;
};

// Butterfly reduce-scatter of U (8 or 16) per-lane partial sums, one per row
// of a batch, over the 32 lanes.  Halving stages (xor 16, 8, ...) leave each
// lane with one row's partial; the remaining xor stages complete the sum.
// Afterwards the lanes with (lane % (32 / U)) == 0 hold the full sum of row
// scatter_row<U>(lane).
template <int U>
__device__ __forceinline__ int scatter_row(int lane) {
  int r = 0;
#pragma unroll
  for (int b = 4, w = U / 2; w >= 1; --b, w >>= 1) r += ((lane >> b) & 1) * w;
  return r;
}

template <int U>
__device__ __forceinline__ float reduce_scatter(float (&v)[U], int lane) {
#pragma unroll
  for (int half = U / 2, b = 16; half >= 1; half >>= 1, b >>= 1) {
    const bool up = lane & b;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = up ? v[i] : v[i + half];
      const float keep = up ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(kFull, send, b);
    }
  }
  float t = v[0];
#pragma unroll
  for (int b = 16 / U; b >= 1; b >>= 1) t += __shfl_xor_sync(kFull, t, b);
  return t;
}

// One warp walks whole tasks: task_rows consecutive rows of one head of one
// of Q, K, V (a whole number of top-level blocks, so every level's sums start
// and end inside a task).  The grid is one CTA per SM; warp w takes tasks w,
// w + W, w + 2W, ... (W = warps in the grid).  The rows reach shared memory
// through a per-warp ring of kStages bulk copies of kStageBytes, issued by
// lane 0 kStages stages ahead of the rows being summed, so about
// kPoolWarps * kStages * kStageBytes bytes per SM are in flight at all times.
// Lane l holds channels [l*VE, l*VE+VE) of every row, so the pooled sums need
// no cross-lane work; only the norms of Q and K rows are reduced across lanes.
template <typename T, int D, int NL>
__global__ void __launch_bounds__(kPoolWarps * 32, 1) pool_kernel(PoolArgs a) {
  constexpr int VE = D / 32;
  constexpr int ROWB = D * (int)sizeof(T);
  constexpr int SR = kStageBytes / ROWB;  // rows per stage
  constexpr int U = 8;                    // rows summed per batch
  static_assert(SR % U == 0, "stage rows");
  using Raw = typename RawVec<sizeof(T) * VE>::type;
  extern __shared__ __align__(128) uint8_t pool_ring[];
  __shared__ __align__(8) uint64_t pool_bars[kPoolWarps][kStages];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint8_t* ring = pool_ring + warp * (kStages * kStageBytes);
  uint64_t* bar = pool_bars[warp];
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) mbar_init(&bar[s], 1);
    fence_mbar_init();
  }
  __syncwarp();
  const int64_t nw = (int64_t)gridDim.x * kPoolWarps;
  const int64_t gw = (int64_t)blockIdx.x * kPoolWarps + warp;
  const int log2p = a.log2p;
  const int rid = scatter_row<U>(lane);
  // rows u of an aligned batch of U after which a level-1 block ends: every
  // p-th row when p <= U, else the last row (when the batch ends a block)
  constexpr int kLog2U = 3;
  static_assert(U == 1 << kLog2U, "batch");
  uint32_t bmask = 1u << (U - 1);
  if (log2p < kLog2U)
    for (int u = (1 << log2p) - 1; u < U; u += 1 << log2p) bmask |= 1u << u;

  // task t: tensor t % 3, head (t / 3) / tasks_per_head, rows from row0
  // (task counts fit 32 bits: the host checks)
  const uint32_t tph = (uint32_t)a.tasks_per_head, ntasks = (uint32_t)a.tasks;
  auto task_at = [&](uint32_t t, int& tensor, int64_t& bh, int64_t& row0) {
    tensor = (int)(t % 3u);
    const uint32_t rest = t / 3u;
    bh = rest / tph;
    row0 = (int64_t)(rest % tph) * a.task_rows;
    return (int)min((int64_t)a.task_rows, a.N - row0);
  };

  // producer cursor, kept by every lane (lane 0 alone issues the copies):
  // task pt, its first source byte and row count, row pr within it
  uint32_t pt = (uint32_t)gw;
  int pr = 0, prows = 0;
  const uint8_t* psrc = nullptr;
  auto producer_task = [&]() {
    if (pt >= ntasks) return;
    int tensor;
    int64_t bh, row0;
    prows = task_at(pt, tensor, bh, row0);
    psrc = static_cast<const uint8_t*>(a.x[tensor]) + (bh * a.N + row0) * ROWB;
  };
  producer_task();
  uint32_t pending = 0;  // slots with a copy issued and not yet consumed
  auto issue = [&](int slot) {
    if (pt >= ntasks) return;
    const int n = min(SR, prows - pr);
    if (lane == 0) {
      mbar_expect_tx(&bar[slot], (uint32_t)(n * ROWB));
      bulk_load(ring + slot * kStageBytes, psrc + (int64_t)pr * ROWB, (uint32_t)(n * ROWB), &bar[slot]);
    }
    pending |= 1u << slot;
    pr += SR;
    if (pr >= prows) {
      pr = 0;
      pt += (uint32_t)nw;
      producer_task();
    }
  };
#pragma unroll
  for (int s = 0; s < kStages; ++s) issue(s);

  // bf16 rows are widened and summed as fp32 pairs (f32x2 arithmetic): one
  // packed fma for the squares and one packed add per two channels
  constexpr bool kPacked = std::is_same<T, __nv_bfloat16>::value && VE % 2 == 0;
  constexpr int NP = kPacked ? VE / 2 : 1;
  float acc[NL + 1][kPacked ? 1 : VE];
  uint64_t acc2[NL + 1][NP];

  uint32_t phase = 0;
  int slot = 0;
  for (uint32_t t = (uint32_t)gw; t < ntasks; t += (uint32_t)nw) {
    int tensor;
    int64_t bh, row0;
    const int rows = task_at(t, tensor, bh, row0);
    T* dst = static_cast<T*>(a.pyr[tensor]) + bh * a.upper_entries * D + lane * VE;
    const bool want_norm = tensor < 2;
    float* norm_out = a.norms + ((int64_t)tensor * a.BH + bh) * a.N + row0;
#pragma unroll
    for (int l = 0; l <= NL; ++l) {
#pragma unroll
      for (int i = 0; i < (kPacked ? 1 : VE); ++i) acc[l][i] = 0.f;
#pragma unroll
      for (int i = 0; i < NP; ++i) acc2[l][i] = 0ull;
    }

    auto process = [&](const Raw (&x)[U], int r0) {
      // bit u: a level-1 block of this task ends after row r0 + u (blocks are
      // aligned to the task; rows past the task's end never end one)
      uint32_t bnd = 0;
      if constexpr (NL > 1) {
        bnd = (log2p <= kLog2U || ((r0 + U) & ((1 << log2p) - 1)) == 0) ? bmask : 0u;
        if (rows - r0 < U) bnd &= (1u << (rows - r0)) - 1u;
      }
      float sq[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if constexpr (kPacked) {
          const uint32_t* wd = reinterpret_cast<const uint32_t*>(&x[u]);  // channels 2i, 2i+1 in word i
          uint64_t q2 = 0ull;
#pragma unroll
          for (int i = 0; i < NP; ++i) {
            const uint64_t v2 = f2_pack(__uint_as_float(wd[i] << 16), __uint_as_float(wd[i] & 0xffff0000u));
            q2 = f2_fma(v2, v2, q2);
            if constexpr (NL > 1) acc2[1][i] = f2_add(acc2[1][i], v2);
          }
          float qa, qb;
          f2_unpack(q2, qa, qb);
          sq[u] = qa + qb;
        } else {
          const T* e = reinterpret_cast<const T*>(&x[u]);
          float v[VE];
#pragma unroll
          for (int i = 0; i < VE; ++i) v[i] = Elem<T>::to_f(e[i]);
          float q = 0.f;
#pragma unroll
          for (int i = 0; i < VE; ++i) q = fmaf(v[i], v[i], q);
          sq[u] = q;
          if constexpr (NL > 1) {
#pragma unroll
            for (int i = 0; i < VE; ++i) acc[1][i] += v[i];
          }
        }
        if constexpr (NL > 1) {
          const int done = r0 + u + 1;  // rows of this task consumed
          if (bnd >> u & 1u) {
#pragma unroll
            for (int l = 1; l < NL; ++l) {
              if ((done & ((1 << (l * log2p)) - 1)) != 0) break;
              const float inv = __int_as_float((127 - l * log2p) << 23);  // 2^(-l log2p), exact
              const int64_t e_idx = ((row0 + done) >> (l * log2p)) - 1;
              if constexpr (kPacked) {
                const uint64_t inv2 = f2_pack(inv, inv);
                if (l >= a.first_level) {
                  Raw o;
                  uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                  for (int i = 0; i < NP; ++i) {
                    float ma, mb;
                    f2_unpack(f2_mul(acc2[l][i], inv2), ma, mb);
                    ow[i] = pack_bf16x2(ma, mb);
                  }
                  *reinterpret_cast<Raw*>(dst + (a.upper_off[l] + e_idx) * D) = o;
                }
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                  acc2[l + 1][i] = f2_add(acc2[l + 1][i], acc2[l][i]);
                  acc2[l][i] = 0ull;
                }
              } else {
                float m[VE];
#pragma unroll
                for (int i = 0; i < VE; ++i) m[i] = acc[l][i] * inv;
                if (l >= a.first_level) store_vec<T, VE>(dst + (a.upper_off[l] + e_idx) * D, m);
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
      if (want_norm) {
        const float tot = reduce_scatter<U>(sq, lane);
        const int r = r0 + rid;
        if ((lane & (32 / U - 1)) == 0 && r < rows) norm_out[r] = sqrtf(tot);
      }
    };

    for (int r0 = 0; r0 < rows; r0 += SR) {
      if (!mbar_wait_bounded_warp(&bar[slot], (phase >> slot) & 1u)) {
        // a copy never landed: report it, give the other copies in flight a
        // bounded time to land (the CTA must not exit with copies pending
        // into its shared memory) and leave
        report_error(a.errw, ERRW_TIMEOUT);
#pragma unroll 1
        for (int s = 0; s < kStages; ++s)
          if (s != slot && (pending >> s & 1u)) mbar_wait_bounded_warp(&bar[s], (phase >> s) & 1u);
        return;
      }
      // rows of a stage past the task's end hold stale bytes: their sums are
      // never written (no block ends there, their norms are not stored) and
      // the task's sums are reset before the next task
      const Raw* stage = reinterpret_cast<const Raw*>(ring + slot * kStageBytes) + lane;
      const int stage_rows = min(SR, rows - r0);
#pragma unroll 1
      for (int b = 0; b < stage_rows; b += U) {
        Raw x[U];
#pragma unroll
        for (int u = 0; u < U; ++u) x[u] = stage[(b + u) * (ROWB / (int)sizeof(Raw))];
        process(x, r0 + b);
      }
      __syncwarp();  // every lane has read the stage before it is refilled
      pending &= ~(1u << slot);
      phase ^= 1u << slot;
      issue(slot);
      slot = slot + 1 == kStages ? 0 : slot + 1;
    }
  }
}

// The same pass for bf16 rows of 128 channels, with about a third of the
// instructions per row (the pass above issues on ~80% of its cycles there).
// Each half-warp takes every other row of the warp's task: lane l holds
// channels [8 (l mod 16), +8) of row 2u + (l div 16) at step u, so one
// 16-byte shared-memory load per lane moves two rows and each half-warp
// reduces its own row's norm over 16 lanes.  The half-warps keep partial
// sums of the levels (each holds the rows of its parity), which are linear,
// and add them together only when a materialised entry is written.  Rows are
// summed straight into the lowest materialised level (first_level): the
// levels below it are never formed.
// Warps per SM x ring stages of 4 KB, measured on the 512K-token layer (16
// heads): 16 x 2: 1.016 ms; 20 x 2: 1.038; 24 x 2: 1.115 (at 80 registers,
// with spills); 16 x 3: 1.087; 12 x 2: 1.101; 12 x 4: 1.103; 8 x 4: 1.354.
// The pass above takes 1.148 ms on the same layer.
constexpr int kPairWarps = 16;
constexpr int kPairStages = 2;
template <int NL>
__global__ void __launch_bounds__(kPairWarps * 32, 1) pool_pairs_kernel(PoolArgs a) {
  constexpr int D = 128;
  constexpr int ROWB = D * 2;
  constexpr int SR = kStageBytes / ROWB;  // 16 rows per stage
  constexpr int NPAIR = SR / 2;           // two rows per step
  static_assert(SR % 2 == 0 && NPAIR == 8, "stage rows");
  extern __shared__ __align__(128) uint8_t pool_ring[];
  __shared__ __align__(8) uint64_t pool_bars[kPairWarps][kPairStages];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int half = lane >> 4;
  uint8_t* ring = pool_ring + warp * (kPairStages * kStageBytes);
  uint64_t* bar = pool_bars[warp];
  if (lane == 0) {
#pragma unroll
    for (int st = 0; st < kPairStages; ++st) mbar_init(&bar[st], 1);
    fence_mbar_init();
  }
  __syncwarp();
  const int64_t nw = (int64_t)gridDim.x * kPairWarps;
  const int64_t gw = (int64_t)blockIdx.x * kPairWarps + warp;
  const int log2p = a.log2p, fl = a.first_level;
  // a block of the lowest materialised level ends after `done` rows of the
  // task when done & fl_mask == 0 (never when no level is materialised)
  const int fl_mask = fl < NL ? (1 << (fl * log2p)) - 1 : -1;
  // the norms are reduced every 4 steps: after the two halving stages of the
  // reduction, lane l's partial belongs to step rid of the 4, and lanes with
  // l mod 4 == 0 end with that row's whole sum
  const int rid = ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);

  const uint32_t tph = (uint32_t)a.tasks_per_head, ntasks = (uint32_t)a.tasks;
  auto task_at = [&](uint32_t t, int& tensor, int64_t& bh, int64_t& row0) {
    tensor = (int)(t % 3u);
    const uint32_t rest = t / 3u;
    bh = rest / tph;
    row0 = (int64_t)(rest % tph) * a.task_rows;
    return (int)min((int64_t)a.task_rows, a.N - row0);
  };
  uint32_t pt = (uint32_t)gw;
  int pr = 0, prows = 0;
  const uint8_t* psrc = nullptr;
  auto producer_task = [&]() {
    if (pt >= ntasks) return;
    int tensor;
    int64_t bh, row0;
    prows = task_at(pt, tensor, bh, row0);
    psrc = static_cast<const uint8_t*>(a.x[tensor]) + (bh * a.N + row0) * ROWB;
  };
  producer_task();
  uint32_t pending = 0;
  auto issue = [&](int sl) {
    if (pt >= ntasks) return;
    const int n = min(SR, prows - pr);
    if (lane == 0) {
      mbar_expect_tx(&bar[sl], (uint32_t)(n * ROWB));
      bulk_load(ring + sl * kStageBytes, psrc + (int64_t)pr * ROWB, (uint32_t)(n * ROWB), &bar[sl]);
    }
    pending |= 1u << sl;
    pr += SR;
    if (pr >= prows) {
      pr = 0;
      pt += (uint32_t)nw;
      producer_task();
    }
  };
#pragma unroll
  for (int st = 0; st < kPairStages; ++st) issue(st);

  uint32_t phase = 0;
  int slot = 0;
  for (uint32_t t = (uint32_t)gw; t < ntasks; t += (uint32_t)nw) {
    int tensor;
    int64_t bh, row0;
    const int rows = task_at(t, tensor, bh, row0);
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.pyr[tensor]) + bh * a.upper_entries * D + (lane & 15) * 8;
    float* norm_out = a.norms + ((int64_t)tensor * a.BH + bh) * a.N + row0;
    uint64_t run[4], acc[NL][4];  // this half's sums: the open block of level fl, and of the levels above it
#pragma unroll
    for (int i = 0; i < 4; ++i) run[i] = 0ull;
#pragma unroll
    for (int l = 0; l < NL; ++l)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[l][i] = 0ull;

    // a block of level fl ended after `done` rows: write it and every level
    // above that ends there, carrying each sum one level up
    auto cascade = [&](int done) {
      uint64_t sm[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        sm[i] = run[i];
        run[i] = 0ull;
      }
#pragma unroll
      for (int l = 1; l < NL; ++l) {
        if (l < fl) continue;
        // both halves' parts of the entry, scaled by p^-l (exact) and rounded once
        const float inv = __int_as_float((127 - l * log2p) << 23);
        const uint64_t inv2 = f2_pack(inv, inv);
        uint4 o;
        uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float x0, x1;
          f2_unpack(sm[i], x0, x1);
          const uint64_t other = f2_pack(__shfl_xor_sync(kFull, x0, 16), __shfl_xor_sync(kFull, x1, 16));
          float m0, m1;
          f2_unpack(f2_mul(f2_add(sm[i], other), inv2), m0, m1);
          ow[i] = pack_bf16x2(m0, m1);
        }
        const int64_t e_idx = ((row0 + done) >> (l * log2p)) - 1;
        if (half == 0) *reinterpret_cast<uint4*>(dst + (a.upper_off[l] + e_idx) * D) = o;
        if (l + 1 == NL) break;
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[l + 1][i] = f2_add(acc[l + 1][i], sm[i]);
        if ((done & ((1 << ((l + 1) * log2p)) - 1)) != 0) break;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          sm[i] = acc[l + 1][i];
          acc[l + 1][i] = 0ull;
        }
      }
    };

    // one stage: NPAIR steps of two rows; the norms of Q and K rows
    auto stage_pass = [&](const uint4* st4, int r0, auto norm) {
      constexpr bool kNorm = decltype(norm)::value;
      float sq[4];
#pragma unroll
      for (int u = 0; u < NPAIR; ++u) {
        const uint4 x = st4[u * 32];
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
        uint64_t q2 = 0ull;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint64_t v2 = f2_pack(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
          if constexpr (kNorm) q2 = f2_fma(v2, v2, q2);
          run[i] = f2_add(run[i], v2);
        }
        if constexpr (kNorm) {
          float qa, qb;
          f2_unpack(q2, qa, qb);
          sq[u & 3] = qa + qb;
          if ((u & 3) == 3) {
            // reduce-scatter of each half's 4 rows over its 16 lanes
#pragma unroll
            for (int hw = 2, b = 8; hw >= 1; hw >>= 1, b >>= 1) {
              const bool up = lane & b;
#pragma unroll
              for (int i = 0; i < hw; ++i) {
                const float send = up ? sq[i] : sq[i + hw];
                const float keep = up ? sq[i + hw] : sq[i];
                sq[i] = keep + __shfl_xor_sync(kFull, send, b);
              }
            }
            float tot = sq[0] + __shfl_xor_sync(kFull, sq[0], 2);
            tot += __shfl_xor_sync(kFull, tot, 1);
            const int r = r0 + 2 * ((u & ~3) + rid) + half;
            if ((lane & 3) == 0 && r < rows) norm_out[r] = sqrtf(tot);
          }
        }
        const int done = r0 + 2 * u + 2;
        if ((done & fl_mask) == 0 && done <= rows) cascade(done);
      }
    };

    const bool want_norm = tensor < 2;
    for (int r0 = 0; r0 < rows; r0 += SR) {
      if (!mbar_wait_bounded_warp(&bar[slot], (phase >> slot) & 1u)) {
        report_error(a.errw, ERRW_TIMEOUT);
#pragma unroll 1
        for (int st = 0; st < kPairStages; ++st)
          if (st != slot && (pending >> st & 1u)) mbar_wait_bounded_warp(&bar[st], (phase >> st) & 1u);
        return;
      }
      // rows of a stage past the task's end hold stale bytes: they only reach
      // sums that are never written (no block ends past the task) and are
      // reset with the next task, and their norms are not stored
      const uint4* st4 = reinterpret_cast<const uint4*>(ring + slot * kStageBytes) + lane;
      if (want_norm) stage_pass(st4, r0, std::true_type{});
      else stage_pass(st4, r0, std::false_type{});
      __syncwarp();  // every lane has read the stage before it is refilled
      pending &= ~(1u << slot);
      phase ^= 1u << slot;
      issue(slot);
      slot = slot + 1 == kPairStages ? 0 : slot + 1;
    }
  }
}

// ---------------------------------------------------------------------------
// adjoint: dX_t = sum_l [kept(l, t >> l log2p)] p^-l dXs[slot]  (fp32, rounded once)
// 16-byte output lanes, R (1 or 2) rows per warp instruction; the rows of an
// instruction share every entry of level >= 1 (t is even when R = 2 and p >= 2),
// whose scaled contributions are cached and refreshed at level-1 boundaries.
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

template <typename T, int D>
struct RowLayout {
  static constexpr int VE = 16 / sizeof(T) <= D / 16 ? 16 / sizeof(T) : D / 16;  // elements per lane
  static constexpr int LPR = D / VE;                                            // lanes per row
  static constexpr int R = 32 / LPR;                                            // rows per instruction
  static_assert(R == 1 || R == 2, "layout");
};

template <typename T, int D, int NL>
__global__ void __launch_bounds__(kWarps * 32) pool_adjoint_kernel(PoolAdjArgs a) {
  using Lay = RowLayout<T, D>;
  constexpr int VE = Lay::VE, LPR = Lay::LPR, R = Lay::R;
  const int lane = threadIdx.x & 31;
  const int lr = lane / LPR, cv = lane % LPR;
  const int64_t wid = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int tensor = (int)(wid % 3);
  const int64_t rest = wid / 3;
  const int64_t bh = rest / a.tasks_per_head;
  if (bh >= a.BH) return;
  const int64_t row0 = (rest % a.tasks_per_head) * a.task_rows;
  const int rows = (int)min((int64_t)a.task_rows, a.N - row0);
  const int log2p = a.log2p;
  const int32_t* so = a.slot_of + bh * a.pyr_entries;
  const float* xs = a.dxs[tensor] + bh * a.S * D + cv * VE;
  T* out = static_cast<T*>(a.dx[tensor]) + (bh * a.N + row0) * D + cv * VE;

  // contribution of level 1, refreshed at level-1 boundaries, and the summed
  // contribution of levels >= 2, refreshed at level-2 boundaries
  float up1[VE], high[VE];
#pragma unroll
  for (int i = 0; i < VE; ++i) up1[i] = high[i] = 0.f;
  auto contribution = [&](int l, int64_t i, float (&acc)[VE]) {
    const int s = so[a.level_off[l] + i];
    if (s >= 0) {
      float v[VE];
      load_f32<VE>(xs + (int64_t)s * D, v);
      const float inv = __int_as_float((127 - l * log2p) << 23);  // 2^(-l log2p), exact
#pragma unroll
      for (int c = 0; c < VE; ++c) acc[c] = fmaf(v[c], inv, acc[c]);
    }
  };
  int s0w = -1;
  for (int r = 0; r < rows; r += R) {
    const int64_t t = row0 + r;  // first row of this instruction
    if ((r & 31) == 0) s0w = (r + lane < rows) ? so[a.level_off[0] + t + lane] : -1;
    if constexpr (NL > 1) {
      if ((t & ((1 << log2p) - 1)) == 0) {
#pragma unroll
        for (int c = 0; c < VE; ++c) up1[c] = 0.f;
        contribution(1, t >> log2p, up1);
        if constexpr (NL > 2) {
          if ((t & ((1 << (2 * log2p)) - 1)) == 0) {
#pragma unroll
            for (int c = 0; c < VE; ++c) high[c] = 0.f;
#pragma unroll
            for (int l = NL - 1; l >= 2; --l) contribution(l, t >> (l * log2p), high);
          }
        }
      }
    }
    const int s0 = __shfl_sync(kFull, s0w, (r & 31) + lr);
    float y[VE];
#pragma unroll
    for (int c = 0; c < VE; ++c) y[c] = up1[c] + high[c];
    if (s0 >= 0) {
      float v[VE];
      load_f32<VE>(xs + (int64_t)s0 * D, v);
#pragma unroll
      for (int c = 0; c < VE; ++c) y[c] += v[c];
    }
    // streaming stores: measured 1.157 -> 1.138 ms inside the 512K step (they
    // do not displace the lines the kernels after this one read)
    if (r + lr < rows) store_vec_stream<T, VE>(out + (int64_t)(r + lr) * D, y);
  }
}

// persistent grid: as many CTAs as fit on the GPU at once, fewer for small inputs
template <typename T, int D, int NL>
cudaError_t pool_launch(const PoolArgs& a, cudaStream_t st) {
  constexpr int smem = kPoolWarps * kStages * kStageBytes;
  cudaError_t e = cudaFuncSetAttribute(pool_kernel<T, D, NL>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  int dev = 0, sms = 0, per_sm = 0;
  if (e == cudaSuccess) e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, pool_kernel<T, D, NL>, kPoolWarps * 32, smem);
  if (e != cudaSuccess) return e;
  const int64_t blocks = std::min<int64_t>((int64_t)sms * std::max(per_sm, 1), (a.tasks + kPoolWarps - 1) / kPoolWarps);
  pool_kernel<T, D, NL><<<(unsigned)blocks, kPoolWarps * 32, smem, st>>>(a);
  return cudaGetLastError();
}

template <int NL>
cudaError_t pool_pairs_launch(const PoolArgs& a, cudaStream_t st) {
  constexpr int smem = kPairWarps * kPairStages * kStageBytes;
  cudaError_t e = cudaFuncSetAttribute(pool_pairs_kernel<NL>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  int dev = 0, sms = 0, per_sm = 0;
  if (e == cudaSuccess) e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess)
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, pool_pairs_kernel<NL>, kPairWarps * 32, smem);
  if (e != cudaSuccess) return e;
  const int64_t blocks = std::min<int64_t>((int64_t)sms * std::max(per_sm, 1), (a.tasks + kPairWarps - 1) / kPairWarps);
  pool_pairs_kernel<NL><<<(unsigned)blocks, kPairWarps * 32, smem, st>>>(a);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t pool_dispatch_L(int L, const PoolArgs& a, cudaStream_t st) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value && D == 128) {
    // the common layout: two rows per warp step (levels 1 to 4 in registers)
    switch (L) {
      case 2: return pool_pairs_launch<2>(a, st);
      case 3: return pool_pairs_launch<3>(a, st);
      case 4: return pool_pairs_launch<4>(a, st);
      case 5: return pool_pairs_launch<5>(a, st);
      default: break;
    }
  }
  switch (L) {
#define LH_CASE(n) \
  case n: return pool_launch<T, D, n>(a, st);
    LH_CASE(1) LH_CASE(2) LH_CASE(3) LH_CASE(4) LH_CASE(5) LH_CASE(6) LH_CASE(7) LH_CASE(8)
#undef LH_CASE
    default: return cudaErrorInvalidValue;
  }
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

// rows per warp task: a whole number of top-level blocks, and at least
// min_rows so that the first loads' latency is paid once per long run
int task_rows_for(const Dims& D, int min_rows) {
  const int64_t ptop = (int64_t)1 << ((D.L - 1) * D.log2p);
  return (int)(ptop > min_rows ? ptop : min_rows);
}

}  // namespace

cudaError_t launch_pool(const Dims& D, const void* q, const void* k, const void* v, void* pq, void* pk, void* pv,
                        float* norms, int* errw, cudaStream_t st, int first_level) {
  PoolArgs a{};
  a.x[0] = q; a.x[1] = k; a.x[2] = v;
  a.pyr[0] = pq; a.pyr[1] = pk; a.pyr[2] = pv;
  a.norms = norms;
  a.errw = errw;
  a.BH = D.BH; a.N = D.N; a.upper_entries = D.upper_entries;
  for (int l = 0; l < LH_MAX_LEVELS; ++l) a.upper_off[l] = D.upper_off[l];
  a.task_rows = task_rows_for(D, 64);
  a.tasks_per_head = (D.N + a.task_rows - 1) / a.task_rows;
  a.tasks = 3 * D.BH * a.tasks_per_head;
  if (a.tasks >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;  // task ids are 32-bit in the kernel
  a.log2p = D.log2p;
  a.first_level = first_level;
  if (D.dtype == LH_BF16) {
    return D.d == 128 ? pool_dispatch_L<__nv_bfloat16, 128>(D.L, a, st)
                      : pool_dispatch_L<__nv_bfloat16, 64>(D.L, a, st);
  }
  return D.d == 128 ? pool_dispatch_L<float, 128>(D.L, a, st) : pool_dispatch_L<float, 64>(D.L, a, st);
}

cudaError_t launch_pool_adjoint(const Dims& D, const float* dqs, const float* dks, const float* dvs,
                                const int32_t* slot_of, void* dq, void* dk, void* dv, cudaStream_t st) {
  PoolAdjArgs a{};
  a.dxs[0] = dqs; a.dxs[1] = dks; a.dxs[2] = dvs;
  a.dx[0] = dq; a.dx[1] = dk; a.dx[2] = dv;
  a.slot_of = slot_of;
  a.BH = D.BH; a.N = D.N; a.S = D.S; a.pyr_entries = D.pyr_entries;
  for (int l = 0; l < LH_MAX_LEVELS; ++l) a.level_off[l] = D.level_off[l];
  a.task_rows = task_rows_for(D, 64);
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
