// Stage 3 (gather into the causally ordered sequence), stage 5 (scatter-back)
// and the scatter-back adjoint.
//
// Kept triples are sorted into causal order and form one contiguous sequence
// of length S (techllm post "Lighthouse Attention: long-context pretraining",
// How it works (3)).  Each output returns to its shifted range R(l,i) over the
// original positions and every position sums what it receives (aitrends.kr
// summary, Technical details (4); techllm post, How it works (4)).
//
// Entry (l, i) covers tokens [i p^l, (i+1) p^l); its key is
// (e = (i+1) p^l - 1, -l) and its range is R(l,i) = [e, e + p^l).  The slot of
// an entry is the number of kept entries with a smaller key, counted level by
// level with searches over the sorted parent lists (or, when levels are
// selected directly, the sorted lists of kept entries), so no sort runs.
#include <algorithm>
#include <type_traits>

#include "lh_common.cuh"

namespace lh {
namespace {

constexpr int kWarps = 8;
// warps per block of the one-warp-per-item kernels, whose items differ in
// size: a block stays resident until its slowest warp is done, so smaller
// blocks keep more warps busy.  Measured on the 512K-token layer (blocks of
// 8 / 4 / 2 / 1 warps): gather 0.163 / 0.158 / 0.158 / 0.165 ms, scatter
// adjoint 0.417 / 0.406 / 0.406 / 0.384 ms.
constexpr int kGatherWarps = 4;
constexpr int kSadjWarps = 1;

constexpr unsigned kFull = 0xffffffffu;

struct GatherArgs {
  const void* x0[3];   // q, k, v (level 0)
  const void* pyr[3];  // pyramid levels >= 1
  const int32_t* sel;
  __nv_bfloat16* out[3];
  int32_t* seq_map;
  int32_t* slot_of;
  int* errw;
  int64_t BH, N, S, upper_entries, pyr_entries, sel_per_head;
  int64_t level_len[LH_MAX_LEVELS];
  int64_t level_off[LH_MAX_LEVELS];
  int64_t upper_off[LH_MAX_LEVELS];
  int64_t sel_off[LH_MAX_LEVELS];
  int64_t cnt_off[LH_MAX_LEVELS + 1];  // first sequence entry id of each level's kept list
  int32_t kprime[LH_MAX_LEVELS];
  int L, log2p, first_level;
  int direct;  // sel lists the kept entries themselves (not parents)
  // warp searches of the sorted lists: `rounds` rounds of 32 probes, the
  // first at stride stride0 = 32^(rounds-1) >= every list's length / 32
  int rounds, stride0;
  // one shard of the tokens (context parallelism): only the entries whose key
  // lies in [t0, t1) are gathered, from rows that hold that shard alone (x0:
  // n_loc tokens per head, pyr: the shard's own pyramid), into a per-head
  // segment of out_rows rows that starts at slot seg_off[bh]; seq_map and
  // slot_of are the segment's and the shard's.  The whole layer is the shard
  // [0, N) with seg_off null and out_rows = S.
  int64_t t0, t1, out_rows, n_loc, upper_loc, pyr_loc;
  const int64_t* seg_off;
  int64_t upper_off_loc[LH_MAX_LEVELS];
  int64_t level_off_loc[LH_MAX_LEVELS];
};

// Kept entries of every level whose key is below (e, -l), excluding level l
// itself.  A coarser level lv > l counts its entries i' with (i'+1) p^lv <=
// e + 1, a finer one those with (i'+1) p^lv <= e; the top level keeps all of
// its entries.  The other levels search their sorted lists (the kept
// parents, or the kept entries when levels are selected directly) with the
// whole warp: a round probes 32 positions of every list at once, each round
// at 1/32 of the previous stride, so a list of n entries takes ceil(log32 n)
// rounds of one load per lane and level instead of log2 n dependent loads.
template <int NL>
__device__ __forceinline__ int64_t kept_below_warp(const GatherArgs& a, const int32_t* sel_h, int l, int64_t e,
                                                   int lane) {
  const int log2p = a.log2p;
  const int top = NL - 1;
  auto target = [&](int lv) -> int64_t { return (lv > l ? e + 1 : e) >> (lv * log2p); };
  int64_t total = 0;
  if (top != l) total += min(target(top), a.level_len[top]);
  if constexpr (NL > 1) {
    constexpr int K = NL - 1;
    int tgt[K], rem[K], base[K], n[K], elem[K];
#pragma unroll
    for (int lv = 0; lv < K; ++lv) {
      const int64_t X = target(lv);  // candidates below X (entries, or parents' children)
      tgt[lv] = (int)(a.direct ? X : X >> log2p);
      rem[lv] = a.direct ? 0 : (int)(X & ((1 << log2p) - 1));
      n[lv] = lv == l ? 0 : (a.direct ? a.kprime[lv] << log2p : a.kprime[lv]);
      base[lv] = 0;
      elem[lv] = -1;
    }
    int st = a.stride0;
    for (int rd = 0; rd < a.rounds; ++rd, st >>= 5) {
      int v[K];
#pragma unroll
      for (int lv = 0; lv < K; ++lv) {
        const int pos = base[lv] + lane * st;
        v[lv] = pos < n[lv] ? sel_h[a.sel_off[lv] + pos] : 0x7fffffff;
      }
#pragma unroll
      for (int lv = 0; lv < K; ++lv) {
        // the probes below the target are a prefix: the list is ascending
        const int c = __popc(__ballot_sync(kFull, v[lv] < tgt[lv]));
        if (st == 1) elem[lv] = __shfl_sync(kFull, v[lv], c & 31);  // the entry at base + c, if probed
        if (c > 0) base[lv] += (c - 1) * st + 1;
      }
    }
#pragma unroll
    for (int lv = 0; lv < K; ++lv) {
      if (lv == l) continue;
      const int lo = base[lv];  // entries of the list below the target
      if (a.direct) {
        total += lo;
      } else {
        // parents before m contribute p children each; parent m itself, if
        // kept, its first rem children
        total += (int64_t)lo << log2p;
        if (rem[lv] > 0 && lo < n[lv] && elem[lv] == tgt[lv]) total += rem[lv];
      }
    }
  }
  return total;
}

// 16 blocks per SM (32 registers, a few spilled): 0.128 ms at 512K x 16 heads,
// against 0.134 at the 48 registers the search takes unconstrained
// SHARD: one shard of the tokens (context parallelism; the whole layer is
// compiled without its offsets)
template <typename T, int D, int NL, bool SHARD>
__global__ void __launch_bounds__(kGatherWarps * 32, 16) gather_kernel(GatherArgs a) {
  const int lane = threadIdx.x & 31;
  const int64_t wid = (int64_t)blockIdx.x * kGatherWarps + (threadIdx.x >> 5);
  const int64_t bh = wid / a.S;
  if (bh >= a.BH) return;
  const int64_t id = wid % a.S;
  const int32_t* sel_h = a.sel + bh * a.sel_per_head;
  int l = 0;
  while (l + 1 < NL && id >= a.cnt_off[l + 1]) ++l;
  const int64_t j = id - a.cnt_off[l];
  int64_t i;
  if (l < NL - 1)
    i = a.direct ? (int64_t)sel_h[a.sel_off[l] + j]
                 : ((int64_t)sel_h[a.sel_off[l] + (j >> a.log2p)] << a.log2p) + (j & ((1 << a.log2p) - 1));
  else i = j;
  const int64_t e = ((i + 1) << (l * a.log2p)) - 1;
  // the entry's slot: the kept entries whose key is below (e, -l), level l's
  // own j included
  if (SHARD && (e < a.t0 || e >= a.t1)) return;  // another shard's entry
  const int64_t slot = j + kept_below_warp<NL>(a, sel_h, l, e, lane);
  // the row in this segment, and the entry's index in the shard's level l
  const int64_t srow = SHARD ? slot - a.seg_off[bh] : slot;
  const int64_t il = SHARD ? i - (a.t0 >> (l * a.log2p)) : i;
  if (srow < 0 || srow >= a.out_rows || i < 0 || i >= a.level_len[l] || il < 0) {
    if (lane == 0) report_error(a.errw, ERRW_BOUNDS);
    return;
  }
  if (lane == 0) {
    a.seq_map[bh * a.out_rows + srow] = (int32_t)(((int64_t)l << 28) | il);
    a.slot_of[bh * a.pyr_loc + a.level_off_loc[l] + il] = (int32_t)srow;
  }
  constexpr int CH = D / 8;
  if (l >= 1 && l < a.first_level) {
    // entry not materialised: average its p^l level-0 rows (fp32, rounded once)
    const int nr = 1 << (l * a.log2p);
    const float inv = __int_as_float((127 - l * a.log2p) << 23);  // 2^(-l log2p), exact
    for (int c = lane; c < 3 * CH; c += 32) {
      const int t = c / CH, off = (c % CH) * 8;
      const T* src = static_cast<const T*>(a.x0[t]) + (bh * a.n_loc + (il << (l * a.log2p))) * D + off;
      float acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = 0.f;
      for (int r = 0; r < nr; ++r) {
        float x[8];
        if constexpr (sizeof(T) == 2) {
          load_vec<T, 8>(src + (int64_t)r * D, x);
        } else {
          load_f32<4>(reinterpret_cast<const float*>(src + (int64_t)r * D), *reinterpret_cast<float(*)[4]>(x));
          load_f32<4>(reinterpret_cast<const float*>(src + (int64_t)r * D) + 4, *reinterpret_cast<float(*)[4]>(x + 4));
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += x[e];
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] *= inv;
      if constexpr (sizeof(T) == 2) {
        // the materialised pyramid rounds the mean to bf16 once; do the same
        store_vec<__nv_bfloat16, 8>(a.out[t] + (bh * a.out_rows + srow) * D + off, acc);
      } else {
        store_vec<__nv_bfloat16, 8>(a.out[t] + (bh * a.out_rows + srow) * D + off, acc);
      }
    }
    return;
  }
  // copy the three rows, 8 elements per lane step, converting to bf16
  for (int c = lane; c < 3 * CH; c += 32) {
    const int t = c / CH, off = (c % CH) * 8;
    const T* src = (l == 0) ? static_cast<const T*>(a.x0[t]) + (bh * a.n_loc + il) * D
                            : static_cast<const T*>(a.pyr[t]) + (bh * a.upper_loc + a.upper_off_loc[l] + il) * D;
    __nv_bfloat16* dst = a.out[t] + (bh * a.out_rows + srow) * D + off;
    if constexpr (sizeof(T) == 2) {
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src + off);
    } else {
      float x[8];
      load_f32<4>(reinterpret_cast<const float*>(src) + off, *reinterpret_cast<float(*)[4]>(x));
      load_f32<4>(reinterpret_cast<const float*>(src) + off + 4, *reinterpret_cast<float(*)[4]>(x + 4));
      store_vec<__nv_bfloat16, 8>(dst, x);
    }
  }
}

// ---------------------------------------------------------------------------
// scatter-back: Y_j = sum_l [kept] Os[slot(l, ((j+1) >> l log2p) - 1)]
// 16-byte output lanes, R (1 or 2) rows per warp instruction.  Each lane keeps
// the summed contribution of levels >= 1 for its own row and refreshes it when
// that row's level-1 entry changes (coarser boundaries are level-1 boundaries).
// ---------------------------------------------------------------------------
struct ScatterArgs {
  const float* os;
  const int32_t* slot_of;
  void* y;
  int64_t BH, N, S, pyr_entries;
  int64_t level_off[LH_MAX_LEVELS];
  int64_t level_len[LH_MAX_LEVELS];
  int64_t tasks_per_head;
  int task_rows, log2p;
  int tbl_ints;  // slot indices of one task's entries of levels >= 1 (the streaming kernel's table)
  // one shard of the tokens (context parallelism): the Os rows of the
  // previous shard's last entry of each level l >= 1 ([BH][L-1][d], zeros
  // where that entry is not kept), whose ranges reach this shard's first
  // p^l - 1 rows; null for the whole layer
  const float* halo;
  int L;
};

template <typename T, int D>
struct RowLayout {
  static constexpr int VE = 16 / sizeof(T) <= D / 16 ? 16 / sizeof(T) : D / 16;  // elements per lane
  static constexpr int LPR = D / VE;                                            // lanes per row
  static constexpr int R = 32 / LPR;                                            // rows per instruction
  static_assert(R == 1 || R == 2, "layout");
};

// A warp runs R tasks side by side, one per group of LPR lanes (R = 2 for a
// bf16 row of 128: two half-warps).  Task t of a head covers the rows
// j = t*task_rows - 1 ... (t+1)*task_rows - 2 (keys j+1 from t*task_rows), one
// row per step, so a step of the warp stores one row of each task.  Tasks
// start on top-level boundaries, so every task meets its level boundaries at
// the same steps: the refreshes of the cached contributions are uniform over
// the warp while their lookups (slot index, then the Os row) go out for all
// of the warp's tasks at once.
template <typename T, int D, int NL>
__global__ void __launch_bounds__(kWarps * 32) scatter_back_kernel(ScatterArgs a) {
  using Lay = RowLayout<T, D>;
  constexpr int VE = Lay::VE, LPR = Lay::LPR, R = Lay::R;
  const int lane = threadIdx.x & 31;
  const int lr = lane / LPR, cv = lane % LPR;
  const int64_t wid = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int64_t ntasks = a.BH * a.tasks_per_head;
  if (wid * R >= ntasks) return;
  const int64_t task = wid * R + lr;  // this lane group's task
  const bool active = task < ntasks;
  const int64_t bh = active ? task / a.tasks_per_head : 0;
  const int u0 = active ? (int)(task % a.tasks_per_head) * a.task_rows : 0;  // rows within a head fit 32 bits
  const int N = (int)a.N;
  const int log2p = a.log2p;
  const int32_t* so = a.slot_of + bh * a.pyr_entries;
  const float* os = a.os + bh * a.S * D + cv * VE;
  T* out = static_cast<T*>(a.y) + bh * a.N * D + cv * VE;

  // contribution of level 1, refreshed at level-1 boundaries, and the summed
  // contribution of levels >= 2, refreshed at level-2 boundaries
  float up1[VE], high[VE];
#pragma unroll
  for (int c = 0; c < VE; ++c) up1[c] = high[c] = 0.f;
  // live: a row of this task inside the head (keys past N would index past
  // the level tables); i < 0 is the part of a level before its first entry
  auto contribution = [&](bool live, int l, int i, float (&acc)[VE]) {
    const int s = (live && i >= 0) ? so[a.level_off[l] + i] : -1;
    if (s >= 0) {
      float v[VE];
      load_f32<VE>(os + (int64_t)s * D, v);
#pragma unroll
      for (int c = 0; c < VE; ++c) acc[c] += v[c];
    }
  };
  constexpr int SW = 32 / R;  // level-0 slots fetched per lane group at a time
  int s0w = -1;
  for (int r = 0; r < a.task_rows; ++r) {
    const int key = u0 + r;  // j + 1
    const int j = key - 1;
    const bool live = active && j < N;
    if (r % SW == 0) {
      const int jw = j + cv % SW;
      s0w = (active && jw >= 0 && jw < N) ? so[a.level_off[0] + jw] : -1;
    }
    if constexpr (NL > 1) {
      if ((r & ((1 << log2p) - 1)) == 0) {
#pragma unroll
        for (int c = 0; c < VE; ++c) up1[c] = 0.f;
        contribution(live, 1, (key >> log2p) - 1, up1);
        if constexpr (NL > 2) {
          if ((r & ((1 << (2 * log2p)) - 1)) == 0) {
#pragma unroll
            for (int c = 0; c < VE; ++c) high[c] = 0.f;
#pragma unroll
            for (int l = NL - 1; l >= 2; --l) contribution(live, l, (key >> (l * log2p)) - 1, high);
          }
        }
      }
    }
    const int s0 = __shfl_sync(kFull, s0w, lr * LPR + r % SW);
    float y[VE];
#pragma unroll
    for (int c = 0; c < VE; ++c) y[c] = up1[c] + high[c];
    if (s0 >= 0) {
      float v[VE];
      load_f32<VE>(os + (int64_t)s0 * D, v);
#pragma unroll
      for (int c = 0; c < VE; ++c) y[c] = v[c] + y[c];
    }
    if (live && j >= 0) store_vec<T, VE>(out + (int64_t)j * D, y);
  }
}

// The scatter-back for bf16 rows of 128 channels as a store stream: one task
// of task_rows keys per warp, two rows per step (lane l: channels
// [8 (l mod 16), +8) of row 2s + l div 16; p is even, so both rows of a step
// share their entries of every level >= 1).  When a task starts, the slot
// indices of its entries of levels >= 1 go to a per-warp table in shared
// memory, and the level-0 ones are fetched 32 rows ahead, so a step waits on
// memory only where a kept entry's Os row is read.  Levels are refreshed at
// their own boundaries: the top level's row once per top-level block, the
// levels between it and level 1 summed at level-2 boundaries, level 1 at
// level-1 boundaries.
// HALO: one shard of the tokens with the previous shard's boundary rows (the
// whole layer is compiled without them)
template <int NL, bool HALO>
__global__ void __launch_bounds__(kWarps * 32) scatter_back_stream_kernel(ScatterArgs a) {
  constexpr int D = 128;
  extern __shared__ int32_t sb_tbl[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int lr = lane >> 4, cv = lane & 15;
  const int64_t task = (int64_t)blockIdx.x * kWarps + warp;
  if (task >= a.BH * a.tasks_per_head) return;
  const int64_t bh = task / a.tasks_per_head;
  const int T = a.task_rows;
  const int u0 = (int)(task % a.tasks_per_head) * T;  // the task's first key j' = j + 1
  const int N = (int)a.N, log2p = a.log2p;
  const int32_t* so = a.slot_of + bh * a.pyr_entries;
  const float* os = a.os + bh * a.S * D + cv * 8;
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.y) + bh * a.N * D + cv * 8;
  int32_t* tbl = sb_tbl + warp * a.tbl_ints;
  // level l (>= 1): T >> l log2p entries from (u0 >> l log2p) - 1; -1 where
  // the level has no such entry
  int toff[NL > 1 ? NL : 1];
  {
    int off = 0;
#pragma unroll
    for (int l = 1; l < NL; ++l) {
      toff[l] = off;
      const int n = T >> (l * log2p);
      const int64_t i0 = (int64_t)(u0 >> (l * log2p)) - 1;
      for (int k = lane; k < n; k += 32) {
        const int64_t i = i0 + k;
        // -1: no entry; -1 - l: the previous shard's entry of level l (halo)
        tbl[off + k] = (i >= 0 && i < a.level_len[l]) ? so[a.level_off[l] + i] : ((HALO && i == -1) ? -1 - l : -1);
      }
      off += n;
    }
  }
  __syncwarp();
  auto add_row = [&](int slot, float (&acc)[8]) {
    const float4* src = reinterpret_cast<const float4*>(
        (!HALO || slot >= 0) ? os + (int64_t)slot * D : a.halo + ((bh * (a.L - 1)) + (-2 - slot)) * D + cv * 8);
    const float4 v0 = __ldg(src), v1 = __ldg(src + 1);
    acc[0] += v0.x; acc[1] += v0.y; acc[2] += v0.z; acc[3] += v0.w;
    acc[4] += v1.x; acc[5] += v1.y; acc[6] += v1.z; acc[7] += v1.w;
  };
  // level-0 slots of task rows r (j = u0 - 1 + r), 32 at a time, one batch ahead
  auto s0_load = [&](int r) -> int {
    const int j = u0 - 1 + r;
    return (r < T && j >= 0 && j < N) ? so[a.level_off[0] + j] : -1;
  };
  int s0_cur = s0_load(lane), s0_next = s0_load(32 + lane);
  float ctop[8], high[8], cs[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) ctop[c] = high[c] = cs[c] = 0.f;
  const int pm1 = (1 << log2p) - 1, pm2 = (1 << (2 * log2p)) - 1;
  const int pmt = NL > 1 ? (1 << ((NL - 1) * log2p)) - 1 : 0;
  // rows of the task that exist: j = u0 - 1 + r in [0, N)
  const int rlo = u0 == 0 ? 1 : 0, rhi = min(T, N + 1 - u0);
  // T is a multiple of 64: batches of 32 rows, 16 steps each, unrolled
  for (int rb = 0; rb < T; rb += 32) {
    if (rb > 0) {
      s0_cur = s0_next;
      s0_next = s0_load(rb + 32 + lane);
    }
    const int64_t jb = (int64_t)u0 - 1 + rb + lr;  // output row of step 0 of the batch (-1 before the head)
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int r0 = rb + 2 * u;
      if constexpr (NL > 1) {
        if ((r0 & pm1) == 0) {
          if ((r0 & pmt) == 0) {
#pragma unroll
            for (int c = 0; c < 8; ++c) ctop[c] = 0.f;
            const int st = tbl[toff[NL - 1] + (r0 >> ((NL - 1) * log2p))];
            if (st != -1) add_row(st, ctop);
          }
          if constexpr (NL > 2) {
            if ((r0 & pm2) == 0) {
#pragma unroll
              for (int c = 0; c < 8; ++c) high[c] = ctop[c];
#pragma unroll
              for (int l = 2; l < NL - 1; ++l) {
                const int sl = tbl[toff[l] + (r0 >> (l * log2p))];
                if (sl != -1) add_row(sl, high);
              }
            }
#pragma unroll
            for (int c = 0; c < 8; ++c) cs[c] = high[c];
            const int s1 = tbl[toff[1] + (r0 >> log2p)];
            if (s1 != -1) add_row(s1, cs);
          } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) cs[c] = ctop[c];
          }
        }
      }
      const int s0 = __shfl_sync(kFull, s0_cur, 2 * u + lr);
      const int r = r0 + lr;
      const bool ok = r >= rlo && r < rhi;
      // Y with streaming stores (evict first): it is read by no later kernel
      if (s0 >= 0) {
        float y[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) y[c] = cs[c];
        add_row(s0, y);
        if (ok) store_vec_stream<__nv_bfloat16, 8>(out + (jb + 2 * u) * D, y);
      } else if (ok) {
        store_vec_stream<__nv_bfloat16, 8>(out + (jb + 2 * u) * D, cs);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// scatter-back adjoint: dOs[s] = sum_{j in R(l,i)} dY_j (fp32), Delta[s] = dOs[s] . Os[s]
// one warp per slot, R rows per warp instruction.  dOs is rounded once to
// bf16 (the attention's 16-bit input) and stored as fp16, which holds every
// bf16 value of magnitude up to 65504 exactly; the attention backward reads it
// as the fp16 operand of its dV and dP products.  A larger magnitude sets the
// range bit of the error word.
// ---------------------------------------------------------------------------
struct ScatterAdjArgs {
  const void* dy;
  const int32_t* seq_map;
  const float* os;
  __half* dos;
  float* delta;
  int* errw;
  int64_t BH, N, S;
  int L, log2p;
  // one shard of the tokens: the sums of dY over the next shard's first
  // p^l - 1 rows ([BH][L-1][d] fp32), which the range of this shard's last
  // entry of each level l >= 1 covers beyond its end; null for the whole layer
  const float* halo;
};

template <typename T, int D>
__global__ void __launch_bounds__(kSadjWarps * 32) scatter_adjoint_kernel(ScatterAdjArgs a) {
  constexpr int VE = (sizeof(T) == 2 && D == 128) ? 8 : 4;
  constexpr int LPR = D / VE, R = 32 / LPR;
  // row loads in flight per lane; at 512K: 4 -> 0.375, 8 -> 0.377, 12 or 16 -> 0.369 ms
  constexpr int U = 16;
  using Raw = typename RawVec<sizeof(T) * VE>::type;
  const int lane = threadIdx.x & 31;
  const int64_t wid = (int64_t)blockIdx.x * kSadjWarps + (threadIdx.x >> 5);
  const int64_t bh = wid / a.S;
  if (bh >= a.BH) return;
  const int64_t s = wid % a.S;
  const int lr = lane / LPR, cv = lane % LPR;
  const int32_t code = a.seq_map[bh * a.S + s];
  const int l = code >> 28;
  const int64_t i = code & ((1 << 28) - 1);
  if (l >= a.L) {
    if (lane == 0) report_error(a.errw, ERRW_BOUNDS);
    return;
  }
  const int64_t b = (int64_t)1 << (l * a.log2p);
  const int64_t r0 = min((i + 1) * b - 1, a.N), r1 = min((i + 2) * b - 1, a.N);
  const int n = (int)(r1 - r0);
  const T* src = static_cast<const T*>(a.dy) + (bh * a.N + r0) * D + cv * VE;
  float acc[VE];
#pragma unroll
  for (int c = 0; c < VE; ++c) acc[c] = 0.f;
  for (int g = 0; g < n; g += R * U) {
    Raw x[U];  // raw rows: widened to fp32 as they are summed
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int row = g + u * R + lr;
      x[u] = row < n ? __ldg(reinterpret_cast<const Raw*>(src + (int64_t)row * D)) : Raw{};
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const T* e = reinterpret_cast<const T*>(&x[u]);
#pragma unroll
      for (int c = 0; c < VE; ++c) acc[c] += Elem<T>::to_f(e[c]);
    }
  }
#pragma unroll
  for (int c = 0; c < VE; ++c)
#pragma unroll
    for (int o = LPR; o < 32; o <<= 1) acc[c] += __shfl_xor_sync(kFull, acc[c], o);
  if (a.halo && l >= 1 && (i + 2) * b - 1 > a.N) {  // the range runs into the next shard
    const float* hr = a.halo + (bh * (a.L - 1) + (l - 1)) * D + cv * VE;
#pragma unroll
    for (int c = 0; c < VE; ++c) acc[c] += hr[c];
  }
  // round to bf16 once (stored as fp16, exact in range); Delta from the
  // rounded values and the fp32 Os
  __half h[VE];
  float o_row[VE];
  load_f32<VE>(a.os + (bh * a.S + s) * D + cv * VE, o_row);
  float dot = 0.f;
  bool in_range = true;
#pragma unroll
  for (int c = 0; c < VE; ++c) {
    const float r = __bfloat162float(__float2bfloat16_rn(acc[c]));
    in_range &= fabsf(r) <= 65504.f;
    h[c] = __float2half_rn(r);
    dot = fmaf(r, o_row[c], dot);
  }
  if (!in_range) report_error(a.errw, ERRW_RANGE);
#pragma unroll
  for (int o = LPR / 2; o >= 1; o >>= 1) dot += __shfl_xor_sync(kFull, dot, o);
  if (lr == 0) {
    using V = typename RawVec<2 * VE>::type;
    *reinterpret_cast<V*>(a.dos + (bh * a.S + s) * D + cv * VE) = *reinterpret_cast<const V*>(h);
    if (cv == 0) a.delta[bh * a.S + s] = dot;
  }
}

// Sums of dY over the first p^l - 1 rows of every head, l = 1 .. L-1, in
// fp32: under context parallelism, the part of the previous shard's last
// level-l entry's range R(l, i) that lies in this shard.
template <typename T, int D>
__global__ void __launch_bounds__(D) head_sums_kernel(const T* __restrict__ dy, float* __restrict__ sums, int64_t N,
                                                      int L, int log2p) {
  const int64_t bh = blockIdx.x;
  const int l = (int)blockIdx.y + 1;
  const int c = threadIdx.x;  // one channel per thread: each row read is one coalesced access
  const int64_t rows = min(((int64_t)1 << (l * log2p)) - 1, N);
  const T* src = dy + bh * N * D + c;
  float acc = 0.f;
  for (int64_t r = 0; r < rows; ++r) acc += Elem<T>::to_f(src[r * D]);
  sums[(bh * (L - 1) + (l - 1)) * D + c] = acc;
}

template <typename T, int D>
cudaError_t scatter_dispatch_L(int L, const ScatterArgs& a, int64_t tasks, cudaStream_t st) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value && D == 128) {
    const size_t smem = (size_t)kWarps * a.tbl_ints * sizeof(int32_t);
    if (smem <= 48 * 1024 && L <= 8) {
      const int64_t blocks = (tasks + kWarps - 1) / kWarps;
      switch (L) {
#define LH_CASE(n) \
  case n:                                                                             \
    if (a.halo) scatter_back_stream_kernel<n, true><<<(unsigned)blocks, kWarps * 32, smem, st>>>(a); \
    else scatter_back_stream_kernel<n, false><<<(unsigned)blocks, kWarps * 32, smem, st>>>(a);       \
    break;
        LH_CASE(1) LH_CASE(2) LH_CASE(3) LH_CASE(4) LH_CASE(5) LH_CASE(6) LH_CASE(7) LH_CASE(8)
#undef LH_CASE
        default: return cudaErrorInvalidValue;
      }
      return cudaGetLastError();
    }
  }
  if (a.halo) return cudaErrorNotSupported;  // halo rows: the stream kernel's layouts only
  constexpr int R = RowLayout<T, D>::R;  // tasks per warp
  const int64_t blocks = ((tasks + R - 1) / R + kWarps - 1) / kWarps;
  switch (L) {
#define LH_CASE(n) \
  case n: scatter_back_kernel<T, D, n><<<(unsigned)blocks, kWarps * 32, 0, st>>>(a); break;
    LH_CASE(1) LH_CASE(2) LH_CASE(3) LH_CASE(4) LH_CASE(5) LH_CASE(6) LH_CASE(7) LH_CASE(8)
#undef LH_CASE
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t gather_dispatch_L(int L, const GatherArgs& a, int64_t blocks, cudaStream_t st) {
  switch (L) {
#define LH_CASE(n) \
  case n:                                                                      \
    if (a.seg_off) gather_kernel<T, D, n, true><<<(unsigned)blocks, kGatherWarps * 32, 0, st>>>(a); \
    else gather_kernel<T, D, n, false><<<(unsigned)blocks, kGatherWarps * 32, 0, st>>>(a);         \
    break;
    LH_CASE(1) LH_CASE(2) LH_CASE(3) LH_CASE(4) LH_CASE(5) LH_CASE(6) LH_CASE(7) LH_CASE(8)
#undef LH_CASE
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gather(const Dims& D, const void* q, const void* k, const void* v, const void* pq,
                          const void* pk, const void* pv, const int32_t* sel, void* qs, void* ks, void* vs,
                          int32_t* seq_map, int32_t* slot_of, int* errw, cudaStream_t st, int first_level,
                          const Dims* shard, int64_t t0, const int64_t* seg_off, int64_t seg_rows) {
  GatherArgs a{};
  a.x0[0] = q; a.x0[1] = k; a.x0[2] = v;
  a.pyr[0] = pq; a.pyr[1] = pk; a.pyr[2] = pv;
  a.sel = sel;
  a.out[0] = static_cast<__nv_bfloat16*>(qs);
  a.out[1] = static_cast<__nv_bfloat16*>(ks);
  a.out[2] = static_cast<__nv_bfloat16*>(vs);
  a.seq_map = seq_map;
  a.slot_of = slot_of;
  a.errw = errw;
  a.BH = D.BH; a.N = D.N; a.S = D.S;
  a.upper_entries = D.upper_entries; a.pyr_entries = D.pyr_entries; a.sel_per_head = D.sel_per_head;
  for (int l = 0; l < LH_MAX_LEVELS; ++l) {
    a.level_len[l] = D.level_len[l];
    a.level_off[l] = D.level_off[l];
    a.upper_off[l] = D.upper_off[l];
    a.sel_off[l] = D.sel_off[l];
    a.kprime[l] = D.kprime[l];
  }
  a.cnt_off[0] = 0;
  for (int l = 0; l < D.L - 1; ++l) a.cnt_off[l + 1] = a.cnt_off[l] + ((int64_t)D.kprime[l] << D.log2p);
  a.L = D.L;
  a.log2p = D.log2p;
  a.first_level = first_level;
  a.direct = D.selection == LH_SELECT_DIRECT;
  int64_t max_n = 1;
  for (int l = 0; l + 1 < D.L; ++l) {
    const int64_t n = a.direct ? ((int64_t)D.kprime[l] << D.log2p) : D.kprime[l];
    if (n > max_n) max_n = n;
  }
  a.rounds = 1;
  a.stride0 = 1;
  while ((int64_t)a.stride0 * 32 < max_n) {
    ++a.rounds;
    a.stride0 *= 32;
  }
  // the shard (the whole layer unless one is given): its token range, row
  // counts and table offsets
  const Dims& Ls = shard ? *shard : D;
  a.t0 = shard ? t0 : 0;
  a.t1 = a.t0 + Ls.N;
  a.seg_off = seg_off;
  a.out_rows = shard ? seg_rows : D.S;
  a.n_loc = Ls.N;
  a.upper_loc = Ls.upper_entries;
  a.pyr_loc = Ls.pyr_entries;
  for (int l = 0; l < LH_MAX_LEVELS; ++l) {
    a.upper_off_loc[l] = Ls.upper_off[l];
    a.level_off_loc[l] = Ls.level_off[l];
  }
  cudaError_t e = cudaMemsetAsync(slot_of, 0xff, (size_t)D.BH * Ls.pyr_entries * sizeof(int32_t), st);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (D.BH * D.S + kGatherWarps - 1) / kGatherWarps;
  if (D.dtype == LH_BF16) {
    return D.d == 128 ? gather_dispatch_L<__nv_bfloat16, 128>(D.L, a, blocks, st)
                      : gather_dispatch_L<__nv_bfloat16, 64>(D.L, a, blocks, st);
  }
  return D.d == 128 ? gather_dispatch_L<float, 128>(D.L, a, blocks, st)
                    : gather_dispatch_L<float, 64>(D.L, a, blocks, st);
}

cudaError_t launch_scatter_back(const Dims& D, const float* os, const int32_t* slot_of, void* y, cudaStream_t st,
                                const float* halo) {
  ScatterArgs a{};
  a.os = os;
  a.slot_of = slot_of;
  a.y = y;
  a.halo = halo;
  a.L = D.L;
  a.BH = D.BH; a.N = D.N; a.S = D.S; a.pyr_entries = D.pyr_entries;
  for (int l = 0; l < LH_MAX_LEVELS; ++l) {
    a.level_off[l] = D.level_off[l];
    a.level_len[l] = D.level_len[l];
  }
  const int64_t ptop = (int64_t)1 << ((D.L - 1) * D.log2p);
  a.task_rows = (int)(ptop > 64 ? ptop : 64);
  a.tasks_per_head = (D.N + 1 + a.task_rows - 1) / a.task_rows;  // steps cover rows -1 .. N-1
  a.log2p = D.log2p;
  int64_t tbl = 0;
  for (int l = 1; l < D.L; ++l) tbl += a.task_rows >> (l * D.log2p);
  a.tbl_ints = (int)std::min<int64_t>(tbl, 1 << 20);
  const int64_t tasks = D.BH * a.tasks_per_head;
  if (D.dtype == LH_BF16) {
    return D.d == 128 ? scatter_dispatch_L<__nv_bfloat16, 128>(D.L, a, tasks, st)
                      : scatter_dispatch_L<__nv_bfloat16, 64>(D.L, a, tasks, st);
  }
  return D.d == 128 ? scatter_dispatch_L<float, 128>(D.L, a, tasks, st)
                    : scatter_dispatch_L<float, 64>(D.L, a, tasks, st);
}

cudaError_t launch_scatter_adjoint(const Dims& D, const void* dy, const int32_t* seq_map, const float* os,
                                   void* dos, float* delta, int* errw, cudaStream_t st, const float* halo) {
  ScatterAdjArgs a{};
  a.halo = halo;
  a.dy = dy;
  a.seq_map = seq_map;
  a.os = os;
  a.dos = static_cast<__half*>(dos);
  a.delta = delta;
  a.errw = errw;
  a.BH = D.BH; a.N = D.N; a.S = D.S;
  a.L = D.L;
  a.log2p = D.log2p;
  const int64_t blocks = (D.BH * D.S + kSadjWarps - 1) / kSadjWarps;
  if (D.dtype == LH_BF16) {
    if (D.d == 128) scatter_adjoint_kernel<__nv_bfloat16, 128><<<(unsigned)blocks, kSadjWarps * 32, 0, st>>>(a);
    else scatter_adjoint_kernel<__nv_bfloat16, 64><<<(unsigned)blocks, kSadjWarps * 32, 0, st>>>(a);
  } else {
    if (D.d == 128) scatter_adjoint_kernel<float, 128><<<(unsigned)blocks, kSadjWarps * 32, 0, st>>>(a);
    else scatter_adjoint_kernel<float, 64><<<(unsigned)blocks, kSadjWarps * 32, 0, st>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_head_sums(const Dims& D, const void* dy, float* sums, cudaStream_t st) {
  if (D.L < 2) return cudaSuccess;
  const dim3 grid((unsigned)D.BH, (unsigned)(D.L - 1));
  if (D.dtype == LH_BF16) {
    if (D.d == 128)
      head_sums_kernel<__nv_bfloat16, 128><<<grid, 128, 0, st>>>(static_cast<const __nv_bfloat16*>(dy), sums, D.N, D.L,
                                                                   D.log2p);
    else
      head_sums_kernel<__nv_bfloat16, 64><<<grid, 64, 0, st>>>(static_cast<const __nv_bfloat16*>(dy), sums, D.N, D.L,
                                                                 D.log2p);
  } else {
    if (D.d == 128)
      head_sums_kernel<float, 128><<<grid, 128, 0, st>>>(static_cast<const float*>(dy), sums, D.N, D.L, D.log2p);
    else
      head_sums_kernel<float, 64><<<grid, 64, 0, st>>>(static_cast<const float*>(dy), sums, D.N, D.L, D.log2p);
  }
  return cudaGetLastError();
}

}  // namespace lh
