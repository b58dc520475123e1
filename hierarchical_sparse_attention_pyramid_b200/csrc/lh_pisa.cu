// PISA block selection: a coarse-to-fine top-K over a pooled key pyramid,
// each candidate block scored by the LogSumExp of its logits (the
// blog.secrett2633.cloud review "[논문리뷰] Block Sparse Attention with
// Log-Linear Complexity", sections 1 and 3: keys are pooled into a
// fine-to-coarse hierarchy, selection starts at the coarsest level, every
// level scores a small candidate set with LSE, keeps the top K and expands
// them into their sub-blocks one level down).
//
// pisa_pool_kernel   - the key pyramid: level l entry j is the mean of key rows
//   [j p^l, (j+1) p^l), summed exactly in fp64 and rounded once to bf16 (round
//   to nearest even).  One warp per top-level span of p^(L-1) rows.
//
// pisa_select_kernel - one CTA per (query group of 128 rows, head).  The group
//   makes one selection.  Warp roles:
//     warp 0      TMA producer: the group's Q tile once, then the visible
//                 candidates' key blocks, 128 key rows (one unit: two blocks
//                 of 64 or one of 128) per stage of a 2-stage ring
//     warp 1      MMA issuer: S = Q K_unit^T (128 x 128, fp32) per unit into
//                 one of two TMEM buffers
//     warps 2-9   scorers, thread = (query row, column half): the row's
//                 max and sum of 2^(s - max) over its half of the block
//                 (masked only where the warp sees a causal edge), reduced
//                 over the warp's 32 rows into one log2 partial per
//                 candidate; at the end of a
//                 level they combine the four partials into each candidate's
//                 score, rank the candidates, write the kept blocks and build
//                 the next level's candidate list (the kept blocks' p
//                 sub-blocks each), then release the producer and MMA warps
//                 for that level.
//   A candidate none of whose entries the group can see (its first entry ends
//   after the group's last query) scores -inf without being loaded.
#include <cudaTypedefs.h>
#include <math.h>
#include <string.h>

#include <type_traits>

#include "lh_common.cuh"
#include "sm100.cuh"

namespace lh {

bool make_seq_map(CUtensorMap* m, const void* base, int64_t BH, int64_t rows, int D, int box_rows);

namespace {
using namespace sm100;

constexpr int kG = 128;          // queries per group: the MMA's M
constexpr int kMaxCand = 256;    // candidates of one level held in shared memory
constexpr int kScorers = 256;    // 8 scorer warps
constexpr int kThreads = 64 + kScorers;  // producer, MMA issuer, scorers
constexpr int kMaxLevels = 8;

struct PisaArgs {
  int N, n_groups, L, log2p, K;
  int level_off[kMaxLevels];  // first row of level l >= 1 in the key pyramid
  float scale_log2;           // log2(e) / sqrt(d)
  int32_t* kept_idx;          // [BH][n_groups][L][K]
  float* kept_score;          // [BH][n_groups][L][K]
  int* errw;
};

// A "unit" is 128 key rows: two blocks of 64 (scored by one MMA of N = 128)
// or one block of 128.
template <int D, int C>
struct PisaSmem {
  static constexpr int BPU = 128 / C;          // blocks per unit
  static constexpr int NST = 2;                // key stages, one unit each
  static constexpr int NBUF = 2;               // TMEM score buffers, 128 columns each
  static constexpr int kQChunk = kG * 128;     // [128 rows][64 bf16]
  static constexpr int kKChunk = 128 * 128;    // [128 key rows][64 bf16]
  static constexpr int kQ = D / 64 * kQChunk;
  static constexpr int kKStage = D / 64 * kKChunk;
  static constexpr int oQ = 0;
  static constexpr int oK = oQ + kQ;
  static constexpr int oCand = oK + NST * kKStage;          // int [2][kMaxCand]
  static constexpr int oScore = oCand + 2 * kMaxCand * 4;   // float [kMaxCand]
  static constexpr int oPart = oScore + kMaxCand * 4;       // float [8][kMaxCand], then int flags [kMaxCand]
  static constexpr int oMisc = oPart + 8 * kMaxCand * 4;    // int counts [2], tmem slot, abort flag
  static constexpr int oBar = oMisc + 64;
  static constexpr int kBytes = oBar + 256;
  static constexpr int kAlloc = kBytes + 1024;
};

// maximum over the warp (redux.sync on sm_100a)
__device__ __forceinline__ float warp_max_f32(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// is block b of level l seen by any query of the group?  (its first entry's
// last averaged token (bC+1) p^l - 1 is at or before the group's last query)
__device__ __forceinline__ bool block_visible(int b, int l, int log2p, int C, int last_query) {
  return ((((int64_t)b * C + 1) << (l * log2p)) - 1) <= (int64_t)last_query;
}

template <int D, int C>
__global__ void __launch_bounds__(kThreads, 2)
    pisa_select_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK0,
                       const __grid_constant__ CUtensorMap tmKU, const PisaArgs a) {
  using Lay = PisaSmem<D, C>;
  constexpr int NST = Lay::NST, NBUF = Lay::NBUF, BPU = Lay::BPU;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::oBar);
  uint64_t* bQ = bars + 0;
  uint64_t* bLevel = bars + 1;             // a level's candidate list is ready (one arrival per scorer)
  uint64_t* bK = bars + 2;                 // [NST] key block landed
  uint64_t* bKfree = bars + 2 + NST;       // [NST] its MMA is done
  uint64_t* bS = bars + 2 + 2 * NST;       // [NBUF] scores in TMEM
  uint64_t* bSfree = bars + 2 + 2 * NST + NBUF;  // [NBUF] scores read (one arrival per scorer)
  int32_t* cand = reinterpret_cast<int32_t*>(smem + Lay::oCand);
  float* score = reinterpret_cast<float*>(smem + Lay::oScore);
  float* part = reinterpret_cast<float*>(smem + Lay::oPart);
  int32_t* flag = reinterpret_cast<int32_t*>(smem + Lay::oPart);  // reuses part once it is consumed
  volatile int32_t* count = reinterpret_cast<volatile int32_t*>(smem + Lay::oMisc);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::oMisc + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::oMisc + 12);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = a.n_groups - 1 - (int)blockIdx.x;  // groups with the most visible blocks first
  const int bh = (int)blockIdx.y;
  const int first_query = g * kG, last_query = first_query + kG - 1;
  const int L = a.L, log2p = a.log2p;

  if (threadIdx.x == 0) {
    mbar_init(bQ, 1);
    mbar_init(bLevel, kScorers);
    for (int s = 0; s < NST; ++s) {
      mbar_init(&bK[s], 1);
      mbar_init(&bKfree[s], 1);
    }
    for (int s = 0; s < NBUF; ++s) {
      mbar_init(&bS[s], 1);
      mbar_init(&bSfree[s], kScorers);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK0);
      tma_prefetch_desc(&tmKU);
      mbar_expect_tx(bQ, kG * D * 2);
      for (int ch = 0; ch < D / 64; ++ch)
        tma_load_3d(smem + Lay::oQ + ch * Lay::kQChunk, &tmQ, bQ, ch * 64, first_query, bh);
      uint32_t u = 0;  // units loaded so far
      bool ok = true;
      for (int li = 0; ok && li < L; ++li) {
        const int l = L - 1 - li, buf = li & 1;
        if (!mbar_wait(bLevel, li & 1, abort_flag)) break;
        const int n = count[buf];
        const int* cl = cand + buf * kMaxCand;
        int nv = 0;  // visible candidates: a prefix of the ascending list
        while (nv < n && block_visible(cl[nv], l, log2p, C, last_query)) ++nv;
        const CUtensorMap* map = l == 0 ? &tmK0 : &tmKU;
        const int row0 = l == 0 ? 0 : a.level_off[l];
        for (int c = 0; c < nv; c += BPU) {
          const int nb = nv - c < BPU ? nv - c : BPU;
          const int st = (int)(u % NST);
          if (u >= (uint32_t)NST && !mbar_wait(&bKfree[st], ((u / NST) - 1) & 1, abort_flag)) { ok = false; break; }
          mbar_expect_tx(&bK[st], nb * C * D * 2);
          for (int j = 0; j < nb; ++j)
            for (int ch = 0; ch < D / 64; ++ch)
              tma_load_3d(smem + Lay::oK + st * Lay::kKStage + ch * Lay::kKChunk + j * C * 128, map, &bK[st],
                          ch * 64, row0 + cl[c + j] * C, bh);
          ++u;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idFull = idesc_bf16(kG, 128, false, false);
    constexpr uint32_t idHalf = idesc_bf16(kG, C, false, false);  // a unit holding one block of 64
    const uint64_t dQ = sdesc_sw128(smem_u32(smem + Lay::oQ), 16, 1024);
    const uint64_t dK = sdesc_sw128(smem_u32(smem + Lay::oK), 16, 1024);
    bool ok = mbar_wait_warp(bQ, 0, abort_flag);
    uint32_t u = 0;
    for (int li = 0; ok && li < L; ++li) {
      const int l = L - 1 - li, buf = li & 1;
      if (!mbar_wait_warp(bLevel, li & 1, abort_flag)) break;
      const int n = count[buf];
      const int* cl = cand + buf * kMaxCand;
      int nv = 0;
      while (nv < n && block_visible(cl[nv], l, log2p, C, last_query)) ++nv;
      for (int c = 0; c < nv; c += BPU) {
        const uint32_t id = nv - c >= BPU ? idFull : idHalf;
        const int st = (int)(u % NST), sb = (int)(u % NBUF);
        if (!mbar_wait_warp(&bK[st], (u / NST) & 1, abort_flag)) { ok = false; break; }
        if (u >= (uint32_t)NBUF && !mbar_wait_warp(&bSfree[sb], ((u / NBUF) - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t kb = dK + ((st * Lay::kKStage) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t oq = ((kk >> 2) * Lay::kQChunk + (kk & 3) * 32) >> 4;
          const uint32_t ok_ = ((kk >> 2) * Lay::kKChunk + (kk & 3) * 32) >> 4;
          umma_bf16_w(tmem + sb * 128, dQ + oq, kb + ok_, id, kk > 0 ? 1u : 0u);
        }
        umma_commit_w(&bKfree[st]);
        umma_commit_w(&bS[sb]);
        ++u;
      }
    }
  } else {
    // ------------------------------------------------------------ scorers
    // Thread (h, row): query row `row` of the group (TMEM lane row) and
    // columns [h C/2, h C/2 + C/2) of each candidate's score tile.  Each warp
    // reduces its 32 rows into one log2-sum-exp2 partial per candidate; the
    // eight partials are combined at the end of the level.
    const int t = threadIdx.x - 64;              // 0..255
    const int q = warp & 3;                      // TMEM lane quarter of this warp
    const int h = (warp - 2) >> 2;               // column half
    const int wp = h * 4 + q;                    // partial slot of this warp
    const int row = q * 32 + lane;               // query row of the group
    const int i = first_query + row;
    constexpr int HC = C / 2;                    // columns per thread
    const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16) + h * HC;
    const float ln2 = 0.69314718055994530942f;
    const float sl2 = a.scale_log2;
    const int64_t out0 = ((int64_t)bh * a.n_groups + g) * L * a.K;
    auto sync_scorers = [] { asm volatile("bar.sync 1, 256;" ::: "memory"); };

    // the coarsest level's candidates: all its blocks
    const int n_top = (a.N >> ((L - 1) * log2p)) / C;
    for (int c = t; c < n_top; c += kScorers) cand[c] = c;
    if (t == 0) count[0] = n_top;
    sync_scorers();
    mbar_arrive(bLevel);

    uint32_t u = 0;
    bool ok = true;
    for (int li = 0; li < L; ++li) {
      const int l = L - 1 - li, buf = li & 1;
      const int n = count[buf];
      const int* cl = cand + buf * kMaxCand;
      // the list is ascending and visibility falls with the block index, so
      // the visible candidates are a prefix of it
      int nv = 0;
      while (nv < n && block_visible(cl[nv], l, log2p, C, last_query)) ++nv;
      if (lane == 0)
        for (int c = nv; c < n; ++c) part[wp * kMaxCand + c] = -INFINITY;
      const int lbase = ((i + 1) >> (l * log2p)) - 1 - h * HC;
      // one unit at a time: both blocks of a unit of two are scored
      // together, so their exponentials and warp reductions interleave
      auto score_blocks = [&](auto nb_tag, int c0) {
        constexpr int NB = decltype(nb_tag)::value;  // blocks of this unit
        uint32_t r[NB][HC / 32][32];
        const int sb = (int)(u % NBUF);
        ok = __all_sync(0xffffffffu, mbar_wait(&bS[sb], (u / NBUF) & 1, abort_flag));
        if (!ok) return;
        tc_fence_after();
#pragma unroll
        for (int j = 0; j < NB; ++j)
#pragma unroll
          for (int x = 0; x < HC / 32; ++x) tmem_ld32(tl + sb * 128 + j * C + x * 32, r[j][x]);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&bSfree[sb]);
        ++u;
        // last column of this thread's half the row sees, per candidate:
        // entry j = bC + col is visible while (j+1) p^l - 1 <= i
        int lim[NB];
        bool all_vis = true;
#pragma unroll
        for (int j = 0; j < NB; ++j) {
          lim[j] = lbase - cl[c0 + j] * C;
          all_vis = all_vis && lim[j] >= HC - 1;
        }
        float m_row[NB], s_row[NB];
        if (__all_sync(0xffffffffu, all_vis)) {
          // every column visible to every row of the warp: no masks
#pragma unroll
          for (int j = 0; j < NB; ++j) {
            float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int x = 0; x < HC / 32; ++x)
#pragma unroll
              for (int y = 0; y < 32; y += 8)
#pragma unroll
                for (int z = 0; z < 4; ++z)
                  mx[z] = max3f(mx[z], __uint_as_float(r[j][x][y + 2 * z]), __uint_as_float(r[j][x][y + 2 * z + 1]));
            m_row[j] = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;
          }
#pragma unroll
          for (int j = 0; j < NB; ++j) {
            const uint64_t c2 = f2_pack(sl2, sl2), nm2 = f2_pack(-m_row[j], -m_row[j]);
            uint64_t acc0 = f2_pack(0.f, 0.f), acc1 = acc0;
#pragma unroll
            for (int x = 0; x < HC / 32; ++x)
#pragma unroll
              for (int y = 0; y < 32; y += 4) {
                float e0, e1, e2, e3;
                f2_unpack(f2_fma(f2_pack(__uint_as_float(r[j][x][y]), __uint_as_float(r[j][x][y + 1])), c2, nm2), e0, e1);
                f2_unpack(f2_fma(f2_pack(__uint_as_float(r[j][x][y + 2]), __uint_as_float(r[j][x][y + 3])), c2, nm2), e2,
                          e3);
                acc0 = f2_add(acc0, f2_pack(fast_exp2(e0), fast_exp2(e1)));
                acc1 = f2_add(acc1, f2_pack(fast_exp2(e2), fast_exp2(e3)));
              }
            float s0, s1;
            f2_unpack(f2_add(acc0, acc1), s0, s1);
            s_row[j] = s0 + s1;
          }
        } else {
#pragma unroll
          for (int j = 0; j < NB; ++j) {
            float mx = -INFINITY;
#pragma unroll
            for (int x = 0; x < HC / 32; ++x)
#pragma unroll
              for (int y = 0; y < 32; ++y)
                if (x * 32 + y <= lim[j]) mx = fmaxf(mx, __uint_as_float(r[j][x][y]));
            m_row[j] = -INFINITY;
            s_row[j] = 0.f;
            if (mx != -INFINITY) {
              m_row[j] = mx * sl2;
              float s0 = 0.f, s1 = 0.f;
#pragma unroll
              for (int x = 0; x < HC / 32; ++x)
#pragma unroll
                for (int y = 0; y < 32; y += 2) {
                  const float e0 = fast_exp2(fmaf(__uint_as_float(r[j][x][y]), sl2, -m_row[j]));
                  const float e1 = fast_exp2(fmaf(__uint_as_float(r[j][x][y + 1]), sl2, -m_row[j]));
                  s0 += x * 32 + y <= lim[j] ? e0 : 0.f;
                  s1 += x * 32 + y + 1 <= lim[j] ? e1 : 0.f;
                }
              s_row[j] = s0 + s1;
            }
          }
        }
        // the warp's 32 rows: one log2-sum-exp2 partial per candidate
#pragma unroll
        for (int j = 0; j < NB; ++j) {
          const float M = warp_max_f32(m_row[j]);
          float S = M == -INFINITY || m_row[j] == -INFINITY ? 0.f : s_row[j] * fast_exp2(m_row[j] - M);
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
          if (lane == 0) part[wp * kMaxCand + c0 + j] = S > 0.f ? M + __log2f(S) : -INFINITY;
        }
      };
      int c = 0;
      if constexpr (Lay::BPU == 2)
        for (; ok && c + 1 < nv; c += 2) score_blocks(std::integral_constant<int, 2>{}, c);
      for (; ok && c < nv; ++c) score_blocks(std::integral_constant<int, 1>{}, c);
      // level end: scores, ranks, kept blocks, next candidates.  Every scorer
      // thread runs all L levels and reaches each barrier, also after an
      // abort (its waits then fail at once and the level's lists hold
      // placeholders of bounded size), so no warp waits at a barrier alone.
      sync_scorers();
      for (int c = t; c < n; c += kScorers) {
        float pv[8];
        float M = -INFINITY;
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          pv[x] = part[x * kMaxCand + c];
          M = fmaxf(M, pv[x]);
        }
        float sc = -INFINITY;
        if (M != -INFINITY) {
          float S = 0.f;
#pragma unroll
          for (int x = 0; x < 8; ++x) S += fast_exp2(pv[x] - M);
          sc = (M + __log2f(S)) * ln2;
        }
        score[c] = sc;
      }
      sync_scorers();
      const int kk = n < a.K ? n : a.K;
      for (int c = t; c < n; c += kScorers) {
        const float s = score[c];
        int rank = 0;
        for (int c2 = 0; c2 < n; ++c2) {
          const float s2 = score[c2];
          rank += (s2 > s) || (s2 == s && c2 < c);  // list order is block order
        }
        flag[c] = rank < kk;
      }
      sync_scorers();
      const int nbuf = buf ^ 1;
      int32_t* nl = cand + nbuf * kMaxCand;
      const int p = 1 << log2p;
      for (int c = t; c < n; c += kScorers) {
        if (!flag[c]) continue;
        int pos = 0;
        for (int c2 = 0; c2 < c; ++c2) pos += flag[c2];
        a.kept_idx[out0 + (int64_t)l * a.K + pos] = cl[c];
        a.kept_score[out0 + (int64_t)l * a.K + pos] = score[c];
        if (l > 0)
          for (int x = 0; x < p; ++x) nl[pos * p + x] = cl[c] * p + x;
      }
      for (int pos = kk + t; pos < a.K; pos += kScorers) {
        a.kept_idx[out0 + (int64_t)l * a.K + pos] = -1;
        a.kept_score[out0 + (int64_t)l * a.K + pos] = -INFINITY;
      }
      if (t == 0) count[nbuf] = kk * p;
      sync_scorers();
      if (l > 0) mbar_arrive(bLevel);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
  if (threadIdx.x == 0 && *abort_flag) report_error(a.errw, ERRW_TIMEOUT);
}

// ---------------------------------------------------------------------------
// key pyramid
// ---------------------------------------------------------------------------

// x rounded to the nearest bf16 value, ties to even, as if straight from
// binary64: x is first rounded to fp32 with round-to-odd (truncate, then set
// the last bit when anything was cut off), then to bf16 with round-to-nearest-
// even.  Rounding to odd at a precision at least two bits above the target's
// makes the second rounding the correct one (Boldo and Melquiond, "Emulation
// of FMA and correctly rounded sums: proved algorithms using rounding to
// odd", IEEE Trans. Computers 57(4), 2008); fp32 keeps 24 bits, bf16 8.
__device__ __forceinline__ uint16_t bf16_from_double_rne(double x) {
  float r = __double2float_rz(x);
  if ((double)r != x) r = __uint_as_float(__float_as_uint(r) | 1u);
  return __bfloat16_as_ushort(__float2bfloat16_rn(r));
}

struct PoolKArgs {
  const __nv_bfloat16* k;
  __nv_bfloat16* pyr;  // [BH][upper][D]
  int64_t BH, N, upper;
  int L, log2p;
  int64_t level_off[kMaxLevels];
};

template <int D, int NL>
__global__ void __launch_bounds__(256) pisa_pool_kernel(PoolKArgs a) {
  constexpr int VE = D / 32;  // columns per lane
  using Raw = typename RawVec<2 * VE>::type;
  const int lane = threadIdx.x & 31;
  const int span_log = (NL - 1) * a.log2p;
  const int64_t spans = a.N >> span_log;
  const int64_t w = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (w >= a.BH * spans) return;
  const int64_t bh = w / spans, s = w % spans;
  const int span = 1 << span_log;
  const __nv_bfloat16* src = a.k + ((bh * a.N + (s << span_log)) * D) + lane * VE;
  double acc[NL][VE];  // acc[l]: running sum of the level-l entry being built (l >= 1)
#pragma unroll
  for (int l = 0; l < NL; ++l)
#pragma unroll
    for (int v = 0; v < VE; ++v) acc[l][v] = 0.0;
  constexpr int U = 16;  // rows in flight per lane
  for (int r0 = 0; r0 < span; r0 += U) {
    Raw raw[U];
#pragma unroll
    for (int x = 0; x < U; ++x)
      if (r0 + x < span) raw[x] = __ldg(reinterpret_cast<const Raw*>(src + (int64_t)(r0 + x) * D));
#pragma unroll
    for (int x = 0; x < U; ++x) {
      if (r0 + x >= span) break;
      const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&raw[x]);
#pragma unroll
      for (int v = 0; v < VE; ++v) acc[1][v] += (double)__bfloat162float(e[v]);
      const int done = r0 + x + 1;  // rows of the span summed so far
#pragma unroll
      for (int l = 1; l < NL; ++l) {
        if ((done & ((1 << (l * a.log2p)) - 1)) != 0) break;
        // level l entry complete: mean = sum * 2^-(l log2 p), exact
        const double inv = ldexp(1.0, -l * a.log2p);
        const int64_t entry = ((s << span_log) + done) >> (l * a.log2p);
        uint16_t o[VE];
#pragma unroll
        for (int v = 0; v < VE; ++v) o[v] = bf16_from_double_rne(acc[l][v] * inv);
        Raw packed;
        memcpy(&packed, o, sizeof(packed));
        *reinterpret_cast<Raw*>(a.pyr + (bh * a.upper + a.level_off[l] + entry - 1) * D + lane * VE) = packed;
        if (l + 1 < NL) {
#pragma unroll
          for (int v = 0; v < VE; ++v) acc[l + 1][v] += acc[l][v];
        }
#pragma unroll
        for (int v = 0; v < VE; ++v) acc[l][v] = 0.0;
      }
    }
  }
}

template <int D>
cudaError_t launch_pool_keys_t(const PoolKArgs& a, unsigned blocks, cudaStream_t st) {
  switch (a.L) {
#define LH_CASE(n) \
  case n: pisa_pool_kernel<D, n><<<blocks, 256, 0, st>>>(a); break;
    LH_CASE(2) LH_CASE(3) LH_CASE(4) LH_CASE(5) LH_CASE(6) LH_CASE(7) LH_CASE(8)
#undef LH_CASE
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

lh_status fail(lh_status s, const char* what) {
  set_error_message("%s", what);
  return s;
}

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int log2_exact(int64_t x) {
  int r = 0;
  while (((int64_t)1 << r) < x) ++r;
  return ((int64_t)1 << r) == x ? r : -1;
}

lh_status pisa_plan_impl(const lh_pisa_config* cfg, lh_pisa_info* info) {
  if (!cfg || !info) return fail(LH_ERR_INVALID_ARG, "lh_pisa_plan: NULL argument");
  memset(info, 0, sizeof(*info));
  const int64_t B = cfg->B, H = cfg->H, N = cfg->N;
  const int d = cfg->d, p = cfg->p, L = cfg->L, C = cfg->block, G = cfg->group, K = cfg->topk;
  if (B < 1 || H < 1 || N < 1 || d < 1 || p < 1 || L < 1 || C < 1 || G < 1 || K < 1)
    return fail(LH_ERR_INVALID_ARG, "lh_pisa_plan: sizes must be positive");
  if (d != 64 && d != 128) return fail(LH_ERR_UNSUPPORTED, "lh_pisa_plan: d must be 64 or 128");
  if (C != 64 && C != 128) return fail(LH_ERR_UNSUPPORTED, "lh_pisa_plan: block must be 64 or 128");
  if (G != kG) return fail(LH_ERR_UNSUPPORTED, "lh_pisa_plan: group must be 128");
  const int log2p = log2_exact(p);
  if (p < 2 || log2p < 0) return fail(LH_ERR_UNSUPPORTED, "lh_pisa_plan: p must be a power of two >= 2");
  if (L > kMaxLevels) return fail(LH_ERR_UNSUPPORTED, "lh_pisa_plan: L must be <= 8");
  if (N >= ((int64_t)1 << 28)) return fail(LH_ERR_UNSUPPORTED, "lh_pisa_plan: N must be < 2^28");
  if (B * H > 65535) return fail(LH_ERR_UNSUPPORTED, "lh_pisa_plan: B*H must be <= 65535");
  if ((int64_t)(L - 1) * log2p + 7 >= 28) return fail(LH_ERR_UNSUPPORTED, "lh_pisa_plan: C p^(L-1) too large");
  const int64_t top_span = (int64_t)C << ((L - 1) * log2p);
  if (N % top_span != 0) return fail(LH_ERR_UNSUPPORTED, "lh_pisa_plan: N must be divisible by block * p^(L-1)");
  if (N % G != 0) return fail(LH_ERR_UNSUPPORTED, "lh_pisa_plan: N must be divisible by the group size");
  const int64_t n_top = N / top_span;
  if (n_top > kMaxCand) return fail(LH_ERR_UNSUPPORTED, "lh_pisa_plan: the coarsest level has more than 256 blocks");
  if ((int64_t)p * K > kMaxCand && L > 1)
    return fail(LH_ERR_UNSUPPORTED, "lh_pisa_plan: p * topk must be <= 256");
  int64_t upper = 0;
  for (int l = 0; l < L; ++l) {
    info->blocks[l] = (N >> (l * log2p)) / C;
    if (l >= 1) {
      info->level_off[l] = upper;
      upper += N >> (l * log2p);
    }
  }
  info->n_groups = N / G;
  info->upper_entries = upper;
  info->pyr_bytes = (size_t)(B * H) * upper * d * 2;
  info->kept_elems = (size_t)(B * H) * info->n_groups * L * K;
  info->max_candidates = (int32_t)(n_top > (int64_t)p * K ? n_top : (int64_t)p * K);
  return LH_OK;
}

template <int D, int C>
cudaError_t launch_select_t(dim3 grid, const CUtensorMap& mq, const CUtensorMap& mk0, const CUtensorMap& mku,
                            const PisaArgs& a, cudaStream_t st) {
  const int smem = PisaSmem<D, C>::kAlloc;
  cudaError_t e = cudaFuncSetAttribute(pisa_select_kernel<D, C>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  pisa_select_kernel<D, C><<<grid, kThreads, smem, st>>>(mq, mk0, mku, a);
  return cudaGetLastError();
}

}  // namespace
}  // namespace lh

using namespace lh;

extern "C" {

lh_status lh_pisa_plan(const lh_pisa_config* cfg, lh_pisa_info* info) { return pisa_plan_impl(cfg, info); }

lh_status lh_pisa_pool_keys(const lh_pisa_config* cfg, const void* k, void* kpyr, lh_stream_t stream) {
  lh_pisa_info info;
  lh_status s = pisa_plan_impl(cfg, &info);
  if (s != LH_OK) return s;
  if (cfg->L == 1) return LH_OK;
  if (!aligned16(k) || !aligned16(kpyr)) return fail(LH_ERR_INVALID_ARG, "lh_pisa_pool_keys: k or kpyr is NULL or not 16-byte aligned");
  PoolKArgs a{};
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.pyr = static_cast<__nv_bfloat16*>(kpyr);
  a.BH = cfg->B * cfg->H;
  a.N = cfg->N;
  a.upper = info.upper_entries;
  a.L = cfg->L;
  a.log2p = log2_exact(cfg->p);
  for (int l = 0; l < kMaxLevels; ++l) a.level_off[l] = info.level_off[l];
  const int64_t warps = a.BH * (a.N >> ((a.L - 1) * a.log2p));
  const unsigned blocks = (unsigned)((warps + 7) / 8);
  const cudaError_t e = cfg->d == 128 ? launch_pool_keys_t<128>(a, blocks, (cudaStream_t)stream)
                                      : launch_pool_keys_t<64>(a, blocks, (cudaStream_t)stream);
  if (e != cudaSuccess) {
    set_error_message("lh_pisa_pool_keys: %s", cudaGetErrorString(e));
    return LH_ERR_CUDA;
  }
  return LH_OK;
}

lh_status lh_pisa_select(const lh_pisa_config* cfg, const void* q, const void* k, const void* kpyr,
                         int32_t* kept_idx, float* kept_score, void* ws, lh_stream_t stream) {
  lh_pisa_info info;
  lh_status s = pisa_plan_impl(cfg, &info);
  if (s != LH_OK) return s;
  if (!aligned16(q) || !aligned16(k) || (cfg->L > 1 && !aligned16(kpyr)) || !aligned16(kept_idx) ||
      !aligned16(kept_score) || !aligned16(ws))
    return fail(LH_ERR_INVALID_ARG, "lh_pisa_select: a pointer is NULL or not 16-byte aligned");
  const int64_t BH = cfg->B * cfg->H;
  CUtensorMap mq, mk0, mku;
  const int C = cfg->block, d = cfg->d;
  if (!make_seq_map(&mq, q, BH, cfg->N, d, kG) || !make_seq_map(&mk0, k, BH, cfg->N, d, C) ||
      !make_seq_map(&mku, cfg->L > 1 ? kpyr : k, BH, cfg->L > 1 ? info.upper_entries : cfg->N, d, C))
    return fail(LH_ERR_CUDA, "lh_pisa_select: tensor map encoding failed");
  PisaArgs a{};
  a.N = (int)cfg->N;
  a.n_groups = (int)info.n_groups;
  a.L = cfg->L;
  a.log2p = log2_exact(cfg->p);
  a.K = cfg->topk;
  for (int l = 0; l < kMaxLevels; ++l) a.level_off[l] = (int)info.level_off[l];
  a.scale_log2 = (float)(1.4426950408889634 / sqrt((double)d));
  a.kept_idx = kept_idx;
  a.kept_score = kept_score;
  a.errw = static_cast<int*>(ws);
  const dim3 grid((unsigned)info.n_groups, (unsigned)BH);
  cudaError_t e;
  if (d == 128)
    e = C == 64 ? launch_select_t<128, 64>(grid, mq, mk0, mku, a, (cudaStream_t)stream)
                : launch_select_t<128, 128>(grid, mq, mk0, mku, a, (cudaStream_t)stream);
  else
    e = C == 64 ? launch_select_t<64, 64>(grid, mq, mk0, mku, a, (cudaStream_t)stream)
                : launch_select_t<64, 128>(grid, mq, mk0, mku, a, (cudaStream_t)stream);
  if (e != cudaSuccess) {
    set_error_message("lh_pisa_select: %s", cudaGetErrorString(e));
    return LH_ERR_CUDA;
  }
  return LH_OK;
}

}  // extern "C"
