// Stage 2: max-pooled score pyramid and stratified chunked top-k.
//
// Level-0 scores come from ||Q_t||_2 and ||K_t||_2 and coarser levels take the
// max over their p children (aitrends.kr summary, Technical details (2)).
// The top-k is stratified: every interval of candidates contributes a fixed
// number (techllm post, Limitations and caveats, stratified top-K bullet).
//
// Selection here is an exact radix select on the fp32 score bits (scores are
// non-negative, so the bit patterns order like the values) followed by an
// ordered compaction, so ties go to the lower index and the output is already
// in ascending order.
#include "lh_common.cuh"

namespace lh {
namespace {

constexpr int kScoreTile = 2048;
constexpr int kScoreThreads = 256;
constexpr int kTopkThreads = 512;

struct ScoreArgs {
  const float* norms;  // [2][BH][N]
  float* spyr;         // [BH][upper_entries]
  float* s0;           // [BH][N] level-0 scores, written when levels are selected directly (else null)
  int64_t BH, N, upper_entries;
  int64_t upper_off[LH_MAX_LEVELS];
  int64_t level_len[LH_MAX_LEVELS];
  int src_level, n_levels, log2p, scorer;
};

__device__ __forceinline__ float level0_score(float nq, float nk, int scorer) {
  return scorer == LH_SCORE_QK_SUM ? nq + nk : (scorer == LH_SCORE_K ? nk : nq);
}

// One block max-pools a tile of kScoreTile source entries through n_levels levels.
__global__ void __launch_bounds__(kScoreThreads) score_pyramid_kernel(ScoreArgs a) {
  __shared__ float buf[2][kScoreTile];
  const int64_t bh = blockIdx.y;
  const int64_t start = (int64_t)blockIdx.x * kScoreTile;
  const int64_t n_src = a.level_len[a.src_level];
  const int n = (int)min((int64_t)kScoreTile, n_src - start);
  for (int i = threadIdx.x; i < n; i += kScoreThreads) {
    float s;
    if (a.src_level == 0) {
      const float nq = a.norms[bh * a.N + start + i];
      const float nk = a.norms[(a.BH + bh) * a.N + start + i];
      s = level0_score(nq, nk, a.scorer);
      if (a.s0) a.s0[bh * a.N + start + i] = s;
    } else {
      s = a.spyr[bh * a.upper_entries + a.upper_off[a.src_level] + start + i];
    }
    buf[0][i] = s;
  }
  __syncthreads();
  const int p = 1 << a.log2p;
  int cur = 0, cnt = n;
  for (int j = 1; j <= a.n_levels; ++j) {
    const int cnt_out = cnt >> a.log2p;
    const int lvl = a.src_level + j;
    float* out = a.spyr + bh * a.upper_entries + a.upper_off[lvl] + (start >> (j * a.log2p));
    for (int i = threadIdx.x; i < cnt_out; i += kScoreThreads) {
      float m = buf[cur][i * p];
      for (int c = 1; c < p; ++c) m = fmaxf(m, buf[cur][i * p + c]);
      buf[cur ^ 1][i] = m;
      out[i] = m;
    }
    __syncthreads();
    cur ^= 1;
    cnt = cnt_out;
  }
}

struct TopkArgs {
  const float* spyr;
  const float* s0;  // level-0 scores (direct selection of level 0)
  int32_t* sel;
  int64_t N, upper_entries, sel_per_head;
  int64_t level_len[LH_MAX_LEVELS];
  int64_t upper_off[LH_MAX_LEVELS];
  int64_t sel_off[LH_MAX_LEVELS];
  int32_t kprime[LH_MAX_LEVELS];
  // per selection level l: the candidates are cand_len[l] contiguous scores at
  // src_off[l] of the head's score pyramid (or the level-0 scores when
  // src_off[l] < 0); budget[l] of them are kept
  int64_t cand_len[LH_MAX_LEVELS];
  int64_t src_off[LH_MAX_LEVELS];
  int32_t budget[LH_MAX_LEVELS];
  int32_t chunks[LH_MAX_LEVELS];
  int32_t chunk_prefix[LH_MAX_LEVELS + 1];
  int L, log2p, chunk;
  int smem_keys;  // chunks up to this size are staged in shared memory
};

// exclusive scan of one int per thread over the block; returns the block total in *total
__device__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int nw = kTopkThreads / 32;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) warp_sums[lane] = w;  // inclusive
  }
  __syncthreads();
  const int before = (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
  *total = warp_sums[nw - 1];
  __syncthreads();
  return before;
}

struct SelectShared {
  uint32_t hist[256];
  uint32_t prefix, remaining;
  int warp_sums[kTopkThreads / 32];
};

// The q largest of K[0..size) (fp32 score bits: non-negative, so the bits
// order like the values), ties to the lower position: an exact radix select
// of the q-th largest key, 8 bits per pass from the top, then an ordered
// compaction.  emit(rank, pos) is called for the kept positions with ranks
// 0..q-1 in ascending position order.  Called by the whole block.
template <class Emit>
__device__ void select_top(const uint32_t* K, int size, int q, SelectShared& sh, Emit emit) {
  uint32_t prefix = 0, mask = 0, remaining = (uint32_t)q;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    if (threadIdx.x < 256) sh.hist[threadIdx.x] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < size; i += kTopkThreads) {
      const uint32_t k = K[i];
      if ((k & mask) == prefix) atomicAdd(&sh.hist[(k >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      uint32_t local = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) local += sh.hist[255 - 8 * lane - j];
      uint32_t incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t before = incl - local;
      if (before < remaining && remaining <= incl) {
        uint32_t run = before;
        for (int j = 0; j < 8; ++j) {
          const uint32_t bin = 255u - 8u * lane - j;
          const uint32_t h = sh.hist[bin];
          if (run + h >= remaining) {
            sh.prefix = prefix | (bin << shift);
            sh.remaining = remaining - run;
            break;
          }
          run += h;
        }
      }
    }
    __syncthreads();
    prefix = sh.prefix;
    remaining = sh.remaining;
    mask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t tau = prefix;
  const int need_eq = (int)remaining;

  // ordered compaction: each thread owns a contiguous segment
  const int seg = (size + kTopkThreads - 1) / kTopkThreads;
  const int i0 = min(size, (int)threadIdx.x * seg), i1 = min(size, i0 + seg);
  int n_eq = 0;
  for (int i = i0; i < i1; ++i) n_eq += K[i] == tau;
  int tot;
  const int eq_rank = block_exclusive_scan(n_eq, sh.warp_sums, &tot);
  int n_sel = 0;
  {
    int r = eq_rank;
    for (int i = i0; i < i1; ++i) {
      const uint32_t k = K[i];
      if (k > tau) ++n_sel;
      else if (k == tau) { n_sel += r < need_eq; ++r; }
    }
  }
  int pos = block_exclusive_scan(n_sel, sh.warp_sums, &tot);
  {
    int r = eq_rank;
    for (int i = i0; i < i1; ++i) {
      const uint32_t k = K[i];
      bool take = false;
      if (k > tau) take = true;
      else if (k == tau) { take = r < need_eq; ++r; }
      if (take) emit(pos++, i);
    }
  }
}

// chunk c of C over M candidates: [start, start + size), quota q of budget kp
__device__ __forceinline__ void chunk_of(int64_t M, int C, int kp, int c, int64_t& start, int& size, int& q) {
  const int64_t base = M / C, extra = M % C;
  start = c * base + min((int64_t)c, extra);
  size = (int)(base + (c < extra ? 1 : 0));
  q = kp / C + (c < kp % C ? 1 : 0);
}

// One block per (head, selection level, chunk) of contiguous candidates
// (the parents and direct readings).
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(TopkArgs a) {
  extern __shared__ uint32_t keys[];
  __shared__ SelectShared sh;
  const int64_t bh = blockIdx.y;
  const int b = blockIdx.x;
  int l = 0;
  while (l + 1 < a.L - 1 && b >= a.chunk_prefix[l + 1]) ++l;
  const int c = b - a.chunk_prefix[l];
  const int kp = a.budget[l];
  int64_t start;
  int size, q;
  chunk_of(a.cand_len[l], a.chunks[l], kp, c, start, size, q);
  const int C = a.chunks[l];
  int32_t* out = a.sel + bh * a.sel_per_head + a.sel_off[l] + (int64_t)c * (kp / C) + min(c, kp % C);
  const float* src =
      (a.src_off[l] < 0 ? a.s0 + bh * a.N : a.spyr + bh * a.upper_entries + a.src_off[l]) + start;
  if (q <= 0) return;
  if (q >= size) {
    for (int i = threadIdx.x; i < size; i += kTopkThreads) out[i] = (int32_t)(start + i);
    return;
  }
  // a chunk that fits the dynamic shared memory is staged there; a larger one
  // (a global top-k over a whole level) is read from the score pyramid in
  // every pass, where it stays L2-resident
  const bool staged = size <= a.smem_keys;
  const uint32_t* K = staged ? keys : reinterpret_cast<const uint32_t*>(src);
  if (staged)
    for (int i = threadIdx.x; i < size; i += kTopkThreads) keys[i] = __float_as_uint(src[i]);
  __syncthreads();
  select_top(K, size, q, sh, [&](int rank, int pos) { out[rank] = (int32_t)(start + pos); });
}

// The nested reading: one block per head walks the levels from the top down;
// the candidates of level l+1 are the entries kept there (the whole top
// level, or the p children of every parent chosen one step earlier, in
// ascending order), chunked by their position in that list.
__global__ void __launch_bounds__(kTopkThreads) nested_topk_kernel(TopkArgs a, int* errw) {
  extern __shared__ uint32_t keys[];
  __shared__ SelectShared sh;
  const int64_t bh = blockIdx.y;
  int32_t* sel_h = a.sel + bh * a.sel_per_head;
  const int p = 1 << a.log2p;
  for (int l = a.L - 2; l >= 0; --l) {
    const bool top = l + 1 == a.L - 1;
    const int64_t M = top ? a.level_len[a.L - 1] : (int64_t)p * a.kprime[l + 1];
    const int32_t* up = sel_h + a.sel_off[l + 1];
    auto cand = [&](int64_t i) -> int64_t { return top ? i : ((int64_t)up[i >> a.log2p] << a.log2p) + (i & (p - 1)); };
    const float* scores = a.spyr + bh * a.upper_entries + a.upper_off[l + 1];
    const int kp = a.kprime[l];
    const int C = (int)(M / a.chunk > 1 ? M / a.chunk : 1);
    for (int c = 0; c < C; ++c) {
      int64_t start;
      int size, q;
      chunk_of(M, C, kp, c, start, size, q);
      int32_t* out = sel_h + a.sel_off[l] + (int64_t)c * (kp / C) + min(c, kp % C);
      if (q <= 0) continue;
      if (q >= size) {
        for (int i = threadIdx.x; i < size; i += kTopkThreads) out[i] = (int32_t)cand(start + i);
        continue;
      }
      if (size > a.smem_keys) {  // the plan keeps nested chunks within the staging buffer
        if (threadIdx.x == 0) report_error(errw, ERRW_BOUNDS);
        return;
      }
      for (int i = threadIdx.x; i < size; i += kTopkThreads) keys[i] = __float_as_uint(scores[cand(start + i)]);
      __syncthreads();
      select_top(keys, size, q, sh, [&](int rank, int pos) { out[rank] = (int32_t)cand(start + pos); });
      __syncthreads();
    }
    __syncthreads();  // this level's parents are written before the next level reads them
  }
}

}  // namespace

cudaError_t launch_score_topk(const Dims& D, const float* norms, float* spyr, int32_t* sel, int* errw,
                              cudaStream_t st) {
  if (D.L < 2) return cudaSuccess;
  const bool direct = D.selection == LH_SELECT_DIRECT, nested = D.selection == LH_SELECT_NESTED;
  // the level-0 scores follow the score pyramid (256-byte aligned) when level 0 is selected directly
  float* s0 = direct ? spyr + (((size_t)D.BH * D.upper_entries * 4 + 255) & ~(size_t)255) / 4 : nullptr;
  ScoreArgs s{};
  s.norms = norms;
  s.spyr = spyr;
  s.s0 = s0;
  s.BH = D.BH; s.N = D.N; s.upper_entries = D.upper_entries;
  for (int l = 0; l < LH_MAX_LEVELS; ++l) { s.upper_off[l] = D.upper_off[l]; s.level_len[l] = D.level_len[l]; }
  s.log2p = D.log2p;
  s.scorer = D.scorer;
  int per_launch = 0;
  while ((1 << ((per_launch + 1) * D.log2p)) <= kScoreTile) ++per_launch;
  for (int src = 0; src < D.L - 1; src += per_launch) {
    s.src_level = src;
    s.n_levels = (D.L - 1 - src) < per_launch ? (D.L - 1 - src) : per_launch;
    const int64_t tiles = (D.level_len[src] + kScoreTile - 1) / kScoreTile;
    score_pyramid_kernel<<<dim3((unsigned)tiles, (unsigned)D.BH), kScoreThreads, 0, st>>>(s);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    s.s0 = nullptr;  // written by the first launch only
  }
  TopkArgs t{};
  t.spyr = spyr;
  t.s0 = s0;
  t.sel = sel;
  t.N = D.N;
  t.upper_entries = D.upper_entries;
  t.sel_per_head = D.sel_per_head;
  for (int l = 0; l < LH_MAX_LEVELS; ++l) {
    t.upper_off[l] = D.upper_off[l];
    t.level_len[l] = D.level_len[l];
    t.sel_off[l] = D.sel_off[l];
    t.kprime[l] = D.kprime[l];
  }
  t.L = D.L;
  t.log2p = D.log2p;
  t.chunk = D.chunk;
  constexpr int64_t kSmemKeys = 48 * 1024;  // 192 KB of staged keys
  t.smem_keys = (int)kSmemKeys;
  int total = 0;
  t.chunk_prefix[0] = 0;
  int64_t max_size = 1;
  for (int l = 0; l < D.L - 1; ++l) {
    // parents: the N/p^(l+1) entries of level l+1; direct: the N/p^l of level l;
    // nested: the kept entries of level l+1
    int64_t M;
    if (nested) M = l + 1 == D.L - 1 ? D.level_len[D.L - 1] : ((int64_t)D.kprime[l + 1] << D.log2p);
    else M = direct ? D.level_len[l] : D.level_len[l + 1];
    t.cand_len[l] = M;
    t.budget[l] = direct ? (D.kprime[l] << D.log2p) : D.kprime[l];
    t.src_off[l] = direct ? (l == 0 ? -1 : D.upper_off[l]) : D.upper_off[l + 1];
    const int64_t C = M / D.chunk > 1 ? M / D.chunk : 1;
    t.chunks[l] = (int32_t)C;
    total += (int)C;
    t.chunk_prefix[l + 1] = total;
    const int64_t sz = M / C + (M % C ? 1 : 0);
    if (sz > max_size) max_size = sz;
  }
  const size_t smem = (size_t)(max_size < kSmemKeys ? max_size : kSmemKeys) * sizeof(uint32_t);
  if (nested) {
    if (smem > 48 * 1024) {
      const cudaError_t e =
          cudaFuncSetAttribute(nested_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
    }
    nested_topk_kernel<<<dim3(1, (unsigned)D.BH), kTopkThreads, smem, st>>>(t, errw);
    return cudaGetLastError();
  }
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  topk_kernel<<<dim3((unsigned)total, (unsigned)D.BH), kTopkThreads, smem, st>>>(t);
  return cudaGetLastError();
}

}  // namespace lh
