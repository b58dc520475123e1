// C ABI of liblh: argument checks, planning of the buffers, and the stage and
// whole-layer entry points declared in include/lh.h.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "lh_common.cuh"

namespace lh {

static thread_local char g_msg[512] = "";

void set_error_message(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
}

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

lh_status fail(lh_status s, const char* what) {
  set_error_message("%s", what);
  return s;
}

lh_status cuda_fail(cudaError_t e, const char* where) {
  set_error_message("%s: %s", where, cudaGetErrorString(e));
  return LH_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int ilog2(int64_t x) {
  int r = 0;
  while (((int64_t)1 << r) < x) ++r;
  return r;
}

// fill the plan (sizes and offsets) of a validated configuration
lh_status plan_impl(const lh_config* cfg, lh_plan_info* info, Dims* D) {
  if (!cfg || !info) return fail(LH_ERR_INVALID_ARG, "lh_plan: NULL argument");
  memset(info, 0, sizeof(*info));
  const int64_t B = cfg->B, H = cfg->H, N = cfg->N;
  const int d = cfg->d, L = cfg->L, p = cfg->p, k = cfg->k;
  const int chunk = cfg->chunk == 0 ? 2048 : cfg->chunk;
  if (B < 1 || H < 1 || N < 1 || L < 1 || p < 1 || k < 1 || chunk < 1)
    return fail(LH_ERR_INVALID_ARG, "lh_plan: sizes must be positive");
  if (cfg->dtype != LH_BF16 && cfg->dtype != LH_FP32) return fail(LH_ERR_INVALID_ARG, "lh_plan: bad dtype");
  if (cfg->scorer < LH_SCORE_QK_SUM || cfg->scorer > LH_SCORE_Q) return fail(LH_ERR_INVALID_ARG, "lh_plan: bad scorer");
  if (cfg->selection < LH_SELECT_PARENTS || cfg->selection > LH_SELECT_NESTED)
    return fail(LH_ERR_INVALID_ARG, "lh_plan: bad selection");
  if (d != 64 && d != 128) return fail(LH_ERR_UNSUPPORTED, "lh_plan: d must be 64 or 128");
  if (p < 2 || (p & (p - 1)) != 0) return fail(LH_ERR_UNSUPPORTED, "lh_plan: p must be a power of two >= 2");
  if (L > 8) return fail(LH_ERR_UNSUPPORTED, "lh_plan: L must be <= 8");
  if (N >= ((int64_t)1 << 28)) return fail(LH_ERR_UNSUPPORTED, "lh_plan: N must be < 2^28");
  if (B * H > (int64_t)65535 * 65535 || H > 65535) return fail(LH_ERR_UNSUPPORTED, "lh_plan: too many heads");
  const int log2p = ilog2(p);
  if ((int64_t)(L - 1) * log2p >= 28) return fail(LH_ERR_UNSUPPORTED, "lh_plan: p^(L-1) too large");
  const int64_t ptop = (int64_t)1 << ((L - 1) * log2p);
  if (N % ptop != 0) return fail(LH_ERR_UNSUPPORTED, "lh_plan: N must be divisible by p^(L-1)");

  const int64_t BH = B * H;
  int64_t pyr = 0, upper = 0, selsum = 0;
  for (int l = 0; l < L; ++l) {
    info->level_len[l] = N >> (l * log2p);
    info->level_off[l] = pyr;
    pyr += info->level_len[l];
    if (l >= 1) {
      info->upper_off[l] = upper;
      upper += info->level_len[l];
    }
  }
  // k'_l = min(k, candidates): N/p^(l+1) (parents, direct), or the kept
  // entries of level l+1 (nested: the whole top level for l = L-2)
  const int sel_mode = cfg->selection;
  if (sel_mode == LH_SELECT_NESTED) {
    int64_t cand = info->level_len[L - 1];
    for (int l = L - 2; l >= 0; --l) {
      info->kprime[l] = (int32_t)(k < cand ? k : cand);
      cand = (int64_t)p * info->kprime[l];
    }
  } else {
    for (int l = 0; l + 1 < L; ++l) {
      const int64_t M = info->level_len[l + 1];
      info->kprime[l] = (int32_t)(k < M ? k : M);
    }
  }
  if (sel_mode == LH_SELECT_NESTED) {
    // the nested top-k stages every chunk of a level's candidates in shared memory
    for (int l = 0; l + 1 < L; ++l) {
      const int64_t M = l + 1 == L - 1 ? info->level_len[L - 1] : (int64_t)p * info->kprime[l + 1];
      const int64_t C = M / chunk > 1 ? M / chunk : 1;
      if ((M + C - 1) / C > 48 * 1024)
        return fail(LH_ERR_UNSUPPORTED, "lh_plan: nested selection needs chunks of at most 49152 candidates");
    }
  }
  // sel holds k'_l parents per level, or the p k'_l kept entries (direct)
  int64_t S = info->level_len[L - 1];
  for (int l = 0; l + 1 < L; ++l) {
    info->sel_off[l] = selsum;
    selsum += sel_mode == LH_SELECT_DIRECT ? (int64_t)p * info->kprime[l] : info->kprime[l];
    S += (int64_t)p * info->kprime[l];
  }
  if (S >= ((int64_t)1 << 31)) return fail(LH_ERR_UNSUPPORTED, "lh_plan: S too large");
  info->S = S;
  info->pyr_entries = pyr;
  info->upper_entries = upper;
  info->sel_per_head = selsum;

  const size_t e = cfg->dtype == LH_BF16 ? 2 : 4;
  info->pyr_bytes = (size_t)BH * upper * d * e;
  info->norms_bytes = (size_t)2 * BH * N * 4;
  // score pyramid (levels >= 1), plus the level-0 scores when level 0 is
  // selected directly
  info->topk_ws_bytes = LH_ERR_WORD_BYTES + align_up((size_t)BH * upper * 4) +
                        (sel_mode == LH_SELECT_DIRECT ? align_up((size_t)BH * N * 4) : 0);
  info->sel_bytes = (size_t)BH * selsum * 4;
  info->seq_bytes = (size_t)BH * S * d * 2;
  info->os_bytes = (size_t)BH * S * d * 4;
  info->seq_map_bytes = (size_t)BH * S * 4;
  info->slot_of_bytes = (size_t)BH * pyr * 4;
  info->lse_bytes = (size_t)BH * S * 4;
  info->grad_seq_bytes = (size_t)BH * S * d * 4;
  info->attn_bwd_ws_bytes = LH_ERR_WORD_BYTES;

  size_t off = 0;
  auto take = [&](size_t n) { const size_t o = off; off = align_up(off + n); return o; };
  info->ctx_off_sel = take(info->sel_bytes > 0 ? info->sel_bytes : 4);
  info->ctx_off_seq_map = take(info->seq_map_bytes);
  info->ctx_off_slot_of = take(info->slot_of_bytes);
  info->ctx_off_qs = take(info->seq_bytes);
  info->ctx_off_ks = take(info->seq_bytes);
  info->ctx_off_vs = take(info->seq_bytes);
  info->ctx_off_os = take(info->os_bytes);
  info->ctx_off_lse = take(info->lse_bytes);
  info->ctx_bytes = off;

  // forward scratch
  off = LH_ERR_WORD_BYTES;
  info->ws_off_pyr_q = take(info->pyr_bytes);
  info->ws_off_pyr_k = take(info->pyr_bytes);
  info->ws_off_pyr_v = take(info->pyr_bytes);
  info->ws_off_norms = take(info->norms_bytes);
  info->ws_off_topk = take(info->topk_ws_bytes);
  const size_t fwd = off;
  // backward scratch (overlaps the forward's)
  off = LH_ERR_WORD_BYTES;
  info->ws_off_dos = take(info->seq_bytes);
  info->ws_off_delta = take(info->lse_bytes);
  info->ws_off_dqs = take(info->grad_seq_bytes);
  info->ws_off_dks = take(info->grad_seq_bytes);
  info->ws_off_dvs = take(info->grad_seq_bytes);
  const size_t bwd = off;
  info->ws_bytes = fwd > bwd ? fwd : bwd;

  {
    Dims tmp;
    Dims* T = D ? D : &tmp;
    T->L = L; T->log2p = log2p;
    for (int l = 0; l < LH_MAX_LEVELS; ++l) {
      T->level_len[l] = info->level_len[l];
      T->kprime[l] = info->kprime[l];
    }
    info->first_level = materialized_level(*T);
  }
  if (D) {
    D->BH = BH; D->N = N; D->S = S;
    D->d = d; D->L = L; D->p = p; D->log2p = log2p; D->chunk = chunk;
    D->dtype = cfg->dtype; D->scorer = cfg->scorer; D->selection = cfg->selection;
    for (int l = 0; l < LH_MAX_LEVELS; ++l) {
      D->level_len[l] = info->level_len[l];
      D->level_off[l] = info->level_off[l];
      D->upper_off[l] = info->upper_off[l];
      D->kprime[l] = info->kprime[l];
      D->sel_off[l] = info->sel_off[l];
    }
    D->upper_entries = upper;
    D->pyr_entries = pyr;
    D->sel_per_head = selsum;
  }
  return LH_OK;
}

#define LH_CHECK_PTR(p)                                                           \
  do {                                                                            \
    if (!(p) || !aligned16(p)) return fail(LH_ERR_INVALID_ARG, #p " is NULL or not 16-byte aligned"); \
  } while (0)

#define LH_CUDA(call, where)                       \
  do {                                             \
    const cudaError_t e_ = (call);                 \
    if (e_ != cudaSuccess) return cuda_fail(e_, where); \
  } while (0)

int* err_word(void* ws) { return static_cast<int*>(ws); }

}  // namespace

lh_status make_dims(const lh_config* cfg, lh_plan_info* info, Dims* D) { return plan_impl(cfg, info, D); }

int materialized_level(const Dims& D) {
  // level l (< top) costs N/p^l rows to write whole, or p^(l+1) k' rows to
  // read back for its kept entries; coarser levels only favour writing more
  for (int l = 1; l < D.L - 1; ++l)
    if ((D.level_len[l]) <= ((int64_t)D.kprime[l] << ((l + 1) * D.log2p))) return l;
  return D.L > 1 ? D.L - 1 : 1;
}

}  // namespace lh

using namespace lh;

extern "C" {

lh_status lh_plan(const lh_config* cfg, lh_plan_info* info) { return plan_impl(cfg, info, nullptr); }

lh_status lh_pyramid_pool(const lh_config* cfg, const void* q, const void* k, const void* v, void* pyr_q,
                          void* pyr_k, void* pyr_v, float* norms, lh_stream_t stream) {
  lh_plan_info info;
  Dims D;
  lh_status s = plan_impl(cfg, &info, &D);
  if (s != LH_OK) return s;
  LH_CHECK_PTR(q); LH_CHECK_PTR(k); LH_CHECK_PTR(v); LH_CHECK_PTR(norms);
  if (D.L > 1) { LH_CHECK_PTR(pyr_q); LH_CHECK_PTR(pyr_k); LH_CHECK_PTR(pyr_v); }
  LH_CUDA(launch_pool(D, q, k, v, pyr_q, pyr_k, pyr_v, norms, nullptr, (cudaStream_t)stream), "lh_pyramid_pool");
  return LH_OK;
}

lh_status lh_pyramid_pool_from(const lh_config* cfg, int32_t first_level, const void* q, const void* k,
                               const void* v, void* pyr_q, void* pyr_k, void* pyr_v, float* norms,
                               lh_stream_t stream) {
  lh_plan_info info;
  Dims D;
  lh_status s = plan_impl(cfg, &info, &D);
  if (s != LH_OK) return s;
  if (first_level < 1 || first_level > (D.L > 1 ? D.L - 1 : 1))
    return fail(LH_ERR_INVALID_ARG, "lh_pyramid_pool_from: first_level outside [1, max(1, L-1)]");
  LH_CHECK_PTR(q); LH_CHECK_PTR(k); LH_CHECK_PTR(v); LH_CHECK_PTR(norms);
  if (D.L > 1) { LH_CHECK_PTR(pyr_q); LH_CHECK_PTR(pyr_k); LH_CHECK_PTR(pyr_v); }
  LH_CUDA(launch_pool(D, q, k, v, pyr_q, pyr_k, pyr_v, norms, nullptr, (cudaStream_t)stream, first_level),
          "lh_pyramid_pool_from");
  return LH_OK;
}

lh_status lh_score_topk(const lh_config* cfg, const float* norms, void* ws, int32_t* sel, lh_stream_t stream) {
  lh_plan_info info;
  Dims D;
  lh_status s = plan_impl(cfg, &info, &D);
  if (s != LH_OK) return s;
  if (D.L == 1) return LH_OK;
  LH_CHECK_PTR(norms); LH_CHECK_PTR(ws); LH_CHECK_PTR(sel);
  float* spyr = reinterpret_cast<float*>(static_cast<char*>(ws) + LH_ERR_WORD_BYTES);
  LH_CUDA(launch_score_topk(D, norms, spyr, sel, err_word(ws), (cudaStream_t)stream), "lh_score_topk");
  return LH_OK;
}

lh_status lh_gather(const lh_config* cfg, const void* q, const void* k, const void* v, const void* pyr_q,
                    const void* pyr_k, const void* pyr_v, const int32_t* sel, void* qs, void* ks, void* vs,
                    int32_t* seq_map, int32_t* slot_of, lh_stream_t stream) {
  lh_plan_info info;
  Dims D;
  lh_status s = plan_impl(cfg, &info, &D);
  if (s != LH_OK) return s;
  LH_CHECK_PTR(q); LH_CHECK_PTR(k); LH_CHECK_PTR(v);
  if (D.L > 1) { LH_CHECK_PTR(pyr_q); LH_CHECK_PTR(pyr_k); LH_CHECK_PTR(pyr_v); LH_CHECK_PTR(sel); }
  LH_CHECK_PTR(qs); LH_CHECK_PTR(ks); LH_CHECK_PTR(vs); LH_CHECK_PTR(seq_map); LH_CHECK_PTR(slot_of);
  LH_CUDA(launch_gather(D, q, k, v, pyr_q, pyr_k, pyr_v, sel, qs, ks, vs, seq_map, slot_of, nullptr,
                        (cudaStream_t)stream),
          "lh_gather");
  return LH_OK;
}

lh_status lh_gather_from(const lh_config* cfg, int32_t first_level, const void* q, const void* k, const void* v,
                         const void* pyr_q, const void* pyr_k, const void* pyr_v, const int32_t* sel, void* qs,
                         void* ks, void* vs, int32_t* seq_map, int32_t* slot_of, lh_stream_t stream) {
  lh_plan_info info;
  Dims D;
  lh_status s = plan_impl(cfg, &info, &D);
  if (s != LH_OK) return s;
  if (first_level < 1 || first_level > (D.L > 1 ? D.L - 1 : 1))
    return fail(LH_ERR_INVALID_ARG, "lh_gather_from: first_level outside [1, max(1, L-1)]");
  LH_CHECK_PTR(q); LH_CHECK_PTR(k); LH_CHECK_PTR(v);
  if (D.L > 1) { LH_CHECK_PTR(pyr_q); LH_CHECK_PTR(pyr_k); LH_CHECK_PTR(pyr_v); LH_CHECK_PTR(sel); }
  LH_CHECK_PTR(qs); LH_CHECK_PTR(ks); LH_CHECK_PTR(vs); LH_CHECK_PTR(seq_map); LH_CHECK_PTR(slot_of);
  LH_CUDA(launch_gather(D, q, k, v, pyr_q, pyr_k, pyr_v, sel, qs, ks, vs, seq_map, slot_of, nullptr,
                        (cudaStream_t)stream, first_level),
          "lh_gather_from");
  return LH_OK;
}

lh_status lh_attn_fwd(const lh_config* cfg, int64_t S, const void* qs, const void* ks, const void* vs, float* os,
                      float* lse, void* ws, lh_stream_t stream) {
  if (!cfg) return fail(LH_ERR_INVALID_ARG, "lh_attn_fwd: NULL cfg");
  if (cfg->B < 1 || cfg->H < 1 || S < 1) return fail(LH_ERR_INVALID_ARG, "lh_attn_fwd: sizes must be positive");
  if (cfg->d != 64 && cfg->d != 128) return fail(LH_ERR_UNSUPPORTED, "lh_attn_fwd: d must be 64 or 128");
  if (cfg->H > 65535 || cfg->B * cfg->H > 65535) return fail(LH_ERR_UNSUPPORTED, "lh_attn_fwd: B*H must be <= 65535");
  if (S >= ((int64_t)1 << 31)) return fail(LH_ERR_UNSUPPORTED, "lh_attn_fwd: S too large");
  LH_CHECK_PTR(qs); LH_CHECK_PTR(ks); LH_CHECK_PTR(vs); LH_CHECK_PTR(os); LH_CHECK_PTR(lse); LH_CHECK_PTR(ws);
  LH_CUDA(launch_attn_fwd(cfg->B * cfg->H, S, cfg->d, qs, ks, vs, os, lse, err_word(ws), (cudaStream_t)stream),
          "lh_attn_fwd");
  return LH_OK;
}

lh_status lh_attn_bwd(const lh_config* cfg, int64_t S, const void* qs, const void* ks, const void* vs,
                      const float* lse, const void* dos, const float* delta, float* dqs, float* dks, float* dvs,
                      void* ws, lh_stream_t stream) {
  if (!cfg) return fail(LH_ERR_INVALID_ARG, "lh_attn_bwd: NULL cfg");
  if (cfg->B < 1 || cfg->H < 1 || S < 1) return fail(LH_ERR_INVALID_ARG, "lh_attn_bwd: sizes must be positive");
  if (cfg->d != 64 && cfg->d != 128) return fail(LH_ERR_UNSUPPORTED, "lh_attn_bwd: d must be 64 or 128");
  if (cfg->H > 65535 || cfg->B * cfg->H > 65535) return fail(LH_ERR_UNSUPPORTED, "lh_attn_bwd: B*H must be <= 65535");
  if (S >= ((int64_t)1 << 31)) return fail(LH_ERR_UNSUPPORTED, "lh_attn_bwd: S too large");
  LH_CHECK_PTR(qs); LH_CHECK_PTR(ks); LH_CHECK_PTR(vs); LH_CHECK_PTR(lse); LH_CHECK_PTR(dos); LH_CHECK_PTR(delta);
  LH_CHECK_PTR(dqs); LH_CHECK_PTR(dks); LH_CHECK_PTR(dvs); LH_CHECK_PTR(ws);
  const int64_t BH = cfg->B * cfg->H;
  LH_CUDA(launch_attn_bwd(BH, S, cfg->d, qs, ks, vs, lse, dos, delta, dqs, dks, dvs, err_word(ws),
                          (cudaStream_t)stream),
          "lh_attn_bwd");
  return LH_OK;
}

lh_status lh_gather_shard(const lh_config* cfg, int64_t t0, int64_t t1, const int64_t* seg_off, int64_t seg_rows,
                         const void* q, const void* k, const void* v, const void* pyr_q, const void* pyr_k,
                         const void* pyr_v, const int32_t* sel, void* qs, void* ks, void* vs, int32_t* seq_map,
                         int32_t* slot_of, lh_stream_t stream) {
  lh_plan_info info;
  Dims D;
  lh_status s = plan_impl(cfg, &info, &D);
  if (s != LH_OK) return s;
  const int64_t ptop = (int64_t)1 << ((D.L - 1) * D.log2p);
  if (t0 < 0 || t1 > D.N || t0 >= t1 || t0 % ptop != 0 || t1 % ptop != 0)
    return fail(LH_ERR_INVALID_ARG, "lh_gather_shard: [t0, t1) must be a non-empty range of multiples of p^(L-1) in [0, N]");
  if (seg_rows < 1 || seg_rows > D.S) return fail(LH_ERR_INVALID_ARG, "lh_gather_shard: seg_rows outside [1, S]");
  // the shard's own plan: a layer of its t1 - t0 tokens
  lh_config sc = *cfg;
  sc.N = t1 - t0;
  lh_plan_info sinfo;
  Dims SD;
  s = plan_impl(&sc, &sinfo, &SD);
  if (s != LH_OK) return s;
  if (!seg_off) return fail(LH_ERR_INVALID_ARG, "lh_gather_shard: NULL seg_off");
  LH_CHECK_PTR(q); LH_CHECK_PTR(k); LH_CHECK_PTR(v);
  if (D.L > 1) { LH_CHECK_PTR(pyr_q); LH_CHECK_PTR(pyr_k); LH_CHECK_PTR(pyr_v); LH_CHECK_PTR(sel); }
  LH_CHECK_PTR(qs); LH_CHECK_PTR(ks); LH_CHECK_PTR(vs); LH_CHECK_PTR(seq_map); LH_CHECK_PTR(slot_of);
  LH_CUDA(launch_gather(D, q, k, v, pyr_q, pyr_k, pyr_v, sel, qs, ks, vs, seq_map, slot_of, nullptr,
                        (cudaStream_t)stream, 1, &SD, t0, seg_off, seg_rows),
          "lh_gather_shard");
  return LH_OK;
}

// the kernels' default bound on each of their waits, in SM clock cycles
// (about 2 s at the B200's 1965 MHz maximum)
constexpr long long kLaunchWaitCycles = 4000000000ll;

// a row window [lo, hi) of the sequence as 128-row tiles: lo a multiple of
// 128, hi a multiple of 128 or S
static bool tile_window(int64_t S, int64_t lo, int64_t hi, int64_t* t0, int64_t* t1) {
  if (lo < 0 || hi > S || lo > hi || lo % 128 != 0 || (hi % 128 != 0 && hi != S)) return false;
  *t0 = lo / 128;
  *t1 = (hi + 127) / 128;
  return true;
}

lh_status lh_attn_fwd_rows(const lh_config* cfg, int64_t S, int64_t row_lo, int64_t row_hi, const void* qs,
                           const void* ks, const void* vs, float* os, float* lse, void* ws, lh_stream_t stream) {
  if (!cfg) return fail(LH_ERR_INVALID_ARG, "lh_attn_fwd_rows: NULL cfg");
  if (cfg->B < 1 || cfg->H < 1 || S < 1) return fail(LH_ERR_INVALID_ARG, "lh_attn_fwd_rows: sizes must be positive");
  if (cfg->d != 64 && cfg->d != 128) return fail(LH_ERR_UNSUPPORTED, "lh_attn_fwd_rows: d must be 64 or 128");
  if (cfg->H > 65535 || cfg->B * cfg->H > 65535)
    return fail(LH_ERR_UNSUPPORTED, "lh_attn_fwd_rows: B*H must be <= 65535");
  if (S >= ((int64_t)1 << 31)) return fail(LH_ERR_UNSUPPORTED, "lh_attn_fwd_rows: S too large");
  int64_t t0, t1;
  if (!tile_window(S, row_lo, row_hi, &t0, &t1))
    return fail(LH_ERR_INVALID_ARG, "lh_attn_fwd_rows: rows must be [lo, hi) with lo % 128 == 0 and hi % 128 == 0 or S");
  if (t0 == t1) return LH_OK;
  LH_CHECK_PTR(qs); LH_CHECK_PTR(ks); LH_CHECK_PTR(vs); LH_CHECK_PTR(os); LH_CHECK_PTR(lse); LH_CHECK_PTR(ws);
  LH_CUDA(launch_attn_fwd(cfg->B * cfg->H, S, cfg->d, qs, ks, vs, os, lse, err_word(ws), (cudaStream_t)stream,
                          kLaunchWaitCycles, 1, t0, t1),
          "lh_attn_fwd_rows");
  return LH_OK;
}

lh_status lh_attn_bwd_rows(const lh_config* cfg, int64_t S, int64_t q_lo, int64_t q_hi, int64_t k_lo, int64_t k_hi,
                           const void* qs, const void* ks, const void* vs, const float* lse, const void* dos,
                           const float* delta, float* dqs, float* dks, float* dvs, void* ws, lh_stream_t stream) {
  if (!cfg) return fail(LH_ERR_INVALID_ARG, "lh_attn_bwd_rows: NULL cfg");
  if (cfg->B < 1 || cfg->H < 1 || S < 1) return fail(LH_ERR_INVALID_ARG, "lh_attn_bwd_rows: sizes must be positive");
  if (cfg->d != 64 && cfg->d != 128) return fail(LH_ERR_UNSUPPORTED, "lh_attn_bwd_rows: d must be 64 or 128");
  if (cfg->H > 65535 || cfg->B * cfg->H > 65535)
    return fail(LH_ERR_UNSUPPORTED, "lh_attn_bwd_rows: B*H must be <= 65535");
  if (S >= ((int64_t)1 << 31)) return fail(LH_ERR_UNSUPPORTED, "lh_attn_bwd_rows: S too large");
  int64_t qt0, qt1, kt0, kt1;
  if (!tile_window(S, q_lo, q_hi, &qt0, &qt1) || !tile_window(S, k_lo, k_hi, &kt0, &kt1))
    return fail(LH_ERR_INVALID_ARG, "lh_attn_bwd_rows: rows must be [lo, hi) with lo % 128 == 0 and hi % 128 == 0 or S");
  if (qt0 == qt1 && kt0 == kt1) return LH_OK;
  LH_CHECK_PTR(qs); LH_CHECK_PTR(ks); LH_CHECK_PTR(vs); LH_CHECK_PTR(lse); LH_CHECK_PTR(dos); LH_CHECK_PTR(delta);
  LH_CHECK_PTR(dqs); LH_CHECK_PTR(dks); LH_CHECK_PTR(dvs); LH_CHECK_PTR(ws);
  LH_CUDA(launch_attn_bwd(cfg->B * cfg->H, S, cfg->d, qs, ks, vs, lse, dos, delta, dqs, dks, dvs, err_word(ws),
                          (cudaStream_t)stream, qt0, qt1, kt0, kt1),
          "lh_attn_bwd_rows");
  return LH_OK;
}

lh_status lh_scatter_back(const lh_config* cfg, const float* os, const int32_t* slot_of, void* y,
                          lh_stream_t stream) {
  lh_plan_info info;
  Dims D;
  lh_status s = plan_impl(cfg, &info, &D);
  if (s != LH_OK) return s;
  LH_CHECK_PTR(os); LH_CHECK_PTR(slot_of); LH_CHECK_PTR(y);
  LH_CUDA(launch_scatter_back(D, os, slot_of, y, (cudaStream_t)stream), "lh_scatter_back");
  return LH_OK;
}

lh_status lh_scatter_back_adjoint(const lh_config* cfg, const void* dy, const int32_t* seq_map, const float* os,
                                  void* dos, float* delta, lh_stream_t stream) {
  lh_plan_info info;
  Dims D;
  lh_status s = plan_impl(cfg, &info, &D);
  if (s != LH_OK) return s;
  LH_CHECK_PTR(dy); LH_CHECK_PTR(seq_map); LH_CHECK_PTR(os); LH_CHECK_PTR(dos); LH_CHECK_PTR(delta);
  LH_CUDA(launch_scatter_adjoint(D, dy, seq_map, os, dos, delta, nullptr, (cudaStream_t)stream),
          "lh_scatter_back_adjoint");
  return LH_OK;
}

// the plan of one shard's layer (cfg->N = the shard's tokens) with its
// segment of seg_rows sequence rows per head in place of the plan's S
static lh_status shard_dims(const lh_config* cfg, int64_t seg_rows, Dims* D, const char* who) {
  lh_plan_info info;
  lh_status s = plan_impl(cfg, &info, D);
  if (s != LH_OK) return s;
  if (seg_rows < 1 || seg_rows >= ((int64_t)1 << 31)) return fail(LH_ERR_INVALID_ARG, who);
  D->S = seg_rows;
  return LH_OK;
}

lh_status lh_scatter_back_shard(const lh_config* cfg, int64_t seg_rows, const float* os, const int32_t* slot_of,
                                const float* halo, void* y, lh_stream_t stream) {
  Dims D;
  lh_status s = shard_dims(cfg, seg_rows, &D, "lh_scatter_back_shard: seg_rows outside [1, 2^31)");
  if (s != LH_OK) return s;
  if (D.dtype != LH_BF16 || D.d != 128)
    return fail(LH_ERR_UNSUPPORTED, "lh_scatter_back_shard: bf16 rows of 128 channels only");
  LH_CHECK_PTR(os); LH_CHECK_PTR(slot_of); LH_CHECK_PTR(y);
  if (D.L > 1) LH_CHECK_PTR(halo);
  LH_CUDA(launch_scatter_back(D, os, slot_of, y, (cudaStream_t)stream, D.L > 1 ? halo : nullptr),
          "lh_scatter_back_shard");
  return LH_OK;
}

lh_status lh_scatter_back_adjoint_shard(const lh_config* cfg, int64_t seg_rows, const void* dy,
                                        const int32_t* seq_map, const float* os, const float* halo, void* dos,
                                        float* delta, lh_stream_t stream) {
  Dims D;
  lh_status s = shard_dims(cfg, seg_rows, &D, "lh_scatter_back_adjoint_shard: seg_rows outside [1, 2^31)");
  if (s != LH_OK) return s;
  LH_CHECK_PTR(dy); LH_CHECK_PTR(seq_map); LH_CHECK_PTR(os); LH_CHECK_PTR(dos); LH_CHECK_PTR(delta);
  if (halo) LH_CHECK_PTR(halo);
  LH_CUDA(launch_scatter_adjoint(D, dy, seq_map, os, dos, delta, nullptr, (cudaStream_t)stream,
                                 D.L > 1 ? halo : nullptr),
          "lh_scatter_back_adjoint_shard");
  return LH_OK;
}

lh_status lh_pool_adjoint_shard(const lh_config* cfg, int64_t seg_rows, const float* dqs, const float* dks,
                                const float* dvs, const int32_t* slot_of, void* dq, void* dk, void* dv,
                                lh_stream_t stream) {
  Dims D;
  lh_status s = shard_dims(cfg, seg_rows, &D, "lh_pool_adjoint_shard: seg_rows outside [1, 2^31)");
  if (s != LH_OK) return s;
  LH_CHECK_PTR(dqs); LH_CHECK_PTR(dks); LH_CHECK_PTR(dvs); LH_CHECK_PTR(slot_of);
  LH_CHECK_PTR(dq); LH_CHECK_PTR(dk); LH_CHECK_PTR(dv);
  LH_CUDA(launch_pool_adjoint(D, dqs, dks, dvs, slot_of, dq, dk, dv, (cudaStream_t)stream), "lh_pool_adjoint_shard");
  return LH_OK;
}

lh_status lh_head_sums(const lh_config* cfg, const void* dy, float* sums, lh_stream_t stream) {
  lh_plan_info info;
  Dims D;
  lh_status s = plan_impl(cfg, &info, &D);
  if (s != LH_OK) return s;
  if (D.L < 2) return LH_OK;
  LH_CHECK_PTR(dy); LH_CHECK_PTR(sums);
  LH_CUDA(launch_head_sums(D, dy, sums, (cudaStream_t)stream), "lh_head_sums");
  return LH_OK;
}

lh_status lh_pool_adjoint(const lh_config* cfg, const float* dqs, const float* dks, const float* dvs,
                          const int32_t* slot_of, void* dq, void* dk, void* dv, lh_stream_t stream) {
  lh_plan_info info;
  Dims D;
  lh_status s = plan_impl(cfg, &info, &D);
  if (s != LH_OK) return s;
  LH_CHECK_PTR(dqs); LH_CHECK_PTR(dks); LH_CHECK_PTR(dvs); LH_CHECK_PTR(slot_of);
  LH_CHECK_PTR(dq); LH_CHECK_PTR(dk); LH_CHECK_PTR(dv);
  LH_CUDA(launch_pool_adjoint(D, dqs, dks, dvs, slot_of, dq, dk, dv, (cudaStream_t)stream), "lh_pool_adjoint");
  return LH_OK;
}

lh_status lh_forward(const lh_config* cfg, const void* q, const void* k, const void* v, void* y, void* ctx,
                     size_t ctx_bytes, void* ws, size_t ws_bytes, lh_stream_t stream) {
  lh_plan_info I;
  Dims D;
  lh_status s = plan_impl(cfg, &I, &D);
  if (s != LH_OK) return s;
  LH_CHECK_PTR(q); LH_CHECK_PTR(k); LH_CHECK_PTR(v); LH_CHECK_PTR(y); LH_CHECK_PTR(ctx); LH_CHECK_PTR(ws);
  if (ctx_bytes < I.ctx_bytes || ws_bytes < I.ws_bytes) return fail(LH_ERR_WORKSPACE, "lh_forward: ctx or ws too small");
  const cudaStream_t st = (cudaStream_t)stream;
  char* c = static_cast<char*>(ctx);
  char* w = static_cast<char*>(ws);
  int* errw = err_word(ws);
  LH_CUDA(cudaMemsetAsync(errw, 0, sizeof(int), st), "lh_forward");
  void* pq = w + I.ws_off_pyr_q;
  void* pk = w + I.ws_off_pyr_k;
  void* pv = w + I.ws_off_pyr_v;
  float* norms = reinterpret_cast<float*>(w + I.ws_off_norms);
  float* spyr = reinterpret_cast<float*>(w + I.ws_off_topk + LH_ERR_WORD_BYTES);
  int32_t* sel = reinterpret_cast<int32_t*>(c + I.ctx_off_sel);
  int32_t* seq_map = reinterpret_cast<int32_t*>(c + I.ctx_off_seq_map);
  int32_t* slot_of = reinterpret_cast<int32_t*>(c + I.ctx_off_slot_of);
  void* qs = c + I.ctx_off_qs;
  void* ks = c + I.ctx_off_ks;
  void* vs = c + I.ctx_off_vs;
  float* os = reinterpret_cast<float*>(c + I.ctx_off_os);
  float* lse = reinterpret_cast<float*>(c + I.ctx_off_lse);
  const int first = I.first_level;
  LH_CUDA(launch_pool(D, q, k, v, pq, pk, pv, norms, errw, st, first), "lh_forward: pool");
  LH_CUDA(launch_score_topk(D, norms, spyr, sel, errw, st), "lh_forward: score_topk");
  LH_CUDA(launch_gather(D, q, k, v, pq, pk, pv, sel, qs, ks, vs, seq_map, slot_of, errw, st, first),
          "lh_forward: gather");
  LH_CUDA(launch_attn_fwd(D.BH, D.S, D.d, qs, ks, vs, os, lse, errw, st), "lh_forward: attn_fwd");
  LH_CUDA(launch_scatter_back(D, os, slot_of, y, st), "lh_forward: scatter_back");
  return LH_OK;
}

lh_status lh_backward(const lh_config* cfg, const void* dy, const void* ctx, size_t ctx_bytes, void* dq,
                      void* dk, void* dv, void* ws, size_t ws_bytes, lh_stream_t stream) {
  lh_plan_info I;
  Dims D;
  lh_status s = plan_impl(cfg, &I, &D);
  if (s != LH_OK) return s;
  LH_CHECK_PTR(dy); LH_CHECK_PTR(ctx); LH_CHECK_PTR(dq); LH_CHECK_PTR(dk); LH_CHECK_PTR(dv); LH_CHECK_PTR(ws);
  if (ctx_bytes < I.ctx_bytes || ws_bytes < I.ws_bytes) return fail(LH_ERR_WORKSPACE, "lh_backward: ctx or ws too small");
  const cudaStream_t st = (cudaStream_t)stream;
  const char* c = static_cast<const char*>(ctx);
  char* w = static_cast<char*>(ws);
  int* errw = err_word(ws);
  LH_CUDA(cudaMemsetAsync(errw, 0, sizeof(int), st), "lh_backward");
  const int32_t* seq_map = reinterpret_cast<const int32_t*>(c + I.ctx_off_seq_map);
  const int32_t* slot_of = reinterpret_cast<const int32_t*>(c + I.ctx_off_slot_of);
  const void* qs = c + I.ctx_off_qs;
  const void* ks = c + I.ctx_off_ks;
  const void* vs = c + I.ctx_off_vs;
  const float* os = reinterpret_cast<const float*>(c + I.ctx_off_os);
  const float* lse = reinterpret_cast<const float*>(c + I.ctx_off_lse);
  void* dos = w + I.ws_off_dos;
  float* delta = reinterpret_cast<float*>(w + I.ws_off_delta);
  float* dqs = reinterpret_cast<float*>(w + I.ws_off_dqs);
  float* dks = reinterpret_cast<float*>(w + I.ws_off_dks);
  float* dvs = reinterpret_cast<float*>(w + I.ws_off_dvs);
  LH_CUDA(launch_scatter_adjoint(D, dy, seq_map, os, dos, delta, errw, st), "lh_backward: scatter_adjoint");
  LH_CUDA(launch_attn_bwd(D.BH, D.S, D.d, qs, ks, vs, lse, dos, delta, dqs, dks, dvs, errw, st),
          "lh_backward: attn_bwd");
  LH_CUDA(launch_pool_adjoint(D, dqs, dks, dvs, slot_of, dq, dk, dv, st), "lh_backward: pool_adjoint");
  return LH_OK;
}

lh_status lh_selftest_wait_timeout(void* ws, size_t ws_bytes, int64_t wait_cycles, lh_stream_t stream) {
  LH_CHECK_PTR(ws);
  if (ws_bytes < LH_SELFTEST_WS_BYTES)
    return fail(LH_ERR_WORKSPACE, "lh_selftest_wait_timeout: ws smaller than LH_SELFTEST_WS_BYTES");
  if (wait_cycles < 1 || wait_cycles > kLaunchWaitCycles)
    return fail(LH_ERR_INVALID_ARG, "lh_selftest_wait_timeout: wait_cycles outside [1, 4e9]");
  // one 128 x 64 tile each of Qs, Ks, Vs (bf16, 16 KB) after the error word,
  // then O (fp32, 32 KB) and LSE (512 B): 256 + 3 * 16384 + 32768 + 512 bytes
  char* w = static_cast<char*>(ws);
  const int64_t S = 128;
  const int d = 64;
  void* qs = w + LH_ERR_WORD_BYTES;
  void* ks = w + LH_ERR_WORD_BYTES + 16384;
  void* vs = w + LH_ERR_WORD_BYTES + 2 * 16384;
  float* os = reinterpret_cast<float*>(w + LH_ERR_WORD_BYTES + 3 * 16384);
  float* lse = reinterpret_cast<float*>(w + LH_ERR_WORD_BYTES + 3 * 16384 + 32768);
  LH_CUDA(launch_attn_fwd(1, S, d, qs, ks, vs, os, lse, err_word(ws), (cudaStream_t)stream, (long long)wait_cycles,
                          /*issue_loads=*/0),
          "lh_selftest_wait_timeout");
  return LH_OK;
}

lh_status lh_check_error(void* ws, lh_stream_t stream) {
  if (!ws) return fail(LH_ERR_INVALID_ARG, "lh_check_error: NULL ws");
  const cudaStream_t st = (cudaStream_t)stream;
  LH_CUDA(cudaStreamSynchronize(st), "lh_check_error");
  int word = 0;
  LH_CUDA(cudaMemcpy(&word, ws, sizeof(int), cudaMemcpyDeviceToHost), "lh_check_error");
  LH_CUDA(cudaMemset(ws, 0, sizeof(int)), "lh_check_error");
  if (word & ERRW_TIMEOUT) return fail(LH_ERR_TIMEOUT, "a bounded device wait ran out");
  if (word & ERRW_BOUNDS) return fail(LH_ERR_DEVICE, "a device-side index check failed");
  if (word & ERRW_RANGE) return fail(LH_ERR_DEVICE, "a value kept in fp16 by the backward (dOs or Vs) exceeds 65504");
  return LH_OK;
}

lh_status lh_clear_error(void* ws, lh_stream_t stream) {
  if (!ws) return fail(LH_ERR_INVALID_ARG, "lh_clear_error: NULL ws");
  LH_CUDA(cudaMemsetAsync(ws, 0, sizeof(int), (cudaStream_t)stream), "lh_clear_error");
  return LH_OK;
}

const char* lh_status_string(lh_status status) {
  switch (status) {
    case LH_OK: return "ok";
    case LH_ERR_INVALID_ARG: return "invalid argument";
    case LH_ERR_UNSUPPORTED: return "unsupported configuration";
    case LH_ERR_WORKSPACE: return "workspace too small";
    case LH_ERR_CUDA: return "CUDA error";
    case LH_ERR_TIMEOUT: return "device wait timed out";
    case LH_ERR_DEVICE: return "device-side check failed";
  }
  return "unknown status";
}

const char* lh_last_error_message(void) { return g_msg; }

}  // extern "C"
