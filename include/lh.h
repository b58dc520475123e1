/*
 * lh.h - C ABI of liblh, one Lighthouse attention layer (forward and backward)
 * on an NVIDIA B200 (sm_100a).
 *
 * Lighthouse Attention (arXiv:2605.06554) wraps an unmodified causal attention
 * in four stages.  Citations below name the two pages that describe it:
 *   LH-summary: the aitrends.kr summary of Lighthouse Attention
 *               ("Method", "Technical details" (1)-(4)).
 *   LH-post:    the techllm.github.io post "Lighthouse Attention: long-context
 *               pretraining" ("How it works" (1)-(4), "Key formulas").
 *
 * Conventions shared by every call
 *  - Ownership: the caller allocates and frees every buffer.  liblh never
 *    allocates device memory, never frees, and never synchronises a stream,
 *    except lh_check_error.  All calls are asynchronous on `stream`.
 *  - Pointers are device pointers (cudaMalloc / torch CUDA tensors) unless a
 *    parameter says "host", and must be 16-byte aligned.
 *  - Layouts are dense row-major.  "BH" = B*H flattened; Q, K, V, Y, dY, dQ,
 *    dK, dV are [B][H][N][d] in cfg->dtype.  The gathered sequence tensors
 *    Qs, Ks, Vs are [BH][S][d] bf16, dOs [BH][S][d] fp16 (holding bf16
 *    values); Os, dQs, dKs, dVs are [BH][S][d]
 *    fp32; LSE and Delta are [BH][S] fp32.
 *  - Support: d in {64, 128}; p a power of two >= 2; 1 <= L <= 8;
 *    N divisible by p^(L-1); N < 2^28; k >= 1; B*H <= 65535 * 65535.
 *    dtype LH_FP32 pools and scores in fp32 and casts the gathered sequence
 *    to bf16 for the tensor cores.
 *  - Errors: argument checks run on the host and return a status at once
 *    (no work is queued).  A failed launch returns LH_ERR_CUDA; details are
 *    in lh_last_error_message().  Device-side problems (a bounded wait that
 *    ran out, an index out of range) set the error word held in the first
 *    LH_ERR_WORD_BYTES bytes of `ws`; lh_check_error reports and clears it.
 *  - Re-entrancy: no global state except the per-thread error message; calls
 *    on different streams are independent when each has its own ws and ctx.
 */
#ifndef LH_H
#define LH_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* a cudaStream_t; NULL is the legacy default stream */
typedef struct CUstream_st *lh_stream_t;

typedef enum {
  LH_OK = 0,
  LH_ERR_INVALID_ARG = 1,  /* NULL or misaligned pointer, negative size, bad enum */
  LH_ERR_UNSUPPORTED = 2,  /* valid but outside the support list above */
  LH_ERR_WORKSPACE = 3,    /* ctx_bytes or ws_bytes smaller than lh_plan asks */
  LH_ERR_CUDA = 4,         /* a CUDA runtime call failed */
  LH_ERR_TIMEOUT = 5,      /* a bounded device wait ran out (from lh_check_error) */
  LH_ERR_DEVICE = 6        /* a device-side index check failed (from lh_check_error) */
} lh_status;

typedef enum { LH_BF16 = 0, LH_FP32 = 1 } lh_dtype;

/* Level-0 score s0_t from the l2 norms of Q_t and K_t (LH-summary
 * "Technical details" (2): ||Q_i||_2, ||K_i||_2 are the scores at level 0). */
typedef enum {
  LH_SCORE_QK_SUM = 0, /* ||Q_t|| + ||K_t|| */
  LH_SCORE_K = 1,      /* ||K_t||  (the "projection-norm" scorer) */
  LH_SCORE_Q = 2       /* ||Q_t|| */
} lh_scorer;

/* What a level below the top keeps (the pages fix only the count p*k per
 * level: LH-post "Key formulas"; these are the three readings of it). */
typedef enum {
  LH_SELECT_PARENTS = 0, /* k' parents at level l+1 by max-pooled score, each with its p children (default) */
  LH_SELECT_DIRECT = 1,  /* p*k' entries of level l by their own score */
  LH_SELECT_NESTED = 2   /* as PARENTS, parents only among the entries kept at level l+1 (the whole
                            top level for l = L-2); k' = min(k, candidates) */
} lh_selection;

typedef struct {
  int64_t B, H, N; /* batch, heads, sequence length */
  int32_t d;       /* head dimension */
  int32_t L;       /* pyramid levels */
  int32_t p;       /* pooling factor */
  int32_t k;       /* selection budget per level */
  int32_t chunk;   /* top-k stratification chunk T (candidates); 0 = 2048 */
  int32_t dtype;   /* lh_dtype of Q, K, V, Y, dY, dQ, dK, dV */
  int32_t scorer;  /* lh_scorer */
  int32_t selection; /* lh_selection */
} lh_config;

#define LH_MAX_LEVELS 16
#define LH_ERR_WORD_BYTES 256

/* Everything a caller needs to size and view the buffers.  Offsets are in
 * bytes from the start of ctx or ws and are 256-byte aligned. */
typedef struct {
  int64_t S;                          /* gathered length N/p^(L-1) + sum_l p*kprime[l] */
  int64_t pyr_entries;                /* sum over l of N/p^l */
  int64_t level_len[LH_MAX_LEVELS];   /* N/p^l */
  int64_t level_off[LH_MAX_LEVELS];   /* first row of level l in slot_of */
  int64_t upper_off[LH_MAX_LEVELS];   /* first row of level l>=1 in the pyramid buffers */
  int64_t upper_entries;              /* sum over l>=1 of N/p^l */
  int32_t kprime[LH_MAX_LEVELS];      /* min(k, N/p^(l+1)) for l < L-1 */
  int64_t sel_off[LH_MAX_LEVELS];     /* first entry of level l in sel */
  int64_t sel_per_head;               /* sum of kprime */
  /* stage-call buffer sizes (whole B*H) */
  size_t pyr_bytes;     /* one of pyr_q/pyr_k/pyr_v: [BH][upper_entries][d] in dtype */
  size_t norms_bytes;   /* [2][BH][N] fp32 */
  size_t topk_ws_bytes; /* ws of lh_score_topk */
  size_t sel_bytes;     /* [BH][sel_per_head] int32 */
  size_t seq_bytes;     /* one of qs/ks/vs/dos: [BH][S][d], 2 bytes an element */
  size_t os_bytes;      /* os: [BH][S][d] fp32 */
  size_t seq_map_bytes; /* [BH][S] int32 */
  size_t slot_of_bytes; /* [BH][pyr_entries] int32 */
  size_t lse_bytes;     /* [BH][S] fp32 (also Delta) */
  size_t grad_seq_bytes;/* one of dqs/dks/dvs: [BH][S][d] fp32 */
  size_t attn_bwd_ws_bytes;
  /* lh_forward / lh_backward */
  size_t ctx_bytes, ws_bytes;
  size_t ctx_off_sel, ctx_off_seq_map, ctx_off_slot_of, ctx_off_qs, ctx_off_ks, ctx_off_vs, ctx_off_os,
      ctx_off_lse;
  size_t ws_off_pyr_q, ws_off_pyr_k, ws_off_pyr_v, ws_off_norms, ws_off_topk;
  size_t ws_off_dos, ws_off_delta, ws_off_dqs, ws_off_dks, ws_off_dvs;
  /* lowest pyramid level that lh_forward writes (1 <= first_level <= max(1, L-1)):
   * a level l < L-1 is written whole only when N/p^l rows cost no more than
   * reading back the p^(l+1) kprime[l] level-0 rows of its kept entries;
   * the gather averages the kept entries of the levels below from level 0 */
  int32_t first_level;
} lh_plan_info;

/* Validate cfg and fill *info (host only, no CUDA call).
 * Cite: LH-post "Key formulas" (S = N/p^(L-1) + (L-1)*p*k; where k exceeds the
 * M = N/p^(l+1) candidates of a level, kprime = min(k, M) is kept). */
lh_status lh_plan(const lh_config *cfg, lh_plan_info *info);

/* Stage 1 - symmetric pyramid pooling plus level-0 norms.
 * Cite: LH-post "How it works" (1) (Q, K, V average-pooled with the same
 * factor p over L levels); LH-summary "Technical details" (1)-(2).
 * In:  q, k, v [BH][N][d] dtype.
 * Out: pyr_q, pyr_k, pyr_v [BH][upper_entries][d] dtype: level l >= 1 starts
 *      at row upper_off[l]; entry i is the mean of tokens [i p^l, (i+1) p^l),
 *      summed in fp32 and rounded once.
 *      norms [2][BH][N] fp32: plane 0 = ||Q_t||_2, plane 1 = ||K_t||_2.
 * With L = 1 the pyramid buffers are not touched (may be NULL).
 * The rows reach shared memory by bulk copies whose waits are bounded; this
 * call has no workspace, so a wait that runs out (a copy that never lands)
 * leaves the outputs incomplete without a status (lh_forward reports it
 * through its error word). */
lh_status lh_pyramid_pool(const lh_config *cfg, const void *q, const void *k, const void *v, void *pyr_q,
                          void *pyr_k, void *pyr_v, float *norms, lh_stream_t stream);

/* Stage 1 as lh_forward runs it: the same pooling and norms, but only levels
 * first_level..L-1 are written (rows of levels 1..first_level-1 of the
 * pyramid buffers are left untouched).  first_level in [1, max(1, L-1)];
 * plan_info.first_level is the value lh_forward uses.  lh_pyramid_pool is
 * this call with first_level = 1.  Same citations as lh_pyramid_pool. */
lh_status lh_pyramid_pool_from(const lh_config *cfg, int32_t first_level, const void *q, const void *k, const void *v,
                               void *pyr_q, void *pyr_k, void *pyr_v, float *norms, lh_stream_t stream);

/* Stage 2 - max-pooled scores and stratified chunked top-k.
 * Cite: LH-summary "Technical details" (2) (coarser levels take max-pooled
 * scores; top-K yields the index set I); LH-post "Limitations" (the top-K is
 * stratified: every interval contributes a fixed number).
 * In:  norms from lh_pyramid_pool; ws of topk_ws_bytes (score pyramid scratch,
 *      preceded by the error word).
 * Out: sel [BH][sel_per_head] int32: for level l < L-1, at sel_off[l], in
 *      ascending order, kprime[l] parent indices at level l+1 (PARENTS,
 *      NESTED) or p * kprime[l] entry indices at level l (DIRECT).  The M
 *      candidates of a level (all N/p^(l+1) entries of level l+1; all N/p^l of
 *      level l for DIRECT; the kept entries of level l+1 in ascending order for
 *      NESTED) are split into C = max(1, M / chunk) contiguous chunks (the
 *      first M mod C one longer); chunk c keeps its floor(b/C) + [c < b mod C]
 *      highest fp32 scores of the budget b, ties to the lower index.
 *      A chunk of at least M candidates makes C = 1: an exact global top-k per
 *      level (chunks above 48K candidates are read from the score pyramid in
 *      every radix pass instead of being staged in shared memory). */
lh_status lh_score_topk(const lh_config *cfg, const float *norms, void *ws, int32_t *sel, lh_stream_t stream);

/* Stage 2 without workspace, for callers that cannot allocate device memory
 * (a host whose allocator owns every device buffer, a runtime whose memory
 * plan is fixed, a plugin that only receives its inputs and outputs).  The
 * pages have no counterpart: this is lh_score_topk with its scratch kept in a
 * file-scope device array of 16 MiB that every GPU loading the library holds
 * until exit.  It calls no allocator.  The scratch a call needs is lh_plan's
 * topk_ws_bytes - LH_ERR_WORD_BYTES: the score pyramid, B*H * upper_entries * 4
 * bytes, plus B*H * N * 4 bytes of level-0 scores with LH_SELECT_DIRECT;
 * configurations above 16 MiB return LH_ERR_UNSUPPORTED.
 * In:  norms as for lh_score_topk.  Out: sel as for lh_score_topk.
 * The first call on a device (and the first after a cudaDeviceReset, which
 * makes a new context) looks up the array's device address with
 * cudaGetSymbolAddress and caches it per device and context; make that first
 * call before any stream capture.  All calls share the array: calls that
 * overlap on the GPU (other streams, other threads) race and must be
 * serialised by the caller.  The array keeps the last call's contents; every
 * call rewrites all it reads.  There is no error word: the selection's one
 * device-side check is kept unreachable by lh_plan's limits. */
lh_status lh_score_topk_static(const lh_config *cfg, const float *norms, int32_t *sel, lh_stream_t stream);

/* Stage 3 - gather the kept entries into one causally ordered sequence.
 * Cite: LH-post "How it works" (3) (kept entries sorted into causal order
 * form a contiguous sequence of length S); LH-summary "Technical details" (3).
 * Kept entries: the p children (l, m*p + c) of every parent m in sel level l
 * (or, with LH_SELECT_DIRECT, the entries listed in sel level l), and every
 * entry of the top level L-1.  Entry (l, i) has key
 * (e = (i+1) p^l - 1, -l); slots are the ranks of the keys.
 * In:  q, k, v (level 0) and pyr_q/k/v (levels >= 1), sel.
 * Out: qs, ks, vs [BH][S][d] bf16; seq_map [BH][S] int32 = (l << 28) | i;
 *      slot_of [BH][pyr_entries] int32 = slot of (l, i) at level_off[l] + i,
 *      -1 if not kept. */
lh_status lh_gather(const lh_config *cfg, const void *q, const void *k, const void *v, const void *pyr_q,
                    const void *pyr_k, const void *pyr_v, const int32_t *sel, void *qs, void *ks, void *vs,
                    int32_t *seq_map, int32_t *slot_of, lh_stream_t stream);

/* Stage 3 as lh_forward runs it: identical outputs, but a kept entry of a
 * level l < first_level is computed as the fp32 mean of its p^l level-0 rows
 * of q, k, v (rounded once), so the pyramid buffers are read only for levels
 * >= first_level (as written by lh_pyramid_pool_from with the same value).
 * lh_gather is this call with first_level = 1. */
lh_status lh_gather_from(const lh_config *cfg, int32_t first_level, const void *q, const void *k, const void *v,
                         const void *pyr_q, const void *pyr_k, const void *pyr_v, const int32_t *sel, void *qs,
                         void *ks, void *vs, int32_t *seq_map, int32_t *slot_of, lh_stream_t stream);

/* Stage 4 - dense causal attention over the S-token sequence (tcgen05).
 * Cite: LH-summary "Technical details" (3) (stock attention over the gathered
 * S tokens); LH-post "How it works" (3).  Softmax scale 1/sqrt(d); slot t
 * attends to slots u <= t.  Uses cfg->B, H, d only; S is any length >= 1.
 * The bf16 inputs are multiplied exactly and accumulated in fp32; the
 * probabilities enter P V as a bf16 pair (hi + lo), so O keeps fp32 accuracy.
 * Out: os [BH][S][d] fp32; lse [BH][S] fp32, natural log of the row's sum of
 *      exp(scaled logits).  ws: at least LH_ERR_WORD_BYTES (error word). */
lh_status lh_attn_fwd(const lh_config *cfg, int64_t S, const void *qs, const void *ks, const void *vs, float *os,
                      float *lse, void *ws, lh_stream_t stream);

/* Stage 4 backward.  Cite: LH-summary "Method" step 5 (the gradient flows
 * back through the attention kernel).  dS enters dQ and dK as a bf16 hi + lo
 * pair (fp32 accuracy); P enters dV = P^T dOs as one fp16 value (P is in
 * [0, 1], summed with positive weights), and dV and dP^T = Vs dOs^T are fp16
 * products (the kernel converts its Vs tile to fp16; Vs and dOs hold bf16
 * values, exact in fp16 up to magnitude 65504 - a larger one sets the error
 * word's range bit, reported by lh_check_error as LH_ERR_DEVICE).
 * In:  qs, ks, vs (bf16), lse from the forward; dos [BH][S][d] fp16 holding
 *      bf16 values and delta [BH][S] fp32 (rowsum(dOs * Os)), both as
 *      lh_scatter_back_adjoint writes them.
 * Out: dqs, dks, dvs [BH][S][d] fp32, each row written once (no accumulation).
 * ws: at least attn_bwd_ws_bytes (error word). */
lh_status lh_attn_bwd(const lh_config *cfg, int64_t S, const void *qs, const void *ks, const void *vs,
                      const float *lse, const void *dos, const float *delta, float *dqs, float *dks, float *dvs,
                      void *ws, lh_stream_t stream);

/* Stage 3 for one shard of the tokens (context parallelism: each GPU holds
 * the tokens [t0, t1) of every head).  Cite: LH-post "How it works" (3) (the
 * kept triples in causal order form one sequence); the entries whose key
 * e = (i+1) p^l - 1 lies in [t0, t1) form one contiguous segment of that
 * sequence, and their blocks lie inside the shard.
 * In:  cfg and sel of the whole layer (the selection every shard shares);
 *      t0 < t1 multiples of p^(L-1) in [0, N]; q, k, v [B][H][t1-t0][d] the
 *      shard's tokens; pyr_q/k/v the shard's pyramid, as lh_pyramid_pool
 *      writes it for a layer of the shard's t1 - t0 tokens (all levels);
 *      seg_off [B*H] int64 on the device: the slot of each head's first
 *      entry in the shard (the kept entries of the earlier shards).
 * Out: qs, ks, vs [B*H][seg_rows][d] bf16 and seq_map [B*H][seg_rows]: row
 *      r of head h is the entry at slot seg_off[h] + r (rows past the
 *      head's segment are left as they are; seg_rows >= the longest
 *      segment); seq_map holds (level << 28) | index within the shard's
 *      level; slot_of [B*H][pyr_entries of the shard's layer]: the row of
 *      each of the shard's entries in the segment, or -1.
 * Errors: LH_ERR_INVALID_ARG for a bad range, seg_rows outside [1, S] or a
 * NULL or misaligned pointer.  An entry whose segment row falls outside
 * [0, seg_rows) (seg_off or seg_rows too small) is skipped without a report
 * (the call takes no error word): size seg_rows from the selection. */
lh_status lh_gather_shard(const lh_config *cfg, int64_t t0, int64_t t1, const int64_t *seg_off, int64_t seg_rows,
                          const void *q, const void *k, const void *v, const void *pyr_q, const void *pyr_k,
                          const void *pyr_v, const int32_t *sel, void *qs, void *ks, void *vs, int32_t *seq_map,
                          int32_t *slot_of, lh_stream_t stream);

/* Stages 5, 5 backward and 1 backward for one shard of the tokens (context
 * parallelism), with cfg the layer of the shard's tokens (cfg->N = t1 - t0)
 * and the shard's segment of seg_rows sequence rows per head in place of the
 * plan's S (os, dos, delta, dqs/dks/dvs and seq_map as [B*H][seg_rows][...]).
 * slot_of and seq_map are the shard's, as lh_gather_shard writes them; rows
 * of seq_map past a head's segment must hold (0 << 28) | cfg->N (an empty
 * range).  Each equals the whole-layer call on the shard's rows except where
 * an entry's range R(l, i) crosses the shard's edge:
 *  - lh_scatter_back_shard adds halo [B*H][L-1][d] fp32: for l >= 1 the Os row
 *    of the previous shard's last level-l entry (zeros where it is not kept;
 *    all zeros on the first shard), whose range covers this shard's first
 *    p^l - 1 rows; the sum is rounded once.  bf16 rows of 128 channels only
 *    (else LH_ERR_UNSUPPORTED).
 *  - lh_scatter_back_adjoint_shard adds halo [B*H][L-1][d] fp32 (NULL on the
 *    last shard): for l >= 1 the next shard's sum of dY over its first
 *    p^l - 1 rows (lh_head_sums), to this shard's last level-l entry before
 *    the rounding and delta.
 *  - lh_pool_adjoint_shard: no halo (an entry's block lies in its shard).
 * lh_head_sums writes sums [B*H][L-1][d] fp32: for l = 1 .. L-1 the sum of
 * dY over the first p^l - 1 rows of each head (the part of the previous
 * shard's last level-l range that lies in this shard).
 * Errors as the whole-layer calls, and LH_ERR_INVALID_ARG for seg_rows
 * outside [1, 2^31). */
lh_status lh_scatter_back_shard(const lh_config *cfg, int64_t seg_rows, const float *os, const int32_t *slot_of,
                                const float *halo, void *y, lh_stream_t stream);
lh_status lh_scatter_back_adjoint_shard(const lh_config *cfg, int64_t seg_rows, const void *dy,
                                        const int32_t *seq_map, const float *os, const float *halo, void *dos,
                                        float *delta, lh_stream_t stream);
lh_status lh_pool_adjoint_shard(const lh_config *cfg, int64_t seg_rows, const float *dqs, const float *dks,
                                const float *dvs, const int32_t *slot_of, void *dq, void *dk, void *dv,
                                lh_stream_t stream);
lh_status lh_head_sums(const lh_config *cfg, const void *dy, float *sums, lh_stream_t stream);

/* Stage 4 over a row window of the sequence: the rows [row_lo, row_hi) of
 * lh_attn_fwd's os and lse (each query row still attends every key row up to
 * itself), for running the attention of one sequence in pieces (one piece per
 * GPU under context parallelism).  row_lo a multiple of 128; row_hi a
 * multiple of 128 or S.  Rows outside the window are not written; an empty
 * window queues nothing.  Other arguments and errors as lh_attn_fwd; the
 * window's rows equal lh_attn_fwd's bit for bit. */
lh_status lh_attn_fwd_rows(const lh_config *cfg, int64_t S, int64_t row_lo, int64_t row_hi, const void *qs,
                           const void *ks, const void *vs, float *os, float *lse, void *ws, lh_stream_t stream);

/* Stage 4 backward over row windows: dqs rows [q_lo, q_hi) and dks, dvs rows
 * [k_lo, k_hi) of lh_attn_bwd (every query and key row of the sequence is
 * read).  Each bound as for lh_attn_fwd_rows; either window may be empty.
 * Rows outside the windows are not written; the windows' rows equal
 * lh_attn_bwd's bit for bit. */
lh_status lh_attn_bwd_rows(const lh_config *cfg, int64_t S, int64_t q_lo, int64_t q_hi, int64_t k_lo, int64_t k_hi,
                           const void *qs, const void *ks, const void *vs, const float *lse, const void *dos,
                           const float *delta, float *dqs, float *dks, float *dvs, void *ws, lh_stream_t stream);

/* Stage 5 - scatter-back.  Cite: LH-summary "Technical details" (4) (outputs
 * return to the N positions and each position j sums over the ranges
 * R(l, i)); LH-post "How it works" (4) (shifted ranges keep causality).
 * Y_j = sum over l of Os[slot(l, floor((j+1)/p^l) - 1)] for kept entries,
 * summed in fp32 and rounded once; R(l, i) =
 * [(i+1) p^l - 1, (i+2) p^l - 1).  Positions with no contributor get 0.
 * Out: y [BH][N][d] dtype. */
lh_status lh_scatter_back(const lh_config *cfg, const float *os, const int32_t *slot_of, void *y,
                          lh_stream_t stream);

/* Stage 5 backward: dOs[slot(l,i)] = sum of dY_j over j in R(l, i) (fp32,
 * rounded once to bf16), and delta[s] = sum_c dOs[s,c] * Os[s,c] (fp32, from
 * the rounded dOs and the fp32 Os).  Cite: LH-summary "Method" step 5.
 * Out: dos [BH][S][d] fp16 (the bf16-rounded values, exact in fp16; a
 *      magnitude above 65504 sets the error word's range bit, reported by
 *      lh_check_error as LH_ERR_DEVICE), delta [BH][S] fp32. */
lh_status lh_scatter_back_adjoint(const lh_config *cfg, const void *dy, const int32_t *seq_map, const float *os,
                                  void *dos, float *delta, lh_stream_t stream);

/* Stages 3 and 1 backward: dX_t = sum over l of p^-l * dXs[slot(l, floor(t/p^l))]
 * for kept entries (fp32, rounded once), X in {Q, K, V}.  No gradient flows
 * through the scores: the top-k is not differentiable (LH-post "How it
 * works" (2)).  In: dqs, dks, dvs fp32.  Out: dq, dk, dv [BH][N][d] dtype. */
lh_status lh_pool_adjoint(const lh_config *cfg, const float *dqs, const float *dks, const float *dvs,
                          const int32_t *slot_of, void *dq, void *dk, void *dv, lh_stream_t stream);

/* Whole forward: stages 1-5.  ctx (ctx_bytes) receives what the backward
 * needs (sel, seq_map, slot_of, Qs, Ks, Vs, Os, LSE at the ctx_off_* offsets)
 * and must live until lh_backward.  ws (ws_bytes) is scratch; its error word
 * is cleared at entry. */
lh_status lh_forward(const lh_config *cfg, const void *q, const void *k, const void *v, void *y, void *ctx,
                     size_t ctx_bytes, void *ws, size_t ws_bytes, lh_stream_t stream);

/* Whole backward: stage 5 adjoint, attention backward, pool/gather adjoint.
 * ctx is read only.  ws (ws_bytes) is scratch; its error word is cleared at entry. */
lh_status lh_backward(const lh_config *cfg, const void *dy, const void *ctx, size_t ctx_bytes, void *dq,
                      void *dk, void *dv, void *ws, size_t ws_bytes, lh_stream_t stream);

/* ---------------------------------------------------------------------------
 * PISA block selection (a second workload on the same pyramid idea).
 * Cite: the blog.secrett2633.cloud review "[논문리뷰] Block Sparse Attention
 * with Log-Linear Complexity" (PISA-review), section 1 (block sparse
 * attention selects key blocks per query; LSE scores the candidate blocks)
 * and section 3 (keys pooled fine-to-coarse; selection starts at the
 * coarsest level, keeps the top K by LSE and expands them into sub-blocks
 * level by level down to the finest; O(N log N)).
 *
 * Readings of what the page leaves open:
 *  - level l entry j is the mean of keys [j p^l, (j+1) p^l) (level 0 = the
 *    keys), stored in bf16 rounded to nearest even from the exact mean;
 *  - a block is `block` (C) consecutive entries of one level; block b of
 *    level l has sub-blocks p b .. p b + p - 1 at level l-1;
 *  - `group` (G) consecutive queries share one selection;
 *  - the score of block b of level l for group g is
 *      ln sum_{i in g} sum_{j in b, (j+1) p^l - 1 <= i} exp(q_i . k^(l)_j / sqrt(d)),
 *    -inf when no pair is visible;
 *  - the coarsest level's candidates are all its blocks; a level keeps
 *    min(topk, candidates) blocks, higher score first, equal scores (-inf
 *    included) to the lower block index.
 * Support: bf16 Q and K [B][H][N][d]; d in {64, 128}; block in {64, 128};
 * group = 128; p a power of two >= 2; 1 <= L <= 8; N divisible by
 * block * p^(L-1) and < 2^28; blocks[L-1] <= 256 and p * topk <= 256;
 * B*H <= 65535.
 * ------------------------------------------------------------------------- */
typedef struct {
  int64_t B, H, N; /* batch, heads, sequence length */
  int32_t d;       /* head dimension */
  int32_t p;       /* pooling factor between levels */
  int32_t L;       /* levels of the key pyramid (level 0 = the keys) */
  int32_t block;   /* C: entries per block, every level */
  int32_t group;   /* G: queries per selection */
  int32_t topk;    /* K: blocks kept per level */
} lh_pisa_config;

typedef struct {
  int64_t n_groups;                   /* N / group */
  int64_t blocks[LH_MAX_LEVELS];      /* N / (block p^l) */
  int64_t level_off[LH_MAX_LEVELS];   /* first row of level l >= 1 in the key pyramid */
  int64_t upper_entries;              /* sum over l >= 1 of N / p^l */
  size_t pyr_bytes;                   /* key pyramid [BH][upper_entries][d] bf16 */
  size_t kept_elems;                  /* BH * n_groups * L * topk */
  int32_t max_candidates;             /* most candidates one level scores */
} lh_pisa_info;

/* Validate cfg and fill *info (host only, no CUDA call). */
lh_status lh_pisa_plan(const lh_pisa_config *cfg, lh_pisa_info *info);

/* The key pyramid.  In: k [BH][N][d] bf16.  Out: kpyr [BH][upper_entries][d]
 * bf16, level l >= 1 from row level_off[l]; each entry is summed exactly (fp64)
 * from the level-0 keys and rounded once.  L = 1: nothing is written (kpyr
 * may be NULL). */
lh_status lh_pisa_pool_keys(const lh_pisa_config *cfg, const void *k, void *kpyr, lh_stream_t stream);

/* The coarse-to-fine selection.  In: q, k [BH][N][d] bf16; kpyr from
 * lh_pisa_pool_keys (unused when L = 1); ws: at least LH_ERR_WORD_BYTES (the
 * error word; a bounded wait that runs out sets it).
 * Out: kept_idx [BH][n_groups][L][topk] int32 and kept_score (same shape,
 * fp32, natural log): for every group and level the kept blocks in
 * ascending block order with their scores, padded with -1 / -inf when a
 * level has fewer than topk candidates.  Level 0 is the selection. */
lh_status lh_pisa_select(const lh_pisa_config *cfg, const void *q, const void *k, const void *kpyr,
                         int32_t *kept_idx, float *kept_score, void *ws, lh_stream_t stream);

/* Self-test of the device-side timeout path (the pages have no counterpart).
 * Launches the stage-4 forward kernel on one 128-row tile (d = 64) with its
 * TMA producer told to load nothing and every barrier wait bounded by
 * `wait_cycles` SM clocks.  Its MMA and softmax warps then wait on barriers
 * that never complete; the first wait to run out stops every role, the kernel
 * returns (no copy or MMA was ever issued, so nothing is in flight) and sets
 * the timeout bit of the error word at the start of ws.  The GPU context
 * stays usable.
 * In:  wait_cycles in [1, 4e9] (about 2 s at the boost clock for 4e9).
 * ws:  device buffer of at least LH_SELFTEST_WS_BYTES bytes: the error word,
 *      then room the kernel's tensor maps and outputs point into.
 * Returns LH_OK once the kernel is queued; lh_check_error(ws, stream) then
 * returns LH_ERR_TIMEOUT, which is the expected outcome. */
#define LH_SELFTEST_WS_BYTES 131072
lh_status lh_selftest_wait_timeout(void *ws, size_t ws_bytes, int64_t wait_cycles, lh_stream_t stream);

/* Synchronise `stream`, read the error word at the start of ws, clear it and
 * return LH_OK, LH_ERR_TIMEOUT or LH_ERR_DEVICE (or LH_ERR_CUDA). */
lh_status lh_check_error(void *ws, lh_stream_t stream);

/* Zero the error word at the start of ws (asynchronous). */
lh_status lh_clear_error(void *ws, lh_stream_t stream);

/* Static text of a status. */
const char *lh_status_string(lh_status status);

/* Text of the last failure on the calling thread ("" if none). */
const char *lh_last_error_message(void);

#ifdef __cplusplus
}
#endif

#endif /* LH_H */
