// Stage 4 backward: gradients of the dense causal attention over the S-token
// sequence (aitrends.kr summary of Lighthouse Attention, Method step 5: the
// gradient flows back through the attention kernel; the top-k passes none).
//
// With P = softmax(Qs Ks^T / sqrt(d)) (causal) recomputed from the saved LSE,
//   dVs = P^T dOs,  dP = dOs Vs^T,  dS = P * (dP - Delta) / sqrt(d),
//   dQs = dS Ks,    dKs = dS^T Qs,  Delta = rowsum(dOs * Os).
// P and dS enter their products as bf16 (hi + lo) pairs, so the bf16
// roundings of the probabilities and of dS do not show in the gradients.
//
// Two kernels, each writing its gradient once (no atomics):
//
// attn_bwd_kv_kernel (dKs, dVs) - one CTA per 128-row key tile; it steps over
//   64-query half tiles from the diagonal to the end.  For half step s the MMA
//   warp computes S^T = K Q_h^T and dP^T = V dO_h^T into TMEM buffer s&1 while
//   the compute warpgroups work on the other buffer; they write P^T and dS^T
//   (hi/lo) back over the columns they read, and the MMA warp then adds
//   dV += P^T dO_h and dK += dS^T Q_h with both A operands read from TMEM.
//   Q_h, dO_h stream through a 4-slot ring.
//
// attn_bwd_q_kernel (dQs) - one CTA per 128-row query tile; it steps over
//   64-key half tiles up to the diagonal: S = Q K_h^T and dP = dO V_h^T into
//   TMEM buffer u&1, the compute warpgroups write dS (hi/lo) over the dP
//   columns, and dQ += dS K_h reads it from TMEM.  K_h and V_h stream through
//   4-slot rings, each slot released by the last product that reads it.
//
// Warp roles in both: warps 0-7 two compute warpgroups (thread (g, t) owns
// TMEM lane t and columns [32g, 32g+32) of each 64-column half), warp 8 TMA
// producer, warp 9 MMA issuer (one thread) and TMEM owner.
#include <math.h>

#include "lh_common.cuh"
#include "sm100.cuh"

namespace lh {

bool make_seq_map(CUtensorMap* m, const void* base, int64_t BH, int64_t rows, int D, int box_rows);

namespace {
using namespace sm100;

constexpr int kCompute = 256;
constexpr int kThreads = kCompute + 64;
constexpr int kRegion = 128 * 128;  // one [128 rows][64 bf16] SW128 region
constexpr int kHalfRegion = 64 * 128;

__device__ __forceinline__ void compute_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// P^T / dS (hi, lo) of 32 columns c0..c0+31 of one row as bf16 pairs over the
// 32 TMEM columns they were read from: hi in the first 16, lo in the last 16.
__device__ __forceinline__ void store_pair_chunk(uint32_t taddr, const uint32_t (&hi)[16], const uint32_t (&lo)[16]) {
  tmem_st16(taddr, hi);
  tmem_st16(taddr + 16, lo);
}

// ===========================================================================
// dKs, dVs
// ===========================================================================
template <int D>
struct KvSmem {
  static constexpr int kTile = D / 64 * kRegion;         // K or V tile, 128 rows
  static constexpr int kHalf = D / 64 * kHalfRegion;     // Q_h or dO_h, 64 rows
  static constexpr int oK = 0;
  static constexpr int oV = oK + kTile;
  static constexpr int oRing = oV + kTile;               // 4 slots of (Q_h, dO_h)
  static constexpr int kSlot = 2 * kHalf;
  static constexpr int oVec = oRing + 4 * kSlot;         // [2][128] floats: LSE*log2e [64], Delta [64]
  static constexpr int oBar = oVec + 1024;
  static constexpr int kBytes = oBar + 256;
  static constexpr int kAlloc = kBytes + 1024;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_kv_kernel(const __grid_constant__ CUtensorMap tmQh, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmOh,
                       const float* __restrict__ LSE, const float* __restrict__ Delta, float* __restrict__ dK,
                       float* __restrict__ dV, int* errw, int S, float scale_log2, float scale) {
  using Lay = KvSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::oBar);
  uint64_t* bKV = bars + 0;        // K, V landed
  uint64_t* bLoad = bars + 1;      // [4] Q_h, dO_h of a ring slot landed
  uint64_t* bSlotFree = bars + 5;  // [4] dV, dK products done with a slot
  uint64_t* bF = bars + 9;         // [2] S^T, dP^T of a half step in TMEM buffer
  uint64_t* bPS = bars + 11;       // [2] P^T, dS^T written back (256 arrivals)
  uint64_t* bDone = bars + 13;     // every product done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::oBar + 128);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::oBar + 132);
  float* sVec = reinterpret_cast<float*>(smem + Lay::oVec);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_qt = (S + 127) / 128;
  const int kt = (int)blockIdx.x;  // key tile; small kt = most query tiles, launched first
  const int bh = (int)blockIdx.y;
  const int NS = 2 * (n_qt - kt);  // half steps

  if (threadIdx.x == 0) {
    mbar_init(bKV, 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&bLoad[i], 1);
      mbar_init(&bSlotFree[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bF[i], 1);
      mbar_init(&bPS[i], kCompute);
    }
    mbar_init(bDone, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  constexpr uint32_t tSP = 0, tDP = 128, tDV = 256, tDK = 256 + D;  // SP/DP: [2] x 64 columns

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQh);
      tma_prefetch_desc(&tmOh);
      mbar_expect_tx(bKV, 2 * 128 * D * 2);
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(smem + Lay::oK + c * kRegion, &tmK, bKV, c * 64, kt * 128, bh);
        tma_load_3d(smem + Lay::oV + c * kRegion, &tmV, bKV, c * 64, kt * 128, bh);
      }
      for (int s = 0; s < NS; ++s) {
        const int slot = s & 3;
        if (s >= 4 && !mbar_wait(&bSlotFree[slot], ((s >> 2) - 1) & 1, abort_flag)) break;
        const int q0 = (kt + (s >> 1)) * 128 + (s & 1) * 64;
        uint8_t* base = smem + Lay::oRing + slot * Lay::kSlot;
        mbar_expect_tx(&bLoad[slot], 2 * 64 * D * 2);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(base + c * kHalfRegion, &tmQh, &bLoad[slot], c * 64, q0, bh);
          tma_load_3d(base + Lay::kHalf + c * kHalfRegion, &tmOh, &bLoad[slot], c * 64, q0, bh);
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    {  // the whole warp; one elected lane issues each instruction
      constexpr uint32_t idF = idesc_bf16(128, 64, false, false);  // S^T, dP^T: N = 64 queries
      constexpr uint32_t idG = idesc_bf16(128, D, false, true);    // dV, dK: A from TMEM, B MN-major
      const uint32_t sRing = smem_u32(smem + Lay::oRing);
      const uint64_t kK = sdesc_sw128(smem_u32(smem + Lay::oK), 16, 1024);
      const uint64_t kV = sdesc_sw128(smem_u32(smem + Lay::oV), 16, 1024);
      const uint64_t kRing = sdesc_sw128(sRing, 16, 1024);
      const uint64_t mRing = sdesc_sw128(sRing, kHalfRegion, 1024);
      bool ok = mbar_wait_warp(bKV, 0, abort_flag);
      // the loads of half step s landed (waited for before the products that
      // precede its F in the issue order, so no wait sits between them)
      auto wait_f = [&](int s) -> bool { return mbar_wait_warp(&bLoad[s & 3], (s >> 2) & 1, abort_flag); };
      auto issue_f = [&](int s) {
        const int slot = s & 3, b = s & 1;
        tc_fence_after();
        const uint32_t qo = (slot * Lay::kSlot) >> 4, oo = (slot * Lay::kSlot + Lay::kHalf) >> 4;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t at = ((kk >> 2) * kRegion + (kk & 3) * 32) >> 4;    // K, V tile (128 rows)
          const uint32_t bt = ((kk >> 2) * kHalfRegion + (kk & 3) * 32) >> 4;  // Q_h, dO_h (64 rows)
          umma_bf16_w(tmem + tSP + b * 64, kK + at, kRing + qo + bt, idF, kk > 0 ? 1u : 0u);
          umma_bf16_w(tmem + tDP + b * 64, kV + at, kRing + oo + bt, idF, kk > 0 ? 1u : 0u);
        }
        umma_commit_w(&bF[b]);
      };
      if (ok && (ok = wait_f(0))) issue_f(0);
      if (ok && NS > 1 && (ok = wait_f(1))) issue_f(1);
      for (int s = 0; ok && s < NS; ++s) {
        const int slot = s & 3, b = s & 1;
        if (s + 2 < NS && !wait_f(s + 2)) { ok = false; break; }
        if (!mbar_wait_warp(&bPS[b], (s >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t qo = (slot * Lay::kSlot) >> 4, oo = (slot * Lay::kSlot + Lay::kHalf) >> 4;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {  // 16 queries per step; hi of chunk kk/2 at +(kk&1)*8, lo at +16
          const uint32_t a = (kk >> 1) * 32 + (kk & 1) * 8;
          const uint32_t acc = (s > 0 || kk > 0) ? 1u : 0u;
          const uint32_t bq = (kk * 2048) >> 4;
          umma_bf16_tmem_a_w(tmem + tDV, tmem + tSP + b * 64 + a, mRing + oo + bq, idG, acc);
          umma_bf16_tmem_a_w(tmem + tDV, tmem + tSP + b * 64 + a + 16, mRing + oo + bq, idG, 1u);
          umma_bf16_tmem_a_w(tmem + tDK, tmem + tDP + b * 64 + a, mRing + qo + bq, idG, acc);
          umma_bf16_tmem_a_w(tmem + tDK, tmem + tDP + b * 64 + a + 16, mRing + qo + bq, idG, 1u);
        }
        umma_commit_w(&bSlotFree[slot]);
        // the next half step that uses this TMEM buffer; its S^T, dP^T land
        // after the products above have read P^T and dS^T (in-order issue)
        if (s + 2 < NS) issue_f(s + 2);
      }
      if (ok) umma_commit_w(bDone);
    }
  } else {
    // ------------------------------------------------------------ compute warpgroups
    const int ct = threadIdx.x;            // 0..255
    const int g = warp >> 2;               // query columns [32g, 32g+32) of each half
    const int t = (warp & 3) * 32 + lane;  // key row of the tile (TMEM lane)
    const int kv_g = kt * 128 + t;
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    bool ok = true;
    // LSE (ct < 64) or Delta (64 <= ct < 128) of query row ct & 63 of half
    // step s, loaded one half step ahead and converted when it is stored
    auto vec_row = [&](int s) { return (kt + (s >> 1)) * 128 + (s & 1) * 64 + (ct & 63); };
    auto vec_raw = [&](int s) -> float {
      const int qg = vec_row(s);
      return qg < S ? ldg_nc_f32((ct < 64 ? LSE : Delta) + (int64_t)bh * S + qg) : 0.f;
    };
    float vec_next = ct < 128 ? vec_raw(0) : 0.f;
    const uint64_t c2 = f2_pack(scale_log2, scale_log2), sc2 = f2_pack(scale, scale);
    for (int s = 0; s < NS; ++s) {
      const int b = s & 1;
      const float vec_cur = vec_next;
      if (ct < 128 && s + 1 < NS) vec_next = vec_raw(s + 1);
      if (ct < 64) sVec[b * 128 + ct] = vec_row(s) < S ? vec_cur * 1.4426950408889634f : INFINITY;
      else if (ct < 128) sVec[b * 128 + ct] = vec_cur;
      compute_sync();
      const float* lse = sVec + b * 128;
      const float* del = lse + 64;
      const int q0 = (kt + (s >> 1)) * 128 + (s & 1) * 64;
      const bool diag = (s >> 1) == 0;  // the diagonal query tile
      // warp-uniform outcome for the collective TMEM accesses; after a failed
      // wait the loop keeps its compute_sync count and skips the work
      ok = __all_sync(0xffffffffu, ok && mbar_wait(&bF[b], (s >> 1) & 1, abort_flag));
      if (!ok) continue;
      tc_fence_after();
      uint32_t sr[32], dr[32];
      tmem_ld32(tl + tSP + b * 64 + g * 32, sr);
      tmem_ld32(tl + tDP + b * 64 + g * 32, dr);
      tmem_ld_wait();
      uint32_t phi[16], plo[16], dhi[16], dlo[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        const int qi = g * 32 + e;
        const float2 l2 = *reinterpret_cast<const float2*>(lse + qi);
        const float2 d2 = *reinterpret_cast<const float2*>(del + qi);
        float pa, pb;
        f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])), c2, f2_pack(-l2.x, -l2.y)), pa,
                  pb);
        pa = fast_exp2(pa);
        pb = fast_exp2(pb);
        if (diag) {
          if (q0 + qi < kv_g) pa = 0.f;
          if (q0 + qi + 1 < kv_g) pb = 0.f;
        }
        const uint64_t p2 = f2_pack(pa, pb);
        const uint64_t diff2 = f2_sub(f2_pack(__uint_as_float(dr[e]), __uint_as_float(dr[e + 1])), f2_pack(d2.x, d2.y));
        float da, db;
        f2_unpack(f2_mul(f2_mul(p2, sc2), diff2), da, db);
        split_bf16x2(pa, pb, phi[e >> 1], plo[e >> 1]);
        split_bf16x2(da, db, dhi[e >> 1], dlo[e >> 1]);
      }
      store_pair_chunk(tl + tSP + b * 64 + g * 32, phi, plo);
      store_pair_chunk(tl + tDP + b * 64 + g * 32, dhi, dlo);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bPS[b]);
    }
    if (__all_sync(0xffffffffu, ok && mbar_wait(bDone, 0, abort_flag))) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        const int col = g * (D / 2) + c * 32;
        uint32_t rv[32], rk[32];
        tmem_ld32(tl + tDV + col, rv);
        tmem_ld32(tl + tDK + col, rk);
        tmem_ld_wait();
        if (kv_g < S) {
          float4* dv4 = reinterpret_cast<float4*>(dV + ((int64_t)bh * S + kv_g) * D + col);
          float4* dk4 = reinterpret_cast<float4*>(dK + ((int64_t)bh * S + kv_g) * D + col);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            dv4[q] = make_float4(__uint_as_float(rv[4 * q]), __uint_as_float(rv[4 * q + 1]),
                                 __uint_as_float(rv[4 * q + 2]), __uint_as_float(rv[4 * q + 3]));
            dk4[q] = make_float4(__uint_as_float(rk[4 * q]), __uint_as_float(rk[4 * q + 1]),
                                 __uint_as_float(rk[4 * q + 2]), __uint_as_float(rk[4 * q + 3]));
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && *abort_flag) report_error(errw, ERRW_TIMEOUT);
}

// ===========================================================================
// dQs
// ===========================================================================
template <int D>
struct QSmem {
  static constexpr int kTile = D / 64 * kRegion;      // Q or dO tile, 128 rows
  static constexpr int kHalf = D / 64 * kHalfRegion;  // K_h or V_h, 64 rows
  static constexpr int oQ = 0;
  static constexpr int oO = oQ + kTile;     // dO
  static constexpr int oK = oO + kTile;     // 4 slots of K_h
  static constexpr int oV = oK + 4 * kHalf; // 4 slots of V_h
  static constexpr int oBar = oV + 4 * kHalf;
  static constexpr int kBytes = oBar + 256;
  static constexpr int kAlloc = kBytes + 1024;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_q_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKh,
                      const __grid_constant__ CUtensorMap tmVh, const __grid_constant__ CUtensorMap tmO,
                      const float* __restrict__ LSE, const float* __restrict__ Delta, float* __restrict__ dQ,
                      int* errw, int S, float scale_log2, float scale) {
  using Lay = QSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::oBar);
  uint64_t* bQO = bars + 0;     // Q, dO landed
  uint64_t* bK = bars + 1;      // [4] K_h of a slot landed
  uint64_t* bV = bars + 5;      // [4] V_h of a slot landed
  uint64_t* bKfree = bars + 9;  // [4] the dQ product is done with K_h
  uint64_t* bVfree = bars + 13; // [4] the dP product is done with V_h
  uint64_t* bF = bars + 17;     // [2] S, dP of a half step in TMEM buffer
  uint64_t* bPS = bars + 19;    // [2] dS written back (256 arrivals)
  uint64_t* bDone = bars + 21;  // every product done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::oBar + 192);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::oBar + 196);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_qt = (S + 127) / 128;
  const int qt = n_qt - 1 - (int)blockIdx.x;  // longest rows first
  const int bh = (int)blockIdx.y;
  const int NU = 2 * (qt + 1);  // 64-key half steps up to the diagonal

  if (threadIdx.x == 0) {
    mbar_init(bQO, 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&bK[i], 1);
      mbar_init(&bV[i], 1);
      mbar_init(&bKfree[i], 1);
      mbar_init(&bVfree[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bF[i], 1);
      mbar_init(&bPS[i], kCompute);
    }
    mbar_init(bDone, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  constexpr uint32_t tS = 0, tDP = 128, tDQ = 256;  // S, dP: [2] x 64 columns

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    // K_h and V_h of half step u go to slot u & 3; V_h is released by the dP
    // product of its half step, K_h by the dQ product, so each reloads as
    // soon as its last reader is done
    if (lane == 0) {
      tma_prefetch_desc(&tmKh);
      tma_prefetch_desc(&tmVh);
      mbar_expect_tx(bQO, 2 * 128 * D * 2);
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(smem + Lay::oQ + c * kRegion, &tmQ, bQO, c * 64, qt * 128, bh);
        tma_load_3d(smem + Lay::oO + c * kRegion, &tmO, bQO, c * 64, qt * 128, bh);
      }
      for (int u = 0; u < NU; ++u) {
        const int slot = u & 3, k0 = u * 64;
        const uint32_t par = ((u >> 2) - 1) & 1;
        if (u >= 4 && !mbar_wait(&bVfree[slot], par, abort_flag)) break;
        mbar_expect_tx(&bV[slot], 64 * D * 2);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + Lay::oV + slot * Lay::kHalf + c * kHalfRegion, &tmVh, &bV[slot], c * 64, k0, bh);
        if (u >= 4 && !mbar_wait(&bKfree[slot], par, abort_flag)) break;
        mbar_expect_tx(&bK[slot], 64 * D * 2);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + Lay::oK + slot * Lay::kHalf + c * kHalfRegion, &tmKh, &bK[slot], c * 64, k0, bh);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    {  // the whole warp; one elected lane issues each instruction
      constexpr uint32_t idF = idesc_bf16(128, 64, false, false);  // S, dP: N = 64 keys
      constexpr uint32_t idG = idesc_bf16(128, D, false, true);    // dQ: A from TMEM, B MN-major
      const uint64_t kQ = sdesc_sw128(smem_u32(smem + Lay::oQ), 16, 1024);
      const uint64_t kO = sdesc_sw128(smem_u32(smem + Lay::oO), 16, 1024);
      const uint64_t kK = sdesc_sw128(smem_u32(smem + Lay::oK), 16, 1024);
      const uint64_t kV = sdesc_sw128(smem_u32(smem + Lay::oV), 16, 1024);
      const uint64_t mK = sdesc_sw128(smem_u32(smem + Lay::oK), kHalfRegion, 1024);
      bool ok = mbar_wait_warp(bQO, 0, abort_flag);
      auto wait_f = [&](int u) -> bool {
        return mbar_wait_warp(&bK[u & 3], (u >> 2) & 1, abort_flag) && mbar_wait_warp(&bV[u & 3], (u >> 2) & 1, abort_flag);
      };
      auto issue_f = [&](int u) {
        const int slot = u & 3, b = u & 1;
        tc_fence_after();
        const uint32_t so = (slot * Lay::kHalf) >> 4;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qoff = ((kk >> 2) * kRegion + (kk & 3) * 32) >> 4;      // Q, dO (128 rows)
          const uint32_t hoff = ((kk >> 2) * kHalfRegion + (kk & 3) * 32) >> 4;  // K_h, V_h (64 rows)
          umma_bf16_w(tmem + tS + b * 64, kQ + qoff, kK + so + hoff, idF, kk > 0 ? 1u : 0u);
          umma_bf16_w(tmem + tDP + b * 64, kO + qoff, kV + so + hoff, idF, kk > 0 ? 1u : 0u);
        }
        umma_commit_w(&bVfree[slot]);
        umma_commit_w(&bF[b]);
      };
      if (ok && (ok = wait_f(0))) issue_f(0);
      if (ok && NU > 1 && (ok = wait_f(1))) issue_f(1);
      for (int u = 0; ok && u < NU; ++u) {
        const int slot = u & 3, b = u & 1;
        if (u + 2 < NU && !wait_f(u + 2)) { ok = false; break; }
        if (!mbar_wait_warp(&bPS[b], (u >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint64_t mk = mK + ((slot * Lay::kHalf) >> 4);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {  // 16 keys per step
          const uint32_t a = tmem + tDP + b * 64 + (kk >> 1) * 32 + (kk & 1) * 8;
          const uint64_t bk = mk + ((kk * 2048) >> 4);
          umma_bf16_tmem_a_w(tmem + tDQ, a, bk, idG, (u > 0 || kk > 0) ? 1u : 0u);
          umma_bf16_tmem_a_w(tmem + tDQ, a + 16, bk, idG, 1u);
        }
        umma_commit_w(&bKfree[slot]);
        if (u + 2 < NU) issue_f(u + 2);
      }
      if (ok) umma_commit_w(bDone);
    }
  } else {
    // ------------------------------------------------------------ compute warpgroups
    const int g = warp >> 2;               // key columns [32g, 32g+32) of each half
    const int t = (warp & 3) * 32 + lane;  // query row of the tile (TMEM lane)
    const int qg = qt * 128 + t;
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const float lse = qg < S ? LSE[(int64_t)bh * S + qg] * 1.4426950408889634f : INFINITY;
    const float del = qg < S ? Delta[(int64_t)bh * S + qg] : 0.f;
    const uint64_t c2 = f2_pack(scale_log2, scale_log2), sc2 = f2_pack(scale, scale);
    const uint64_t nl2 = f2_pack(-lse, -lse), d2 = f2_pack(del, del);
    bool ok = true;
    for (int u = 0; u < NU; ++u) {
      const int b = u & 1;
      const int k0 = (u >> 1) * 128 + (u & 1) * 64 + g * 32;  // first key of this thread's chunk
      const bool diag = (u >> 1) == qt;
      ok = __all_sync(0xffffffffu, mbar_wait(&bF[b], (u >> 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[32], dr[32];
      tmem_ld32(tl + tS + b * 64 + g * 32, sr);
      tmem_ld32(tl + tDP + b * 64 + g * 32, dr);
      tmem_ld_wait();
      uint32_t dhi[16], dlo[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        float pa, pb;
        f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])), c2, nl2), pa, pb);
        pa = fast_exp2(pa);
        pb = fast_exp2(pb);
        if (diag) {
          if (k0 + e > qg) pa = 0.f;
          if (k0 + e + 1 > qg) pb = 0.f;
        }
        const uint64_t diff2 = f2_sub(f2_pack(__uint_as_float(dr[e]), __uint_as_float(dr[e + 1])), d2);
        float da, db;
        f2_unpack(f2_mul(f2_mul(f2_pack(pa, pb), sc2), diff2), da, db);
        split_bf16x2(da, db, dhi[e >> 1], dlo[e >> 1]);
      }
      store_pair_chunk(tl + tDP + b * 64 + g * 32, dhi, dlo);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bPS[b]);
    }
    if (__all_sync(0xffffffffu, ok && mbar_wait(bDone, 0, abort_flag))) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        const int col = g * (D / 2) + c * 32;
        uint32_t r[32];
        tmem_ld32(tl + tDQ + col, r);
        tmem_ld_wait();
        if (qg < S) {
          float4* dq4 = reinterpret_cast<float4*>(dQ + ((int64_t)bh * S + qg) * D + col);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dq4[q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]), __uint_as_float(r[4 * q + 2]),
                                 __uint_as_float(r[4 * q + 3]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && *abort_flag) report_error(errw, ERRW_TIMEOUT);
}

// TMA maps of the sequences: full 128-row boxes and 64-row half boxes
struct SeqMaps {
  CUtensorMap q, qh, kh, k, v, vh, o, oh;
};

template <int D>
cudaError_t launch_bwd_d(int64_t BH, int64_t S, const SeqMaps& m, const float* lse, const float* delta, float* dqs,
                         float* dks, float* dvs, int* errw, float scale_log2, float scale, cudaStream_t st) {
  const unsigned n_qt = (unsigned)((S + 127) / 128);
  int smem = KvSmem<D>::kAlloc;
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_kv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  attn_bwd_kv_kernel<D><<<dim3(n_qt, (unsigned)BH), kThreads, smem, st>>>(m.qh, m.k, m.v, m.oh, lse, delta, dks, dvs,
                                                                         errw, (int)S, scale_log2, scale);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  smem = QSmem<D>::kAlloc;
  e = cudaFuncSetAttribute(attn_bwd_q_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  attn_bwd_q_kernel<D><<<dim3(n_qt, (unsigned)BH), kThreads, smem, st>>>(m.q, m.kh, m.vh, m.o, lse, delta, dqs, errw,
                                                                        (int)S, scale_log2, scale);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bwd(int64_t BH, int64_t S, int d, const void* qs, const void* ks, const void* vs,
                            const float* lse, const void* dos, const float* delta, float* dqs, float* dks,
                            float* dvs, int* errw, cudaStream_t st) {
  SeqMaps m;
  if (!make_seq_map(&m.q, qs, BH, S, d, 128) || !make_seq_map(&m.qh, qs, BH, S, d, 64) ||
      !make_seq_map(&m.k, ks, BH, S, d, 128) || !make_seq_map(&m.kh, ks, BH, S, d, 64) ||
      !make_seq_map(&m.v, vs, BH, S, d, 128) || !make_seq_map(&m.vh, vs, BH, S, d, 64) ||
      !make_seq_map(&m.o, dos, BH, S, d, 128) || !make_seq_map(&m.oh, dos, BH, S, d, 64))
    return cudaErrorInvalidValue;
  const double scale = 1.0 / sqrt((double)d);
  const float scale_log2 = (float)(1.4426950408889634 * scale);
  if (d == 128) return launch_bwd_d<128>(BH, S, m, lse, delta, dqs, dks, dvs, errw, scale_log2, (float)scale, st);
  return launch_bwd_d<64>(BH, S, m, lse, delta, dqs, dks, dvs, errw, scale_log2, (float)scale, st);
}

}  // namespace lh
