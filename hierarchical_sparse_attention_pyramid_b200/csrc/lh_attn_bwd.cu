// Stage 4 backward: gradients of the dense causal attention over the S-token
// sequence (aitrends.kr summary of Lighthouse Attention, Method step 5: the
// gradient flows back through the attention kernel; the top-k passes none).
//
// With P = softmax(Qs Ks^T / sqrt(d)) (causal) recomputed from the saved LSE,
//   dVs = P^T dOs,  dP = dOs Vs^T,  dS = P * (dP - Delta) / sqrt(d),
//   dQs = dS Ks,    dKs = dS^T Qs,  Delta = rowsum(dOs * Os).
// dS enters its products as a bf16 (hi + lo) pair, so its rounding does not
// show in dQ and dK.  P enters dV = P^T dO as one fp16 value (11 significant
// bits; P is in [0, 1] and its products with dO are summed with positive
// weights, so no cancellation amplifies that rounding), and dV and dP = dO V^T
// are fp16 products: dOs arrives in fp16 and the dK/dV kernel converts its V
// tile to fp16 in shared memory (both hold bf16 values, exact in fp16 up to
// 65504; larger ones set the range bit of the error word).  The dQ kernel
// converts its dO tile back to bf16 for dP = dO V^T.
//
// Two kernels, each writing its gradient once (no atomics):
//
// attn_bwd_kv_kernel (dKs, dVs) - one CTA per 128-row key tile; it steps over
//   128-query tiles from the diagonal to the end.  For step j the MMA warp
//   computes S^T = K Q_j^T and dP^T = V dO_j^T (N = 128) into TMEM; the
//   compute warpgroups write P^T and dS^T (hi/lo) back over the columns they
//   read, and the MMA warp adds dV += P^T dO_j and dK += dS^T Q_j with both A
//   operands read from TMEM.  The next step's S^T is issued right after dV(j)
//   and its dP^T right after dK(j), so the tensor core works on one step's
//   products while the compute warps turn the other's scores around.  Q_j
//   streams through a 3-slot ring (it is needed first, by S^T(j), and held
//   longest, until dK(j)), dO_j through a 2-slot ring.
//
// attn_bwd_q_kernel (dQs) - one CTA per 128-row query tile; it steps over the
//   128-key tiles up to the diagonal.  S = Q K_j^T runs two tiles ahead into a
//   double-buffered TMEM region and dP = dO V_j^T one tile ahead; the compute
//   warpgroups turn the scores into P as soon as they land, take dP into
//   registers (which frees it for the next tile's dP), then write dS (hi/lo)
//   over the tile's S columns, and dQ += dS K_j reads it from TMEM.  K streams
//   through 3 stages (read by S(j) and, two tiles later, by dQ(j)), V
//   through 2.
//
// Warp roles in both: warps 0-7 two compute warpgroups (thread (g, t) owns
// TMEM lane t and 64 columns of each step: [64g, 64g+64) in the dK/dV kernel,
// the columns [32g, 32g+32) of each 64-column half in the dQ kernel), warp 8
// TMA producer, warp 9 MMA issuer (a converged warp; one elected lane issues)
// and TMEM owner.
#include <math.h>

#include <type_traits>

#include "lh_common.cuh"
#include "sm100.cuh"

namespace lh {

bool make_seq_map(CUtensorMap* m, const void* base, int64_t BH, int64_t rows, int D, int box_rows);

namespace {
using namespace sm100;

constexpr int kCompute = 256;    // dQ kernel: two compute warpgroups
constexpr int kThreads = kCompute + 64;
constexpr int kComputeKV = 512;  // dK/dV kernel: four compute warpgroups
constexpr int kThreadsKV = kComputeKV + 64;
constexpr int kRegion = 128 * 128;  // one [128 rows][64 bf16] SW128 region

__device__ __forceinline__ void compute_sync_kv() { asm volatile("bar.sync 1, 512;" ::: "memory"); }

// P^T / dS (hi, lo) of 32 columns c0..c0+31 of one row as bf16 pairs over the
// 32 TMEM columns they were read from: hi in the first 16, lo in the last 16.
__device__ __forceinline__ void store_pair_chunk(uint32_t taddr, const uint32_t (&hi)[16], const uint32_t (&lo)[16]) {
  tmem_st16(taddr, hi);
  tmem_st16(taddr + 16, lo);
}

// ===========================================================================
// dKs, dVs
// ===========================================================================
// 224 KB of tiles at D = 128: with the vectors and barriers the layout fills
// the 227 KB a CTA can have only without alignment slack, so the kernel
// relies on the dynamic shared memory starting 1024-byte aligned (it does
// when the kernel has no static shared memory) and checks that it does.
template <int D>
struct KvSmem {
  static constexpr int kTile = D / 64 * kRegion;         // one 128-row tile: K, V, Q_j or dO_j
  static constexpr int oK = 0;
  static constexpr int oV = oK + kTile;
  static constexpr int oQ = oV + kTile;                  // 3 slots of Q_j
  static constexpr int oO = oQ + 3 * kTile;              // 2 slots of dO_j
  static constexpr int oVec = oO + 2 * kTile;            // [2][256] floats: LSE*log2e [128], Delta [128]
  static constexpr int oBar = oVec + 2048;
  static constexpr int kBytes = oBar + 256;
  static constexpr int kAlloc = kBytes;
};

template <int D>
__global__ void __launch_bounds__(kThreadsKV, 1)
    attn_bwd_kv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                       const float* __restrict__ LSE, const float* __restrict__ Delta, float* __restrict__ dK,
                       float* __restrict__ dV, int* errw, int S, float scale_log2, float scale, int kt0, int kt1) {
  using Lay = KvSmem<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (reinterpret_cast<uintptr_t>(smem_raw) & 1023) {  // the layout has no slack to align it
    if (threadIdx.x == 0) report_error(errw, ERRW_BOUNDS);
    return;
  }
  uint8_t* smem = smem_raw;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::oBar);
  uint64_t* bKV = bars + 0;        // K, V landed
  uint64_t* bQload = bars + 1;     // [3] Q_j of a slot landed
  uint64_t* bQfree = bars + 4;     // [3] dK product done with a Q slot
  uint64_t* bOload = bars + 7;     // [2] dO_j of a slot landed
  uint64_t* bOfree = bars + 9;     // [2] dV product done with a dO slot
  uint64_t* bS = bars + 11;        // S^T of the step in TMEM
  uint64_t* bDP = bars + 12;       // dP^T of the step in TMEM
  uint64_t* bP = bars + 13;        // P^T written back (one arrival per compute thread)
  uint64_t* bDS = bars + 14;       // dS^T written back (one arrival per compute thread)
  uint64_t* bDone = bars + 15;     // every product done
  uint64_t* bVconv = bars + 16;    // V converted to fp16 in shared memory (one arrival per compute thread)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::oBar + 192);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::oBar + 196);
  float* sVec = reinterpret_cast<float*>(smem + Lay::oVec);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_qt = (S + 127) / 128;
  // one CTA per (key tile, head) of the key tiles [kt0, kt1), tile-major:
  // small kt (most query tiles) of every head is started first, the short
  // tiles fill the tail
  const int BHn = (int)(gridDim.x / (unsigned)(kt1 - kt0));
  const int kt = kt0 + (int)(blockIdx.x / (unsigned)BHn);
  const int bh = (int)(blockIdx.x % (unsigned)BHn);
  const int NJ = n_qt - kt;        // 128-query steps, from the diagonal tile on

  if (threadIdx.x == 0) {
    mbar_init(bKV, 1);
    for (int i = 0; i < 3; ++i) {
      mbar_init(&bQload[i], 1);
      mbar_init(&bQfree[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bOload[i], 1);
      mbar_init(&bOfree[i], 1);
    }
    mbar_init(bS, 1);
    mbar_init(bDP, 1);
    mbar_init(bP, kComputeKV);
    mbar_init(bDS, kComputeKV);
    mbar_init(bDone, 1);
    mbar_init(bVconv, kComputeKV);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 17) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  constexpr uint32_t tS = 0, tDP = 128, tDV = 256, tDK = 256 + D;

  if (warp == 16) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmO);
      mbar_expect_tx(bKV, 2 * 128 * D * 2);
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(smem + Lay::oK + c * kRegion, &tmK, bKV, c * 64, kt * 128, bh);
        tma_load_3d(smem + Lay::oV + c * kRegion, &tmV, bKV, c * 64, kt * 128, bh);
      }
      for (int j = 0; j < NJ; ++j) {
        const int qs = j % 3, os = j & 1;
        const int q0 = (kt + j) * 128;
        if (j >= 3 && !mbar_wait(&bQfree[qs], ((j / 3) - 1) & 1, abort_flag)) break;
        mbar_expect_tx(&bQload[qs], 128 * D * 2);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + Lay::oQ + qs * Lay::kTile + c * kRegion, &tmQ, &bQload[qs], c * 64, q0, bh);
        if (j >= 2 && !mbar_wait(&bOfree[os], ((j >> 1) - 1) & 1, abort_flag)) break;
        mbar_expect_tx(&bOload[os], 128 * D * 2);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + Lay::oO + os * Lay::kTile + c * kRegion, &tmO, &bOload[os], c * 64, q0, bh);
      }
    }
  } else if (warp == 17) {
    // ------------------------------------------------------------ MMA issuer
    // Order per step j: dV(j) once P^T(j) is back, S^T(j+1) (over the P^T
    // columns dV(j) has read: the tensor core runs in issue order), dK(j) once
    // dS^T(j) is back, dP^T(j+1) (over the dS^T columns dK(j) has read).
    {  // the whole warp; one elected lane issues each instruction
      constexpr uint32_t idF = idesc_bf16(128, 128, false, false);  // S^T = K Q^T: N = 128 queries
      constexpr uint32_t idF16 = idesc_f16(128, 128, false, false); // dP^T = V dO^T, fp16 both
      constexpr uint32_t idG = idesc_bf16(128, D, false, true);     // dK: A (dS^T) from TMEM, B MN-major
      constexpr uint32_t idG16 = idesc_f16(128, D, false, true);    // dV: A (P^T, fp16) from TMEM, dO fp16
      const uint32_t sQ = smem_u32(smem + Lay::oQ), sO = smem_u32(smem + Lay::oO);
      const uint64_t kK = sdesc_sw128(smem_u32(smem + Lay::oK), 16, 1024);
      const uint64_t kV = sdesc_sw128(smem_u32(smem + Lay::oV), 16, 1024);
      const uint64_t kQ = sdesc_sw128(sQ, 16, 1024), mQ = sdesc_sw128(sQ, kRegion, 1024);
      const uint64_t kO = sdesc_sw128(sO, 16, 1024), mO = sdesc_sw128(sO, kRegion, 1024);
      auto wait_q = [&](int j) -> bool { return mbar_wait_warp(&bQload[j % 3], (j / 3) & 1, abort_flag); };
      auto wait_o = [&](int j) -> bool { return mbar_wait_warp(&bOload[j & 1], (j >> 1) & 1, abort_flag); };
      auto issue_s = [&](int j) {
        const uint32_t qo = ((j % 3) * Lay::kTile) >> 4;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t at = ((kk >> 2) * kRegion + (kk & 3) * 32) >> 4;
          umma_bf16_w(tmem + tS, kK + at, kQ + qo + at, idF, kk > 0 ? 1u : 0u);
        }
        umma_commit_w(bS);
      };
      auto issue_dp = [&](int j) {
        const uint32_t oo = ((j & 1) * Lay::kTile) >> 4;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t at = ((kk >> 2) * kRegion + (kk & 3) * 32) >> 4;
          umma_bf16_w(tmem + tDP, kV + at, kO + oo + at, idF16, kk > 0 ? 1u : 0u);
        }
        umma_commit_w(bDP);
      };
      bool ok = mbar_wait_warp(bKV, 0, abort_flag) && wait_q(0);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        // dP^T reads V as fp16: after the compute warps have converted it
        ok = wait_o(0) && mbar_wait_warp(bVconv, 0, abort_flag);
      }
      if (ok) {
        tc_fence_after();
        issue_dp(0);
      }
      for (int j = 0; ok && j < NJ; ++j) {
        const uint32_t qo = ((j % 3) * Lay::kTile) >> 4, oo = ((j & 1) * Lay::kTile) >> 4;
        // dV += P^T dO_j (16 queries per MMA: P^T of chunk kk/2, fp16, at +(kk&1)*8)
        if (!mbar_wait_warp(bP, j & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t a = tmem + tS + (kk >> 1) * 32 + (kk & 1) * 8;
          const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
          const uint64_t bo = mO + oo + ((kk * 2048) >> 4);
          umma_bf16_tmem_a_w(tmem + tDV, a, bo, idG16, acc);
        }
        umma_commit_w(&bOfree[j & 1]);  // dV(j) was the last reader of dO_j
        if (j + 1 < NJ) {
          if (!wait_q(j + 1)) { ok = false; break; }
          tc_fence_after();
          issue_s(j + 1);
        }
        // dK += dS^T Q_j
        if (!mbar_wait_warp(bDS, j & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t a = tmem + tDP + (kk >> 1) * 32 + (kk & 1) * 8;
          const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
          const uint64_t bq = mQ + qo + ((kk * 2048) >> 4);
          umma_bf16_tmem_a_w(tmem + tDK, a, bq, idG, acc);
          umma_bf16_tmem_a_w(tmem + tDK, a + 16, bq, idG, 1u);
        }
        umma_commit_w(&bQfree[j % 3]);  // dK(j) was the last reader of Q_j
        if (j + 1 < NJ) {
          if (!wait_o(j + 1)) { ok = false; break; }
          tc_fence_after();
          issue_dp(j + 1);
        }
      }
      if (ok) umma_commit_w(bDone);
    }
  } else {
    // ------------------------------------------------------------ compute warpgroups
    const int ct = threadIdx.x;            // 0..511
    const int g = warp >> 2;               // query columns [32g, 32g+32) of each step
    const int t = (warp & 3) * 32 + lane;  // key row of the tile (TMEM lane)
    const int kv_g = kt * 128 + t;
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    bool ok = true;
    // LSE (ct < 128) or Delta (128 <= ct < 256) of query row ct & 127 of
    // step j, loaded one step ahead and converted when it is stored
    auto vec_row = [&](int j) { return (kt + j) * 128 + (ct & 127); };
    auto vec_raw = [&](int j) -> float {
      const int qg = vec_row(j);
      return qg < S ? ldg_nc_f32((ct < 128 ? LSE : Delta) + (int64_t)bh * S + qg) : 0.f;
    };
    float vec_next = ct < 256 ? vec_raw(0) : 0.f;
    const uint64_t c2 = f2_pack(scale_log2, scale_log2);
    const uint64_t sc2 = f2_pack(scale, scale);
    // V to fp16 in place (the operand type of dP^T = V dO^T): every thread
    // converts its share of the tile once the TMA has landed it
    ok = mbar_wait(bKV, 0, abort_flag);
    if (ok) {
      constexpr int kPer = Lay::kTile / 16 / kComputeKV;  // 16-byte words per thread
      uint4* vt = reinterpret_cast<uint4*>(smem + Lay::oV);
      bool in_range = true;
#pragma unroll
      for (int w = 0; w < kPer; ++w) {
        uint4 u = vt[ct + w * kComputeKV];
        uint32_t* e = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float lo = __uint_as_float(e[c] << 16), hi = __uint_as_float(e[c] & 0xffff0000u);
          in_range &= fabsf(lo) <= 65504.f && fabsf(hi) <= 65504.f;
          e[c] = pack_f16x2(lo, hi);
        }
        vt[ct + w * kComputeKV] = u;
      }
      if (!in_range) report_error(errw, ERRW_RANGE);
      fence_proxy_async_smem();  // the tensor core reads the tile through the async proxy
    }
    mbar_arrive(bVconv);
    for (int j = 0; j < NJ; ++j) {
      const int b = j & 1;
      const float vec_cur = vec_next;
      if (ct < 256 && j + 1 < NJ) vec_next = vec_raw(j + 1);
      if (ct < 128) sVec[b * 256 + ct] = vec_row(j) < S ? vec_cur * 1.4426950408889634f : INFINITY;
      else if (ct < 256) sVec[b * 256 + ct] = vec_cur;
      compute_sync_kv();
      const float* lse = sVec + b * 256;
      const float* del = lse + 128;
      const int q0 = (kt + j) * 128;
      const bool diag = j == 0;  // the diagonal query tile
      // warp-uniform outcome for the collective TMEM accesses; after a failed
      // wait the loop keeps its compute_sync_kv count and skips the work
      ok = __all_sync(0xffffffffu, ok && mbar_wait(bS, j & 1, abort_flag));
      if (!ok) continue;
      tc_fence_after();
      // P^T in fp16 over the first 16 of the 32 S^T columns just read; dV
      // starts on it while dP^T is still being computed
      float p[32];
      {
        uint32_t sr[32];
        tmem_ld32(tl + tS + g * 32, sr);
        tmem_ld_wait();
        uint32_t ph[16];
        // queries before the key are masked on the diagonal tile only
        auto p_pass = [&](auto masked) {
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int qi = g * 32 + e;
            const float2 l2 = *reinterpret_cast<const float2*>(lse + qi);
            float pa, pb;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])), c2, f2_pack(-l2.x, -l2.y)),
                      pa, pb);
            pa = fast_exp2(pa);
            pb = fast_exp2(pb);
            if constexpr (decltype(masked)::value) {
              if (q0 + qi < kv_g) pa = 0.f;
              if (q0 + qi + 1 < kv_g) pb = 0.f;
            }
            p[e] = pa;
            p[e + 1] = pb;
            ph[e >> 1] = pack_f16x2(pa, pb);
          }
        };
        if (diag) p_pass(std::true_type{});
        else p_pass(std::false_type{});
        tmem_st16(tl + tS + g * 32, ph);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bP);
      ok = __all_sync(0xffffffffu, mbar_wait(bDP, j & 1, abort_flag));
      if (!ok) continue;
      tc_fence_after();
      // dS^T = P^T (dP^T - Delta) / sqrt(d) as bf16 pairs over the dP^T columns
      {
        uint32_t dr[32];
        tmem_ld32(tl + tDP + g * 32, dr);
        tmem_ld_wait();
        uint32_t dhi[16], dlo[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float2 d2 = *reinterpret_cast<const float2*>(del + g * 32 + e);
          const uint64_t diff2 =
              f2_sub(f2_pack(__uint_as_float(dr[e]), __uint_as_float(dr[e + 1])), f2_pack(d2.x, d2.y));
          float da, db;
          f2_unpack(f2_mul(f2_mul(f2_pack(p[e], p[e + 1]), sc2), diff2), da, db);
          split_bf16x2(da, db, dhi[e >> 1], dlo[e >> 1]);
        }
        store_pair_chunk(tl + tDP + g * 32, dhi, dlo);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bDS);
    }
    // dV and dK of this thread's key row, columns [g D/4, (g+1) D/4)
    if (__all_sync(0xffffffffu, ok && mbar_wait(bDone, 0, abort_flag))) {
      tc_fence_after();
      constexpr int CW = D / 4;
      uint32_t rv[CW], rk[CW];
      if constexpr (CW == 32) {
        tmem_ld32(tl + tDV + g * CW, rv);
        tmem_ld32(tl + tDK + g * CW, rk);
      } else {
        tmem_ld16(tl + tDV + g * CW, rv);
        tmem_ld16(tl + tDK + g * CW, rk);
      }
      tmem_ld_wait();
      if (kv_g < S) {
        float4* dv4 = reinterpret_cast<float4*>(dV + ((int64_t)bh * S + kv_g) * D + g * CW);
        float4* dk4 = reinterpret_cast<float4*>(dK + ((int64_t)bh * S + kv_g) * D + g * CW);
#pragma unroll
        for (int q = 0; q < CW / 4; ++q) {
          dv4[q] = make_float4(__uint_as_float(rv[4 * q]), __uint_as_float(rv[4 * q + 1]),
                               __uint_as_float(rv[4 * q + 2]), __uint_as_float(rv[4 * q + 3]));
          dk4[q] = make_float4(__uint_as_float(rk[4 * q]), __uint_as_float(rk[4 * q + 1]),
                               __uint_as_float(rk[4 * q + 2]), __uint_as_float(rk[4 * q + 3]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 17) {
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
  static constexpr int kTile = D / 64 * kRegion;  // one 128-row tile of Q, dO, K or V
  static constexpr int oQ = 0;
  static constexpr int oO = oQ + kTile;      // dO
  static constexpr int oK = oO + kTile;      // 3 stages: K_j is read by S(j) two steps before dQ(j)
  static constexpr int oV = oK + 3 * kTile;  // 2 stages
  static constexpr int oBar = oV + 2 * kTile;
  static constexpr int kBytes = oBar + 256;
  static constexpr int kAlloc = kBytes + 1024;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_q_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                      const float* __restrict__ LSE, const float* __restrict__ Delta, float* __restrict__ dQ,
                      int* errw, int S, float scale_log2, float scale, int qt0, int qt1) {
  using Lay = QSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::oBar);
  uint64_t* bQO = bars + 0;     // Q, dO landed
  uint64_t* bK = bars + 1;      // [3] K tile of a stage landed
  uint64_t* bV = bars + 4;      // [2] V tile of a stage landed
  uint64_t* bKfree = bars + 6;  // [3] the dQ product is done with a K stage
  uint64_t* bVfree = bars + 9;  // [2] the dP product is done with a V stage
  uint64_t* bS = bars + 11;     // [2] S of a key tile in TMEM buffer
  uint64_t* bDPread = bars + 13;  // dP of the key tile is in registers (256 arrivals)
  uint64_t* bDP = bars + 15;    // dP of the current key tile in TMEM
  uint64_t* bPS = bars + 16;    // dS written over the tile's S columns (256 arrivals)
  uint64_t* bDone = bars + 17;  // every product done
  uint64_t* bOconv = bars + 18; // dO converted to bf16 in shared memory (one arrival per compute thread)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::oBar + 192);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::oBar + 196);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // one CTA per (query tile, head) of the query tiles [qt0, qt1), tile-major
  // with the longest rows first
  const int BHn = (int)(gridDim.x / (unsigned)(qt1 - qt0));
  const int qt = qt1 - 1 - (int)(blockIdx.x / (unsigned)BHn);
  const int bh = (int)(blockIdx.x % (unsigned)BHn);
  const int NJ = qt + 1;  // key tiles up to the diagonal

  if (threadIdx.x == 0) {
    mbar_init(bQO, 1);
    for (int i = 0; i < 3; ++i) {
      mbar_init(&bK[i], 1);
      mbar_init(&bKfree[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bV[i], 1);
      mbar_init(&bVfree[i], 1);
      mbar_init(&bS[i], 1);
    }
    mbar_init(bDPread, kCompute);
    mbar_init(bDP, 1);
    mbar_init(bPS, kCompute);
    mbar_init(bDone, 1);
    mbar_init(bOconv, kCompute);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  constexpr uint32_t tS = 0, tDP = 256, tDQ = 384;  // S, then dS (hi/lo): [2] x 128 columns; dP: 128

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    // K_j to stage j % 3 once the dQ product of key tile j-3 is done, V_j to
    // stage j & 1 once the dP product of key tile j-2 is done
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_expect_tx(bQO, 2 * 128 * D * 2);
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(smem + Lay::oQ + c * kRegion, &tmQ, bQO, c * 64, qt * 128, bh);
        tma_load_3d(smem + Lay::oO + c * kRegion, &tmO, bQO, c * 64, qt * 128, bh);
      }
      for (int j = 0; j < NJ; ++j) {
        const int sk = j % 3, sv = j & 1;
        if (j >= 3 && !mbar_wait(&bKfree[sk], ((j / 3) - 1) & 1, abort_flag)) break;
        mbar_expect_tx(&bK[sk], 128 * D * 2);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + Lay::oK + sk * Lay::kTile + c * kRegion, &tmK, &bK[sk], c * 64, j * 128, bh);
        if (j >= 2 && !mbar_wait(&bVfree[sv], ((j >> 1) - 1) & 1, abort_flag)) break;
        mbar_expect_tx(&bV[sv], 128 * D * 2);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + Lay::oV + sv * Lay::kTile + c * kRegion, &tmV, &bV[sv], c * 64, j * 128, bh);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    // Per key tile j: dP(j+1) = dO V_{j+1}^T as soon as the compute warps hold
    // dP(j) in registers, then dQ += dS(j) K_j once dS(j) is written over
    // tile j's S columns, then S(j+2) = Q K_{j+2}^T into that S buffer (after
    // dQ(j) has read it: the tensor core runs in issue order).  The scores
    // are two tiles ahead of the softmax-gradient pass and dP one tile ahead.
    {  // the whole warp; one elected lane issues each instruction
      constexpr uint32_t idF = idesc_bf16(128, 128, false, false);  // S, dP: N = 128 keys
      constexpr uint32_t idG = idesc_bf16(128, D, false, true);     // dQ: A from TMEM, B MN-major
      const uint64_t kQ = sdesc_sw128(smem_u32(smem + Lay::oQ), 16, 1024);
      const uint64_t kO = sdesc_sw128(smem_u32(smem + Lay::oO), 16, 1024);
      const uint64_t kK = sdesc_sw128(smem_u32(smem + Lay::oK), 16, 1024);
      const uint64_t kV = sdesc_sw128(smem_u32(smem + Lay::oV), 16, 1024);
      const uint64_t mK = sdesc_sw128(smem_u32(smem + Lay::oK), kRegion, 1024);
      auto issue_s = [&](int j) {  // S(j) = Q K_j^T into buffer j & 1
        const uint32_t ko = ((j % 3) * Lay::kTile) >> 4;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * kRegion + (kk & 3) * 32) >> 4;
          umma_bf16_w(tmem + tS + (j & 1) * 128, kQ + off, kK + ko + off, idF, kk > 0 ? 1u : 0u);
        }
        umma_commit_w(&bS[j & 1]);
      };
      auto issue_dp = [&](int j) {  // dP(j) = dO V_j^T; then V_j is free
        const uint32_t vo = ((j & 1) * Lay::kTile) >> 4;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * kRegion + (kk & 3) * 32) >> 4;
          umma_bf16_w(tmem + tDP, kO + off, kV + vo + off, idF, kk > 0 ? 1u : 0u);
        }
        umma_commit_w(bDP);
        umma_commit_w(&bVfree[j & 1]);
      };
      bool ok = mbar_wait_warp(bQO, 0, abort_flag) && mbar_wait_warp(&bK[0], 0, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        // dP reads dO as bf16: after the compute warps have converted it
        ok = mbar_wait_warp(&bV[0], 0, abort_flag) && mbar_wait_warp(bOconv, 0, abort_flag);
      }
      if (ok) {
        tc_fence_after();
        issue_dp(0);
        if (NJ > 1 && (ok = mbar_wait_warp(&bK[1], 0, abort_flag))) {
          tc_fence_after();
          issue_s(1);
        }
      }
      for (int j = 0; ok && j < NJ; ++j) {
        if (j + 1 < NJ) {
          if (!mbar_wait_warp(&bV[(j + 1) & 1], ((j + 1) >> 1) & 1, abort_flag)) { ok = false; break; }
          if (!mbar_wait_warp(bDPread, j & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_dp(j + 1);
        }
        if (!mbar_wait_warp(bPS, j & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint64_t mk = mK + (((j % 3) * Lay::kTile) >> 4);
        const uint32_t sb = tmem + tS + (j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // 16 keys per step; hi of chunk kk/2 at +(kk&1)*8, lo at +16
          const uint32_t a = sb + (kk >> 1) * 32 + (kk & 1) * 8;
          const uint64_t bk = mk + ((kk * 2048) >> 4);
          umma_bf16_tmem_a_w(tmem + tDQ, a, bk, idG, (j > 0 || kk > 0) ? 1u : 0u);
          umma_bf16_tmem_a_w(tmem + tDQ, a + 16, bk, idG, 1u);
        }
        umma_commit_w(&bKfree[j % 3]);
        if (j + 2 < NJ) {
          if (!mbar_wait_warp(&bK[(j + 2) % 3], ((j + 2) / 3) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_s(j + 2);
        }
      }
      if (ok) umma_commit_w(bDone);
    }
  } else {
    // ------------------------------------------------------------ compute warpgroups
    const int g = warp >> 2;               // keys [64g, 64g+64) of every key tile
    const int t = (warp & 3) * 32 + lane;  // query row of the tile (TMEM lane)
    const int qg = qt * 128 + t;
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const float lse = qg < S ? LSE[(int64_t)bh * S + qg] * 1.4426950408889634f : INFINITY;
    const float del = qg < S ? Delta[(int64_t)bh * S + qg] : 0.f;
    const uint64_t c2 = f2_pack(scale_log2, scale_log2), sc2 = f2_pack(scale, scale);
    const uint64_t nl2 = f2_pack(-lse, -lse), d2 = f2_pack(del, del);
    // dO arrives in fp16 (the operand type of the dK/dV kernel); its values
    // are bf16 values, so converting the tile back to bf16 in place is exact
    bool ok = mbar_wait(bQO, 0, abort_flag);
    if (ok) {
      constexpr int kPer = Lay::kTile / 16 / kCompute;  // 16-byte words per thread
      uint4* ot = reinterpret_cast<uint4*>(smem + Lay::oO);
#pragma unroll
      for (int w = 0; w < kPer; ++w) {
        uint4 u = ot[threadIdx.x + w * kCompute];
        uint32_t* e = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&e[c]));
          e[c] = pack_bf16x2(f.x, f.y);
        }
        ot[threadIdx.x + w * kCompute] = u;
      }
      fence_proxy_async_smem();  // the tensor core reads the tile through the async proxy
    }
    mbar_arrive(bOconv);
    for (int j = 0; j < NJ; ++j) {
      const int b = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&bS[b], (j >> 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      // P = 2^(s*scale*log2e - lse*log2e) of this thread's 64 keys
      uint32_t r[2][32];
      tmem_ld32(tl + tS + b * 128 + g * 64, r[0]);
      tmem_ld32(tl + tS + b * 128 + g * 64 + 32, r[1]);
      tmem_ld_wait();
      // keys after the row are masked on the diagonal tile only
      float p[2][32];
      auto p_pass = [&](auto masked) {
        const int limit = t - g * 64;
#pragma unroll
        for (int ch = 0; ch < 2; ++ch)
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float pa, pb;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(r[ch][e]), __uint_as_float(r[ch][e + 1])), c2, nl2), pa, pb);
            pa = fast_exp2(pa);
            pb = fast_exp2(pb);
            if constexpr (decltype(masked)::value) {
              pa = ch * 32 + e > limit ? 0.f : pa;
              pb = ch * 32 + e + 1 > limit ? 0.f : pb;
            }
            p[ch][e] = pa;
            p[ch][e + 1] = pb;
          }
      };
      if (j == qt) p_pass(std::true_type{});
      else p_pass(std::false_type{});
      ok = __all_sync(0xffffffffu, mbar_wait(bDP, j & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      // dS = P (dP - Delta) / sqrt(d) as a bf16 pair over this tile's S
      // columns (read into registers above): per 32 keys, hi in the first 16
      // columns and lo in the last 16.  dP is released as soon as it is in
      // registers, so the next tile's dP can be computed meanwhile.
      uint32_t dr[2][32];
      tmem_ld32(tl + tDP + g * 64, dr[0]);
      tmem_ld32(tl + tDP + g * 64 + 32, dr[1]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(bDPread);
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t dhi[16], dlo[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const uint64_t diff2 = f2_sub(f2_pack(__uint_as_float(dr[ch][e]), __uint_as_float(dr[ch][e + 1])), d2);
          float da, db;
          f2_unpack(f2_mul(f2_mul(f2_pack(p[ch][e], p[ch][e + 1]), sc2), diff2), da, db);
          split_bf16x2(da, db, dhi[e >> 1], dlo[e >> 1]);
        }
        store_pair_chunk(tl + tS + b * 128 + g * 64 + ch * 32, dhi, dlo);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bPS);
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

// TMA maps of the sequences, 128-row boxes
struct SeqMaps {
  CUtensorMap q, k, v, o;
};

template <int D>
cudaError_t launch_bwd_d(int64_t BH, int64_t S, const SeqMaps& m, const float* lse, const float* delta, float* dqs,
                         float* dks, float* dvs, int* errw, float scale_log2, float scale, cudaStream_t st,
                         int64_t qt0, int64_t qt1, int64_t kt0, int64_t kt1) {
  // dK/dV of the key tiles [kt0, kt1), dQ of the query tiles [qt0, qt1); an
  // empty window launches nothing
  cudaError_t e;
  if (kt1 > kt0) {
    if ((kt1 - kt0) * BH > 0x7fffffffll) return cudaErrorInvalidConfiguration;  // one grid dimension
    const int smem = KvSmem<D>::kAlloc;
    e = cudaFuncSetAttribute(attn_bwd_kv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attn_bwd_kv_kernel<D><<<dim3((unsigned)((kt1 - kt0) * BH)), kThreadsKV, smem, st>>>(
        m.q, m.k, m.v, m.o, lse, delta, dks, dvs, errw, (int)S, scale_log2, scale, (int)kt0, (int)kt1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (qt1 > qt0) {
    if ((qt1 - qt0) * BH > 0x7fffffffll) return cudaErrorInvalidConfiguration;
    const int smem = QSmem<D>::kAlloc;
    e = cudaFuncSetAttribute(attn_bwd_q_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attn_bwd_q_kernel<D><<<dim3((unsigned)((qt1 - qt0) * BH)), kThreads, smem, st>>>(
        m.q, m.k, m.v, m.o, lse, delta, dqs, errw, (int)S, scale_log2, scale, (int)qt0, (int)qt1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_attn_bwd(int64_t BH, int64_t S, int d, const void* qs, const void* ks, const void* vs,
                            const float* lse, const void* dos, const float* delta, float* dqs, float* dks,
                            float* dvs, int* errw, cudaStream_t st, int64_t qt0, int64_t qt1, int64_t kt0,
                            int64_t kt1) {
  const int64_t n_qt = (S + 127) / 128;
  if (qt1 < 0) qt1 = n_qt;
  if (kt1 < 0) kt1 = n_qt;
  if (qt0 < 0 || qt0 > qt1 || qt1 > n_qt || kt0 < 0 || kt0 > kt1 || kt1 > n_qt) return cudaErrorInvalidValue;
  SeqMaps m;
  if (!make_seq_map(&m.q, qs, BH, S, d, 128) || !make_seq_map(&m.k, ks, BH, S, d, 128) ||
      !make_seq_map(&m.v, vs, BH, S, d, 128) || !make_seq_map(&m.o, dos, BH, S, d, 128))
    return cudaErrorInvalidValue;
  const double scale = 1.0 / sqrt((double)d);
  const float scale_log2 = (float)(1.4426950408889634 * scale);
  if (d == 128)
    return launch_bwd_d<128>(BH, S, m, lse, delta, dqs, dks, dvs, errw, scale_log2, (float)scale, st, qt0, qt1, kt0, kt1);
  return launch_bwd_d<64>(BH, S, m, lse, delta, dqs, dks, dvs, errw, scale_log2, (float)scale, st, qt0, qt1, kt0, kt1);
}

}  // namespace lh
