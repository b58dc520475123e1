// Stage 4 backward: gradients of the dense causal attention over the S-token
// sequence (aitrends.kr summary of Lighthouse Attention, Method step 5: the
// gradient flows back through the attention kernel; the top-k passes none).
//
// With P = softmax(Qs Ks^T / sqrt(d)) (causal) recomputed from the saved LSE,
//   dVs = P^T dOs,  dP = dOs Vs^T,  dS = P * (dP - Delta) / sqrt(d),
//   dQs = dS Ks,    dKs = dS^T Qs,  Delta = rowsum(dOs * Os).
// P^T and dS^T enter their products as bf16 (hi + lo) pairs, so the bf16
// roundings of the probabilities and of dS do not show in the gradients.
//
// One CTA owns a 128-row key/value tile of one (batch, head) and walks the
// query tiles from the diagonal to the end.  Warp roles:
//   warps 0-7  two compute warpgroups; thread (g, t) owns key row t (TMEM lane
//              t) and query columns [64g, 64g+64) of the tile.  One pass turns
//              S^T and dP^T into P^T (hi/lo, written back into the S^T
//              columns of TMEM, where the dV product reads it as its A
//              operand) and dS^T (hi/lo, to shared memory); then each reads
//              half of the tile's dQ from TMEM into shared memory, and one
//              thread adds the tile to dQs with a TMA reduce-add; at the end
//              they write dKs and dVs
//   warp 8     TMA producer: K, V once; Q and dO per query tile, each as
//              soon as the product that last reads it (dK, dV) is done
//   warp 9     MMA issuer (one thread) and TMEM owner
// TMEM columns: S^T/P^T [0,128), dP^T/dQ [128,256), dV [256,256+D), dK [256+D,256+2D).
#include <math.h>

#include "lh_common.cuh"
#include "sm100.cuh"

namespace lh {

bool make_seq_map(CUtensorMap* m, const void* base, int64_t BH, int64_t rows, int D, int box_rows);

// [BH][rows][D] fp32 viewed as (D, rows, BH); box of 32 x box_rows x 1, 128-byte swizzle
bool make_f32_map(CUtensorMap* m, const void* base, int64_t BH, int64_t rows, int D, int box_rows);

namespace {
using namespace sm100;

constexpr int BM = 128;  // query rows per tile
constexpr int BN = 128;  // key rows per CTA
constexpr int kCompute = 256;
constexpr int kThreads = kCompute + 64;

template <int D>
struct BwdSmem {
  static constexpr int kChunk = 128 * 128;
  static constexpr int kTile = D / 64 * kChunk;
  static constexpr int oK = 0;
  static constexpr int oV = oK + kTile;
  static constexpr int oQ = oV + kTile;
  static constexpr int oO = oQ + kTile;          // dO
  static constexpr int oHi = oO + kTile;         // dS^T, bf16 high part; later the fp32 dQ tile
  static constexpr int oLo = oHi + 2 * kChunk;   // bf16 of the remainder
  static constexpr int oVec = oLo + 2 * kChunk;  // LSE*log2e [128], Delta [128]
  static constexpr int oBar = oVec + 1024;
  static constexpr int kBytes = oBar + 256;
  static constexpr int kAlloc = kBytes + 1024;
};

__device__ __forceinline__ void compute_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
// the 128 threads of compute warpgroup g
__device__ __forceinline__ void group_sync(int g) { asm volatile("bar.sync %0, 128;" ::"r"(2 + g) : "memory"); }

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    const __grid_constant__ CUtensorMap tmDQ,
                    const float* __restrict__ LSE, const float* __restrict__ Delta,
                    float* __restrict__ dK, float* __restrict__ dV, int* errw, int S, float scale_log2,
                    float scale) {
  using Lay = BwdSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::oBar);
  uint64_t* bKV = bars + 0;      // K, V landed
  uint64_t* bQ = bars + 1;       // Q_i landed
  uint64_t* bQfree = bars + 2;   // dK product of tile i done: Q buffer free
  uint64_t* bO = bars + 7;       // dO_i landed
  uint64_t* bOfree = bars + 8;   // dV product of tile i done: dO buffer free
  uint64_t* bSdP = bars + 3;     // S^T and dP^T of tile i in TMEM
  uint64_t* bPS = bars + 4;      // P^T in TMEM and dS^T in shared memory (256 arrivals)
  uint64_t* bDQ = bars + 5;      // dQ of tile i in TMEM (all products of tile i done)
  uint64_t* bDQfree = bars + 6;  // dQ read out of TMEM (256 arrivals)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::oBar + 128);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::oBar + 132);
  float* sVec = reinterpret_cast<float*>(smem + Lay::oVec);  // [0,128) LSE*log2e, [128,256) Delta

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_qt = (S + BM - 1) / BM;
  const int kt = (int)blockIdx.x;  // key tile; small kt = most query tiles, launched first
  const int bh = (int)blockIdx.y;
  const int n_q = n_qt - kt;

  if (threadIdx.x == 0) {
    mbar_init(bKV, 1);
    mbar_init(bQ, 1);
    mbar_init(bQfree, 1);
    mbar_init(bO, 1);
    mbar_init(bOfree, 1);
    mbar_init(bSdP, 1);
    mbar_init(bPS, kCompute);
    mbar_init(bDQ, 1);
    mbar_init(bDQfree, kCompute);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  constexpr uint32_t tS = 0, tDP = 128, tDV = 256, tDK = 256 + D;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmO);
      mbar_expect_tx(bKV, 2 * BN * D * 2);
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(smem + Lay::oK + c * Lay::kChunk, &tmK, bKV, c * 64, kt * BN, bh);
        tma_load_3d(smem + Lay::oV + c * Lay::kChunk, &tmV, bKV, c * 64, kt * BN, bh);
      }
      // Q is released by the dK product and dO by the dV product of the
      // previous tile; each reloads as soon as its buffer is free
      for (int it = 0; it < n_q; ++it) {
        const int i = kt + it;
        if (it >= 1 && !mbar_wait(bQfree, (it - 1) & 1, abort_flag)) break;
        mbar_expect_tx(bQ, BM * D * 2);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + Lay::oQ + c * Lay::kChunk, &tmQ, bQ, c * 64, i * BM, bh);
        if (it >= 1 && !mbar_wait(bOfree, (it - 1) & 1, abort_flag)) break;
        mbar_expect_tx(bO, BM * D * 2);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + Lay::oO + c * Lay::kChunk, &tmO, bO, c * 64, i * BM, bh);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idSS = idesc_bf16(128, 128, false, false);
      constexpr uint32_t idKM = idesc_bf16(128, D, false, true);  // A K-major, B MN-major
      constexpr uint32_t idMM = idesc_bf16(128, D, true, true);   // A MN-major, B MN-major
      const uint32_t sK = smem_u32(smem + Lay::oK), sV = smem_u32(smem + Lay::oV);
      const uint32_t sQ = smem_u32(smem + Lay::oQ), sO = smem_u32(smem + Lay::oO);
      const uint32_t sHi = smem_u32(smem + Lay::oHi), sLo = smem_u32(smem + Lay::oLo);
      // base descriptors: an operand at byte offset off is base + (off >> 4)
      const uint64_t kK = sdesc_sw128(sK, 16, 1024), kQ = sdesc_sw128(sQ, 16, 1024);
      const uint64_t kV = sdesc_sw128(sV, 16, 1024), kO = sdesc_sw128(sO, 16, 1024);
      const uint64_t kHi = sdesc_sw128(sHi, 16, 1024), kLo = sdesc_sw128(sLo, 16, 1024);
      const uint64_t mO = sdesc_sw128(sO, Lay::kChunk, 1024), mQ = sdesc_sw128(sQ, Lay::kChunk, 1024);
      const uint64_t mK = sdesc_sw128(sK, Lay::kChunk, 1024);
      const uint64_t mHi = sdesc_sw128(sHi, Lay::kChunk, 1024), mLo = sdesc_sw128(sLo, Lay::kChunk, 1024);
      bool ok = mbar_wait(bKV, 0, abort_flag);
      for (int it = 0; ok && it < n_q; ++it) {
        if (!mbar_wait(bQ, it & 1, abort_flag)) break;
        tc_fence_after();
        // S^T = K Q^T  (M = keys, N = queries, K = d); the S^T columns held P^T of
        // the previous tile, whose dV product was issued before this one
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * Lay::kChunk + (kk & 3) * 32) >> 4;
          umma_bf16(tmem + tS, kK + off, kQ + off, idSS, kk > 0 ? 1u : 0u);
        }
        // dP^T = V dO^T into the dQ columns, once dO has landed and the previous
        // dQ has been read out
        if (!mbar_wait(bO, it & 1, abort_flag)) break;
        if (it >= 1 && !mbar_wait(bDQfree, (it - 1) & 1, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * Lay::kChunk + (kk & 3) * 32) >> 4;
          umma_bf16(tmem + tDP, kV + off, kO + off, idSS, kk > 0 ? 1u : 0u);
        }
        umma_commit(bSdP);
        if (!mbar_wait(bPS, it & 1, abort_flag)) break;
        tc_fence_after();
        // dK += dS^T Q: A = dS^T (hi, lo) K-major from shared memory; then Q is free
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk) {
          const uint32_t aoff = ((kk >> 2) * Lay::kChunk + (kk & 3) * 32) >> 4;
          const uint64_t b = mQ + ((kk * 2048) >> 4);
          umma_bf16(tmem + tDK, kHi + aoff, b, idKM, (it > 0 || kk > 0) ? 1u : 0u);
          umma_bf16(tmem + tDK, kLo + aoff, b, idKM, 1u);
        }
        umma_commit(bQfree);
        // dV += P^T dO: A = P^T (hi, lo) from TMEM, B = dO MN-major (K = queries); then dO is free
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk) {
          const uint32_t a = tmem + tS + (kk >> 1) * 32 + (kk & 1) * 8;
          const uint64_t b = mO + ((kk * 2048) >> 4);
          umma_bf16_tmem_a(tmem + tDV, a, b, idKM, (it > 0 || kk > 0) ? 1u : 0u);
          umma_bf16_tmem_a(tmem + tDV, a + 16, b, idKM, 1u);
        }
        umma_commit(bOfree);
        // dQ = dS K  (M = queries, K = keys, N = d): dS^T read M-major
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint32_t off = (kk * 2048) >> 4;
          umma_bf16(tmem + tDP, mHi + off, mK + off, idMM, kk > 0 ? 1u : 0u);
          umma_bf16(tmem + tDP, mLo + off, mK + off, idMM, 1u);
        }
        umma_commit(bDQ);
      }
    }
  } else {
    // ------------------------------------------------------------ compute warpgroups
    const int ct = threadIdx.x;            // 0..255
    const int g = warp >> 2;               // warpgroup: query columns [64g, 64g+64)
    const int t = (warp & 3) * 32 + lane;  // key row of the tile (TMEM lane)
    const int kv_g = kt * BN + t;
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    uint8_t* sHib = smem + Lay::oHi;
    uint8_t* sLob = smem + Lay::oLo;
    bool ok = true;
    // LSE (ct < 128) or Delta (ct >= 128) of one query row of the tile at q0
    auto vec_of = [&](int q0) -> float {
      const int qg = q0 + (ct & 127);
      if (ct < 128) return qg < S ? LSE[(int64_t)bh * S + qg] * 1.4426950408889634f : INFINITY;
      return qg < S ? Delta[(int64_t)bh * S + qg] : 0.f;
    };
    float vec_next = vec_of(kt * BM);
    for (int it = 0; it < n_q; ++it) {
      const int q0 = (kt + it) * BM;
      const float vec_cur = vec_next;
      if (it + 1 < n_q) vec_next = vec_of(q0 + BM);  // one tile ahead
      compute_sync();  // every thread is done with the previous tile's LSE / Delta
      sVec[ct] = vec_cur;
      compute_sync();
      if (!mbar_wait(bSdP, it & 1, abort_flag)) { ok = false; break; }
      __syncwarp();
      tc_fence_after();
      const bool diag = (it == 0);
#pragma unroll 1
      for (int cc = 0; cc < 2; ++cc) {
        const int c = 2 * g + cc;  // 32-column chunk of the tile
        uint32_t sr[32], dr[32];
        tmem_ld32(tl + tS + c * 32, sr);
        tmem_ld32(tl + tDP + c * 32, dr);
        tmem_ld_wait();
        uint32_t phi[16], plo[16], dhi[16], dlo[16];
        const uint64_t c2 = f2_pack(scale_log2, scale_log2), sc2 = f2_pack(scale, scale);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int qi = c * 32 + e;
          const float2 lse2 = *reinterpret_cast<const float2*>(sVec + qi);
          const float2 del2 = *reinterpret_cast<const float2*>(sVec + 128 + qi);
          float pa, pb;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])), c2, f2_pack(-lse2.x, -lse2.y)),
                    pa, pb);
          pa = fast_exp2(pa);
          pb = fast_exp2(pb);
          if (diag) {
            if (q0 + qi < kv_g) pa = 0.f;
            if (q0 + qi + 1 < kv_g) pb = 0.f;
          }
          const uint64_t p2 = f2_pack(pa, pb);
          const uint64_t diff2 = f2_sub(f2_pack(__uint_as_float(dr[e]), __uint_as_float(dr[e + 1])), f2_pack(del2.x, del2.y));
          float da, db;
          f2_unpack(f2_mul(f2_mul(p2, sc2), diff2), da, db);
          split_bf16x2(pa, pb, phi[e >> 1], plo[e >> 1]);
          split_bf16x2(da, db, dhi[e >> 1], dlo[e >> 1]);
        }
        // P^T over the S^T columns just read: hi in the first 16, lo in the last 16
        tmem_st16(tl + tS + c * 32, phi);
        tmem_st16(tl + tS + c * 32 + 16, plo);
        if (cc == 0) {
          // this group's previous dQ reduce must have read the regions it reuses
          if (t == 0) bulk_wait_read_all();
          group_sync(g);
        }
        // dS^T row t, query columns c*32..c*32+31: 4 chunks of 16 bytes in region c/2 = g
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int ch = (c & 1) * 4 + q;
          const int off = (c >> 1) * Lay::kChunk + t * 128 + ((ch ^ (t & 7)) << 4);
          *reinterpret_cast<uint4*>(sHib + off) = make_uint4(dhi[4 * q], dhi[4 * q + 1], dhi[4 * q + 2], dhi[4 * q + 3]);
          *reinterpret_cast<uint4*>(sLob + off) = make_uint4(dlo[4 * q], dlo[4 * q + 1], dlo[4 * q + 2], dlo[4 * q + 3]);
        }
      }
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bPS);
      // dQ of query row q0 + t, columns [D/2 g, D/2 (g+1)): TMEM -> shared memory,
      // into the two regions (hi and lo, region g) that this group's dS writes
      // use, then one TMA reduce-add per 32-column chunk into dQs, issued by
      // the group; the dS buffers are free once the dQ product is done
      if (!mbar_wait(bDQ, it & 1, abort_flag)) { ok = false; break; }
      __syncwarp();
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        const int col = g * (D / 2) + c * 32;
        uint32_t r[32];
        tmem_ld32(tl + tDP + col, r);
        tmem_ld_wait();
        uint8_t* dst = smem + (c == 0 ? Lay::oHi : Lay::oLo) + g * (128 * 128) + t * 128;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          *reinterpret_cast<uint4*>(dst + ((k ^ (t & 7)) << 4)) = make_uint4(r[4 * k], r[4 * k + 1], r[4 * k + 2], r[4 * k + 3]);
      }
      tc_fence_before();
      mbar_arrive(bDQfree);
      fence_proxy_async_smem();
      group_sync(g);
      if (t == 0) {
        for (int c = 0; c < D / 64; ++c)
          tma_reduce_add_3d(&tmDQ, smem + (c == 0 ? Lay::oHi : Lay::oLo) + g * (128 * 128), g * (D / 2) + c * 32, q0, bh);
        bulk_commit_group();
      }
    }
    if (ok && !*abort_flag) {
      // bDQ of the last tile has completed: dV and dK are final
      __syncwarp();
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
  if (threadIdx.x == 0 || threadIdx.x == 128) bulk_wait_all();  // every dQ reduce has landed
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && *abort_flag) report_error(errw, ERRW_TIMEOUT);
}

}  // namespace

cudaError_t launch_attn_bwd(int64_t BH, int64_t S, int d, const void* qs, const void* ks, const void* vs,
                            const float* lse, const void* dos, const float* delta, float* dqs, float* dks,
                            float* dvs, int* errw, cudaStream_t st) {
  CUtensorMap mq, mk, mv, mo, mdq;
  if (!make_seq_map(&mq, qs, BH, S, d, BM) || !make_seq_map(&mk, ks, BH, S, d, BN) ||
      !make_seq_map(&mv, vs, BH, S, d, BN) || !make_seq_map(&mo, dos, BH, S, d, BM) ||
      !make_f32_map(&mdq, dqs, BH, S, d, BM))
    return cudaErrorInvalidValue;
  const double scale = 1.0 / sqrt((double)d);
  const float scale_log2 = (float)(1.4426950408889634 * scale);
  const dim3 grid((unsigned)((S + BN - 1) / BN), (unsigned)BH);
  if (d == 128) {
    const int smem = BwdSmem<128>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attn_bwd_kernel<128><<<grid, kThreads, smem, st>>>(mq, mk, mv, mo, mdq, lse, delta, dks, dvs, errw, (int)S,
                                                        scale_log2, (float)scale);
  } else {
    const int smem = BwdSmem<64>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attn_bwd_kernel<64><<<grid, kThreads, smem, st>>>(mq, mk, mv, mo, mdq, lse, delta, dks, dvs, errw, (int)S,
                                                       scale_log2, (float)scale);
  }
  return cudaGetLastError();
}

}  // namespace lh
