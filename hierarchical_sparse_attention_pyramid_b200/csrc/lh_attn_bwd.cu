// Stage 4 backward: gradients of the dense causal attention over the S-token
// sequence (aitrends.kr summary of Lighthouse Attention, Method step 5: the
// gradient flows back through the attention kernel; the top-k passes none).
//
// With P = softmax(Qs Ks^T / sqrt(d)) (causal) recomputed from the saved LSE,
//   dVs = P^T dOs,  dP = dOs Vs^T,  dS = P * (dP - Delta) / sqrt(d),
//   dQs = dS Ks,    dKs = dS^T Qs,  Delta = rowsum(dOs * Os).
//
// One CTA owns a 128-row key/value tile of one (batch, head) and walks the
// query tiles from the diagonal to the end.  Warp roles:
//   warps 0-3  thread t owns key row t for S^T/dP^T (TMEM lane t): writes
//              P^T, then dS^T, to shared memory as bf16 hi + lo pairs (so the
//              products keep fp32-level accuracy), then reads dQ row t of the
//              query tile from TMEM and adds it to dQs with fp32 vector
//              atomics; at the end writes dKs and dVs rows
//   warp 4     TMA producer: K, V once; Q and dO per query tile
//   warp 5     MMA issuer (one thread) and TMEM owner
// TMEM columns: S^T [0,128), dP^T / dQ [128,256), dV [256,256+D), dK [256+D,256+2D).
#include <math.h>

#include "lh_common.cuh"
#include "sm100.cuh"

namespace lh {

bool make_seq_map(CUtensorMap* m, const void* base, int64_t BH, int64_t rows, int D, int box_rows);

namespace {
using namespace sm100;

constexpr int BM = 128;  // query rows per tile
constexpr int BN = 128;  // key rows per CTA
constexpr int kThreads = 192;

template <int D>
struct BwdSmem {
  static constexpr int kChunk = 128 * 128;
  static constexpr int kTile = D / 64 * kChunk;
  static constexpr int oK = 0;
  static constexpr int oV = oK + kTile;
  static constexpr int oQ = oV + kTile;
  static constexpr int oO = oQ + kTile;  // dO
  static constexpr int oHi = oO + kTile;        // P^T, then dS^T: bf16 high part
  static constexpr int oLo = oHi + 2 * kChunk;  // bf16 of the remainder
  static constexpr int oVec = oLo + 2 * kChunk;  // LSE*log2e [128], Delta [128]
  static constexpr int oBar = oVec + 1024;
  static constexpr int kBytes = oBar + 256;
  static constexpr int kAlloc = kBytes + 1024;
};

__device__ __forceinline__ void wg_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    const float* __restrict__ LSE, const float* __restrict__ Delta, float* __restrict__ dQ,
                    float* __restrict__ dK, float* __restrict__ dV, int* errw, int S, float scale_log2,
                    float scale) {
  using Lay = BwdSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::oBar);
  uint64_t* bKV = bars + 0;     // K, V landed
  uint64_t* bQO = bars + 1;     // Q_i, dO_i landed
  uint64_t* bSdP = bars + 2;    // S^T and dP^T in TMEM
  uint64_t* bP = bars + 3;      // P^T hi/lo in shared memory (128 arrivals)
  uint64_t* bMM = bars + 4;     // dK, dQ MMAs of the tile done
  uint64_t* bDQfree = bars + 5; // dQ read out of TMEM (128 arrivals)
  uint64_t* bPfree = bars + 6;  // dV MMAs done: the hi/lo buffers may take dS^T
  uint64_t* bDS = bars + 7;     // dS^T hi/lo in shared memory (128 arrivals)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::oBar + 128);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::oBar + 132);
  float* sLSE = reinterpret_cast<float*>(smem + Lay::oVec);
  float* sDel = sLSE + 128;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_qt = (S + BM - 1) / BM;
  const int kt = (int)blockIdx.x;  // key tile; small kt = most query tiles, launched first
  const int bh = (int)blockIdx.y;
  const int n_q = n_qt - kt;

  if (threadIdx.x == 0) {
    mbar_init(bKV, 1);
    mbar_init(bQO, 1);
    mbar_init(bSdP, 1);
    mbar_init(bP, 128);
    mbar_init(bMM, 1);
    mbar_init(bDQfree, 128);
    mbar_init(bPfree, 1);
    mbar_init(bDS, 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  constexpr uint32_t tS = 0, tDP = 128, tDV = 256, tDK = 256 + D;

  if (warp == 4) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmO);
      mbar_expect_tx(bKV, 2 * BN * D * 2);
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(smem + Lay::oK + c * Lay::kChunk, &tmK, bKV, c * 64, kt * BN, bh);
        tma_load_3d(smem + Lay::oV + c * Lay::kChunk, &tmV, bKV, c * 64, kt * BN, bh);
      }
      for (int it = 0; it < n_q; ++it) {
        const int i = kt + it;
        if (it >= 1 && !mbar_wait(bMM, (it - 1) & 1, abort_flag)) break;
        mbar_expect_tx(bQO, 2 * BM * D * 2);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(smem + Lay::oQ + c * Lay::kChunk, &tmQ, bQO, c * 64, i * BM, bh);
          tma_load_3d(smem + Lay::oO + c * Lay::kChunk, &tmO, bQO, c * 64, i * BM, bh);
        }
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      constexpr uint32_t idSS = idesc_bf16(128, 128, false, false);
      constexpr uint32_t idKM = idesc_bf16(128, D, false, true);  // A K-major, B MN-major
      constexpr uint32_t idMM = idesc_bf16(128, D, true, true);   // A MN-major, B MN-major
      const uint32_t sK = smem_u32(smem + Lay::oK), sV = smem_u32(smem + Lay::oV);
      const uint32_t sQ = smem_u32(smem + Lay::oQ), sO = smem_u32(smem + Lay::oO);
      const uint32_t sHi = smem_u32(smem + Lay::oHi), sLo = smem_u32(smem + Lay::oLo);
      bool ok = mbar_wait(bKV, 0, abort_flag);
      for (int it = 0; ok && it < n_q; ++it) {
        if (!mbar_wait(bQO, it & 1, abort_flag)) break;
        tc_fence_after();
        // S^T = K Q^T  (M = keys, N = queries, K = d)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * Lay::kChunk + (kk & 3) * 32;
          umma_bf16(tmem + tS, sdesc_sw128(sK + off, 16, 1024), sdesc_sw128(sQ + off, 16, 1024), idSS,
                    kk > 0 ? 1u : 0u);
        }
        // dP^T = V dO^T into the dQ region, once the previous dQ has been read out
        if (it >= 1 && !mbar_wait(bDQfree, (it - 1) & 1, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * Lay::kChunk + (kk & 3) * 32;
          umma_bf16(tmem + tDP, sdesc_sw128(sV + off, 16, 1024), sdesc_sw128(sO + off, 16, 1024), idSS,
                    kk > 0 ? 1u : 0u);
        }
        umma_commit(bSdP);
        if (!mbar_wait(bP, it & 1, abort_flag)) break;
        tc_fence_after();
        // dV += P^T dO   (M = keys, K = queries, N = d), P^T = hi + lo
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk) {
          const uint32_t aoff = (kk >> 2) * Lay::kChunk + (kk & 3) * 32;
          const uint64_t b = sdesc_sw128(sO + kk * 2048, Lay::kChunk, 1024);
          umma_bf16(tmem + tDV, sdesc_sw128(sHi + aoff, 16, 1024), b, idKM, (it > 0 || kk > 0) ? 1u : 0u);
          umma_bf16(tmem + tDV, sdesc_sw128(sLo + aoff, 16, 1024), b, idKM, 1u);
        }
        umma_commit(bPfree);
        if (!mbar_wait(bDS, it & 1, abort_flag)) break;
        tc_fence_after();
        // dK += dS^T Q   (M = keys, K = queries, N = d), dS^T = hi + lo
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk) {
          const uint32_t aoff = (kk >> 2) * Lay::kChunk + (kk & 3) * 32;
          const uint64_t b = sdesc_sw128(sQ + kk * 2048, Lay::kChunk, 1024);
          umma_bf16(tmem + tDK, sdesc_sw128(sHi + aoff, 16, 1024), b, idKM, (it > 0 || kk > 0) ? 1u : 0u);
          umma_bf16(tmem + tDK, sdesc_sw128(sLo + aoff, 16, 1024), b, idKM, 1u);
        }
        // dQ = dS K  (M = queries, K = keys, N = d): dS^T read M-major
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint32_t off = kk * 2048;
          const uint64_t b = sdesc_sw128(sK + off, Lay::kChunk, 1024);
          umma_bf16(tmem + tDP, sdesc_sw128(sHi + off, Lay::kChunk, 1024), b, idMM, kk > 0 ? 1u : 0u);
          umma_bf16(tmem + tDP, sdesc_sw128(sLo + off, Lay::kChunk, 1024), b, idMM, 1u);
        }
        umma_commit(bMM);
      }
    }
  } else {
    // ------------------------------------------------------------ compute warpgroup
    const int t = threadIdx.x;  // 0..127
    const int kv_g = kt * BN + t;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    uint8_t* sHib = smem + Lay::oHi;
    uint8_t* sLob = smem + Lay::oLo;
    bool ok = true;
    // write 32 consecutive query columns (chunk c) of this key row as bf16 hi + lo
    auto put_row_chunk = [&](int c, const float (&x)[32]) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a = x[8 * q + 2 * e], b = x[8 * q + 2 * e + 1];
          const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
          hi[e] = *reinterpret_cast<const uint32_t*>(&h);
          lo[e] = pack_bf16x2(a - __low2float(h), b - __high2float(h));
        }
        const int ch = (c & 1) * 4 + q;  // 16-byte chunk within the 128-byte row
        const int off = (c >> 1) * Lay::kChunk + t * 128 + ((ch ^ (t & 7)) << 4);
        *reinterpret_cast<uint4*>(sHib + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(sLob + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
    };
    for (int it = 0; it < n_q; ++it) {
      const int q0 = (kt + it) * BM;
      wg_sync();  // every thread is done with the previous tile's LSE / Delta
      {
        const int qg = q0 + t;
        sLSE[t] = qg < S ? LSE[(int64_t)bh * S + qg] * 1.4426950408889634f : INFINITY;
        sDel[t] = qg < S ? Delta[(int64_t)bh * S + qg] : 0.f;
      }
      wg_sync();
      if (!mbar_wait(bSdP, it & 1, abort_flag)) { ok = false; break; }
      __syncwarp();
      tc_fence_after();
      // pass 1: P^T
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t sr[32];
        tmem_ld32(tl + tS + c * 32, sr);
        tmem_ld_wait();
        float pv[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int qi = c * 32 + e;
          pv[e] = (q0 + qi) >= kv_g ? exp2f(__uint_as_float(sr[e]) * scale_log2 - sLSE[qi]) : 0.f;
        }
        put_row_chunk(c, pv);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bP);
      // pass 2: dS^T, once the dV MMAs have read P^T
      if (!mbar_wait(bPfree, it & 1, abort_flag)) { ok = false; break; }
      __syncwarp();
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t sr[32], dr[32];
        tmem_ld32(tl + tS + c * 32, sr);
        tmem_ld32(tl + tDP + c * 32, dr);
        tmem_ld_wait();
        float dv[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int qi = c * 32 + e;
          const float p = (q0 + qi) >= kv_g ? exp2f(__uint_as_float(sr[e]) * scale_log2 - sLSE[qi]) : 0.f;
          dv[e] = p * (__uint_as_float(dr[e]) - sDel[qi]) * scale;
        }
        put_row_chunk(c, dv);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bDS);
      // dQ of query row q0 + t
      if (!mbar_wait(bMM, it & 1, abort_flag)) { ok = false; break; }
      __syncwarp();
      tc_fence_after();
      const int qg = q0 + t;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tl + tDP + c * 32, r);
        tmem_ld_wait();
        if (qg < S) {
          float4* dst = reinterpret_cast<float4*>(dQ + ((int64_t)bh * S + qg) * D + c * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            atomicAdd(dst + q, make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                           __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3])));
        }
      }
      tc_fence_before();
      mbar_arrive(bDQfree);
    }
    if (ok && !*abort_flag) {
      // bMM of the last tile has completed: dV and dK are final
      __syncwarp();
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t rv[32], rk[32];
        tmem_ld32(tl + tDV + c * 32, rv);
        tmem_ld32(tl + tDK + c * 32, rk);
        tmem_ld_wait();
        if (kv_g < S) {
          float4* dv4 = reinterpret_cast<float4*>(dV + ((int64_t)bh * S + kv_g) * D + c * 32);
          float4* dk4 = reinterpret_cast<float4*>(dK + ((int64_t)bh * S + kv_g) * D + c * 32);
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
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && *abort_flag) report_error(errw, ERRW_TIMEOUT);
}

}  // namespace

cudaError_t launch_attn_bwd(int64_t BH, int64_t S, int d, const void* qs, const void* ks, const void* vs,
                            const float* lse, const void* dos, const float* delta, float* dqs, float* dks,
                            float* dvs, int* errw, cudaStream_t st) {
  CUtensorMap mq, mk, mv, mo;
  if (!make_seq_map(&mq, qs, BH, S, d, BM) || !make_seq_map(&mk, ks, BH, S, d, BN) ||
      !make_seq_map(&mv, vs, BH, S, d, BN) || !make_seq_map(&mo, dos, BH, S, d, BM))
    return cudaErrorInvalidValue;
  const double scale = 1.0 / sqrt((double)d);
  const float scale_log2 = (float)(1.4426950408889634 * scale);
  const dim3 grid((unsigned)((S + BN - 1) / BN), (unsigned)BH);
  if (d == 128) {
    const int smem = BwdSmem<128>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attn_bwd_kernel<128><<<grid, kThreads, smem, st>>>(mq, mk, mv, mo, lse, delta, dqs, dks, dvs, errw, (int)S,
                                                        scale_log2, (float)scale);
  } else {
    const int smem = BwdSmem<64>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attn_bwd_kernel<64><<<grid, kThreads, smem, st>>>(mq, mk, mv, mo, lse, delta, dqs, dks, dvs, errw, (int)S,
                                                       scale_log2, (float)scale);
  }
  return cudaGetLastError();
}

}  // namespace lh
