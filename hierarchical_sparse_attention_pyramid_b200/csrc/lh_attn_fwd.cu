// Stage 4 forward: dense causal softmax attention over the gathered S-token
// sequence (aitrends.kr summary of Lighthouse Attention, Technical details
// (3): the kept Q/K/V form S tokens and an unmodified attention runs on them).
//
// One CTA owns a 128-row query tile of one (batch, head) and walks the key
// tiles 0..qt (causal; the diagonal tile is masked).  Warp roles:
//   warps 0-3  softmax: thread t owns query row t (TMEM lane t); reads S from
//              TMEM, keeps the running max / sum, writes P (bf16) to shared
//              memory in the 128-byte-swizzled K-major layout, rescales O in
//              TMEM when the max moves, and writes O / LSE at the end
//   warp 4     TMA producer: Q once, then K and V tiles into a 2-stage ring
//   warp 5     MMA issuer (one thread): S = Q K^T into one of two TMEM
//              buffers, O += P V into a third; owns the TMEM allocation
// TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+D).
#include <cudaTypedefs.h>
#include <math.h>

#include "lh_common.cuh"
#include "sm100.cuh"

namespace lh {
namespace {
using namespace sm100;

constexpr int BM = 128, BN = 128;
constexpr int kThreads = 192;

template <int D>
struct FwdSmem {
  static constexpr int kChunk = 128 * 128;  // [128 rows][64 bf16] region
  static constexpr int kTile = D / 64 * kChunk;
  static constexpr int oQ = 0;
  static constexpr int oK = oQ + kTile;
  static constexpr int oV = oK + 2 * kTile;
  static constexpr int oP = oV + 2 * kTile;     // P_hi: bf16(P)
  static constexpr int oPl = oP + 2 * kChunk;   // P_lo: bf16(P - P_hi)
  static constexpr int oBar = oPl + 2 * kChunk;
  static constexpr int kBytes = oBar + 256;
  static constexpr int kAlloc = kBytes + 1024;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, float* __restrict__ O, float* __restrict__ LSE,
                    int* errw, int S, float scale_log2) {
  using Lay = FwdSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::oBar);
  uint64_t* bQ = bars + 0;
  uint64_t* bK = bars + 1;       // [2]
  uint64_t* bV = bars + 3;       // [2]
  uint64_t* bKVfree = bars + 5;  // [2]
  uint64_t* bS = bars + 7;       // [2]
  uint64_t* bSfree = bars + 9;   // [2]
  uint64_t* bP = bars + 11;
  uint64_t* bO = bars + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::oBar + 128);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::oBar + 132);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_qt = (S + BM - 1) / BM;
  const int qt = n_qt - 1 - (int)blockIdx.x;  // longest rows first
  const int bh = (int)blockIdx.y;
  const int n_kv = qt + 1;

  if (threadIdx.x == 0) {
    mbar_init(bQ, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bK[s], 1);
      mbar_init(&bV[s], 1);
      mbar_init(&bKVfree[s], 1);
      mbar_init(&bS[s], 1);
      mbar_init(&bSfree[s], 128);
    }
    mbar_init(bP, 128);
    mbar_init(bO, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_expect_tx(bQ, BM * D * 2);
      for (int c = 0; c < D / 64; ++c) tma_load_3d(smem + Lay::oQ + c * Lay::kChunk, &tmQ, bQ, c * 64, qt * BM, bh);
      for (int j = 0; j < n_kv; ++j) {
        const int st = j & 1, use = j >> 1;
        if (j >= 2 && !mbar_wait(&bKVfree[st], (use - 1) & 1, abort_flag)) break;
        mbar_expect_tx(&bK[st], BN * D * 2);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + Lay::oK + st * Lay::kTile + c * Lay::kChunk, &tmK, &bK[st], c * 64, j * BN, bh);
        mbar_expect_tx(&bV[st], BN * D * 2);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + Lay::oV + st * Lay::kTile + c * Lay::kChunk, &tmV, &bV[st], c * 64, j * BN, bh);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idQK = idesc_bf16(BM, BN, false, false);
      constexpr uint32_t idPV = idesc_bf16(BM, D, false, true);
      const uint32_t sQ = smem_u32(smem + Lay::oQ), sK = smem_u32(smem + Lay::oK);
      const uint32_t sV = smem_u32(smem + Lay::oV), sP = smem_u32(smem + Lay::oP);
      const uint32_t sPl = smem_u32(smem + Lay::oPl);
      auto issue_pv = [&](int jj) -> bool {
        const int st = jj & 1;
        if (!mbar_wait(bP, jj & 1, abort_flag)) return false;
        if (!mbar_wait(&bV[st], (jj >> 1) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t vb = sV + st * Lay::kTile;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint32_t aoff = (kk >> 2) * Lay::kChunk + (kk & 3) * 32;
          const uint64_t b = sdesc_sw128(vb + kk * 2048, Lay::kChunk, 1024);
          umma_bf16(tmem + 256, sdesc_sw128(sP + aoff, 16, 1024), b, idPV, (jj > 0 || kk > 0) ? 1u : 0u);
          umma_bf16(tmem + 256, sdesc_sw128(sPl + aoff, 16, 1024), b, idPV, 1u);
        }
        umma_commit(bO);
        umma_commit(&bKVfree[st]);
        return true;
      };
      bool ok = mbar_wait(bQ, 0, abort_flag);
      for (int j = 0; ok && j < n_kv; ++j) {
        const int st = j & 1, use = j >> 1;
        if (!mbar_wait(&bK[st], use & 1, abort_flag)) { ok = false; break; }
        if (j >= 2 && !mbar_wait(&bSfree[st], (use - 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kb = sK + st * Lay::kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = sdesc_sw128(sQ + (kk >> 2) * Lay::kChunk + (kk & 3) * 32, 16, 1024);
          const uint64_t b = sdesc_sw128(kb + (kk >> 2) * Lay::kChunk + (kk & 3) * 32, 16, 1024);
          umma_bf16(tmem + st * 128, a, b, idQK, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bS[st]);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok) issue_pv(n_kv - 1);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int row = threadIdx.x;  // 0..127
    const int row_g = qt * BM + row;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    uint8_t* sPb = smem + Lay::oP;
    uint8_t* sPlb = smem + Lay::oPl;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int st = j & 1;
      if (!mbar_wait(&bS[st], (j >> 1) & 1, abort_flag)) { ok = false; break; }
      __syncwarp();
      tc_fence_after();
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tl + st * 128 + c * 32, r[c]);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bSfree[st]);
      float s[128];
      float mx = -INFINITY;
      const bool diag = (j == n_kv - 1);
      const int lim = row_g - j * BN;  // columns c > lim are in the future
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        float v = __uint_as_float(r[c >> 5][c & 31]) * scale_log2;
        if (diag && c > lim) v = -INFINITY;
        s[c] = v;
        mx = fmaxf(mx, v);
      }
      const float m_new = fmaxf(m_run, mx);
      const float alpha = exp2f(m_run - m_new);
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        s[c] = exp2f(s[c] - m_new);
        rs += s[c];
      }
      if (j >= 1) {
        // PV of the previous tile must be done: O is stable and the P buffers free
        if (!mbar_wait(bO, (j - 1) & 1, abort_flag)) { ok = false; break; }
        __syncwarp();
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tl + 256 + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tl + 256 + c * 32, o);
          }
          tmem_st_wait();
        }
      }
      l_run = l_run * alpha + rs;
      m_run = m_new;
      // P = P_hi + P_lo, both bf16, so that P V keeps fp32-level accuracy
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float a = s[8 * ch + 2 * q], b = s[8 * ch + 2 * q + 1];
          const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
          hi[q] = *reinterpret_cast<const uint32_t*>(&h);
          lo[q] = pack_bf16x2(a - __low2float(h), b - __high2float(h));
        }
        const int off = (ch >> 3) * Lay::kChunk + row * 128 + (((ch & 7) ^ (row & 7)) << 4);
        *reinterpret_cast<uint4*>(sPb + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(sPlb + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bP);
    }
    if (ok && mbar_wait(bO, (n_kv - 1) & 1, abort_flag)) {
      __syncwarp();
      tc_fence_after();
      const float inv_l = 1.f / l_run;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tl + 256 + c * 32, o);
        tmem_ld_wait();
        if (row_g < S) {
          float4* dst = reinterpret_cast<float4*>(O + ((int64_t)bh * S + row_g) * D + c * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(__uint_as_float(o[4 * q]) * inv_l, __uint_as_float(o[4 * q + 1]) * inv_l,
                                 __uint_as_float(o[4 * q + 2]) * inv_l, __uint_as_float(o[4 * q + 3]) * inv_l);
        }
      }
      if (row_g < S) LSE[(int64_t)bh * S + row_g] = (m_run + log2f(l_run)) * 0.69314718055994530942f;
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

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

}  // namespace

// [BH][rows][D] bf16 viewed as a 3-D tensor (D, rows, BH); box of 64 x box_rows x 1, 128-byte swizzle
bool make_seq_map(CUtensorMap* m, const void* base, int64_t BH, int64_t rows, int D, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_attn_fwd(int64_t BH, int64_t S, int d, const void* qs, const void* ks, const void* vs, float* os,
                            float* lse, int* errw, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (!make_seq_map(&mq, qs, BH, S, d, BM) || !make_seq_map(&mk, ks, BH, S, d, BN) ||
      !make_seq_map(&mv, vs, BH, S, d, BN))
    return cudaErrorInvalidValue;
  const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)d));
  const dim3 grid((unsigned)((S + BM - 1) / BM), (unsigned)BH);
  if (d == 128) {
    const int smem = FwdSmem<128>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attn_fwd_kernel<128><<<grid, kThreads, smem, st>>>(mq, mk, mv, os, lse, errw,
                                                        (int)S, scale_log2);
  } else {
    const int smem = FwdSmem<64>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attn_fwd_kernel<64><<<grid, kThreads, smem, st>>>(mq, mk, mv, os, lse, errw,
                                                       (int)S, scale_log2);
  }
  return cudaGetLastError();
}

}  // namespace lh
