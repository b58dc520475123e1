// Stage 4 forward: dense causal softmax attention over the gathered S-token
// sequence (aitrends.kr summary of Lighthouse Attention, Technical details
// (3): the kept Q/K/V form S tokens and an unmodified attention runs on them).
//
// One CTA owns two 128-row query tiles (A = 2c, B = 2c+1) of one (batch,
// head) and streams the key/value tiles 0..2c+1 once for both (causal; each
// tile's diagonal block is masked).  Warp roles:
//   warps 0-7  softmax, one warpgroup per query tile (warps 0-3 tile A, 4-7
//              tile B): thread t of a group owns query row t (TMEM lane t) and
//              all 128 keys of a key tile, so the row max needs no exchange
//              between threads; it keeps the running max and row sum,
//              rescales its O row in TMEM when the max moves, and writes P
//              back over the S columns it came from as a bf16 pair (per 32
//              keys: 16 columns of hi, 16 of lo), where the P V product reads it
//   warp 8     TMA producer: both Q tiles once, K and V tiles into a 2-stage ring
//   warp 9     MMA issuer (the converged warp; one elected lane issues):
//              for each key tile, P_A V, then the next S_A = Q_A K^T, then
//              P_B V and the next S_B.  One tile's softmax runs while the
//              tensor core works on the other tile's products, so the two
//              groups take turns rather than sharing the issue slots.
// TMEM columns: S_A/P_A [0,128), S_B/P_B [128,256), O_A [256,256+D), O_B [256+D,256+2D).
// The P pair keeps P V at fp32 accuracy (the backward's Delta = rowsum(dO O)
// cancels against P (dP - Delta), so O errors would reach dQ); O is written
// in fp32.
#include <cudaTypedefs.h>
#include <math.h>

#include <type_traits>

#include "lh_common.cuh"
#include "sm100.cuh"

namespace lh {
namespace {
using namespace sm100;

constexpr int BM = 128, BN = 128;
constexpr int kSoftmax = 256;          // two warpgroups, one per query tile
constexpr int kPair = kSoftmax / 2;    // softmax threads of one query tile (one per row)
constexpr int kThreads = kSoftmax + 64;
constexpr int kWarpTma = kSoftmax / 32, kWarpMma = kWarpTma + 1;


template <int D>
struct FwdSmem {
  static constexpr int kChunk = 128 * 128;  // [128 rows][64 bf16] region
  static constexpr int kTile = D / 64 * kChunk;
  static constexpr int oQ = 0;              // Q_A, Q_B
  static constexpr int oK = oQ + 2 * kTile; // 2 stages
  static constexpr int oV = oK + 2 * kTile; // 2 stages
  static constexpr int oBar = oV + 2 * kTile;
  static constexpr int kBytes = oBar + 256;
  static constexpr int kAlloc = kBytes + 1024;
};

// 10 warps, three on some SM sub-partitions: at most 168 registers a thread
// (a sub-partition holds 16384).  A softmax thread holds its row's 128 scores
// in registers and writes P back 16 keys at a time.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, float* __restrict__ O, float* __restrict__ LSE,
                    int* errw, int S, float scale_log2, long long wait_cycles, int issue_loads, int qt0, int qt1) {
  using Lay = FwdSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::oBar);
  uint64_t* bQ = bars + 0;
  uint64_t* bK = bars + 1;       // [2] stages
  uint64_t* bV = bars + 3;       // [2]
  uint64_t* bKVfree = bars + 5;  // [2]
  uint64_t* bS = bars + 7;       // [2] tiles: S of the tile in TMEM (and its previous P V done)
  uint64_t* bP = bars + 9;       // [2] tiles: P in TMEM, O rescaled (one arrival per thread of the tile's pair)
  uint64_t* bO = bars + 11;      // [2] tiles: a P V product of the tile done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::oBar + 192);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::oBar + 196);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // the query tiles [qt0, qt1) of the sequence (all of them, except for a
  // row window of the sequence); key tiles run from 0 to each query tile
  const int n_pairs = (qt1 - qt0 + 1) / 2;
  // one CTA per (tile pair, head), pair-major: the block scheduler starts
  // blocks in index order, so every head's longest pairs run first and the
  // short ones fill the tail
  const int BHn = (int)(gridDim.x / (unsigned)n_pairs);
  const int c = n_pairs - 1 - (int)(blockIdx.x / (unsigned)BHn);
  const int bh = (int)(blockIdx.x % (unsigned)BHn);
  const int qtile[2] = {qt0 + 2 * c, qt0 + 2 * c + 1};
  const bool hasB = qtile[1] < qt1;
  const int last[2] = {qtile[0], hasB ? qtile[1] : -1};  // last key tile of each query tile
  const int n_kv = (hasB ? qtile[1] : qtile[0]) + 1;

  if (threadIdx.x == 0) {
    mbar_init(bQ, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bK[s], 1);
      mbar_init(&bV[s], 1);
      mbar_init(&bKVfree[s], 1);
      mbar_init(&bS[s], 1);
      mbar_init(&bP[s], kPair);
      mbar_init(&bO[s], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ TMA producer
    // issue_loads == 0 only in the timeout self-test: nothing is loaded, so
    // the other roles' bounded waits run out with no copy or MMA in flight
    if (lane == 0 && issue_loads) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_expect_tx(bQ, (hasB ? 2 : 1) * BM * D * 2);
      for (int x = 0; x < (hasB ? 2 : 1); ++x)
        for (int ch = 0; ch < D / 64; ++ch)
          tma_load_3d(smem + Lay::oQ + x * Lay::kTile + ch * Lay::kChunk, &tmQ, bQ, ch * 64, qtile[x] * BM, bh);
      for (int j = 0; j < n_kv; ++j) {
        const int st = j & 1, use = j >> 1;
        if (j >= 2 && !mbar_wait(&bKVfree[st], (use - 1) & 1, abort_flag, wait_cycles)) break;
        mbar_expect_tx(&bK[st], BN * D * 2);
        for (int ch = 0; ch < D / 64; ++ch)
          tma_load_3d(smem + Lay::oK + st * Lay::kTile + ch * Lay::kChunk, &tmK, &bK[st], ch * 64, j * BN, bh);
        mbar_expect_tx(&bV[st], BN * D * 2);
        for (int ch = 0; ch < D / 64; ++ch)
          tma_load_3d(smem + Lay::oV + st * Lay::kTile + ch * Lay::kChunk, &tmV, &bV[st], ch * 64, j * BN, bh);
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    {  // the whole warp; one elected lane issues each instruction
      constexpr uint32_t idQK = idesc_bf16(BM, BN, false, false);
      constexpr uint32_t idPV = idesc_bf16(BM, D, false, true);
      const uint32_t sQ = smem_u32(smem + Lay::oQ), sK = smem_u32(smem + Lay::oK), sV = smem_u32(smem + Lay::oV);
      // base descriptors: an operand at byte offset off is base + (off >> 4)
      const uint64_t kQ = sdesc_sw128(sQ, 16, 1024), kK = sdesc_sw128(sK, 16, 1024);
      const uint64_t mV = sdesc_sw128(sV, Lay::kChunk, 1024);
      auto issue_s = [&](int x, int j) {
        const uint64_t qb = kQ + ((x * Lay::kTile) >> 4), kb = kK + (((j & 1) * Lay::kTile) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * Lay::kChunk + (kk & 3) * 32) >> 4;
          umma_bf16_w(tmem + x * 128, qb + off, kb + off, idQK, kk > 0 ? 1u : 0u);
        }
        umma_commit_w(&bS[x]);
      };
      bool ok = mbar_wait_warp(bQ, 0, abort_flag, wait_cycles) && mbar_wait_warp(&bK[0], 0, abort_flag, wait_cycles);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        if (hasB) issue_s(1, 0);
      }
      for (int j = 0; ok && j < n_kv; ++j) {
        const int st = j & 1;
        bool v_ready = false, k_next_ready = false;
        for (int x = 0; x < 2 && ok; ++x) {
          if (j > last[x]) continue;
          if (!mbar_wait_warp(&bP[x], j & 1, abort_flag, wait_cycles)) { ok = false; break; }
          if (!v_ready) {
            if (!mbar_wait_warp(&bV[st], (j >> 1) & 1, abort_flag, wait_cycles)) { ok = false; break; }
            v_ready = true;
          }
          tc_fence_after();
          const uint64_t vb = mV + ((st * Lay::kTile) >> 4);
          const uint32_t pa = tmem + x * 128;
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint64_t b = vb + ((kk * 2048) >> 4);
            const uint32_t a = pa + (kk >> 1) * 32 + (kk & 1) * 8;  // hi of keys 16kk..16kk+15
            umma_bf16_tmem_a_w(tmem + 256 + x * D, a, b, idPV, (j > 0 || kk > 0) ? 1u : 0u);
            umma_bf16_tmem_a_w(tmem + 256 + x * D, a + 16, b, idPV, 1u);
          }
          umma_commit_w(&bO[x]);
          if (j + 1 <= last[x]) {
            if (!k_next_ready) {
              if (!mbar_wait_warp(&bK[(j + 1) & 1], ((j + 1) >> 1) & 1, abort_flag, wait_cycles)) { ok = false; break; }
              k_next_ready = true;
              tc_fence_after();
            }
            issue_s(x, j + 1);  // after P V of this tile: the S columns hold P until then
          }
        }
        if (ok) umma_commit_w(&bKVfree[st]);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    // Warpgroup x (warps 4x .. 4x+3) works on query tile x; thread t owns
    // query row t (TMEM lane t) and all 128 keys of each key tile.  It loads
    // the row's scores from TMEM once, takes their max, keeps the running max
    // and row sum, rescales its O row when the max moves, and writes P back
    // over the S columns it came from as a bf16 pair (per 32 keys: 16
    // columns of hi, 16 of lo), where the P V product reads it.
    const int x = warp >> 2;
    const int row = (warp & 3) * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t ts = tl + x * 128, to = tl + 256 + x * D;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; ok && j <= last[x]; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bS[x], j & 1, abort_flag, wait_cycles));
      if (!ok) break;
      tc_fence_after();
      const bool diag = (j == last[x]);
      // row max of the raw scores (the scale is positive), as eight
      // independent chains over two 64-key halves loaded in turn (the scores
      // are read again for the P pass, so no more than 64 are held at once);
      // on the diagonal tile the keys after the row are masked
      uint32_t r[2][32];
      float mc[8];
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) mc[c8] = -INFINITY;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        tmem_ld32(ts + hh * 64, r[0]);
        tmem_ld32(ts + hh * 64 + 32, r[1]);
        tmem_ld_wait();
        if (diag) {
#pragma unroll
          for (int ch = 0; ch < 2; ++ch)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (hh * 64 + ch * 32 + i <= row)
                mc[ch * 4 + (i >> 3)] = fmaxf(mc[ch * 4 + (i >> 3)], __uint_as_float(r[ch][i]));
        } else {
#pragma unroll
          for (int ch = 0; ch < 2; ++ch)
#pragma unroll
            for (int i = 0; i < 32; i += 2)
              mc[ch * 4 + (i >> 3)] =
                  max3f(mc[ch * 4 + (i >> 3)], __uint_as_float(r[ch][i]), __uint_as_float(r[ch][i + 1]));
        }
      }
      const float mx = fmaxf(fmaxf(max3f(mc[0], mc[1], mc[2]), max3f(mc[3], mc[4], mc[5])), fmaxf(mc[6], mc[7]));
      // Lazy rescaling: the reference m_run moves only when the row max
      // exceeds it by more than 8 (so every P stays <= 2^8); O and l share
      // the reference, so the result is exact either way.
      const float m_tile = mx * scale_log2;
      const bool move = m_tile > m_run + 8.f;
      const float m_new = move ? m_tile : m_run;
      const float alpha = move ? fast_exp2(m_run - m_new) : 1.f;
      // P = 2^(s*scale - m) as a bf16 pair written back over the chunk it
      // came from: chunk ch (keys 32ch..32ch+31) holds hi in its first 16
      // columns and lo in its last 16, where P V reads them.  Keys after the
      // row are masked on the diagonal tile only.
      const uint64_t c2 = f2_pack(scale_log2, scale_log2), nm2 = f2_pack(-m_new, -m_new);
      uint64_t rs2[4];
      auto p_pass = [&](auto masked) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          tmem_ld32(ts + hh * 64, r[0]);
          tmem_ld32(ts + hh * 64 + 32, r[1]);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int ch = hh * 2 + c;
            rs2[ch] = f2_pack(0.f, 0.f);
#pragma unroll
            for (int h = 0; h < 2; ++h) {  // keys 32ch+16h .. +15: hi to columns 32ch+8h, lo to 32ch+16+8h
              uint32_t hi[8], lo[8];
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const int e = 16 * h + 2 * q;
                float a, b;
                f2_unpack(f2_fma(f2_pack(__uint_as_float(r[c][e]), __uint_as_float(r[c][e + 1])), c2, nm2), a, b);
                a = fast_exp2(a);
                b = fast_exp2(b);
                if constexpr (decltype(masked)::value) {
                  const int col = ch * 32 + e;
                  a = col > row ? 0.f : a;
                  b = col + 1 > row ? 0.f : b;
                }
                rs2[ch] = f2_add(rs2[ch], f2_pack(a, b));
                split_bf16x2(a, b, hi[q], lo[q]);
              }
              tmem_st8(ts + ch * 32 + 8 * h, hi);
              tmem_st8(ts + ch * 32 + 16 + 8 * h, lo);
            }
          }
        }
      };
      if (diag) p_pass(std::true_type{});
      else p_pass(std::false_type{});
      float rsa, rsb;
      f2_unpack(f2_add(f2_add(rs2[0], rs2[1]), f2_add(rs2[2], rs2[3])), rsa, rsb);
      const float rs = rsa + rsb;
      // rescale the O row; the previous P V of this tile is done (its
      // completion preceded this S)
      if (j >= 1 && __any_sync(0xffffffffu, move)) {
#pragma unroll 1
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t o[32];
          tmem_ld32(to + ch * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(to + ch * 32, o);
        }
      }
      l_run = l_run * alpha + rs;
      m_run = m_new;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bP[x]);
    }
    if (ok && last[x] >= 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bO[x], last[x] & 1, abort_flag, wait_cycles));
      if (ok) {
        tc_fence_after();
        const float inv_l = 1.f / l_run;
        const int row_g = qtile[x] * BM + row;
#pragma unroll 1
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t o[32];
          tmem_ld32(to + ch * 32, o);
          tmem_ld_wait();
          if (row_g < S) {
            float4* dst = reinterpret_cast<float4*>(O + ((int64_t)bh * S + row_g) * D + ch * 32);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              dst[q] = make_float4(__uint_as_float(o[4 * q]) * inv_l, __uint_as_float(o[4 * q + 1]) * inv_l,
                                   __uint_as_float(o[4 * q + 2]) * inv_l, __uint_as_float(o[4 * q + 3]) * inv_l);
          }
        }
        if (row_g < S) LSE[(int64_t)bh * S + row_g] = (m_run + log2f(l_run)) * 0.69314718055994530942f;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
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

// [BH][rows][D] fp32 viewed as a 3-D tensor (D, rows, BH); box of 32 x box_rows x 1, 128-byte swizzle
bool make_f32_map(CUtensorMap* m, const void* base, int64_t BH, int64_t rows, int D, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)rows * D * 4};
  cuuint32_t box[3] = {32, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_attn_fwd(int64_t BH, int64_t S, int d, const void* qs, const void* ks, const void* vs, float* os,
                            float* lse, int* errw, cudaStream_t st, long long wait_cycles, int issue_loads, int64_t qt0,
                            int64_t qt1) {
  CUtensorMap mq, mk, mv;
  if (!make_seq_map(&mq, qs, BH, S, d, BM) || !make_seq_map(&mk, ks, BH, S, d, BN) ||
      !make_seq_map(&mv, vs, BH, S, d, BN))
    return cudaErrorInvalidValue;
  const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)d));
  const int64_t n_qt = (S + BM - 1) / BM;
  if (qt1 < 0) qt1 = n_qt;
  if (qt0 < 0 || qt0 >= qt1 || qt1 > n_qt) return cudaErrorInvalidValue;
  if (((qt1 - qt0 + 1) / 2) * BH > 0x7fffffffll) return cudaErrorInvalidConfiguration;  // one grid dimension
  const dim3 grid((unsigned)(((qt1 - qt0 + 1) / 2) * BH));
  if (d == 128) {
    const int smem = FwdSmem<128>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attn_fwd_kernel<128><<<grid, kThreads, smem, st>>>(mq, mk, mv, os, lse, errw, (int)S, scale_log2, wait_cycles,
                                                               issue_loads, (int)qt0, (int)qt1);
  } else {
    const int smem = FwdSmem<64>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attn_fwd_kernel<64><<<grid, kThreads, smem, st>>>(mq, mk, mv, os, lse, errw, (int)S, scale_log2, wait_cycles,
                                                               issue_loads, (int)qt0, (int)qt1);
  }
  return cudaGetLastError();
}

}  // namespace lh
