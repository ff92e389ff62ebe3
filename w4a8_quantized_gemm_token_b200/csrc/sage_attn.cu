// sage_attn.cu -- INT8 attention (scores from INT8 q and k, softmax and P V in
// floating point), head dim 128, no mask.
//
// Computes ("qlip-mlx" README, intro bullet "sage_attention" and the "Exact
// where it matters" bullet: INT8 Q K^T inside a flash-attention structure,
// exact online softmax, per-token scales, softmax and P V in floating point),
// per batch b, head h, query i:
//     s[i, j] = (qc_i . kc_j) * sq[i] * sk[j] * scale       (integer dot, exact)
//     o_i     = sum_j softmax_j(s[i, :]) v_j                 (bf16 out)
// where qc, sq and kc, sk are the per-token INT8 codes and scales of q and k
// (the activation rule of act_quant.cuh, one 128-element row per token).
//
// Design (sm_100a), one CTA per (128-query block, head), 8 warps:
//  * warp 0: TMA producer -- the query block's codes once, then per 128-key
//    block the key codes (128 x 128 B, 128-byte swizzle), the value block
//    transposed (v^T: 128 dims x 128 keys bf16, two 128-byte slabs) and the
//    block's key scales, into a 2-stage ring;
//  * warp 1: MMA issuer -- S_j = Q K_j^T by tcgen05.mma kind::i8 (M = N = 128,
//    K = 32 x 4) into one of two int32 TMEM buffers, then, once the softmax
//    warps have written P_j (bf16, K-major, swizzled) to shared memory,
//    O_j = P_j V_j by tcgen05.mma kind::f16 (bf16 in, fp32 accumulate, K = 16
//    x 8) into one of two fp32 TMEM buffers;
//  * warps 4-7 (one query row per thread): read S_j twice from TMEM (the row
//    maximum of acc sk, then p = 2^(s log2 e - m) with s log2 e = cq acc sk and
//    cq = sq scale log2 e >= 0), keep the running maximum m and sum l
//    in fp32, write P_j as bf16, and fold the previous block's O_{j-1} into
//    the output accumulator held in registers, o = 2^(m_{j-2} - m_{j-1}) o +
//    O_{j-1}, one block behind so the tensor cores are never waited for; at
//    the end o / l is rounded to bf16.
// Keys past L (the last block) get p = 0.  Every mbarrier wait is bounded
// (sm100.cuh); no load uses cluster multicast.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "qk_internal.h"
#include "sm100.cuh"

namespace qk {
namespace {

constexpr int D = 128;          // head dim (bytes of a code row)
constexpr int BQ = 128;         // queries per tile (TMEM lanes)
constexpr int kTiles = 2;       // query tiles per CTA, one softmax warpgroup each
constexpr int BKV = 128;        // keys per block
constexpr int kStages = 2;
constexpr int Q_BYTES = BQ * D;                 // 16 KiB of codes per tile
constexpr int K_BYTES = BKV * D;                // 16 KiB of codes
constexpr int VT_BYTES = D * BKV * 2;           // 32 KiB: 128 dims x 128 keys bf16
constexpr int P_BYTES = BQ * BKV * 2;           // 32 KiB: 128 queries x 128 keys bf16
constexpr int SK_BYTES = BKV * 4;
constexpr int SMEM_Q = 0;
constexpr int SMEM_K = SMEM_Q + kTiles * Q_BYTES;
constexpr int SMEM_VT = SMEM_K + kStages * K_BYTES;
constexpr int SMEM_P = SMEM_VT + kStages * VT_BYTES;  // one P buffer per tile
constexpr int SMEM_SK = SMEM_P + kTiles * P_BYTES;
constexpr int SMEM_BAR = SMEM_SK + kStages * SK_BYTES;
// qfull, kvfull[2], kvempty[2], then per tile sfull, sfree, pfull, pfree, ofull
constexpr int kNumBars = 1 + 2 * kStages + 5 * kTiles;
constexpr int SMEM_SLOT = SMEM_BAR + kNumBars * 8;
constexpr int SMEM_ALLOC = SMEM_SLOT + 16 + 1024;
constexpr int kThreads = 128 * (1 + kTiles);  // warpgroup 0: producer, MMA, 2 idle
constexpr int kSoftWarps = 4;                 // per tile
// Registers: launched with kRegsLaunch per thread; warpgroup 0 keeps kRegsCtl
// and the softmax warpgroups (o[128] in registers) take the rest.
constexpr int kRegsLaunch = 168;
constexpr int kRegsCtl = 56;
constexpr int kRegsSoft = 224;
static_assert(128 * kRegsCtl + 128 * kTiles * kRegsSoft <= kThreads * kRegsLaunch,
              "register split exceeds the launch allocation");
constexpr uint32_t KV_TX = K_BYTES + VT_BYTES + SK_BYTES;
static_assert(kTiles * 2 * 128 <= 512, "S and O of every tile fit the 512 TMEM columns");
constexpr uint32_t kIdescS = i8_idesc(BQ, BKV, true, true);
// kind::f16 instruction descriptor: D fp32 (bits 4-5 = 1), A and B bf16 (bits
// 7-9, 10-12 = 1), both K-major, N >> 3 at bits 17-22, M >> 4 at bits 24-28.
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(D >> 3) << 17) |
                              ((uint32_t)(BQ >> 4) << 24);

static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
static_assert(SMEM_K % 1024 == 0 && SMEM_VT % 1024 == 0 && SMEM_P % 1024 == 0,
              "swizzled tiles need 1024-byte alignment");

// D[tmem] (+)= A[smem] * B[smem]^T, one K = 16 step of bf16 operands.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 2^x by the hardware approximation (relative error below 2^-22).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// One pass over a block's scores: y[key] = acc * sk for the 128 keys (acc the
// int32 dot products in TMEM); returns the maximum over the keys below kvalid
// (all of them unless masked).
template <bool kMasked>
__device__ __forceinline__ float load_scores(uint32_t t_s, const float* skb, int kvalid,
                                             float (&y)[BKV]) {
  float my = -INFINITY;
#pragma unroll
  for (int c = 0; c < BKV / 32; ++c) {
    uint32_t v[32];
    tmem_ld32(t_s + (uint32_t)(32 * c), v);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
      const float4 s4 = reinterpret_cast<const float4*>(skb)[(32 * c + i) >> 2];
      const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = 32 * c + i + e;
        y[key] = __int2float_rn((int)v[i + e]) * sv[e];
        if (!kMasked || key < kvalid) my = fmaxf(my, y[key]);
      }
    }
  }
  return my;
}

// p = 2^(cq y + neg_m) rounded to bf16 (0 for keys past kvalid when masked),
// written as this row of P (K-major, 128-byte swizzle, two slabs of 64 keys);
// returns the sum of the rounded weights, the ones P V uses.
template <bool kMasked>
__device__ __forceinline__ float write_p(const float (&y)[BKV], int kvalid, float cq, float neg_m,
                                         uint8_t* prow, int row) {
  float rs = 0.0f;
#pragma unroll
  for (int c = 0; c < BKV / 32; ++c) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      const int key = 32 * c + i;
      const float p0 = (!kMasked || key < kvalid) ? ex2(fmaf(cq, y[key], neg_m)) : 0.0f;
      const float p1 = (!kMasked || key + 1 < kvalid) ? ex2(fmaf(cq, y[key + 1], neg_m)) : 0.0f;
      const uint32_t w = pack_bf16x2(p0, p1);
      rs += __uint_as_float(w << 16) + __uint_as_float(w & 0xFFFF0000u);
      pk[i >> 1] = w;
    }
    uint8_t* srow = prow + (c >> 1) * (P_BYTES / 2);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int ch = (c & 1) * 4 + u;  // 16-byte chunk of the 128-byte row
      *reinterpret_cast<uint4*>(srow + ((ch ^ (row & 7)) * 16)) =
          make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
    }
  }
  return rs;
}

// v [BH, L, 128] bf16 -> vt [BH, 128, L] bf16 (64 x 64 tiles through shared
// memory; L % 8 == 0).
__global__ void __launch_bounds__(256) transpose_v_kernel(const uint16_t* __restrict__ v,
                                                          uint16_t* __restrict__ vt, int L) {
  __shared__ uint16_t tile[64][66];
  const int bh = blockIdx.z;
  const int l0 = blockIdx.x * 64, d0 = blockIdx.y * 64;
  const uint16_t* src = v + (size_t)bh * L * D;
  uint16_t* dst = vt + (size_t)bh * D * L;
  const int tx = threadIdx.x & 63, ty = threadIdx.x >> 6;  // 64 x 4
  for (int r = ty; r < 64; r += 4) {
    const int l = l0 + r;
    tile[r][tx] = l < L ? src[(size_t)l * D + d0 + tx] : (uint16_t)0;
  }
  __syncthreads();
  for (int r = ty; r < 64; r += 4) {
    const int l = l0 + tx;
    if (l < L) dst[(size_t)(d0 + r) * L + l] = tile[tx][r];
  }
}


__global__ void __launch_bounds__(kThreads, 1)
    sage_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmVt, const float* __restrict__ sq,
                     const float* __restrict__ sk, uint16_t* __restrict__ out, int L,
                     float scale_log2e, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem<1024>(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + SMEM_BAR;
  const uint32_t qfull = bar0;
  auto kvfull = [&](int s) { return bar0 + 8u * (1 + s); };
  auto kvempty = [&](int s) { return bar0 + 8u * (3 + s); };
  // per query tile t: 0 sfull, 1 sfree, 2 pfull, 3 pfree, 4 ofull
  auto tbar = [&](int t, int which) { return bar0 + 8u * (5 + 5 * t + which); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SMEM_SLOT);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int q0 = blockIdx.x * (kTiles * BQ);  // first query of this CTA, within the head
  const int nkb = (L + BKV - 1) / BKV;
  const int row_base = bh * L;                // this head's first row of the [BH * L] arrays

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmVt);
    mbar_init(qfull, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(kvfull(s), 1);
      mbar_init(kvempty(s), 1);
    }
    for (int t = 0; t < kTiles; ++t) {
      mbar_init(tbar(t, 0), 1);           // S ready (MMA commit)
      mbar_init(tbar(t, 1), kSoftWarps);  // S read
      mbar_init(tbar(t, 2), kSoftWarps);  // P written
      mbar_init(tbar(t, 3), 1);           // P read (MMA commit)
      mbar_init(tbar(t, 4), 1);           // O updated (MMA commit)
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);  // S of tile t: columns 128 t; O: 256 + 128 t
    tmem_relinquish();
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait();  // codes, scales and v^T come from the preparation kernels

  if (warp < 4) {
    // warpgroup 0: warp 0 loads, warp 1 issues the MMAs, warps 2-3 idle; most
    // of its registers go to the softmax warpgroups
    regs_dec<kRegsCtl>();
    if (warp == 0) {
      // ---------------------------------------------------------- producer
      if (lane == 0) {
        mbar_arrive_expect_tx(qfull, kTiles * Q_BYTES);
        for (int t = 0; t < kTiles; ++t)
          tma_load_2d(sbase + SMEM_Q + t * Q_BYTES, &tmQ, 0, row_base + q0 + t * BQ, qfull);
        for (int j = 0; j < nkb; ++j) {
          const int s = j & 1;
          if (!mbar_wait(kvempty(s), ((j >> 1) & 1) ^ 1u, err)) break;
          mbar_arrive_expect_tx(kvfull(s), KV_TX);
          tma_load_2d(sbase + SMEM_K + s * K_BYTES, &tmK, 0, row_base + j * BKV, kvfull(s));
#pragma unroll
          for (int sl = 0; sl < 2; ++sl)  // keys [64 sl, 64 sl + 64) of the block
            tma_load_2d(sbase + SMEM_VT + s * VT_BYTES + sl * (VT_BYTES / 2), &tmVt,
                        j * BKV + 64 * sl, bh * D, kvfull(s));
          bulk_load(sbase + SMEM_SK + s * SK_BYTES, sk + row_base + j * BKV, SK_BYTES,
                    kvfull(s));
        }
      }
    } else if (warp == 1) {
      // -------------------------------------------------------- MMA issuer
      if (lane == 0) {
        auto issue_s = [&](int t, int j) -> bool {  // S_t = Q_t K_j^T (int32)
          const int s = j & 1;
          if (!mbar_wait(tbar(t, 1), (j & 1) ^ 1u, err)) return false;  // S_t read
          tc_fence_after();
          const uint32_t a = sbase + SMEM_Q + t * Q_BYTES, b = sbase + SMEM_K + s * K_BYTES;
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)
            mma_i8(tmem_base + (uint32_t)(t * BQ), sw128_kmajor_desc(a + 32 * kk),
                   sw128_kmajor_desc(b + 32 * kk), kIdescS, kk);
          mma_commit(tbar(t, 0));
          return true;
        };
        bool ok = mbar_wait(qfull, 0, err) && mbar_wait(kvfull(0), 0, err);
        for (int t = 0; t < kTiles && ok; ++t) ok = issue_s(t, 0);
        for (int j = 0; j < nkb && ok; ++j) {
          const int s = j & 1;
          const bool next = j + 1 < nkb;
          if (next && !mbar_wait(kvfull(s ^ 1), ((j + 1) >> 1) & 1, err)) break;
          for (int t = 0; t < kTiles && ok; ++t) {
            // O_t += P_t V_j once tile t's softmax wrote P_t (and rescaled O_t if
            // its reference maximum moved)
            if (!mbar_wait(tbar(t, 2), j & 1, err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a = sbase + SMEM_P + t * P_BYTES, b = sbase + SMEM_VT + s * VT_BYTES;
#pragma unroll
            for (int kk = 0; kk < BKV / 16; ++kk)  // K = 16 keys per step: slab kk / 4
              mma_bf16(tmem_base + (uint32_t)(256 + t * D),
                       sw128_kmajor_desc(a + (kk >> 2) * (P_BYTES / 2) + 32 * (kk & 3)),
                       sw128_kmajor_desc(b + (kk >> 2) * (VT_BYTES / 2) + 32 * (kk & 3)),
                       kIdescPV, (j | kk) != 0 ? 1u : 0u);
            mma_commit(tbar(t, 4));  // O_t updated
            mma_commit(tbar(t, 3));  // P_t read
            // the next scores of this tile (its S buffer was read before P_t was written)
            if (next && !issue_s(t, j + 1)) ok = false;
          }
          mma_commit(kvempty(s));  // K_j and v^T_j read by every tile
        }
      }
    }
  } else {
    // ------------------------------------------------- softmax and output
    regs_inc<kRegsSoft>();
    const int t = (warp >> 2) - 1;           // query tile of this warpgroup
    const int q = warp & 3;                  // TMEM lane quarter
    const int row = q * 32 + lane;           // query row of the tile (TMEM lane)
    const int qi = q0 + t * BQ + row;
    const bool live = qi < L;
    const float cq = live ? __ldg(sq + row_base + qi) * scale_log2e : 0.0f;
    const uint32_t t_lane = tmem_base + ((uint32_t)(q * 32) << 16);
    const uint32_t t_s = t_lane + (uint32_t)(t * BQ);
    const uint32_t t_o = t_lane + (uint32_t)(256 + t * D);
    uint8_t* prow = smem + SMEM_P + t * P_BYTES + row * 128;
    // reference maximum m (log2 units) and sum l; the output accumulates in
    // TMEM (O_t += P V), rescaled only when a row's reference maximum moves
    float m = -INFINITY, l = 0.0f;
    bool ok = true;
    for (int j = 0; j < nkb; ++j) {
      const int s = j & 1;
      if (!mbar_wait(tbar(t, 0), j & 1, err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* skb = reinterpret_cast<const float*>(smem + SMEM_SK + s * SK_BYTES);
      const int kvalid = min(BKV, L - j * BKV);  // keys of this block inside the head
      float y[BKV];
      const float my = kvalid == BKV ? load_scores<false>(t_s, skb, kvalid, y)
                                     : load_scores<true>(t_s, skb, kvalid, y);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tbar(t, 1));  // S_t read: the next scores may start
      // keep the reference unless the block's maximum exceeds it by more than
      // 2^8 (weights then stay below 256); a new reference rescales O and l
      const float mb = cq * my;
      const float m_new = mb > m + 8.0f ? mb : m;
      const float alpha = ex2(m - m_new);  // 1 when kept; 0 on the first block
      if (j >= 1 && __any_sync(0xFFFFFFFFu, alpha != 1.0f)) {
        // O_t holds P V up to block j - 1: wait for it, scale this warp's rows
        if (!mbar_wait(tbar(t, 4), (j - 1) & 1, err)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(t_o + (uint32_t)(32 * c), v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
          tmem_st32(t_o + (uint32_t)(32 * c), v);
        }
        tmem_st_wait();
        tc_fence_before();
      }
      // P_t of this block (the buffer is free once P V of the last block ran)
      if (!mbar_wait(tbar(t, 3), (j & 1) ^ 1u, err)) {
        ok = false;
        break;
      }
      const float rs = kvalid == BKV ? write_p<false>(y, kvalid, cq, -m_new, prow, row)
                                     : write_p<true>(y, kvalid, cq, -m_new, prow, row);
      fence_proxy_async_smem();  // P_t stores before the tensor cores read them
      __syncwarp();
      if (lane == 0) mbar_arrive(tbar(t, 2));
      l = alpha * l + rs;
      m = m_new;
    }
    // the output: O_t after the last block's P V, divided by l
    if (ok && nkb >= 1 && mbar_wait(tbar(t, 4), (nkb - 1) & 1, err)) {
      tc_fence_after();
      const float inv = 1.0f / l;
      uint4* dst = reinterpret_cast<uint4*>(out + (size_t)(row_base + qi) * D);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(t_o + (uint32_t)(32 * c), v);
        tmem_ld_wait();
        if (live) {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            dst[4 * c + u] = make_uint4(
                pack_bf16x2(__uint_as_float(v[8 * u]) * inv, __uint_as_float(v[8 * u + 1]) * inv),
                pack_bf16x2(__uint_as_float(v[8 * u + 2]) * inv, __uint_as_float(v[8 * u + 3]) * inv),
                pack_bf16x2(__uint_as_float(v[8 * u + 4]) * inv, __uint_as_float(v[8 * u + 5]) * inv),
                pack_bf16x2(__uint_as_float(v[8 * u + 6]) * inv, __uint_as_float(v[8 * u + 7]) * inv));
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, 512);
}

bool g_attr_done[64];

}  // namespace

cudaError_t launch_sage_attention(const int8_t* qc, const float* sq, const int8_t* kc,
                                  const float* sk, const uint16_t* vt, int64_t BH, int64_t L,
                                  float scale, uint16_t* out, cudaStream_t s) {
  CUtensorMap tQ, tK, tV;
  if (!encode_tmap_2d(&tQ, CU_TENSOR_MAP_DATA_TYPE_UINT8, qc, (uint64_t)D, (uint64_t)(BH * L),
                      (uint64_t)D, D, BQ, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tK, CU_TENSOR_MAP_DATA_TYPE_UINT8, kc, (uint64_t)D, (uint64_t)(BH * L),
                      (uint64_t)D, D, BKV, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, vt, (uint64_t)L, (uint64_t)(BH * D),
                      (uint64_t)L * 2, 64, D, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !g_attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(sage_attn_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    // the softmax warpgroups' register increase is only satisfiable with the
    // launch allocation the split was computed for
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, sage_attn_kernel)) != cudaSuccess) return e;
    if (fa.numRegs != kRegsLaunch) return cudaErrorInvalidKernelImage;
    g_attr_done[dev] = true;
  }
  int* err = device_error_word();
  if (err == nullptr) return cudaErrorUnknown;
  const float scale_log2e = scale * 1.4426950408889634f;
  dim3 grid((unsigned)((L + kTiles * BQ - 1) / (kTiles * BQ)), (unsigned)BH);
  sage_attn_kernel<<<grid, kThreads, SMEM_ALLOC, s>>>(tQ, tK, tV, sq, sk, out, (int)L, scale_log2e,
                                                      err);
  return cudaGetLastError();
}

cudaError_t launch_transpose_v(const uint16_t* v, int64_t BH, int64_t L, uint16_t* vt,
                               cudaStream_t s) {
  dim3 grid((unsigned)((L + 63) / 64), (unsigned)(D / 64), (unsigned)BH);
  transpose_v_kernel<<<grid, 256, 0, s>>>(v, vt, (int)L);
  return cudaGetLastError();
}

}  // namespace qk
