// gemm_w8a8.cu -- the W8A8 tensor-core GEMM with the fused dequant epilogue.
//
// Computes ("qlip-mlx" README, "w8a8_linear / W8A8Linear": INT8 x INT8 ->
// INT32 matmul with dequant + bias fused behind it)
//     acc[m, n] = sum_k xq[m, k] * Wq[n, k]                  (exact int32)
//     y[m, n]   = bf16( acc * sx[m] * sw[n] + bias[n] )      (one rounding)
// within 1 bf16 ulp of the exact value rounded once (see the epilogue below).
//
// Design (sm_100a):
//  * CTA pairs (clusters of 2) run one tcgen05.mma.cta_group::2 kind::i8 over
//    both SMs: a pair owns a 256 x 256 output tile, each CTA loads its 128 rows
//    of xq and its 128 rows of Wq (so each SM moves 32 KiB of operands per
//    128-deep K block instead of 48 KiB for a 128 x 256 tile on one SM) and
//    holds a 128 x 256 int32 accumulator in its own TMEM;
//  * persistent grid (one pair per two SMs), tiles in a grouped raster;
//  * warp 0: TMA producer into a 3-stage shared-memory ring of 256-deep K
//    blocks (64 KiB per stage per CTA, as two 128-byte-wide swizzled slabs per
//    operand); both CTAs' loads complete on the pair leader's full barrier;
//  * warp 1 of the leader issues the MMAs (M = 256, N = 256, K = 32 each) into
//    one of two 256-column accumulators and commits each stage and each
//    finished accumulator to the barriers of both CTAs;
//  * warps 2-5 (4 per CTA): epilogue.  tcgen05.ld of 32 columns at a time,
//    then a guarded fp32 fast path: v32 = fma(fp32(acc) * sx, sw, bias) with
//    per-column {sw, bias, guard, gate} built once per tile in shared memory.
//    Where |v32| >= 2^-12 |bias| (and v32 is far from fp32 underflow) its error
//    is below 1/8 bf16 ulp, so its rounding is within 1 ulp of the exact value
//    rounded once; the few elements that fail the guard (cancellation against
//    the bias) take the exact path: int32 -> fp64 by the 2^52 magic number,
//    acc * sx exact in fp64, one fused multiply-add with sw and bias, and the
//    fp64 -> bf16 round-to-nearest-even done with integer operations on the
//    double's bits.  Rows are staged in a swizzled shared buffer and written
//    with TMA stores that clip the M and N edges.  Conversions avoid the XU
//    pipe, whose throughput had made the epilogue the bottleneck.
// Every mbarrier wait is bounded (sm100.cuh); no load uses cluster multicast.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <chrono>
#include <cstdint>

#include "act_quant.cuh"
#include "qk_internal.h"
#include "sm100.cuh"

namespace qk {
namespace {

constexpr int BM = 128;   // rows per CTA (the pair covers 256)
constexpr int BN = 256;   // columns per tile (each CTA loads 128 rows of Wq)
constexpr int BK = 256;   // K per stage (bytes = elements): two 128-byte swizzled slabs
constexpr int kSlabs = BK / 128;
#ifndef QK_W8A8_STAGES
#define QK_W8A8_STAGES 3
#endif
#ifndef QK_W8A8_STG_BUFS
#define QK_W8A8_STG_BUFS 1
#endif
constexpr int STAGES = QK_W8A8_STAGES;
constexpr int kEpiWarps = 4;  // 6 warps: at most 2 per SM sub-partition, 255 registers each
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int A_BYTES = BM * BK;                  // 32 KiB
constexpr int B_BYTES = (BN / 2) * BK;            // 32 KiB
constexpr uint32_t STAGE_TX = 2 * (A_BYTES + B_BYTES);  // both CTAs' loads
constexpr int STG_BYTES = 32 * 128;               // 32 rows x 128 B
constexpr int TAB_BYTES = BN * 16;                // per column {sw, bias, guard, gate}
constexpr int SMEM_A = 0;
constexpr int SMEM_B = SMEM_A + STAGES * A_BYTES;
constexpr int SMEM_STG = SMEM_B + STAGES * B_BYTES;
constexpr int kStgBufs = QK_W8A8_STG_BUFS;        // staging buffers per epilogue warp
constexpr int SMEM_TAB = SMEM_STG + kEpiWarps * kStgBufs * STG_BYTES;
constexpr int SMEM_BAR = SMEM_TAB + 2 * TAB_BYTES;  // two tile tables
constexpr int kNumBars = 2 * STAGES + 6;          // + two table-ready barriers
constexpr int SMEM_SLOT = SMEM_BAR + kNumBars * 8;
constexpr int SMEM_USED = SMEM_SLOT + 16;
constexpr int SMEM_ALLOC = SMEM_USED + 1024;      // room to align the base to 1024 B
constexpr int kTmemCols = 2 * BN;                 // two accumulators
constexpr uint32_t kIdesc = i8_idesc(2 * BM, BN, true, true);

static_assert(SMEM_ALLOC <= 232448, "shared memory budget");

// An output takes the fp32 fast path when |v32| >= max(kGuard |bias|, kTiny).
constexpr float kGuard = 0.000244140625f;   // 2^-12
constexpr float kTiny = 7.888609052210118e-31f;  // 2^-100
// The gated fast path holds when |y| >= kGuardGate |gate| (|u| + |bias|) + kTiny.
constexpr float kGuardGate = 0.0001220703125f;  // 2^-13

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// bf16 bits -> fp64, exactly: integer operations on the bits for normal
// values (rebias the exponent, move the 7 mantissa bits), through fp32 for
// zeros and subnormals.
__device__ __forceinline__ double bf16_bits_to_f64(uint32_t b) {
  const uint32_t e = (b >> 7) & 0xFFu;
  if (e == 0u) return (double)__uint_as_float(b << 16);
  const uint32_t hi = ((b & 0x8000u) << 16) | ((e + 896u) << 20) | ((b & 0x7Fu) << 13);
  return __hiloint2double((int)hi, 0);
}

// Raster: groups of `group_m` M tiles; inside a group, consecutive tiles walk
// down the M tiles first, then across N, so the CTA pairs running at the same
// time share the group's rows of xq (kept in L2) and a few Wq tiles.
__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int group_m, int& mb,
                                            int& nb) {
  const int per_group = group_m * tiles_n;
  const int gid = t / per_group;
  const int first_m = gid * group_m;
  const int gm = min(tiles_m - first_m, group_m);
  const int r = t - gid * per_group;
  mb = first_m + r % gm;
  nb = r / gm;
}

// Exact int32 -> fp64 without a conversion instruction: the double with high
// word 0x43300000 and low word a + 2^31 is 2^52 + 2^31 + a.
__device__ __forceinline__ double i32_to_f64(uint32_t a) {
  return __hiloint2double(0x43300000, (int)(a ^ 0x80000000u)) - 4503601774854144.0;
}

// fp64 -> bf16 with one rounding to nearest-even, for |v| >= 2^-126 by integer
// operations on the bits (keep the sign, the 11-bit exponent and 7 mantissa
// bits; round on bit 12 of the high word with the rest as sticky bits), and for
// smaller magnitudes through round-to-odd into fp32.
__device__ __forceinline__ uint32_t f64_to_bf16_bits(double v) {
  const uint32_t hi = (uint32_t)__double2hiint(v);
  const uint32_t lo = (uint32_t)__double2loint(v);
  const uint32_t sign = (hi >> 16) & 0x8000u;
  const uint32_t mag = hi & 0x7FFFFFFFu;
  if (mag < 0x38100000u) {  // |v| < 2^-126 (bf16 subnormal range) or zero
    if ((mag | lo) == 0u) return sign;
    float f = __double2float_rz(v);
    if ((double)f != v) f = __uint_as_float(__float_as_uint(f) | 1u);
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f));
  }
  const uint32_t keep = mag >> 13;                          // exponent | 7 mantissa bits
  const uint32_t low13 = (mag & 0x1FFFu) | min(lo, 1u);     // round bit 12, sticky below
  const uint32_t up = (low13 + 0x0FFFu + (keep & 1u)) >> 13;
  const uint32_t bits = min(keep + up - (896u << 7), 0x7F80u);  // rebias 1023 -> 127
  return sign | bits;
}

// ---- readiness of the quantized rows (the fused-quantization kernel)
//
// Row r of xq / sx is ready when the 64-bit word ready[r] holds the launch's
// epoch (a value the host never reuses): the warp that quantized the row
// stores it with release semantics after its codes and scale.  No word is
// ever incremented, so none needs clearing between launches, and a word left
// by an earlier launch (or any garbage) never reads as ready.

__device__ __forceinline__ void ready_publish(unsigned long long* p, unsigned long long epoch) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(epoch) : "memory");
}

__device__ __forceinline__ unsigned long long ready_load(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Warp-collective: waits (bounded) until rows [r0, r0 + nrows) (nrows <= 128)
// are ready, each lane watching four of them.  Returns the same value in
// every lane; afterwards the TMA (async proxy) reads of lane 0 are ordered
// after the generic-proxy writes the warp observed.
__device__ __forceinline__ bool ready_wait_rows(const unsigned long long* ready, int r0, int nrows,
                                                unsigned long long epoch, int lane, int* err) {
  const long long t0 = clock64();
  bool ok = true;
  while (true) {
    bool mine = true;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = lane + 32 * i;
      if (r < nrows && ready_load(ready + r0 + r) != epoch) mine = false;
    }
    if (__all_sync(0xFFFFFFFFu, mine)) break;
    if (clock64() - t0 > QK_WAIT_LIMIT_CYCLES) {
      if (lane == 0) record_timeout(err);
      ok = false;
      break;
    }
    __nanosleep(32);
  }
  __syncwarp();
  asm volatile("fence.proxy.async.global;" ::: "memory");
  return ok;
}

// One lane's row: waits (bounded) until it is ready.
__device__ __forceinline__ void ready_wait_row(const unsigned long long* p,
                                               unsigned long long epoch, int* err) {
  const long long t0 = clock64();
  while (ready_load(p) != epoch) {
    if (clock64() - t0 > QK_WAIT_LIMIT_CYCLES) {
      record_timeout(err);
      return;
    }
    __nanosleep(32);
  }
}

// Quantizes RB = min(16, 32 / CPL) rows of x held in registers at once (rows r0,
// r0 + stride, ...; the first nrows of them), each row <= 32 CPL 16-byte
// chunks (the rule of act_quant.cuh); writes their codes, then their scales
// and readiness words (all lanes' writes fenced before the release).
template <int CPL>
__device__ __forceinline__ void quant_rows(const uint16_t* __restrict__ x, int K, int nch, int r0,
                                           int stride, int nrows, int8_t* xq, float* sxo,
                                           unsigned long long* ready, unsigned long long epoch,
                                           int lane) {
  constexpr int RB = 32 / CPL < 16 ? 32 / CPL : 16;
  uint4 v[RB][CPL];
#pragma unroll
  for (int i = 0; i < RB; ++i) {
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)(r0 + i * stride) * K);
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      const int cc = c * 32 + lane;
      v[i][c] = (i < nrows && cc < nch) ? __ldcs(src + cc) : make_uint4(0u, 0u, 0u, 0u);
    }
  }
  float amax[RB];
#pragma unroll
  for (int i = 0; i < RB; ++i) {
    uint32_t m = 0;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      m = bf16x2_absmax_bits(m, v[i][c].x);
      m = bf16x2_absmax_bits(m, v[i][c].y);
      m = bf16x2_absmax_bits(m, v[i][c].z);
      m = bf16x2_absmax_bits(m, v[i][c].w);
    }
    amax[i] = warp_max_bits_to_float(m);
  }
  int dummy = 0;
#pragma unroll
  for (int i = 0; i < RB; ++i) {
    if (i < nrows) {
      const float q = act_multiplier(amax[i]);
      uint2* dst = reinterpret_cast<uint2*>(xq + (size_t)(r0 + i * stride) * K);
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        const int cc = c * 32 + lane;
        if (cc < nch) dst[cc] = quant_chunk(v[i][c], q, &dummy);
      }
      if (lane == 0) sxo[r0 + i * stride] = act_scale(amax[i]);
    }
  }
  // every lane's codes (and the scales) before any of the rows counts as done
  asm volatile("fence.proxy.async.global;" ::: "memory");
  __threadfence();
  __syncwarp();
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < RB; ++i)
      if (i < nrows) ready_publish(ready + r0 + i * stride, epoch);
  }
}

// kAccOut: store the int32 sums instead of y.  kGated: the gated residual
// epilogue ("mlx-kquant PR #89", commit list), y = bf16(residual + gate[n] *
// (acc * sx * sw + bias)) in fp64 for every output.
// kFused: the activations arrive as bf16 x and the epilogue warps quantize
// them into xq / sx (the workspace the TMA loads read) while the tiles run;
// the producers wait for each 128-row block's readiness word (see above).
template <bool kAccOut, bool kGated, bool kFused>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    w8a8_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, const float* __restrict__ sx,
                     const float* __restrict__ sw, const float* __restrict__ bias,
                     const float* __restrict__ gate, const uint16_t* residual, int M, int N,
                     int K, int group_m, int* err, const uint16_t* __restrict__ x,
                     int8_t* xq_out, float* sx_out, unsigned long long* ready,
                     unsigned long long epoch) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem<1024>(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + SMEM_BAR;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  auto table_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 4 + b); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SMEM_SLOT);
  float4* tab = reinterpret_cast<float4*>(smem + SMEM_TAB);

  const uint32_t rank = cluster_ctarank();  // 0 leads the pair
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int pair = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;
  const int tiles_m = (M + 2 * BM - 1) / (2 * BM);
  const int tiles_n = (N + BN - 1) / BN;
  const int num_tiles = tiles_m * tiles_n;
  const int num_kb = (K + BK - 1) / BK;

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmC);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 2 * kEpiWarps);
      mbar_init(table_bar(a), 32 * kEpiWarps);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync();  // barriers and TMEM of both CTAs are ready
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // The next kernel in the stream may become resident now (it waits for this
  // grid to finish before it touches anything this grid reads or writes).
  pdl_launch_dependents();
  // Everything below reads what the previous kernel (activation quant) wrote.
  pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // (lane 0 issues the loads; with fused quantization the whole warp first
    // checks that the CTA's 128 rows of the tile are quantized)
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int t = pair; t < num_tiles && ok; t += num_pairs) {
      int mb, nb;
      tile_coords(t, tiles_m, tiles_n, group_m, mb, nb);
      const int arow = mb * 2 * BM + (int)rank * BM;
      const int brow = nb * BN + (int)rank * (BN / 2);
      if constexpr (kFused) {
        const int nrows = min(BM, M - arow);
        if (nrows > 0 && !ready_wait_rows(ready, arow, nrows, epoch, lane, err)) break;
      }
      if (lane == 0) {
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, err)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), STAGE_TX);
          const uint32_t lead_full = mapa_shared(full_bar(stage), 0);
#pragma unroll
          for (int sl = 0; sl < kSlabs; ++sl) {  // 128-byte-wide K slabs
            tma_load_2d_pair(sbase + SMEM_A + stage * A_BYTES + sl * (A_BYTES / kSlabs), &tmA,
                             kb * BK + 128 * sl, arow, lead_full);
            tma_load_2d_pair(sbase + SMEM_B + stage * B_BYTES + sl * (B_BYTES / kSlabs), &tmB,
                             kb * BK + 128 * sl, brow, lead_full);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
    }
  } else if (warp == 1) {
    // ------------------------------------------- MMA issuer (pair leader)
    if (rank == 0 && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t aphase = 0;
      bool ok = true;
      for (int t = pair; t < num_tiles && ok; t += num_pairs) {
        if (!mbar_wait(tempty_bar(acc), aphase ^ 1u, err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = sbase + SMEM_A + stage * A_BYTES;
          const uint32_t b_addr = sbase + SMEM_B + stage * B_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            // K step kk: slab kk / 4, 32-byte column (kk % 4) inside the swizzle atom
            const uint32_t ao = (kk >> 2) * (A_BYTES / kSlabs) + 32 * (kk & 3);
            const uint32_t bo = (kk >> 2) * (B_BYTES / kSlabs) + 32 * (kk & 3);
            mma_i8_pair(d_tmem, sw128_kmajor_desc(a_addr + ao),
                        sw128_kmajor_desc(b_addr + bo), kIdesc, (kb | kk) != 0 ? 1u : 0u);
          }
          mma_commit_pair(empty_bar(stage), 0x3);  // frees this stage in both CTAs
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        mma_commit_pair(tfull_bar(acc), 0x3);  // accumulator ready in both CTAs
        if (++acc == 2) {
          acc = 0;
          aphase ^= 1u;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int e = warp - 2;           // 0..3
    const int q = warp & 3;           // TMEM lane quarter this warp may access
    const int et = threadIdx.x - 64;  // 0..127
    const uint32_t stg0 = sbase + SMEM_STG + (uint32_t)(e * kStgBufs * STG_BYTES);
    uint8_t* stg0_ptr = smem + SMEM_STG + e * kStgBufs * STG_BYTES;
    int acc = 0;
    uint32_t aphase = 0;
    int iter = 0;
    int use = 0;  // staging-buffer use counter (alternates the two buffers)
    const uint64_t y_policy = l2_policy_evict_first();
    // gated: each lane sends its row of a tile's residual (up to 512 bytes) to
    // L2 one tile ahead of the tile's epilogue, so the per-chunk register loads
    // below meet L2 rather than HBM latency
    auto prefetch_residual = [&](int tt) {
      if (tt >= num_tiles) return;
      int pm, pn;
      tile_coords(tt, tiles_m, tiles_n, group_m, pm, pn);
      const int prow = pm * 2 * BM + (int)rank * BM + q * 32 + lane;
      const int pcol = pn * BN;
      if (prow < M && pcol < N)
        bulk_prefetch_l2(residual + (size_t)prow * N + pcol, (uint32_t)(min(BN, N - pcol) * 2));
    };
    // ---- fused quantization: rows qw, qw + QW, qw + 2 QW, ... of x are this
    // warp's (QW = all epilogue warps of the grid, so the first rows are spread
    // over every SM).  Rows of up to 4096 elements are quantized in batches held
    // in registers (min(16, 32 / CPL) rows of up to 32 CPL chunks each); longer rows take
    // two passes over 4096-element segments (the second from L2).
    const int QW = (int)gridDim.x * kEpiWarps;
    int qrow = (int)blockIdx.x * kEpiWarps + e;
    const int nch = K >> 3;  // 16-byte chunks of bf16 per row
    const int cpl = nch <= 32 ? 1 : nch <= 64 ? 2 : nch <= 128 ? 4 : nch <= 256 ? 8 : 16;
    auto quantize_until = [&](int limit) {
      if constexpr (kFused) {
        limit = min(limit, M);
        while (qrow < limit) {
          if (nch <= 512) {
            const int rb = min(16, 32 / cpl);
            const int n = min(rb, (limit - qrow + QW - 1) / QW);
            switch (cpl) {
              case 1: quant_rows<1>(x, K, nch, qrow, QW, n, xq_out, sx_out, ready, epoch, lane); break;
              case 2: quant_rows<2>(x, K, nch, qrow, QW, n, xq_out, sx_out, ready, epoch, lane); break;
              case 4: quant_rows<4>(x, K, nch, qrow, QW, n, xq_out, sx_out, ready, epoch, lane); break;
              case 8: quant_rows<8>(x, K, nch, qrow, QW, n, xq_out, sx_out, ready, epoch, lane); break;
              default: quant_rows<16>(x, K, nch, qrow, QW, n, xq_out, sx_out, ready, epoch, lane); break;
            }
            qrow += n * QW;
          } else {
            const int r0 = qrow;
            const uint4* s0 = reinterpret_cast<const uint4*>(x + (size_t)r0 * K);
            uint2* d0 = reinterpret_cast<uint2*>(xq_out + (size_t)r0 * K);
            uint32_t m0 = 0;
            for (int seg = 0; seg < nch; seg += 512) {  // warp-uniform
              uint4 v[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const int c = seg + i * 32 + lane;
                v[i] = c < nch ? __ldcs(s0 + c) : make_uint4(0u, 0u, 0u, 0u);
              }
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                m0 = bf16x2_absmax_bits(m0, v[i].x);
                m0 = bf16x2_absmax_bits(m0, v[i].y);
                m0 = bf16x2_absmax_bits(m0, v[i].z);
                m0 = bf16x2_absmax_bits(m0, v[i].w);
              }
            }
            const float a0 = warp_max_bits_to_float(m0);
            const float q0 = act_multiplier(a0);
            int dummy = 0;
            for (int seg = 0; seg < nch; seg += 512) {
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const int c = seg + i * 32 + lane;
                if (c < nch) d0[c] = quant_chunk(__ldcg(s0 + c), q0, &dummy);
              }
            }
            if (lane == 0) sx_out[r0] = act_scale(a0);
            asm volatile("fence.proxy.async.global;" ::: "memory");
            __threadfence();
            __syncwarp();
            if (lane == 0) ready_publish(ready + r0, epoch);
            qrow += QW;
          }
        }
      }
    };
    // rows that the tiles before index T need (whole raster groups)
    auto rows_before = [&](int T) {
      const int last = min(T, num_tiles) - 1;
      const int gid = last / (group_m * tiles_n);
      return min(M, (gid + 1) * group_m * 2 * BM);
    };
    if constexpr (kGated) prefetch_residual(pair);
    for (int t = pair; t < num_tiles; t += num_pairs, ++iter) {
      int mb, nb;
      tile_coords(t, tiles_m, tiles_n, group_m, mb, nb);
      // keep this warp's share of the rows two waves ahead of the tiles
      if constexpr (kFused) quantize_until(rows_before(t + 2 * num_pairs + 1));
      if constexpr (kGated) prefetch_residual(t + num_pairs);
      const int ncol0 = nb * BN;
      float4* tcol = tab + (iter & 1) * BN;
      if constexpr (!kAccOut) {
        // this tile's per-column constants (one column per epilogue thread);
        // the barrier also tells each thread that all others finished the tile
        // before the previous one, the last user of this table buffer
#pragma unroll
        for (int k = 0; k < BN / (32 * kEpiWarps); ++k) {
          const int col = et + 32 * kEpiWarps * k;
          const int n = ncol0 + col;
          const float w = n < N ? __ldg(sw + n) : 0.0f;
          const float b = (n < N && bias != nullptr) ? __ldg(bias + n) : 0.0f;
          const float g = (kGated && n < N) ? __ldg(gate + n) : 0.0f;
          const float z = kGated ? kGuardGate * fabsf(g) : fmaxf(kGuard * fabsf(b), kTiny);
          tcol[col] = make_float4(w, b, z, g);
        }
        mbar_arrive(table_bar(iter & 1));
        if (!mbar_wait(table_bar(iter & 1), (uint32_t)(iter >> 1) & 1u, err)) break;
      }
      if (!mbar_wait(tfull_bar(acc), aphase, err)) break;
      tc_fence_after();
      const int row0 = mb * 2 * BM + (int)rank * BM + q * 32;  // this warp's 32-row slab
      const int row = row0 + lane;
      float sxf = 0.0f;
      if constexpr (kFused) {
        // the scale was written in this launch by another warp: acquire the
        // row's readiness word, then read past L1
        if (row < M) {
          ready_wait_row(ready + row, epoch, err);
          sxf = __ldcg(sx + row);
        }
      } else {
        sxf = (!kAccOut && row < M) ? __ldg(sx + row) : 0.0f;
      }
      const uint32_t t_lane = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      constexpr int kChunk = kAccOut ? 32 : 64;  // columns per 128-byte staged row
      constexpr int kChunks = BN / kChunk;
#pragma unroll 1
      for (int c = 0; c < kChunks; ++c) {
        const int col0 = c * kChunk;
        const int n0 = ncol0 + col0;
        uint32_t out[32];
        // gated: this row's residual for the chunk (64 bf16 = 8 x 16 bytes),
        // loaded before the accumulator so the latency overlaps
        uint4 res[kGated ? kChunk / 8 : 1];
        if constexpr (kGated) {
#pragma unroll
          for (int i = 0; i < kChunk / 8; ++i)
            res[i] = (row < M && n0 + 8 * i < N)
                         ? *reinterpret_cast<const uint4*>(residual + (size_t)row * N + n0 + 8 * i)
                         : make_uint4(0u, 0u, 0u, 0u);
        }
        // two 32-column halves per chunk keep the live registers down
#pragma unroll
        for (int h = 0; h < kChunk / 32; ++h) {
          uint32_t v[32];
          tmem_ld32(t_lane + (uint32_t)(col0 + 32 * h), v);
          tmem_ld_wait();
          if (c == kChunks - 1 && h == kChunk / 32 - 1) {
            // all TMEM reads of this accumulator are done: hand it back to the leader
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(tempty_bar(acc), 0));
          }
          if constexpr (kAccOut) {
#pragma unroll
            for (int j = 0; j < 32; ++j) out[j] = v[j];
          } else if constexpr (kGated) {
            // fast path in fp32: u32 = fma(fp32(acc) * sx, sw, bias) and
            // y32 = fma(gate, u32, residual).  Their error is below
            // |gate| (|u32| + |bias|) 2^-22.4 + 2^-24 |y32|, under 2^-9 |y32|
            // (half a bf16 ulp) when |y32| >= 2^-13 |gate| (|u32| + |bias|);
            // y32 then rounds to within 1 ulp of the exact value.  Other
            // outputs (the residual cancelling the update, magnitudes near the
            // fp32 underflow) take the exact fp64 path.
            const float4* tc = tcol + col0 + 32 * h;
            uint32_t* o = out + 16 * h;
            uint32_t slow = 0;
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const uint4 rq = res[(32 * h + j) / 8];
              const int w4 = ((32 * h + j) % 8) / 2;  // which 32-bit word of the 16-byte piece
              const uint32_t rw = w4 == 0 ? rq.x : w4 == 1 ? rq.y : w4 == 2 ? rq.z : rq.w;
              const float4 c0 = tc[j], c1 = tc[j + 1];
              const float u0 = __fmaf_rn(__fmul_rn(__int2float_rn((int)v[j]), sxf), c0.x, c0.y);
              const float u1 = __fmaf_rn(__fmul_rn(__int2float_rn((int)v[j + 1]), sxf), c1.x, c1.y);
              const float r0 = __fmaf_rn(c0.w, u0, __uint_as_float(rw << 16));
              const float r1 = __fmaf_rn(c1.w, u1, __uint_as_float(rw & 0xFFFF0000u));
              // c.z = 2^-13 |gate|
              const bool s0 = !(fabsf(r0) >= __fmaf_rn(c0.z, fabsf(u0) + fabsf(c0.y), kTiny));
              const bool s1 = !(fabsf(r1) >= __fmaf_rn(c1.z, fabsf(u1) + fabsf(c1.y), kTiny));
              slow |= ((s0 ? 1u : 0u) | (s1 ? 2u : 0u)) << j;
              o[j >> 1] = pack_bf16x2(r0, r1);
            }
            if (__any_sync(0xFFFFFFFFu, slow != 0u)) {
              const double sxd = (double)sxf;
#pragma unroll
              for (int g = 0; g < 4; ++g) {
                const uint32_t m8 = (slow >> (8 * g)) & 0xFFu;
                if (__any_sync(0xFFFFFFFFu, m8 != 0u)) {
#pragma unroll
                  for (int i = 0; i < 8; ++i) {
                    const int j = 8 * g + i;
                    if ((m8 >> i) & 1u) {
                      const uint4 rq = res[(32 * h + j) / 8];
                      const int w4 = ((32 * h + j) % 8) / 2;
                      const uint32_t rw = w4 == 0 ? rq.x : w4 == 1 ? rq.y : w4 == 2 ? rq.z : rq.w;
                      const uint32_t rb = (j & 1) ? (rw >> 16) : (rw & 0xFFFFu);
                      const float4 cj = tc[j];
                      const double u = fma(i32_to_f64(v[j]) * sxd, (double)cj.x, (double)cj.y);
                      const uint32_t hb = f64_to_bf16_bits(fma((double)cj.w, u, bf16_bits_to_f64(rb)));
                      o[j >> 1] = (j & 1) ? ((o[j >> 1] & 0x0000FFFFu) | (hb << 16))
                                          : ((o[j >> 1] & 0xFFFF0000u) | hb);
                    }
                  }
                }
              }
            }
          } else {
            // fast path in fp32: v32 = fma(fp32(acc) * sx, sw, bias).  Its error
            // is at most 2^-23 |acc sx sw| + 2^-24 |v32|, below 1/8 bf16 ulp when
            // |v32| >= 2^-12 |bias|, so it then rounds to within 1 ulp of the
            // exact value.  Other outputs (cancellation against the bias, or
            // magnitudes near the fp32 underflow) take the exact fp64 path.
            const float4* tc = tcol + col0 + 32 * h;
            uint32_t* o = out + 16 * h;
            uint32_t slow = 0;
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const float4 c0 = tc[j], c1 = tc[j + 1];
              const float r0 = __fmaf_rn(__fmul_rn(__int2float_rn((int)v[j]), sxf), c0.x, c0.y);
              const float r1 = __fmaf_rn(__fmul_rn(__int2float_rn((int)v[j + 1]), sxf), c1.x, c1.y);
              const bool s0 = !(fabsf(r0) >= c0.z) && v[j] != 0u;
              const bool s1 = !(fabsf(r1) >= c1.z) && v[j + 1] != 0u;
              slow |= ((s0 ? 1u : 0u) | (s1 ? 2u : 0u)) << j;
              o[j >> 1] = pack_bf16x2(r0, r1);
            }
            if (__any_sync(0xFFFFFFFFu, slow != 0u)) {
              const double sxd = (double)sxf;
#pragma unroll
              for (int g = 0; g < 4; ++g) {
                const uint32_t m8 = (slow >> (8 * g)) & 0xFFu;
                if (__any_sync(0xFFFFFFFFu, m8 != 0u)) {
#pragma unroll
                  for (int i = 0; i < 8; ++i) {
                    const int j = 8 * g + i;
                    if ((m8 >> i) & 1u) {
                      const float4 cj = tc[j];
                      const double yj =
                          fma(i32_to_f64(v[j]) * sxd, (double)cj.x, (double)cj.y);
                      const uint32_t hb = f64_to_bf16_bits(yj);
                      o[j >> 1] = (j & 1) ? ((o[j >> 1] & 0x0000FFFFu) | (hb << 16))
                                          : ((o[j >> 1] & 0xFFFF0000u) | hb);
                    }
                  }
                }
              }
            }
          }
        }
        if (n0 >= N || row0 >= M) continue;  // whole box outside y
        // the TMA store that last used this staging buffer must be done reading it
        const int buf = use % kStgBufs;
        if (lane == 0) bulk_wait_read<kStgBufs - 1>();
        __syncwarp();
        uint8_t* rowp = stg0_ptr + buf * STG_BYTES + lane * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int phys = j ^ (lane & 7);  // 128-byte swizzle of the TMA box
          *reinterpret_cast<uint4*>(rowp + phys * 16) =
              make_uint4(out[4 * j], out[4 * j + 1], out[4 * j + 2], out[4 * j + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          // y is written once and never read here: evict it first from L2
          tma_store_2d_hint(&tmC, stg0 + (uint32_t)(buf * STG_BYTES), n0, row0, y_policy);
          bulk_commit();
        }
        ++use;
      }
      if (++acc == 2) {
        acc = 0;
        aphase ^= 1u;
      }
    }
    // the rest of this warp's rows (tiles of other CTAs may still need them)
    if constexpr (kFused) quantize_until(M);
    if (lane == 0) bulk_wait<0>();
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync();  // every remote arrival and MMA of the pair is done
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, kTmemCols);
}

bool g_attr_done[4][64];  // plain, accumulator dump, gated, fused quantization

std::atomic<unsigned long long> g_epoch{0};

// Pairs of CTAs that can be resident at once (the fused kernel's producers wait
// for rows that other CTAs quantize, so its whole grid must be resident).
int resident_pairs(const void* kernel) {
  int dev = 0;
  cudaGetDevice(&dev);
  static int cached[64];
  if (dev < 64 && cached[dev] > 0) return cached[dev];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (num_sms() / 2));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM_ALLOC;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = num_sms() / 2;
  }
  n = n < num_sms() / 2 ? n : num_sms() / 2;
  if (dev < 64) cached[dev] = n;
  return n;
}

}  // namespace

unsigned long long next_epoch() {
  static const unsigned long long seed = [] {
    const unsigned long long t =
        (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count();
    return (t * 0x9E3779B97F4A7C15ull) >> 9;
  }();
  unsigned long long e = (seed + g_epoch.fetch_add(1, std::memory_order_relaxed)) & ((1ull << 56) - 1);
  return e == 0 ? 1 : e;
}

cudaError_t launch_w8a8_gemm(const int8_t* xq, const float* sx, int64_t M, int64_t K,
                             const int8_t* Wq, const float* sw, const float* bias, int64_t N,
                             uint16_t* y, int32_t* acc_out, bool pdl, cudaStream_t s,
                             const float* gate, const uint16_t* residual) {
  if (w8a8_use_skinny(M, K, N))
    return launch_w8a8_skinny(xq, sx, M, K, Wq, sw, bias, N, y, acc_out, pdl, s, gate, residual);
  const bool acc_mode = acc_out != nullptr;
  CUtensorMap tA, tB, tC;
  if (!encode_tmap_2d(&tA, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, (uint64_t)K, (uint64_t)M,
                      (uint64_t)K, 128, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, (uint64_t)K, (uint64_t)N,
                      (uint64_t)K, 128, BN / 2, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (acc_mode) {
    if (!encode_tmap_2d(&tC, CU_TENSOR_MAP_DATA_TYPE_INT32, acc_out, (uint64_t)N, (uint64_t)M,
                        (uint64_t)N * 4, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  } else {
    if (!encode_tmap_2d(&tC, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, (uint64_t)N, (uint64_t)M,
                        (uint64_t)N * 2, 64, 32, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  int dev = 0;
  cudaGetDevice(&dev);
  const bool gated = gate != nullptr;
  auto kernel = acc_mode ? w8a8_gemm_kernel<true, false, false>
                         : (gated ? w8a8_gemm_kernel<false, true, false>
                                  : w8a8_gemm_kernel<false, false, false>);
  const int variant = acc_mode ? 1 : (gated ? 2 : 0);
  if (dev < 64 && !g_attr_done[variant][dev]) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    g_attr_done[variant][dev] = true;
  }
  int* err = device_error_word();
  if (err == nullptr) return cudaErrorUnknown;
  const long long tiles_m = (M + 2 * BM - 1) / (2 * BM);
  const long long tiles = tiles_m * ((N + BN - 1) / BN);
  // A raster group's rows of xq (256 rows x K bytes per M tile) should stay in
  // L2 while the group sweeps all of Wq: about 40 MB of the 126 MB L2.
  long long group_m = (40ll << 20) / (2 * BM * K);
  group_m = group_m < 1 ? 1 : (group_m > tiles_m ? tiles_m : group_m);
  const long long pairs = num_sms() / 2;
  const int grid = 2 * (int)(tiles < pairs ? tiles : pairs);

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM_ALLOC;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, tA, tB, tC, sx, sw, bias, gate, residual, (int)M,
                            (int)N, (int)K, (int)group_m, err, (const uint16_t*)nullptr,
                            (int8_t*)nullptr, (float*)nullptr, (unsigned long long*)nullptr,
                            0ull);
}

bool w8a8_use_fused(int64_t M, int64_t K, int64_t N) { return !w8a8_use_skinny(M, K, N); }

cudaError_t launch_w8a8_fused(const uint16_t* x, int64_t M, int64_t K, const int8_t* Wq,
                              const float* sw, const float* bias, int64_t N, uint16_t* y,
                              int8_t* xq, float* sx, unsigned long long* ready, bool pdl,
                              cudaStream_t s) {
  CUtensorMap tA, tB, tC;
  if (!encode_tmap_2d(&tA, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, (uint64_t)K, (uint64_t)M,
                      (uint64_t)K, 128, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, (uint64_t)K, (uint64_t)N,
                      (uint64_t)K, 128, BN / 2, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tC, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, (uint64_t)N, (uint64_t)M,
                      (uint64_t)N * 2, 64, 32, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  int dev = 0;
  cudaGetDevice(&dev);
  auto kernel = w8a8_gemm_kernel<false, false, true>;
  if (dev < 64 && !g_attr_done[3][dev]) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    g_attr_done[3][dev] = true;
  }
  int* err = device_error_word();
  if (err == nullptr) return cudaErrorUnknown;
  const long long tiles_m = (M + 2 * BM - 1) / (2 * BM);
  const long long tiles_n = (N + BN - 1) / BN;
  const long long tiles = tiles_m * tiles_n;
  const long long pairs = resident_pairs((const void*)kernel);
  const long long used = tiles < pairs ? tiles : pairs;
  // Raster groups just large enough that one wave of tiles stays inside one
  // group: the first wave then needs only the rows of its group's M tiles.
  long long group_m = (used + tiles_n - 1) / tiles_n;
  group_m = group_m < 1 ? 1 : (group_m > tiles_m ? tiles_m : group_m);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (int)used);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM_ALLOC;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, tA, tB, tC, (const float*)sx, sw, bias,
                            (const float*)nullptr, (const uint16_t*)nullptr, (int)M, (int)N,
                            (int)K, (int)group_m, err, x, xq, sx, ready, next_epoch());
}

}  // namespace qk
