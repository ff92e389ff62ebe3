// gemm_w8a8.cu -- the W8A8 tensor-core GEMM with the fused dequant epilogue.
//
// Computes ("qlip-mlx" README, "w8a8_linear / W8A8Linear": INT8 x INT8 ->
// INT32 matmul with dequant + bias fused behind it)
//     acc[m, n] = sum_k xq[m, k] * Wq[n, k]                  (exact int32)
//     y[m, n]   = bf16( acc * sx[m] * sw[n] + bias[n] )      (fp64, one rounding)
//
// Design (sm_100a):
//  * CTA pairs (clusters of 2) run one tcgen05.mma.cta_group::2 kind::i8 over
//    both SMs: a pair owns a 256 x 256 output tile, each CTA loads its 128 rows
//    of xq and its 128 rows of Wq (so each SM moves 32 KiB of operands per
//    128-deep K block instead of 48 KiB for a 128 x 256 tile on one SM) and
//    holds a 128 x 256 int32 accumulator in its own TMEM;
//  * persistent grid (one pair per two SMs), tiles in a grouped raster;
//  * warp 0: TMA producer into a 5-stage shared-memory ring; both CTAs' loads
//    complete on the pair leader's (rank 0's) full barrier;
//  * warp 1 of the leader issues the MMAs (M = 256, N = 256, K = 32 each) into
//    one of two 256-column accumulators and commits each stage and each
//    finished accumulator to the barriers of both CTAs;
//  * warps 2-9 (8 per CTA): epilogue.  tcgen05.ld, then exact int32 -> fp64
//    (2^52 magic number), acc * sx exact in fp64, one fused multiply-add with
//    sw and bias (pre-converted to fp64 once per tile in shared memory), and
//    the fp64 -> bf16 round-to-nearest-even done with integer operations on the
//    double's bits; rows staged in a swizzled shared buffer and written with TMA
//    stores that clip the M and N edges.  Conversions avoid the XU pipe, whose
//    throughput made the epilogue the bottleneck.
// Every mbarrier wait is bounded (sm100.cuh); no load uses cluster multicast.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "qk_internal.h"
#include "sm100.cuh"

namespace qk {
namespace {

constexpr int BM = 128;   // rows per CTA (the pair covers 256)
constexpr int BN = 256;   // columns per tile (each CTA loads 128 rows of Wq)
constexpr int BK = 128;   // K per stage (bytes = elements)
constexpr int STAGES = 5;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int A_BYTES = BM * BK;                  // 16 KiB
constexpr int B_BYTES = (BN / 2) * BK;            // 16 KiB
constexpr uint32_t STAGE_TX = 2 * (A_BYTES + B_BYTES);  // both CTAs' loads
constexpr int STG_BYTES = 32 * 128;               // 32 rows x 128 B
constexpr int TAB_DOUBLES = 2 * BN;               // sw then bias, one tile
constexpr int SMEM_A = 0;
constexpr int SMEM_B = SMEM_A + STAGES * A_BYTES;
constexpr int SMEM_STG = SMEM_B + STAGES * B_BYTES;
constexpr int SMEM_TAB = SMEM_STG + kEpiWarps * STG_BYTES;
constexpr int SMEM_BAR = SMEM_TAB + 2 * TAB_DOUBLES * 8;  // two tile tables
constexpr int kNumBars = 2 * STAGES + 6;          // + two table-ready barriers
constexpr int SMEM_SLOT = SMEM_BAR + kNumBars * 8;
constexpr int SMEM_USED = SMEM_SLOT + 16;
constexpr int SMEM_ALLOC = SMEM_USED + 1024;      // room to align the base to 1024 B
constexpr int kTmemCols = 2 * BN;                 // two accumulators
constexpr int kGroupM = 8;                        // M tiles per raster group
constexpr uint32_t kIdesc = i8_idesc(2 * BM, BN, true, true);

static_assert(SMEM_ALLOC <= 232448, "shared memory budget");

__device__ __forceinline__ void tile_coords(int t, int tiles_m, int tiles_n, int& mb, int& nb) {
  const int per_group = kGroupM * tiles_n;
  const int gid = t / per_group;
  const int first_m = gid * kGroupM;
  const int gm = min(tiles_m - first_m, kGroupM);
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

template <bool kAccOut>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    w8a8_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, const float* __restrict__ sx,
                     const float* __restrict__ sw, const float* __restrict__ bias, int M, int N,
                     int K, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + SMEM_BAR;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  auto table_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 4 + b); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SMEM_SLOT);
  double* tab = reinterpret_cast<double*>(smem + SMEM_TAB);

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

  // Everything below reads what the previous kernel (activation quant) wrote.
  pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = pair; t < num_tiles && ok; t += num_pairs) {
        int mb, nb;
        tile_coords(t, tiles_m, tiles_n, mb, nb);
        const int arow = mb * 2 * BM + (int)rank * BM;
        const int brow = nb * BN + (int)rank * (BN / 2);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, err)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), STAGE_TX);
          const uint32_t lead_full = mapa_shared(full_bar(stage), 0);
          tma_load_2d_pair(sbase + SMEM_A + stage * A_BYTES, &tmA, kb * BK, arow, lead_full);
          tma_load_2d_pair(sbase + SMEM_B + stage * B_BYTES, &tmB, kb * BK, brow, lead_full);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
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
            mma_i8_pair(d_tmem, sw128_kmajor_desc(a_addr + 32 * kk),
                        sw128_kmajor_desc(b_addr + 32 * kk), kIdesc, (kb | kk) != 0 ? 1u : 0u);
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
    const int e = warp - 2;           // 0..7
    const int q = warp & 3;           // TMEM lane quarter this warp may access
    const int half = e >> 2;          // column half of the tile
    const int et = threadIdx.x - 64;  // 0..255
    const uint32_t stg = sbase + SMEM_STG + (uint32_t)(e * STG_BYTES);
    uint8_t* stg_ptr = smem + SMEM_STG + e * STG_BYTES;
    int acc = 0;
    uint32_t aphase = 0;
    int iter = 0;
    for (int t = pair; t < num_tiles; t += num_pairs, ++iter) {
      int mb, nb;
      tile_coords(t, tiles_m, tiles_n, mb, nb);
      const int ncol0 = nb * BN;
      double* tsw = tab + (iter & 1) * TAB_DOUBLES;
      double* tb = tsw + BN;
      if constexpr (!kAccOut) {
        // this tile's sw and bias as fp64 (one column per epilogue thread); the
        // barrier also tells each thread that all others finished the tile
        // before the previous one, the last user of this table buffer
        const int n = ncol0 + et;
        tsw[et] = n < N ? (double)__ldg(sw + n) : 0.0;
        tb[et] = (n < N && bias != nullptr) ? (double)__ldg(bias + n) : 0.0;
        mbar_arrive(table_bar(iter & 1));
        if (!mbar_wait(table_bar(iter & 1), (uint32_t)(iter >> 1) & 1u, err)) break;
      }
      if (!mbar_wait(tfull_bar(acc), aphase, err)) break;
      tc_fence_after();
      const int row0 = mb * 2 * BM + (int)rank * BM + q * 32;  // this warp's 32-row slab
      const int row = row0 + lane;
      const double sxd = (!kAccOut && row < M) ? (double)__ldg(sx + row) : 0.0;
      const uint32_t t_lane = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      constexpr int kChunk = kAccOut ? 32 : 64;  // columns per 128-byte staged row
      constexpr int kChunks = (BN / 2) / kChunk;
#pragma unroll 1
      for (int c = 0; c < kChunks; ++c) {
        const int col0 = half * (BN / 2) + c * kChunk;
        const int n0 = ncol0 + col0;
        uint32_t v[kChunk];
        tmem_ld32(t_lane + (uint32_t)col0, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        if constexpr (!kAccOut)
          tmem_ld32(t_lane + (uint32_t)(col0 + 32), *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_ld_wait();
        if (c == kChunks - 1) {
          // all TMEM reads of this accumulator are done: hand it back to the leader
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(mapa_shared(tempty_bar(acc), 0));
        }
        if (n0 >= N || row0 >= M) continue;  // whole box outside y
        uint32_t out[32];
        if constexpr (kAccOut) {
#pragma unroll
          for (int j = 0; j < 32; ++j) out[j] = v[j];
        } else {
#pragma unroll
          for (int j = 0; j < 64; j += 2) {
            const double y0 = fma(i32_to_f64(v[j]) * sxd, tsw[col0 + j], tb[col0 + j]);
            const double y1 = fma(i32_to_f64(v[j + 1]) * sxd, tsw[col0 + j + 1], tb[col0 + j + 1]);
            out[j >> 1] = f64_to_bf16_bits(y0) | (f64_to_bf16_bits(y1) << 16);
          }
        }
        // the TMA store that last read the staging buffer must be done with it
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
        uint8_t* rowp = stg_ptr + lane * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int phys = j ^ (lane & 7);  // 128-byte swizzle of the TMA box
          *reinterpret_cast<uint4*>(rowp + phys * 16) =
              make_uint4(out[4 * j], out[4 * j + 1], out[4 * j + 2], out[4 * j + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tmC, stg, n0, row0);
          bulk_commit();
        }
      }
      if (++acc == 2) {
        acc = 0;
        aphase ^= 1u;
      }
    }
    if (lane == 0) bulk_wait<0>();
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync();  // every remote arrival and MMA of the pair is done
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, kTmemCols);
}

bool g_attr_done[2][64];

}  // namespace

cudaError_t launch_w8a8_gemm(const int8_t* xq, const float* sx, int64_t M, int64_t K,
                             const int8_t* Wq, const float* sw, const float* bias, int64_t N,
                             uint16_t* y, int32_t* acc_out, bool pdl, cudaStream_t s) {
  const bool acc_mode = acc_out != nullptr;
  CUtensorMap tA, tB, tC;
  if (!encode_tmap_2d(&tA, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, (uint64_t)K, (uint64_t)M,
                      (uint64_t)K, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, (uint64_t)K, (uint64_t)N,
                      (uint64_t)K, BK, BN / 2, CU_TENSOR_MAP_SWIZZLE_128B))
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
  auto kernel = acc_mode ? w8a8_gemm_kernel<true> : w8a8_gemm_kernel<false>;
  if (dev < 64 && !g_attr_done[acc_mode][dev]) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    g_attr_done[acc_mode][dev] = true;
  }
  int* err = device_error_word();
  if (err == nullptr) return cudaErrorUnknown;
  const long long tiles = ((M + 2 * BM - 1) / (2 * BM)) * ((N + BN - 1) / BN);
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
  return cudaLaunchKernelEx(&cfg, kernel, tA, tB, tC, sx, sw, bias, (int)M, (int)N, (int)K, err);
}

}  // namespace qk
