// gemm_w8a8.cu -- the W8A8 tensor-core GEMM with the fused dequant epilogue.
//
// Computes ("qlip-mlx" README, "w8a8_linear / W8A8Linear": INT8 x INT8 ->
// INT32 matmul with dequant + bias fused behind it)
//     acc[m, n] = sum_k xq[m, k] * Wq[n, k]                  (exact int32)
//     y[m, n]   = bf16( acc * sx[m] * sw[n] + bias[n] )      (fp64, one rounding)
//
// Design (sm_100a):
//  * persistent grid, one 128 x 256 output tile at a time per CTA, tiles in a
//    grouped raster (16 M-tiles per group) so concurrent CTAs share operand
//    tiles in L2;
//  * warp 0: TMA producer -- 128 x 128 int8 tiles of xq and 256 x 128 of Wq
//    (both K-major, 128-byte swizzle) into a 4-stage shared-memory ring;
//  * warp 1: allocates all 512 TMEM columns and issues tcgen05.mma kind::i8
//    (M = 128, N = 256, K = 32 per instruction) into one of two 256-column
//    int32 accumulators, so the epilogue of tile i overlaps the mainloop of
//    tile i + 1;
//  * warps 2-5: epilogue -- tcgen05.ld 32 lanes x 32 columns, dequant in fp64
//    (int32 -> fp64 is exact, acc * sx is exact in fp64, one fused multiply-add
//    with sw and bias), fp64 -> bf16 rounded once (round-to-odd into fp32, then
//    nearest-even into bf16, which equals direct nearest-even), staged in a
//    swizzled shared buffer and written with TMA stores that clip the M and N
//    edges.
// Every mbarrier wait is bounded (sm100.cuh) so a fault ends the kernel.
#include <cuda_runtime.h>

#include <cstdint>

#include "qk_internal.h"
#include "sm100.cuh"

namespace qk {
namespace {

constexpr int BM = 128, BN = 256, BK = 128, STAGES = 4;
constexpr int kThreads = 192;
constexpr int kEpiWarps = 4;
constexpr int A_BYTES = BM * BK;                  // 16 KiB
constexpr int B_BYTES = BN * BK;                  // 32 KiB
constexpr int STG_BYTES = 32 * 128;               // 32 rows x 128 B per staging buffer
constexpr int SMEM_A = 0;
constexpr int SMEM_B = SMEM_A + STAGES * A_BYTES;
constexpr int SMEM_STG = SMEM_B + STAGES * B_BYTES;
constexpr int SMEM_BAR = SMEM_STG + kEpiWarps * 2 * STG_BYTES;
constexpr int kNumBars = 2 * STAGES + 4;          // full, empty, tmem_full x2, tmem_empty x2
constexpr int SMEM_SLOT = SMEM_BAR + kNumBars * 8;
constexpr int SMEM_USED = SMEM_SLOT + 16;
constexpr int SMEM_ALLOC = SMEM_USED + 1024;      // room to align the base to 1024 B
constexpr int kTmemCols = 2 * BN;                 // two accumulators
constexpr int kGroupM = 16;
constexpr uint32_t kIdesc = i8_idesc(BM, BN, true, true);

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

// fp64 -> bf16 with one rounding to nearest-even: round to odd into fp32 (24
// bits, at least two more than bf16's 8), then nearest-even to bf16.
__device__ __forceinline__ float f64_to_f32_odd(double v) {
  float f = __double2float_rz(v);
  if ((double)f != v) f = __uint_as_float(__float_as_uint(f) | 1u);
  return f;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

template <bool kAccOut>
__global__ void __launch_bounds__(kThreads, 1)
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
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SMEM_SLOT);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tiles_m = (M + BM - 1) / BM;
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
      mbar_init(tempty_bar(a), kEpiWarps);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
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
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        int mb, nb;
        tile_coords(t, tiles_m, tiles_n, mb, nb);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full_bar(stage), A_BYTES + B_BYTES);
          tma_load_2d(sbase + SMEM_A + stage * A_BYTES, &tmA, kb * BK, mb * BM, full_bar(stage));
          tma_load_2d(sbase + SMEM_B + stage * B_BYTES, &tmB, kb * BK, nb * BN, full_bar(stage));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t aphase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
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
            mma_i8(d_tmem, sw128_kmajor_desc(a_addr + 32 * kk), sw128_kmajor_desc(b_addr + 32 * kk),
                   kIdesc, (kb | kk) != 0 ? 1u : 0u);
          }
          mma_commit(empty_bar(stage));  // frees the smem stage when these MMAs finish
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        mma_commit(tfull_bar(acc));  // accumulator ready for the epilogue
        if (++acc == 2) {
          acc = 0;
          aphase ^= 1u;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const uint32_t stg0 = sbase + SMEM_STG + (uint32_t)((warp - 2) * 2 * STG_BYTES);
    uint8_t* stg0_ptr = smem + SMEM_STG + (warp - 2) * 2 * STG_BYTES;
    int acc = 0;
    uint32_t aphase = 0;
    int use = 0;  // staging-buffer use counter (alternates the two buffers)
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
      int mb, nb;
      tile_coords(t, tiles_m, tiles_n, mb, nb);
      if (!mbar_wait(tfull_bar(acc), aphase, err)) break;
      tc_fence_after();
      const int row0 = mb * BM + q * 32;  // first row of this warp's 32-row slab
      const int row = row0 + lane;
      const double sxd = (!kAccOut && row < M) ? (double)sx[row] : 0.0;
      const uint32_t t_lane = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      constexpr int kChunk = kAccOut ? 32 : 64;  // columns per 128-byte staged row
      for (int c = 0; c < BN / kChunk; ++c) {
        const int n0 = nb * BN + c * kChunk;
        uint32_t v[kChunk];
        tmem_ld32(t_lane + (uint32_t)(c * kChunk), *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        if constexpr (!kAccOut)
          tmem_ld32(t_lane + (uint32_t)(c * kChunk + 32), *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_ld_wait();
        if (c == BN / kChunk - 1) {
          // all TMEM reads of this accumulator are done: hand it back
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty_bar(acc));
        }
        if (n0 >= N || row0 >= M) continue;  // whole box outside y
        uint32_t out[32];
        if constexpr (kAccOut) {
#pragma unroll
          for (int j = 0; j < 32; ++j) out[j] = v[j];
        } else {
#pragma unroll
          for (int j4 = 0; j4 < 16; ++j4) {
            const int n = n0 + 4 * j4;
            float4 w4 = make_float4(0.f, 0.f, 0.f, 0.f), b4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (n < N) {
              w4 = __ldg(reinterpret_cast<const float4*>(sw + n));
              if (bias != nullptr) b4 = __ldg(reinterpret_cast<const float4*>(bias + n));
            }
            const double p0 = (double)(int)v[4 * j4 + 0] * sxd;
            const double p1 = (double)(int)v[4 * j4 + 1] * sxd;
            const double p2 = (double)(int)v[4 * j4 + 2] * sxd;
            const double p3 = (double)(int)v[4 * j4 + 3] * sxd;
            const float y0 = f64_to_f32_odd(fma(p0, (double)w4.x, (double)b4.x));
            const float y1 = f64_to_f32_odd(fma(p1, (double)w4.y, (double)b4.y));
            const float y2 = f64_to_f32_odd(fma(p2, (double)w4.z, (double)b4.z));
            const float y3 = f64_to_f32_odd(fma(p3, (double)w4.w, (double)b4.w));
            out[2 * j4] = pack_bf16x2(y0, y1);
            out[2 * j4 + 1] = pack_bf16x2(y2, y3);
          }
        }
        // staging buffer: wait until the TMA store that used it two chunks ago
        // has finished reading it
        const int buf = use & 1;
        if (lane == 0) bulk_wait_read<1>();
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
          tma_store_2d(&tmC, stg0 + (uint32_t)(buf * STG_BYTES), n0, row0);
          bulk_commit();
        }
        ++use;
      }
      if (++acc == 2) {
        acc = 0;
        aphase ^= 1u;
      }
    }
    if (lane == 0) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
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
                      (uint64_t)K, BK, BN, CU_TENSOR_MAP_SWIZZLE_128B))
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
  const long long tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int grid = (int)(tiles < num_sms() ? tiles : num_sms());

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
