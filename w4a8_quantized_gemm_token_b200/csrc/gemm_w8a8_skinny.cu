// gemm_w8a8_skinny.cu -- the W8A8 product for thin outputs (N <= 64): split-K
// over a thread-block cluster with exact int32 partial sums.
//
// Same arithmetic as the main W8A8 GEMM ("qlip-mlx" README, "w8a8_linear /
// W8A8Linear": INT8 x INT8 -> INT32, dequant + bias fused behind it):
//     acc[m, n] = sum_k xq[m, k] * Wq[n, k]                  (exact int32)
//     y[m, n]   = bf16( acc * sx[m] * sw[n] + bias[n] )      (fp64, one rounding)
//
// With N = 48 a 256 x 256 output tile is mostly empty and M = 2048 gives only
// eight tiles, so the main kernel keeps 16 SMs busy on an HBM-bound shape.
// Here a 128-row M tile is split along K over a cluster of S CTAs (S <= 8):
//  * warp 0: TMA producer of the CTA's K range -- per 128-deep K block the
//    128 x 128 xq tile and the Np x 128 Wq tile (Np = N rounded up to 16, rows
//    past N zero-filled), 128-byte swizzled, into a 3-stage ring;
//  * warp 1: tcgen05.mma kind::i8 (M = 128, N = Np, K = 32) into one int32
//    TMEM accumulator;
//  * warps 2-5: read the accumulator (one TMEM lane = one row per thread) and
//    store it, through distributed shared memory, into the slot of this K
//    range in the CTA that owns the row (128 / S rows per CTA); after a
//    cluster barrier each CTA adds its rows' S partial sums in a fixed order
//    (integer addition: exact and deterministic) and applies the dequant
//    (and, with a gate, the gated residual epilogue).
// Every wait is bounded; a CTA that gives up still takes part in the cluster
// barrier.  No load uses cluster multicast.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "qk_internal.h"
#include "sm100.cuh"

namespace qk {
namespace {

constexpr int BM = 128;        // rows per M tile (TMEM lanes)
constexpr int BK = 128;        // K bytes per stage (one swizzled 128-byte row)
constexpr int kMaxN = 64;      // widest output handled here
constexpr int STAGES = 3;     // ~100 KB per CTA: two CTAs fit an SM
constexpr int kThreads = 192;  // producer, MMA, 4 epilogue warps
constexpr int A_BYTES = BM * BK;
constexpr int kTmemCols = 64;

struct SkinnyLayout {
  int Np, S, RO;
  size_t a, b, red, bars, slot, total;
  __host__ __device__ SkinnyLayout(int N, int S_) {
    Np = (N + 15) / 16 * 16;
    S = S_;
    RO = BM / S;
    size_t off = 0;
    a = off;    off += (size_t)STAGES * A_BYTES;            // xq stages (1024-aligned)
    b = off;    off += (size_t)STAGES * Np * BK;            // Wq stages (Np * 128, 1024-aligned)
    red = off;  off += (size_t)S * RO * Np * 4;             // int32 partials [slot][row][col]
    bars = off; off += (size_t)(2 * STAGES + 1) * 8;        // full, empty, accumulator
    slot = off; off += 16;                                  // TMEM address
    total = off + 1024;
  }
};

__device__ __forceinline__ double i32_to_f64(uint32_t a) {
  return __hiloint2double(0x43300000, (int)(a ^ 0x80000000u)) - 4503601774854144.0;
}

// fp64 -> bf16 bits with one rounding to nearest-even (integer operations on
// the bits for |v| >= 2^-126, round-to-odd into fp32 below).
__device__ __forceinline__ uint16_t f64_to_bf16_bits(double v) {
  const uint32_t hi = (uint32_t)__double2hiint(v);
  const uint32_t lo = (uint32_t)__double2loint(v);
  const uint32_t sign = (hi >> 16) & 0x8000u;
  const uint32_t mag = hi & 0x7FFFFFFFu;
  if (mag < 0x38100000u) {
    if ((mag | lo) == 0u) return (uint16_t)sign;
    float f = __double2float_rz(v);
    if ((double)f != v) f = __uint_as_float(__float_as_uint(f) | 1u);
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
  }
  const uint32_t keep = mag >> 13;
  const uint32_t low13 = (mag & 0x1FFFu) | min(lo, 1u);
  const uint32_t up = (low13 + 0x0FFFu + (keep & 1u)) >> 13;
  return (uint16_t)(sign | min(keep + up - (896u << 7), 0x7F80u));
}

__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                              uint32_t d) {
  asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b),
               "r"(c), "r"(d)
               : "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Grid (S, ceil(M / 128)), cluster (S, 1, 1).  kAccOut: store the int32 sums
// (acc_out [M, N]) instead of y.
template <bool kAccOut>
__global__ void __launch_bounds__(kThreads, 1)
    w8a8_skinny_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const float* __restrict__ sx, const float* __restrict__ sw,
                       const float* __restrict__ bias, const float* __restrict__ gate,
                       const uint16_t* residual, int M, int N, int K, int S,
                       uint16_t* y, int32_t* __restrict__ acc_out, int* err) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint8_t* smem = align_smem<1024>(smem_raw);
  const SkinnyLayout L(N, S);
  const int Np = L.Np, RO = L.RO;
  const int crank = (int)blockIdx.x;  // K range of this CTA = rank in the cluster
  const int m0 = (int)blockIdx.y * BM;
  const int nkb = (K + BK - 1) / BK;
  const int kb0 = (int)((long long)nkb * crank / S), kb1 = (int)((long long)nkb * (crank + 1) / S);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + (uint32_t)L.bars;
  auto full_bar = [&](int i) { return bar0 + 8u * i; };
  auto empty_bar = [&](int i) { return bar0 + 8u * (STAGES + i); };
  const uint32_t acc_bar = bar0 + 8u * (2 * STAGES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.slot);
  uint32_t* red = reinterpret_cast<uint32_t*>(smem + L.red);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t b_bytes = (uint32_t)(Np * BK);

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(full_bar(i), 1);
      mbar_init(empty_bar(i), 1);
    }
    mbar_init(acc_bar, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  // peers write into this CTA's shared memory only after every CTA of the
  // cluster has arrived here (it has started)
  if (S > 1) cluster_arrive_relaxed();
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait();  // xq and sx come from the activation-quant kernel

  bool ok = true;
  if (warp == 0) {
    if (lane == 0) {
      for (int kb = kb0, it = 0; kb < kb1; ++kb, ++it) {
        const int s = it % STAGES;
        if (!mbar_wait(empty_bar(s), ((it / STAGES) & 1) ^ 1u, err)) break;
        mbar_arrive_expect_tx(full_bar(s), (uint32_t)A_BYTES + b_bytes);
        tma_load_2d(sbase + (uint32_t)L.a + (uint32_t)(s * A_BYTES), &tmA, kb * BK, m0, full_bar(s));
        tma_load_2d(sbase + (uint32_t)L.b + (uint32_t)s * b_bytes, &tmB, kb * BK, 0, full_bar(s));
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = i8_idesc(BM, Np, true, true);
      for (int kb = kb0, it = 0; kb < kb1; ++kb, ++it) {
        const int s = it % STAGES;
        if (!mbar_wait(full_bar(s), (it / STAGES) & 1, err)) break;
        tc_fence_after();
        const uint32_t a_addr = sbase + (uint32_t)L.a + (uint32_t)(s * A_BYTES);
        const uint32_t b_addr = sbase + (uint32_t)L.b + (uint32_t)s * b_bytes;
#pragma unroll
        for (int kk = 0; kk < BK / 32; ++kk)
          mma_i8(tmem_base, sw128_kmajor_desc(a_addr + 32 * kk), sw128_kmajor_desc(b_addr + 32 * kk),
                 idesc, (it > 0 || kk > 0) ? 1u : 0u);
        mma_commit(empty_bar(s));
      }
      mma_commit(acc_bar);  // the accumulator is complete (or, with no K block, untouched)
    }
  } else {
    // ---- epilogue warps: TMEM lane quarter q = warp % 4 (rows 32 q .. 32 q + 31)
    const int q = warp & 3;
    const int r = q * 32 + lane;  // row of the M tile
    ok = mbar_wait(acc_bar, 0, err);
    tc_fence_after();
    uint32_t v[kMaxN];
#pragma unroll
    for (int h = 0; h < kMaxN / 8; ++h)
      tmem_ld8(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(8 * h),
               *reinterpret_cast<uint32_t(*)[8]>(&v[8 * h]));
    tmem_ld_wait();
    if (kb1 == kb0 || !ok) {
#pragma unroll
      for (int c = 0; c < kMaxN; ++c) v[c] = 0u;  // no K range here: contributes zero
    }
    // partial sums of this K range -> slot `crank` of the owning CTA (after the
    // start barrier: every CTA of the cluster is running)
    if (S > 1) cluster_wait_acquire();
    const int owner = r / RO, lr = r - owner * RO;
    uint32_t* dst = red + ((size_t)crank * RO + lr) * Np;
    // 16-byte stores (a row of the slot is Np * 4 bytes, a multiple of 64)
    if (S > 1) {
      const uint32_t raddr = mapa_shared(smem_u32(dst), (uint32_t)owner);
#pragma unroll
      for (int c = 0; c < kMaxN; c += 4)
        if (c < Np) st_cluster_v4(raddr + 4u * c, v[c], v[c + 1], v[c + 2], v[c + 3]);
    } else {
#pragma unroll
      for (int c = 0; c < kMaxN; c += 4)
        if (c < Np) *reinterpret_cast<uint4*>(dst + c) = make_uint4(v[c], v[c + 1], v[c + 2], v[c + 3]);
    }
  }
  __syncwarp();
  if (S > 1) {
    if (warp < 2) cluster_wait_acquire();  // the start barrier (warp-uniform)
    cluster_arrive_release();
    cluster_wait_acquire();
  } else {
    __syncthreads();
  }
  // ---- this CTA's rows [crank RO, crank RO + RO) of the tile: the S slots in a
  // fixed order, then the dequant and one rounding
  for (int idx = threadIdx.x; idx < RO * N; idx += kThreads) {
    const int lr = idx / N, c = idx - lr * N;
    const int m = m0 + crank * RO + lr;
    if (m >= M) continue;
    uint32_t acc = 0u;
    for (int s = 0; s < S; ++s) acc += red[((size_t)s * RO + lr) * Np + c];
    if constexpr (kAccOut) {
      acc_out[(size_t)m * N + c] = (int32_t)acc;
    } else {
      double v = fma(i32_to_f64(acc) * (double)__ldg(sx + m), (double)__ldg(sw + c),
                     bias != nullptr ? (double)__ldg(bias + c) : 0.0);
      if (gate != nullptr)  // gated residual epilogue: residual + gate * v
        v = fma((double)__ldg(gate + c), v,
                (double)__uint_as_float((uint32_t)residual[(size_t)m * N + c] << 16));
      y[(size_t)m * N + c] = f64_to_bf16_bits(v);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

bool g_attr_done[2][64];
// resident clusters of 2, 4, 8 CTAs per (mode, cluster size, N / 16, device); -1 = not asked yet
int g_active[2][3][4][64];
bool g_active_init = [] {
  for (auto& a : g_active)
    for (auto& b : a)
      for (auto& c : b)
        for (int& d : c) d = -1;
  return true;
}();

}  // namespace

// Thin outputs with few M tiles: the cluster split-K kernel keeps more SMs busy
// than 256 x 256 tiles would.
bool w8a8_use_skinny(int64_t M, int64_t K, int64_t N) {
  return N <= kMaxN && M >= 1 && M <= 8192 && K >= 32;
}

cudaError_t launch_w8a8_skinny(const int8_t* xq, const float* sx, int64_t M, int64_t K,
                               const int8_t* Wq, const float* sw, const float* bias, int64_t N,
                               uint16_t* y, int32_t* acc_out, bool pdl, cudaStream_t s,
                               const float* gate, const uint16_t* residual) {
  const bool acc_mode = acc_out != nullptr;
  const int mtiles = (int)((M + BM - 1) / BM);
  const int nkb = (int)((K + BK - 1) / BK);
  auto kernel = acc_mode ? w8a8_skinny_kernel<true> : w8a8_skinny_kernel<false>;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 64 || !g_attr_done[acc_mode][dev]) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SkinnyLayout(kMaxN, 8).total);
    if (e != cudaSuccess) return e;
    if (dev < 64) g_attr_done[acc_mode][dev] = true;
  }
  // cluster size S: the most K ranges (<= 8, a power of two, at least one K
  // block each) such that every cluster is resident at once (the device's
  // answer for this cluster shape and shared memory) and the grid stays within
  // one CTA per SM
  int S = 1;
  for (int c = 8; c >= 2; c /= 2) {
    if (c > nkb || (long long)c * mtiles > num_sms()) continue;
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3((unsigned)c, (unsigned)mtiles);
    q.blockDim = dim3(kThreads);
    q.dynamicSmemBytes = SkinnyLayout((int)N, c).total;
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = (unsigned)c;
    qa[0].val.clusterDim.y = 1;
    qa[0].val.clusterDim.z = 1;
    q.attrs = qa;
    q.numAttrs = 1;
    // the answer depends on the cluster shape and shared memory only: cached
    int& active = g_active[acc_mode][c == 2 ? 0 : c == 4 ? 1 : 2][(N + 15) / 16 - 1][dev < 64 ? dev : 0];
    if (active < 0 || dev >= 64) {
      int a = 0;
      if (cudaOccupancyMaxActiveClusters(&a, kernel, &q) != cudaSuccess) {
        cudaGetLastError();  // clear it: fall back to a smaller cluster
        a = 0;
      }
      active = a;
    }
    if (active >= mtiles) {
      S = c;
      break;
    }
  }
  const SkinnyLayout L((int)N, S);
  CUtensorMap tA, tB;
  if (!encode_tmap_2d(&tA, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, (uint64_t)K, (uint64_t)M,
                      (uint64_t)K, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq, (uint64_t)K, (uint64_t)N,
                      (uint64_t)K, BK, (uint32_t)L.Np, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  int* err = device_error_word();
  if (err == nullptr) return cudaErrorUnknown;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)S, (unsigned)mtiles);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (S > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = (unsigned)S;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kernel, tA, tB, sx, sw, bias, gate, residual, (int)M, (int)N,
                            (int)K, S, y, acc_out, err);
}

}  // namespace qk
