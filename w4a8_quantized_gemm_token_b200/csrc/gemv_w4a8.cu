// gemv_w4a8.cu -- the W4A8 product for M <= 16 rows ("qlip-mlx" README,
// "w4a8_linear / W4A8Linear": a small-batch path for M <= 16 that runs at
// weight-bandwidth speed).
//
// Same arithmetic as the GEMM route: per group g of 64 along K the exact int32
// acc[m, n, g] = sum_k xq[m, k] * q[n, k] on the raw codes 0..15, then
//   y[m, n] = bf16( sx[m] * sum_g (s[n,g] * acc + o[n,g] * xsum[m,g]) + bias[n] )
// with the fold in fp64 and one rounding to bf16.
//
// Design (HBM-bound: the packed weights are ~97% of the bytes):
//  * each CTA owns R = 16 * RT weight rows; at kernel start, before waiting on
//    the activation-quant kernel it depends on (programmatic dependent launch),
//    warp 0 bulk-copies the CTA's whole weight slice (rows padded by 16 bytes
//    against bank conflicts) and its fp16 scales / offsets into shared memory,
//    so the weight stream is in flight while the previous kernel finishes;
//  * the 8 warps split into RT row tiles x (8 / RT) K ranges; each K range has
//    its own mbarrier so a warp starts as soon as its part has landed;
//  * nibbles are unpacked in registers (two AND/shift + two byte permutes per
//    8 codes) straight into the A fragments of mma.sync m16n8k32 u8 x s8
//    (weights as A, tokens as the N = 8 side); K is permuted identically in A
//    and B so each lane reads 8 consecutive codes and 8 consecutive xq bytes;
//  * partial fp64 sums of the K ranges are added in a fixed order (so results
//    are deterministic), then scaled by sx, biased, rounded and stored.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "qk_internal.h"
#include "sm100.cuh"

namespace qk {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = 8;
constexpr int kGemvSmemLimit = 227 * 1024;

struct GemvSmem {
  __host__ __device__ static int row_stride(int K) { return K / 2 + 16; }
  __host__ __device__ static size_t weights(int R, int K) { return (size_t)R * row_stride(K); }
  // R = 16 * RT rows; the 8 warps form RT row tiles x (8 / RT) K ranges.
  __host__ __device__ static size_t partials(int R) { return (size_t)(kWarps / (R / 16)) * R * 16 * sizeof(double); }
  __host__ __device__ static size_t bytes(int R, int K) {
    const int G = K / 64;
    size_t b = 0;
    b += weights(R, K);                        // packed codes
    b += (size_t)R * G * 2 * 2;                // fp16 scales + offsets
    b = (b + 15) & ~size_t(15);
    b += partials(R);                          // fp64 partial sums of the K ranges
    b += 16 * 8;                               // mbarriers
    return b;
  }
};

__device__ __forceinline__ void unpack8(uint32_t w, uint32_t& lo4, uint32_t& hi4) {
  // w holds codes c0..c7 (c0 = low nibble of byte 0).  Output bytes:
  // lo4 = {c0, c1, c2, c3}, hi4 = {c4, c5, c6, c7}.
  const uint32_t even = w & 0x0F0F0F0Fu;         // c0, c2, c4, c6
  const uint32_t odd = (w >> 4) & 0x0F0F0F0Fu;   // c1, c3, c5, c7
  lo4 = __byte_perm(even, odd, 0x5140);
  hi4 = __byte_perm(even, odd, 0x7362);
}

__device__ __forceinline__ void mma_u8s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float f64_to_f32_odd(double v) {
  float f = __double2float_rz(v);
  if ((double)f != v) f = __uint_as_float(__float_as_uint(f) | 1u);
  return f;
}

__device__ __forceinline__ uint16_t f64_to_bf16_bits(double v) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f64_to_f32_odd(v)));
}

// TT token tiles of 8 (M <= 8 * TT).  RT row tiles of 16 per CTA.
template <int TT>
__global__ void __launch_bounds__(kThreads, 1)
    w4a8_gemv_kernel(const int8_t* __restrict__ xq, const float* __restrict__ sx,
                     const int32_t* __restrict__ xsum, int M, int K,
                     const uint8_t* __restrict__ Wp, const uint16_t* __restrict__ wscale,
                     const uint16_t* __restrict__ woffset, const float* __restrict__ bias, int N,
                     uint16_t* __restrict__ y, int32_t* __restrict__ acc_out, int m0, int m1,
                     int RT, int* err) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int G = K / 64;
  const int R = 16 * RT;
  const int KS = kWarps / RT;  // K ranges
  const int RS = GemvSmem::row_stride(K);
  const int n0 = blockIdx.x * R;
  const int rows = min(R, N - n0);  // valid rows of this CTA (a multiple of 8)

  uint8_t* w_sm = smem;
  uint16_t* s_sm = reinterpret_cast<uint16_t*>(smem + GemvSmem::weights(R, K));
  uint16_t* o_sm = s_sm + (size_t)R * G;
  size_t off = GemvSmem::weights(R, K) + (size_t)R * G * 4;
  off = (off + 15) & ~size_t(15);
  double* part = reinterpret_cast<double*>(smem + off);
  off += GemvSmem::partials(R);
  const uint32_t bars = smem_u32(smem + off);  // KS weight barriers, then 1 scale barrier

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto g_lo = [&](int q) { return q * G / KS; };

  if (threadIdx.x == 0) {
    for (int q = 0; q <= KS; ++q) mbar_init(bars + 8u * q, 1);
    fence_mbar_init();
  }
  __syncthreads();

  // ---- weight stream: issued before the dependency wait
  if (warp == 0) {
    if (lane == 0) {
      for (int q = 0; q < KS; ++q)
        mbar_arrive_expect_tx(bars + 8u * q, (uint32_t)(rows * (g_lo(q + 1) - g_lo(q)) * 32));
      const bool with_scales = acc_out == nullptr;
      mbar_arrive_expect_tx(bars + 8u * KS, with_scales ? (uint32_t)(rows * G * 2 * 2) : 0u);
      if (with_scales) {
        bulk_load(smem_u32(s_sm), wscale + (size_t)n0 * G, (uint32_t)(rows * G * 2), bars + 8u * KS);
        bulk_load(smem_u32(o_sm), woffset + (size_t)n0 * G, (uint32_t)(rows * G * 2), bars + 8u * KS);
      }
    }
    __syncwarp();
    for (int i = lane; i < rows * KS; i += 32) {
      const int q = i / rows, r = i - q * rows;
      const int glo = g_lo(q), ghi = g_lo(q + 1);
      if (ghi > glo)
        bulk_load(smem_u32(w_sm + (size_t)r * RS + glo * 32),
                  Wp + (size_t)(n0 + r) * (K / 2) + glo * 32, (uint32_t)((ghi - glo) * 32),
                  bars + 8u * q);
    }
  }

  // ---- activations come from the previous kernel
  pdl_wait();

  const int rt = warp % RT, q = warp / RT;
  const int grp = lane >> 2, tq = lane & 3;
  const int glo = g_lo(q), ghi = g_lo(q + 1);
  bool ok = mbar_wait(bars + 8u * q, 0, err);
  ok = mbar_wait(bars + 8u * KS, 0, err) && ok;

  double f[TT][4];
#pragma unroll
  for (int tt = 0; tt < TT; ++tt)
#pragma unroll
    for (int i = 0; i < 4; ++i) f[tt][i] = 0.0;

  const int rloc = rt * 16 + grp;  // this lane's first weight row (second: +8)
  const uint8_t* wrow0 = w_sm + (size_t)rloc * RS;
  const uint8_t* wrow1 = wrow0 + (size_t)8 * RS;

  for (int g = glo; g < ghi && ok; ++g) {
    int acc[TT][4];
#pragma unroll
    for (int tt = 0; tt < TT; ++tt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[tt][i] = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int kb = 64 * g + 32 * h + 8 * tq;  // this lane's 8 consecutive k
      uint32_t a[4];
      const uint32_t w0 = *reinterpret_cast<const uint32_t*>(wrow0 + kb / 2);
      const uint32_t w1 = *reinterpret_cast<const uint32_t*>(wrow1 + kb / 2);
      unpack8(w0, a[0], a[2]);
      unpack8(w1, a[1], a[3]);
#pragma unroll
      for (int tt = 0; tt < TT; ++tt) {
        const int m = tt * 8 + grp;
        uint2 b = make_uint2(0u, 0u);
        if (m < M) b = __ldg(reinterpret_cast<const uint2*>(xq + (size_t)m * K + kb));
        mma_u8s8(acc[tt], a, b.x, b.y);
      }
    }
    if (acc_out != nullptr) {
      // accumulator dump: acc[(m - m0), n, g] for rows m0 <= m < m1
#pragma unroll
      for (int tt = 0; tt < TT; ++tt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int m = tt * 8 + 2 * tq + (i & 1);
          const int n = n0 + rloc + (i >> 1) * 8;
          if (m >= m0 && m < m1 && n < N) acc_out[((size_t)(m - m0) * N + n) * G + g] = acc[tt][i];
        }
      continue;
    }
    const double s_a = (double)__half2float(__ushort_as_half(s_sm[(size_t)rloc * G + g]));
    const double s_b = (double)__half2float(__ushort_as_half(s_sm[(size_t)(rloc + 8) * G + g]));
    const double o_a = (double)__half2float(__ushort_as_half(o_sm[(size_t)rloc * G + g]));
    const double o_b = (double)__half2float(__ushort_as_half(o_sm[(size_t)(rloc + 8) * G + g]));
#pragma unroll
    for (int tt = 0; tt < TT; ++tt) {
      const int m = tt * 8 + 2 * tq;
      const double x0 = m < M ? (double)__ldg(xsum + (size_t)m * G + g) : 0.0;
      const double x1 = m + 1 < M ? (double)__ldg(xsum + (size_t)(m + 1) * G + g) : 0.0;
      f[tt][0] = fma(o_a, x0, fma(s_a, (double)acc[tt][0], f[tt][0]));
      f[tt][1] = fma(o_a, x1, fma(s_a, (double)acc[tt][1], f[tt][1]));
      f[tt][2] = fma(o_b, x0, fma(s_b, (double)acc[tt][2], f[tt][2]));
      f[tt][3] = fma(o_b, x1, fma(s_b, (double)acc[tt][3], f[tt][3]));
    }
  }
  if (acc_out != nullptr) return;

  // ---- partial sums of the K ranges, added in a fixed order
#pragma unroll
  for (int tt = 0; tt < TT; ++tt)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = tt * 8 + 2 * tq + (i & 1);
      const int r = rloc + (i >> 1) * 8;
      part[((size_t)q * R + r) * 16 + m] = f[tt][i];
    }
  __syncthreads();
  for (int idx = threadIdx.x; idx < R * M; idx += kThreads) {
    const int m = idx / R, r = idx - m * R;  // consecutive threads -> consecutive n
    const int n = n0 + r;
    if (r >= rows) continue;
    double acc = 0.0;
    for (int qq = 0; qq < KS; ++qq) acc += part[((size_t)qq * R + r) * 16 + m];
    const double v = fma((double)sx[m], acc, bias != nullptr ? (double)bias[n] : 0.0);
    y[(size_t)m * N + n] = f64_to_bf16_bits(v);
  }
}

size_t g_smem_set[2][64];

}  // namespace

cudaError_t launch_w4a8_gemv(const int8_t* xq, const float* sx, const int32_t* xsum, int64_t M,
                             int64_t K, const uint8_t* Wp, const uint16_t* ws, const uint16_t* wo,
                             const float* bias, int64_t N, uint16_t* y, int32_t* acc_out,
                             int64_t m0, int64_t m1, bool pdl, cudaStream_t s) {
  const int sms = num_sms();
  int RT = 1;  // fewest rows per CTA that still fit all CTAs in one wave
  while (RT < 4 && (N + 16 * RT - 1) / (16 * RT) > sms &&
         GemvSmem::bytes(32 * RT, (int)K) <= (size_t)kGemvSmemLimit)
    RT *= 2;
  const int R = 16 * RT;
  const unsigned grid = (unsigned)((N + R - 1) / R);
  const size_t smem = GemvSmem::bytes(R, (int)K);
  if (smem > (size_t)kGemvSmemLimit) return cudaErrorInvalidValue;
  int* err = device_error_word();
  if (err == nullptr) return cudaErrorUnknown;
  auto kernel = M <= 8 ? w4a8_gemv_kernel<1> : w4a8_gemv_kernel<2>;
  int dev = 0;
  cudaGetDevice(&dev);
  const int tt = M <= 8 ? 0 : 1;
  if (dev >= 64 || g_smem_set[tt][dev] < smem) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kGemvSmemLimit);
    if (e != cudaSuccess) return e;
    if (dev < 64) g_smem_set[tt][dev] = kGemvSmemLimit;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, xq, sx, xsum, (int)M, (int)K, Wp, ws, wo, bias, (int)N,
                            y, acc_out, (int)m0, (int)m1, RT, err);
}

}  // namespace qk
