// gemv1_w4a8.cu -- the W4A8 product for one token (M = 1), the decode-style
// case of the small-batch path ("qlip-mlx" README, "w4a8_linear / W4A8Linear":
// a register-dequant GEMV for M <= 16 that runs at weight-bandwidth speed).
//
// Same arithmetic as every W4A8 route: per group g of 64 along K the exact
// int32 acc[n, g] = sum_k xq[k] * q[n, k] on the raw codes 0..15, then
//   y[n] = bf16( sx * sum_g (s[n,g] * acc + o[n,g] * xsum[g]) + bias[n] )
// with the fold in fp64 and one rounding to bf16.
//
// With one token an m16n8k32 MMA would use one of its eight token columns, so
// this kernel uses 4-way byte dot products (dp4a) instead, and keeps every
// lane busy:
//  * a CTA owns 32 weight rows (4 per warp); before the programmatic-dependency
//    wait one thread bulk-copies each warp's rows (contiguous, 4 x K/2 bytes)
//    and the CTA's fp16 scales / offsets into shared memory, and the scales
//    become an fp64 {s, o} table -- all off the critical path;
//  * lane l owns the 16-byte chunks l, l + 32, l + 64, ... of a packed row
//    (one 512-byte, conflict-free shared load per chunk index for the warp);
//    after the wait every lane holds the matching activation codes in
//    registers -- read straight from xq, or quantized by the CTA from bf16 x
//    (the rule of the stand-alone kernel);
//    nibbles split into even / odd codes feed dp4a against xq permuted the same
//    way; the two halves of a group (lanes 2m, 2m + 1) add by one shuffle;
//  * even lanes fold s * acc, odd lanes o * xsum, in fp64; a fixed-order
//    butterfly over the warp gives the row, which lane 0 rounds once and
//    stores -- no shared-memory reduction, no block barrier at the end.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "act_quant.cuh"
#include "qk_internal.h"
#include "sm100.cuh"

namespace qk {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = 8;
constexpr int kRows = 32;          // weight rows per CTA
constexpr int kRowsPerWarp = kRows / kWarps;
constexpr int kSmemTwoPerSm = 113 * 1024;

struct Gemv1Layout {
  int K, G, KB;
  size_t w, s16, so, xq, xs, amx, bias, bars, total;
  __host__ __device__ explicit Gemv1Layout(int K_) {
    K = K_;
    G = K / 64;
    KB = K / 2;  // packed bytes per row
    size_t off = 0;
    w = off;    off += (size_t)kRows * KB;           // packed rows, contiguous
    s16 = off;  off += (size_t)kRows * G * 2 * 2;    // fp16 scales [row][g], then offsets
    so = off;   off += (size_t)kRows * G * 16;       // {s, o} in fp64 [row][g]
    xq = off;   off += (size_t)K;                    // codes (in-kernel quantization only)
    xs = off;   off += (size_t)G * 8;                // group sums in fp64 (ditto)
    amx = off;  off += kWarps * 4;                   // per-warp absmax (ditto)
    bias = off; off += kRows * 4;
    off = (off + 15) & ~size_t(15);
    bars = off; off += (kWarps + 1) * 8;             // one per warp's rows, one for the scales
    total = off + 128;                               // base alignment slack
  }
};

__device__ __forceinline__ double i32_to_f64(int a) {
  return __hiloint2double(0x43300000, a ^ (int)0x80000000) - 4503601774854144.0;
}

__device__ __forceinline__ double h2d(uint16_t h) {
  return (double)__half2float(__ushort_as_half(h));
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

// The four even codes then the four odd codes of 8 consecutive activation
// bytes (the order in which the nibble split delivers the weight codes).
__device__ __forceinline__ uint2 even_odd(uint32_t lo, uint32_t hi) {
  return make_uint2(__byte_perm(lo, hi, 0x6420), __byte_perm(lo, hi, 0x7531));
}

// dot of the 8 codes of one packed word with their 8 activation codes
__device__ __forceinline__ int dot8(uint32_t w, uint32_t x_even, uint32_t x_odd, int acc) {
  acc = __dp4a((int)(w & 0x0F0F0F0Fu), (int)x_even, acc);
  return __dp4a((int)((w >> 4) & 0x0F0F0F0Fu), (int)x_odd, acc);
}

// NJ = K / 1024: 16-byte chunks of a packed row per lane.  kQuantX: x arrives
// as bf16 and is quantized here.  kDump: store the per-group int32 sums
// (acc_out [1, N, G]) instead of y.  Grid ceil(N / 32), 256 threads.
template <bool kQuantX, bool kDump, int NJ>
__global__ void __launch_bounds__(kThreads, 2)
    w4a8_gemv1_kernel(const uint16_t* __restrict__ x, const int8_t* __restrict__ xq,
                      const float* __restrict__ sx, const int32_t* __restrict__ xsum, int K,
                      const uint8_t* __restrict__ Wp, const uint16_t* __restrict__ wscale,
                      const uint16_t* __restrict__ woffset, const float* __restrict__ bias, int N,
                      uint16_t* __restrict__ y, int32_t* __restrict__ acc_out, int early_trigger,
                      int* err) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint8_t* smem = align_smem<128>(smem_raw);
  const Gemv1Layout L(K);
  const int G = L.G, KB = L.KB;
  const int n0 = (int)blockIdx.x * kRows;
  const int rows = min(kRows, N - n0);  // a multiple of 8
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const uint8_t* w_sm = smem + L.w;
  const uint16_t* s16 = reinterpret_cast<const uint16_t*>(smem + L.s16);
  const uint16_t* o16 = s16 + (size_t)kRows * G;
  double2* so_sm = reinterpret_cast<double2*>(smem + L.so);
  int8_t* xq_sm = reinterpret_cast<int8_t*>(smem + L.xq);
  double* xs_sm = reinterpret_cast<double*>(smem + L.xs);
  unsigned int* amx_sm = reinterpret_cast<unsigned int*>(smem + L.amx);
  float* bias_sm = reinterpret_cast<float*>(smem + L.bias);
  const uint32_t bars = smem_u32(smem + L.bars);
  const uint32_t sbar = bars + 8u * kWarps;

  // ---- before the dependency wait: weights, scales / offsets, bias
  if (threadIdx.x == 0) {
    for (int i = 0; i <= kWarps; ++i) mbar_init(bars + 8u * i, 1);
    fence_mbar_init();
    if (!kDump) {
      mbar_arrive_expect_tx(sbar, (uint32_t)(2 * rows * G * 2));
      bulk_load(smem_u32(smem + L.s16), wscale + (size_t)n0 * G, (uint32_t)(rows * G * 2), sbar);
      bulk_load(smem_u32(smem + L.s16) + (uint32_t)(kRows * G * 2), woffset + (size_t)n0 * G,
                (uint32_t)(rows * G * 2), sbar);
    }
    for (int w = 0; w < kWarps; ++w) {
      const int r0 = w * kRowsPerWarp;
      const int nr = min(kRowsPerWarp, rows - r0);
      if (nr <= 0) break;
      mbar_arrive_expect_tx(bars + 8u * w, (uint32_t)(nr * KB));
      bulk_load(smem_u32(smem + L.w) + (uint32_t)(r0 * KB), Wp + (size_t)(n0 + r0) * KB,
                (uint32_t)(nr * KB), bars + 8u * w);
    }
  }
  if (!kDump && threadIdx.x < kRows)
    bias_sm[threadIdx.x] =
        (bias != nullptr && (int)threadIdx.x < rows) ? __ldg(bias + n0 + threadIdx.x) : 0.0f;
  if (early_trigger) pdl_launch_dependents();
  __syncthreads();  // barriers initialized
  if (!kDump && mbar_wait(sbar, 0, err)) {
    for (int i = threadIdx.x; i < rows * G; i += kThreads)
      so_sm[i] = make_double2(h2d(s16[i]), h2d(o16[i]));
  }

  // ---- activations (they come from the previous kernel).  Lane l owns chunks
  // c = l + 32 j, i.e. codes 32 c .. 32 c + 31, of group 16 j + l / 2, and
  // keeps their codes in registers.  Quantized activations are read by every
  // warp straight from global memory (no warp waits on another); bf16 x is
  // quantized by the whole CTA (one absmax) through shared memory.
  pdl_wait();
  if (!early_trigger) pdl_launch_dependents();
  uint32_t xr[NJ][8];  // codes, even / odd permuted per 8 (the nibble-split order)
  double xsj[NJ];      // xsum of the lane's group of chunk j
  float sxv = 1.0f;
  if constexpr (kQuantX) {
    // cooperative: every thread quantizes two 16-byte chunks of x (absmax by a
    // block reduction), the codes go to shared memory in the even / odd order,
    // then each lane picks up its own
    const int nch = K >> 3;
    const uint4* src = reinterpret_cast<const uint4*>(x);
    uint4 v[2];
    uint32_t mb = 0u;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int c = threadIdx.x + kThreads * i;
      v[i] = c < nch ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
      mb = bf16x2_absmax_bits(mb, v[i].x);
      mb = bf16x2_absmax_bits(mb, v[i].y);
      mb = bf16x2_absmax_bits(mb, v[i].z);
      mb = bf16x2_absmax_bits(mb, v[i].w);
    }
    const unsigned wmax = __reduce_max_sync(0xFFFFFFFFu, max(mb & 0xFFFFu, mb >> 16));
    if (lane == 0) amx_sm[warp] = wmax;
    __syncthreads();
    unsigned amax_bits = amx_sm[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) amax_bits = max(amax_bits, amx_sm[w]);
    const float amax = __uint_as_float(amax_bits << 16);
    const float r = act_multiplier(amax);
    sxv = act_scale(amax);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      if (kThreads * i >= nch) break;  // block-uniform
      const int c = threadIdx.x + kThreads * i;
      int sum = 0;
      if (c < nch) {
        const uint2 qc = quant_chunk(v[i], r, &sum);
        *reinterpret_cast<uint2*>(xq_sm + 8 * c) = even_odd(qc.x, qc.y);
      }
      // the 8 chunks of a group sit in 8 consecutive lanes (nch % 8 == 0)
      sum = group8_sum(sum);
      if ((lane & 7) == 0 && c < nch) xs_sm[c >> 3] = i32_to_f64(sum);
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const uint4* p = reinterpret_cast<const uint4*>(xq_sm + 32 * (lane + 32 * j));
      const uint4 a = p[0], b = p[1];
      xr[j][0] = a.x; xr[j][1] = a.y; xr[j][2] = a.z; xr[j][3] = a.w;
      xr[j][4] = b.x; xr[j][5] = b.y; xr[j][6] = b.z; xr[j][7] = b.w;
      xsj[j] = xs_sm[16 * j + (lane >> 1)];
    }
  } else {
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const uint4* p = reinterpret_cast<const uint4*>(xq) + 2 * (lane + 32 * j);
      const uint4 a = __ldg(p), b = __ldg(p + 1);
      const uint2 e0 = even_odd(a.x, a.y), e1 = even_odd(a.z, a.w);
      const uint2 e2 = even_odd(b.x, b.y), e3 = even_odd(b.z, b.w);
      xr[j][0] = e0.x; xr[j][1] = e0.y; xr[j][2] = e1.x; xr[j][3] = e1.y;
      xr[j][4] = e2.x; xr[j][5] = e2.y; xr[j][6] = e3.x; xr[j][7] = e3.y;
      xsj[j] = kDump ? 0.0 : i32_to_f64(__ldg(xsum + 16 * j + (lane >> 1)));
    }
    if (!kDump) sxv = __ldg(sx);
  }

  // A warp's four rows are all valid or all past N (rows is a multiple of 8),
  // so they run as one straight-line block and their chains interleave.
  const int r0 = warp * kRowsPerWarp;
  if (r0 < rows) {
    mbar_wait(bars + 8u * warp, 0, err);  // this warp's rows landed
    const bool odd = (lane & 1) != 0;
    double f[kRowsPerWarp];
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
      const int r = r0 + rr;
      const uint8_t* wrow = w_sm + (size_t)r * KB;
      f[rr] = 0.0;
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const uint4 wv = *reinterpret_cast<const uint4*>(wrow + 16 * (lane + 32 * j));
        int acc = dot8(wv.x, xr[j][0], xr[j][1], 0);
        acc = dot8(wv.y, xr[j][2], xr[j][3], acc);
        acc = dot8(wv.z, xr[j][4], xr[j][5], acc);
        acc = dot8(wv.w, xr[j][6], xr[j][7], acc);
        const int accg = acc + __shfl_xor_sync(0xFFFFFFFFu, acc, 1);  // both halves of the group
        const int g = 16 * j + (lane >> 1);
        if constexpr (kDump) {
          if (!odd) acc_out[(size_t)(n0 + r) * G + g] = accg;
        } else {
          // even lanes the scale term, odd lanes the offset term of group g
          const double2 so = so_sm[r * G + g];
          f[rr] = fma(odd ? so.y : so.x, odd ? xsj[j] : i32_to_f64(accg), f[rr]);
        }
      }
    }
    if constexpr (!kDump) {
      // fixed-order butterflies, the four rows interleaved
#pragma unroll
      for (int o = 1; o < 32; o <<= 1)
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; ++rr) f[rr] += __shfl_xor_sync(0xFFFFFFFFu, f[rr], o);
      if (lane < kRowsPerWarp) {
        double fr = f[0];
#pragma unroll
        for (int rr = 1; rr < kRowsPerWarp; ++rr) fr = lane == rr ? f[rr] : fr;
        y[n0 + r0 + lane] = f64_to_bf16_bits(fma((double)sxv, fr, (double)bias_sm[r0 + lane]));
      }
    }
  }
}

bool g_attr_set[2][2][4][64];

}  // namespace

bool gemv1_fits(int64_t M, int64_t K, int64_t N) {
  return M == 1 && K % 1024 == 0 && K >= 1024 && K <= 4096 && N >= 8 &&
         Gemv1Layout((int)K).total <= (size_t)kSmemTwoPerSm;
}

cudaError_t launch_w4a8_gemv1(const uint16_t* x, const int8_t* xq, const float* sx,
                              const int32_t* xsum, int64_t K, const uint8_t* Wp,
                              const uint16_t* ws, const uint16_t* wo, const float* bias, int64_t N,
                              uint16_t* y, int32_t* acc_out, bool pdl, cudaStream_t s) {
  if (!gemv1_fits(1, K, N)) return cudaErrorInvalidValue;
  const bool qx = x != nullptr, dump = acc_out != nullptr;
  if (qx && dump) return cudaErrorInvalidValue;
  const int nj = (int)(K / 1024);
  using Kern = decltype(&w4a8_gemv1_kernel<false, false, 1>);
  auto pick = [&](auto q, auto d) -> Kern {
    constexpr bool Q = decltype(q)::value, D = decltype(d)::value;
    return nj == 1 ? w4a8_gemv1_kernel<Q, D, 1>
         : nj == 2 ? w4a8_gemv1_kernel<Q, D, 2>
         : nj == 3 ? w4a8_gemv1_kernel<Q, D, 3>
                   : w4a8_gemv1_kernel<Q, D, 4>;
  };
  const Kern kernel = qx ? pick(std::true_type{}, std::false_type{})
                    : dump ? pick(std::false_type{}, std::true_type{})
                           : pick(std::false_type{}, std::false_type{});
  const size_t smem = Gemv1Layout((int)K).total;
  int dev = 0;
  cudaGetDevice(&dev);
  bool& done = g_attr_set[qx][dump][nj - 1][dev < 64 ? dev : 0];
  if (dev >= 64 || !done) {
    cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (dev < 64) done = true;
  }
  int* err = device_error_word();
  if (err == nullptr) return cudaErrorUnknown;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((N + kRows - 1) / kRows));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, x, xq, sx, xsum, (int)K, Wp, ws, wo, bias, (int)N, y,
                            acc_out, 0, err);
}

}  // namespace qk
