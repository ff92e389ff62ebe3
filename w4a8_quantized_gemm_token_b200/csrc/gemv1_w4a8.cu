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
//    and the CTA's fp16 scales / offsets into shared memory, the scales become
//    an fp64 {s, o} table, every warp waits for its rows and the activations
//    are prefetched into L2 -- all off the critical path;
//  * after the wait the CTA stages the activation codes in shared memory
//    (quantizing bf16 x with the rule of the stand-alone kernel, or permuting
//    xq), one block barrier, and lane l picks up the codes of the 16-byte
//    packed chunks l, l + 32, l + 64, ... of a row (one 512-byte, conflict-free
//    shared load per chunk index for the warp) with the sum of those 32 codes;
//  * the low nibbles (even k) and the masked high nibbles (odd k, 16 times
//    too large, one exact shift) feed dp4a against codes permuted the same
//    way, and each lane folds s * acc + o * (its code sum) for its half-group
//    in fp64;
//  * a fixed-order reduction over the warp (two row-halving steps, then a
//    butterfly) gives the four rows, each rounded once and stored -- no
//    shared-memory reduction, no block barrier at the end.
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
    xq = off;   off += (size_t)K;                    // codes, even / odd permuted per 8
    xs = off;   off += (size_t)(K / 32) * 8;         // half-group sums of the codes in fp64
    amx = off;  off += kWarps * 4;                   // per-warp absmax (in-kernel quantization)
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

// The activation rule on 8 bf16 values (one 16-byte chunk), codes returned in
// the even / odd order of `even_odd`: q = rint(fl(v * r)) with ties to even.
// Adding 1.5 * 2^23 to the rounded product leaves rint(product) in the low
// bits (the sum lies in [2^23, 2^24), where the fp32 spacing is 1, and rounds
// to nearest-even); the product is rounded first, as the rule says, because
// the multiply and the add are separate roundings (no contraction).  No clamp
// is needed: with a finite absmax, |v| <= absmax makes |fl(v * r)| < 127.5.
// (A row holding an inf or a NaN takes the general conversion instead.)
__device__ __forceinline__ uint32_t rint_bits(float v, float r) {
  return __float_as_uint(__fadd_rn(__fmul_rn(v, r), 12582912.0f));
}
__device__ __forceinline__ uint32_t pack4_low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}
__device__ __forceinline__ uint2 quant_chunk_even_odd(uint4 c, float r) {
  // bf16 pairs: the low half of each word is the even k, the high half the odd
  const uint32_t e0 = rint_bits(__uint_as_float(c.x << 16), r);
  const uint32_t e1 = rint_bits(__uint_as_float(c.y << 16), r);
  const uint32_t e2 = rint_bits(__uint_as_float(c.z << 16), r);
  const uint32_t e3 = rint_bits(__uint_as_float(c.w << 16), r);
  const uint32_t o0 = rint_bits(__uint_as_float(c.x & 0xFFFF0000u), r);
  const uint32_t o1 = rint_bits(__uint_as_float(c.y & 0xFFFF0000u), r);
  const uint32_t o2 = rint_bits(__uint_as_float(c.z & 0xFFFF0000u), r);
  const uint32_t o3 = rint_bits(__uint_as_float(c.w & 0xFFFF0000u), r);
  return make_uint2(pack4_low_bytes(e0, e1, e2, e3), pack4_low_bytes(o0, o1, o2, o3));
}

// dp4a with unsigned bytes in a and signed bytes in b
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Sum of the 32 codes of one packed 16-byte weight chunk times their
// activation codes.  The low nibbles (even k) go through dp4a as they are; the
// high nibbles (odd k) are only masked, so each byte holds 16 q and their dot
// product is 16 times the wanted one -- exact, removed by one shift at the end.
__device__ __forceinline__ int dot32(uint4 w, const uint32_t (&xe)[8]) {
  int lo = 0, hi = 0;
  lo = __dp4a((int)(w.x & 0x0F0F0F0Fu), (int)xe[0], lo);
  hi = dp4a_us(w.x & 0xF0F0F0F0u, xe[1], hi);
  lo = __dp4a((int)(w.y & 0x0F0F0F0Fu), (int)xe[2], lo);
  hi = dp4a_us(w.y & 0xF0F0F0F0u, xe[3], hi);
  lo = __dp4a((int)(w.z & 0x0F0F0F0Fu), (int)xe[4], lo);
  hi = dp4a_us(w.z & 0xF0F0F0F0u, xe[5], hi);
  lo = __dp4a((int)(w.w & 0x0F0F0F0Fu), (int)xe[6], lo);
  hi = dp4a_us(w.w & 0xF0F0F0F0u, xe[7], hi);
  return lo + (hi >> 4);
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

  // ---- before the dependency wait: weights, scales / offsets, bias, and an
  // L2 prefetch of the activations (a hint only: the loads that use them come
  // after the wait, and L2 is coherent for every SM)
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
    if constexpr (kQuantX) bulk_prefetch_l2(x, (uint32_t)K * 2u);
    else bulk_prefetch_l2(xq, (uint32_t)K);
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
  __syncthreads();  // the {s, o} table is complete (read by every warp)
  // A warp's four rows are all valid or all past N (rows is a multiple of 8).
  // Its rows have landed long before the previous kernel releases this one,
  // so the wait costs nothing there and none is left after the release.
  const int r0 = warp * kRowsPerWarp;
  if (r0 < rows) mbar_wait(bars + 8u * warp, 0, err);

  // ---- activations (they come from the previous kernel).  The CTA stages
  // the codes in shared memory (quantizing bf16 x with one absmax, or
  // permuting xq) with the sum of every 32 codes; then lane l picks up the
  // codes of its 16-byte packed chunks c = l + 32 j, i.e. codes 32 c .. 32 c +
  // 31 (half of group c / 2), into registers with the sum of those codes as a
  // double (the offset term of each half-group is folded by its own lane).
  pdl_wait();
  if (!early_trigger) pdl_launch_dependents();
  uint32_t xr[NJ][8];  // codes, even / odd permuted per 8 (the nibble-split order)
  double xh[NJ];       // sum of the lane's 32 codes of chunk j
  float sxv = 1.0f;
  if constexpr (kQuantX) {
    // cooperative: every thread quantizes 16-byte chunks of x (absmax by a
    // block reduction), the codes go to shared memory in the even / odd order,
    // then each lane picks up its own
    constexpr int kPer = (128 * NJ + kThreads - 1) / kThreads;  // 8-value chunks per thread
    const int nch = K >> 3;
    const uint4* src = reinterpret_cast<const uint4*>(x);
    uint4 v[kPer];
    uint32_t mb = 0u;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
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
    const bool finite = amax_bits < 0x7F80u;  // block-uniform
    sxv = act_scale(amax);
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
      if (kThreads * i >= nch) break;  // block-uniform
      const int c = threadIdx.x + kThreads * i;
      int sum = 0;
      if (c < nch) {
        uint2 qc;
        if (finite) {
          qc = quant_chunk_even_odd(v[i], r);
          sum = __dp4a((int)qc.x, 0x01010101, __dp4a((int)qc.y, 0x01010101, 0));
        } else {  // an inf or NaN in the row: the general conversion
          const uint2 qn = quant_chunk(v[i], r, &sum);
          qc = even_odd(qn.x, qn.y);
        }
        *reinterpret_cast<uint2*>(xq_sm + 8 * c) = qc;
      }
      // the 4 chunks of a 32-code half-group sit in 4 consecutive lanes
      sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 1);
      sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 2);
      if ((lane & 3) == 0 && c < nch) xs_sm[c >> 2] = (double)sum;
    }
  } else {
    // cooperative: every thread permutes one 16-byte piece of xq into shared
    // memory and sums its codes; the two pieces of a half-group are in
    // consecutive lanes
    const int nc = K >> 4;  // <= kThreads
    const int c = threadIdx.x;
    if (!kDump) sxv = __ldg(sx);
    const uint4 a = c < nc ? __ldg(reinterpret_cast<const uint4*>(xq) + c) : make_uint4(0u, 0u, 0u, 0u);
    const uint2 e0 = even_odd(a.x, a.y), e1 = even_odd(a.z, a.w);
    if (c < nc) *reinterpret_cast<uint4*>(xq_sm + 16 * c) = make_uint4(e0.x, e0.y, e1.x, e1.y);
    if constexpr (!kDump) {
      int hs = __dp4a((int)a.x, 0x01010101, __dp4a((int)a.y, 0x01010101, 0));
      hs = __dp4a((int)a.z, 0x01010101, __dp4a((int)a.w, 0x01010101, hs));
      hs += __shfl_xor_sync(0xFFFFFFFFu, hs, 1);
      if ((lane & 1) == 0 && c < nc) xs_sm[c >> 1] = (double)hs;
    }
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const uint4* p = reinterpret_cast<const uint4*>(xq_sm + 32 * (lane + 32 * j));
    const uint4 a = p[0], b = p[1];
    xr[j][0] = a.x; xr[j][1] = a.y; xr[j][2] = a.z; xr[j][3] = a.w;
    xr[j][4] = b.x; xr[j][5] = b.y; xr[j][6] = b.z; xr[j][7] = b.w;
    xh[j] = kDump ? 0.0 : xs_sm[lane + 32 * j];
  }

  // The four rows run as one straight-line block and their chains interleave.
  if (r0 < rows) {
    double f[kRowsPerWarp];
#pragma unroll
    for (int rr = 0; rr < kRowsPerWarp; ++rr) {
      const int r = r0 + rr;
      const uint8_t* wrow = w_sm + (size_t)r * KB;
      f[rr] = 0.0;
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const uint4 wv = *reinterpret_cast<const uint4*>(wrow + 16 * (lane + 32 * j));
        const int acc = dot32(wv, xr[j]);
        if constexpr (kDump) {
          const int accg = acc + __shfl_xor_sync(0xFFFFFFFFu, acc, 1);  // both halves of the group
          if ((lane & 1) == 0) acc_out[(size_t)(n0 + r) * G + 16 * j + (lane >> 1)] = accg;
        } else {
          // each lane folds its half-group: s * acc + o * (sum of its codes)
          const double2 so = so_sm[r * G + 16 * j + (lane >> 1)];
          f[rr] = fma(so.x, i32_to_f64(acc), f[rr]);
          f[rr] = fma(so.y, xh[j], f[rr]);
        }
      }
    }
    if constexpr (!kDump) {
      // fixed-order reduction of the four rows over the warp: halve the rows
      // held per lane at the first two steps, then a butterfly; lane 8 q ends
      // with row q
      const bool up16 = (lane & 16) != 0, up8 = (lane & 8) != 0;
      double a0 = up16 ? f[2] : f[0], a1 = up16 ? f[3] : f[1];
      const double b0 = up16 ? f[0] : f[2], b1 = up16 ? f[1] : f[3];
      a0 += __shfl_xor_sync(0xFFFFFFFFu, b0, 16);
      a1 += __shfl_xor_sync(0xFFFFFFFFu, b1, 16);
      double c = up8 ? a1 : a0;
      c += __shfl_xor_sync(0xFFFFFFFFu, up8 ? a0 : a1, 8);
      c += __shfl_xor_sync(0xFFFFFFFFu, c, 4);
      c += __shfl_xor_sync(0xFFFFFFFFu, c, 2);
      c += __shfl_xor_sync(0xFFFFFFFFu, c, 1);
      if ((lane & 7) == 0) {
        const int rr = lane >> 3;
        y[n0 + r0 + rr] = f64_to_bf16_bits(fma((double)sxv, c, (double)bias_sm[r0 + rr]));
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
