// quant.cu -- quantization kernels.
//
//  * quant_act: per-token dynamic symmetric int8 quantization of bf16
//    activations ("qlip-mlx" README, "w8a8_linear / W8A8Linear": activations
//    quantized dynamically inside the op; "MLX PR #4722", "SIMD fix": a kernel
//    of its own quantizes x).  HBM-bound: 2 bytes read and 1 written per
//    element.  One warp owns one row; each lane moves 16-byte chunks (8 bf16),
//    so a warp-wide load covers 512 contiguous bytes.  Rows of up to
//    32 * 8 * NCH elements stay in registers between the absmax and the
//    quantize pass; longer rows are read twice (the second read hits L2).
//  * quant_w8: the same rule per output channel on fp32 weights (offline).
//  * quant_w4: affine group-64 4-bit weights ("qlip-mlx" README,
//    "w4a8_linear / W4A8Linear"; "MLX PR #4722", "Selector rules"), offline.
//
// Rounding (act_quant.cuh): the scale is absmax / 127 and the multiplier
// 127 / absmax, both correctly rounded fp32 divisions; each code is
// round-half-even of the fp32 product x * multiplier, clamped to [-127, 127].
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "act_quant.cuh"
#include "qk_internal.h"
#include "sm100.cuh"

namespace qk {
namespace {

constexpr int kQuantWarps = 8;  // rows per 256-thread block

// NCH > 0: the row (<= 256 * NCH elements) stays in registers.
// NCH == 0: two passes over the row.
template <int NCH>
__global__ void __launch_bounds__(256) quant_act_kernel(const uint16_t* __restrict__ x, int M,
                                                        int K, int8_t* __restrict__ xq,
                                                        float* __restrict__ sx,
                                                        int32_t* __restrict__ xsum) {
  // The dependent GEMM may start its prologue now; it waits for this grid's
  // completion before it reads xq / sx.
  pdl_launch_dependents();
  // When launched as a programmatic dependent, wait for the previous grid (it
  // may produce x, or still read the xq / sx this kernel overwrites).
  pdl_wait();
  const int row = blockIdx.x * kQuantWarps + (threadIdx.x >> 5);
  if (row >= M) return;
  const int lane = threadIdx.x & 31;
  const int nch = K >> 3;  // 16-byte chunks per row
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)row * K);
  uint2* dst = reinterpret_cast<uint2*>(xq + (size_t)row * K);
  const int G = K >> 6;

  uint32_t mb = 0;
  float r;
  if constexpr (NCH > 0) {
    uint4 v[NCH];
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int c = i * 32 + lane;
      if (c < nch) {
        v[i] = __ldcs(src + c);
        mb = bf16x2_absmax_bits(mb, v[i].x);
        mb = bf16x2_absmax_bits(mb, v[i].y);
        mb = bf16x2_absmax_bits(mb, v[i].z);
        mb = bf16x2_absmax_bits(mb, v[i].w);
      }
    }
    const float amax = warp_max_bits_to_float(mb);
    r = act_multiplier(amax);
    if (lane == 0) sx[row] = act_scale(amax);
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int c = i * 32 + lane;
      int s = 0;
      if (c < nch) dst[c] = quant_chunk(v[i], r, &s);
      if (xsum != nullptr && i * 32 < nch) {  // warp-uniform
        s = group8_sum(s);
        if ((lane & 7) == 0 && c < nch) xsum[(size_t)row * G + (c >> 3)] = s;
      }
    }
  } else {
    for (int c = lane; c < nch; c += 32) {
      const uint4 v = __ldg(src + c);
      mb = bf16x2_absmax_bits(mb, v.x);
      mb = bf16x2_absmax_bits(mb, v.y);
      mb = bf16x2_absmax_bits(mb, v.z);
      mb = bf16x2_absmax_bits(mb, v.w);
    }
    const float amax = warp_max_bits_to_float(mb);
    r = act_multiplier(amax);
    if (lane == 0) sx[row] = act_scale(amax);
    for (int base = 0; base < nch; base += 32) {  // warp-uniform trip count
      const int c = base + lane;
      int s = 0;
      if (c < nch) dst[c] = quant_chunk(__ldcs(src + c), r, &s);
      if (xsum != nullptr) {
        s = group8_sum(s);
        if ((lane & 7) == 0 && c < nch) xsum[(size_t)row * G + (c >> 3)] = s;
      }
    }
  }
}

// W8: one warp per output channel, fp32 input, two passes (offline op).
// Long rows: WPR warps share a row (8 / WPR rows per 256-thread block), each
// thread holding CPT 16-byte chunks (chunk c = i * 32 WPR + thread-in-row) in
// registers; the row's absmax is combined across its warps through shared
// memory.  More, lighter warps per SM keep more loads in flight than one warp
// per row holding the whole row.
template <int WPR, int CPT>
__global__ void __launch_bounds__(256) quant_act_split_kernel(const uint16_t* __restrict__ x, int M,
                                                              int K, int8_t* __restrict__ xq,
                                                              float* __restrict__ sx,
                                                              int32_t* __restrict__ xsum) {
  pdl_launch_dependents();
  pdl_wait();
  constexpr int T = 32 * WPR;  // threads per row
  __shared__ uint32_t red[kQuantWarps];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (kQuantWarps / WPR) + warp / WPR;
  const int t = (warp % WPR) * 32 + lane;
  const bool live = row < M;
  const int nch = K >> 3;
  const int G = K >> 6;
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)(live ? row : 0) * K);
  uint2* dst = reinterpret_cast<uint2*>(xq + (size_t)(live ? row : 0) * K);
  uint4 v[CPT];
  uint32_t mb = 0;
#pragma unroll
  for (int i = 0; i < CPT; ++i) {
    const int c = i * T + t;
    if (live && c < nch) {
      v[i] = __ldcs(src + c);
      mb = bf16x2_absmax_bits(mb, v[i].x);
      mb = bf16x2_absmax_bits(mb, v[i].y);
      mb = bf16x2_absmax_bits(mb, v[i].z);
      mb = bf16x2_absmax_bits(mb, v[i].w);
    }
  }
  uint32_t m = warp_max_bits(mb);
  if (lane == 0) red[warp] = m;
  __syncthreads();  // every thread of the block reaches it (no early return above)
#pragma unroll
  for (int w = 0; w < WPR; ++w) m = max(m, red[(warp / WPR) * WPR + w]);
  if (!live) return;
  const float amax = __uint_as_float(m << 16);
  const float r = act_multiplier(amax);
  if (t == 0) sx[row] = act_scale(amax);
#pragma unroll
  for (int i = 0; i < CPT; ++i) {
    const int c = i * T + t;
    int s = 0;
    if (c < nch) dst[c] = quant_chunk(v[i], r, &s);
    if (xsum != nullptr && i * T < nch) {  // warp-uniform
      s = group8_sum(s);
      if ((lane & 7) == 0 && c < nch) xsum[(size_t)row * G + (c >> 3)] = s;
    }
  }
}

__global__ void __launch_bounds__(256) quant_w8_kernel(const float* __restrict__ W, int N, int K,
                                                       int8_t* __restrict__ Wq,
                                                       float* __restrict__ sw) {
  const int row = blockIdx.x * kQuantWarps + (threadIdx.x >> 5);
  if (row >= N) return;
  const int lane = threadIdx.x & 31;
  const float4* src = reinterpret_cast<const float4*>(W + (size_t)row * K);
  uint32_t* dst = reinterpret_cast<uint32_t*>(Wq + (size_t)row * K);
  const int nch = K >> 2;
  float amax = 0.0f;
  for (int c = lane; c < nch; c += 32) {
    const float4 v = __ldg(src + c);
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  const float r = act_multiplier(amax);
  if (lane == 0) sw[row] = act_scale(amax);
  for (int c = lane; c < nch; c += 32) {
    const float4 v = __ldg(src + c);
    const int q0 = quant1(v.x, r), q1 = quant1(v.y, r), q2 = quant1(v.z, r), q3 = quant1(v.w, r);
    dst[c] = (uint32_t)(q0 & 0xFF) | ((uint32_t)(q1 & 0xFF) << 8) | ((uint32_t)(q2 & 0xFF) << 16) |
             ((uint32_t)(q3 & 0xFF) << 24);
  }
}

// W4 affine, group 64: eight lanes per group, eight weights per lane.
__global__ void __launch_bounds__(256) quant_w4_kernel(const float* __restrict__ W, int N, int K,
                                                       uint8_t* __restrict__ Wp,
                                                       uint16_t* __restrict__ wscale,
                                                       uint16_t* __restrict__ woffset) {
  const int G = K >> 6;
  const long long total = (long long)N * G;
  const long long grp = ((long long)blockIdx.x * 256 + threadIdx.x) >> 3;
  const int t = threadIdx.x & 7;
  const bool valid = grp < total;  // whole 8-lane teams are valid or not
  const long long g_safe = valid ? grp : 0;
  const int n = (int)(g_safe / G), g = (int)(g_safe % G);
  const float4* src = reinterpret_cast<const float4*>(W + (size_t)n * K + 64 * g + 8 * t);
  float w[8];
  if (valid) {
    const float4 a = __ldg(src), b = __ldg(src + 1);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = 0.0f;
  }
  float lo = w[0], hi = w[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) {
    lo = fminf(lo, w[i]);
    hi = fmaxf(hi, w[i]);
  }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xFFFFFFFFu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xFFFFFFFFu, hi, o));
  }
  if (!valid) return;
  const __half sh = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 15.0f));
  const __half oh = __float2half_rn(lo);
  const float s = __half2float(sh);
  const float off = __half2float(oh);
  uint32_t packed = 0;
  if (s != 0.0f) {
    const float r = __fdiv_rn(1.0f, s);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      int q = __float2int_rn(__fmul_rn(__fsub_rn(w[i], off), r));
      q = max(0, min(15, q));
      packed |= (uint32_t)q << (4 * i);  // k = 2j low nibble, 2j + 1 high nibble
    }
  }
  reinterpret_cast<uint32_t*>(Wp + (size_t)n * (K / 2) + 32 * g)[t] = packed;
  if (t == 0) {
    wscale[(size_t)n * G + g] = __half_as_ushort(sh);
    woffset[(size_t)n * G + g] = __half_as_ushort(oh);
  }
}

}  // namespace

cudaError_t launch_quant_act(const uint16_t* x, int64_t M, int64_t K, int8_t* xq, float* sx,
                             int32_t* xsum, cudaStream_t s, bool pdl) {
  const int m = (int)M, k = (int)K;
  const int nch = (int)(K / 8);                    // 16-byte chunks per row
  const int per_lane = (nch + 31) / 32;            // ... per lane of one warp
  using Kern = void (*)(const uint16_t*, int, int, int8_t*, float*, int32_t*);
  Kern kernel = nullptr;
  int rows_per_block = kQuantWarps;
  // rows of up to 8 chunks per lane: one warp per row; longer rows: 2, 4 or 8
  // warps per row with at most 8 chunks per thread; beyond 16384 elements,
  // one warp per row reading the row twice
  auto split = [&](int wpr) -> Kern {
    const int cpt = (nch + 32 * wpr - 1) / (32 * wpr);
    rows_per_block = kQuantWarps / wpr;
    switch (wpr * 16 + cpt) {
      case 2 * 16 + 5: return quant_act_split_kernel<2, 5>;
      case 2 * 16 + 6: return quant_act_split_kernel<2, 6>;
      case 2 * 16 + 7: return quant_act_split_kernel<2, 7>;
      case 2 * 16 + 8: return quant_act_split_kernel<2, 8>;
      case 4 * 16 + 5: return quant_act_split_kernel<4, 5>;
      case 4 * 16 + 6: return quant_act_split_kernel<4, 6>;
      case 4 * 16 + 7: return quant_act_split_kernel<4, 7>;
      case 4 * 16 + 8: return quant_act_split_kernel<4, 8>;
      case 8 * 16 + 5: return quant_act_split_kernel<8, 5>;
      case 8 * 16 + 6: return quant_act_split_kernel<8, 6>;
      case 8 * 16 + 7: return quant_act_split_kernel<8, 7>;
      case 8 * 16 + 8: return quant_act_split_kernel<8, 8>;
      default: return nullptr;
    }
  };
  // Few rows (at most one block per SM either way): a whole block per row,
  // so that each thread holds at most four chunks and the call's latency is
  // one round of loads.
  if (M <= 148 && nch >= 128 && nch <= 1024) {
    const int cpt = (nch + 255) / 256;
    kernel = cpt == 1 ? quant_act_split_kernel<8, 1>
           : cpt == 2 ? quant_act_split_kernel<8, 2>
           : cpt == 3 ? quant_act_split_kernel<8, 3> : quant_act_split_kernel<8, 4>;
    rows_per_block = 1;
  } else if (per_lane <= 1)
    kernel = quant_act_kernel<1>;
  else if (per_lane <= 2)
    kernel = quant_act_kernel<2>;
  else if (per_lane <= 4)
    kernel = quant_act_kernel<4>;
  else if (per_lane <= 8)
    kernel = quant_act_kernel<8>;
  else if (per_lane <= 16)
    kernel = split(2);
  else if (per_lane <= 32)
    kernel = split(4);
  else if (per_lane <= 64)
    kernel = split(8);
  if (kernel == nullptr) {
    kernel = quant_act_kernel<0>;
    rows_per_block = kQuantWarps;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((M + rows_per_block - 1) / rows_per_block));
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, x, m, k, xq, sx, xsum);
}

cudaError_t launch_quant_w8(const float* W, int64_t N, int64_t K, int8_t* Wq, float* sw,
                            cudaStream_t s) {
  const dim3 grid((unsigned)((N + kQuantWarps - 1) / kQuantWarps)), block(256);
  quant_w8_kernel<<<grid, block, 0, s>>>(W, (int)N, (int)K, Wq, sw);
  return cudaGetLastError();
}

cudaError_t launch_quant_w4(const float* W, int64_t N, int64_t K, uint8_t* Wp, uint16_t* ws,
                            uint16_t* wo, cudaStream_t s) {
  const long long threads = N * (K / 64) * 8;
  const dim3 grid((unsigned)((threads + 255) / 256)), block(256);
  quant_w4_kernel<<<grid, block, 0, s>>>(W, (int)N, (int)K, Wp, ws, wo);
  return cudaGetLastError();
}

}  // namespace qk
