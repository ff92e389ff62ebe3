// act_quant.cuh -- the per-token int8 activation quantization rule, shared by
// the stand-alone quantization kernel and the small-M W4A8 kernel that
// quantizes its activations itself ("qlip-mlx" README, "w8a8_linear /
// W8A8Linear": activations quantized dynamically inside the op).
//
// Rounding: the scale is absmax / 127 and the multiplier 127 / absmax, both
// correctly rounded fp32 divisions; each code is round-half-even of the fp32
// product x * multiplier (no fused multiply-add), clamped to [-127, 127]; an
// all-zero row gets scale 1 and codes 0.
#pragma once

#include <cstdint>

namespace qk {

__device__ __forceinline__ uint32_t bf16x2_absmax_bits(uint32_t acc, uint32_t w) {
  // |bf16| bit patterns order like the values they encode, so a 16-bit integer
  // max of the magnitudes is the absmax.
  return __vmaxu2(acc, w & 0x7FFF7FFFu);
}

__device__ __forceinline__ int quant1(float v, float r) {
  int q = __float2int_rn(__fmul_rn(v, r));
  return max(-127, min(127, q));
}

// 8 bf16 (one 16-byte chunk) -> 8 int8 codes packed in a uint2; adds the codes
// to *sum.
__device__ __forceinline__ uint2 quant_chunk(uint4 c, float r, int* sum) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  uint32_t out[2];
  int s = 0;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t packed = 0;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint32_t u = w[2 * h + j];
      const int q0 = quant1(__uint_as_float(u << 16), r);
      const int q1 = quant1(__uint_as_float(u & 0xFFFF0000u), r);
      s += q0 + q1;
      packed |= ((uint32_t)(q0 & 0xFF) | ((uint32_t)(q1 & 0xFF) << 8)) << (16 * j);
    }
    out[h] = packed;
  }
  *sum += s;
  return make_uint2(out[0], out[1]);
}

// Warp-wide max of two packed |bf16| bit patterns per lane: the bf16 bits of
// the absmax (as an integer that orders like the value).
__device__ __forceinline__ uint32_t warp_max_bits(uint32_t bits2) {
  uint32_t m = max(bits2 & 0xFFFFu, bits2 >> 16);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  return m;
}

__device__ __forceinline__ float warp_max_bits_to_float(uint32_t bits2) {
  return __uint_as_float(warp_max_bits(bits2) << 16);
}

// Sum over the 8 lanes that hold one group of 64 codes.
__device__ __forceinline__ int group8_sum(int v) {
  v += __shfl_xor_sync(0xFFFFFFFFu, v, 1);
  v += __shfl_xor_sync(0xFFFFFFFFu, v, 2);
  v += __shfl_xor_sync(0xFFFFFFFFu, v, 4);
  return v;
}

// Multiplier and scale of a row from its absmax.
__device__ __forceinline__ float act_multiplier(float amax) {
  return (amax == 0.0f) ? 0.0f : __fdiv_rn(127.0f, amax);
}
__device__ __forceinline__ float act_scale(float amax) {
  return (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 127.0f);
}

}  // namespace qk
