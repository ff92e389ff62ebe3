// gemm_w4a8_planes.cu -- the W4A8 tensor-core GEMM (M > 16 rows) as int8 GEMMs
// on the bytes of the dequantized weight.
//
// Computes what the per-group fold of gemm_w4a8.cu computes ("qlip-mlx"
// README, "w4a8_linear / W4A8Linear": packed 4-bit weights, the same INT8
// compute; "MLX PR #4722": affine 4-bit weights of group size 64 staged as int8
// for the matmul), with G = K / 64:
//   y[m, n] = bf16( sx[m] * sum_g (s[n,g] * acc[m,n,g] + o[n,g] * xsum[m,g]) + bias[n] ).
//
// The exact reformulation.  A nonzero fp16 value is an odd integer times a
// power of two.  For weight row n let e_n be the smallest such exponent over
// the row's nonzero scales and offsets; then S_g = s[n,g] / 2^e_n and
// O_g = o[n,g] / 2^e_n are integers, every dequantized weight s q + o of the
// row is 2^e_n W with the integer W = S_g q + O_g, and
//   sum_g (s acc + o xsum) = 2^e_n sum_k xq[m,k] W[n,k]            (exactly).
// With c_P = 0x80..80 (P bytes) and U = W + c_P: when every U of the matrix lies
// in [0, 2^(8P)) for some P <= 3 (Gaussian or trained weights need 2, or 3 when
// a row holds a group of unusually small range), W has the signed base-256
// digits d_p = U_p - 128 in [-128, 127] (U_p the bytes of U), W = sum_p 256^p d_p,
// and the integer sum is P int8 GEMMs on those digits:
//   Y[m,n] = sum_p 256^p sum_k xq[m,k] d_p[n,k].
// Each digit GEMM is exact in int32 (|xq| <= 127, |d_p| <= 128, K <= 65536) and Y
// is exact in fp64, so
//   y = bf16( sx[m] 2^e_n Y + bias[n] )
// is the exact value of the fold rounded once (with one fused multiply-add,
// as the fold kernel rounds it).  The per-group fp64 fold is itself exact under
// the same bound on the integers, so both kernels give the same bits.
//
// Kernels (one call of the GEMM route runs them in this order, each a
// programmatic dependent of the one before):
//  * w4a8_plane_count_kernel: one warp per weight row finds e_n (written to
//    the call's scratch) and the bytes its integers need; the launch's P (the
//    maximum, or 255 when some row needs more than 3 bytes or holds a
//    non-finite value) goes into a 64-bit word as (epoch << 8) | P, with the
//    launch's epoch (a value never reused): a word of another epoch is
//    replaced, one of this epoch raised, so the word needs no clearing.  A row
//    that needs three digits also claims one of 8 slots in its block of 60
//    rows (the same epoch-tagged words); a block with more sets an overflow
//    word;
//  * w4a8_plane_build_kernel: memory-bound; writes the digit rows of every
//    weight row to the scratch (one thread per 16 codes: 8 packed bytes in,
//    16-byte stores out): uniform layout, the P digit rows of row n at n P + p;
//    mixed layout (P = 3 without overflow), the two low digit rows of every row
//    at 2 n + p and the top digit of a three-digit row at 2 N + 8 (n / 60) +
//    its slot (2.13 digit rows per weight row on average instead of 3);
//  * (the per-group fold kernel of gemm_w4a8.cu, gated by the same word: it
//    computes only when P > 3);
//  * w4a8_planes_kernel: the W8A8 GEMM's structure on those rows -- CTA pairs
//    (clusters of 2) run tcgen05.mma.cta_group::2 kind::i8 with M = 256 rows of
//    xq and N = 256 digit rows (uniform: 256 / P weight rows, 64 for P = 3;
//    mixed: 120 weight rows, each CTA's half holding its 60 rows' low digits
//    and its 8 top-digit rows), both operands loaded by TMA into a 5-stage
//    ring, one MMA covering every digit row of the tile; two epilogue
//    warpgroups, one per TMEM accumulator (so consecutive tiles drain in
//    parallel), tcgen05.ld the digit sums of 16 outputs at a time and round
//    y = sx 2^e_n Y + bias once to bf16: in fp32 where an error bound proves
//    that v - err and v + err round to the same bf16 value (which is then the
//    exact value's), else Y in int64 and one fp64 fused multiply-add for the
//    pair of outputs; TMA stores that clip the edges write y.
//    The plane GEMM does nothing unless the word holds 1..3 planes of this
//    launch's epoch.
// A prepared weight (qk_w4a8_prepare) runs the count and the build once, into
// caller-owned memory with a fixed epoch after zeroing its words; its products
// then run the gated fold and the plane GEMM only.
// (Building the planes inside the GEMM was measured and not kept: a transform
// split over the pair needs a cluster-scope handoff per stage, about a
// microsecond of release and acquire, and one done by the issuing CTA alone
// runs at a third of the tensor pipe's pace.)
// Every mbarrier wait is bounded (sm100.cuh); no load uses cluster multicast.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "qk_internal.h"
#include "sm100.cuh"

namespace qk {
namespace {

constexpr int BM = 128;                 // rows of xq per CTA (the pair covers 256)
constexpr int BK = 128;                 // K per stage: two groups of 64
constexpr int STAGES = 5;
constexpr int kEpiWarps = 8;            // two warpgroups, one per TMEM accumulator
constexpr int kThreads = 32 * (2 + kEpiWarps);  // 320
constexpr int A_BYTES = BM * BK;        // 16 KiB of xq per stage
constexpr int B_BYTES = 128 * BK;       // 16 KiB: up to 128 plane rows per CTA
constexpr int STG_BYTES = 32 * 128;     // 32 output rows x 64 bf16
constexpr int SMEM_A = 0;
constexpr int SMEM_B = SMEM_A + STAGES * A_BYTES;
constexpr int SMEM_STG = SMEM_B + STAGES * B_BYTES;
// per epilogue warp, the current tile's column constants: {2^e_n, bias} for
// the up to 256 weight rows of a uniform tile, or {2^e_n, bias, top-digit
// offset} for the kMixRows rows of a mixed one (the same 2 KiB)
struct ColInfo {
  float p2;    // 2^e_n
  float bias;
};
struct MixInfo {
  float p2;
  float bias;
  uint32_t exoff;  // byte offset of the row's top-digit sum in a lane's ex row (8: none)
  uint32_t pad;
};
constexpr int COL_BYTES = 256 * (int)sizeof(ColInfo);  // 2 KiB
// per epilogue warp, each lane's top-digit sums of the current mixed half:
// kMixExtra words and a zero, one 9-word row per lane (an odd stride: no bank
// conflicts when every lane reads its own row)
constexpr int kExStride = 9;
constexpr int EX_BYTES = 32 * kExStride * 4;
constexpr int SMEM_COL = SMEM_STG + kEpiWarps * STG_BYTES;
constexpr int SMEM_EX = SMEM_COL + kEpiWarps * COL_BYTES;
constexpr int SMEM_BAR = SMEM_EX + kEpiWarps * EX_BYTES;
constexpr int kNumBars = 2 * STAGES + 4;  // full, empty per stage; tfull, tempty per accumulator
constexpr int SMEM_SLOT = SMEM_BAR + kNumBars * 8;
constexpr int SMEM_USED = SMEM_SLOT + 16;
constexpr int SMEM_ALLOC = SMEM_USED + 1024;
constexpr int kTmemCols = 512;          // two accumulators of up to 256 columns
constexpr int kMaxPlanes = 3;
// Mixed mode (the matrix needs three digits but few rows do): tiles of
// kMixRows weight rows, each CTA's half (kMixHalf rows) holding the two low
// digit planes of its rows (2 kMixHalf plane rows) and the top digit of up to
// kMixExtra of them that need it, 2 kMixHalf + kMixExtra = 128 plane rows.
constexpr int kMixHalf = 60;
constexpr int kMixRows = 2 * kMixHalf;
constexpr int kMixExtra = 8;
constexpr int kMixBox = 40;             // TMA box rows of the two low planes (three per half)
static_assert(2 * kMixHalf + kMixExtra == 128, "mixed half = 128 plane rows");
static_assert((2 * kMixHalf) % kMixBox == 0 && kMixBox % 8 == 0, "whole swizzle atoms per box");

static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
static_assert(SMEM_B % 1024 == 0 && B_BYTES % 1024 == 0, "swizzled operand tiles");
static_assert(SMEM_STG % 1024 == 0, "swizzled output stages");

constexpr int kNoExp = 1 << 20;         // "no nonzero value" in a minimum of exponents

__host__ __device__ constexpr int tile_rows_of(int P) { return P == 3 ? 64 : 256 / P; }

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  return __byte_perm(a, b, sel);
}

// Exponent of the lowest set bit of a nonzero finite fp16 value (its value is
// an odd integer times 2^this), or kNoExp for +-0.
__device__ __forceinline__ int f16_low_exp(uint32_t h) {
  const uint32_t E = (h >> 10) & 31u;
  const uint32_t m = h & 1023u;
  const uint32_t mant = E != 0u ? (m | 1024u) : m;
  if (mant == 0u) return kNoExp;
  return (E != 0u ? (int)E - 25 : -24) + (__ffs((int)mant) - 1);
}

// Left shift that puts the 11-bit significand of fp16 h on the grid 2^eb
// (negative: a right shift of trailing zero bits).
__device__ __forceinline__ int f16_grid_shift(uint32_t h, int eb) {
  const uint32_t E = (h >> 10) & 31u;
  return (E != 0u ? (int)E - 25 : -24) - eb;
}

// fp16 value / 2^eb as an integer (exact when eb <= f16_low_exp(h)); 64-bit so
// that the plane count below sees every value, however far from the grid.
__device__ __forceinline__ long long f16_on_grid64(uint32_t h, int eb) {
  const uint32_t E = (h >> 10) & 31u;
  const uint32_t m = h & 1023u;
  const long long mant = E != 0u ? (long long)(m | 1024u) : (long long)m;
  if (mant == 0) return 0;
  const int sh = (E != 0u ? (int)E - 25 : -24) - eb;
  const long long v = sh >= 0 ? (mant << sh) : (mant >> -sh);
  return (h & 0x8000u) ? -v : v;
}

// Same, as 32 bits (the plane count guarantees the value fits when P <= 4).
__device__ __forceinline__ uint32_t f16_on_grid32(uint32_t h, int eb) {
  const uint32_t E = (h >> 10) & 31u;
  const uint32_t m = h & 1023u;
  const uint32_t mant = E != 0u ? (m | 1024u) : m;
  if (mant == 0u) return 0u;
  const int sh = (E != 0u ? (int)E - 25 : -24) - eb;
  const uint32_t v = sh >= 0 ? (mant << sh) : (mant >> -sh);
  return (h & 0x8000u) ? (0u - v) : v;
}

__host__ __device__ constexpr uint32_t plane_bias(int P) {
  return P == 1 ? 0x80u : P == 2 ? 0x8080u : P == 3 ? 0x808080u : 0x80808080u;
}

// ------------------------------------------------------------ plane count

constexpr int kCountRowsPerBlock = 8;

__global__ void __launch_bounds__(32 * kCountRowsPerBlock)
    w4a8_plane_count_kernel(const uint16_t* __restrict__ wscale,
                            const uint16_t* __restrict__ woffset, int N, int K, int* ebase,
                            int* slot, unsigned long long* hcount, unsigned long long* pword,
                            unsigned long long* oword, unsigned long long epoch) {
  __shared__ int s_p[kCountRowsPerBlock];
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = blockIdx.x * kCountRowsPerBlock + warp;
  const int G = K >> 6;
  int prow = 0;
  if (n < N) {
    const uint16_t* s = wscale + (size_t)n * G;
    const uint16_t* o = woffset + (size_t)n * G;
    int eb = kNoExp;
    bool bad = false;
    for (int g = lane; g < G; g += 32) {
      const uint32_t hs = s[g], ho = o[g];
      bad |= ((hs >> 10) & 31u) == 31u || ((ho >> 10) & 31u) == 31u;
      eb = min(eb, min(f16_low_exp(hs), f16_low_exp(ho)));
    }
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) eb = min(eb, __shfl_xor_sync(0xFFFFFFFFu, eb, d));
    bad = __any_sync(0xFFFFFFFFu, bad);
    if (eb == kNoExp) eb = 0;
    if (lane == 0) ebase[n] = eb;
    long long lo = 0, hi = 0;
    for (int g = lane; g < G && !bad; g += 32) {
      const uint32_t hs = s[g], ho = o[g];
      // 11 significant bits shifted by more than 40 would leave the int64 range
      // of 15 S + O; such a row is far outside the four planes anyway
      if (f16_grid_shift(hs, eb) > 40 || f16_grid_shift(ho, eb) > 40) {
        bad = true;
        break;
      }
      const long long S = f16_on_grid64(hs, eb), O = f16_on_grid64(ho, eb);
      const long long a = O, b = O + 15 * S;
      lo = min(lo, min(a, b));
      hi = max(hi, max(a, b));
    }
    bad = __any_sync(0xFFFFFFFFu, bad);
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) {
      lo = min(lo, (long long)__shfl_xor_sync(0xFFFFFFFFu, lo, d));
      hi = max(hi, (long long)__shfl_xor_sync(0xFFFFFFFFu, hi, d));
    }
    prow = 255;
    if (!bad) {
      for (int p = kMaxPlanes; p >= 1; --p) {
        const long long c = (long long)plane_bias(p);
        if (lo + c >= 0 && hi + c < (1ll << (8 * p))) prow = p;
      }
    }
  }
  if (lane == 0) s_p[warp] = prow;
  __syncthreads();
  // an earlier kernel of the stream may still read the words until the
  // dependency wait returns
  pdl_wait();
  if (n < N && lane == 0) {
    // a row that needs a third digit takes one of its mixed-mode half tile's
    // kMixExtra top-digit slots (counters tagged with the epoch, as the word
    // below); a half tile with more such rows sets the overflow word
    int sl = -1;
    if (prow == 3) {
      unsigned long long* c = hcount + n / kMixHalf;
      unsigned long long old = *reinterpret_cast<volatile unsigned long long*>(c);
      while (true) {
        const bool same = (old >> 8) == epoch;
        const unsigned long long want = same ? old + 1 : ((epoch << 8) | 1ull);
        const unsigned long long prev = atomicCAS(c, old, want);
        if (prev == old) {
          sl = same ? (int)(old & 0xFFull) : 0;
          break;
        }
        old = prev;
      }
      if (sl >= kMixExtra) {
        const unsigned long long want = (epoch << 8) | 1ull;
        unsigned long long o = *reinterpret_cast<volatile unsigned long long*>(oword);
        while (o != want) {
          const unsigned long long prev = atomicCAS(oword, o, want);
          if (prev == o) break;
          o = prev;
        }
      }
    }
    slot[n] = sl;
  }
  if (threadIdx.x == 0) {
    int pmax = 0;
    for (int w = 0; w < kCountRowsPerBlock; ++w) pmax = max(pmax, s_p[w]);
    // The word holds (epoch << 8) | P.  A word of another epoch (an earlier
    // launch, or whatever the scratch held) is replaced, one of this epoch is
    // raised to pmax if below it: a compare-and-swap loop that most blocks
    // leave after one read, since the first block already wrote their P.
    const unsigned long long want = (epoch << 8) | (unsigned long long)pmax;
    unsigned long long old = *reinterpret_cast<volatile unsigned long long*>(pword);
    while (pmax > 0 && ((old >> 8) != epoch || (old & 0xFFull) < (unsigned long long)pmax)) {
      const unsigned long long prev = atomicCAS(pword, old, want);
      if (prev == old) break;
      old = prev;
    }
  }
}

// ------------------------------------------------------------ plane build

constexpr int kBuildThreads = 256;

// 8 packed bytes (16 codes) of one weight row -> the 16 signed digits of each
// of the P planes at the same K offset.  S and Op = O + c_P are the row's integers for
// the codes' group.
template <int P>
__device__ __forceinline__ void planes_of16(const uint2 w2, uint32_t S, uint32_t Op,
                                            uint4 (&out)[P]) {
  const uint32_t w[2] = {w2.x, w2.y};
  uint32_t pl[P][4];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint32_t even = w[i] & 0x0F0F0F0Fu, odd = (w[i] >> 4) & 0x0F0F0F0Fu;
    if constexpr (P == 1) {
      // four codes per word: bytes S q + O + 128, no carries between them
      const uint32_t O4 = Op * 0x01010101u;
      pl[0][2 * i] = S * prmt(even, odd, 0x5140) + O4;      // codes 8i .. 8i + 3
      pl[0][2 * i + 1] = S * prmt(even, odd, 0x7362) + O4;  // codes 8i + 4 .. 8i + 7
    } else if constexpr (P == 2) {
      // two codes per word (16-bit halves): U0 + 2^16 U2 = S (q0 + 2^16 q2) + O (1 + 2^16)
      const uint32_t O2 = Op * 0x00010001u;
      const uint32_t ya = S * prmt(even, 0u, 0x4140) + O2;  // codes 0, 2 of the word
      const uint32_t yb = S * prmt(odd, 0u, 0x4140) + O2;   // codes 1, 3
      const uint32_t yc = S * prmt(even, 0u, 0x4342) + O2;  // codes 4, 6
      const uint32_t yd = S * prmt(odd, 0u, 0x4342) + O2;   // codes 5, 7
      pl[0][2 * i] = prmt(ya, yb, 0x6240);
      pl[1][2 * i] = prmt(ya, yb, 0x7351);
      pl[0][2 * i + 1] = prmt(yc, yd, 0x6240);
      pl[1][2 * i + 1] = prmt(yc, yd, 0x7351);
    } else {
      // one code per word, then a 4 x 4 byte transpose into the planes
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t q4 = h == 0 ? prmt(even, odd, 0x5140) : prmt(even, odd, 0x7362);
        const uint32_t u0 = S * prmt(q4, 0u, 0x4440) + Op;
        const uint32_t u1 = S * prmt(q4, 0u, 0x4441) + Op;
        const uint32_t u2 = S * prmt(q4, 0u, 0x4442) + Op;
        const uint32_t u3 = S * prmt(q4, 0u, 0x4443) + Op;
        const uint32_t a_lo = prmt(u0, u1, 0x5140), a_hi = prmt(u0, u1, 0x7362);
        const uint32_t b_lo = prmt(u2, u3, 0x5140), b_hi = prmt(u2, u3, 0x7362);
        pl[0][2 * i + h] = prmt(a_lo, b_lo, 0x5410);
        pl[1][2 * i + h] = prmt(a_lo, b_lo, 0x7632);
        pl[2][2 * i + h] = prmt(a_hi, b_hi, 0x5410);
      }
    }
  }
#pragma unroll
  // signed digits d_p = U_p - 128: flip the top bit of every byte
  for (int p = 0; p < P; ++p)
    out[p] = make_uint4(pl[p][0] ^ 0x80808080u, pl[p][1] ^ 0x80808080u, pl[p][2] ^ 0x80808080u,
                        pl[p][3] ^ 0x80808080u);
}

// kMixed: the matrix needs three digits; the two low digit planes of every row
// go to rows 2 n + p, the top digit of a row holding a slot to row
// 2 N + kMixExtra (n / kMixHalf) + slot.
template <int P, bool kMixed>
__device__ __forceinline__ void build_rows(const uint8_t* __restrict__ Wp,
                                           const uint16_t* __restrict__ wscale,
                                           const uint16_t* __restrict__ woffset,
                                           const int* __restrict__ ebase,
                                           const int* __restrict__ slot, int N, int K,
                                           uint8_t* __restrict__ planes) {
  const int G = K >> 6;
  const int units_per_row = K >> 4;  // 16 codes each
  const long long total = (long long)N * units_per_row;
  for (long long u = (long long)blockIdx.x * blockDim.x + threadIdx.x; u < total;
       u += (long long)gridDim.x * blockDim.x) {
    const int n = (int)(u / units_per_row);
    const int c = (int)(u - (long long)n * units_per_row);  // codes 16c .. 16c + 15
    const int g = c >> 2;
    const int eb = __ldg(ebase + n);
    const uint32_t S = f16_on_grid32(__ldg(wscale + (size_t)n * G + g), eb);
    const uint32_t Op = f16_on_grid32(__ldg(woffset + (size_t)n * G + g), eb) + plane_bias(P);
    const uint2 w2 = __ldg(reinterpret_cast<const uint2*>(Wp + (size_t)n * (K / 2)) + c);
    uint4 out[P];
    planes_of16<P>(w2, S, Op, out);
    if constexpr (kMixed) {
      __stcg(reinterpret_cast<uint4*>(planes + ((size_t)n * 2) * K) + c, out[0]);
      __stcg(reinterpret_cast<uint4*>(planes + ((size_t)n * 2 + 1) * K) + c, out[1]);
      const int sl = __ldg(slot + n);
      if (sl >= 0)
        __stcg(reinterpret_cast<uint4*>(planes + ((size_t)2 * N + (size_t)kMixExtra * (n / kMixHalf) +
                                                  sl) * K) + c,
               out[2]);
    } else {
#pragma unroll
      for (int p = 0; p < P; ++p)
        __stcg(reinterpret_cast<uint4*>(planes + ((size_t)n * P + p) * K) + c, out[p]);
    }
  }
}

// The launch's plane mode from the plane-count words: 1..3 uniform planes,
// 4 = mixed (three digits needed, every half tile's top digits fit its
// slots), 0 = nothing for the plane kernels (the fold computes).
__device__ __forceinline__ int plane_mode(const unsigned long long* pword,
                                          const unsigned long long* oword,
                                          unsigned long long epoch) {
  const unsigned long long pw = *reinterpret_cast<const volatile unsigned long long*>(pword);
  const unsigned long long ow = *reinterpret_cast<const volatile unsigned long long*>(oword);
  const int P = (pw >> 8) == epoch ? (int)(pw & 0xFFull) : 0;
  const bool over = (ow >> 8) == epoch && (ow & 1ull) != 0;
  if (P == 3) return over ? 3 : 4;
  return (P >= 1 && P <= 2) ? P : 0;
}

__global__ void __launch_bounds__(kBuildThreads)
    w4a8_plane_build_kernel(const uint8_t* __restrict__ Wp, const uint16_t* __restrict__ wscale,
                            const uint16_t* __restrict__ woffset, const int* ebase,
                            const int* slot, int N, int K, uint8_t* planes,
                            const unsigned long long* pword, const unsigned long long* oword,
                            unsigned long long epoch) {
  pdl_launch_dependents();
  pdl_wait();  // e_n, the slots and the plane count come from the kernel before
  switch (plane_mode(pword, oword, epoch)) {
    case 1: build_rows<1, false>(Wp, wscale, woffset, ebase, slot, N, K, planes); break;
    case 2: build_rows<2, false>(Wp, wscale, woffset, ebase, slot, N, K, planes); break;
    case 3: build_rows<3, false>(Wp, wscale, woffset, ebase, slot, N, K, planes); break;
    case 4: build_rows<3, true>(Wp, wscale, woffset, ebase, slot, N, K, planes); break;
    default: break;  // the fold kernel computes the product
  }
}

// -------------------------------------------------------- the plane GEMM

// Raster: groups of group_m M tiles walked down M first (as the W8A8 GEMM).
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

// fp64 -> bf16 bits, one rounding to nearest-even (as in gemm_w8a8.cu).
__device__ __forceinline__ uint32_t f64_to_bf16_bits(double v) {
  const uint32_t hi = (uint32_t)__double2hiint(v);
  const uint32_t lo = (uint32_t)__double2loint(v);
  const uint32_t sign = (hi >> 16) & 0x8000u;
  const uint32_t mag = hi & 0x7FFFFFFFu;
  if (mag < 0x38100000u) {
    if ((mag | lo) == 0u) return sign;
    float f = __double2float_rz(v);
    if ((double)f != v) f = __uint_as_float(__float_as_uint(f) | 1u);
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f));
  }
  const uint32_t keep = mag >> 13;
  const uint32_t low13 = (mag & 0x1FFFu) | min(lo, 1u);
  const uint32_t up = (low13 + 0x0FFFu + (keep & 1u)) >> 13;
  return sign | min(keep + up - (896u << 7), 0x7F80u);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// The fp32 fast path of one output.  With the digit sums A_p converted to
// fp32 (one rounding each) and combined by fused multiply-adds, |yf - Y| is at
// most 3 2^-24 T (1 + 2^-22), where T = sum_p 256^p |A_p| is formed the same way
// (P = 3; fewer roundings for fewer planes); v = fma(sc, yf, bias) with
// sc = sx 2^e_n exact in fp32 (sx a normal value in [2^-100, 2^100], or 0).
// So |v - y| <= 3 2^-24 sc T (1 + 2^-22) + 2^-24 |v| for the exact
// y = sc Y + bias while v is normal, and
//   err = 2^-23 (1 + 2^-16) (1.5 sc T + |v|) + 2^-99
// exceeds |v - y| + 2^-24 (|v| + err), the bound plus the roundings of v - err
// and v + err, through every rounding of its own computation.  The absolute
// term covers a subnormal v, whose rounding error is absolute: the interval
// then straddles a bf16 midpoint whenever |v| is below about 2^-92.
// Round-to-nearest-even to bf16 is monotone, so when v - err and v + err round
// to the same bf16 value, y (and v) round to it too: those are the bits of the
// exact path.  Returns the two roundings (low half: of v - err; high half: of
// v + err).  A NaN v (from a NaN bias) must not reach here, since both halves
// would agree; an infinite v gives a NaN and an infinity, which differ.
__device__ __forceinline__ uint32_t fast_pair(float yf, float T, float sc, float bias) {
  const float v = __fmaf_rn(sc, yf, bias);
  const float err = __fmaf_rn(__fmaf_rn(1.5f * sc, T, fabsf(v)),
                              1.192111085401848e-07f,   // 2^-23 (1 + 2^-16)
                              1.5777218104420236e-30f); // 2^-99
  return pack_bf16x2(v - err, v + err);
}

// Two outputs of the fast path, packed: the bf16 of outputs j (low half) and
// j + 1 (high half), and in `dp` the halves where the two roundings differ.
__device__ __forceinline__ uint32_t pack_pair(uint32_t hl0, uint32_t hl1, uint32_t& dp) {
  const uint32_t lo = __byte_perm(hl0, hl1, 0x5410);  // the roundings of v - err
  dp = lo ^ __byte_perm(hl0, hl1, 0x7632);            // against those of v + err
  return lo;
}

// yf and T of one output from its P digit sums (int32 bit patterns).
template <int P>
__device__ __forceinline__ void digits_to_f32(const uint32_t* a, float& yf, float& T) {
  const float a0 = __int2float_rn((int)a[0]);
  yf = a0;
  T = fabsf(a0);
  if constexpr (P >= 2) {
    const float a1 = __int2float_rn((int)a[1]);
    yf = __fmaf_rn(a1, 256.0f, yf);
    T = __fmaf_rn(fabsf(a1), 256.0f, T);
  }
  if constexpr (P >= 3) {
    const float a2 = __int2float_rn((int)a[2]);
    yf = __fmaf_rn(a2, 65536.0f, yf);
    T = __fmaf_rn(fabsf(a2), 65536.0f, T);
  }
}

// 0xFFFFFFFF (every output of the lane takes the exact path) when sx is
// outside the fast path's range: nonzero below 2^-100, where sx 2^e_n could lose
// bits to fp32 underflow, or above 2^100, where it could overflow.
__device__ __forceinline__ uint32_t sx_force_exact(float sxf) {
  const float a = fabsf(sxf);
  return ((a != 0.0f && a < 7.888609052210118e-31f) || a > 1.2676506002282294e30f) ? 0xFFFFFFFFu
                                                                                     : 0u;
}

// The exact path of one output: Y in fp64 (exact, |Y| < 2^53), one fused
// multiply-add with sx 2^e_n and the bias, one rounding to bf16.
__device__ __forceinline__ uint32_t exact_value(long long Y, double sxd, float p2, float bias) {
  return f64_to_bf16_bits(fma(sxd * (double)p2, __ll2double_rn(Y), (double)bias));
}

// The epilogue of one tile for a fixed P: 16 outputs per TMEM load group,
// 64 outputs per staged 128-byte row and TMA store.  `force` is the lane's
// sx_force_exact, or'ed with all-ones when a column of the tile has a
// non-finite bias.
template <int P>
__device__ __forceinline__ void epilogue_tile(uint32_t t_lane, const ColInfo* col, float sxf,
                                              uint32_t force, uint8_t* stg_ptr, uint32_t stg,
                                              const CUtensorMap* tmY, int ncol0, int row0, int M,
                                              int N, int lane, uint32_t lead_tempty, bool& used) {
  constexpr int TR = tile_rows_of(P);
  constexpr int kChunks = TR / 64;
#pragma unroll 1
  for (int ch = 0; ch < kChunks; ++ch) {
    uint32_t out[32];
#pragma unroll
    for (int sub = 0; sub < 4; ++sub) {
      const int r0 = ch * 64 + sub * 16;  // first weight row of this load group
      uint32_t v[16 * P];
      const uint32_t a = t_lane + (uint32_t)(r0 * P);
      if constexpr (P == 1) {
        uint32_t (&vv)[16] = *reinterpret_cast<uint32_t(*)[16]>(v);
        tmem_ld16(a, vv);
      } else if constexpr (P == 2) {
        uint32_t (&vv)[32] = *reinterpret_cast<uint32_t(*)[32]>(v);
        tmem_ld32(a, vv);
      } else {
#pragma unroll
        for (int j = 0; j < 3; ++j) {
          uint32_t (&vv)[16] = *reinterpret_cast<uint32_t(*)[16]>(v + 16 * j);
          tmem_ld16(a + 16u * j, vv);
        }
      }
      tmem_ld_wait();
      if (ch == kChunks - 1 && sub == 3) {
        // every TMEM read of this accumulator is done: hand it back to the leader
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(lead_tempty);
      }
      uint32_t dp[8];
      uint32_t differs = force;
#pragma unroll
      for (int j = 0; j < 16; j += 2) {
        uint32_t hl[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const ColInfo ci = col[r0 + j + h];  // the same for every lane
          float yf, T;
          digits_to_f32<P>(v + (j + h) * P, yf, T);
          hl[h] = fast_pair(yf, T, sxf * ci.p2, ci.bias);
        }
        out[sub * 8 + (j >> 1)] = pack_pair(hl[0], hl[1], dp[j >> 1]);
        differs |= dp[j >> 1];
      }
      if (__any_sync(0xFFFFFFFFu, differs != 0u)) {
        // the exact path, for each pair of outputs that some lane needs it for
        const double sxd = (double)sxf;
#pragma unroll
        for (int j = 0; j < 16; j += 2) {
          if (__any_sync(0xFFFFFFFFu, (dp[j >> 1] | force) != 0u)) {
            uint32_t hb[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              long long y = (long long)(int)v[(j + h) * P + P - 1];
#pragma unroll
              for (int p = P - 2; p >= 0; --p) y = y * 256 + (long long)(int)v[(j + h) * P + p];
              const volatile ColInfo* cv = col + r0 + j + h;  // not merged with the fast path's reads
              hb[h] = exact_value(y, sxd, cv->p2, cv->bias);
            }
            out[sub * 8 + (j >> 1)] = hb[0] | (hb[1] << 16);
          }
        }
      }
    }
    const int n0 = ncol0 + ch * 64;
    if (n0 >= N || row0 >= M) continue;  // whole box outside y
    if (lane == 0 && used) bulk_wait_read<0>();
    __syncwarp();
    uint8_t* rowp = stg_ptr + lane * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4)) =
          make_uint4(out[4 * j], out[4 * j + 1], out[4 * j + 2], out[4 * j + 3]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tmY, stg, n0, row0);
      bulk_commit();
    }
    used = true;
  }
}

// The epilogue of one mixed-mode tile (kMixRows weight rows): per half h, the
// two low digit sums of row lr in columns h 128 + 2 lr + {0, 1} and the top
// digit sums of the half's slots in columns h 128 + 2 kMixHalf + slot, which
// each lane parks in its row of `ex` so that a row's top digit is one shared
// load at the offset its column entry holds.  The kMixRows outputs of the
// thread's row are assembled in registers and written as a 64-column TMA box
// (once its outputs are final) and a 56-column one.
__device__ __forceinline__ void epilogue_mixed(uint32_t t_lane, const MixInfo* col, float sxf,
                                               uint32_t force, uint8_t* ex_ptr, uint8_t* stg_ptr,
                                               uint32_t stg, const CUtensorMap* tmY,
                                               const CUtensorMap* tmY56, int ncol0, int row0,
                                               int M, int N, int lane, uint32_t lead_tempty,
                                               bool& used) {
  uint32_t out[kMixRows / 2];
  uint8_t* exrow = ex_ptr + lane * (kExStride * 4);
  // box 0 holds outputs 0..63, box 1 outputs 64..119 (56 columns, 112 bytes)
  auto store_box = [&](int ch) {
    const int n0 = ncol0 + 64 * ch;
    if (n0 >= N || row0 >= M) return;  // whole box outside y
    if (lane == 0 && used) bulk_wait_read<0>();
    __syncwarp();
    uint8_t* rowp = stg_ptr + lane * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (ch == 1 && j == 7) break;
      *reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4)) =
          make_uint4(out[32 * ch + 4 * j], out[32 * ch + 4 * j + 1], out[32 * ch + 4 * j + 2],
                     out[32 * ch + 4 * j + 3]);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(ch == 0 ? tmY : tmY56, stg, n0, row0);
      bulk_commit();
    }
    used = true;
  };
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t hb = t_lane + (uint32_t)(h * 128);
    {
      uint32_t ex[8];
      tmem_ld8(hb + 2 * kMixHalf, ex);  // the half's top-digit sums
      tmem_ld_wait();
      // (each lane reads only its own row: no synchronisation between lanes)
#pragma unroll
      for (int k = 0; k < 8; ++k) reinterpret_cast<uint32_t*>(exrow)[k] = ex[k];
      reinterpret_cast<uint32_t*>(exrow)[8] = 0u;
    }
#pragma unroll
    for (int sub = 0; sub < 4; ++sub) {
      constexpr int kSub[4] = {16, 16, 16, kMixHalf - 48};
      const int lr0 = 16 * sub;
      const int cnt = kSub[sub];
      uint32_t v[32];
      if (sub < 3) {
        tmem_ld32(hb + (uint32_t)(2 * lr0), v);
      } else {
        uint32_t (&v16)[16] = *reinterpret_cast<uint32_t(*)[16]>(v);
        uint32_t (&v8)[8] = *reinterpret_cast<uint32_t(*)[8]>(v + 16);
        tmem_ld16(hb + (uint32_t)(2 * lr0), v16);
        tmem_ld8(hb + (uint32_t)(2 * lr0 + 16), v8);
      }
      tmem_ld_wait();
      if (h == 1 && sub == 3) {
        // every TMEM read of this accumulator is done: hand it back to the leader
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(lead_tempty);
      }
      uint32_t dp[8];
      uint32_t differs = force;
#pragma unroll
      for (int j = 0; j < 16; j += 2) {
        if (j < cnt) {
          uint32_t hl[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const MixInfo ci = col[h * kMixHalf + lr0 + j + e];  // the same for every lane
            uint32_t d[3] = {v[2 * (j + e)], v[2 * (j + e) + 1],
                             *reinterpret_cast<const uint32_t*>(exrow + ci.exoff)};
            float yf, T;
            digits_to_f32<3>(d, yf, T);
            hl[e] = fast_pair(yf, T, sxf * ci.p2, ci.bias);
          }
          out[(h * kMixHalf + lr0 + j) >> 1] = pack_pair(hl[0], hl[1], dp[j >> 1]);
          differs |= dp[j >> 1];
        }
      }
      if (__any_sync(0xFFFFFFFFu, differs != 0u)) {
        // the exact path, for each pair of outputs that some lane needs it for
        const double sxd = (double)sxf;
#pragma unroll
        for (int j = 0; j < 16; j += 2) {
          if (j < cnt && __any_sync(0xFFFFFFFFu, (dp[j >> 1] | force) != 0u)) {
            uint32_t hv[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const volatile MixInfo* cv = col + h * kMixHalf + lr0 + j + e;
              const long long top =
                  (long long)*reinterpret_cast<const volatile int*>(exrow + cv->exoff);
              const long long y = (top * 256 + (long long)(int)v[2 * (j + e) + 1]) * 256 +
                                  (long long)(int)v[2 * (j + e)];
              hv[e] = exact_value(y, sxd, cv->p2, cv->bias);
            }
            out[(h * kMixHalf + lr0 + j) >> 1] = hv[0] | (hv[1] << 16);
          }
        }
      }
      if (h == 1 && sub == 0) store_box(0);  // outputs 0..63 are final: free their registers
    }
  }
  store_box(1);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    w4a8_planes_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmB40, const __grid_constant__ CUtensorMap tmB8,
                       const __grid_constant__ CUtensorMap tmY,
                       const __grid_constant__ CUtensorMap tmY56, const float* __restrict__ sx,
                       const int* __restrict__ ebase, const int* __restrict__ slot,
                       const float* __restrict__ bias, int M, int N, int K, int group_m,
                       const unsigned long long* pword, const unsigned long long* oword,
                       unsigned long long epoch, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem<1024>(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + SMEM_BAR;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SMEM_SLOT);

  const uint32_t rank = cluster_ctarank();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int pair = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmB40);
    prefetch_tmap(&tmB8);
    prefetch_tmap(&tmY);
    prefetch_tmap(&tmY56);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 2 * (kEpiWarps / 2));  // one warpgroup in each CTA
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  pdl_launch_dependents();
  pdl_wait();  // xq, sx, e_n, the planes and the plane-count word come from earlier kernels

  const int mode = plane_mode(pword, oword, epoch);
  if (mode != 0) {
    const bool mixed = mode == 4;
    const int P = mixed ? 3 : mode;        // digits per weight
    const int TR = mixed ? kMixRows : tile_rows_of(P);
    const int RC = TR / 2;                 // weight rows of each CTA's half
    const int nplane = mixed ? 128 : P * RC;  // plane rows of each CTA's half
    const int tiles_m = (M + 2 * BM - 1) / (2 * BM);
    const int tiles_n = (N + TR - 1) / TR;
    const int num_tiles = tiles_m * tiles_n;
    const int num_kb = (K + BK - 1) / BK;

    if (warp == 0) {
      // ---------------------------------------------------------- producer
      // each CTA loads its 128 rows of xq and its P RC plane rows (32-row
      // boxes), completing on the leader's barrier
      if (lane == 0) {
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        const uint32_t tx = 2u * (uint32_t)(A_BYTES + nplane * BK);
        for (int t = pair; t < num_tiles && ok; t += num_pairs) {
          int mb, nb;
          tile_coords(t, tiles_m, tiles_n, group_m, mb, nb);
          const int arow = mb * 2 * BM + (int)rank * BM;
          // uniform: rows (nb TR + rank RC) P ..; mixed: the two low planes of
          // the half's rows and its kMixExtra top-digit rows after the 2 N
          const int brow = mixed ? (nb * TR + (int)rank * RC) * 2 : (nb * TR + (int)rank * RC) * P;
          const int xrow = 2 * N + kMixExtra * (2 * nb + (int)rank);
          for (int kb = 0; kb < num_kb; ++kb) {
            if (!mbar_wait(empty_bar(stage), phase ^ 1u, err)) {
              ok = false;
              break;
            }
            if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), tx);
            const uint32_t lead_full = mapa_shared(full_bar(stage), 0);
            tma_load_2d_pair(sbase + SMEM_A + stage * A_BYTES, &tmA, kb * BK, arow, lead_full);
            if (mixed) {
              for (int i = 0; i < 2 * kMixHalf / kMixBox; ++i)
                tma_load_2d_pair(sbase + SMEM_B + stage * B_BYTES + i * kMixBox * BK, &tmB40,
                                 kb * BK, brow + kMixBox * i, lead_full);
              tma_load_2d_pair(sbase + SMEM_B + stage * B_BYTES + 2 * kMixHalf * BK, &tmB8,
                               kb * BK, xrow, lead_full);
            } else {
              for (int i = 0; i < P * RC / 32; ++i)
                tma_load_2d_pair(sbase + SMEM_B + stage * B_BYTES + i * 32 * BK, &tmB, kb * BK,
                                 brow + 32 * i, lead_full);
            }
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
        const uint32_t idesc = i8_idesc(2 * BM, 2 * nplane, true, true);
        int stage = 0;
        uint32_t phase = 0;
        int acc = 0;
        uint32_t aphase = 0;
        bool ok = true;
        for (int t = pair; t < num_tiles && ok; t += num_pairs) {
          if (!mbar_wait(tempty_bar(acc), aphase ^ 1u, err)) break;
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + (uint32_t)(acc * 256);
          for (int kb = 0; kb < num_kb; ++kb) {
            if (!mbar_wait(full_bar(stage), phase, err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a_addr = sbase + SMEM_A + stage * A_BYTES;
            const uint32_t b_addr = sbase + SMEM_B + stage * B_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / 32; ++kk)
              mma_i8_pair(d_tmem, sw128_kmajor_desc(a_addr + 32 * kk),
                          sw128_kmajor_desc(b_addr + 32 * kk), idesc, (kb | kk) != 0 ? 1u : 0u);
            mma_commit_pair(empty_bar(stage), 0x3);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          mma_commit_pair(tfull_bar(acc), 0x3);
          if (++acc == 2) {
            acc = 0;
            aphase ^= 1u;
          }
        }
      }
    } else {
      // ---------------------------------------------------------- epilogue
      // warpgroup eg drains accumulator eg: the pair's tiles 2i + eg
      const int e = warp - 2;             // 0..7
      const int eg = e >> 2;              // warpgroup = accumulator
      const int q = warp & 3;             // TMEM lane quarter
      uint8_t* stg_ptr = smem + SMEM_STG + e * STG_BYTES;
      const uint32_t stg = sbase + SMEM_STG + (uint32_t)(e * STG_BYTES);
      ColInfo* col = reinterpret_cast<ColInfo*>(smem + SMEM_COL + e * COL_BYTES);
      MixInfo* mcol = reinterpret_cast<MixInfo*>(smem + SMEM_COL + e * COL_BYTES);
      uint8_t* ex_ptr = smem + SMEM_EX + e * EX_BYTES;
      uint32_t aphase = 0;
      bool used = false;
      for (int t = pair + eg * num_pairs; t < num_tiles; t += 2 * num_pairs) {
        int mb, nb;
        tile_coords(t, tiles_m, tiles_n, group_m, mb, nb);
        const int row0 = mb * 2 * BM + (int)rank * BM + q * 32;
        const int row = row0 + lane;
        const float sxf = row < M ? __ldg(sx + row) : 0.0f;
        // this tile's column constants, one table per warp (columns past N:
        // e_n 0, no bias, no slot -- their outputs are clipped by the stores);
        // a non-finite bias sends the whole tile to the exact path
        __syncwarp();  // every lane is done with the previous tile's table
        bool bad_bias = false;
        for (int r = lane; r < TR; r += 32) {
          const int n = nb * TR + r;
          const float p2 = __uint_as_float((uint32_t)(127 + (n < N ? __ldg(ebase + n) : 0)) << 23);
          const float bv = (bias != nullptr && n < N) ? __ldg(bias + n) : 0.0f;
          bad_bias |= !(fabsf(bv) <= 3.4028234663852886e38f);
          if (mixed) {
            const int sl = n < N ? __ldg(slot + n) : -1;
            MixInfo mi;
            mi.p2 = p2;
            mi.bias = bv;
            mi.exoff = (uint32_t)(sl >= 0 ? sl : kMixExtra) * 4u;
            mi.pad = 0u;
            mcol[r] = mi;
          } else {
            ColInfo ci;
            ci.p2 = p2;
            ci.bias = bv;
            col[r] = ci;
          }
        }
        const uint32_t force = sx_force_exact(sxf) |
                               (__any_sync(0xFFFFFFFFu, bad_bias) ? 0xFFFFFFFFu : 0u);
        __syncwarp();
        if (!mbar_wait(tfull_bar(eg), aphase, err)) break;
        tc_fence_after();
        const uint32_t t_lane = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(eg * 256);
        const uint32_t lead_tempty = mapa_shared(tempty_bar(eg), 0);
        switch (mode) {
          case 1: epilogue_tile<1>(t_lane, col, sxf, force, stg_ptr, stg, &tmY, nb * TR, row0, M, N, lane, lead_tempty, used); break;
          case 2: epilogue_tile<2>(t_lane, col, sxf, force, stg_ptr, stg, &tmY, nb * TR, row0, M, N, lane, lead_tempty, used); break;
          case 3: epilogue_tile<3>(t_lane, col, sxf, force, stg_ptr, stg, &tmY, nb * TR, row0, M, N, lane, lead_tempty, used); break;
          default: epilogue_mixed(t_lane, mcol, sxf, force, ex_ptr, stg_ptr, stg, &tmY, &tmY56, nb * TR, row0, M, N, lane, lead_tempty, used); break;
        }
        aphase ^= 1u;
      }
      if (lane == 0) bulk_wait<0>();
    }
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync();  // every remote arrival and MMA of the pair is done
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, kTmemCols);
}

bool g_attr_done[64];

}  // namespace

// Scratch of the GEMM route: the plane-count and overflow words, e_n and the
// top-digit slot of every row, the mixed-mode half-tile counters, then the
// planes ([3 N, K] int8: P N rows uniform, or 2 N rows + the top-digit rows).
struct PlaneScratch {
  size_t words, ebase, slot, hcount, planes, total;
  PlaneScratch(int64_t N, int64_t K) {
    auto r = [](size_t b) { return (b + 255u) & ~size_t(255u); };
    words = 0;
    ebase = words + r(16);
    slot = ebase + r((size_t)N * 4u);
    hcount = slot + r((size_t)N * 4u);
    planes = hcount + r((size_t)((N + kMixHalf - 1) / kMixHalf) * 8u);
    total = planes + (size_t)kMaxPlanes * (size_t)N * (size_t)K;
  }
};

size_t w4a8_plane_scratch_bytes(int64_t N, int64_t K) { return PlaneScratch(N, K).total; }

namespace {

// The words of a prepared weight carry this fixed epoch: qk_w4a8_prepare
// zeroes them before counting, so no word of an earlier preparation of the
// same buffer survives, and every product with the prepared form passes it.
constexpr unsigned long long kPreparedEpoch = 1;

struct PlanePtrs {
  unsigned long long* pword;
  unsigned long long* oword;
  int* ebase;
  int* slot;
  unsigned long long* hcount;
  uint8_t* planes;
  PlanePtrs(const void* scratch, int64_t N, int64_t K) {
    const PlaneScratch L(N, K);
    uint8_t* base = static_cast<uint8_t*>(const_cast<void*>(scratch));
    pword = reinterpret_cast<unsigned long long*>(base + L.words);
    oword = pword + 1;
    ebase = reinterpret_cast<int*>(base + L.ebase);
    slot = reinterpret_cast<int*>(base + L.slot);
    hcount = reinterpret_cast<unsigned long long*>(base + L.hcount);
    planes = base + L.planes;
  }
};

template <typename Kernel, typename... Args>
cudaError_t launch_ex(Kernel kernel, dim3 grid, dim3 block, size_t smem, bool dep, cudaStream_t s,
                      Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dep ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// The plane count (e_n, the slots, the plane-count word) and the digit rows
// of a weight, tagged with `epoch`.
cudaError_t launch_count_build(const uint8_t* Wp, const uint16_t* ws, const uint16_t* wo,
                               int64_t N, int64_t K, void* scratch, unsigned long long epoch,
                               bool pdl, cudaStream_t s) {
  const PlanePtrs P(scratch, N, K);
  // 1. plane count and e_n
  cudaError_t e = launch_ex(w4a8_plane_count_kernel,
                            dim3((unsigned)((N + kCountRowsPerBlock - 1) / kCountRowsPerBlock)),
                            dim3(32 * kCountRowsPerBlock), 0, pdl, s, ws, wo, (int)N, (int)K,
                            P.ebase, P.slot, P.hcount, P.pword, P.oword, epoch);
  if (e != cudaSuccess) return e;
  // 2. the planes (a few waves of the SMs; each thread loops over 16-code units)
  const long long units = N * (K / 16);
  long long blocks = (units + kBuildThreads - 1) / kBuildThreads;
  const long long cap = 8ll * num_sms();
  return launch_ex(w4a8_plane_build_kernel, dim3((unsigned)(blocks < cap ? blocks : cap)),
                   dim3(kBuildThreads), 0, true, s, Wp, ws, wo, (const int*)P.ebase,
                   (const int*)P.slot, (int)N, (int)K, P.planes,
                   (const unsigned long long*)P.pword, (const unsigned long long*)P.oword,
                   epoch);
}

// The product on counted and built planes: the per-group fold (it computes
// only when the planes cannot serve; launched as a programmatic dependent when
// fold_dep), then the plane GEMM.
cudaError_t launch_plane_product(const int8_t* xq, const float* sx, const int32_t* xsum,
                                 int64_t M, int64_t K, const uint8_t* Wp, const uint16_t* ws,
                                 const uint16_t* wo, const float* bias, int64_t N, uint16_t* y,
                                 const void* scratch, unsigned long long epoch, bool fold_dep,
                                 cudaStream_t s) {
  const PlanePtrs P(scratch, N, K);
  const unsigned long long* pword = P.pword;
  const unsigned long long* oword = P.oword;
  const int* ebase = P.ebase;
  const int* slot = P.slot;
  const uint8_t* planes = P.planes;
  // 3. the per-group fold, which computes only when the planes cannot
  cudaError_t e = launch_w4a8_fold(xq, sx, xsum, M, K, Wp, ws, wo, bias, N, y, nullptr, 0, 0,
                                   fold_dep, s, pword, epoch);
  if (e != cudaSuccess) return e;
  // 4. the plane GEMM
  CUtensorMap tA, tB, tB40, tB8, tY, tY56;
  if (!encode_tmap_2d(&tA, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, (uint64_t)K, (uint64_t)M,
                      (uint64_t)K, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, planes, (uint64_t)K,
                      (uint64_t)(kMaxPlanes * N), (uint64_t)K, BK, 32, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tB40, CU_TENSOR_MAP_DATA_TYPE_UINT8, planes, (uint64_t)K,
                      (uint64_t)(kMaxPlanes * N), (uint64_t)K, BK, kMixBox,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tB8, CU_TENSOR_MAP_DATA_TYPE_UINT8, planes, (uint64_t)K,
                      (uint64_t)(kMaxPlanes * N), (uint64_t)K, BK, 8, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, (uint64_t)N, (uint64_t)M,
                      (uint64_t)N * 2, 64, 32, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tY56, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, (uint64_t)N, (uint64_t)M,
                      (uint64_t)N * 2, 56, 32, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !g_attr_done[dev]) {
    e = cudaFuncSetAttribute(w4a8_planes_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    g_attr_done[dev] = true;
  }
  int* err = device_error_word();
  if (err == nullptr) return cudaErrorUnknown;
  // the tile count depends on the plane count, which only the device knows:
  // size the grid for the smallest tiles (64 weight rows, P = 3); pairs
  // without a tile at the actual P exit at once
  const long long tiles_m = (M + 2 * BM - 1) / (2 * BM);
  const long long max_tiles = tiles_m * ((N + 63) / 64);
  const long long pairs = num_sms() / 2;
  const int grid = 2 * (int)(max_tiles < pairs ? max_tiles : pairs);
  // a raster group's rows of xq (256 rows x K bytes per M tile) stay in L2
  long long group_m = (40ll << 20) / (2 * BM * K);
  group_m = group_m < 1 ? 1 : (group_m > tiles_m ? tiles_m : group_m);
  return launch_ex(w4a8_planes_kernel, dim3(grid), dim3(kThreads), (size_t)SMEM_ALLOC, true, s,
                   tA, tB, tB40, tB8, tY, tY56, sx, ebase, slot, bias, (int)M, (int)N, (int)K,
                   (int)group_m, pword, oword, epoch, err);
}

}  // namespace

cudaError_t launch_w4a8_gemm(const int8_t* xq, const float* sx, const int32_t* xsum, int64_t M,
                             int64_t K, const uint8_t* Wp, const uint16_t* ws, const uint16_t* wo,
                             const float* bias, int64_t N, uint16_t* y, void* scratch, bool pdl,
                             cudaStream_t s) {
  const unsigned long long epoch = next_epoch();
  cudaError_t e = launch_count_build(Wp, ws, wo, N, K, scratch, epoch, pdl, s);
  if (e != cudaSuccess) return e;
  return launch_plane_product(xq, sx, xsum, M, K, Wp, ws, wo, bias, N, y, scratch, epoch, true,
                              s);
}

cudaError_t launch_w4a8_prepare(const uint8_t* Wp, const uint16_t* ws, const uint16_t* wo,
                                int64_t N, int64_t K, void* prepared, int* planes,
                                cudaStream_t s) {
  const PlaneScratch L(N, K);
  // zero the words, e_n, the slots and the slot counters (not the planes)
  cudaError_t e = cudaMemsetAsync(prepared, 0, L.planes, s);
  if (e != cudaSuccess) return e;
  e = launch_count_build(Wp, ws, wo, N, K, prepared, kPreparedEpoch, false, s);
  if (e != cudaSuccess || planes == nullptr) return e;
  unsigned long long word = 0;
  e = cudaMemcpyAsync(&word, prepared, sizeof(word), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) *planes = (word >> 8) == kPreparedEpoch ? (int)(word & 0xFFull) : 0;
  return e;
}

cudaError_t launch_w4a8_gemm_prepared(const int8_t* xq, const float* sx, const int32_t* xsum,
                                      int64_t M, int64_t K, const uint8_t* Wp,
                                      const uint16_t* ws, const uint16_t* wo,
                                      const void* prepared, const float* bias, int64_t N,
                                      uint16_t* y, bool pdl, cudaStream_t s) {
  return launch_plane_product(xq, sx, xsum, M, K, Wp, ws, wo, bias, N, y, prepared,
                              kPreparedEpoch, pdl, s);
}


cudaError_t launch_w4a8_plane_count(const uint16_t* ws, const uint16_t* wo, int64_t N, int64_t K,
                                    void* scratch, unsigned long long epoch, bool pdl,
                                    cudaStream_t s) {
  const PlaneScratch L(N, K);
  uint8_t* base = static_cast<uint8_t*>(scratch);
  auto* pword = reinterpret_cast<unsigned long long*>(base + L.words);
  auto* ebase = reinterpret_cast<int*>(base + L.ebase);
  auto* slot = reinterpret_cast<int*>(base + L.slot);
  auto* hcount = reinterpret_cast<unsigned long long*>(base + L.hcount);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((N + kCountRowsPerBlock - 1) / kCountRowsPerBlock));
  cfg.blockDim = dim3(32 * kCountRowsPerBlock);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, w4a8_plane_count_kernel, ws, wo, (int)N, (int)K, ebase, slot,
                            hcount, pword, pword + 1, epoch);
}

}  // namespace qk
