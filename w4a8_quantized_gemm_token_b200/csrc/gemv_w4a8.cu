// gemv_w4a8.cu -- the W4A8 product for M <= 16 rows ("qlip-mlx" README,
// "w4a8_linear / W4A8Linear": a small-batch path for M <= 16 that runs at
// weight-bandwidth speed).
//
// Same arithmetic as the GEMM route: per group g of 64 along K the exact int32
// acc[m, n, g] = sum_k xq[m, k] * q[n, k] on the raw codes 0..15, then
//   y[m, n] = bf16( sx[m] * sum_g (s[n,g] * acc + o[n,g] * xsum[m,g]) + bias[n] )
// with the fold in fp64 and one rounding to bf16.
//
// Design (HBM-bound: the packed weights are ~97% of the bytes; every operand of
// the inner loop comes from shared memory so the loop never waits on L2):
//  * each CTA owns R = 16 * RT weight rows; at kernel start, before waiting on
//    the activation-quant kernel it depends on (programmatic dependent launch),
//    one thread issues 2-D TMA copies of the CTA's whole weight slice -- boxes
//    of R rows x 128 packed bytes (four groups), 128-byte swizzled so the
//    fragment reads are free of bank conflicts -- and bulk copies of its fp16
//    scales / offsets, one mbarrier per box, so the weight stream is in flight
//    while the previous kernel finishes (few large copies: per-copy overhead
//    of many small ones dominated an earlier version);
//  * after the wait: xq (all M rows, padded rows) by bulk copy, xsum as fp64 and the
//    scales / offsets as fp64 (converted once per CTA) into padded tables;
//  * 16 warps = RT row tiles x (16 / RT) K ranges; each warp starts as soon as
//    its K range has landed;
//  * nibbles are split in registers (one AND, one shift + AND per 8 codes)
//    straight into the A fragments of mma.sync m16n8k32 u8 x s8 (weights as A,
//    tokens as the N = 8 side); K is permuted identically in A and B (xq is
//    byte-permuted once in shared memory) so a lane reads 16 consecutive codes
//    and 16 xq bytes per group with one load each;
//  * per-group sums fold into fp64 (exact int -> fp64 by the 2^52 magic
//    number); the K ranges' partial sums add in a fixed order (deterministic),
//    then sx, bias and one rounding to bf16.
// The route is used only when weights, xq and the tables fit shared memory
// (K <= 4096 at M = 16); larger K goes to the GEMM.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "act_quant.cuh"
#include "qk_internal.h"
#include "sm100.cuh"

namespace qk {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = 16;
constexpr int kSmemLimit = 227 * 1024;
// In-kernel activation quantization keeps up to this many 16-byte chunks of
// x per thread in registers (M * K <= kQuantChunks * 8 * kThreads = 65536).
constexpr int kQuantChunks = 16;

// Shared-memory layout for R weight rows, K, and M token rows.
struct GemvLayout {
  int G, KS, Mp, nbox, XS;
  size_t w, so16, so64, xq, xs, sxo, amx, part, bars, total;
  __host__ __device__ GemvLayout(int R, int K, int M) {
    G = K / 64;
    KS = kWarps / (R / 16);
    Mp = M <= 8 ? 8 : 16;
    nbox = (G + 3) / 4;                                    // 128-byte boxes per row
    size_t off = 0;
    w = off;    off += (size_t)nbox * R * 128;             // packed codes, swizzled boxes
    so16 = off; off += (size_t)R * G * 2 * 2;              // fp16 scales then offsets
    off = (off + 15) & ~size_t(15);
    so64 = off; off += (size_t)R * (G + 1) * 16;           // {s, o} fp64, padded rows
    // xq row stride = 64 (mod 128): the two token rows of one 16-byte load
    // phase fall in opposite halves of the banks
    XS = (K + 63) / 128 * 128 + 64;
    xq = off;   off += (size_t)Mp * XS;                    // xq rows (zero past M)
    off = (off + 15) & ~size_t(15);
    xs = off;   off += (size_t)Mp * (G + 1) * 8;           // xsum fp64, padded rows
    sxo = off;  off += 16 * 4;                             // sx
    amx = off;  off += 16 * 4;                             // row absmax (in-kernel quant)
    // fp64 partial sums [K range][token][row], rows padded to R + 4 so the
    // reduce (consecutive rows per lane) and the stores are conflict-free
    part = off; off += (size_t)KS * 16 * (R + 4) * 8;
    bars = off; off += (size_t)(nbox + 2) * 8;             // mbarriers
    total = off + 1024;                                    // base alignment slack
  }
};

__device__ __forceinline__ void mma_u8s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ double i32_to_f64(int a) {
  return __hiloint2double(0x43300000, a ^ (int)0x80000000) - 4503601774854144.0;
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

// TT token tiles of 8 (M <= 8 * TT).  RT row tiles of 16 per CTA.  kFold:
// the product y; otherwise the per-group int32 sums go to acc_out.  kQuantX:
// the activations arrive as bf16 x and are quantized here (xq, sx, xsum are
// unused), with the rule of the stand-alone quantization kernel.
template <int TT, bool kFold, bool kQuantX>
__global__ void __launch_bounds__(kThreads, 1)
    w4a8_gemv_kernel(const __grid_constant__ CUtensorMap tmW, const uint16_t* __restrict__ x,
                     const int8_t* __restrict__ xq,
                     const float* __restrict__ sx,
                     const int32_t* __restrict__ xsum, int M, int K,
                     const uint8_t* __restrict__ Wp, const uint16_t* __restrict__ wscale,
                     const uint16_t* __restrict__ woffset, const float* __restrict__ bias, int N,
                     uint16_t* __restrict__ y, int32_t* __restrict__ acc_out, int m0, int m1,
                     int RT, int* err) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint8_t* smem = align_smem<1024>(smem_raw);
  const int R = 16 * RT;
  const GemvLayout L(R, K, M);
  const int G = L.G, KS = L.KS, nbox = L.nbox;
  const int XS = L.XS;         // xq row stride
  const int n0 = blockIdx.x * R;
  const int rows = min(R, N - n0);  // valid rows of this CTA (a multiple of 8)

  uint8_t* w_sm = smem + L.w;
  const uint16_t* s16 = reinterpret_cast<const uint16_t*>(smem + L.so16);
  const uint16_t* o16 = s16 + (size_t)R * G;
  double2* so_sm = reinterpret_cast<double2*>(smem + L.so64);
  int8_t* xq_sm = reinterpret_cast<int8_t*>(smem + L.xq);
  double* xs_sm = reinterpret_cast<double*>(smem + L.xs);
  float* sx_sm = reinterpret_cast<float*>(smem + L.sxo);
  double* part = reinterpret_cast<double*>(smem + L.part);
  // one barrier per weight box, then one for the scales, one for the activations
  const uint32_t bars = smem_u32(smem + L.bars);
  const uint32_t sbar = bars + 8u * nbox, abar = bars + 8u * (nbox + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    prefetch_tmap(&tmW);
    for (int q = 0; q < nbox + 2; ++q) mbar_init(bars + 8u * q, 1);
    fence_mbar_init();
  }
  __syncthreads();

  // ---- weights: issued before the dependency wait.  The scales / offsets go
  // first (small, needed first), then the boxes in K order, so the boxes land
  // roughly in the order the warps consume them.  A box always moves R rows x
  // 128 bytes; rows past N and bytes past K/2 are zero-filled.
  if (threadIdx.x == 0) {
    if (kFold) {
      mbar_arrive_expect_tx(sbar, (uint32_t)(rows * G * 2 * 2));
      bulk_load(smem_u32(smem + L.so16), wscale + (size_t)n0 * G, (uint32_t)(rows * G * 2), sbar);
      bulk_load(smem_u32(smem + L.so16) + (uint32_t)(R * G * 2), woffset + (size_t)n0 * G,
                (uint32_t)(rows * G * 2), sbar);
    }
    for (int j = 0; j < nbox; ++j) {
      mbar_arrive_expect_tx(bars + 8u * j, (uint32_t)(R * 128));
      tma_load_2d(smem_u32(w_sm + (size_t)j * R * 128), &tmW, 128 * j, n0, bars + 8u * j);
    }
  }
  // The next kernel may start its own prologue now; it waits for this grid to
  // finish before it touches anything this grid reads or writes.
  pdl_launch_dependents();

  // scales / offsets to fp64 once they land (rows beyond `rows` are never read)
  auto scales_to_fp64 = [&]() {
    if (!mbar_wait(sbar, 0, err)) return;
    for (int r = warp; r < rows; r += kWarps)
      for (int g = lane; g < G; g += 32)
        so_sm[r * (G + 1) + g] =
            make_double2((double)__half2float(__ushort_as_half(s16[(size_t)r * G + g])),
                         (double)__half2float(__ushort_as_half(o16[(size_t)r * G + g])));
  };

  // ---- activations come from the previous kernel
  bool ok = true;
  if constexpr (kQuantX) {
    // Every CTA quantizes the whole of x (L2-resident, M * K <= 65536): per
    // row the absmax, then the codes go straight into xq_sm in the even / odd
    // order of the K map below, and the group sums into xs_sm.
    unsigned int* amax_sm = reinterpret_cast<unsigned int*>(smem + L.amx);
    if (threadIdx.x < 16) amax_sm[threadIdx.x] = 0u;
    pdl_wait();
    const int nch = K >> 3;     // 16-byte chunks per row
    const int total = M * nch;  // chunk c of the flattened rows: row c / nch
    const uint4* src = reinterpret_cast<const uint4*>(x);
    uint4 v[kQuantChunks];
#pragma unroll
    for (int i = 0; i < kQuantChunks; ++i) {
      const int c = threadIdx.x + kThreads * i;
      v[i] = c < total ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
    }
    __syncthreads();  // amax_sm zeroed
#pragma unroll
    for (int i = 0; i < kQuantChunks; ++i) {
      if (kThreads * i >= total) break;  // warp-uniform
      const int c = threadIdx.x + kThreads * i;
      uint32_t mb = bf16x2_absmax_bits(0u, v[i].x);
      mb = bf16x2_absmax_bits(mb, v[i].y);
      mb = bf16x2_absmax_bits(mb, v[i].z);
      mb = bf16x2_absmax_bits(mb, v[i].w);
      const uint32_t m16 = max(mb & 0xFFFFu, mb >> 16);
      const int m = c < total ? c / nch : -1;
      // one shared-memory atomic per row present in the warp
      const unsigned same = __match_any_sync(0xFFFFFFFFu, m);
      const unsigned red = __reduce_max_sync(same, m16);
      if (m >= 0 && lane == __ffs(same) - 1) atomicMax(amax_sm + m, red);
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kQuantChunks; ++i) {
      if (kThreads * i >= total) break;  // warp-uniform
      const int c = threadIdx.x + kThreads * i;
      int sum = 0, m = 0, col = 0;
      if (c < total) {
        m = c / nch;
        col = c - m * nch;
        const float r = act_multiplier(__uint_as_float(amax_sm[m] << 16));
        const uint2 qc = quant_chunk(v[i], r, &sum);
        *reinterpret_cast<uint2*>(xq_sm + (size_t)m * XS + 8 * col) =
            make_uint2(__byte_perm(qc.x, qc.y, 0x6420), __byte_perm(qc.x, qc.y, 0x7531));
      }
      // the 8 chunks of a group sit in 8 consecutive lanes (nch % 8 == 0)
      sum = group8_sum(sum);
      if ((lane & 7) == 0 && c < total) xs_sm[m * (G + 1) + (col >> 3)] = i32_to_f64(sum);
    }
    if (threadIdx.x < M) sx_sm[threadIdx.x] = act_scale(__uint_as_float(amax_sm[threadIdx.x] << 16));
    for (int m = M + warp; m < L.Mp; m += kWarps)
      for (int g = lane; g < G; g += 32) xs_sm[m * (G + 1) + g] = 0.0;
    scales_to_fp64();
  } else {
    if (warp == 1) {
      pdl_wait();
      if (lane == 0) mbar_arrive_expect_tx(abar, (uint32_t)(M * K));
      __syncwarp();
      for (int m = lane; m < M; m += 32)
        bulk_load(smem_u32(xq_sm + (size_t)m * XS), xq + (size_t)m * K, (uint32_t)K, abar);
    }
    // (weights: no dependency wait needed)
    if (kFold) scales_to_fp64();
    if (warp != 1) pdl_wait();
    if (kFold) {
      if (threadIdx.x < M) sx_sm[threadIdx.x] = __ldg(sx + threadIdx.x);
      for (int m = warp; m < L.Mp; m += kWarps)
        for (int g = lane; g < G; g += 32)
          xs_sm[m * (G + 1) + g] = m < M ? i32_to_f64(__ldg(xsum + (size_t)m * G + g)) : 0.0;
    }
    // xq: within every 8 bytes put the even k first, then the odd k, to match
    // the even / odd nibble split of the weight codes (see the K map below)
    ok = mbar_wait(abar, 0, err);
    if (ok) {
      for (int m = warp; m < M; m += kWarps)
        for (int c = lane; c < K / 16; c += 32) {
          uint4* v = reinterpret_cast<uint4*>(xq_sm + (size_t)m * XS + 16 * c);
          const uint4 x = *v;
          *v = make_uint4(__byte_perm(x.x, x.y, 0x6420), __byte_perm(x.x, x.y, 0x7531),
                          __byte_perm(x.z, x.w, 0x6420), __byte_perm(x.z, x.w, 0x7531));
        }
    }
  }
  // token rows past M read as zeros
  for (int m = M + warp; m < L.Mp; m += kWarps)
    for (int c = lane; c < K / 16; c += 32)
      *reinterpret_cast<uint4*>(xq_sm + (size_t)m * XS + 16 * c) = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();

  // ---- warp (rt, q): row tile rt, groups g = q, q + KS, q + 2 KS, ...  The
  // groups interleave so that every box (four consecutive groups) is shared by
  // KS / 4 ... 4 warps per row tile and all warps work while the boxes land.
  const int rt = warp % RT, q = warp / RT;
  const int grp = lane >> 2, tq = lane & 3;
  const int rloc = rt * 16 + grp;  // this lane's first weight row (second: +8)
  // rows past the CTA's valid rows are read clamped (their results are dropped)
  const int ra = min(rloc, rows - 1), rb = min(rloc + 8, rows - 1);
  const double2* so_a = so_sm + (size_t)ra * (G + 1);
  const double2* so_b = so_sm + (size_t)rb * (G + 1);
  const double* xsp[TT];
  const int8_t* xb[TT];
#pragma unroll
  for (int tt = 0; tt < TT; ++tt) {
    xb[tt] = xq_sm + (size_t)(tt * 8 + grp) * XS + 16 * tq;
    xsp[tt] = xs_sm + (size_t)(tt * 8 + 2 * tq) * (G + 1);
  }

  // Offset term first, while the weight boxes are still in flight:
  // f = sum over this warp's groups of o[n, g] * xsum[m, g].
  double f[TT][4];
#pragma unroll
  for (int tt = 0; tt < TT; ++tt)
#pragma unroll
    for (int i = 0; i < 4; ++i) f[tt][i] = 0.0;
  if (kFold) {
    for (int g = q; g < G; g += KS) {
      const double oa = so_a[g].y, ob = so_b[g].y;
#pragma unroll
      for (int tt = 0; tt < TT; ++tt) {
        const double x0 = xsp[tt][g], x1 = xsp[tt][(G + 1) + g];
        f[tt][0] = fma(oa, x0, f[tt][0]);
        f[tt][1] = fma(oa, x1, f[tt][1]);
        f[tt][2] = fma(ob, x0, f[tt][2]);
        f[tt][3] = fma(ob, x1, f[tt][3]);
      }
    }
  }

  // K map.  For group g, lane (grp, tq) handles the 16 consecutive codes
  // k = 64 g + 16 tq + 0..15 (8 packed bytes).  Splitting a packed word into its
  // low nibbles (codes 0, 2, 4, 6) and high nibbles (codes 1, 3, 5, 7) gives the
  // A registers of one m16n8k32 MMA directly; xq was permuted to the same
  // even / odd order, so each MMA sums the same 32 k on both sides, and the two
  // MMAs of a group cover its 64 k once.
  // Packed byte p of row r sits in box p / 128, 16-byte chunk ((p % 128) / 16)
  // ^ (r % 8); here p = 32 g + 8 tq and g % 4 = q % 4 for every group of the
  // warp (KS is a multiple of 4), so the offsets inside a box are fixed.
  const int c = 2 * (q & 3) + (tq >> 1);
  const uint32_t offa = (uint32_t)(ra * 128 + ((c ^ (ra & 7)) << 4) + 8 * (tq & 1));
  const uint32_t offb = (uint32_t)(rb * 128 + ((c ^ (rb & 7)) << 4) + 8 * (tq & 1));
  const uint32_t box_bytes = (uint32_t)R * 128;

#pragma unroll 2
  for (int g = q; g < G; g += KS) {
    if (!mbar_wait(bars + 8u * (uint32_t)(g >> 2), 0, err)) { ok = false; break; }
    const uint8_t* box = w_sm + (size_t)(g >> 2) * box_bytes;
    const uint2 wa = *reinterpret_cast<const uint2*>(box + offa);
    const uint2 wb = *reinterpret_cast<const uint2*>(box + offb);
    // A registers: {row grp, row grp + 8} x {even codes, odd codes}, per MMA
    const uint32_t a0[4] = {wa.x & 0x0F0F0F0Fu, wb.x & 0x0F0F0F0Fu, (wa.x >> 4) & 0x0F0F0F0Fu,
                            (wb.x >> 4) & 0x0F0F0F0Fu};
    const uint32_t a1[4] = {wa.y & 0x0F0F0F0Fu, wb.y & 0x0F0F0F0Fu, (wa.y >> 4) & 0x0F0F0F0Fu,
                            (wb.y >> 4) & 0x0F0F0F0Fu};
    int acc[TT][4];
#pragma unroll
    for (int tt = 0; tt < TT; ++tt) {
      const uint4 b = *reinterpret_cast<const uint4*>(xb[tt] + 64 * g);
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[tt][i] = 0;
      mma_u8s8(acc[tt], a0, b.x, b.y);
      mma_u8s8(acc[tt], a1, b.z, b.w);
    }
    if constexpr (!kFold) {
      // accumulator dump: acc[(m - m0), n, g] for rows m0 <= m < m1
#pragma unroll
      for (int tt = 0; tt < TT; ++tt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int m = tt * 8 + 2 * tq + (i & 1);
          const int r = rloc + (i >> 1) * 8;
          if (m >= m0 && m < m1 && r < rows)
            acc_out[((size_t)(m - m0) * N + n0 + r) * G + g] = acc[tt][i];
        }
    } else {
      const double sa = so_a[g].x, sb = so_b[g].x;
#pragma unroll
      for (int tt = 0; tt < TT; ++tt) {
        f[tt][0] = fma(sa, i32_to_f64(acc[tt][0]), f[tt][0]);
        f[tt][1] = fma(sa, i32_to_f64(acc[tt][1]), f[tt][1]);
        f[tt][2] = fma(sb, i32_to_f64(acc[tt][2]), f[tt][2]);
        f[tt][3] = fma(sb, i32_to_f64(acc[tt][3]), f[tt][3]);
      }
    }
  }
  if constexpr (kFold) {
    // ---- partial sums of the warps of a row tile, added in a fixed order
#pragma unroll
    for (int tt = 0; tt < TT; ++tt)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = tt * 8 + 2 * tq + (i & 1);
        const int r = rloc + (i >> 1) * 8;
        part[((size_t)q * 16 + m) * (R + 4) + r] = f[tt][i];
      }
    __syncthreads();
    for (int m = threadIdx.x / R; m < M; m += kThreads / R) {
      const int r = threadIdx.x % R;  // consecutive threads -> consecutive n
      if (r >= rows) continue;
      double acc = 0.0;
      for (int qq = 0; qq < KS; ++qq) acc += part[((size_t)qq * 16 + m) * (R + 4) + r];
      const double v = fma((double)sx_sm[m], acc, bias != nullptr ? (double)bias[n0 + r] : 0.0);
      y[(size_t)m * N + n0 + r] = f64_to_bf16_bits(v);
    }
  }
}

size_t g_smem_set[6][64];

// Rows per CTA: the fewest (16, 32, 64) that still fit all CTAs in one wave.
int choose_rt(int64_t M, int64_t K, int64_t N) {
  const int sms = num_sms();
  int RT = 1;
  while (RT < 4 && (N + 16 * RT - 1) / (16 * RT) > sms &&
         GemvLayout(32 * RT, (int)K, (int)M).total <= (size_t)kSmemLimit)
    RT *= 2;
  return RT;
}

}  // namespace

size_t gemv_smem_bytes(int64_t M, int64_t K, int64_t N) {
  return GemvLayout(16 * choose_rt(M, K, N), (int)K, (int)M).total;
}

namespace {

// One launcher for both activation forms: x != nullptr quantizes x in the
// kernel, else xq / sx / xsum come from the caller.
cudaError_t launch_gemv(const uint16_t* x, const int8_t* xq, const float* sx,
                        const int32_t* xsum, int64_t M, int64_t K, const uint8_t* Wp,
                        const uint16_t* ws, const uint16_t* wo, const float* bias, int64_t N,
                        uint16_t* y, int32_t* acc_out, int64_t m0, int64_t m1, bool pdl,
                        cudaStream_t s) {
  const int RT = choose_rt(M, K, N);
  const int R = 16 * RT;
  const unsigned grid = (unsigned)((N + R - 1) / R);
  const size_t smem = GemvLayout(R, (int)K, (int)M).total;
  if (smem > (size_t)kSmemLimit) return cudaErrorInvalidValue;
  CUtensorMap tW;
  if (!encode_tmap_2d(&tW, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wp, (uint64_t)(K / 2), (uint64_t)N,
                      (uint64_t)(K / 2), 128, (uint32_t)R, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  int* err = device_error_word();
  if (err == nullptr) return cudaErrorUnknown;
  const bool fold = acc_out == nullptr;
  const bool qx = x != nullptr;
  if (qx && (!fold || M * K > (int64_t)kQuantChunks * 8 * kThreads)) return cudaErrorInvalidValue;
  decltype(&w4a8_gemv_kernel<1, true, false>) kernel;
  int variant;
  if (qx) {
    kernel = M <= 8 ? w4a8_gemv_kernel<1, true, true> : w4a8_gemv_kernel<2, true, true>;
    variant = M <= 8 ? 4 : 5;
  } else {
    kernel = M <= 8 ? (fold ? w4a8_gemv_kernel<1, true, false> : w4a8_gemv_kernel<1, false, false>)
                    : (fold ? w4a8_gemv_kernel<2, true, false> : w4a8_gemv_kernel<2, false, false>);
    variant = (M <= 8 ? 0 : 2) + (fold ? 0 : 1);
  }
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 64 || g_smem_set[variant][dev] < smem) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemLimit);
    if (e != cudaSuccess) return e;
    if (dev < 64) g_smem_set[variant][dev] = kSmemLimit;
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
  return cudaLaunchKernelEx(&cfg, kernel, tW, x, xq, sx, xsum, (int)M, (int)K, Wp, ws, wo, bias,
                            (int)N, y, acc_out, (int)m0, (int)m1, RT, err);
}

}  // namespace

bool gemv_quant_fits(int64_t M, int64_t K, int64_t N) {
  return gemv_fits(M, K, N) && M * K <= (int64_t)kQuantChunks * 8 * kThreads;
}

cudaError_t launch_w4a8_gemv(const int8_t* xq, const float* sx, const int32_t* xsum, int64_t M,
                             int64_t K, const uint8_t* Wp, const uint16_t* ws, const uint16_t* wo,
                             const float* bias, int64_t N, uint16_t* y, int32_t* acc_out,
                             int64_t m0, int64_t m1, bool pdl, cudaStream_t s) {
  return launch_gemv(nullptr, xq, sx, xsum, M, K, Wp, ws, wo, bias, N, y, acc_out, m0, m1, pdl,
                     s);
}

cudaError_t launch_w4a8_gemv_quant(const uint16_t* x, int64_t M, int64_t K, const uint8_t* Wp,
                                   const uint16_t* ws, const uint16_t* wo, const float* bias,
                                   int64_t N, uint16_t* y, bool pdl, cudaStream_t s) {
  return launch_gemv(x, nullptr, nullptr, nullptr, M, K, Wp, ws, wo, bias, N, y, nullptr, 0, 0,
                     pdl, s);
}

}  // namespace qk

