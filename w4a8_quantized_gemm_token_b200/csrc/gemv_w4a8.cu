// gemv_w4a8.cu -- the W4A8 product for M <= 16 rows ("qlip-mlx" README,
// "w4a8_linear / W4A8Linear": a small-batch path for M <= 16 that runs at
// weight-bandwidth speed).
//
// Same arithmetic as the GEMM route: per group g of 64 along K the exact int32
// acc[m, n, g] = sum_k xq[m, k] * q[n, k] on the raw codes 0..15, then
//   y[m, n] = bf16( sx[m] * sum_g (s[n,g] * acc + o[n,g] * xsum[m,g]) + bias[n] )
// with the fold in fp64 and one rounding to bf16.
//
// Design.  The packed weights are ~97% of the bytes, and a call at
// N = K = 4096 moves only ~9.5 MB, so a lone launch is dominated by fixed
// latencies.  The kernel is therefore built for back-to-back calls (the
// layers of a model, graph replays): while one call computes, the next call's
// CTAs are already resident with their weights in flight.
//  * A cluster of C CTAs shares R weight rows; CTA c takes the groups of one
//    K slice [c GC, (c + 1) GC).  The host picks (R, C) so that every warp
//    covers at most 16 groups, two CTAs fit an SM (this call's and the next
//    one's) and the grid is at most one CTA per SM.
//  * At kernel start, before the programmatic-dependency wait, one thread
//    issues 2-D TMA copies of the CTA's packed codes (boxes of R rows x 128
//    bytes, 128-byte swizzled so the fragment reads are conflict-free) and
//    bulk / TMA copies of its fp16 scales / offsets; the bias of the CTA's rows
//    is read too.  (An earlier form loaded the codes into registers with
//    per-lane loads: the flood of loads then delayed the co-resident CTA's
//    latency-critical activation loads.)  Weights, scales, offsets and bias
//    are therefore read before the previous kernel in the stream has
//    finished: they must not be written by a kernel that triggers its
//    dependents early (no kernel of this library that writes weights does).
//  * After the wait the CTA either quantizes its K slice of bf16 x itself
//    (the rule of the stand-alone quantization kernel; with C > 1 the per-row
//    absmax is exchanged through distributed shared memory) or reads
//    quantized xq / sx / xsum.
//  * 8 warps = R/16 row tiles x KW group ranges.  Nibbles are split in
//    registers and put back in K order (two byte permutes per packed word)
//    as the A fragments of mma.sync m16n8k32 u8 x s8 (weights as A, tokens as
//    the N = 8 side), so each lane pairs its 8 packed bytes of a group with 16
//    consecutive activation bytes, and the activations stay in their natural
//    order: the quantized rows arrive by bulk copies issued by one thread.
//  * Per-group sums fold into fp64 (exact int -> fp64 by the 2^52 magic
//    number).  With one token the lanes first gather one group each by
//    shuffles, so no lane folds an all-zero token column.  When the kernel
//    quantizes x itself (up to 8 tokens), the fp16 scales and offsets are
//    first widened into an fp64 table before the dependency wait.
//  * The partial sums of all warps of all CTAs of a cluster go, through
//    distributed shared memory, to the CTA that owns the row (R / C rows
//    each), which adds them in a fixed order (deterministic), applies sx and
//    the bias and rounds once to bf16.
// Every wait is bounded; a CTA that gives up still takes part in every
// cluster barrier, so its peers never wait on it forever.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "act_quant.cuh"
#include "qk_internal.h"
#include "sm100.cuh"

namespace qk {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = 8;
constexpr int kSmemLimit = 227 * 1024;
// Two CTAs per SM: 228 KB of shared memory per SM, 1 KB reserved per CTA.
constexpr int kSmemTwoPerSm = 113 * 1024;
// In-kernel activation quantization keeps up to this many 16-byte chunks of
// x per thread in registers (M * KC <= kQuantChunks * 8 * kThreads = 16384,
// KC = the K slice of one CTA).
constexpr int kQuantChunks = 8;
// Groups of 64 codes one warp covers (straight-line code over all of them).
constexpr int kWarpGroups = 16;

// Shared-memory layout of one CTA: R weight rows, cluster of C CTAs along K,
// M token rows.
struct GemvLayout {
  int R, C, M, G, GC, RT, KW, GW, RO, Mp, XS, nbox;
  bool tab;                    // M <= 8 quantizing x in the kernel: fp64 scale table
  size_t w, s16, xq, st, xs, sx, amx, bias, part, bars, total;
  __host__ __device__ GemvLayout(int R_, int C_, int K, int M_, bool quant_x) {
    R = R_;
    C = C_;
    M = M_;
    G = K / 64;
    GC = (G + C - 1) / C;      // groups per K slice (C > 1: C divides G)
    RT = R / 16;               // row tiles
    KW = kWarps / RT;          // group ranges per row tile
    GW = (GC + KW - 1) / KW;   // groups per warp (at most kWarpGroups)
    RO = R / C;                // rows each CTA finalizes
    Mp = M <= 8 ? 8 : 16;      // token columns of the MMAs
    // xq row stride = 64 (mod 128): the two token rows of one 16-byte load
    // phase fall in opposite halves of the banks
    XS = (GC * 64 + 127) / 128 * 128 + 64;
    nbox = (GC + 3) / 4;       // 128-byte weight boxes per row of the slice
    tab = quant_x && M <= 8;
    size_t off = 0;
    w = off;    off += (size_t)nbox * R * 128;        // packed codes, 128-byte-swizzled boxes
    s16 = off;                                        // fp16 scales [R][GC], then offsets
    if (tab) {
      // the fp16 scales are consumed into the table before the dependency
      // wait; the xq rows land in the same bytes after it
      xq = off; off += std::max((size_t)R * GC * 2 * 2, (size_t)M * XS);
      off = (off + 15) & ~size_t(15);
      st = off; off += (size_t)R * (GC + 1) * 8;      // {hi(s), hi(o)} [R][GC + 1]
    } else {
      off += (size_t)R * GC * 2 * 2;
      off = (off + 127) & ~size_t(127);
      xq = off; off += (size_t)M * XS;                // xq rows of the slice
      st = off;
    }
    off = (off + 15) & ~size_t(15);
    xs = off;   off += (size_t)Mp * (GC + 1) * 8;     // xsum as fp64, zero past M
    sx = off;   off += 16 * 4;                        // sx
    amx = off;  off += (size_t)(C + 1) * 16 * 4 + 256 * 4 + 16 * 4;  // absmax: [C] exchange slots,
                                                      // local; group maxima; row multipliers
    bias = off; off += (size_t)RO * 4;                // bias of the rows this CTA finalizes
    off = (off + 15) & ~size_t(15);
    part = off; off += (size_t)C * KW * M * RO * 8;   // fp64 partials [slot][token][row]
    bars = off; off += (size_t)(nbox + 2) * 8;        // mbarriers: the boxes, the scales,
                                                      // the activation rows
    total = off + 1024;                               // base alignment slack
  }
};

// D = A (16 x 32, u8) * B (32 x 8, s8), int32, from a zero accumulator.  Not
// volatile: it has no side effects, so the compiler may interleave the MMAs
// of independent groups.
__device__ __forceinline__ void mma_u8s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(0));
}

__device__ __forceinline__ double i32_to_f64(int a) {
  return __hiloint2double(0x43300000, a ^ (int)0x80000000) - 4503601774854144.0;
}

__device__ __forceinline__ double h2d(uint16_t h) {
  return (double)__half2float(__ushort_as_half(h));
}

// An fp16 value widened to fp64 has a zero low word: the table keeps the
// high words only.
__device__ __forceinline__ double hi_to_f64(uint32_t hi) { return __hiloint2double((int)hi, 0); }

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

// ---- distributed shared memory (cluster-window addresses from mapa_shared)
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void st_cluster_f64(uint32_t addr, double v) {
  asm volatile("st.shared::cluster.f64 [%0], %1;" ::"r"(addr), "d"(v) : "memory");
}
// Split cluster barrier: every thread of every CTA arrives once, then waits.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The A fragment of one m16n8k32 MMA from 4 packed bytes (8 codes, code 2i
// in the low nibble of byte i) of each of the lane's two rows: the codes back
// in K order, four per register.
__device__ __forceinline__ void split_codes(uint32_t wa, uint32_t wb, uint32_t (&a)[4]) {
  const uint32_t la = wa & 0x0F0F0F0Fu, ha = (wa >> 4) & 0x0F0F0F0Fu;  // even, odd codes
  const uint32_t lb = wb & 0x0F0F0F0Fu, hb = (wb >> 4) & 0x0F0F0F0Fu;
  a[0] = __byte_perm(la, ha, 0x5140);  // row ra:     codes 0..3
  a[1] = __byte_perm(lb, hb, 0x5140);  // row ra + 8: codes 0..3
  a[2] = __byte_perm(la, ha, 0x7362);  // row ra:     codes 4..7
  a[3] = __byte_perm(lb, hb, 0x7362);  // row ra + 8: codes 4..7
}


// TT token tiles of 8 (M <= 8 TT).  kFold: the product y; otherwise the
// per-group int32 sums of rows [m0, m1) go to acc_out.  kQuantX: the
// activations arrive as bf16 x and are quantized here (xq, sx, xsum unused).
// kOne: M == 1, the one-token fold.  C: CTAs per cluster along K.
// Grid (C, ceil(N / R)), cluster (C, 1, 1).
template <int TT, bool kFold, bool kQuantX, bool kOne, int C>
__global__ void __launch_bounds__(kThreads, 2)
    w4a8_gemv_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmS,
                     const __grid_constant__ CUtensorMap tmO,
                     const uint16_t* __restrict__ x, const int8_t* __restrict__ xq,
                     const float* __restrict__ sx, const int32_t* __restrict__ xsum, int M, int K,
                     const uint8_t* __restrict__ Wp, const uint16_t* __restrict__ wscale,
                     const uint16_t* __restrict__ woffset, const float* __restrict__ bias, int N,
                     uint16_t* __restrict__ y, int32_t* __restrict__ acc_out, int m0, int m1, int R,
                     int early_trigger, int* err) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint8_t* smem = align_smem<1024>(smem_raw);
  const GemvLayout L(R, C, K, M, kQuantX);
  const int G = L.G, GC = L.GC, RT = L.RT, KW = L.KW, RO = L.RO, XS = L.XS;
  const int crank = (int)blockIdx.x;  // rank in the cluster = K slice
  const int n0 = (int)blockIdx.y * R;
  const int rows = min(R, N - n0);    // valid rows of this row block (a multiple of 8)
  const int g0 = crank * GC;
  const int gcount = min(GC, G - g0);  // groups of this slice (GC when C > 1)

  const uint16_t* s16 = reinterpret_cast<const uint16_t*>(smem + L.s16);
  const uint16_t* o16 = s16 + (size_t)R * GC;
  int8_t* xq_sm = reinterpret_cast<int8_t*>(smem + L.xq);
  double* xs_sm = reinterpret_cast<double*>(smem + L.xs);
  float* sx_sm = reinterpret_cast<float*>(smem + L.sx);
  unsigned int* amx_sm = reinterpret_cast<unsigned int*>(smem + L.amx);  // [C][16], local [16]
  float* bias_sm = reinterpret_cast<float*>(smem + L.bias);
  double* part = reinterpret_cast<double*>(smem + L.part);
  const uint8_t* w_sm = smem + L.w;
  const uint32_t wbar0 = smem_u32(smem + L.bars);      // box j: wbar0 + 8 j
  const uint32_t sbar = wbar0 + 8u * (uint32_t)L.nbox;
  const uint32_t abar = sbar + 8u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rt = warp % RT, kw = warp / RT;
  const int grp = lane >> 2, tq = lane & 3;
  const int ra = rt * 16 + grp;  // this lane's weight rows: ra and ra + 8
  // this warp's groups of the slice: [gbeg, gbeg + gn)
  const int gbeg = kw * L.GW;
  const int gn = max(0, min(L.GW, gcount - gbeg));

  // ---- before the dependency wait: scales / offsets by bulk copy, the
  // packed codes of this lane's two rows into registers, the bias.
  if (threadIdx.x == 0) {
    prefetch_tmap(&tmW);
    for (int q = 0; q <= L.nbox + 1; ++q) mbar_init(wbar0 + 8u * q, 1);
    fence_mbar_init();
    if (kFold) {
      if (C > 1) {
        mbar_arrive_expect_tx(sbar, (uint32_t)(2 * R * GC * 2));
        tma_load_2d(smem_u32(smem + L.s16), &tmS, g0, n0, sbar);
        tma_load_2d(smem_u32(smem + L.s16) + (uint32_t)(R * GC * 2), &tmO, g0, n0, sbar);
      } else {
        mbar_arrive_expect_tx(sbar, (uint32_t)(2 * rows * G * 2));
        bulk_load(smem_u32(smem + L.s16), wscale + (size_t)n0 * G, (uint32_t)(rows * G * 2), sbar);
        bulk_load(smem_u32(smem + L.s16) + (uint32_t)(R * G * 2), woffset + (size_t)n0 * G,
                  (uint32_t)(rows * G * 2), sbar);
      }
    }
  }
  // the packed codes: boxes of R rows x 128 bytes (four groups), 128-byte
  // swizzled, in K order; rows past N and bytes past K/2 are zero-filled
  if (threadIdx.x == 0) {
    for (int j = 0; j < L.nbox; ++j) {
      mbar_arrive_expect_tx(wbar0 + 8u * j, (uint32_t)(R * 128));
      tma_load_2d(smem_u32(w_sm + (size_t)j * R * 128), &tmW, 32 * g0 + 128 * j, n0, wbar0 + 8u * j);
    }
  }
  if (kFold && threadIdx.x < RO && crank * RO + (int)threadIdx.x < rows)
    bias_sm[threadIdx.x] = bias != nullptr ? __ldg(bias + n0 + crank * RO + threadIdx.x) : 0.0f;
  if (early_trigger) pdl_launch_dependents();
  // token rows past M: zero xsum (their MMA columns are zero too)
  for (int i = threadIdx.x; i < (L.Mp - M) * (GC + 1); i += kThreads)
    xs_sm[(size_t)M * (GC + 1) + i] = 0.0;
  if (threadIdx.x < 16) amx_sm[C * 16 + threadIdx.x] = 0u;
  // M <= 8 quantizing x in the kernel: the scales and offsets widened to fp64
  // (high words) in a table with rows padded to GC + 1 entries (the eight rows
  // a warp reads at once fall in distinct banks), so the product loop
  // converts nothing.  Built before the dependency wait (calls of this form
  // follow one another, and the scales have long landed); the activation
  // codes land on the fp16 scales after the wait.  (With xq from the
  // quantization kernel in front, the GEMV starts too shortly before its
  // release: waiting for the scales there, or building the table after the
  // release, measured slower than converting in the loop.)
  auto build_table = [&]() {
    __all_sync(0xFFFFFFFFu, mbar_wait(sbar, 0, err));
    uint2* stab = reinterpret_cast<uint2*>(smem + L.st);
    const int dr = kThreads / GC, dg = kThreads - dr * GC;
    int r = (int)threadIdx.x / GC, g = (int)threadIdx.x - r * GC;
    while (r < R) {
      stab[r * (GC + 1) + g] = make_uint2((uint32_t)__double2hiint(h2d(s16[r * GC + g])),
                                          (uint32_t)__double2hiint(h2d(o16[r * GC + g])));
      r += dr;
      g += dg;
      if (g >= GC) {
        g -= GC;
        ++r;
      }
    }
  };
  if constexpr (kFold && TT == 1 && kQuantX) {  // (exactly when L.tab)
    __syncthreads();  // thread 0 has initialized the barriers
    build_table();
  }
  // peers write into this CTA's shared memory only after every CTA of the
  // cluster has arrived here (it has started); with the table, every thread
  // is done with the fp16 scales before the activation rows overwrite them
  if (C > 1) cluster_arrive_relaxed();
  __syncthreads();

  // ---- activations (they come from the previous kernel)
  pdl_wait();
  if (!early_trigger) pdl_launch_dependents();
  if constexpr (kQuantX) {
    const int nch = GC * 8;         // 16-byte chunks per row of the slice
    const int total = M * nch;      // chunk c = threadIdx.x + kThreads i: row c / nch
    // (row, chunk) of c for every i, by steps of kThreads (one division each)
    const int dm = kThreads / nch, dr = kThreads - dm * nch;
    const int m_first = (int)threadIdx.x / nch, r_first = (int)threadIdx.x - m_first * nch;
    const uint4* src = reinterpret_cast<const uint4*>(x);
    uint4 v[kQuantChunks];
    {
      int m = m_first, r = r_first;
#pragma unroll
      for (int i = 0; i < kQuantChunks; ++i) {
        v[i] = make_uint4(0u, 0u, 0u, 0u);
        if (m < M) v[i] = __ldg(src + (((size_t)m * K + (size_t)g0 * 64) >> 3) + r);
        m += dm;
        r += dr;
        if (r >= nch) {
          r -= nch;
          ++m;
        }
      }
    }
    unsigned int* amx_local = amx_sm + C * 16;
    unsigned int* gmax_sm = amx_sm + (C + 1) * 16;                    // [M][GC] group maxima
    float* rmul_sm = reinterpret_cast<float*>(gmax_sm + 256);          // [16] row multipliers
    // Group maxima: the 8 chunks of a group sit in 8 consecutive lanes of one
    // row (nch % 8 == 0), so three shuffles and one plain store per group.
#pragma unroll
    for (int i = 0; i < kQuantChunks; ++i) {
      if (kThreads * i >= total) break;  // warp-uniform
      const int c = threadIdx.x + kThreads * i;
      uint32_t mb = bf16x2_absmax_bits(0u, v[i].x);
      mb = bf16x2_absmax_bits(mb, v[i].y);
      mb = bf16x2_absmax_bits(mb, v[i].z);
      mb = bf16x2_absmax_bits(mb, v[i].w);
      uint32_t m16 = max(mb & 0xFFFFu, mb >> 16);
      m16 = max(m16, __shfl_xor_sync(0xFFFFFFFFu, m16, 1));
      m16 = max(m16, __shfl_xor_sync(0xFFFFFFFFu, m16, 2));
      m16 = max(m16, __shfl_xor_sync(0xFFFFFFFFu, m16, 4));
      if ((lane & 7) == 0 && c < total) gmax_sm[c >> 3] = m16;  // index m * GC + g
    }
    __syncthreads();
    // row maxima over this slice: warp w takes rows w and w + 8
    for (int m = warp; m < M; m += kWarps) {
      uint32_t mr = 0u;
      for (int g = lane; g < GC; g += 32) mr = max(mr, gmax_sm[m * GC + g]);
      mr = __reduce_max_sync(0xFFFFFFFFu, mr);
      if (lane == 0) amx_local[m] = mr;
    }
    __syncthreads();
    if (C > 1) {
      cluster_wait_acquire();  // (the start barrier) every peer is running
      // this slice's absmax of every row, to every CTA of the cluster
      if (threadIdx.x < C * M) {
        const int peer = threadIdx.x / M, m = threadIdx.x - peer * M;
        st_cluster_u32(mapa_shared(smem_u32(amx_sm + crank * 16 + m), (uint32_t)peer),
                       amx_local[m]);
      }
      __syncwarp();
      cluster_arrive_release();
      cluster_wait_acquire();
    }
    // the row's absmax over the whole K, its multiplier and scale (one
    // division each per row)
    if (threadIdx.x < M) {
      unsigned int b = amx_local[threadIdx.x];
      if (C > 1) {
        b = amx_sm[threadIdx.x];
#pragma unroll
        for (int q = 1; q < C; ++q) b = max(b, amx_sm[q * 16 + threadIdx.x]);
      }
      const float amax = __uint_as_float(b << 16);
      rmul_sm[threadIdx.x] = act_multiplier(amax);
      sx_sm[threadIdx.x] = act_scale(amax);
    }
    __syncthreads();
    {
      int m = m_first, cc = r_first;
#pragma unroll
      for (int i = 0; i < kQuantChunks; ++i) {
        if (kThreads * i >= total) break;  // warp-uniform
        int sum = 0;
        if (m < M) {
          const uint2 qc = quant_chunk(v[i], rmul_sm[m], &sum);
          *reinterpret_cast<uint2*>(xq_sm + (size_t)m * XS + 8 * cc) = qc;
        }
        // the 8 chunks of a group sit in 8 consecutive lanes (nch % 8 == 0)
        sum = group8_sum(sum);
        if ((lane & 7) == 0 && m < M) xs_sm[m * (GC + 1) + (cc >> 3)] = i32_to_f64(sum);
        m += dm;
        cc += dr;
        if (cc >= nch) {
          cc -= nch;
          ++m;
        }
      }
    }
    __syncthreads();
  } else {
    // quantized activations: the M rows of the slice by bulk copy (issued by
    // one thread), the group sums and sx by plain loads meanwhile
    if (threadIdx.x == 0) {
      mbar_arrive_expect_tx(abar, (uint32_t)(M * gcount * 64));
      for (int m = 0; m < M; ++m)
        bulk_load(smem_u32(xq_sm + (size_t)m * XS), xq + (size_t)m * K + (size_t)g0 * 64,
                  (uint32_t)(gcount * 64), abar);
    }
    if (kFold) {
      // (row, group) pairs by steps of kThreads (one division each)
      const int dm = kThreads / GC, dg = kThreads - dm * GC;
      int m = (int)threadIdx.x / GC, g = (int)threadIdx.x - m * GC;
      constexpr int kXs = 8;    // M * GC <= kXs * kThreads in every plan with K <= 4096
      int xv[kXs];
      int mi[kXs], gi[kXs];
#pragma unroll
      for (int i = 0; i < kXs; ++i) {
        mi[i] = m;
        gi[i] = g;
        xv[i] = m < M ? __ldg(xsum + (size_t)m * G + g0 + g) : 0;
        m += dm;
        g += dg;
        if (g >= GC) {
          g -= GC;
          ++m;
        }
      }
      if ((int)threadIdx.x < M) sx_sm[threadIdx.x] = __ldg(sx + threadIdx.x);
#pragma unroll
      for (int i = 0; i < kXs; ++i)
        if (mi[i] < M) xs_sm[mi[i] * (GC + 1) + gi[i]] = i32_to_f64(xv[i]);
      // the rest (a larger K slice)
      for (; m < M;) {
        xs_sm[m * (GC + 1) + g] = i32_to_f64(__ldg(xsum + (size_t)m * G + g0 + g));
        m += dm;
        g += dg;
        if (g >= GC) {
          g -= GC;
          ++m;
        }
      }
    }
    // (if the rows never land the results are wrong and the error word is set)
    __all_sync(0xFFFFFFFFu, mbar_wait(abar, 0, err));
    __syncthreads();
    if (C > 1) cluster_wait_acquire();  // the start barrier
  }

  // ---- products.  Warp (rt, kw): row tile rt, groups [gbeg, gbeg + gn)
  const int8_t* xb[TT];
  bool tv[TT];
#pragma unroll
  for (int tt = 0; tt < TT; ++tt) {
    const int t = tt * 8 + grp;  // this lane's token column
    tv[tt] = t < M;
    xb[tt] = xq_sm + (size_t)(tv[tt] ? t : 0) * XS + 16 * tq;
  }
  double f[TT][4];
#pragma unroll
  for (int tt = 0; tt < TT; ++tt)
#pragma unroll
    for (int i = 0; i < 4; ++i) f[tt][i] = 0.0;
  double fa = 0.0, fb = 0.0;  // one token: rows ra, ra + 8
  // (if the scales or a box never land the results are wrong and the error
  // word is set)
  if (kFold) __all_sync(0xFFFFFFFFu, mbar_wait(sbar, 0, err));
  if (gn > 0)
    for (int j = gbeg / 4; j <= (gbeg + gn - 1) / 4; ++j)
      __all_sync(0xFFFFFFFFu, mbar_wait(wbar0 + 8u * j, 0, err));
  // Packed byte p of row r sits in box p / 128, 16-byte chunk
  // ((p % 128) / 16) ^ (r % 8), and r % 8 == grp for both rows of the lane.
  const uint32_t offa = (uint32_t)(ra * 128 + 8 * (tq & 1));
  const uint32_t offb = offa + 8u * 128u;

  // K map.  For group g, lane (grp, tq) handles the 16 consecutive codes
  // k = 64 g + 16 tq + 0..15 (8 packed bytes, 16 bytes of xq).  The first MMA
  // takes codes 0..7 of every lane's 16 (A: split_codes of the first packed
  // word; B: xq bytes 0..7), the second codes 8..15, so each MMA sums the same
  // 32 k on both sides and the two MMAs of a group cover its 64 k once.
  //
  // All kWarpGroups groups in straight-line code (no branch between them, so
  // the loads, MMAs and folds of different groups overlap); groups past gn
  // re-read the last group and their results are dropped.
#pragma unroll
  for (int blk = 0; blk < kWarpGroups / 4; ++blk) {
    int A0[4], A2[4];                 // one token: the block's group sums
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = 4 * blk + u;
      const int gl = gbeg + min(i, gn - 1);  // group within the slice (clamped)
      const uint8_t* box = w_sm + (size_t)(gl >> 2) * R * 128;
      const uint32_t sw = (uint32_t)(((2 * (gl & 3) + (tq >> 1)) ^ grp) << 4);
      const uint2 wa = *reinterpret_cast<const uint2*>(box + offa + sw);
      const uint2 wb = *reinterpret_cast<const uint2*>(box + offb + sw);
      // A registers of the two MMAs: codes 0..7 and 8..15 of the lane's 16
      uint32_t a0[4], a1[4];
      split_codes(wa.x, wb.x, a0);
      split_codes(wa.y, wb.y, a1);
      // two independent MMAs per token tile (half a group each), then one add
      int acc[TT][4];
#pragma unroll
      for (int tt = 0; tt < TT; ++tt) {
        const uint4 b = tv[tt] ? *reinterpret_cast<const uint4*>(xb[tt] + 64 * gl)
                               : make_uint4(0u, 0u, 0u, 0u);
        int h0[4], h1[4];
        mma_u8s8(h0, a0, b.x, b.y);
        mma_u8s8(h1, a1, b.z, b.w);
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[tt][q] = h0[q] + h1[q];
      }
      if constexpr (!kFold) {
        // accumulator dump: acc[(m - m0), n, g] for rows m0 <= m < m1
#pragma unroll
        for (int tt = 0; tt < TT; ++tt)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int m = tt * 8 + 2 * tq + (q & 1);
            const int r = ra + (q >> 1) * 8;
            if (i < gn && m >= m0 && m < m1 && r < rows)
              acc_out[((size_t)(m - m0) * N + n0 + r) * G + g0 + gl] = acc[tt][q];
          }
      } else if constexpr (kOne) {
        A0[u] = acc[0][0];  // token 0 lives in the lanes with tq == 0
        A2[u] = acc[0][2];
      } else if (i < gn) {
        double sa, sb, oa, ob;
        if constexpr (TT == 1 && kQuantX) {
          const uint2* stab = reinterpret_cast<const uint2*>(smem + L.st);
          const uint2 ta = stab[ra * (GC + 1) + gl], tb = stab[(ra + 8) * (GC + 1) + gl];
          sa = hi_to_f64(ta.x);
          oa = hi_to_f64(ta.y);
          sb = hi_to_f64(tb.x);
          ob = hi_to_f64(tb.y);
        } else {
          sa = h2d(s16[ra * GC + gl]);
          sb = h2d(s16[(ra + 8) * GC + gl]);
          oa = h2d(o16[ra * GC + gl]);
          ob = h2d(o16[(ra + 8) * GC + gl]);
        }
#pragma unroll
        for (int tt = 0; tt < TT; ++tt) {
          const double x0 = xs_sm[(tt * 8 + 2 * tq) * (GC + 1) + gl];
          const double x1 = xs_sm[(tt * 8 + 2 * tq + 1) * (GC + 1) + gl];
          f[tt][0] = fma(oa, x0, fma(sa, i32_to_f64(acc[tt][0]), f[tt][0]));
          f[tt][1] = fma(oa, x1, fma(sa, i32_to_f64(acc[tt][1]), f[tt][1]));
          f[tt][2] = fma(ob, x0, fma(sb, i32_to_f64(acc[tt][2]), f[tt][2]));
          f[tt][3] = fma(ob, x1, fma(sb, i32_to_f64(acc[tt][3]), f[tt][3]));
        }
      }
    }
    if constexpr (kFold && kOne) {
      // lane (grp, tq) folds group 4 blk + tq of the warp, gathered from
      // lane (grp, 0)
      int s0 = 0, s2 = 0;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v0 = __shfl_sync(0xFFFFFFFFu, A0[u], lane & ~3);
        const int v2 = __shfl_sync(0xFFFFFFFFu, A2[u], lane & ~3);
        if (tq == u) {
          s0 = v0;
          s2 = v2;
        }
      }
      const int ig = 4 * blk + tq;
      if (ig < gn) {
        const int g = gbeg + ig;
        const double x0 = xs_sm[g];
        if constexpr (kQuantX) {
          const uint2* stab = reinterpret_cast<const uint2*>(smem + L.st);
          const uint2 ta = stab[ra * (GC + 1) + g], tb = stab[(ra + 8) * (GC + 1) + g];
          fa = fma(hi_to_f64(ta.y), x0, fma(hi_to_f64(ta.x), i32_to_f64(s0), fa));
          fb = fma(hi_to_f64(tb.y), x0, fma(hi_to_f64(tb.x), i32_to_f64(s2), fb));
        } else {
          fa = fma(h2d(o16[ra * GC + g]), x0, fma(h2d(s16[ra * GC + g]), i32_to_f64(s0), fa));
          fb = fma(h2d(o16[(ra + 8) * GC + g]), x0,
                   fma(h2d(s16[(ra + 8) * GC + g]), i32_to_f64(s2), fb));
        }
      }
    }
  }

  if constexpr (kFold) {
    // ---- partial sums to the CTA that owns the rows, slot (slice, group range)
    const int slot = crank * KW + kw;
    const int owner = (rt * 16) / RO;
    const int lr = rt * 16 - owner * RO + grp;  // ra within the owner's rows
    double* pbase = part + (size_t)slot * M * RO;
    auto put = [&](double* p, double v) {
      if (C > 1)
        st_cluster_f64(mapa_shared(smem_u32(p), (uint32_t)owner), v);
      else
        *p = v;
    };
    if constexpr (kOne) {
      fa += __shfl_xor_sync(0xFFFFFFFFu, fa, 1);
      fb += __shfl_xor_sync(0xFFFFFFFFu, fb, 1);
      fa += __shfl_xor_sync(0xFFFFFFFFu, fa, 2);
      fb += __shfl_xor_sync(0xFFFFFFFFu, fb, 2);
      if (tq == 0) {
        put(pbase + lr, fa);
        put(pbase + lr + 8, fb);
      }
    } else {
#pragma unroll
      for (int tt = 0; tt < TT; ++tt)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int t = tt * 8 + 2 * tq + (q & 1);
          if (t < M) put(pbase + (size_t)t * RO + lr + (q >> 1) * 8, f[tt][q]);
        }
    }
    __syncwarp();
    if (C > 1) {
      cluster_arrive_release();
      cluster_wait_acquire();
    } else {
      __syncthreads();
    }
    // ---- this CTA's rows [crank RO, crank RO + RO): the slots in a fixed
    // order, then sx, bias and one rounding
    const int nslots = C * KW;
    for (int idx = threadIdx.x; idx < M * RO; idx += kThreads) {
      const int t = idx / RO, r = idx - t * RO;
      const int rr = crank * RO + r;
      if (rr >= rows) continue;
      double s = 0.0;
      for (int q = 0; q < nslots; ++q) s += part[((size_t)q * M + t) * RO + r];
      const double v = fma((double)sx_sm[t], s, (double)bias_sm[r]);
      y[(size_t)t * N + n0 + rr] = f64_to_bf16_bits(v);
    }
  }
}

// Tiling of one GEMV call: R weight rows per CTA, C CTAs per cluster along K.
struct GemvPlan {
  int R = 0, C = 0;
  size_t smem = 0;
};

// Picks (R, C) for M <= 16.  A warp covers at most kWarpGroups groups.  In order of preference: a CTA fits two per SM (the
// next call's CTAs can be resident while this call computes); the grid fits
// one wave; at most 16 KB of activations per CTA (they are read after the
// dependency wait, on the critical path); the most CTAs (the most SMs
// streaming weights); the smallest cluster.  quant_x: x is quantized in the kernel, so the K slice
// of the activations must fit the registers too.
bool choose_plan(int64_t M, int64_t K, int64_t N, bool quant_x, GemvPlan* out) {
  if (M < 1 || M > 16 || K % 64 != 0 || K > 65536) return false;
  const int sms = num_sms();
  const int G = (int)(K / 64);
  bool found = false;
  long best[5] = {0, 0, 0, 0, 0};
  for (int C : {1, 2, 4}) {
    if (C > 1 && (G % C != 0 || (G / C) % 8 != 0)) continue;
    for (int R : {32, 64, 128}) {
      if (R / C < 16) continue;
      const GemvLayout L(R, C, (int)K, (int)M, quant_x);
      if (L.total > (size_t)kSmemLimit || L.GW > kWarpGroups) continue;
      if (quant_x && M * L.GC * 64 > (int64_t)kQuantChunks * 8 * kThreads) continue;
      const long grid = (long)C * ((N + R - 1) / R);
      const long one_wave = grid <= sms;
      // activation bytes one CTA reads after the dependency wait, beyond 16 KB
      const long act_excess = -std::max(0L, (long)(M * L.GC * 64) - 16384L);
      const long score[5] = {L.total <= (size_t)kSmemTwoPerSm, one_wave, act_excess,
                             one_wave ? grid : -grid, -C};
      bool better = !found;
      for (int i = 0; i < 5 && !better; ++i) {
        if (score[i] != best[i]) {
          better = score[i] > best[i];
          break;
        }
      }
      if (better) {
        found = true;
        for (int i = 0; i < 5; ++i) best[i] = score[i];
        out->R = R;
        out->C = C;
        out->smem = L.total;
      }
    }
  }
  return found;
}

using GemvKernel = decltype(&w4a8_gemv_kernel<1, true, false, false, 1>);

template <int TT, bool kFold, bool kQuantX, bool kOne>
GemvKernel pick_c(int C) {
  return C == 1 ? w4a8_gemv_kernel<TT, kFold, kQuantX, kOne, 1>
       : C == 2 ? w4a8_gemv_kernel<TT, kFold, kQuantX, kOne, 2>
                : w4a8_gemv_kernel<TT, kFold, kQuantX, kOne, 4>;
}

GemvKernel pick_kernel(int64_t M, bool fold, bool quant_x, int C, int* id) {
  // id: a small index of the instantiation, for the once-per-device attribute
  const int ci = C == 1 ? 0 : C == 2 ? 1 : 2;
  if (!fold) {
    *id = 18 + ci * 2 + (M > 8);
    return M <= 8 ? pick_c<1, false, false, false>(C) : pick_c<2, false, false, false>(C);
  }
  const int v = M == 1 ? 0 : M <= 8 ? 1 : 2;
  *id = (quant_x ? 9 : 0) + ci * 3 + v;
  if (quant_x)
    return v == 0 ? pick_c<1, true, true, true>(C)
         : v == 1 ? pick_c<1, true, true, false>(C) : pick_c<2, true, true, false>(C);
  return v == 0 ? pick_c<1, true, false, true>(C)
       : v == 1 ? pick_c<1, true, false, false>(C) : pick_c<2, true, false, false>(C);
}

constexpr int kKernelIds = 24;
constexpr int kMaxDevices = 64;
bool g_attr_set[kKernelIds][kMaxDevices];

// One launcher for both activation forms: x != nullptr quantizes x in the
// kernel, else xq / sx / xsum come from the caller.
cudaError_t launch_gemv(const uint16_t* x, const int8_t* xq, const float* sx,
                        const int32_t* xsum, int64_t M, int64_t K, const uint8_t* Wp,
                        const uint16_t* ws, const uint16_t* wo, const float* bias, int64_t N,
                        uint16_t* y, int32_t* acc_out, int64_t m0, int64_t m1, bool pdl,
                        cudaStream_t s) {
  const bool fold = acc_out == nullptr;
  const bool qx = x != nullptr;
  if (qx && !fold) return cudaErrorInvalidValue;
  if (gemv1_fits(M, K, N) && (fold || (m0 == 0 && m1 == 1)))
    return launch_w4a8_gemv1(x, xq, sx, xsum, K, Wp, ws, wo, bias, N, y, acc_out, pdl, s);
  GemvPlan p;
  if (!choose_plan(M, K, N, qx, &p)) return cudaErrorInvalidValue;
  const int G = (int)(K / 64), GC = G / p.C;
  // scales / offsets [N, G] fp16 as 2-D boxes of GC groups x R rows (C > 1;
  // one CTA's block is then strided); with C == 1 it is contiguous and goes by
  // bulk copy, and the maps are unused
  CUtensorMap tW, tS = {}, tO = {};
  if (!encode_tmap_2d(&tW, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wp, (uint64_t)(K / 2), (uint64_t)N,
                      (uint64_t)(K / 2), 128, (uint32_t)p.R, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (p.C > 1 && fold) {
    if (!encode_tmap_2d(&tS, CU_TENSOR_MAP_DATA_TYPE_UINT16, ws, (uint64_t)G, (uint64_t)N,
                        (uint64_t)G * 2, (uint32_t)GC, (uint32_t)p.R, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !encode_tmap_2d(&tO, CU_TENSOR_MAP_DATA_TYPE_UINT16, wo, (uint64_t)G, (uint64_t)N,
                        (uint64_t)G * 2, (uint32_t)GC, (uint32_t)p.R, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  }
  int* err = device_error_word();
  if (err == nullptr) return cudaErrorUnknown;
  int id = 0;
  const GemvKernel kernel = pick_kernel(M, fold, qx, p.C, &id);
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= kMaxDevices || !g_attr_set[id][dev]) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemLimit);
    if (e != cudaSuccess) return e;
    if (dev < kMaxDevices) g_attr_set[id][dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.C, (unsigned)((N + p.R - 1) / p.R));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (p.C > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = (unsigned)p.C;
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
  return cudaLaunchKernelEx(&cfg, kernel, tW, tS, tO, x, xq, sx, xsum, (int)M, (int)K, Wp, ws, wo,
                            bias, (int)N, y, acc_out, (int)m0, (int)m1, p.R, 0, err);
}

}  // namespace

size_t gemv_smem_bytes(int64_t M, int64_t K, int64_t N) {
  GemvPlan p;
  return choose_plan(M, K, N, false, &p) ? p.smem : ~size_t(0);
}

// The in-kernel quantization pays off up to 6 tokens: at N = K = 4096
// (graph-chained calls) 4 tokens take 8.4 us quantizing in the kernel against
// 9.8 us as the quantization kernel + the GEMV on its codes, 6 tokens 9.5 us
// both ways, and 8 tokens 9.6 us against 9.1 us.
bool gemv_quant_fits(int64_t M, int64_t K, int64_t N) {
  GemvPlan p;
  return M <= 6 && choose_plan(M, K, N, true, &p);
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
