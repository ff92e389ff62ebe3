// gemm_w4a8.cu -- the W4A8 tensor-core GEMM with the per-group fold.
//
// Computes ("qlip-mlx" README, "w4a8_linear / W4A8Linear": packed 4-bit
// weights, the same int8 compute; "MLX PR #4722": affine 4-bit weights with
// group size 64 staged as int8 for the matmul), with G = K / 64,
//   acc[m, n, g] = sum_{k in group g} xq[m, k] * q[n, k]          (exact int32)
//   y[m, n] = bf16( sx[m] * sum_g (s[n,g] * acc + o[n,g] * xsum[m,g]) + bias[n] )
// with the fold in fp64 and one rounding to bf16.
//
// The byte-plane GEMM (gemm_w4a8_planes.cu) computes the same value several
// times faster whenever the scales and offsets of every weight row fit a common
// integer grid within three bytes; this kernel runs beside it for the products
// that do not (it then does the work, gated by the same plane-count word), when
// the per-group fold is asked for explicitly, and for the per-group int32 dump.
//
// The per-group rescaling makes this kernel bound by the fp64 fold (M N G
// multiply-add pairs on the CUDA cores), not by the tensor cores, so the tile is
// chosen for the fold: 128 x 128 outputs per CTA (one CTA per SM, persistent).
//  * warp 0: TMA producer -- per K block of 128 (two groups) the 128 x 128 int8
//    tile of xq (128-byte swizzle) and the 128 x 64-byte packed-nibble tile of
//    Wp, into a 4-stage ring;
//  * warps 2-3: unpack -- expand the nibbles into a 128 x 128 u8 code tile in
//    the swizzled K-major layout the MMA reads (then fence.proxy.async), and
//    convert the block's fp16 scales, offsets and xsum to fp64 into a table ring;
//  * warp 1: per group, two tcgen05.mma kind::i8 (A signed, B unsigned, M = 128,
//    N = 128, K = 32) into one of four 128-column TMEM buffers;
//  * warps 4-11: fold -- tcgen05.ld a group's int32 sums, f += s * acc + o * xsum
//    in fp64 (exact int -> fp64 by the 2^52 magic number), one row and 64
//    columns per thread (two warps per TMEM lane quarter);
//    at the end of the tile y = sx * f + bias is rounded once to bf16 (integer
//    operations on the double's bits) and written with a TMA store.
// A debug mode stores the per-group int32 sums of rows [m0, m1) instead.
// Every mbarrier wait is bounded (sm100.cuh).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "qk_internal.h"
#include "sm100.cuh"

namespace qk {
namespace {

constexpr int BM = 128;                   // rows (TMEM lanes)
constexpr int BN = 128;                   // output columns per tile
constexpr int BK = 128;                   // K per stage: two groups of 64
constexpr int STAGES = 4;
constexpr int UBUFS = 2;                  // unpacked code tiles
constexpr int TSLOTS = 4;                 // scale/offset table slots (one per K block)
constexpr int TBUFS = 4;                  // TMEM group accumulators
constexpr int kUnpackWarps = 2;
constexpr int kFoldWarps = 8;             // two per TMEM lane quarter
constexpr int kFoldCols = BN / (kFoldWarps / 4);  // columns per fold thread
constexpr int kHalf = kFoldCols / 2;              // TMEM columns loaded at a time
constexpr int kThreads = 32 * (2 + kUnpackWarps + kFoldWarps);  // 384: three warpgroups
// Registers: the block is launched with kRegsLaunch per thread; warpgroup 0
// (producer, MMA issuer, unpack) keeps kRegsCtl and hands the rest to the two
// fold warpgroups, whose threads hold 64 fp64 sums each.
constexpr int kRegsLaunch = 168;
constexpr int kRegsCtl = 56;
constexpr int kRegsFold = 224;
static_assert(2 + kUnpackWarps == 4, "warpgroup 0 holds every non-fold warp");
static_assert(128 * kRegsCtl + 32 * kFoldWarps * kRegsFold <= kThreads * kRegsLaunch,
              "register split exceeds the launch allocation");
constexpr int A_BYTES = BM * BK;          // 16 KiB
constexpr int P_BYTES = BN * (BK / 2);    // 4 KiB of packed nibbles
constexpr int U_BYTES = BN * BK;          // 8 KiB of unpacked codes
// table slot: two groups x 64 columns x {s, o} fp64, then two groups x 128
// rows of xsum as fp64
constexpr int T_SO = 2 * BN * 16;
constexpr int T_BYTES = T_SO + 2 * BM * 8;
constexpr int STG_BYTES = 32 * 2 * kFoldCols;  // 32 rows x kFoldCols bf16 (128-byte swizzle)
constexpr int SMEM_A = 0;
constexpr int SMEM_P = SMEM_A + STAGES * A_BYTES;
constexpr int SMEM_U = SMEM_P + STAGES * P_BYTES;
constexpr int SMEM_T = SMEM_U + UBUFS * U_BYTES;
constexpr int SMEM_STG = SMEM_T + TSLOTS * T_BYTES;
constexpr int SMEM_BAR = SMEM_STG + kFoldWarps * STG_BYTES;
constexpr int kNumBars = 2 * STAGES + 2 * UBUFS + 2 * TSLOTS + 2 * TBUFS;
constexpr int SMEM_SLOT = SMEM_BAR + kNumBars * 8;
constexpr int SMEM_ALLOC = SMEM_SLOT + 16 + 1024;
constexpr int kTmemCols = TBUFS * BN;     // 256
constexpr uint32_t kIdesc = i8_idesc(BM, BN, true, false);


static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
static_assert(SMEM_U % 1024 == 0 && U_BYTES % 1024 == 0, "swizzled tiles need 1024-byte alignment");
static_assert(2 * kFoldCols == 128, "the output stage is 128-byte rows with the 128-byte swizzle");
static_assert(SMEM_STG % 1024 == 0 && STG_BYTES % 1024 == 0, "swizzled output stages too");

__device__ __forceinline__ double i32_to_f64(uint32_t a) {
  return __hiloint2double(0x43300000, (int)(a ^ 0x80000000u)) - 4503601774854144.0;
}

// fp64 -> bf16 bits, one rounding to nearest-even (see gemm_w8a8.cu).
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

// 32 lanes x 16 or 32 consecutive TMEM columns.
__device__ __forceinline__ void tmem_ld_cols(uint32_t a, uint32_t (&v)[32]) { tmem_ld32(a, v); }
__device__ __forceinline__ void tmem_ld_cols(uint32_t a, uint32_t (&v)[16]) { tmem_ld16(a, v); }

// 8 packed codes (c0 = low nibble of byte 0) -> two words of 4 u8 codes.
__device__ __forceinline__ void unpack8(uint32_t w, uint32_t& lo4, uint32_t& hi4) {
  const uint32_t even = w & 0x0F0F0F0Fu;
  const uint32_t odd = (w >> 4) & 0x0F0F0F0Fu;
  lo4 = __byte_perm(even, odd, 0x5140);
  hi4 = __byte_perm(even, odd, 0x7362);
}

template <bool kAccOut>
__global__ void __launch_bounds__(kThreads, 1)
    w4a8_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmP,
                     const __grid_constant__ CUtensorMap tmY, const float* __restrict__ sx,
                     const int32_t* __restrict__ xsum, const uint16_t* __restrict__ wscale,
                     const uint16_t* __restrict__ woffset, const float* __restrict__ bias, int M,
                     int N, int K, int32_t* __restrict__ acc_out, int m0, int m1, int* err,
                     const unsigned long long* pword, unsigned long long epoch) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem<1024>(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + SMEM_BAR;
  auto full_bar = [&](int i) { return bar0 + 8u * i; };
  auto empty_bar = [&](int i) { return bar0 + 8u * (STAGES + i); };
  auto ufull_bar = [&](int i) { return bar0 + 8u * (2 * STAGES + i); };
  auto uempty_bar = [&](int i) { return bar0 + 8u * (2 * STAGES + UBUFS + i); };
  auto tabfull_bar = [&](int i) { return bar0 + 8u * (2 * STAGES + 2 * UBUFS + i); };
  auto tabempty_bar = [&](int i) { return bar0 + 8u * (2 * STAGES + 2 * UBUFS + TSLOTS + i); };
  auto tfull_bar = [&](int i) { return bar0 + 8u * (2 * STAGES + 2 * UBUFS + 2 * TSLOTS + i); };
  auto tempty_bar = [&](int i) {
    return bar0 + 8u * (2 * STAGES + 2 * UBUFS + 2 * TSLOTS + TBUFS + i);
  };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SMEM_SLOT);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = K >> 6;
  const int num_kb = (G + 1) >> 1;
  const int tiles_m = (M + BM - 1) / BM;
  const int tiles_n = (N + BN - 1) / BN;
  const int num_tiles = tiles_m * tiles_n;

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmP);
    if (!kAccOut) prefetch_tmap(&tmY);
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(full_bar(i), 1);
      mbar_init(empty_bar(i), 1);
    }
    for (int i = 0; i < UBUFS; ++i) {
      mbar_init(ufull_bar(i), kUnpackWarps);
      mbar_init(uempty_bar(i), 1);
    }
    for (int i = 0; i < TSLOTS; ++i) {
      mbar_init(tabfull_bar(i), kUnpackWarps);
      mbar_init(tabempty_bar(i), kFoldWarps);
    }
    for (int i = 0; i < TBUFS; ++i) {
      mbar_init(tfull_bar(i), 1);
      mbar_init(tempty_bar(i), kFoldWarps);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // The next kernel in the stream may become resident now (it waits for this
  // grid to finish before it touches anything this grid reads or writes).
  pdl_launch_dependents();
  pdl_wait();  // xq, sx and xsum come from the activation-quant kernel

  // Beside the byte-plane GEMM (gemm_w4a8_planes.cu) this kernel computes only
  // the products that one cannot: a plane-count word of this launch's epoch
  // holding 1..3 planes means the plane kernel takes the product.
  bool skip = false;
  if (pword != nullptr) {
    const unsigned long long pw = *reinterpret_cast<const volatile unsigned long long*>(pword);
    const unsigned long long p = pw & 0xFFull;
    skip = (pw >> 8) == epoch && p >= 1 && p <= 3;
  }

  if (skip) {
    // nothing to compute
  } else if (warp < 4) {
    // warpgroup 0: warp 0 loads, warp 1 issues the MMAs, warps 2-3 unpack;
    // most of its registers go to the fold warpgroups
    regs_dec<kRegsCtl>();
    if (warp == 0) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        int it = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
          const int mb = t % tiles_m, nb = t / tiles_m;
          for (int kb = 0; kb < num_kb; ++kb, ++it) {
            const int s = it % STAGES;
            if (!mbar_wait(empty_bar(s), ((it / STAGES) & 1) ^ 1u, err)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(full_bar(s), A_BYTES + P_BYTES);
            tma_load_2d(sbase + SMEM_A + s * A_BYTES, &tmA, kb * BK, mb * BM, full_bar(s));
            tma_load_2d(sbase + SMEM_P + s * P_BYTES, &tmP, kb * (BK / 2), nb * BN, full_bar(s));
          }
        }
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------- MMA issuer
      if (lane == 0) {
        int it = 0, gc = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
          for (int kb = 0; kb < num_kb && ok; ++kb, ++it) {
            const int s = it % STAGES, u = it % UBUFS;
            ok = mbar_wait(ufull_bar(u), (it / UBUFS) & 1, err) &&
                 mbar_wait(full_bar(s), (it / STAGES) & 1, err);
            if (!ok) break;
            tc_fence_after();
            const uint32_t a_addr = sbase + SMEM_A + s * A_BYTES;
            const uint32_t b_addr = sbase + SMEM_U + u * U_BYTES;
            for (int j = 0; j < 2 && 2 * kb + j < G; ++j, ++gc) {
              const int b = gc % TBUFS;
              if (!mbar_wait(tempty_bar(b), ((gc / TBUFS) & 1) ^ 1u, err)) {
                ok = false;
                break;
              }
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < 2; ++kk)
                mma_i8(tmem_base + (uint32_t)(b * BN), sw128_kmajor_desc(a_addr + 64 * j + 32 * kk),
                       sw128_kmajor_desc(b_addr + 64 * j + 32 * kk), kIdesc, kk);
              mma_commit(tfull_bar(b));  // this group's sums are ready
            }
            mma_commit(empty_bar(s));   // xq and packed tiles free
            mma_commit(uempty_bar(u));  // unpacked tile free
          }
        }
      }
    } else {
      // -------------------------------------------------------------- unpack
      const int r = threadIdx.x - 64;  // tile rows (output columns) r and r + 64
      // scales / offsets of K block (tile t, block kb) for these rows, fetched
      // one block ahead so their global-load latency overlaps the current block;
      // v[4 i + 2 j + {0, 1}] = {s, o} of row r + 64 i, group 2 kb + j
      auto fetch_so = [&](int t, int kb, uint16_t (&v)[8]) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int n = (t / tiles_m) * BN + r + 64 * i;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int g = 2 * kb + j;
            const bool in = t < num_tiles && n < N && g < G;
            v[4 * i + 2 * j] = in ? __ldg(wscale + (size_t)n * G + g) : (uint16_t)0;
            v[4 * i + 2 * j + 1] = in ? __ldg(woffset + (size_t)n * G + g) : (uint16_t)0;
          }
        }
      };
      // xsum of K block (tile t, block kb) for rows r and r + 64 of the tile
      auto fetch_xs = [&](int t, int kb, int (&v)[4]) {
        const int mrow = (t % tiles_m) * BM + r;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int m = mrow + 64 * (i >> 1), g = 2 * kb + (i & 1);
          v[i] = (t < num_tiles && m < M && g < G) ? __ldg(xsum + (size_t)m * G + g) : 0;
        }
      };
      uint16_t so_next[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      int xs_next[4] = {0, 0, 0, 0};
      if (!kAccOut) {
        fetch_so(blockIdx.x, 0, so_next);
        fetch_xs(blockIdx.x, 0, xs_next);
      }
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        for (int kb = 0; kb < num_kb; ++kb, ++it) {
          const int s = it % STAGES, u = it % UBUFS, ts = it % TSLOTS;
          uint16_t so_cur[8];
          int xs_cur[4];
#pragma unroll
          for (int i = 0; i < 8; ++i) so_cur[i] = so_next[i];
#pragma unroll
          for (int i = 0; i < 4; ++i) xs_cur[i] = xs_next[i];
          if (!kAccOut) {
            const bool last = kb + 1 == num_kb;
            fetch_so(last ? t + (int)gridDim.x : t, last ? 0 : kb + 1, so_next);
            fetch_xs(last ? t + (int)gridDim.x : t, last ? 0 : kb + 1, xs_next);
          }
          ok = mbar_wait(full_bar(s), (it / STAGES) & 1, err) &&
               mbar_wait(uempty_bar(u), ((it / UBUFS) & 1) ^ 1u, err);
          if (!ok) break;
          // 64 packed bytes of a row -> 128 u8 codes, 128-byte-swizzled row
#pragma unroll
          for (int rr = r; rr < BN; rr += 64) {
            const uint4* src =
                reinterpret_cast<const uint4*>(smem + SMEM_P + s * P_BYTES + rr * 64);
            uint8_t* dst = smem + SMEM_U + u * U_BYTES + rr * 128;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint4 w = src[i];  // codes 32i .. 32i + 31
              uint4 c0, c1;
              unpack8(w.x, c0.x, c0.y);
              unpack8(w.y, c0.z, c0.w);
              unpack8(w.z, c1.x, c1.y);
              unpack8(w.w, c1.z, c1.w);
              *reinterpret_cast<uint4*>(dst + (((2 * i) ^ (rr & 7)) * 16)) = c0;
              *reinterpret_cast<uint4*>(dst + (((2 * i + 1) ^ (rr & 7)) * 16)) = c1;
            }
          }
          fence_proxy_async_smem();  // generic writes -> tensor-core reads
          __syncwarp();
          if (lane == 0) mbar_arrive(ufull_bar(u));
          // this K block's scales and offsets in fp64, for the fold warps
          if (!kAccOut) {
            if (!mbar_wait(tabempty_bar(ts), ((it / TSLOTS) & 1) ^ 1u, err)) {
              ok = false;
              break;
            }
            double2* tab = reinterpret_cast<double2*>(smem + SMEM_T + ts * T_BYTES);
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
              for (int j = 0; j < 2; ++j)
                tab[j * BN + r + 64 * i] = make_double2(
                    (double)__half2float(__ushort_as_half(so_cur[4 * i + 2 * j])),
                    (double)__half2float(__ushort_as_half(so_cur[4 * i + 2 * j + 1])));
            double* xs_tab = reinterpret_cast<double*>(smem + SMEM_T + ts * T_BYTES + T_SO);
#pragma unroll
            for (int i = 0; i < 4; ++i)  // [group][row]
              xs_tab[(i & 1) * BM + r + 64 * (i >> 1)] = i32_to_f64((uint32_t)xs_cur[i]);
            __syncwarp();
            if (lane == 0) mbar_arrive(tabfull_bar(ts));
          }
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- fold
    regs_inc<kRegsFold>();
    const int fw = warp - (2 + kUnpackWarps);  // 0..7
    const int q = warp & 3;                     // TMEM lane quarter
    const int cpart = fw >> 2;                  // columns [kFoldCols cpart, + kFoldCols)
    uint8_t* stg_ptr = smem + SMEM_STG + fw * STG_BYTES;
    const uint32_t stg = sbase + SMEM_STG + (uint32_t)(fw * STG_BYTES);
    int it = 0, gc = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
      const int mb = t % tiles_m, nb = t / tiles_m;
      const int row0 = mb * BM + q * 32;
      const int row = row0 + lane;
      const int n0 = nb * BN + cpart * kFoldCols;
      const uint32_t t_lane =
          tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(cpart * kFoldCols);
      double f[kFoldCols];
#pragma unroll
      for (int c = 0; c < kFoldCols; ++c) f[c] = 0.0;

      for (int kb = 0; kb < num_kb && ok; ++kb, ++it) {
        const int ts = it % TSLOTS;
        if (!kAccOut && !mbar_wait(tabfull_bar(ts), (it / TSLOTS) & 1, err)) {
          ok = false;
          break;
        }
        const double2* tab = reinterpret_cast<const double2*>(smem + SMEM_T + ts * T_BYTES);
        for (int j = 0; j < 2 && 2 * kb + j < G; ++j, ++gc) {
          const int g = 2 * kb + j;
          const int b = gc % TBUFS;
          const double xs = kAccOut ? 0.0
                                    : reinterpret_cast<const double*>(
                                          smem + SMEM_T + ts * T_BYTES + T_SO)[j * BM + q * 32 + lane];
          if (!mbar_wait(tfull_bar(b), (gc / TBUFS) & 1, err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const double2* tj = tab + j * BN + cpart * kFoldCols;
          // two halves keep the live registers down; the buffer goes back to
          // the MMA issuer once the second half is loaded
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t v[kHalf];
            tmem_ld_cols(t_lane + (uint32_t)(b * BN + kHalf * h), v);
            tmem_ld_wait();
            if (h == 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(tempty_bar(b));
            }
            if constexpr (kAccOut) {
              if (row >= m0 && row < m1) {
#pragma unroll
                for (int c = 0; c < kHalf; ++c) {
                  const int n = n0 + kHalf * h + c;
                  if (n < N) acc_out[((size_t)(row - m0) * N + n) * G + g] = (int32_t)v[c];
                }
              }
            } else {
#pragma unroll
              for (int c = 0; c < kHalf; ++c) {
                const double2 so = tj[kHalf * h + c];
                f[kHalf * h + c] = fma(so.y, xs, fma(so.x, i32_to_f64(v[c]), f[kHalf * h + c]));
              }
            }
          }
        }
        if (!kAccOut) {
          __syncwarp();
          if (lane == 0) mbar_arrive(tabempty_bar(ts));
        }
      }
      if (kAccOut || !ok) continue;
      // ---- tile output: y = bf16(sx * f + bias), staged and TMA-stored
      if (row0 >= M || n0 >= N) continue;
      const double sxd = row < M ? (double)__ldg(sx + row) : 0.0;
      uint32_t out[kFoldCols / 2];
#pragma unroll
      for (int c = 0; c < kFoldCols; c += 2) {
        const int n = n0 + c;
        const double b0 = (bias != nullptr && n < N) ? (double)__ldg(bias + n) : 0.0;
        const double b1 = (bias != nullptr && n + 1 < N) ? (double)__ldg(bias + n + 1) : 0.0;
        out[c >> 1] = f64_to_bf16_bits(fma(sxd, f[c], b0)) |
                      (f64_to_bf16_bits(fma(sxd, f[c + 1], b1)) << 16);
      }
      if (lane == 0) bulk_wait_read<0>();
      __syncwarp();
      uint8_t* rowp = stg_ptr + lane * 2 * kFoldCols;  // 128-byte rows, 128-byte swizzle
#pragma unroll
      for (int i = 0; i < kFoldCols / 8; ++i)
        *reinterpret_cast<uint4*>(rowp + 16 * (i ^ (lane & 7))) =
            make_uint4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(&tmY, stg, n0, row0);
        bulk_commit();
      }
    }
    if (lane == 0) bulk_wait<0>();
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

bool g_attr_done[2][64];

}  // namespace

cudaError_t launch_w4a8_fold(const int8_t* xq, const float* sx, const int32_t* xsum, int64_t M,
                             int64_t K, const uint8_t* Wp, const uint16_t* ws, const uint16_t* wo,
                             const float* bias, int64_t N, uint16_t* y, int32_t* acc_out,
                             int64_t m0, int64_t m1, bool pdl, cudaStream_t s,
                             const unsigned long long* pword, unsigned long long epoch) {
  const bool acc_mode = acc_out != nullptr;
  CUtensorMap tA, tP, tY;
  if (!encode_tmap_2d(&tA, CU_TENSOR_MAP_DATA_TYPE_UINT8, xq, (uint64_t)K, (uint64_t)M,
                      (uint64_t)K, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tP, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wp, (uint64_t)(K / 2), (uint64_t)N,
                      (uint64_t)(K / 2), BK / 2, BN, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  if (acc_mode)
    tY = tA;  // unused by the accumulator dump
  else if (!encode_tmap_2d(&tY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, (uint64_t)N, (uint64_t)M,
                           (uint64_t)N * 2, kFoldCols, 32, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  int dev = 0;
  cudaGetDevice(&dev);
  auto kernel = acc_mode ? w4a8_gemm_kernel<true> : w4a8_gemm_kernel<false>;
  if (dev < 64 && !g_attr_done[acc_mode][dev]) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    // the fold warpgroups' register increase is only satisfiable with the
    // launch allocation the split was computed for
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, kernel)) != cudaSuccess) return e;
    if (fa.numRegs != kRegsLaunch) return cudaErrorInvalidKernelImage;
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
  return cudaLaunchKernelEx(&cfg, kernel, tA, tP, tY, sx, xsum, ws, wo, bias, (int)M, (int)N,
                            (int)K, acc_out, (int)m0, (int)m1, err, pword, epoch);
}

}  // namespace qk
