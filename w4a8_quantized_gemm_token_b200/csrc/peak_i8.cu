// peak_i8.cu -- a probe of the INT8 tensor-pipe throughput of the device: the
// denominator the W8A8 GEMM's roofline fraction is measured against.
//
// The B200 datasheet gives a dense INT8 peak, but the rate a kernel can reach
// depends on the clock the part holds under load (power cap) and on the MMA
// shape.  This kernel issues the same instruction stream as the W8A8 GEMM's
// mainloop -- tcgen05.mma.cta_group::2.kind::i8, M = 256, N = 256, K = 32,
// eight per 256-deep K block, operands read from two 64 KiB shared-memory
// stages through 128-byte-swizzled K-major descriptors, int32 accumulation in
// TMEM -- with nothing else: no global loads, no epilogue.  The operands hold
// a fixed pseudo-random byte pattern (all-zero operands would draw less power
// and so flatter the clock).  One CTA pair per two SMs, persistent.
//
// The host times launches with CUDA events; the op count a launch performs is
// 2 * 256 * 256 * 32 per MMA.  The single wait (for the queued MMAs to drain
// after the last one is issued) is bounded and records QK_ERR_TIMEOUT if it
// gives up; a launch is meant to last milliseconds, and longer measurements
// chain launches.
#include <cuda_runtime.h>

#include <cstdint>

#include "qk_internal.h"
#include "sm100.cuh"

namespace qk {
namespace {

constexpr int kPM = 256;            // MMA rows (both CTAs of the pair)
constexpr int kPN = 256;            // MMA columns
constexpr int kPK = 32;             // K per MMA (bytes)
constexpr int kStageA = 128 * 256;  // one CTA's A rows of a 256-deep K block
constexpr int kStageB = 128 * 256;  // one CTA's B rows
constexpr int kStages = 2;
constexpr int kSmemBytes = kStages * (kStageA + kStageB) + 1024 + 64;
constexpr uint32_t kPeakIdesc = i8_idesc(kPM, kPN, true, true);

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(64, 1)
    int8_peak_kernel(long long iters, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem<1024>(smem_raw);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar = sbase + kStages * (kStageA + kStageB);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kStages * (kStageA + kStageB) + 16);
  const uint32_t rank = cluster_ctarank();
  const int warp = threadIdx.x >> 5;

  // fixed pseudo-random operands (a 32-bit LCG per thread)
  uint32_t* w = reinterpret_cast<uint32_t*>(smem);
  uint32_t h = 0x9E3779B9u * (threadIdx.x + 1u) + 0x7F4A7C15u * (blockIdx.x + 1u);
  for (int i = threadIdx.x; i < kStages * (kStageA + kStageB) / 4; i += blockDim.x) {
    h = h * 1664525u + 1013904223u;
    w[i] = h;
  }
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kPN);
    tmem_relinquish_pair();
  }
  __syncthreads();
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (rank == 0 && threadIdx.x == 0) {
    for (long long it = 0; it < iters; ++it) {
      const int s = (int)(it & 1);
      const uint32_t a = sbase + s * kStageA;
      const uint32_t b = sbase + kStages * kStageA + s * kStageB;
#pragma unroll
      for (int kk = 0; kk < 256 / kPK; ++kk) {
        const uint32_t o = (kk >> 2) * (kStageA / 2) + 32 * (kk & 3);
        mma_i8_pair(tmem, sw128_kmajor_desc(a + o), sw128_kmajor_desc(b + o), kPeakIdesc,
                    (it | kk) != 0 ? 1u : 0u);
      }
    }
    mma_commit_pair(bar, 0x3);
  }
  // Every MMA is issued once the issuing thread reaches this barrier; then
  // both CTAs wait (bounded) for the queue to drain before releasing TMEM.
  __syncwarp();
  cluster_sync();
  if (threadIdx.x == 0) mbar_wait(bar, 0, err);
  __syncthreads();
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, kPN);
}

}  // namespace

double int8_peak_ops_per_iter(int num_pairs) {
  return (double)num_pairs * (256.0 / kPK) * 2.0 * kPM * kPN * kPK;
}

namespace {
bool g_peak_attr_done[64];
}  // namespace

cudaError_t launch_int8_peak(long long iters, int* err, int* pairs_out, cudaStream_t s) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 64) return cudaErrorInvalidDevice;
  if (!g_peak_attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(int8_peak_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    g_peak_attr_done[dev] = true;
  }
  const int pairs = num_sms() / 2;
  *pairs_out = pairs;
  int8_peak_kernel<<<2 * pairs, 64, kSmemBytes, s>>>(iters, err);
  return cudaGetLastError();
}

}  // namespace qk
