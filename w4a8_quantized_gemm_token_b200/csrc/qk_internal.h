// qk_internal.h -- host-side declarations shared by the library's .cu files.
// Not installed; the public ABI is include/qk.h.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "qk.h"

namespace qk {

// ------------------------------------------------------------- launchers
// Each returns cudaSuccess or the launch error.  Arguments are already
// validated by the C-ABI layer (qk_api.cu).

// `pdl`: launch as a programmatic dependent of the previous kernel in the
// stream (the kernel waits for it before reading x or writing xq / sx).
cudaError_t launch_quant_act(const uint16_t* x, int64_t M, int64_t K, int8_t* xq, float* sx,
                             int32_t* xsum, cudaStream_t s, bool pdl = false);

cudaError_t launch_quant_w8(const float* W, int64_t N, int64_t K, int8_t* Wq, float* sw,
                            cudaStream_t s);

cudaError_t launch_quant_w4(const float* W, int64_t N, int64_t K, uint8_t* Wp, uint16_t* ws,
                            uint16_t* wo, cudaStream_t s);

// W8A8 GEMM with the fused dequant + bias epilogue (bf16 out), or the raw int32
// accumulator epilogue when `acc_out` is not null (y, sx, sw, bias ignored).
// `pdl` launches it as a programmatic dependent of the previous kernel.
// With `gate` (fp32 [N]) and `residual` (bf16 [M, N]) the gated residual
// epilogue: y = bf16(residual + gate[n] * (acc * sx * sw + bias)); y may be the
// residual buffer itself (each element is read before it is written, by the
// same thread).
cudaError_t launch_w8a8_gemm(const int8_t* xq, const float* sx, int64_t M, int64_t K,
                             const int8_t* Wq, const float* sw, const float* bias, int64_t N,
                             uint16_t* y, int32_t* acc_out, bool pdl, cudaStream_t s,
                             const float* gate = nullptr, const uint16_t* residual = nullptr);

// The W8A8 linear in one kernel: the GEMM's epilogue warps quantize bf16 x
// (per token, the rule of act_quant.cuh) into xq / sx while the tiles run;
// the producers wait for each row through `ready` (M 8-byte words, each set
// to the launch's epoch when its row is quantized: no clearing needed).  For the shapes
// w8a8_use_fused accepts (every shape not routed to the split-K kernel).
bool w8a8_use_fused(int64_t M, int64_t K, int64_t N);
cudaError_t launch_w8a8_fused(const uint16_t* x, int64_t M, int64_t K, const int8_t* Wq,
                              const float* sw, const float* bias, int64_t N, uint16_t* y,
                              int8_t* xq, float* sx, unsigned long long* ready, bool pdl,
                              cudaStream_t s);

// The same product for thin outputs (N <= 64, see w8a8_use_skinny): 128-row
// tiles split along K over a cluster, exact int32 partial sums reduced through
// distributed shared memory.  launch_w8a8_gemm routes such shapes here.
bool w8a8_use_skinny(int64_t M, int64_t K, int64_t N);

// INT8 attention of BH heads of L tokens (head dim 128): per-token codes and
// scales of q and k ([BH * L, 128] int8, [BH * L] fp32; sk readable for 128
// entries past BH * L), v^T ([BH, 128, L] bf16), out [BH, L, 128] bf16.
cudaError_t launch_sage_attention(const int8_t* qc, const float* sq, const int8_t* kc,
                                  const float* sk, const uint16_t* vt, int64_t BH, int64_t L,
                                  float scale, uint16_t* out, cudaStream_t s);
// v [BH, L, 128] bf16 -> vt [BH, 128, L] bf16.
cudaError_t launch_transpose_v(const uint16_t* v, int64_t BH, int64_t L, uint16_t* vt,
                               cudaStream_t s);

// Test hook: one kernel whose two waits can never complete, each bounded by
// `limit_cycles`; both record QK_ERR_TIMEOUT (debug_wait.cu).
cudaError_t launch_wait_timeout_probe(long long limit_cycles, cudaStream_t s);
cudaError_t launch_w8a8_skinny(const int8_t* xq, const float* sx, int64_t M, int64_t K,
                               const int8_t* Wq, const float* sw, const float* bias, int64_t N,
                               uint16_t* y, int32_t* acc_out, bool pdl, cudaStream_t s,
                               const float* gate = nullptr, const uint16_t* residual = nullptr);

// A value never returned before in this process (56 bits, never zero): the
// epoch of a launch whose device words (readiness, plane count) are tagged
// with it, so that words left by earlier launches never match.
unsigned long long next_epoch();

// W4A8 tensor-core GEMM with the per-group fp64 fold (gemm_w4a8.cu).  When
// `acc_out` is not null it stores the per-group int32 accumulators of rows
// [m0, m1) instead of y.  With `pword`, the kernel computes only when that
// plane-count word (written by launch_w4a8_plane_count with `epoch`) does not
// hold 1..3 planes of this epoch: the fallback beside the byte-plane GEMM.
cudaError_t launch_w4a8_fold(const int8_t* xq, const float* sx, const int32_t* xsum, int64_t M,
                             int64_t K, const uint8_t* Wp, const uint16_t* ws, const uint16_t* wo,
                             const float* bias, int64_t N, uint16_t* y, int32_t* acc_out,
                             int64_t m0, int64_t m1, bool pdl, cudaStream_t s,
                             const unsigned long long* pword = nullptr,
                             unsigned long long epoch = 0);

// The byte-plane W4A8 GEMM (gemm_w4a8_planes.cu).  The plane-count kernel
// writes, into the route's scratch (laid out by w4a8_plane_scratch_bytes),
// e_n and the top-digit slot of every weight row and two words tagged with
// `epoch` (raised within an epoch, replacing any other epoch's word; no
// clearing needed): word 0 = (epoch << 8) | P, word 1 = (epoch << 8) | 1 when
// some half tile has more rows needing a third digit than it has slots.
cudaError_t launch_w4a8_plane_count(const uint16_t* ws, const uint16_t* wo, int64_t N, int64_t K,
                                    void* scratch, unsigned long long epoch, bool pdl,
                                    cudaStream_t s);

// Device scratch the W4A8 GEMM route needs: the plane-count words, e_n and
// the top-digit slot of every weight row, the half-tile counters and the digit
// planes of the dequantized weight (3 N K bytes; none for K = 0, which sizes
// the scratch of the count alone).
size_t w4a8_plane_scratch_bytes(int64_t N, int64_t K);

// The W4A8 GEMM route (any M): the plane count, the plane build, the gated
// per-group fold and the plane GEMM -- four launches, one of the two GEMMs
// computing.  `scratch`: w4a8_plane_scratch_bytes(N, K) bytes of device memory
// owned by the call (256-byte aligned).
cudaError_t launch_w4a8_gemm(const int8_t* xq, const float* sx, const int32_t* xsum, int64_t M,
                             int64_t K, const uint8_t* Wp, const uint16_t* ws, const uint16_t* wo,
                             const float* bias, int64_t N, uint16_t* y, void* scratch, bool pdl,
                             cudaStream_t s);

// The prepared form of a weight for the GEMM route (the layout of
// w4a8_plane_scratch_bytes(N, K)): the count and build once, with a fixed
// epoch, after zeroing the words.  With `planes` non-null, synchronizes `s`
// and writes the plane count (1..3, or 255: the per-group fold computes).
cudaError_t launch_w4a8_prepare(const uint8_t* Wp, const uint16_t* ws, const uint16_t* wo,
                                int64_t N, int64_t K, void* prepared, int* planes,
                                cudaStream_t s);

// The GEMM route on a prepared weight: the gated per-group fold and the plane
// GEMM (two launches).
cudaError_t launch_w4a8_gemm_prepared(const int8_t* xq, const float* sx, const int32_t* xsum,
                                      int64_t M, int64_t K, const uint8_t* Wp,
                                      const uint16_t* ws, const uint16_t* wo,
                                      const void* prepared, const float* bias, int64_t N,
                                      uint16_t* y, bool pdl, cudaStream_t s);

// W4A8 weight-streaming GEMV (M <= 16; its per-CTA working set -- the weight
// slice of R rows x one K slice, xq, scales -- must fit shared memory, see
// gemv_fits); per-group accumulator dump as above.
size_t gemv_smem_bytes(int64_t M, int64_t K, int64_t N);
inline bool gemv_fits(int64_t M, int64_t K, int64_t N) {
  return M <= 16 && gemv_smem_bytes(M, K, N) <= 227u * 1024u;
}
// The same GEMV quantizing bf16 x itself (each CTA's K slice of x must fit its
// registers, see gemv_quant_fits): the activation-quant kernel and its launch
// drop out of the small-M linear.
bool gemv_quant_fits(int64_t M, int64_t K, int64_t N);
cudaError_t launch_w4a8_gemv_quant(const uint16_t* x, int64_t M, int64_t K, const uint8_t* Wp,
                                   const uint16_t* ws, const uint16_t* wo, const float* bias,
                                   int64_t N, uint16_t* y, bool pdl, cudaStream_t s);
// One token (M = 1, K a multiple of 1024 up to 4096): a dp4a kernel that keeps
// every lane busy; launch_w4a8_gemv / launch_w4a8_gemv_quant route such shapes
// here.  x != nullptr quantizes x in the kernel; acc_out dumps the group sums.
bool gemv1_fits(int64_t M, int64_t K, int64_t N);
cudaError_t launch_w4a8_gemv1(const uint16_t* x, const int8_t* xq, const float* sx,
                              const int32_t* xsum, int64_t K, const uint8_t* Wp,
                              const uint16_t* ws, const uint16_t* wo, const float* bias, int64_t N,
                              uint16_t* y, int32_t* acc_out, bool pdl, cudaStream_t s);
cudaError_t launch_w4a8_gemv(const int8_t* xq, const float* sx, const int32_t* xsum, int64_t M,
                             int64_t K, const uint8_t* Wp, const uint16_t* ws, const uint16_t* wo,
                             const float* bias, int64_t N, uint16_t* y, int32_t* acc_out,
                             int64_t m0, int64_t m1, bool pdl, cudaStream_t s);

// QK_OK if the current device is an sm_100 device (the answer is cached per
// device after the first query), else QK_ERR_NO_DEVICE.
qk_status check_device();

// The INT8 tensor-pipe probe (peak_i8.cu): one pair of CTAs per two SMs,
// each pair issuing `iters` x 8 tcgen05 kind::i8 MMAs of 256 x 256 x 32.
// *pairs_out receives the number of pairs launched.
cudaError_t launch_int8_peak(long long iters, int* err, int* pairs_out, cudaStream_t s);
double int8_peak_ops_per_iter(int num_pairs);

// Address of this device's error word (a __device__ int of the library),
// resolved once per device with cudaGetSymbolAddress; null on failure.
int* device_error_word();

// Number of SMs of the current device (cached per device).
int num_sms();

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda
// link dependency).  Returns false if the driver call is unavailable or fails.
bool encode_tmap_2d(CUtensorMap* out, CUtensorMapDataType dtype, const void* base,
                    uint64_t inner, uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner,
                    uint32_t box_rows, CUtensorMapSwizzle swizzle);

}  // namespace qk
