/*
 * qk.h -- C ABI of libqk, the B200 (sm_100a) W8A8 / W4A8 quantized linear.
 *
 * What it computes (by page and section of the sources):
 *   - "qlip-mlx" README, intro bullet "w8a8_linear / W8A8Linear": a linear
 *     layer whose activations are quantized per token to int8 on the fly, whose
 *     weights are quantized offline to int8, an INT8 x INT8 -> INT32 matmul,
 *     and a dequant + bias step fused behind it.
 *   - same page, "Quick start" -> "Use it from Python": quantize_weight_int8
 *     turns an [N, K] weight into int8 codes plus fp32 per-output-channel
 *     scales; w8a8_linear(x, w_i8, sw, bias) runs the layer.
 *   - same page, intro bullet "w4a8_linear / W4A8Linear": the same int8 compute
 *     with the weight stored as packed 4-bit codes, and a separate path for
 *     M <= 16 rows that runs at weight-bandwidth speed.
 *   - "MLX PR #4722" (int8-staged quantized matmul), "Selector rules": affine
 *     4-bit weights with group size 64 along K, K % 64 == 0, K <= 65536.
 *
 * Conventions for every call:
 *   - Matrices are row-major.  x is [M, K] (M tokens, K in-features), a weight
 *     is [N, K] (N out-features; the nn.Linear orientation), y is [M, N].
 *   - bf16 and fp16 values are passed as their 16-bit patterns (uint16_t).
 *   - Every pointer is DEVICE memory on the current CUDA device, owned by the
 *     caller.  The library keeps no pointer after a call returns.
 *   - Calls are asynchronous and ordered on `stream` (NULL = the legacy
 *     default stream).  They are deterministic: the same inputs give the same
 *     bits.  The caller must not modify inputs or read outputs until the stream
 *     has reached the call.
 *   - Arguments are checked on the host before anything is launched; a failed
 *     check returns an error code and leaves every output untouched.  A launch
 *     failure returns QK_ERR_CUDA.  Kernels never trap: a kernel wait that
 *     gives up records QK_ERR_TIMEOUT in a per-device error word, read by
 *     qk_check_device_error.
 *   - Inputs must be finite.  Activation rows whose absmax lies in (0, 2^-121)
 *     are outside the contract (127 / absmax overflows fp32).
 *   - Pointer alignment: matrices (x, xq, Wq, Wp, wscale, woffset, xsum, y) and
 *     the workspace need 16-byte alignment; sx, sw and bias need 16 bytes too
 *     (the kernels read them as 16-byte vectors).
 */
#ifndef QK_H
#define QK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t (a CUDA stream handle); NULL is the legacy stream. */
typedef struct CUstream_st *qk_stream_t;

typedef enum {
    QK_OK = 0,
    QK_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad route    */
    QK_ERR_UNSUPPORTED_SHAPE = 2, /* K or N outside the shape contract         */
    QK_ERR_MISALIGNED = 3,        /* a pointer breaks the alignment rule       */
    QK_ERR_NO_DEVICE = 4,         /* no CUDA device, or it is not sm_100       */
    QK_ERR_WORKSPACE = 5,         /* workspace too small or misaligned         */
    QK_ERR_CUDA = 6,              /* a CUDA runtime call or launch failed      */
    QK_ERR_TIMEOUT = 7            /* a kernel wait gave up (device error word) */
} qk_status;

/* Routes of the W4A8 product. */
typedef enum {
    QK_ROUTE_AUTO = 0,     /* GEMV when M <= 16 and it fits, else GEMM          */
    QK_ROUTE_GEMM = 1,     /* tensor-core GEMM (tcgen05), any M: byte planes,   */
                           /* or the per-group fold where planes cannot serve   */
    QK_ROUTE_GEMV = 2,     /* weight-streaming GEMV, M <= 16 only              */
    QK_ROUTE_GEMM_FOLD = 3 /* tensor-core GEMM with the per-group fold, any M  */
} qk_route;

/* Static string for a status code (never NULL). */
const char *qk_status_string(int status);

/* Library ABI version, (major << 16) | minor. */
int qk_version(void);

/* 1 if `device` exists and is compute capability 10.0 (B200, sm_100a), else 0.
 * Never fails: a missing driver or device gives 0.  (The qlip-mlx README,
 * "Key features": is_available() reports False where the INT8 path cannot run.) */
int qk_is_available(int device);

/*
 * Shape contract (qk_w8a8_*): 32 <= K <= 65536 with K % 32 == 0; N >= 8 with
 * N % 8 == 0; M >= 0 (M == 0 returns QK_OK and launches nothing).
 * W4A8 (qk_w4a8_*, qk_quantize_weights_int4): additionally K % 64 == 0.
 * A shape outside the contract returns QK_ERR_UNSUPPORTED_SHAPE.
 */

/* ------------------------------------------------------------- workspace */

/* Bytes of workspace qk_w8a8_linear (and qk_w8a8_linear_fused) needs: int8
 * codes [M, K], fp32 scales [M] and one 8-byte readiness word per row (used
 * by qk_w8a8_linear_fused), each 256-byte aligned inside the block. */
size_t qk_w8a8_workspace_size(int64_t M, int64_t K);

/* Bytes of workspace qk_w4a8_linear needs: codes [M, K], scales [M] and int32
 * group sums [M, K/64], each 256-byte aligned inside the block.  (The GEMM
 * route's byte planes of the weight, up to 3 N K bytes, are allocated
 * stream-ordered by the call itself: see qk_w4a8_linear.) */
size_t qk_w4a8_workspace_size(int64_t M, int64_t K);

/* ------------------------------------------------------ offline weights */

/*
 * W8 weight quantization ("qlip-mlx" README, "Use it from Python":
 * quantize_weight_int8, [N, K] -> int8 + fp32 scales).  Per output channel n:
 * sw[n] = absmax_k |W[n,k]| / 127 and Wq[n,k] = round-half-even(W[n,k] *
 * (127 / absmax)) clamped to [-127, 127]; an all-zero row gets sw = 1 and zero
 * codes.  All arithmetic is IEEE fp32.
 *   W  : fp32 [N, K]          (in)
 *   Wq : int8 [N, K]          (out)
 *   sw : fp32 [N]             (out)
 */
qk_status qk_quantize_weights_int8(const float *W, int64_t N, int64_t K,
                                   int8_t *Wq, float *sw, qk_stream_t stream);

/*
 * W4 affine group-64 quantization ("qlip-mlx" README, "w4a8_linear"; "MLX PR
 * #4722", "Selector rules").  Per row n and group g of 64 consecutive k: lo =
 * min, hi = max, wscale = fp16((hi - lo) / 15), woffset = fp16(lo); codes
 * q = round-half-even((W - float(woffset)) * (1 / float(wscale))) clamped to
 * [0, 15] (all zero when wscale == 0).  The dequantized weight is
 * q * wscale + woffset.  Two codes per byte: k = 2j in the low nibble of byte
 * j, k = 2j + 1 in the high nibble.  |W| must stay below 65504 (fp16 range).
 *   W       : fp32 [N, K]                (in)
 *   Wp      : uint8 [N, K/2]             (out)
 *   wscale  : fp16 bits [N, K/64]        (out)
 *   woffset : fp16 bits [N, K/64]        (out)
 */
qk_status qk_quantize_weights_int4(const float *W, int64_t N, int64_t K,
                                   uint8_t *Wp, uint16_t *wscale, uint16_t *woffset,
                                   qk_stream_t stream);

/* ----------------------------------------------------- activation quant */

/*
 * Per-token dynamic symmetric int8 quantization ("qlip-mlx" README,
 * "w8a8_linear": activations quantized dynamically, no calibration; "MLX PR
 * #4722", "SIMD fix": x quantized by a kernel of its own).  Per row m:
 * sx[m] = absmax / 127, xq = round-half-even(x * (127 / absmax)) clamped to
 * [-127, 127] (fp32 arithmetic); an all-zero row gets sx = 1, codes 0.
 * If xsum is not NULL (needs K % 64 == 0) it also writes the int32 sums of the
 * codes over each group of 64: xsum[m, g] = sum_{k = 64g}^{64g+63} xq[m, k].
 *   x    : bf16 bits [M, K]  (in)
 *   xq   : int8 [M, K]       (out)
 *   sx   : fp32 [M]          (out)
 *   xsum : int32 [M, K/64]   (out, nullable)
 */
qk_status qk_quantize_activations(const uint16_t *x, int64_t M, int64_t K,
                                  int8_t *xq, float *sx, int32_t *xsum,
                                  qk_stream_t stream);

/* ------------------------------------------------------------ W8A8 linear */

/*
 * The W8A8 linear ("qlip-mlx" README, "w8a8_linear / W8A8Linear"):
 *   y[m, n] = bf16( acc[m, n] * sx[m] * sw[n] + bias[n] ),
 *   acc[m, n] = sum_k xq[m, k] * Wq[n, k]  (exact int32),
 * where xq, sx are the per-token quantization of x (qk_quantize_activations).
 * The dequant is evaluated in fp32, fma(fp32(acc) * sx, sw, bias), wherever
 * a per-element guard (|that value| >= 2^-12 |bias|, and no fp32 underflow)
 * proves it within 1/8 bf16 ulp of the exact value; every other element
 * (cancellation against the bias) takes the exact fp64 evaluation.  Each
 * element is rounded once to bf16 (nearest even) and lies within 1 bf16 ulp
 * of the exact value rounded once (0 ulp on most elements).
 *   x         : bf16 bits [M, K]   (in)
 *   Wq, sw    : from qk_quantize_weights_int8 (in)
 *   bias      : fp32 [N] (in, nullable: no bias)
 *   y         : bf16 bits [M, N]   (out)
 *   workspace : device scratch of ws_bytes >= qk_w8a8_workspace_size(M, K),
 *               or NULL: the call then allocates it stream-ordered
 *               (cudaMallocAsync / cudaFreeAsync on `stream`).  Two calls
 *               that may run at the same time need separate workspaces; the
 *               codes and scales of x are left in it.
 */
qk_status qk_w8a8_linear(const uint16_t *x, int64_t M, int64_t K,
                         const int8_t *Wq, const float *sw, const float *bias, int64_t N,
                         uint16_t *y, void *workspace, size_t ws_bytes,
                         qk_stream_t stream);

/*
 * The W8A8 linear as ONE kernel ("qlip-mlx" README, "w8a8_linear /
 * W8A8Linear": the activations quantized dynamically inside the op, the
 * whole linear a single graph node).  Same inputs, outputs, workspace and
 * errors as qk_w8a8_linear, and the same result (the codes and scales left in
 * the workspace are the same bits): the tcgen05 GEMM's epilogue warps
 * quantize the rows of x into the workspace while the tiles run (rows spread
 * over every warp of the grid, kept two waves of tiles ahead), and the loads
 * of each tile wait until its rows are ready (one readiness word per row,
 * set to a per-launch value, so the workspace needs no clearing).  Thin
 * outputs (N <= 64) take the split-K route behind the quantization kernel,
 * as qk_w8a8_linear does.
 * On B200 this is slower than the two kernels of qk_w8a8_linear at the DiT
 * shapes measured (the quantization's memory traffic and latency inside the
 * GEMM cost more than the kernel boundary saves), so qk_w8a8_linear does not
 * use it.
 */
qk_status qk_w8a8_linear_fused(const uint16_t *x, int64_t M, int64_t K,
                               const int8_t *Wq, const float *sw, const float *bias, int64_t N,
                               uint16_t *y, void *workspace, size_t ws_bytes,
                               qk_stream_t stream);

/*
 * The W8A8 linear with a gated residual epilogue ("mlx-kquant PR #89", commit
 * list: a quantized matmul with a gated residual epilogue, each element held
 * within 2 ulp), the update of a DiT block's residual stream:
 *   y[m, n] = bf16( residual[m, n] + gate[n] * (acc[m, n] * sx[m] * sw[n] + bias[n]) )
 * rounded once to bf16 (nearest even); the bracket is the value qk_w8a8_linear
 * rounds.  As there, fp32 evaluates every element a guard proves within half
 * a bf16 ulp of the exact value, and the exact fp64 evaluation takes the rest
 * (cancellation against the residual or the bias): within 1 bf16 ulp of the
 * exact value rounded once.
 *   x, Wq, sw, bias, workspace : as for qk_w8a8_linear
 *   gate      : fp32 [N], one gate per output channel (in)
 *   residual  : bf16 bits [M, N] (in); y may be the residual itself (an
 *               in-place update: each element is read before it is written)
 *   y         : bf16 bits [M, N]   (out)
 * Errors as for qk_w8a8_linear; gate and residual must be non-NULL and
 * 16-byte aligned.
 */
qk_status qk_w8a8_linear_gated(const uint16_t *x, int64_t M, int64_t K,
                               const int8_t *Wq, const float *sw, const float *bias,
                               const float *gate, const uint16_t *residual, int64_t N,
                               uint16_t *y, void *workspace, size_t ws_bytes,
                               qk_stream_t stream);

/*
 * The matmul + dequant half of qk_w8a8_linear, on activations that are already
 * quantized (xq, sx from qk_quantize_activations).  Lets one quantization feed
 * several projections of the same input.
 */
qk_status qk_w8a8_gemm(const int8_t *xq, const float *sx, int64_t M, int64_t K,
                       const int8_t *Wq, const float *sw, const float *bias, int64_t N,
                       uint16_t *y, qk_stream_t stream);

/*
 * The W8A8 linear without any device allocation.  The pages have no
 * counterpart: this exists for callers that may not allocate device memory at
 * call time and cannot hand over a workspace either (a custom allocator that
 * owns all device memory, a fixed-budget real-time host, a plugin whose host
 * forbids allocation in its callbacks).
 *
 * Computes exactly what qk_w8a8_linear computes (same kernels), but keeps the
 * quantized activations in a scratch array built into the library: a
 * file-scope __device__ array of QK_NOALLOC_SCRATCH_BYTES (64 MiB).  Every GPU
 * that loads the library's module holds that array until the process exits
 * (with CUDA's default lazy module loading, from the first call on that
 * device).  The call itself allocates nothing: no cudaMalloc, no cudaFree, no
 * allocating library routine.
 *
 *   - Problems whose scratch, qk_w8a8_workspace_size(M, K), exceeds
 *     QK_NOALLOC_SCRATCH_BYTES are rejected with QK_ERR_WORKSPACE before any
 *     launch (M * K up to about 64 Mi elements; e.g. 16384 x 3072 fits).
 *   - The first call on a device resolves the scratch's device address
 *     (cudaGetSymbolAddress) and loads the kernels; make that first call
 *     before any stream capture.
 *   - All calls on a device share the one scratch array, which keeps whatever
 *     the last call wrote.  Nothing in it needs to start at zero (each call
 *     overwrites the part it reads).  Calls whose executions overlap on the GPU
 *     (for example on two streams without ordering between them) race on the
 *     scratch and give wrong results: order them on one stream or with events.
 *   - The scratch address is resolved once per device and kept; after
 *     cudaDeviceReset (which unloads the module and its array) this entry
 *     point must not be called again in the same process.
 * Arguments, layouts and the other errors are those of qk_w8a8_linear.
 */
#define QK_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

qk_status qk_w8a8_linear_noalloc(const uint16_t *x, int64_t M, int64_t K,
                                 const int8_t *Wq, const float *sw, const float *bias,
                                 int64_t N, uint16_t *y, qk_stream_t stream);

/* ------------------------------------------------------------ W4A8 linear */

/*
 * The W4A8 linear ("qlip-mlx" README, "w4a8_linear / W4A8Linear"; weights in
 * the affine group-64 format of qk_quantize_weights_int4).  With G = K / 64,
 * the dequantized weight q * s + o and the dequantized activation xq * sx:
 *   acc[m, n, g] = sum_{k in group g} xq[m, k] * q[n, k]    (exact int32)
 *   y[m, n] = bf16( sx[m] * sum_g ( s[n,g] * acc[m,n,g] + o[n,g] * xsum[m,g] )
 *                   + bias[n] ),
 * the fold evaluated in fp64 and rounded once to bf16.
 * M <= 16 takes the weight-streaming GEMV when its per-CTA working set fits
 * in shared memory (K <= 4096 at M = 16), otherwise the tensor-core GEMM; both
 * compute the same per-group integers and agree to the fp64 rounding order.
 * The GEMM route computes the same value through byte planes of the
 * dequantized weight: every scale and offset of weight row n is an integer
 * multiple of 2^e_n (e_n the smallest exponent of their lowest set bits), so
 * every dequantized weight is 2^e_n times an integer W; when W + 0x80..80 fits
 * P <= 3 bytes for every weight (Gaussian weights need 2 or 3), the product is
 * P exact int8 GEMMs on those bytes, rounded once -- the fold's exact value
 * (rounded in fp32 where an error bound proves the bf16 result equal to the
 * exact value's, in fp64 otherwise), the same bits as the per-group fold
 * wherever that fold is exact in fp64;
 * otherwise the per-group fold kernel computes it.  The route allocates its
 * scratch (the planes, up to 3 N K bytes) stream-ordered from a memory pool of
 * the library that keeps freed blocks for reuse.
 * When also M <= 6 and each CTA's K slice of x fits its registers (M times
 * the slice <= 16384 elements) the GEMV quantizes x itself (same rule and
 * codes as qk_quantize_activations) and the call is one kernel; the workspace
 * is then checked but not used (qk_w4a8_linear_plan tells which case
 * applies).  From 7 tokens on, the quantization kernel followed by the GEMV
 * on its codes is faster.
 *   x                  : bf16 bits [M, K]            (in)
 *   Wp, wscale, woffset: from qk_quantize_weights_int4 (in)
 *   bias               : fp32 [N] (nullable)
 *   y                  : bf16 bits [M, N]            (out)
 *   workspace          : >= qk_w4a8_workspace_size(M, K) bytes, or NULL
 *                        (stream-ordered allocation as in qk_w8a8_linear).
 */
qk_status qk_w4a8_linear(const uint16_t *x, int64_t M, int64_t K,
                         const uint8_t *Wp, const uint16_t *wscale, const uint16_t *woffset,
                         const float *bias, int64_t N,
                         uint16_t *y, void *workspace, size_t ws_bytes,
                         qk_stream_t stream);

/* Kernel plans of qk_w4a8_linear (see qk_w4a8_linear_plan). */
typedef enum {
    QK_PLAN_NONE = 0,       /* M == 0: nothing is launched                      */
    QK_PLAN_GEMV_QUANT = 1, /* one kernel: the GEMV quantizing x itself          */
    QK_PLAN_QUANT_GEMV = 2, /* activation quantization, then the GEMV            */
    QK_PLAN_QUANT_GEMM = 3  /* activation quantization, then the tcgen05 GEMM    */
} qk_plan;

/*
 * Which kernels qk_w4a8_linear launches for this shape on the current device
 * (a query of this library's routing; the method itself has no such call).
 * Returns a qk_plan, or the negated qk_status of an invalid shape.  The GEMV
 * plans depend on the device's SM count; with no device the count is taken
 * as 1.
 */
int qk_w4a8_linear_plan(int64_t M, int64_t K, int64_t N);

/*
 * The product half of qk_w4a8_linear on quantized activations (xq, sx and
 * xsum from qk_quantize_activations), with an explicit route (qk_route).
 * xsum must be the group sums of xq (as that call writes them): the one-token
 * GEMV (M = 1, K a multiple of 1024 up to 4096) recomputes them from xq and
 * does not read xsum, the other routes read it.
 * QK_ROUTE_GEMV with M > 16 returns QK_ERR_INVALID_ARG; with a shape whose
 * GEMV working set does not fit shared memory, QK_ERR_UNSUPPORTED_SHAPE.
 * QK_ROUTE_GEMM takes the byte planes (or the fold where they cannot serve);
 * QK_ROUTE_GEMM_FOLD always takes the per-group fold kernel (any M).
 */
qk_status qk_w4a8_gemm(const int8_t *xq, const float *sx, const int32_t *xsum,
                       int64_t M, int64_t K,
                       const uint8_t *Wp, const uint16_t *wscale, const uint16_t *woffset,
                       const float *bias, int64_t N, uint16_t *y, int route,
                       qk_stream_t stream);

/*
 * A prepared W4A8 weight, for weights that do not change between calls (the
 * usual inference case).  The GEMM route of qk_w4a8_linear (M > 16) first
 * counts the digit planes of the weight and writes them to a scratch (see
 * qk_w4a8_linear); qk_w4a8_prepare does that once into caller-owned device
 * memory, and the _prepared products below then launch only the activation
 * quantization, the gated per-group fold and the plane GEMM, with the same
 * results bit for bit as qk_w4a8_linear / qk_w4a8_gemm.  (The pages' W4 path
 * unpacks the weight per call; this keeps the unpacked form instead.)
 *
 * qk_w4a8_prepared_size: bytes of the prepared form of an [N, K] weight (the
 * plane-count words, e_n and the top-digit slot of every row, and up to
 * 3 N K bytes of digit rows), or 0 for an unsupported shape (N % 8 != 0,
 * K % 64 != 0, K outside [64, 65536]).
 *
 * qk_w4a8_prepare: writes the prepared form of (Wp, wscale, woffset) to
 * `prepared` (device, 256-byte aligned, >= qk_w4a8_prepared_size(N, K)
 * bytes, owned by the caller and read by every later _prepared call: it must
 * not be written or freed while one is in flight, and must be prepared again
 * after the weight changes).  `planes` (host, nullable): when given, the call
 * synchronizes `stream` and writes the digit-plane count there (1..3; 255
 * when the per-group fold computes the product).  Errors: QK_ERR_INVALID_ARG
 * (NULL pointers), QK_ERR_UNSUPPORTED_SHAPE, QK_ERR_MISALIGNED (inputs not
 * 16-byte or `prepared` not 256-byte aligned), QK_ERR_WORKSPACE (`bytes` too
 * small).
 *
 * qk_w4a8_gemm_prepared / qk_w4a8_linear_prepared: as qk_w4a8_gemm with
 * QK_ROUTE_AUTO / qk_w4a8_linear, with `prepared` (from qk_w4a8_prepare on
 * the same Wp, wscale, woffset, N, K) serving the GEMM route; M <= 16 takes the
 * same GEMV as there (`prepared` is then not read).  Same errors as those
 * calls, plus QK_ERR_INVALID_ARG for a NULL `prepared` and QK_ERR_MISALIGNED
 * for one not 256-byte aligned.
 */
size_t qk_w4a8_prepared_size(int64_t N, int64_t K);

qk_status qk_w4a8_prepare(const uint8_t *Wp, const uint16_t *wscale, const uint16_t *woffset,
                          int64_t N, int64_t K, void *prepared, size_t bytes, int *planes,
                          qk_stream_t stream);

qk_status qk_w4a8_gemm_prepared(const int8_t *xq, const float *sx, const int32_t *xsum,
                                int64_t M, int64_t K,
                                const uint8_t *Wp, const uint16_t *wscale,
                                const uint16_t *woffset, const void *prepared,
                                const float *bias, int64_t N, uint16_t *y,
                                qk_stream_t stream);

qk_status qk_w4a8_linear_prepared(const uint16_t *x, int64_t M, int64_t K,
                                  const uint8_t *Wp, const uint16_t *wscale,
                                  const uint16_t *woffset, const void *prepared,
                                  const float *bias, int64_t N,
                                  uint16_t *y, void *workspace, size_t ws_bytes,
                                  qk_stream_t stream);

/* ---------------------------------------------------------------- errors */

/*
 * Synchronizes `stream`, then reads and clears this device's error word.
 * Returns QK_ERR_TIMEOUT if a kernel wait gave up since the last check,
 * QK_ERR_CUDA if the synchronization failed, else QK_OK.
 */
qk_status qk_check_device_error(qk_stream_t stream);

/* ------------------------------------------------------- INT8 attention */

/* Bytes of workspace qk_sage_attention needs: the INT8 codes and fp32 scales
 * of q and k and a transposed copy of v, each part 256-byte aligned. */
size_t qk_sage_attention_workspace_size(int64_t B, int64_t H, int64_t L);

/*
 * INT8 attention of a diffusion transformer block ("qlip-mlx" README, intro
 * bullet "sage_attention" and the "Exact where it matters" bullet: INT8 Q K^T
 * inside a flash-attention structure with exact online softmax, per-token
 * scales, softmax and P V in floating point; head dim 128; no mask):
 *   qc, sq = per-token quantization of q (the qk_quantize_activations rule on
 *            each 128-element row), likewise kc, sk for k;
 *   s[i, j] = (qc_i . kc_j) * sq[i] * sk[j] * scale;
 *   out_i   = sum_j softmax_j(s[i, :]) v_j.
 * Scores and the softmax are evaluated in fp32 (2^x by the hardware
 * approximation), the weights rounded to bf16 for P V (bf16 tensor-core
 * products, fp32 sums) and normalised by the sum of the rounded weights; out
 * is rounded to bf16.  Relative to the same formula in exact arithmetic the
 * error per element stays below about 2^-8 (max_j |v_j| + |out_i|).
 *   q, k, v   : bf16 bits [B, H, L, 128], contiguous (in)
 *   D         : head dim, must be 128
 *   scale     : the softmax scale, finite and >= 0 (e.g. 1 / sqrt(128))
 *   out       : bf16 bits [B, H, L, 128] (out; must not alias q, k or v)
 *   workspace : >= qk_sage_attention_workspace_size(B, H, L) bytes, or NULL
 *               (allocated stream-ordered on `stream`).
 * Shape contract: B, H >= 1, L >= 1, L % 8 == 0, B * H * L <= 2^31 / 128.
 * Kernels: the activation quantization twice (q, k), a transpose of v, and
 * the attention kernel (tcgen05 kind::i8 for Q K^T, kind::f16 for P V).
 */
qk_status qk_sage_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                            int64_t B, int64_t H, int64_t L, int64_t D, float scale,
                            uint16_t *out, void *workspace, size_t ws_bytes,
                            qk_stream_t stream);

/* ------------------------------------------------------------ test hooks */

/*
 * The W8A8 GEMM mainloop with an epilogue that stores the raw int32
 * accumulators: acc[m, n] = sum_k xq[m, k] * Wq[n, k], acc int32 [M, N].
 * Same kernel, tiles and schedule as qk_w8a8_gemm.
 */
qk_status qk_debug_w8a8_acc(const int8_t *xq, int64_t M, int64_t K,
                            const int8_t *Wq, int64_t N, int32_t *acc,
                            qk_stream_t stream);

/*
 * The per-group int32 accumulators of the W4A8 product for rows [m0, m1):
 * acc[(m - m0), n, g] = sum_{k in group g} xq[m, k] * q[n, k], acc int32
 * [m1 - m0, N, K/64], computed by the mainloop of `route` (QK_ROUTE_GEMM or
 * QK_ROUTE_GEMV; GEMV needs M <= 16).  xq is the full [M, K] matrix.
 */
qk_status qk_debug_w4a8_group_acc(const int8_t *xq, int64_t M, int64_t K,
                                  const uint8_t *Wp, int64_t N,
                                  int64_t m0, int64_t m1, int32_t *acc,
                                  int route, qk_stream_t stream);

/*
 * The plane count the W4A8 GEMM route computes for a weight (the byte-plane
 * reformulation of the fold: with e_n the smallest exponent of the lowest set
 * bit over the nonzero scales and offsets of weight row n, every dequantized
 * weight of the row is 2^e_n times the integer S q + O; the count is the
 * fewest bytes P <= 3 holding S q + O + 0x80..80 for every code q of every row,
 * else 255, or 255 for a non-finite scale or offset).  Writes it to *planes
 * (host) after synchronizing `stream`.  The route uses the byte-plane GEMM
 * for P <= 3, the per-group fold kernel otherwise.  When P = 3 the GEMM takes
 * the mixed layout (two digit planes for every row, the third digit only for
 * the rows that need one, at most 8 in each aligned block of 60 rows) if every
 * block fits; *mixed (host, nullable) receives 1 then, else 0.  Shapes as for
 * the W4A8 calls; N >= 8.
 */
qk_status qk_debug_w4a8_plane_count(const uint16_t *wscale, const uint16_t *woffset,
                                    int64_t N, int64_t K, int *planes, int *mixed,
                                    qk_stream_t stream);

/*
 * A probe of the device's INT8 tensor-pipe throughput (the denominator of the
 * W8A8 GEMM's roofline fraction; the pages have no counterpart).  One CTA pair
 * per two SMs issues `iters` x 8 tcgen05.mma.cta_group::2.kind::i8 of
 * M = 256, N = 256, K = 32 -- the instruction stream of the W8A8 GEMM's
 * mainloop -- on operands resident in shared memory (no global loads, no
 * epilogue).  If `ops` is not NULL it receives (on the host, at return) the
 * int8 operations the launch performs, 2 * 256 * 256 * 32 per MMA; the caller
 * times the launch on `stream`.  1 <= iters <= 2^24 (one iteration takes about
 * half a microsecond at full clock), else QK_ERR_INVALID_ARG.  The one wait
 * (for the issued MMAs to drain) is bounded as in every kernel here.
 */
qk_status qk_debug_int8_peak(int64_t iters, double *ops, qk_stream_t stream);

/*
 * The timeout path of the library's bounded waits, for tests: launches one
 * single-thread kernel that waits on an mbarrier no thread arrives at and on
 * a device word no thread sets.  Each wait gives up after limit_cycles SM
 * clock cycles (1 <= limit_cycles <= 2^31), records QK_ERR_TIMEOUT in the
 * device error word and the kernel returns; qk_check_device_error then
 * returns QK_ERR_TIMEOUT once, and the context stays usable.  Nothing traps.
 * Returns QK_ERR_INVALID_ARG for a limit out of range.
 */
qk_status qk_debug_wait_timeout(int64_t limit_cycles, qk_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* QK_H */
