// qk_api.cu -- the C ABI of include/qk.h: argument checks, device checks,
// workspace carving and the kernel launches.  All checks run on the host before
// any launch; nothing here computes on the CPU.
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <mutex>

#include "qk.h"
#include "qk_internal.h"

namespace qk {

// The device error word (see sm100.cuh).  One per device: every device that
// loads the library's module has its own copy.
__device__ int g_qk_error = 0;

namespace {

constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices];
int g_cc_ok[kMaxDevices];  // 0 unknown, 1 sm_100, -1 other
int* g_err_ptr[kMaxDevices];
std::mutex g_mu;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool log_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("QK_LOG");
    return v != nullptr && v[0] == '1';
  }();
  return on;
}

int current_device() {
  int d = -1;
  if (cudaGetDevice(&d) != cudaSuccess) return -1;
  return d;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round256(size_t b) { return (b + 255u) & ~size_t(255u); }

// Shape contract shared by every product call.
qk_status check_shape(int64_t M, int64_t K, int64_t N, bool w4) {
  if (M < 0 || K < 0 || N < 0) return QK_ERR_INVALID_ARG;
  if (M > INT32_MAX || N > INT32_MAX) return QK_ERR_UNSUPPORTED_SHAPE;
  if (K < 32 || K > 65536 || K % 32 != 0) return QK_ERR_UNSUPPORTED_SHAPE;
  if (w4 && K % 64 != 0) return QK_ERR_UNSUPPORTED_SHAPE;
  if (N < 8 || N % 8 != 0) return QK_ERR_UNSUPPORTED_SHAPE;
  return QK_OK;
}

qk_status from_cuda(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return QK_OK;
  if (log_enabled()) std::fprintf(stderr, "[qk] %s: %s\n", what, cudaGetErrorString(e));
  return QK_ERR_CUDA;
}

// Carves xq / sx / xsum out of a workspace block, allocating it stream-ordered
// when the caller passes none.
struct Workspace {
  int8_t* xq = nullptr;
  float* sx = nullptr;
  int32_t* xsum = nullptr;
  unsigned long long* ready = nullptr;  // W8A8: readiness words of the fused quantization
  void* owned = nullptr;
  cudaStream_t stream = nullptr;

  qk_status init(void* ws, size_t ws_bytes, int64_t M, int64_t K, bool w4, cudaStream_t s) {
    const size_t need = w4 ? qk_w4a8_workspace_size(M, K) : qk_w8a8_workspace_size(M, K);
    uint8_t* base = static_cast<uint8_t*>(ws);
    if (base == nullptr) {
      cudaError_t e = cudaMallocAsync(&owned, need, s);
      if (e != cudaSuccess) return from_cuda(e, "cudaMallocAsync(workspace)");
      stream = s;
      base = static_cast<uint8_t*>(owned);
    } else if (ws_bytes < need || (reinterpret_cast<uintptr_t>(base) & 255u) != 0) {
      return QK_ERR_WORKSPACE;
    }
    xq = reinterpret_cast<int8_t*>(base);
    sx = reinterpret_cast<float*>(base + round256((size_t)M * (size_t)K));
    if (w4)
      xsum = reinterpret_cast<int32_t*>(base + round256((size_t)M * (size_t)K) +
                                        round256((size_t)M * 4u));
    else
      ready = reinterpret_cast<unsigned long long*>(base + round256((size_t)M * (size_t)K) +
                                                    round256((size_t)M * 4u));
    return QK_OK;
  }
  ~Workspace() {
    if (owned != nullptr) cudaFreeAsync(owned, stream);
  }
};

}  // namespace

qk_status check_device() {
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return QK_ERR_NO_DEVICE;
  if (g_cc_ok[d] == 0) g_cc_ok[d] = qk_is_available(d) ? 1 : -1;
  return g_cc_ok[d] == 1 ? QK_OK : QK_ERR_NO_DEVICE;
}

int* device_error_word() {
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return nullptr;
  if (g_err_ptr[d] == nullptr) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_err_ptr[d] == nullptr) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_qk_error) != cudaSuccess) return nullptr;
      g_err_ptr[d] = static_cast<int*>(p);
    }
  }
  return g_err_ptr[d];
}

// The library's stream-ordered memory pool on the current device (created on
// first use): it keeps freed blocks reserved instead of returning them to the
// driver at each synchronization, so the large per-call scratch of the W4A8
// GEMM route (the weight's byte planes) is recycled, not mapped again on every
// call.  Null if the pool cannot be made (callers then use the default pool).
cudaMemPool_t scratch_pool() {
  static cudaMemPool_t pools[kMaxDevices];
  static bool tried[kMaxDevices];
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!tried[d]) {
    tried[d] = true;
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.handleTypes = cudaMemHandleTypeNone;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = d;
    cudaMemPool_t pool = nullptr;
    if (cudaMemPoolCreate(&pool, &props) == cudaSuccess) {
      unsigned long long keep = ~0ull;
      cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
      pools[d] = pool;
    } else {
      cudaGetLastError();
    }
  }
  return pools[d];
}

cudaError_t scratch_alloc(void** p, size_t bytes, cudaStream_t s) {
  cudaMemPool_t pool = scratch_pool();
  return pool != nullptr ? cudaMallocFromPoolAsync(p, bytes, pool, s) : cudaMallocAsync(p, bytes, s);
}

int num_sms() {
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return 1;
  if (g_sm_count[d] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d);
    g_sm_count[d] = n > 0 ? n : 1;
  }
  return g_sm_count[d];
}

bool encode_tmap_2d(CUtensorMap* out, CUtensorMapDataType dtype, const void* base,
                    uint64_t inner, uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner,
                    uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (g_encode == nullptr) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(out, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace qk

using namespace qk;

extern "C" {

const char* qk_status_string(int status) {
  switch (status) {
    case QK_OK: return "QK_OK";
    case QK_ERR_INVALID_ARG: return "QK_ERR_INVALID_ARG: null pointer, negative size or bad route";
    case QK_ERR_UNSUPPORTED_SHAPE: return "QK_ERR_UNSUPPORTED_SHAPE: K or N outside the shape contract";
    case QK_ERR_MISALIGNED: return "QK_ERR_MISALIGNED: a pointer is not 16-byte aligned";
    case QK_ERR_NO_DEVICE: return "QK_ERR_NO_DEVICE: no CUDA device, or not sm_100";
    case QK_ERR_WORKSPACE: return "QK_ERR_WORKSPACE: workspace too small or not 256-byte aligned";
    case QK_ERR_CUDA: return "QK_ERR_CUDA: a CUDA call or kernel launch failed";
    case QK_ERR_TIMEOUT: return "QK_ERR_TIMEOUT: a kernel wait gave up";
    default: return "unknown qk_status";
  }
}

int qk_version(void) { return (0 << 16) | 1; }

int qk_is_available(int device) {
  int n = 0;
  if (cudaGetDeviceCount(&n) != cudaSuccess || device < 0 || device >= n) {
    cudaGetLastError();
    return 0;
  }
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device) != cudaSuccess)
    return 0;
  return (major == 10 && minor == 0) ? 1 : 0;
}

size_t qk_w8a8_workspace_size(int64_t M, int64_t K) {
  if (M < 0 || K < 0) return 0;
  // codes, scales, and one 8-byte readiness word per row
  return round256((size_t)M * (size_t)K) + round256((size_t)M * 4u) + round256((size_t)M * 8u);
}

size_t qk_w4a8_workspace_size(int64_t M, int64_t K) {
  if (M < 0 || K < 0) return 0;
  return round256((size_t)M * (size_t)K) + round256((size_t)M * 4u) +
         round256((size_t)M * (size_t)(K / 64) * 4u);
}

qk_status qk_quantize_weights_int8(const float* W, int64_t N, int64_t K, int8_t* Wq, float* sw,
                                   qk_stream_t stream) {
  if (N < 0 || K < 0) return QK_ERR_INVALID_ARG;
  if (K < 32 || K > 65536 || K % 32 != 0 || N > INT32_MAX) return QK_ERR_UNSUPPORTED_SHAPE;
  if (N == 0) return QK_OK;
  if (!W || !Wq || !sw) return QK_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(Wq) || !aligned16(sw)) return QK_ERR_MISALIGNED;
  qk_status st = check_device();
  if (st != QK_OK) return st;
  return from_cuda(launch_quant_w8(W, N, K, Wq, sw, stream), "quant_w8");
}

qk_status qk_quantize_weights_int4(const float* W, int64_t N, int64_t K, uint8_t* Wp,
                                   uint16_t* wscale, uint16_t* woffset, qk_stream_t stream) {
  if (N < 0 || K < 0) return QK_ERR_INVALID_ARG;
  if (K < 64 || K > 65536 || K % 64 != 0 || N > INT32_MAX) return QK_ERR_UNSUPPORTED_SHAPE;
  if (N == 0) return QK_OK;
  if (!W || !Wp || !wscale || !woffset) return QK_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(Wp) || !aligned16(wscale) || !aligned16(woffset))
    return QK_ERR_MISALIGNED;
  qk_status st = check_device();
  if (st != QK_OK) return st;
  return from_cuda(launch_quant_w4(W, N, K, Wp, wscale, woffset, stream), "quant_w4");
}

qk_status qk_quantize_activations(const uint16_t* x, int64_t M, int64_t K, int8_t* xq, float* sx,
                                  int32_t* xsum, qk_stream_t stream) {
  if (M < 0 || K < 0) return QK_ERR_INVALID_ARG;
  if (K < 32 || K > 65536 || K % 32 != 0 || M > INT32_MAX) return QK_ERR_UNSUPPORTED_SHAPE;
  if (xsum != nullptr && K % 64 != 0) return QK_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return QK_OK;
  if (!x || !xq || !sx) return QK_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(xq) || !aligned16(sx) || (xsum && !aligned16(xsum)))
    return QK_ERR_MISALIGNED;
  qk_status st = check_device();
  if (st != QK_OK) return st;
  return from_cuda(launch_quant_act(x, M, K, xq, sx, xsum, stream), "quant_act");
}

qk_status qk_w8a8_gemm(const int8_t* xq, const float* sx, int64_t M, int64_t K, const int8_t* Wq,
                       const float* sw, const float* bias, int64_t N, uint16_t* y,
                       qk_stream_t stream) {
  qk_status st = check_shape(M, K, N, false);
  if (st != QK_OK || M == 0) return st;
  if (!xq || !sx || !Wq || !sw || !y) return QK_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(sx) || !aligned16(Wq) || !aligned16(sw) || !aligned16(y) ||
      (bias && !aligned16(bias)))
    return QK_ERR_MISALIGNED;
  if ((st = check_device()) != QK_OK) return st;
  return from_cuda(launch_w8a8_gemm(xq, sx, M, K, Wq, sw, bias, N, y, nullptr, true, stream),
                   "w8a8_gemm");
}

qk_status qk_w8a8_linear(const uint16_t* x, int64_t M, int64_t K, const int8_t* Wq,
                         const float* sw, const float* bias, int64_t N, uint16_t* y,
                         void* workspace, size_t ws_bytes, qk_stream_t stream) {
  qk_status st = check_shape(M, K, N, false);
  if (st != QK_OK || M == 0) return st;
  if (!x || !Wq || !sw || !y) return QK_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(Wq) || !aligned16(sw) || !aligned16(y) ||
      (bias && !aligned16(bias)))
    return QK_ERR_MISALIGNED;
  if ((st = check_device()) != QK_OK) return st;
  Workspace ws;
  if ((st = ws.init(workspace, ws_bytes, M, K, false, stream)) != QK_OK) return st;
  if ((st = from_cuda(launch_quant_act(x, M, K, ws.xq, ws.sx, nullptr, stream, true),
                      "quant_act")) != QK_OK)
    return st;
  if (log_enabled())
    std::fprintf(stderr, "[qk] w8a8_linear M=%lld K=%lld N=%lld -> quant_act + tcgen05 GEMM\n",
                 (long long)M, (long long)K, (long long)N);
  return from_cuda(launch_w8a8_gemm(ws.xq, ws.sx, M, K, Wq, sw, bias, N, y, nullptr, true, stream),
                   "w8a8_gemm");
}

qk_status qk_w8a8_linear_fused(const uint16_t* x, int64_t M, int64_t K, const int8_t* Wq,
                               const float* sw, const float* bias, int64_t N, uint16_t* y,
                               void* workspace, size_t ws_bytes, qk_stream_t stream) {
  qk_status st = check_shape(M, K, N, false);
  if (st != QK_OK || M == 0) return st;
  if (!x || !Wq || !sw || !y) return QK_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(Wq) || !aligned16(sw) || !aligned16(y) ||
      (bias && !aligned16(bias)))
    return QK_ERR_MISALIGNED;
  if ((st = check_device()) != QK_OK) return st;
  Workspace ws;
  if ((st = ws.init(workspace, ws_bytes, M, K, false, stream)) != QK_OK) return st;
  if (!w8a8_use_fused(M, K, N)) {
    // thin outputs: the split-K route, behind the quantization kernel
    if ((st = from_cuda(launch_quant_act(x, M, K, ws.xq, ws.sx, nullptr, stream, true),
                        "quant_act")) != QK_OK)
      return st;
    return from_cuda(
        launch_w8a8_gemm(ws.xq, ws.sx, M, K, Wq, sw, bias, N, y, nullptr, true, stream),
        "w8a8_gemm");
  }
  if (log_enabled())
    std::fprintf(stderr, "[qk] w8a8_linear_fused M=%lld K=%lld N=%lld -> one kernel\n",
                 (long long)M, (long long)K, (long long)N);
  return from_cuda(
      launch_w8a8_fused(x, M, K, Wq, sw, bias, N, y, ws.xq, ws.sx, ws.ready, true, stream),
      "w8a8_fused");
}

qk_status qk_w8a8_linear_gated(const uint16_t* x, int64_t M, int64_t K, const int8_t* Wq,
                               const float* sw, const float* bias, const float* gate,
                               const uint16_t* residual, int64_t N, uint16_t* y, void* workspace,
                               size_t ws_bytes, qk_stream_t stream) {
  qk_status st = check_shape(M, K, N, false);
  if (st != QK_OK || M == 0) return st;
  if (!x || !Wq || !sw || !y || !gate || !residual) return QK_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(Wq) || !aligned16(sw) || !aligned16(y) || !aligned16(gate) ||
      !aligned16(residual) || (bias && !aligned16(bias)))
    return QK_ERR_MISALIGNED;
  if ((st = check_device()) != QK_OK) return st;
  Workspace ws;
  if ((st = ws.init(workspace, ws_bytes, M, K, false, stream)) != QK_OK) return st;
  if ((st = from_cuda(launch_quant_act(x, M, K, ws.xq, ws.sx, nullptr, stream, true),
                      "quant_act")) != QK_OK)
    return st;
  if (log_enabled())
    std::fprintf(stderr, "[qk] w8a8_linear_gated M=%lld K=%lld N=%lld\n", (long long)M,
                 (long long)K, (long long)N);
  return from_cuda(launch_w8a8_gemm(ws.xq, ws.sx, M, K, Wq, sw, bias, N, y, nullptr, true, stream,
                                    gate, residual),
                   "w8a8_gemm_gated");
}

static qk_status check_w4_product(const uint8_t* Wp, const uint16_t* wscale,
                                  const uint16_t* woffset, const float* bias, uint16_t* y) {
  if (!Wp || !wscale || !woffset || !y) return QK_ERR_INVALID_ARG;
  if (!aligned16(Wp) || !aligned16(wscale) || !aligned16(woffset) || !aligned16(y) ||
      (bias && !aligned16(bias)))
    return QK_ERR_MISALIGNED;
  return QK_OK;
}

static bool w4a8_takes_gemv(int route, int64_t M, int64_t K, int64_t N) {
  return route == QK_ROUTE_GEMV || (route == QK_ROUTE_AUTO && gemv_fits(M, K, N));
}

// The GEMM route allocates its plane scratch (w4a8_plane_scratch_bytes)
// stream-ordered for the call, from the library's pool (scratch_pool).
static cudaError_t run_w4a8(const int8_t* xq, const float* sx, const int32_t* xsum, int64_t M,
                            int64_t K, const uint8_t* Wp, const uint16_t* ws, const uint16_t* wo,
                            const float* bias, int64_t N, uint16_t* y, int route, bool pdl,
                            cudaStream_t s) {
  const bool gemv = w4a8_takes_gemv(route, M, K, N);
  if (log_enabled())
    std::fprintf(stderr, "[qk] w4a8 M=%lld K=%lld N=%lld -> %s\n", (long long)M, (long long)K,
                 (long long)N,
                 gemv ? "GEMV"
                      : route == QK_ROUTE_GEMM_FOLD ? "tcgen05 GEMM, per-group fold"
                                                    : "tcgen05 GEMM, byte planes (fold if needed)");
  if (gemv)
    return launch_w4a8_gemv(xq, sx, xsum, M, K, Wp, ws, wo, bias, N, y, nullptr, 0, 0, pdl, s);
  if (route == QK_ROUTE_GEMM_FOLD)
    return launch_w4a8_fold(xq, sx, xsum, M, K, Wp, ws, wo, bias, N, y, nullptr, 0, 0, pdl, s);
  void* scratch = nullptr;
  cudaError_t e = scratch_alloc(&scratch, w4a8_plane_scratch_bytes(N, K), s);
  if (e != cudaSuccess) return e;
  e = launch_w4a8_gemm(xq, sx, xsum, M, K, Wp, ws, wo, bias, N, y, scratch, pdl, s);
  const cudaError_t f = cudaFreeAsync(scratch, s);
  return e != cudaSuccess ? e : f;
}

int qk_w4a8_linear_plan(int64_t M, int64_t K, int64_t N) {
  const qk_status st = check_shape(M, K, N, true);
  if (st != QK_OK) return -(int)st;
  if (M == 0) return QK_PLAN_NONE;
  if (gemv_quant_fits(M, K, N)) return QK_PLAN_GEMV_QUANT;
  if (gemv_fits(M, K, N)) return QK_PLAN_QUANT_GEMV;
  return QK_PLAN_QUANT_GEMM;
}

qk_status qk_w4a8_gemm(const int8_t* xq, const float* sx, const int32_t* xsum, int64_t M,
                       int64_t K, const uint8_t* Wp, const uint16_t* wscale,
                       const uint16_t* woffset, const float* bias, int64_t N, uint16_t* y,
                       int route, qk_stream_t stream) {
  qk_status st = check_shape(M, K, N, true);
  if (st != QK_OK) return st;
  if (route != QK_ROUTE_AUTO && route != QK_ROUTE_GEMM && route != QK_ROUTE_GEMV &&
      route != QK_ROUTE_GEMM_FOLD)
    return QK_ERR_INVALID_ARG;
  if (route == QK_ROUTE_GEMV && M > 16) return QK_ERR_INVALID_ARG;
  if (route == QK_ROUTE_GEMV && M > 0 && !gemv_fits(M, K, N)) return QK_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return QK_OK;
  if (!xq || !sx || !xsum) return QK_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(sx) || !aligned16(xsum)) return QK_ERR_MISALIGNED;
  if ((st = check_w4_product(Wp, wscale, woffset, bias, y)) != QK_OK) return st;
  if ((st = check_device()) != QK_OK) return st;
  return from_cuda(run_w4a8(xq, sx, xsum, M, K, Wp, wscale, woffset, bias, N, y, route, true,
                            stream),
                   "w4a8");
}

qk_status qk_w4a8_linear(const uint16_t* x, int64_t M, int64_t K, const uint8_t* Wp,
                         const uint16_t* wscale, const uint16_t* woffset, const float* bias,
                         int64_t N, uint16_t* y, void* workspace, size_t ws_bytes,
                         qk_stream_t stream) {
  qk_status st = check_shape(M, K, N, true);
  if (st != QK_OK || M == 0) return st;
  if (!x) return QK_ERR_INVALID_ARG;
  if (!aligned16(x)) return QK_ERR_MISALIGNED;
  if ((st = check_w4_product(Wp, wscale, woffset, bias, y)) != QK_OK) return st;
  if ((st = check_device()) != QK_OK) return st;
  if (gemv_quant_fits(M, K, N)) {
    // small M: the GEMV quantizes x itself; the workspace is checked, not used
    if (workspace != nullptr && (ws_bytes < qk_w4a8_workspace_size(M, K) ||
                                 (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0))
      return QK_ERR_WORKSPACE;
    if (log_enabled())
      std::fprintf(stderr, "[qk] w4a8 M=%lld K=%lld N=%lld -> GEMV (quantizing x)\n",
                   (long long)M, (long long)K, (long long)N);
    return from_cuda(launch_w4a8_gemv_quant(x, M, K, Wp, wscale, woffset, bias, N, y, true,
                                            stream),
                     "w4a8 gemv");
  }
  Workspace ws;
  if ((st = ws.init(workspace, ws_bytes, M, K, true, stream)) != QK_OK) return st;
  // In front of the GEMV the quantization kernel is launched in plain stream
  // order: as a programmatic dependent it would start the next GEMV (and its
  // weight stream) while the previous GEMV still computes, which measured
  // ~1 us slower per call at 16 tokens.  In front of the GEMM it overlaps the
  // previous kernel's tail.
  const bool pdl_quant = !w4a8_takes_gemv(QK_ROUTE_AUTO, M, K, N);
  if ((st = from_cuda(launch_quant_act(x, M, K, ws.xq, ws.sx, ws.xsum, stream, pdl_quant),
                      "quant_act")) != QK_OK)
    return st;
  return from_cuda(run_w4a8(ws.xq, ws.sx, ws.xsum, M, K, Wp, wscale, woffset, bias, N, y,
                            QK_ROUTE_AUTO, true, stream),
                   "w4a8");
}

// ---- prepared W4A8 weights (the GEMM route's digit planes built once)

static bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

static cudaError_t run_w4a8_prepared(const int8_t* xq, const float* sx, const int32_t* xsum,
                                     int64_t M, int64_t K, const uint8_t* Wp, const uint16_t* ws,
                                     const uint16_t* wo, const void* prepared, const float* bias,
                                     int64_t N, uint16_t* y, bool pdl, cudaStream_t s) {
  const bool gemv = w4a8_takes_gemv(QK_ROUTE_AUTO, M, K, N);
  if (log_enabled())
    std::fprintf(stderr, "[qk] w4a8 M=%lld K=%lld N=%lld -> %s\n", (long long)M, (long long)K,
                 (long long)N, gemv ? "GEMV" : "tcgen05 GEMM, prepared byte planes");
  if (gemv)
    return launch_w4a8_gemv(xq, sx, xsum, M, K, Wp, ws, wo, bias, N, y, nullptr, 0, 0, pdl, s);
  return launch_w4a8_gemm_prepared(xq, sx, xsum, M, K, Wp, ws, wo, prepared, bias, N, y, pdl, s);
}

size_t qk_w4a8_prepared_size(int64_t N, int64_t K) {
  if (check_shape(1, K, N, true) != QK_OK) return 0;
  return w4a8_plane_scratch_bytes(N, K);
}

qk_status qk_w4a8_prepare(const uint8_t* Wp, const uint16_t* wscale, const uint16_t* woffset,
                          int64_t N, int64_t K, void* prepared, size_t bytes, int* planes,
                          qk_stream_t stream) {
  qk_status st = check_shape(1, K, N, true);
  if (st != QK_OK) return st;
  if (!Wp || !wscale || !woffset || !prepared) return QK_ERR_INVALID_ARG;
  if (!aligned16(Wp) || !aligned16(wscale) || !aligned16(woffset) || !aligned256(prepared))
    return QK_ERR_MISALIGNED;
  if (bytes < w4a8_plane_scratch_bytes(N, K)) return QK_ERR_WORKSPACE;
  if ((st = check_device()) != QK_OK) return st;
  int p = 0;
  st = from_cuda(launch_w4a8_prepare(Wp, wscale, woffset, N, K, prepared,
                                     planes != nullptr ? &p : nullptr, stream),
                 "w4a8 prepare");
  if (st == QK_OK && planes != nullptr) *planes = (p >= 1 && p <= 3) ? p : 255;
  return st;
}

qk_status qk_w4a8_gemm_prepared(const int8_t* xq, const float* sx, const int32_t* xsum,
                                int64_t M, int64_t K, const uint8_t* Wp, const uint16_t* wscale,
                                const uint16_t* woffset, const void* prepared, const float* bias,
                                int64_t N, uint16_t* y, qk_stream_t stream) {
  qk_status st = check_shape(M, K, N, true);
  if (st != QK_OK || M == 0) return st;
  if (!xq || !sx || !xsum || !prepared) return QK_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(sx) || !aligned16(xsum) || !aligned256(prepared))
    return QK_ERR_MISALIGNED;
  if ((st = check_w4_product(Wp, wscale, woffset, bias, y)) != QK_OK) return st;
  if ((st = check_device()) != QK_OK) return st;
  return from_cuda(run_w4a8_prepared(xq, sx, xsum, M, K, Wp, wscale, woffset, prepared, bias, N,
                                     y, true, stream),
                   "w4a8 prepared");
}

qk_status qk_w4a8_linear_prepared(const uint16_t* x, int64_t M, int64_t K, const uint8_t* Wp,
                                  const uint16_t* wscale, const uint16_t* woffset,
                                  const void* prepared, const float* bias, int64_t N,
                                  uint16_t* y, void* workspace, size_t ws_bytes,
                                  qk_stream_t stream) {
  qk_status st = check_shape(M, K, N, true);
  if (st != QK_OK || M == 0) return st;
  if (!x || !prepared) return QK_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned256(prepared)) return QK_ERR_MISALIGNED;
  if ((st = check_w4_product(Wp, wscale, woffset, bias, y)) != QK_OK) return st;
  if ((st = check_device()) != QK_OK) return st;
  if (gemv_quant_fits(M, K, N)) {
    // small M: as qk_w4a8_linear (the GEMV quantizes x itself; `prepared` unused)
    if (workspace != nullptr && (ws_bytes < qk_w4a8_workspace_size(M, K) ||
                                 (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0))
      return QK_ERR_WORKSPACE;
    return from_cuda(launch_w4a8_gemv_quant(x, M, K, Wp, wscale, woffset, bias, N, y, true,
                                            stream),
                     "w4a8 gemv");
  }
  Workspace ws;
  if ((st = ws.init(workspace, ws_bytes, M, K, true, stream)) != QK_OK) return st;
  const bool pdl_quant = !w4a8_takes_gemv(QK_ROUTE_AUTO, M, K, N);  // as in qk_w4a8_linear
  if ((st = from_cuda(launch_quant_act(x, M, K, ws.xq, ws.sx, ws.xsum, stream, pdl_quant),
                      "quant_act")) != QK_OK)
    return st;
  return from_cuda(run_w4a8_prepared(ws.xq, ws.sx, ws.xsum, M, K, Wp, wscale, woffset, prepared,
                                     bias, N, y, true, stream),
                   "w4a8 prepared");
}

qk_status qk_check_device_error(qk_stream_t stream) {
  qk_status st = check_device();
  if (st != QK_OK) return st;
  if ((st = from_cuda(cudaStreamSynchronize(stream), "cudaStreamSynchronize")) != QK_OK) return st;
  int* word = device_error_word();
  if (word == nullptr) return QK_ERR_CUDA;
  int h = 0;
  if ((st = from_cuda(cudaMemcpy(&h, word, sizeof h, cudaMemcpyDeviceToHost), "read error word")) !=
      QK_OK)
    return st;
  if (h != 0) {
    const int zero = 0;
    if ((st = from_cuda(cudaMemcpy(word, &zero, sizeof zero, cudaMemcpyHostToDevice),
                        "clear error word")) != QK_OK)
      return st;
    return h == QK_ERR_TIMEOUT ? QK_ERR_TIMEOUT : QK_ERR_CUDA;
  }
  return QK_OK;
}

// INT8 attention workspace: qc, kc [BH L 128] int8; sq [BH L] fp32; sk
// [BH L + 128] fp32 (the last key block reads 128 entries from its start);
// vt [BH, 128, L] bf16.
static size_t sage_parts(int64_t BH, int64_t L, size_t off[5]) {
  const size_t n = (size_t)BH * (size_t)L;
  size_t o = 0;
  off[0] = o; o += round256(n * 128);
  off[1] = o; o += round256(n * 128);
  off[2] = o; o += round256(n * 4);
  off[3] = o; o += round256((n + 128) * 4);
  off[4] = o; o += round256(n * 128 * 2);
  return o;
}

size_t qk_sage_attention_workspace_size(int64_t B, int64_t H, int64_t L) {
  if (B <= 0 || H <= 0 || L <= 0) return 0;
  size_t off[5];
  return sage_parts(B * H, L, off);
}

qk_status qk_sage_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t B,
                            int64_t H, int64_t L, int64_t D, float scale, uint16_t* out,
                            void* workspace, size_t ws_bytes, qk_stream_t stream) {
  if (B < 1 || H < 1 || L < 1 || !(scale >= 0.0f) || !(scale < INFINITY)) return QK_ERR_INVALID_ARG;
  if (D != 128 || L % 8 != 0 || B * H * L > (int64_t(1) << 31) / 128)
    return QK_ERR_UNSUPPORTED_SHAPE;
  if (!q || !k || !v || !out) return QK_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return QK_ERR_MISALIGNED;
  qk_status st = check_device();
  if (st != QK_OK) return st;
  const int64_t BH = B * H;
  size_t off[5];
  const size_t need = sage_parts(BH, L, off);
  void* owned = nullptr;
  uint8_t* base = static_cast<uint8_t*>(workspace);
  if (base == nullptr) {
    if ((st = from_cuda(cudaMallocAsync(&owned, need, stream), "cudaMallocAsync(workspace)")) !=
        QK_OK)
      return st;
    base = static_cast<uint8_t*>(owned);
  } else if (ws_bytes < need || (reinterpret_cast<uintptr_t>(base) & 255u) != 0) {
    return QK_ERR_WORKSPACE;
  }
  int8_t* qc = reinterpret_cast<int8_t*>(base + off[0]);
  int8_t* kc = reinterpret_cast<int8_t*>(base + off[1]);
  float* sq = reinterpret_cast<float*>(base + off[2]);
  float* sk = reinterpret_cast<float*>(base + off[3]);
  uint16_t* vt = reinterpret_cast<uint16_t*>(base + off[4]);
  if (log_enabled())
    std::fprintf(stderr, "[qk] sage_attention B=%lld H=%lld L=%lld\n", (long long)B, (long long)H,
                 (long long)L);
  if ((st = from_cuda(launch_quant_act(q, BH * L, 128, qc, sq, nullptr, stream), "quant_q")) ==
          QK_OK &&
      (st = from_cuda(launch_quant_act(k, BH * L, 128, kc, sk, nullptr, stream), "quant_k")) ==
          QK_OK &&
      (st = from_cuda(launch_transpose_v(v, BH, L, vt, stream), "transpose_v")) == QK_OK)
    st = from_cuda(launch_sage_attention(qc, sq, kc, sk, vt, BH, L, scale, out, stream),
                   "sage_attention");
  if (owned != nullptr) cudaFreeAsync(owned, stream);
  return st;
}

qk_status qk_debug_wait_timeout(int64_t limit_cycles, qk_stream_t stream) {
  if (limit_cycles < 1 || limit_cycles > (int64_t(1) << 31)) return QK_ERR_INVALID_ARG;
  qk_status st = check_device();
  if (st != QK_OK) return st;
  return from_cuda(launch_wait_timeout_probe((long long)limit_cycles, stream), "wait_timeout_probe");
}

qk_status qk_debug_int8_peak(int64_t iters, double* ops, qk_stream_t stream) {
  if (iters < 1 || iters > (int64_t(1) << 24)) return QK_ERR_INVALID_ARG;
  qk_status st = check_device();
  if (st != QK_OK) return st;
  int* err = device_error_word();
  if (err == nullptr) return QK_ERR_CUDA;
  int pairs = 0;
  st = from_cuda(launch_int8_peak((long long)iters, err, &pairs, stream), "int8_peak");
  if (st == QK_OK && ops != nullptr) *ops = int8_peak_ops_per_iter(pairs) * (double)iters;
  return st;
}

qk_status qk_debug_w8a8_acc(const int8_t* xq, int64_t M, int64_t K, const int8_t* Wq, int64_t N,
                            int32_t* acc, qk_stream_t stream) {
  qk_status st = check_shape(M, K, N, false);
  if (st != QK_OK || M == 0) return st;
  if (!xq || !Wq || !acc) return QK_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(Wq) || !aligned16(acc)) return QK_ERR_MISALIGNED;
  if ((st = check_device()) != QK_OK) return st;
  return from_cuda(
      launch_w8a8_gemm(xq, nullptr, M, K, Wq, nullptr, nullptr, N, nullptr, acc, false, stream),
      "w8a8_acc");
}

qk_status qk_debug_w4a8_plane_count(const uint16_t* wscale, const uint16_t* woffset, int64_t N,
                                    int64_t K, int* planes, int* mixed, qk_stream_t stream) {
  qk_status st = check_shape(1, K, N, true);
  if (st != QK_OK) return st;
  if (!wscale || !woffset || !planes) return QK_ERR_INVALID_ARG;
  if (!aligned16(wscale) || !aligned16(woffset)) return QK_ERR_MISALIGNED;
  if ((st = check_device()) != QK_OK) return st;
  void* scratch = nullptr;
  if ((st = from_cuda(cudaMallocAsync(&scratch, w4a8_plane_scratch_bytes(N, 0), stream),
                      "cudaMallocAsync(plane count)")) != QK_OK)
    return st;
  const unsigned long long epoch = next_epoch();
  unsigned long long words[2] = {0, 0};
  cudaError_t e = launch_w4a8_plane_count(wscale, woffset, N, K, scratch, epoch, false, stream);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(words, scratch, sizeof(words), cudaMemcpyDeviceToHost, stream);
  cudaFreeAsync(scratch, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if ((st = from_cuda(e, "w4a8_plane_count")) != QK_OK) return st;
  *planes = (words[0] >> 8) == epoch ? (int)(words[0] & 0xFFull) : 0;
  if (mixed != nullptr)
    *mixed = (*planes == 3 && !((words[1] >> 8) == epoch && (words[1] & 1ull) != 0)) ? 1 : 0;
  return QK_OK;
}

qk_status qk_debug_w4a8_group_acc(const int8_t* xq, int64_t M, int64_t K, const uint8_t* Wp,
                                  int64_t N, int64_t m0, int64_t m1, int32_t* acc, int route,
                                  qk_stream_t stream) {
  qk_status st = check_shape(M, K, N, true);
  if (st != QK_OK) return st;
  if (route != QK_ROUTE_GEMM && route != QK_ROUTE_GEMV) return QK_ERR_INVALID_ARG;
  if (route == QK_ROUTE_GEMV && M > 16) return QK_ERR_INVALID_ARG;
  if (route == QK_ROUTE_GEMV && M > 0 && !gemv_fits(M, K, N)) return QK_ERR_UNSUPPORTED_SHAPE;
  if (m0 < 0 || m1 < m0 || m1 > M) return QK_ERR_INVALID_ARG;
  if (m1 == m0) return QK_OK;
  if (!xq || !Wp || !acc) return QK_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(Wp) || !aligned16(acc)) return QK_ERR_MISALIGNED;
  if ((st = check_device()) != QK_OK) return st;
  cudaError_t e =
      route == QK_ROUTE_GEMV
          ? launch_w4a8_gemv(xq, nullptr, nullptr, M, K, Wp, nullptr, nullptr, nullptr, N,
                             nullptr, acc, m0, m1, false, stream)
          : launch_w4a8_fold(xq, nullptr, nullptr, M, K, Wp, nullptr, nullptr, nullptr, N,
                             nullptr, acc, m0, m1, false, stream);
  return from_cuda(e, "w4a8_group_acc");
}

}  // extern "C"
