// noalloc.cu -- qk_w8a8_linear_noalloc: the W8A8 linear with no device
// allocation at all.
//
// qk_w8a8_linear needs scratch for the quantized activations (int8 codes and
// fp32 row scales).  It takes that scratch from the caller or allocates it with
// cudaMallocAsync.  Some callers can do neither: code that runs where the
// allocator must not be touched (a custom allocator that owns all device
// memory, a real-time or embedded host with a fixed memory budget set at start,
// or a plugin whose host framework forbids allocation inside its callbacks).
// This entry point serves them: its scratch is one file-scope __device__ array
// of QK_NOALLOC_SCRATCH_BYTES, part of the library's module, so every GPU that
// loads this module holds it until the process exits, and no call allocates.
//
// The kernels are the same ones qk_w8a8_linear launches (activation quant, then
// the tcgen05 GEMM); only the scratch pointer differs.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "qk.h"
#include "qk_internal.h"

namespace {

static_assert(QK_NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size must keep 256-byte carving");

// The scratch.  In host code this name is only a stand-in for the symbol: its
// device address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[QK_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
uint8_t* g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of this device's copy of the scratch; resolved on the first
// call made with that device current and kept for the life of the process
// (cudaDeviceReset unloads the module, after which the kept address is stale:
// the header says not to call this entry point after a reset).  Null if the
// lookup fails.
uint8_t* scratch_address(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return nullptr;
    g_scratch_addr[dev] = static_cast<uint8_t*>(p);
  }
  return g_scratch_addr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" qk_status qk_w8a8_linear_noalloc(const uint16_t* x, int64_t M, int64_t K,
                                            const int8_t* Wq, const float* sw, const float* bias,
                                            int64_t N, uint16_t* y, qk_stream_t stream) {
  if (M < 0 || K < 0 || N < 0) return QK_ERR_INVALID_ARG;
  if (M > INT32_MAX || N > INT32_MAX || K < 32 || K > 65536 || K % 32 != 0 || N < 8 || N % 8 != 0)
    return QK_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return QK_OK;
  if (!x || !Wq || !sw || !y) return QK_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(Wq) || !aligned16(sw) || !aligned16(y) ||
      (bias && !aligned16(bias)))
    return QK_ERR_MISALIGNED;
  // codes [M, K] and scales [M] must fit the built-in scratch
  if (qk_w8a8_workspace_size(M, K) > (size_t)QK_NOALLOC_SCRATCH_BYTES) return QK_ERR_WORKSPACE;
  if (qk::check_device() != QK_OK) return QK_ERR_NO_DEVICE;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return QK_ERR_NO_DEVICE;
  uint8_t* scratch = scratch_address(dev);
  if (scratch == nullptr) return QK_ERR_CUDA;

  // Same carving as qk_w8a8_linear's workspace.  Both regions are fully
  // written by the quant kernel before the GEMM reads them, so whatever an
  // earlier call left in the scratch never needs clearing.
  int8_t* xq = reinterpret_cast<int8_t*>(scratch);
  float* sx = reinterpret_cast<float*>(scratch + (((size_t)M * (size_t)K + 255u) & ~size_t(255u)));
  if (qk::launch_quant_act(x, M, K, xq, sx, nullptr, stream) != cudaSuccess) return QK_ERR_CUDA;
  if (qk::launch_w8a8_gemm(xq, sx, M, K, Wq, sw, bias, N, y, nullptr, true, stream) != cudaSuccess)
    return QK_ERR_CUDA;
  return QK_OK;
}
