// debug_wait.cu -- a test hook for the timeout path of the bounded waits.
//
// One single-thread kernel waits on two things nothing will ever complete: an
// mbarrier in shared memory that no thread arrives at, and a device word that
// no thread sets.  Each wait is the same bounded loop the kernels use, with a
// caller-chosen limit; when it gives up it records QK_ERR_TIMEOUT in the
// device error word and the kernel returns normally, so the context stays
// usable and the host reads the status with qk_check_device_error.  Nothing
// traps, faults or spins without a bound.
#include <cuda_runtime.h>

#include <cstdint>

#include "qk_internal.h"
#include "sm100.cuh"

namespace qk {
namespace {

__device__ uint32_t g_never_set;  // no kernel writes it: stays 0

__global__ void wait_timeout_probe_kernel(int* err, long long limit_cycles) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  fence_mbar_init();
  mbar_wait_limit(b, 0, err, limit_cycles);  // no arrival: gives up
  // a device-scope flag nobody sets, polled the same bounded way
  const long long t0 = clock64();
  while (*reinterpret_cast<volatile uint32_t*>(&g_never_set) == 0u) {
    if (clock64() - t0 > limit_cycles) {
      record_timeout(err);
      break;
    }
  }
}

}  // namespace

cudaError_t launch_wait_timeout_probe(long long limit_cycles, cudaStream_t s) {
  int* err = device_error_word();
  if (err == nullptr) return cudaErrorUnknown;
  wait_timeout_probe_kernel<<<1, 1, 0, s>>>(err, limit_cycles);
  return cudaGetLastError();
}

}  // namespace qk
