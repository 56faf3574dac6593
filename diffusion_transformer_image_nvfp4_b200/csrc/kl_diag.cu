// kl_diag.cu -- a self-test of the library's failure path: a kernel whose
// mbarrier wait can never complete, so its bounded wait must run out, record
// KL_ERR_DEVICE_TIMEOUT in the device status word and return, leaving the
// context usable.  It waits with the same code every library kernel uses
// (mbar_wait_limit), only with a short caller-given limit.
#include "../../include/klein.h"
#include "kl_common.cuh"
#include "kl_internal.h"

namespace kl {

// One warp: lane 0 initialises an mbarrier that expects one arrival, then
// the warp waits on its first phase.  Nothing arrives, nothing is in flight
// (no copy, no MMA, no TMEM), so the wait ends only by its limit.
__global__ void __launch_bounds__(32, 1) wait_timeout_kernel(uint64_t limit_ns, int* waited_out) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncwarp();
  const bool ok = __all_sync(0xffffffffu, mbar_wait_limit(&bar, 0, &abort_flag, limit_ns));
  if (threadIdx.x == 0 && waited_out) *waited_out = ok ? 1 : 0;
}

}  // namespace kl

extern "C" kl_status kl_selftest_wait_timeout(uint64_t limit_ns, int* waited_out, void* stream) {
  using namespace kl;
  if (limit_ns < 1000 || limit_ns > 1000000000ull) return KL_ERR_INVALID_ARG;
  if (waited_out && (reinterpret_cast<uintptr_t>(waited_out) & 3)) return KL_ERR_MISALIGNED;
  kl_status st = check_arch();
  if (st != KL_OK) return st;
  wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns, waited_out);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? KL_OK : cuda_fail(e);
}
