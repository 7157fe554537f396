// selftest.cu -- a health check of the library's failure detection: a bounded
// mbarrier wait that nothing completes must give up, report PA_FLAG_TIMEOUT
// (in err_flag and in the device-global watchdog word) and return, leaving the
// context usable.  The kernels' own waits have the same shape (a try-wait loop
// against %globaltimer), with a two-second limit.

#include "pa_common.cuh"
#include "pa_internal.h"

namespace pa {

__global__ void __launch_bounds__(32) selftest_wait_kernel(int32_t* err_flag, uint64_t limit_ns,
                                                           unsigned long long* waited_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_barrier_init();
  const uint64_t t0 = globaltimer_ns();
  const bool ok = mbar_wait_for(&bar, 0, limit_ns);   // no thread ever arrives
  const uint64_t t1 = globaltimer_ns();
  if (!ok) raise_flag(err_flag, PA_FLAG_TIMEOUT);
  if (waited_ns) *waited_ns = (unsigned long long)(t1 - t0);
}

}  // namespace pa

using namespace pa;

extern "C" pa_status pa_selftest_wait_timeout(int32_t* err_flag, uint32_t limit_us,
                                              uint64_t* waited_ns, pa_stream_t stream) {
  if (limit_us == 0 || limit_us > 2000000u)
    return fail(PA_ERR_INVALID_ARG, "limit_us must be in [1, 2000000]");
  cudaError_t e = launch_pdl(selftest_wait_kernel, dim3(1), dim3(32), 0, (cudaStream_t)stream,
                             err_flag, (uint64_t)limit_us * 1000ull,
                             reinterpret_cast<unsigned long long*>(waited_ns));
  if (e != cudaSuccess) return cuda_fail(e, "selftest launch");
  return PA_OK;
}
