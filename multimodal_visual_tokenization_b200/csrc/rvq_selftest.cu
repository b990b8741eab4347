// rvq_selftest.cu -- a self-test of the bounded waits that every spin in the encode kernels uses
// (mbar_wait on a shared-memory mbarrier, wait_count on a global counter): one block waits on an
// mbarrier phase that nothing completes and on a counter that nothing increments, and reports
// through the device status word that both gave up after the limit instead of hanging.
#include "rvq.h"
#include "rvq_device.cuh"
#include "rvq_host.h"

namespace rvq {

__global__ void __launch_bounds__(64) selftest_wait_kernel(const uint32_t *counter, int32_t *status,
                                                           uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int flags[2];
  volatile int *abort_flag = reinterpret_cast<volatile int *>(&flags[0]);
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival would complete phase 0; none comes
    flags[0] = 0;
    flags[1] = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool got = mbar_wait(&bar, 0, abort_flag, limit_ns);
    if (!got) atomicAdd(&flags[1], 1);
  } else if (threadIdx.x == 32) {
    volatile int never = 0;  // a separate flag: the mbarrier wait's give-up must not end this one
    const bool got = wait_count(counter, 1u, counter, &never, limit_ns);
    if (!got) atomicAdd(&flags[1], 1);
  }
  __syncthreads();
  if (threadIdx.x == 0) set_status(status, flags[1] == 2 ? RVQ_ERR_TIMEOUT : RVQ_ERR_ARG);
}

}  // namespace rvq

extern "C" int rvq_selftest_wait_timeout(const uint32_t *counter, int32_t *status, int64_t limit_us, void *stream) {
  using namespace rvq;
  if (!counter || !status || limit_us < 1 || limit_us > 10000000) return RVQ_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(counter) & 3u) return RVQ_ERR_ARG;
  selftest_wait_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(counter, status,
                                                                         static_cast<uint64_t>(limit_us) * 1000u);
  note_launch();
  return check_launch();
}
