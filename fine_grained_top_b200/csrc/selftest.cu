// selftest.cu -- a health check of the bounded-wait machinery.
//
// Every pipeline wait in the library gives up after a time limit and reports
// SA_DEV_TIMEOUT instead of hanging the GPU.  sa_selftest_wait_timeout runs
// one thread that waits on a shared-memory mbarrier that nothing ever arrives
// at, with the caller's (short) limit, so a caller can check that a stalled
// wait comes back as a status word and the context stays usable.
#include "internal.h"
#include "ptx.cuh"

namespace sa {

__global__ void wait_timeout_kernel(unsigned long long limit_ns, int *dev_status) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);       // expects one arrival; none will come
    fence_mbar_init();
    abort_flag = 0;
    if (!mbar_wait(&bar, 0u, &abort_flag, limit_ns)) report(dev_status, SA_DEV_TIMEOUT);
}

}  // namespace sa

extern "C" sa_status sa_selftest_wait_timeout(int limit_us, int *dev_status, sa_stream stream) {
    if (limit_us <= 0 || limit_us > 1000000 || !dev_status) return SA_ERR_INVALID_ARG;
    sa::wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        (unsigned long long)limit_us * 1000ull, dev_status);
    return sa::cuda_ok(cudaGetLastError());
}
