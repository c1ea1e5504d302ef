// kvq_selftest.cu -- failure-detection self-test of the bounded waits.
//
// Runs the library's own bounded mbarrier wait on a barrier that nothing
// ever arrives at.  The wait must give up after `limit_ns` and the kernel
// report KVQ_DEV_TIMEOUT in the caller's status word; the CUDA context stays
// usable.  This is how the timeout path of the attention and append kernels
// is exercised without making any real transfer fail.
#include "kvq_common.cuh"
#include "kvq_internal.h"
#include "kvq_sync.cuh"

namespace kvq {

__global__ void wait_timeout_selftest_kernel(int32_t* status, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    __syncthreads();
    // phase 0 never completes: no thread arrives and no copy is issued
    const bool done = mbar_wait(&bar, 0, limit_ns);
    if (!done && threadIdx.x == 0) set_status(status, KVQ_DEV_TIMEOUT);
}

kvq_status selftest_wait_timeout(int32_t* status, long long limit_ns, cudaStream_t st) {
    wait_timeout_selftest_kernel<<<1, 32, 0, st>>>(status, (unsigned long long)limit_ns);
    return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ECUDA;
}

}  // namespace kvq
