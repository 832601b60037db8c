// Failure-path self test: a kernel whose one bounded mbarrier wait nothing ever
// completes.  It exercises the wait every pass uses: after the limit the wait
// gives up, the kernel raises kDevErrTimeout and returns normally, so the host
// reads FS_ERR_TIMEOUT and the context stays usable.  No copy, MMA or TMEM is
// involved, so giving up leaves nothing in flight.
#include "fs_tc_common.cuh"

namespace fs {
namespace {

__global__ void wait_probe_kernel(unsigned long long timeout_ns, int *err) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0 && !tc::mbar_wait(&bar, 0, timeout_ns)) atomicOr(err, kDevErrTimeout);
}

}  // namespace

cudaError_t launch_wait_probe(unsigned long long timeout_ns, int *err, cudaStream_t s) {
    wait_probe_kernel<<<1, 32, 0, s>>>(timeout_ns, err);
    return cudaGetLastError();
}

}  // namespace fs
