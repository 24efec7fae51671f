// Self-test of the bounded pipeline waits every tensor-core kernel uses.
#include "tc_ptx.cuh"

namespace {

// One thread waits on an mbarrier that nothing arrives at; the bounded wait
// gives up after `limit` cycles, raises HGA_DEV_TIMEOUT and the kernel ends.
__global__ void wait_timeout_kernel(long long limit, unsigned *status) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        hga::tc::mbar_init(&bar, 1);
        abort_flag = 0;
        hga::tc::fence_mbar_init();
        volatile int *ab = &abort_flag;
        hga::tc::mbar_wait(&bar, 0, ab, status, limit);
    }
}

}  // namespace

namespace hga {
hga_status_t launch_selftest_wait_timeout(long long wait_cycles, unsigned *status, cudaStream_t stream) {
    wait_timeout_kernel<<<1, 32, 0, stream>>>(wait_cycles, status);
    return record_cuda(cudaGetLastError());
}
}  // namespace hga
