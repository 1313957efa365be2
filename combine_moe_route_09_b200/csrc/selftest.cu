// Self-test of the bounded waits: one thread runs a wait that nothing will
// complete -- an mbarrier phase with no arrival, or a global word that nothing
// writes -- with a short limit, so that the wait runs out, sets
// MOE_STATUS_TIMEOUT and returns.  These are the same wait routines every
// kernel of the library uses; nothing is left in flight and the context stays
// usable.
#include "common.cuh"
#include "kernels.cuh"
#include "tma.cuh"

namespace moe {

__global__ void wait_selftest_kernel(int which, unsigned long long limit_ns, int32_t *status, const unsigned *flag) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    if (which == 0) {
        const uint32_t b = smem_addr(&bar);
        mbar_init(b, 1);
        fence_mbar_init();
        (void)mbar_wait_for(b, 0, status, limit_ns);  // no thread arrives
    } else {
        (void)wait_changed_for(flag, *(const volatile unsigned *)flag, status, limit_ns);  // nothing writes it
    }
}

cudaError_t launch_wait_selftest(int which, unsigned long long limit_ns, int32_t *status, const unsigned *flag,
                                 cudaStream_t st) {
    wait_selftest_kernel<<<1, 32, 0, st>>>(which, limit_ns, status, flag);
    return cudaGetLastError();
}

}  // namespace moe
