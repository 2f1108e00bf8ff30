// Self-test of the bounded pipeline wait (mbar_wait_bounded), the one every
// TMA / tensor-core kernel of the library uses: a CTA waits on an mbarrier
// phase that nothing completes, so the wait must give up on its own -- after
// its time limit, or as soon as another warp sets the abort flag -- record
// PA_DEVERR_TIMEOUT in the device error word and return, leaving the context
// usable.  Every wait and spin in it ends by itself.
#include "common.cuh"
#include "launch.h"

namespace pa {

__global__ void wait_selftest_kernel(unsigned int *err, uint64_t limit_ns, uint64_t abort_after_ns,
                                     unsigned long long *elapsed_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);  // one arrival expected; none comes
        abort_flag = 0;
        fence_mbarrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 32 && abort_after_ns) {
        // a second warp raises the abort flag after abort_after_ns
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 < abort_after_ns) {
        }
        *reinterpret_cast<volatile int *>(&abort_flag) = 1;
    }
    if (threadIdx.x == 0) {
        const uint64_t t0 = global_timer_ns();
        const bool ok = mbar_wait_bounded(smem_u32(&bar), 0,
                                          reinterpret_cast<volatile int *>(&abort_flag), limit_ns);
        *elapsed_ns = global_timer_ns() - t0;
        if (!ok) raise_device_error(err, PA_DEVERR_TIMEOUT);
    }
}

cudaError_t launch_wait_selftest(unsigned int *err, uint64_t limit_ns, uint64_t abort_after_ns,
                                 unsigned long long *elapsed_ns, cudaStream_t stream) {
    wait_selftest_kernel<<<1, 64, 0, stream>>>(err, limit_ns, abort_after_ns, elapsed_ns);
    return cudaGetLastError();
}

}  // namespace pa
