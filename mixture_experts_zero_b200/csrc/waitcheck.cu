// waitcheck.cu -- a device check of the bounded pipeline waits.
//
// Every mbarrier wait in the GEMMs and the row gather gives up after a time limit and records
// LC_MOE_DEV_WAIT_TIMEOUT (in the GEMMs the wait also raises its CTA's abort flag, which ends the
// other roles' waits), so that a stalled pipeline ends as a status the host reads instead of a
// hung context. This kernel runs the GEMMs' wait (mbar_wait of common.cuh) on a two-role pipeline
// whose first phase never completes, so a caller can see on its own device that the limit ends
// the wait and that the abort reaches the other role:
//   - role 0 waits for phase 0 of bars[0], on which nothing ever arrives, with the limit; it
//     gives up, raises the abort flag and records WAIT_TIMEOUT. (Had it completed, it would have
//     arrived on bars[1].)
//   - role 1 waits for phase 0 of bars[1] with four times the limit, and leaves through the
//     abort flag role 0 raised, after about one limit rather than four.
// Both waits are bounded by their own clocks, so the kernel ends within four limits whatever
// happens.
#include "common.cuh"

namespace lcmoe {

namespace {

__global__ void __launch_bounds__(64) wait_check_kernel(uint32_t* status, uint64_t limit_ns) {
    __shared__ uint64_t bars[2];
    __shared__ int abort_word;
    volatile int* abort_flag = &abort_word;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (lane == 0) {
        if (warp == 0) {
            if (mbar_wait(&bars[0], 0, limit_ns, abort_flag, status)) mbar_arrive(&bars[1]);
        } else {
            mbar_wait(&bars[1], 0, 4 * limit_ns, abort_flag, status);
        }
    }
    __syncthreads();
}

}  // namespace

cudaError_t launch_wait_check(uint32_t* status, uint64_t limit_ns, cudaStream_t st) {
    wait_check_kernel<<<1, 64, 0, st>>>(status, limit_ns);
    return cudaGetLastError();
}

}  // namespace lcmoe
