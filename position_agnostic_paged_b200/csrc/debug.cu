// debug.cu -- test export of the bounded pipeline wait that every
// warp-specialised kernel of the library uses (common.cuh: mbar_wait and
// wait_or_abort).  A kernel whose pipeline stalls -- a copy that never lands,
// a role that never arrives -- must give up, report LAZY_DSTATUS_TIMEOUT and
// exit with its context usable, never hang the GPU.  This kernel arms an
// mbarrier that nothing completes and waits on it with the caller's poll
// limit, the way a stalled consumer would, while a second role waits on
// another barrier and must leave as soon as the first role has aborted.
#include "common.cuh"
#include "kernels.h"

namespace lazy {
namespace {

// One CTA of two warps.  result[0] = 1 if the first role's wait ran out,
// result[1] = 1 if the second role left because of the abort flag.
// complete != 0 completes the first barrier before anyone waits (the normal
// case: the wait succeeds and nothing is reported).
__global__ void __launch_bounds__(64) debug_bounded_wait_kernel(uint32_t polls, int complete, int *result,
                                                                int *d_status) {
    __shared__ uint64_t bars[2];
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && complete) {
        mbar_arrive(&bars[0]);
        mbar_arrive(&bars[1]);
    }
    __syncthreads();
    if (lane == 0) {
        volatile int *flag = &abort_flag;
        if (warp == 0) {
            const bool ok = wait_or_abort(&bars[0], 0, flag, d_status, polls);
            result[0] = ok ? 0 : 1;
        } else {
            // bounded too (16x the first role's limit), but expected to end through the flag
            const bool ok = wait_or_abort(&bars[1], 0, flag, nullptr, 16u * polls);
            result[1] = (!ok && *flag) ? 1 : 0;
        }
    }
}

}  // namespace

cudaError_t launch_debug_bounded_wait(uint32_t polls, int complete, int *result, int *d_status, cudaStream_t s) {
    debug_bounded_wait_kernel<<<1, 64, 0, s>>>(polls, complete, result, d_status);
    return cudaGetLastError();
}

}  // namespace lazy

extern "C" int lazy_debug_bounded_wait(uint32_t polls, int complete, int32_t *result, int *d_status, void *stream) {
    if (!result || polls == 0 || polls > (1u << 24)) return LAZY_EINVAL;
    return lazy::launch_debug_bounded_wait(polls, complete, result, d_status, static_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? LAZY_OK
               : LAZY_ECUDA;
}
