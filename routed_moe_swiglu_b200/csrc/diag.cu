// diag.cu -- moe_check_bounded_wait: exercises, on the device, the bounded
// mbarrier wait that every pipeline wait of the GEMMs goes through, and the
// status word through which a kernel that gave up reports it.
//
// One CTA of two warps.  Nothing ever arrives on either of its two
// mbarriers.  Warp 0 waits with the caller's limit, gives up when it runs
// out, raises the CTA's abort flag and sets MOE_DEV_TIMEOUT; warp 1 waits
// with a limit a second longer and leaves as soon as it sees the abort flag
// (the route by which the other roles of a GEMM CTA stop when one role gave
// up).  Both record how long they waited.  The kernel then exits normally:
// no trap, no fault, and the context stays usable.
#include "moe_internal.cuh"
#include "ptx.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(64) bounded_wait_check_kernel(unsigned long long limit_ns, unsigned* status,
                                                                unsigned long long* elapsed_ns) {
    __shared__ __align__(8) uint64_t bars[2];
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
        volatile int* abort = &abort_flag;
        const unsigned long long t0 = global_timer_ns();
        // phase 0 of a fresh barrier completes only after an arrival, and none comes
        const bool got = mbar_wait_bounded(&bars[warp], 0u, abort,
                                           warp == 0 ? limit_ns : limit_ns + 1000000000ull);
        const unsigned long long dt = global_timer_ns() - t0;
        if (!got && warp == 0) {
            *abort = 1;
            atomicOr(status, MOE_DEV_TIMEOUT);
        }
        if (elapsed_ns != nullptr) elapsed_ns[warp] = dt;
    }
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_check_bounded_wait(unsigned long long limit_ns, unsigned* status_dev,
                                             unsigned long long* elapsed_ns_dev, void* stream) {
    if (status_dev == nullptr) return MOE_ERR_INVALID_ARG;
    if (limit_ns == 0 || limit_ns > 10000000000ull) return MOE_ERR_INVALID_ARG;
    moe::bounded_wait_check_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, status_dev,
                                                                                    elapsed_ns_dev);
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
