// gdn_selftest.cu -- self-test of the bounded device-side waits that every
// warp-specialised kernel of this library relies on instead of spinning
// forever: one CTA waits on an mbarrier phase that nothing completes and on a
// hand-over counter that nothing publishes, with the library's own wait
// helpers. Both waits must give up after their limit and record
// GDN_ERR_TIMEOUT in the status word; nothing else is in flight (no TMA, no
// tensor-core MMA), so the CTA then exits normally and the context stays
// usable.
#include "gdn_internal.cuh"
#include "gdn_warp.cuh"
#include "sm100_ptx.cuh"

namespace gdn {
namespace {

__global__ void __launch_bounds__(64) wait_selftest_kernel(uint64_t limit_ns, unsigned long long *elapsed,
                                                          unsigned *status) {
    __shared__ uint64_t bar;
    __shared__ uint32_t ctr;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);
        ctr = 0;
        abort_flag = 0;
        sm100::fence_barrier_init();
    }
    __syncthreads();
    const int role = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
        const uint64_t t0 = warp::globaltimer();
        // phase 0 of a fresh barrier with one expected arrival, which never comes;
        // a counter that stays at 0
        const bool ok = role == 0 ? warp::wait_bar(&bar, 0, &abort_flag, limit_ns)
                                  : warp::wait_ge(&ctr, 1, &abort_flag, limit_ns);
        const uint64_t t1 = warp::globaltimer();
        elapsed[role] = ok ? ~0ull : (unsigned long long)(t1 - t0);
        if (!ok) set_status(status, GDN_ERR_TIMEOUT);
    }
    __syncthreads();
}

}  // namespace

cudaError_t launch_wait_selftest(uint64_t limit_ns, unsigned long long *elapsed, unsigned *status,
                                 cudaStream_t stream) {
    wait_selftest_kernel<<<1, 64, 0, stream>>>(limit_ns ? limit_ns : warp::kWaitNs, elapsed, status);
    return cudaGetLastError();
}

}  // namespace gdn
