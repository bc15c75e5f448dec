// selftest.cu -- ssd_selftest_bounded_wait: makes a bounded device wait run
// out on purpose, so that a test can check that the give-up path reports
// SSD_ERR_TIMEOUT and leaves the context usable, without any fault.
//
// One thread initialises an mbarrier that expects one arrival, never
// arrives on it, and waits on it with mbar_wait_bounded -- the helper every
// mbarrier wait of the tensor-core scan goes through -- for limit_ns.  The
// helper gives up after the limit, writes SSD_ERR_TIMEOUT into *status and
// marks the CTA aborted; a second wait then returns at once instead of
// waiting again, which the kernel checks too.
#include "ssd.h"
#include "sm100.cuh"

namespace {

using namespace ssd::sm100;

__global__ void bounded_wait_selftest_kernel(int32_t* status, uint64_t limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ int aborted_flag;
    volatile int* aborted = &aborted_flag;
    *aborted = 0;
    mbar_init(&bar, 1);
    fence_mbar_init();
    const uint64_t t0 = globaltimer_ns();
    const bool first = mbar_wait_bounded(&bar, 0u, limit_ns, aborted, status);
    const uint64_t t1 = globaltimer_ns();
    const bool second = mbar_wait_bounded(&bar, 0u, limit_ns, aborted, status);
    const uint64_t t2 = globaltimer_ns();
    // a wait that succeeded, a give-up before the limit, a missing abort
    // mark or a second wait that waited again are all reported as errors
    const bool ok = !first && !second && *aborted == 1 && t1 - t0 >= limit_ns && t2 - t1 < limit_ns;
    if (!ok) atomicExch(reinterpret_cast<int*>(status), (int)SSD_ERR_CUDA);
}

}  // namespace

extern "C" SSD_API ssd_status_t ssd_selftest_bounded_wait(int32_t* status, uint64_t limit_ns,
                                                          cudaStream_t stream)
{
    if (!status || limit_ns == 0 || limit_ns > 1000000000ull) return SSD_ERR_INVALID_ARG;
    bounded_wait_selftest_kernel<<<1, 1, 0, stream>>>(status, limit_ns);
    return cudaGetLastError() == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
