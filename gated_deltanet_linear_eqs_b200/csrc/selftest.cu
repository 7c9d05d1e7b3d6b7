// selftest.cu -- a kernel whose bounded wait is made to run out.
//
// Every wait in the library's kernels is bounded: when it gives up, the kernel records
// GDN_ERR_TIMEOUT in the device status word, unwinds and returns, so that a lost arrival
// becomes an error the host can read instead of a hung GPU.  This kernel takes that path on
// purpose, safely: one thread waits, with a short limit, on an mbarrier that nothing arrives
// on (a flag that nothing sets).  Nothing else is touched, so the context stays usable.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace gdn {

namespace {

using namespace sm100;

__global__ void __launch_bounds__(32) wait_timeout_kernel(int* status, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int never;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);  // expects one arrival; none ever comes
        never = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 &&
        !mbar_wait(&bar, 0, reinterpret_cast<volatile int*>(&never), limit_ns))
        record_status(status, GDN_ERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(int* status, unsigned long long limit_ns, cudaStream_t st) {
    wait_timeout_kernel<<<1, 32, 0, st>>>(status, limit_ns);
    return cudaGetLastError();
}

}  // namespace gdn
