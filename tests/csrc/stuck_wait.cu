// Test-only kernel for the device status path: a bounded wait that runs out.
//
// One block initialises an mbarrier that expects one arrival which nobody
// makes, and every thread waits on it through the library's own bounded wait
// (mbar_wait) with a small poll limit.  The wait gives up, the block records
// the scan's timeout code in the status word with the library's flag_error --
// the same steps the tensor-core scan takes when one of its waits gives up --
// and returns.  Nothing is in flight when it gives up (no copy, no tensor-core
// product), so the kernel ends by itself and the context stays usable.
//
// A second kernel makes the range check of the bounds-checked build fail on
// purpose (an index past the size it is checked against; the access it guards
// is skipped) and records GDN_DEV_BOUNDS the same way.
//
// Built by the tests (with -DGDN_CHECKED) into their own small library, apart
// from libgdn.so.
#include <cuda_runtime.h>

#include "tc_common.cuh"

using namespace gdn;
using namespace gdn::sm100;

__global__ void gdn_test_stuck_wait_kernel(int *status, uint32_t limit, int *polls_gave_up) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    const bool ok = mbar_wait(&bar, 0, limit);
    if (__syncthreads_or(!ok)) {
        if (threadIdx.x == 0) {
            tc::flag_error(status, GDN_DEV_TIMEOUT_SCAN);
            *polls_gave_up = 1;
        }
    }
}

__global__ void gdn_test_bounds_kernel(int *status, int64_t index, int64_t size, float *dst) {
    if (in_bounds(index >= 0 && index < size, status)) dst[index] = 1.f;
}

extern "C" int gdn_test_bounds(int *status, int64_t index, int64_t size, float *dst, cudaStream_t stream) {
    gdn_test_bounds_kernel<<<1, 32, 0, stream>>>(status, index, size, dst);
    return (int)cudaGetLastError();
}

extern "C" int gdn_test_stuck_wait(int *status, uint32_t limit, int *gave_up, cudaStream_t stream) {
    gdn_test_stuck_wait_kernel<<<1, 128, 0, stream>>>(status, limit, gave_up);
    return (int)cudaGetLastError();
}
