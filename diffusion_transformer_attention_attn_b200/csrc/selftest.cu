// Self-test of the bounded wait that every kernel of this library relies on.
// One warp waits on an mbarrier that nothing ever arrives on.  The wait gives
// up after the limit in sm100_ptx.cuh (1 s of %globaltimer), records
// DIT_ERR_TIMEOUT in the device error word, and the kernel returns: the
// failure is reported, and the GPU context stays usable.
#include <cuda_runtime.h>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace ditk {
namespace {

__global__ void wait_selftest_kernel(int* err, int32_t* completed) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncwarp();
    // Phase 0 of a barrier that expects one arrival, and gets none, never
    // completes.
    const bool ok = mbar_wait(&bar, 0, &abort_flag, err);
    if (threadIdx.x == 0) *completed = ok ? 1 : 0;
}

}  // namespace

cudaError_t launch_wait_selftest(int* err, int32_t* completed, cudaStream_t stream) {
    wait_selftest_kernel<<<1, 32, 0, stream>>>(err, completed);
    return cudaGetLastError();
}

}  // namespace ditk
