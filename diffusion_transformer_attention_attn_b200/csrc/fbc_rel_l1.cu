// First-block-cache residual difference on sm_100a:
//   rel = Σ|r_cur − r_prev| / Σ|r_prev|,  skip = rel < threshold.
// "ParaAttention" (diffusers docs), section "First Block Cache": the relative
// L1 change of the first transformer block's residual between two denoising
// steps decides whether the remaining blocks run or the cached residual is
// reused.
//
// One HBM-bound launch of the shared relative-L1 reduction (rel_l1_reduce.cuh)
// whose epilogue writes rel and skip, launched so that it overlaps the tail of
// the kernel before it (programmatic launch with an L2 prefetch of its first
// loads).
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "dit_attn.h"
#include "internal.h"
#include "rel_l1_reduce.cuh"

namespace ditk {
namespace {

struct EpiThreshold {
    static constexpr bool kProgrammatic = true;
    float threshold;
    double* out_rel;
    int32_t* out_skip;
    __device__ bool evaluate() const { return true; }
    __device__ void finish(double num, double den, bool) const {
        const double rel = rl1_ratio(num, den);
        *out_rel = rel;
        *out_skip = (rel < static_cast<double>(threshold)) ? 1 : 0;
    }
};

// The two sums themselves (for a residual sharded across devices).
struct EpiSums {
    static constexpr bool kProgrammatic = true;
    double* out;
    __device__ bool evaluate() const { return true; }
    __device__ void finish(double num, double den, bool) const {
        out[0] = num;
        out[1] = den;
    }
};

__global__ void fbc_finish_kernel(const double* __restrict__ sums, float threshold, double* __restrict__ out_rel,
                                  int32_t* __restrict__ out_skip) {
    if (threadIdx.x == 0 && blockIdx.x == 0) {
        const double rel = rl1_ratio(sums[0], sums[1]);
        *out_rel = rel;
        *out_skip = (rel < static_cast<double>(threshold)) ? 1 : 0;
    }
}

}  // namespace

size_t fbc_workspace_bytes(int64_t /*n*/) {
    return sizeof(FbcWs) + sizeof(double2) * kFbcMaxBlocks;
}

cudaError_t launch_fbc_rel_l1(const void* cur, const void* prev, int64_t n, int dtype, float threshold,
                              double* out_rel, int32_t* out_skip, void* workspace, cudaStream_t stream) {
    return launch_rel_l1<false>(cur, prev, n, dtype, EpiThreshold{threshold, out_rel, out_skip}, workspace, stream);
}

cudaError_t launch_fbc_sums(const void* cur, const void* prev, int64_t n, int dtype, double* out_sums,
                            void* workspace, cudaStream_t stream) {
    return launch_rel_l1<false>(cur, prev, n, dtype, EpiSums{out_sums}, workspace, stream);
}

cudaError_t launch_fbc_finish(const double* sums, float threshold, double* out_rel, int32_t* out_skip,
                              cudaStream_t stream) {
    fbc_finish_kernel<<<1, 32, 0, stream>>>(sums, threshold, out_rel, out_skip);
    return cudaGetLastError();
}

}  // namespace ditk

// ---------------------------------------------------------------------------
// fbc_rel_l1_noalloc: the same reduction for callers that cannot allocate
// device memory.  Such callers hold only their input and output pointers: a
// plugin run by an inference engine, or a module inside a framework whose
// caching allocator owns all device memory.  cudaMalloc is either unavailable
// to them or costs an implicit device-wide synchronisation they cannot take
// inside a denoising step.  The kernel's scratch (the finishing ticket and one
// partial-sum pair per block) lives in the file-scope array below.  Every GPU
// that loads the library holds that array until the process exits.

namespace ditk {
namespace {

// Scratch capacity: the ticket plus the partials of the largest grid the
// kernel launches (kFbcMaxBlocks blocks), i.e. 16 KiB + 16 B.
constexpr size_t kNoAllocScratchBytes = sizeof(FbcWs) + sizeof(double2) * kFbcMaxBlocks;
static __device__ __align__(256) unsigned char g_fbc_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
struct NoAllocDevice {
    std::once_flag once;
    cudaError_t err = cudaSuccess;
    bool sm100 = false;
    void* scratch = nullptr;  // device address of g_fbc_noalloc_scratch on this device
};
NoAllocDevice g_noalloc_dev[kNoAllocMaxDevices];

// Once per device, with that device current: look up the device address of
// the scratch array.  In host code the array's name is only a host-side
// stand-in, so kernels must be given this address, never the name.
NoAllocDevice* noalloc_setup(int dev) {
    NoAllocDevice& d = g_noalloc_dev[dev];
    std::call_once(d.once, [&d, dev] {
        cudaDeviceProp prop;
        d.err = cudaGetDeviceProperties(&prop, dev);
        if (d.err != cudaSuccess) return;
        d.sm100 = (prop.major == 10 && prop.minor == 0);
        d.err = cudaGetSymbolAddress(&d.scratch, g_fbc_noalloc_scratch);
    });
    return &d;
}

}  // namespace
}  // namespace ditk

extern "C" dit_status fbc_rel_l1_noalloc(const void* r_cur, const void* r_prev, int64_t n, int dtype,
                                         float threshold, double* out_rel, int32_t* out_skip, void* stream) {
    using namespace ditk;
    if (!r_cur || !r_prev || !out_rel || !out_skip || n < 1) return DIT_ERR_INVALID_ARG;
    if (dtype != DIT_DTYPE_F32 && dtype != DIT_DTYPE_BF16) return DIT_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(r_cur) & 15u) != 0 || (reinterpret_cast<uintptr_t>(r_prev) & 15u) != 0)
        return DIT_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(out_rel) & 7u) != 0 || (reinterpret_cast<uintptr_t>(out_skip) & 3u) != 0)
        return DIT_ERR_INVALID_ARG;
    if (!(threshold == threshold)) return DIT_ERR_INVALID_ARG;
    // The request must fit the fixed scratch array.
    if (fbc_workspace_bytes(n) > kNoAllocScratchBytes) return DIT_ERR_WORKSPACE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) return DIT_ERR_CUDA;
    NoAllocDevice* d = noalloc_setup(dev);
    if (d->err != cudaSuccess || !d->scratch) return DIT_ERR_CUDA;
    if (!d->sm100) return DIT_ERR_UNSUPPORTED;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    // The ticket must start at zero.  A completed call leaves it at zero, and
    // this clear also covers a call that never finished.
    if (cudaMemsetAsync(d->scratch, 0, sizeof(FbcWs), s) != cudaSuccess) return DIT_ERR_CUDA;
    cudaError_t e = launch_fbc_rel_l1(r_cur, r_prev, n, dtype, threshold, out_rel, out_skip, d->scratch, s);
    return e == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}
