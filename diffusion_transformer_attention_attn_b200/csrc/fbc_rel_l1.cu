// First-block-cache residual difference on sm_100a:
//   rel = Σ|r_cur − r_prev| / Σ|r_prev|,  skip = rel < threshold.
// "ParaAttention" (diffusers docs), section "First Block Cache": the relative
// L1 change of the first transformer block's residual between two denoising
// steps decides whether the remaining blocks run or the cached residual is
// reused.
//
// One launch, HBM-bound: every thread streams 16-byte vectors of both inputs
// (grid-stride, four vectors in flight per array), sums |cur − prev| and
// |prev| in fp32 over at most 32 elements before folding into fp64, and the
// block reduces in fp64 with warp shuffles.  Each block writes its two
// partial sums to the workspace; the last block to finish (a ticket counter)
// adds the partials in block order, writes rel and skip, and re-zeroes the
// ticket.  The grid size depends on n only, so the summation order, and the
// result, are the same on every run.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "dit_attn.h"
#include "internal.h"

namespace ditk {
namespace {

constexpr int kFbcThreads = 512;
constexpr int kFbcMaxBlocks = 1024;
constexpr int kUnroll = 4;

struct FbcWs {
    unsigned int ticket;
    unsigned int pad[3];
    // followed by double2 partials[kFbcMaxBlocks]
};

__device__ __forceinline__ void acc_vec(const float4& c, const float4& p, float& num, float& den) {
    num += fabsf(c.x - p.x) + fabsf(c.y - p.y) + fabsf(c.z - p.z) + fabsf(c.w - p.w);
    den += fabsf(p.x) + fabsf(p.y) + fabsf(p.z) + fabsf(p.w);
}
__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }
__device__ __forceinline__ void acc_vec(const uint4& c, const uint4& p, float& num, float& den) {
    const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
    const uint32_t pw[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float c0 = bf_lo(cw[i]), c1 = bf_hi(cw[i]);
        const float p0 = bf_lo(pw[i]), p1 = bf_hi(pw[i]);
        num += fabsf(c0 - p0) + fabsf(c1 - p1);
        den += fabsf(p0) + fabsf(p1);
    }
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Deterministic block sum of (a, b) in fp64; result valid in thread 0.
__device__ __forceinline__ void block_sum2(double& a, double& b, double2* sh) {
    a = warp_sum(a);
    b = warp_sum(b);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) sh[warp] = make_double2(a, b);
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        double2 v = lane < nw ? sh[lane] : make_double2(0.0, 0.0);
        a = warp_sum(v.x);
        b = warp_sum(v.y);
    }
}

// VecT: float4 (fp32 inputs, 4 elements) or uint4 (bf16 inputs, 8 elements).
template <typename VecT, int kElems>
__global__ void __launch_bounds__(kFbcThreads)
    fbc_rel_l1_kernel(const VecT* __restrict__ cur, const VecT* __restrict__ prev, int64_t nvec,
                      const void* __restrict__ cur_tail, const void* __restrict__ prev_tail, int tail, float threshold,
                      double* __restrict__ out_rel, int32_t* __restrict__ out_skip, FbcWs* ws) {
    __shared__ double2 sh[kFbcThreads / 32];
    __shared__ bool is_last;
    double2* partials = reinterpret_cast<double2*>(ws + 1);

    double num = 0.0, den = 0.0;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    for (; i + (kUnroll - 1) * stride < nvec; i += kUnroll * stride) {
        VecT c[kUnroll], p[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            c[u] = __ldcs(cur + i + u * stride);
            p[u] = __ldcs(prev + i + u * stride);
        }
        float fn = 0.f, fd = 0.f;
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) acc_vec(c[u], p[u], fn, fd);
        num += fn;
        den += fd;
    }
    for (; i < nvec; i += stride) {
        float fn = 0.f, fd = 0.f;
        acc_vec(__ldcs(cur + i), __ldcs(prev + i), fn, fd);
        num += fn;
        den += fd;
    }
    // Elements past the last whole vector (fewer than kElems) go to thread 0 of block 0.
    if (blockIdx.x == 0 && threadIdx.x == 0 && tail > 0) {
        for (int t = 0; t < tail; ++t) {
            float c, p;
            if (kElems == 4) {
                c = static_cast<const float*>(cur_tail)[t];
                p = static_cast<const float*>(prev_tail)[t];
            } else {
                c = __bfloat162float(static_cast<const __nv_bfloat16*>(cur_tail)[t]);
                p = __bfloat162float(static_cast<const __nv_bfloat16*>(prev_tail)[t]);
            }
            num += fabsf(c - p);
            den += fabsf(p);
        }
    }
    block_sum2(num, den, sh);
    if (threadIdx.x == 0) {
        partials[blockIdx.x] = make_double2(num, den);
        __threadfence();
        const unsigned int t = atomicAdd(&ws->ticket, 1u);
        is_last = (t == gridDim.x - 1);
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    // Last block: fixed-order sum of the partials.
    double a = 0.0, b = 0.0;
    for (int k = threadIdx.x; k < static_cast<int>(gridDim.x); k += blockDim.x) {
        const double2 v = __ldcg(&partials[k]);
        a += v.x;
        b += v.y;
    }
    __syncthreads();
    block_sum2(a, b, sh);
    if (threadIdx.x == 0) {
        double rel;
        if (b > 0.0)
            rel = a / b;
        else
            rel = (a > 0.0) ? HUGE_VAL : 0.0;
        *out_rel = rel;
        *out_skip = (rel < static_cast<double>(threshold)) ? 1 : 0;
        ws->ticket = 0u;
    }
}

int fbc_blocks(int64_t nvec) {
    int64_t per = static_cast<int64_t>(kFbcThreads) * kUnroll;
    int64_t nb = (nvec + per - 1) / per;
    if (nb < 1) nb = 1;
    if (nb > kFbcMaxBlocks) nb = kFbcMaxBlocks;
    return static_cast<int>(nb);
}

}  // namespace

size_t fbc_workspace_bytes(int64_t /*n*/) {
    return sizeof(FbcWs) + sizeof(double2) * kFbcMaxBlocks;
}

cudaError_t launch_fbc_rel_l1(const void* cur, const void* prev, int64_t n, int dtype, float threshold,
                              double* out_rel, int32_t* out_skip, void* workspace, cudaStream_t stream) {
    FbcWs* ws = static_cast<FbcWs*>(workspace);
    if (dtype == 0) {
        const int64_t nvec = n / 4;
        const int tail = static_cast<int>(n - nvec * 4);
        const float* c = static_cast<const float*>(cur);
        const float* p = static_cast<const float*>(prev);
        fbc_rel_l1_kernel<float4, 4><<<fbc_blocks(nvec), kFbcThreads, 0, stream>>>(
            reinterpret_cast<const float4*>(c), reinterpret_cast<const float4*>(p), nvec, c + nvec * 4,
            p + nvec * 4, tail, threshold, out_rel, out_skip, ws);
    } else {
        const int64_t nvec = n / 8;
        const int tail = static_cast<int>(n - nvec * 8);
        const __nv_bfloat16* c = static_cast<const __nv_bfloat16*>(cur);
        const __nv_bfloat16* p = static_cast<const __nv_bfloat16*>(prev);
        fbc_rel_l1_kernel<uint4, 8><<<fbc_blocks(nvec), kFbcThreads, 0, stream>>>(
            reinterpret_cast<const uint4*>(c), reinterpret_cast<const uint4*>(p), nvec, c + nvec * 8,
            p + nvec * 8, tail, threshold, out_rel, out_skip, ws);
    }
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
