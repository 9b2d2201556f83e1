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
