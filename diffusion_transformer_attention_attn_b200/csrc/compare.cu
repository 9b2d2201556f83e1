// Error of one output against a reference, per contiguous segment
// (declared in include/dit_attn.h as dit_compare_stats).
//
// TMAP image-to-video blog, "keeping video quality": plotting the attention
// error of every layer over the denoising steps singled out the layers whose
// 8-bit attention is switched back to 16 bits.  This call measures that error
// on the device, so a per-layer probe costs one read of both outputs and no
// host copy of them:
//   rel_l1 = Σ|test − ref| / Σ|ref|
//   cosine = Σ ref·test / sqrt(Σ ref² · Σ test²)
//   max_abs = max |test − ref|
//
// HBM-bound, one launch.  Grid (blocks per segment, segments).  Each thread
// reads 16-byte vectors of both inputs, forms the five sums of a vector in
// fp32 and folds them into fp64; blocks reduce in fp64; the last block of a
// segment (a ticket per segment) adds that segment's partials in block order
// and writes its three results.  The grid depends on the shape only, so the
// results are the same on every run.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "dit_attn.h"
#include "internal.h"

namespace ditk {
namespace {

constexpr int kCmpThreads = 256;
constexpr int kCmpUnroll = 2;
constexpr int kCmpMaxBlocks = 2048;  // all segments together
constexpr int kCmpSums = 6;          // |d|, |ref|, ref·test, ref², test², max|d|

struct Acc {
    double s[kCmpSums];
};

__device__ __forceinline__ void acc_elem(float a, float b, float (&f)[kCmpSums]) {
    const float dlt = fabsf(b - a);
    f[0] += dlt;
    f[1] += fabsf(a);
    f[2] += a * b;
    f[3] += a * a;
    f[4] += b * b;
    f[5] = fmaxf(f[5], dlt);
}

__device__ __forceinline__ void fold(const float (&f)[kCmpSums], Acc& acc) {
#pragma unroll
    for (int k = 0; k < 5; ++k) acc.s[k] += static_cast<double>(f[k]);
    acc.s[5] = fmax(acc.s[5], static_cast<double>(f[5]));
}

__device__ __forceinline__ float bf(uint16_t u) { return __uint_as_float(static_cast<uint32_t>(u) << 16); }

template <bool kBf16>
__device__ __forceinline__ void acc_vec(const uint4& a, const uint4& b, Acc& acc) {
    float f[kCmpSums] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
    const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (kBf16) {
            acc_elem(__uint_as_float(aw[i] << 16), __uint_as_float(bw[i] << 16), f);
            acc_elem(__uint_as_float(aw[i] & 0xFFFF0000u), __uint_as_float(bw[i] & 0xFFFF0000u), f);
        } else {
            acc_elem(__uint_as_float(aw[i]), __uint_as_float(bw[i]), f);
        }
    }
    fold(f, acc);
}

__device__ __forceinline__ double warp_red(double v, bool is_max) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const double w = __shfl_xor_sync(0xffffffffu, v, o);
        v = is_max ? fmax(v, w) : v + w;
    }
    return v;
}

// Block reduction of the six accumulators; valid in thread 0.
__device__ __forceinline__ void block_red(Acc& acc, double (*sh)[kCmpSums]) {
#pragma unroll
    for (int k = 0; k < kCmpSums; ++k) acc.s[k] = warp_red(acc.s[k], k == 5);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
#pragma unroll
        for (int k = 0; k < kCmpSums; ++k) sh[warp][k] = acc.s[k];
    }
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
#pragma unroll
        for (int k = 0; k < kCmpSums; ++k) acc.s[k] = warp_red(lane < nw ? sh[lane][k] : 0.0, k == 5);
    }
}

// kVec: every segment starts 16-byte aligned and holds whole 16-byte vectors.
template <bool kBf16, bool kVec>
__global__ void __launch_bounds__(kCmpThreads)
    compare_kernel(const void* __restrict__ ref, const void* __restrict__ test, int64_t seg_len,
                   double* __restrict__ out, unsigned int* tickets, Acc* partials) {
    __shared__ double sh[kCmpThreads / 32][kCmpSums];
    __shared__ bool is_last;
    const int seg = blockIdx.y;
    const int nb = gridDim.x;
    const int esz = kBf16 ? 2 : 4;
    const char* ra = static_cast<const char*>(ref) + static_cast<int64_t>(seg) * seg_len * esz;
    const char* tb = static_cast<const char*>(test) + static_cast<int64_t>(seg) * seg_len * esz;

    Acc acc;
#pragma unroll
    for (int k = 0; k < kCmpSums; ++k) acc.s[k] = 0.0;
    const int64_t stride = static_cast<int64_t>(nb) * blockDim.x;
    int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (kVec) {
        const int64_t nvec = seg_len * esz / 16;
        const uint4* a4 = reinterpret_cast<const uint4*>(ra);
        const uint4* b4 = reinterpret_cast<const uint4*>(tb);
        for (; i + (kCmpUnroll - 1) * stride < nvec; i += kCmpUnroll * stride) {
            uint4 a[kCmpUnroll], b[kCmpUnroll];
#pragma unroll
            for (int u = 0; u < kCmpUnroll; ++u) {
                a[u] = __ldcs(a4 + i + u * stride);
                b[u] = __ldcs(b4 + i + u * stride);
            }
#pragma unroll
            for (int u = 0; u < kCmpUnroll; ++u) acc_vec<kBf16>(a[u], b[u], acc);
        }
        for (; i < nvec; i += stride) acc_vec<kBf16>(__ldcs(a4 + i), __ldcs(b4 + i), acc);
    } else {
        for (; i < seg_len; i += stride) {
            float f[kCmpSums] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (kBf16)
                acc_elem(bf(reinterpret_cast<const uint16_t*>(ra)[i]), bf(reinterpret_cast<const uint16_t*>(tb)[i]),
                         f);
            else
                acc_elem(reinterpret_cast<const float*>(ra)[i], reinterpret_cast<const float*>(tb)[i], f);
            fold(f, acc);
        }
    }
    block_red(acc, sh);
    Acc* part = partials + static_cast<int64_t>(seg) * nb;
    if (threadIdx.x == 0) {
        part[blockIdx.x] = acc;
        __threadfence();
        const unsigned int t = atomicAdd(&tickets[seg], 1u);
        is_last = (t == static_cast<unsigned int>(nb - 1));
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    Acc tot;
#pragma unroll
    for (int k = 0; k < kCmpSums; ++k) tot.s[k] = 0.0;
    for (int b = threadIdx.x; b < nb; b += blockDim.x) {
#pragma unroll
        for (int k = 0; k < kCmpSums; ++k) {
            const double v = __ldcg(&part[b].s[k]);
            tot.s[k] = k == 5 ? fmax(tot.s[k], v) : tot.s[k] + v;
        }
    }
    __syncthreads();
    block_red(tot, sh);
    if (threadIdx.x == 0) {
        const double num = tot.s[0], den = tot.s[1], xy = tot.s[2], xx = tot.s[3], yy = tot.s[4];
        double rel, cosv;
        if (den > 0.0)
            rel = num / den;
        else
            rel = num > 0.0 ? HUGE_VAL : 0.0;
        if (xx > 0.0 && yy > 0.0)
            cosv = xy / sqrt(xx * yy);
        else
            cosv = (xx == 0.0 && yy == 0.0) ? 1.0 : 0.0;
        out[3 * seg + 0] = rel;
        out[3 * seg + 1] = cosv;
        out[3 * seg + 2] = tot.s[5];
        tickets[seg] = 0u;
    }
}

}  // namespace

int compare_blocks_per_segment(int64_t n_seg, int64_t seg_len, int dtype) {
    const int64_t esz = dtype == DIT_DTYPE_F32 ? 4 : 2;
    const int64_t nvec = (seg_len * esz + 15) / 16;
    const int64_t per = static_cast<int64_t>(kCmpThreads) * kCmpUnroll;
    int64_t nb = (nvec + per - 1) / per;
    int64_t cap = kCmpMaxBlocks / (n_seg > 0 ? n_seg : 1);
    if (cap < 1) cap = 1;
    if (nb > cap) nb = cap;
    if (nb < 1) nb = 1;
    return static_cast<int>(nb);
}

size_t compare_workspace_bytes(int64_t n_seg, int64_t seg_len, int dtype) {
    const size_t tick = ((static_cast<size_t>(n_seg) * sizeof(unsigned int) + 255) / 256) * 256;
    return tick + static_cast<size_t>(n_seg) * compare_blocks_per_segment(n_seg, seg_len, dtype) * sizeof(Acc);
}

cudaError_t launch_compare(const void* ref, const void* test, int64_t n_seg, int64_t seg_len, int dtype,
                           double* out, void* workspace, cudaStream_t stream) {
    const size_t tick = ((static_cast<size_t>(n_seg) * sizeof(unsigned int) + 255) / 256) * 256;
    unsigned int* tickets = static_cast<unsigned int*>(workspace);
    Acc* partials = reinterpret_cast<Acc*>(static_cast<char*>(workspace) + tick);
    const int64_t esz = dtype == DIT_DTYPE_F32 ? 4 : 2;
    const bool vec = (reinterpret_cast<uintptr_t>(ref) % 16 == 0) && (reinterpret_cast<uintptr_t>(test) % 16 == 0) &&
                     ((seg_len * esz) % 16 == 0);
    const dim3 grid(compare_blocks_per_segment(n_seg, seg_len, dtype), static_cast<unsigned int>(n_seg));
    if (dtype == DIT_DTYPE_BF16) {
        if (vec)
            compare_kernel<true, true><<<grid, kCmpThreads, 0, stream>>>(ref, test, seg_len, out, tickets, partials);
        else
            compare_kernel<true, false><<<grid, kCmpThreads, 0, stream>>>(ref, test, seg_len, out, tickets, partials);
    } else {
        if (vec)
            compare_kernel<false, true><<<grid, kCmpThreads, 0, stream>>>(ref, test, seg_len, out, tickets, partials);
        else
            compare_kernel<false, false><<<grid, kCmpThreads, 0, stream>>>(ref, test, seg_len, out, tickets,
                                                                            partials);
    }
    return cudaGetLastError();
}

}  // namespace ditk

extern "C" size_t dit_compare_workspace_bytes(int64_t n_segments, int64_t segment_len, int dtype) {
    if (n_segments < 1 || segment_len < 1 || n_segments > 65535) return 0;
    if (dtype != DIT_DTYPE_F32 && dtype != DIT_DTYPE_BF16) return 0;
    return ditk::compare_workspace_bytes(n_segments, segment_len, dtype);
}

extern "C" dit_status dit_compare_stats(const void* ref, const void* test, int64_t n_segments, int64_t segment_len,
                                        int dtype, double* out, void* workspace, size_t workspace_bytes,
                                        void* stream) {
    using namespace ditk;
    if (!ref || !test || !out) return DIT_ERR_INVALID_ARG;
    if (n_segments < 1 || n_segments > 65535 || segment_len < 1) return DIT_ERR_INVALID_ARG;
    if (dtype != DIT_DTYPE_F32 && dtype != DIT_DTYPE_BF16) return DIT_ERR_INVALID_ARG;
    const uintptr_t esz = dtype == DIT_DTYPE_F32 ? 4 : 2;
    if (reinterpret_cast<uintptr_t>(ref) % esz || reinterpret_cast<uintptr_t>(test) % esz) return DIT_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(out) % 8) return DIT_ERR_INVALID_ARG;
    if (segment_len > (int64_t(1) << 40) / n_segments) return DIT_ERR_INVALID_ARG;
    if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 16 ||
        workspace_bytes < compare_workspace_bytes(n_segments, segment_len, dtype))
        return DIT_ERR_WORKSPACE;
    const dit_status st = check_device();
    if (st != DIT_OK) return st;
    const cudaError_t e = launch_compare(ref, test, n_segments, segment_len, dtype, out, workspace,
                                         static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}
