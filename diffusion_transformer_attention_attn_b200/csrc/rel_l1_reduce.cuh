// One-pass relative-L1 reduction shared by the step-caching calls.
//
// Each call computes num = Σ|cur − prev| and den = Σ|prev| over n elements in
// a single launch and hands the two sums to an epilogue run by thread 0 of the
// last block to finish:
//   * EpiThreshold (fbc_rel_l1): rel = num/den and skip = rel < threshold.
//   * the step policies of cache_step.cu, which also keep device-resident
//     counters and may set a CUDA-graph conditional.
//
// HBM-bound streaming: every thread reads 16-byte vectors of both inputs
// (grid-stride, four vectors of each in flight), sums in fp32 over at most 32
// elements and folds into fp64; blocks reduce in fp64 with warp shuffles.
// Each block writes its partial pair to the workspace; the last block to take
// a ticket adds the partials in block order, runs the epilogue and re-zeroes
// the ticket.  The grid (at most one wave of resident blocks) depends on n
// and the GPU's SM count only, so the summation order, and the result, are
// the same on every run on a given device.
//
// With kCopy the kernel also stores cur into prev in the same pass (each
// element is read before the same thread overwrites it), the update that the
// TeaCache accumulator needs on every step.  An epilogue may declare that the
// sums are not needed (evaluate() false): the kernel then reads nothing and
// only runs the epilogue.
//
// An epilogue with kProgrammatic = true (the plain decision and the sums,
// whose kernels always read their inputs) is launched as a programmatic
// dependent of the kernel before it in the stream: its blocks may become
// resident while that kernel finishes.  Each block then asks L2 for its first
// trip of both inputs (cp.async.bulk.prefetch.L2, a hint) and waits
// (griddepcontrol.wait) for the preceding grid and its memory before any load,
// so the DRAM latency of the first loads overlaps the previous kernel's tail.
// The loads themselves come after the wait and read coherent L2, so inputs
// that the previous kernel writes are seen as written.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

namespace ditk {

constexpr int kFbcThreads = 512;
constexpr int kFbcMaxBlocks = 1024;
constexpr int kFbcUnroll = 4;

struct FbcWs {
    unsigned int ticket;
    unsigned int pad[3];
    // followed by double2 partials[kFbcMaxBlocks]
};

__device__ __forceinline__ void rl1_acc(const float4& c, const float4& p, float& num, float& den) {
    num += fabsf(c.x - p.x) + fabsf(c.y - p.y) + fabsf(c.z - p.z) + fabsf(c.w - p.w);
    den += fabsf(p.x) + fabsf(p.y) + fabsf(p.z) + fabsf(p.w);
}
__device__ __forceinline__ float rl1_bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float rl1_bf_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }
__device__ __forceinline__ void rl1_acc(const uint4& c, const uint4& p, float& num, float& den) {
    const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
    const uint32_t pw[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float c0 = rl1_bf_lo(cw[i]), c1 = rl1_bf_hi(cw[i]);
        const float p0 = rl1_bf_lo(pw[i]), p1 = rl1_bf_hi(pw[i]);
        num += fabsf(c0 - p0) + fabsf(c1 - p1);
        den += fabsf(p0) + fabsf(p1);
    }
}

__device__ __forceinline__ double rl1_warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Deterministic block sum of (a, b) in fp64; result valid in thread 0.
__device__ __forceinline__ void rl1_block_sum2(double& a, double& b, double2* sh) {
    a = rl1_warp_sum(a);
    b = rl1_warp_sum(b);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) sh[warp] = make_double2(a, b);
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        double2 v = lane < nw ? sh[lane] : make_double2(0.0, 0.0);
        a = rl1_warp_sum(v.x);
        b = rl1_warp_sum(v.y);
    }
}

// rel = num / den; den = 0 gives 0 when num = 0 too, else +inf.
__device__ __forceinline__ double rl1_ratio(double num, double den) {
    if (den > 0.0) return num / den;
    return num > 0.0 ? HUGE_VAL : 0.0;
}

// VecT: float4 (fp32 inputs, 4 elements) or uint4 (bf16 inputs, 8 elements).
template <typename VecT, int kElems, bool kCopy, typename Epi>
__global__ void __launch_bounds__(kFbcThreads)
    rel_l1_kernel(const VecT* __restrict__ cur, VecT* prev, int64_t nvec, const void* __restrict__ cur_tail,
                  void* prev_tail, int tail, Epi epi, FbcWs* ws) {
    __shared__ double2 sh[kFbcThreads / 32];
    __shared__ bool is_last;
    if constexpr (Epi::kProgrammatic) {
        // Threads 0 .. 2·kFbcUnroll−1: one contiguous run of this block's
        // first trip each (trip u, input cur or prev).
        if (threadIdx.x < 2 * kFbcUnroll) {
            const int64_t u = threadIdx.x >> 1;
            const int64_t v0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + u * gridDim.x * blockDim.x;
            if (v0 < nvec) {
                const int64_t nv = min(static_cast<int64_t>(blockDim.x), nvec - v0);
                const VecT* base = (threadIdx.x & 1) ? static_cast<const VecT*>(prev) : cur;
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(base + v0),
                             "r"(static_cast<uint32_t>(nv * sizeof(VecT)))
                             : "memory");
            }
        }
        asm volatile("griddepcontrol.wait;" ::: "memory");
    }
    double2* partials = reinterpret_cast<double2*>(ws + 1);
    const bool eval = epi.evaluate();

    double num = 0.0, den = 0.0;
    if (eval || kCopy) {
        const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
        int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
        for (; i + (kFbcUnroll - 1) * stride < nvec; i += kFbcUnroll * stride) {
            VecT c[kFbcUnroll], p[kFbcUnroll];
#pragma unroll
            for (int u = 0; u < kFbcUnroll; ++u) {
                c[u] = __ldcs(cur + i + u * stride);
                p[u] = __ldcs(prev + i + u * stride);
            }
            if (kCopy) {
#pragma unroll
                for (int u = 0; u < kFbcUnroll; ++u) __stcs(prev + i + u * stride, c[u]);
            }
            float fn = 0.f, fd = 0.f;
#pragma unroll
            for (int u = 0; u < kFbcUnroll; ++u) rl1_acc(c[u], p[u], fn, fd);
            num += fn;
            den += fd;
        }
        for (; i < nvec; i += stride) {
            const VecT c = __ldcs(cur + i), p = __ldcs(prev + i);
            if (kCopy) __stcs(prev + i, c);
            float fn = 0.f, fd = 0.f;
            rl1_acc(c, p, fn, fd);
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
                    if (kCopy) static_cast<float*>(prev_tail)[t] = c;
                } else {
                    const __nv_bfloat16 cb = static_cast<const __nv_bfloat16*>(cur_tail)[t];
                    c = __bfloat162float(cb);
                    p = __bfloat162float(static_cast<const __nv_bfloat16*>(prev_tail)[t]);
                    if (kCopy) static_cast<__nv_bfloat16*>(prev_tail)[t] = cb;
                }
                num += fabsf(c - p);
                den += fabsf(p);
            }
        }
    }
    // This block has loaded all it reads: a programmatic dependent of this
    // grid may be scheduled (no effect when there is none).
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    rl1_block_sum2(num, den, sh);
    if (threadIdx.x == 0) {
        partials[blockIdx.x] = make_double2(num, den);
        // Release publishes this block's partial; the last block's acquire
        // (with the barrier below) makes every partial visible to its threads.
        unsigned int t;
        asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;" : "=r"(t) : "l"(&ws->ticket) : "memory");
        is_last = (t == gridDim.x - 1);
    }
    __syncthreads();
    if (!is_last) return;
    // Last block: fixed-order sum of the partials.
    double a = 0.0, b = 0.0;
    for (int k = threadIdx.x; k < static_cast<int>(gridDim.x); k += blockDim.x) {
        const double2 v = __ldcg(&partials[k]);
        a += v.x;
        b += v.y;
    }
    __syncthreads();
    rl1_block_sum2(a, b, sh);
    if (threadIdx.x == 0) {
        epi.finish(a, b, eval);
        ws->ticket = 0u;
    }
}

// Blocks of kFbcThreads that fit on the current GPU at once (4 per SM on
// sm_100: 2048 threads), queried once per device.
inline int rel_l1_resident_blocks() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return kFbcMaxBlocks;
    if (cached[dev] == 0) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
            return kFbcMaxBlocks;
        cached[dev] = sms * (2048 / kFbcThreads);
    }
    return cached[dev];
}

// One wave of resident blocks at most (more only adds a partial second wave),
// never more than the workspace holds.  The grid depends on n and the GPU's
// SM count only, so a given device always sums in the same order.
inline int rel_l1_blocks(int64_t nvec) {
    const int64_t per = static_cast<int64_t>(kFbcThreads) * kFbcUnroll;
    int64_t nb = (nvec + per - 1) / per;
    int64_t cap = rel_l1_resident_blocks();
    if (cap > kFbcMaxBlocks) cap = kFbcMaxBlocks;
    if (nb < 1) nb = 1;
    if (nb > cap) nb = cap;
    return static_cast<int>(nb);
}

// Launch over n elements of dtype 0 (fp32) or 1 (bf16).  prev must be
// writable when kCopy.  Epi::kProgrammatic selects the programmatic
// (overlapped) launch described at the top of this file.
template <bool kCopy, typename Epi>
cudaError_t launch_rel_l1(const void* cur, const void* prev, int64_t n, int dtype, const Epi& epi, void* workspace,
                          cudaStream_t stream) {
    FbcWs* ws = static_cast<FbcWs*>(workspace);
    void* pv = const_cast<void*>(prev);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kFbcThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = Epi::kProgrammatic ? 1 : 0;
    if (dtype == 0) {
        const int64_t nvec = n / 4;
        const int tail = static_cast<int>(n - nvec * 4);
        const float* c = static_cast<const float*>(cur);
        float* p = static_cast<float*>(pv);
        cfg.gridDim = dim3(rel_l1_blocks(nvec));
        return cudaLaunchKernelEx(&cfg, rel_l1_kernel<float4, 4, kCopy, Epi>, reinterpret_cast<const float4*>(c),
                                  reinterpret_cast<float4*>(p), nvec, static_cast<const void*>(c + nvec * 4),
                                  static_cast<void*>(p + nvec * 4), tail, epi, ws);
    }
    const int64_t nvec = n / 8;
    const int tail = static_cast<int>(n - nvec * 8);
    const __nv_bfloat16* c = static_cast<const __nv_bfloat16*>(cur);
    __nv_bfloat16* p = static_cast<__nv_bfloat16*>(pv);
    cfg.gridDim = dim3(rel_l1_blocks(nvec));
    return cudaLaunchKernelEx(&cfg, rel_l1_kernel<uint4, 8, kCopy, Epi>, reinterpret_cast<const uint4*>(c),
                              reinterpret_cast<uint4*>(p), nvec, static_cast<const void*>(c + nvec * 8),
                              static_cast<void*>(p + nvec * 8), tail, epi, ws);
}

}  // namespace ditk
