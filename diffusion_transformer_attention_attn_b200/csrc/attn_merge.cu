// Merge of attention outputs computed over disjoint key chunks
// (declared in include/dit_attn.h as dit_attn_merge).
//
// Ring-style context parallelism splits the keys of one attention into chunks
// ("ParaAttention" (diffusers docs), section "Context Parallelism"; TMAP
// image-to-video blog, section on sequence parallelism).  Each chunk c gives
// a normalised output O_c and the log-sum-exp L_c of its logits; over all
// chunks
//   L = ln Σ_c exp(L_c),   O = Σ_c exp(L_c − L) · O_c,
// which is the attention over the union of the keys.
//
// HBM-bound: each thread owns one 16-byte slice (8 channels) of one query
// row.  It issues the loads of the row's L_c (shared by the slices of the
// row, served from L1) and of the matching slice of every O_c together, forms
// the weights with the largest L_c subtracted first, and writes the bf16
// result.  The first slice of a row also writes L.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "dit_attn.h"
#include "internal.h"

namespace ditk {
namespace {

constexpr int kMergeThreads = 256;

struct MergeParts {
    const __nv_bfloat16* o[kMaxMergeParts];
    const float* lse[kMaxMergeParts];
};

// NP: the number of parts (a template argument, so that every part's loads
// are issued before any of them is used).
template <int NP>
__global__ void __launch_bounds__(kMergeThreads)
    attn_merge_kernel(MergeParts parts, int64_t rows, int H, int N, int d, int64_t sb, int64_t sh, int64_t sn,
                      __nv_bfloat16* __restrict__ o, float* __restrict__ lse_out) {
    const int slices = d / 8;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (t >= rows * slices) return;
    const int64_t r = t / slices;  // row index over (b, h, n)
    const int sl = static_cast<int>(t - r * slices);
    const int64_t bh = r / N;
    const int n = static_cast<int>(r - bh * N);
    const int b = static_cast<int>(bh / H), h = static_cast<int>(bh % H);
    const int64_t off = b * sb + h * sh + static_cast<int64_t>(n) * sn + sl * 8;

    float L[NP];
    uint4 v[NP];
#pragma unroll
    for (int c = 0; c < NP; ++c) {
        L[c] = __ldg(parts.lse[c] + r);
        v[c] = __ldcs(reinterpret_cast<const uint4*>(parts.o[c] + off));
    }
    float lmax = L[0];
#pragma unroll
    for (int c = 1; c < NP; ++c) lmax = fmaxf(lmax, L[c]);
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    float wsum = 0.f;
    if (lmax > -INFINITY) {
#pragma unroll
        for (int c = 0; c < NP; ++c) {
            const float w = expf(L[c] - lmax);
            wsum += w;
            const uint32_t u[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                acc[2 * i] = fmaf(w, __uint_as_float(u[i] << 16), acc[2 * i]);
                acc[2 * i + 1] = fmaf(w, __uint_as_float(u[i] & 0xFFFF0000u), acc[2 * i + 1]);
            }
        }
    }
    const float inv = wsum > 0.f ? 1.0f / wsum : 0.f;
    uint32_t pk[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 p = __floats2bfloat162_rn(acc[2 * i] * inv, acc[2 * i + 1] * inv);
        pk[i] = *reinterpret_cast<const uint32_t*>(&p);
    }
    __stcs(reinterpret_cast<uint4*>(o + off), make_uint4(pk[0], pk[1], pk[2], pk[3]));
    if (lse_out != nullptr && sl == 0) lse_out[r] = wsum > 0.f ? lmax + logf(wsum) : -INFINITY;
}

template <int NP>
cudaError_t launch_np(const MergeParts& p, int64_t rows, int H, int N, int d, int64_t sb, int64_t sh, int64_t sn,
                      void* o, float* lse, cudaStream_t stream) {
    const int64_t threads = rows * (d / 8);
    const int64_t blocks = (threads + kMergeThreads - 1) / kMergeThreads;
    if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
    attn_merge_kernel<NP><<<static_cast<unsigned>(blocks), kMergeThreads, 0, stream>>>(
        p, rows, H, N, d, sb, sh, sn, static_cast<__nv_bfloat16*>(o), lse);
    return cudaGetLastError();
}

template <int NP>
cudaError_t dispatch(int n_parts, const MergeParts& p, int64_t rows, int H, int N, int d, int64_t sb, int64_t sh,
                     int64_t sn, void* o, float* lse, cudaStream_t stream) {
    if (n_parts == NP) return launch_np<NP>(p, rows, H, N, d, sb, sh, sn, o, lse, stream);
    if constexpr (NP < kMaxMergeParts)
        return dispatch<NP + 1>(n_parts, p, rows, H, N, d, sb, sh, sn, o, lse, stream);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_attn_merge(const void* const* o_parts, const float* const* lse_parts, int n_parts, int B, int H,
                              int N, int d, int64_t sb, int64_t sh, int64_t sn, void* o, float* lse,
                              cudaStream_t stream) {
    MergeParts p;
    for (int c = 0; c < kMaxMergeParts; ++c) {
        p.o[c] = c < n_parts ? static_cast<const __nv_bfloat16*>(o_parts[c]) : nullptr;
        p.lse[c] = c < n_parts ? lse_parts[c] : nullptr;
    }
    const int64_t rows = static_cast<int64_t>(B) * H * N;
    return dispatch<1>(n_parts, p, rows, H, N, d, sb, sh, sn, o, lse, stream);
}

}  // namespace ditk
