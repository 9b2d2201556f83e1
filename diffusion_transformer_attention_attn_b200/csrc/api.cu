// C ABI of libditattn.so (declared in include/dit_attn.h): argument
// validation, TMA tensor-map encoding and launches.  Host code only; the
// arithmetic of every call runs in the kernels of attn_bf16.cu, attn_q8.cu,
// q8_prepass.cu, attn_merge.cu and fbc_rel_l1.cu (the step caches and the output comparison
// have their own entry points in cache_step.cu and compare.cu; the bounded-wait self-test
// kernel is in selftest.cu).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "dit_attn.h"
#include "internal.h"

namespace ditk {

// Device-side error word (one per device that loads the library); kernels
// receive its address and write DIT_ERR_TIMEOUT there when a wait runs out.
__device__ int g_dit_error = 0;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
    std::once_flag once;
    cudaError_t init_err = cudaSuccess;
    int* err_word = nullptr;
    bool sm100 = false;
};
DeviceState g_dev[kMaxDevices];

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
std::once_flag g_encode_once;
EncodeTiledFn g_encode = nullptr;

EncodeTiledFn encode_fn() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    });
    return g_encode;
}

// Per-device set-up, done once with that device current: the address of the
// error word and whether the device is an sm_100 part.
DeviceState* device_state(dit_status* st) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        *st = DIT_ERR_CUDA;
        return nullptr;
    }
    DeviceState& s = g_dev[dev];
    std::call_once(s.once, [&s, dev] {
        cudaDeviceProp prop;
        s.init_err = cudaGetDeviceProperties(&prop, dev);
        if (s.init_err != cudaSuccess) return;
        s.sm100 = (prop.major == 10 && prop.minor == 0);
        s.init_err = cudaGetSymbolAddress(reinterpret_cast<void**>(&s.err_word), g_dit_error);
    });
    if (s.init_err != cudaSuccess) {
        *st = DIT_ERR_CUDA;
        return nullptr;
    }
    if (!s.sm100) {
        *st = DIT_ERR_UNSUPPORTED;
        return nullptr;
    }
    *st = DIT_OK;
    return &s;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Byte ranges [p, p + span) of two tensors overlap?
bool overlaps(const void* a, const void* b, int64_t span) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    const uintptr_t s = static_cast<uintptr_t>(span);
    return x < y + s && y < x + s;
}

// Validation shared by the attention calls.  On success fills the strides.
// `o` may be null only when the call writes no output (need_o false).
dit_status check_attn_args(const void* q, const void* k, const void* v, const void* o, int B, int H, int N, int d,
                           const int64_t* strides, int64_t* sb, int64_t* sh, int64_t* sn, bool need_o = true) {
    if (!q || !k || !v || (need_o && !o)) return DIT_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || N < 1 || d < 1) return DIT_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || (o && !aligned16(o))) return DIT_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return DIT_ERR_UNSUPPORTED;
    if (N > (1 << 30) || static_cast<int64_t>(B) * H > (1 << 24)) return DIT_ERR_UNSUPPORTED;
    if (strides) {
        *sb = strides[0];
        *sh = strides[1];
        *sn = strides[2];
    } else {
        *sn = d;
        *sh = static_cast<int64_t>(N) * d;
        *sb = static_cast<int64_t>(H) * N * d;
    }
    // TMA: every stride in bytes a multiple of 16, below 2^40; rows must not alias.
    const int64_t st[3] = {*sb, *sh, *sn};
    for (int i = 0; i < 3; ++i) {
        if (st[i] <= 0 || (st[i] * 2) % 16 != 0 || st[i] * 2 >= (int64_t(1) << 40)) return DIT_ERR_INVALID_ARG;
    }
    if (*sn < d) return DIT_ERR_INVALID_ARG;
    // Extent of one tensor in bytes (for the overlap check on o).
    const int64_t span = ((B - 1) * *sb + (H - 1) * *sh + (N - 1) * *sn + d) * 2;
    if (o && (overlaps(o, q, span) || overlaps(o, k, span) || overlaps(o, v, span))) return DIT_ERR_INVALID_ARG;
    return DIT_OK;
}

// 4-D map {d, N, H, B} over a bf16 tensor, box {64, 128, 1, 1}, 128-B swizzle.
dit_status encode_bf16_map(CUtensorMap* map, const void* base, int B, int H, int N, int d, int64_t sb, int64_t sh,
                           int64_t sn) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return DIT_ERR_CUDA;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(H),
                                static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(sn * 2), static_cast<cuuint64_t>(sh * 2),
                                   static_cast<cuuint64_t>(sb * 2)};
    const cuuint32_t box[4] = {64, 128, 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? DIT_OK : DIT_ERR_INVALID_ARG;
}

float default_scale(int d) { return 1.0f / std::sqrt(static_cast<float>(d)); }

// (b, h, n) element strides of one bf16 [B, H, N, d] operand: given, or those
// of the contiguous layout.  TMA needs every stride in bytes to be a multiple
// of 16 below 2^40; rows must not alias (sn >= d).  span: bytes covered.
dit_status resolve_strides(const int64_t* strides, int B, int H, int N, int d, int64_t* sb, int64_t* sh, int64_t* sn,
                           int64_t* span) {
    if (strides) {
        *sb = strides[0];
        *sh = strides[1];
        *sn = strides[2];
    } else {
        *sn = d;
        *sh = static_cast<int64_t>(N) * d;
        *sb = static_cast<int64_t>(H) * N * d;
    }
    const int64_t st[3] = {*sb, *sh, *sn};
    for (int i = 0; i < 3; ++i)
        if (st[i] <= 0 || (st[i] * 2) % 16 != 0 || st[i] * 2 >= (int64_t(1) << 40)) return DIT_ERR_INVALID_ARG;
    if (*sn < d) return DIT_ERR_INVALID_ARG;
    *span = ((B - 1) * *sb + (H - 1) * *sh + (N - 1) * *sn + d) * 2;
    return DIT_OK;
}

// 4-D map {d B, N, H, B} over contiguous 8-bit codes [B, H, N, d] inside
// the workspace, box {d, 128, 1, 1}: 128-byte swizzle at d = 128, 64-byte
// swizzle at d = 64 (the swizzle spans one d-byte row).
dit_status encode_u8_map(CUtensorMap* map, const void* base, int B, int H, int N, int d) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return DIT_ERR_CUDA;
    const cuuint64_t D = static_cast<cuuint64_t>(d);
    const cuuint64_t dims[4] = {D, static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(B)};
    const cuuint64_t strides[3] = {D, static_cast<cuuint64_t>(N) * D, static_cast<cuuint64_t>(H) * N * D};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(d), 128, 1, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUtensorMapSwizzle sw = d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? DIT_OK : DIT_ERR_INVALID_ARG;
}

// Validation shared by the 8-bit calls (after check_attn_args).
dit_status check_q8_args(int d, int smooth_k, int pv_mode, const void* ws, size_t ws_bytes, int B, int H, int N) {
    if (d != 64 && d != 128) return DIT_ERR_UNSUPPORTED;
    if (smooth_k != 0 && smooth_k != 1) return DIT_ERR_INVALID_ARG;
    if (pv_mode != DIT_PV_FP8_E4M3 && pv_mode != DIT_PV_BF16) return DIT_ERR_INVALID_ARG;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return DIT_ERR_WORKSPACE;
    if (ws_bytes < q8_layout(B, H, N, d, pv_mode == DIT_PV_FP8_E4M3).total) return DIT_ERR_WORKSPACE;
    return DIT_OK;
}

}  // namespace

dit_status check_device() {
    dit_status st;
    device_state(&st);
    return st;
}

}  // namespace ditk

using namespace ditk;

extern "C" {

dit_status dit_attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq,
                           int Nkv, int d, const int64_t* q_strides, const int64_t* kv_strides, float scale,
                           void* stream) {
    if (!q || !k || !v || !o) return DIT_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || Nq < 1 || Nkv < 1 || d < 1) return DIT_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return DIT_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return DIT_ERR_UNSUPPORTED;
    if (Nq > (1 << 30) || Nkv > (1 << 30) || static_cast<int64_t>(B) * H > (1 << 24)) return DIT_ERR_UNSUPPORTED;
    int64_t qb, qh, qn, kb, kh, kn, qspan, kspan;
    dit_status st = resolve_strides(q_strides, B, H, Nq, d, &qb, &qh, &qn, &qspan);
    if (st != DIT_OK) return st;
    if ((st = resolve_strides(kv_strides, B, H, Nkv, d, &kb, &kh, &kn, &kspan)) != DIT_OK) return st;
    const uintptr_t uo = reinterpret_cast<uintptr_t>(o);
    auto hit = [](uintptr_t a, int64_t sa, const void* p, int64_t sp) {
        const uintptr_t b = reinterpret_cast<uintptr_t>(p);
        return a < b + static_cast<uintptr_t>(sp) && b < a + static_cast<uintptr_t>(sa);
    };
    if (hit(uo, qspan, q, qspan) || hit(uo, qspan, k, kspan) || hit(uo, qspan, v, kspan)) return DIT_ERR_INVALID_ARG;
    if (lse) {
        if ((reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return DIT_ERR_INVALID_ARG;
        const int64_t lspan = static_cast<int64_t>(B) * H * Nq * 4;
        const uintptr_t ul = reinterpret_cast<uintptr_t>(lse);
        if (hit(ul, lspan, o, qspan) || hit(ul, lspan, q, qspan) || hit(ul, lspan, k, kspan) ||
            hit(ul, lspan, v, kspan))
            return DIT_ERR_INVALID_ARG;
    }
    if (!(scale == scale) || std::isinf(scale)) return DIT_ERR_INVALID_ARG;
    DeviceState* ds = device_state(&st);
    if (!ds) return st;
    CUtensorMap tq, tk, tv;
    if ((st = encode_bf16_map(&tq, q, B, H, Nq, d, qb, qh, qn)) != DIT_OK) return st;
    if ((st = encode_bf16_map(&tk, k, B, H, Nkv, d, kb, kh, kn)) != DIT_OK) return st;
    if ((st = encode_bf16_map(&tv, v, B, H, Nkv, d, kb, kh, kn)) != DIT_OK) return st;
    const float s = scale > 0.f ? scale : default_scale(d);
    const float scale_log2 = static_cast<float>(static_cast<double>(s) * 1.4426950408889634);
    cudaError_t e = launch_attn_bf16(tq, tk, tv, o, qb, qh, qn, B, H, Nq, Nkv, d, scale_log2, lse, ds->err_word,
                                     static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

dit_status dit_attn_merge(const void* const* o_parts, const float* const* lse_parts, int n_parts, int B, int H, int N,
                          int d, const int64_t* strides, void* o, float* lse, void* stream) {
    if (!o_parts || !lse_parts || !o || n_parts < 1 || n_parts > kMaxMergeParts) return DIT_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || N < 1 || d < 8 || d > 256 || d % 8 != 0) return DIT_ERR_INVALID_ARG;
    if (static_cast<int64_t>(B) * H * N > (int64_t(1) << 36)) return DIT_ERR_UNSUPPORTED;
    int64_t sb, sh, sn, span;
    dit_status st = resolve_strides(strides, B, H, N, d, &sb, &sh, &sn, &span);
    if (st != DIT_OK) return st;
    if (!aligned16(o)) return DIT_ERR_INVALID_ARG;
    const int64_t lspan = static_cast<int64_t>(B) * H * N * 4;
    auto hit = [](const void* a, int64_t sa, const void* p, int64_t sp) {
        const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(p);
        return x < y + static_cast<uintptr_t>(sp) && y < x + static_cast<uintptr_t>(sa);
    };
    for (int c = 0; c < n_parts; ++c) {
        if (!o_parts[c] || !lse_parts[c] || !aligned16(o_parts[c])) return DIT_ERR_INVALID_ARG;
        if ((reinterpret_cast<uintptr_t>(lse_parts[c]) & 3u) != 0) return DIT_ERR_INVALID_ARG;
        // the output may not overwrite an input still to be read
        if (hit(o, span, o_parts[c], span) || hit(o, span, lse_parts[c], lspan)) return DIT_ERR_INVALID_ARG;
        if (lse && (hit(lse, lspan, o_parts[c], span) || hit(lse, lspan, lse_parts[c], lspan)))
            return DIT_ERR_INVALID_ARG;
    }
    if (lse && ((reinterpret_cast<uintptr_t>(lse) & 3u) != 0 || hit(lse, lspan, o, span))) return DIT_ERR_INVALID_ARG;
    if (!device_state(&st)) return st;
    cudaError_t e = launch_attn_merge(o_parts, lse_parts, n_parts, B, H, N, d, sb, sh, sn, o, lse,
                                      static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

dit_status dit_attn_fwd(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d,
                        const int64_t* strides, float scale, void* stream) {
    int64_t sb, sh, sn;
    dit_status st = check_attn_args(q, k, v, o, B, H, N, d, strides, &sb, &sh, &sn);
    if (st != DIT_OK) return st;
    if (!(scale == scale) || std::isinf(scale)) return DIT_ERR_INVALID_ARG;
    DeviceState* ds = device_state(&st);
    if (!ds) return st;
    CUtensorMap tq, tk, tv;
    if ((st = encode_bf16_map(&tq, q, B, H, N, d, sb, sh, sn)) != DIT_OK) return st;
    if ((st = encode_bf16_map(&tk, k, B, H, N, d, sb, sh, sn)) != DIT_OK) return st;
    if ((st = encode_bf16_map(&tv, v, B, H, N, d, sb, sh, sn)) != DIT_OK) return st;
    const float s = scale > 0.f ? scale : default_scale(d);
    const float scale_log2 = static_cast<float>(static_cast<double>(s) * 1.4426950408889634);
    cudaError_t e = launch_attn_bf16(tq, tk, tv, o, sb, sh, sn, B, H, N, N, d, scale_log2, nullptr, ds->err_word,
                                     static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

size_t dit_attn_q8_workspace_bytes(int B, int H, int N, int d, int pv_mode) {
    if (B < 1 || H < 1 || N < 1 || (d != 64 && d != 128)) return 0;
    if (pv_mode != DIT_PV_FP8_E4M3 && pv_mode != DIT_PV_BF16) return 0;
    return q8_layout(B, H, N, d, pv_mode == DIT_PV_FP8_E4M3).total;
}

dit_status dit_attn_q8_workspace_layout(int B, int H, int N, int d, int pv_mode, size_t* offsets) {
    if (!offsets || B < 1 || H < 1 || N < 1) return DIT_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return DIT_ERR_UNSUPPORTED;
    if (pv_mode != DIT_PV_FP8_E4M3 && pv_mode != DIT_PV_BF16) return DIT_ERR_INVALID_ARG;
    const Q8Layout L = q8_layout(B, H, N, d, pv_mode == DIT_PV_FP8_E4M3);
    const size_t o[8] = {L.q_codes, L.k_codes, L.v_codes, L.q_scale, L.k_scale, L.k_mean, L.v_scale, L.v_inv};
    for (int i = 0; i < 8; ++i) offsets[i] = o[i];
    return DIT_OK;
}

dit_status dit_attn_q8_quantize(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                                const int64_t* strides, int smooth_k, int pv_mode, void* workspace,
                                size_t workspace_bytes, void* stream) {
    int64_t sb, sh, sn;
    dit_status st = check_attn_args(q, k, v, nullptr, B, H, N, d, strides, &sb, &sh, &sn, false);
    if (st != DIT_OK) return st;
    if ((st = check_q8_args(d, smooth_k, pv_mode, workspace, workspace_bytes, B, H, N)) != DIT_OK) return st;
    DeviceState* ds = device_state(&st);
    if (!ds) return st;
    cudaError_t e = launch_q8_prepass(q, k, v, sb, sh, sn, B, H, N, d, smooth_k, pv_mode == DIT_PV_FP8_E4M3,
                                      static_cast<uint8_t*>(workspace), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

// ---- token-sharded 8-bit pre-pass and attention from codes ----------------

namespace {
bool overlap_bytes(const void* a, int64_t na, const void* b, int64_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + static_cast<uintptr_t>(nb) && y < x + static_cast<uintptr_t>(na);
}
}  // namespace

dit_status dit_attn_q8_channel_stats(const void* k, const void* v, int B, int H, int N, int d, const int64_t* strides,
                                     int smooth_k, int pv_mode, double* k_sum, float* v_amax, void* workspace,
                                     size_t workspace_bytes, void* stream) {
    int64_t sb, sh, sn;
    dit_status st = check_attn_args(k, k, v, nullptr, B, H, N, d, strides, &sb, &sh, &sn, false);
    if (st != DIT_OK) return st;
    if ((st = check_q8_args(d, smooth_k, pv_mode, workspace, workspace_bytes, B, H, N)) != DIT_OK) return st;
    if (!k_sum || !v_amax || (reinterpret_cast<uintptr_t>(k_sum) & 7u) || (reinterpret_cast<uintptr_t>(v_amax) & 3u))
        return DIT_ERR_INVALID_ARG;
    const int64_t nstat = static_cast<int64_t>(B) * H * d;
    const int64_t wsz = static_cast<int64_t>(q8_layout(B, H, N, d, pv_mode == DIT_PV_FP8_E4M3).total);
    if (overlap_bytes(k_sum, nstat * 8, workspace, wsz) || overlap_bytes(v_amax, nstat * 4, workspace, wsz) ||
        overlap_bytes(k_sum, nstat * 8, v_amax, nstat * 4))
        return DIT_ERR_INVALID_ARG;
    DeviceState* ds = device_state(&st);
    if (!ds) return st;
    cudaError_t e = launch_q8_slice_stats(k, v, sb, sh, sn, B, H, N, d, smooth_k, pv_mode == DIT_PV_FP8_E4M3,
                                          static_cast<uint8_t*>(workspace), k_sum, v_amax,
                                          static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

dit_status dit_attn_q8_quantize_global(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                                       const int64_t* strides, int smooth_k, int pv_mode, const double* k_sum,
                                       const float* v_amax, int64_t n_total, void* workspace, size_t workspace_bytes,
                                       void* stream) {
    int64_t sb, sh, sn;
    dit_status st = check_attn_args(q, k, v, nullptr, B, H, N, d, strides, &sb, &sh, &sn, false);
    if (st != DIT_OK) return st;
    if ((st = check_q8_args(d, smooth_k, pv_mode, workspace, workspace_bytes, B, H, N)) != DIT_OK) return st;
    if (!k_sum || !v_amax || (reinterpret_cast<uintptr_t>(k_sum) & 7u) || (reinterpret_cast<uintptr_t>(v_amax) & 3u))
        return DIT_ERR_INVALID_ARG;
    if (n_total < N) return DIT_ERR_INVALID_ARG;
    DeviceState* ds = device_state(&st);
    if (!ds) return st;
    cudaError_t e = launch_q8_quantize_global(q, k, v, sb, sh, sn, B, H, N, d, smooth_k, pv_mode == DIT_PV_FP8_E4M3,
                                              k_sum, v_amax, n_total, static_cast<uint8_t*>(workspace),
                                              static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

dit_status dit_attn_q8_quantize_scatter(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                                        const int64_t* strides, int smooth_k, int pv_mode, const double* k_sum,
                                        const float* v_amax, int rank, int world, void* const* dst_workspaces,
                                        size_t dst_workspace_bytes, void* workspace, size_t workspace_bytes,
                                        void* stream) {
    int64_t sb, sh, sn;
    dit_status st = check_attn_args(q, k, v, nullptr, B, H, N, d, strides, &sb, &sh, &sn, false);
    if (st != DIT_OK) return st;
    if ((st = check_q8_args(d, smooth_k, pv_mode, workspace, workspace_bytes, B, H, N)) != DIT_OK) return st;
    if (world < 1 || world > kQ8MaxRanks || rank < 0 || rank >= world) return DIT_ERR_INVALID_ARG;
    if (H % world != 0 || (world > 1 && N % 128 != 0)) return DIT_ERR_INVALID_ARG;
    if (static_cast<int64_t>(N) * world > (int64_t(1) << 30)) return DIT_ERR_UNSUPPORTED;
    if (!k_sum || !v_amax || (reinterpret_cast<uintptr_t>(k_sum) & 7u) || (reinterpret_cast<uintptr_t>(v_amax) & 3u))
        return DIT_ERR_INVALID_ARG;
    if (!dst_workspaces) return DIT_ERR_INVALID_ARG;
    const int pv_fp8 = pv_mode == DIT_PV_FP8_E4M3;
    const size_t need = q8_layout(B, H / world, N * world, d, pv_fp8).total;
    if (dst_workspace_bytes < need) return DIT_ERR_WORKSPACE;
    const int64_t local = static_cast<int64_t>(q8_layout(B, H, N, d, pv_fp8).total);
    const int64_t span = ((B - 1) * sb + (H - 1) * sh + (N - 1) * sn + d) * 2;
    uint8_t* dst[kQ8MaxRanks];
    for (int r = 0; r < world; ++r) {
        dst[r] = static_cast<uint8_t*>(dst_workspaces[r]);
        if (!dst[r] || (reinterpret_cast<uintptr_t>(dst[r]) & 255u) != 0) return DIT_ERR_WORKSPACE;
        // every destination is distinct from the others, the slice workspace and the inputs
        if (overlap_bytes(dst[r], static_cast<int64_t>(need), workspace, local)) return DIT_ERR_WORKSPACE;
        for (const void* t : {q, k, v})
            if (overlap_bytes(dst[r], static_cast<int64_t>(need), t, span)) return DIT_ERR_WORKSPACE;
        for (int u = 0; u < r; ++u)
            if (overlap_bytes(dst[r], static_cast<int64_t>(need), dst[u], static_cast<int64_t>(need)))
                return DIT_ERR_WORKSPACE;
    }
    DeviceState* ds = device_state(&st);
    if (!ds) return st;
    cudaError_t e = launch_q8_quantize_scatter(q, k, v, sb, sh, sn, B, H, N, d, smooth_k, pv_fp8, k_sum, v_amax, rank,
                                               world, dst, static_cast<uint8_t*>(workspace),
                                               static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

dit_status dit_attn_fwd_q8_prequantized(const void* workspace, size_t workspace_bytes, const void* v, void* o, int B,
                                        int H, int N, int d, const int64_t* strides, float scale, int pv_mode,
                                        void* stream) {
    if (pv_mode != DIT_PV_FP8_E4M3 && pv_mode != DIT_PV_BF16) return DIT_ERR_INVALID_ARG;
    const int pv_fp8 = pv_mode == DIT_PV_FP8_E4M3;
    const void* vv = pv_fp8 ? o : v;  // stands in for V during validation in FP8 mode
    int64_t sb, sh, sn;
    dit_status st = check_attn_args(o, o, vv, nullptr, B, H, N, d, strides, &sb, &sh, &sn, false);
    if (st != DIT_OK) return st;
    if (!(scale == scale) || std::isinf(scale)) return DIT_ERR_INVALID_ARG;
    if ((st = check_q8_args(d, 0, pv_mode, workspace, workspace_bytes, B, H, N)) != DIT_OK) return st;
    const Q8Layout L = q8_layout(B, H, N, d, pv_fp8);
    const int64_t span = ((B - 1) * sb + (H - 1) * sh + (N - 1) * sn + d) * 2;
    if (overlap_bytes(o, span, workspace, static_cast<int64_t>(L.total))) return DIT_ERR_WORKSPACE;
    if (!pv_fp8 && overlap_bytes(o, span, v, span)) return DIT_ERR_INVALID_ARG;
    DeviceState* ds = device_state(&st);
    if (!ds) return st;
    const uint8_t* ws = static_cast<const uint8_t*>(workspace);
    CUtensorMap tq8, tk8, tv;
    if ((st = encode_u8_map(&tq8, ws + L.q_codes, B, H, N, d)) != DIT_OK) return st;
    if ((st = encode_u8_map(&tk8, ws + L.k_codes, B, H, N, d)) != DIT_OK) return st;
    if (pv_fp8)
        st = encode_u8_map(&tv, ws + L.v_codes, B, H, N, d);
    else
        st = encode_bf16_map(&tv, v, B, H, N, d, sb, sh, sn);
    if (st != DIT_OK) return st;
    const float sc = scale > 0.f ? scale : default_scale(d);
    const float scale_log2 = static_cast<float>(static_cast<double>(sc) * 1.4426950408889634);
    cudaError_t e = launch_attn_q8(tq8, tk8, tv, pv_fp8, ws, L, o, sb, sh, sn, B, H, N, d, scale_log2, ds->err_word,
                                   static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

dit_status dit_attn_fwd_q8(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d,
                           const int64_t* strides, float scale, int smooth_k, int pv_mode, void* workspace,
                           size_t workspace_bytes, void* stream) {
    int64_t sb, sh, sn;
    dit_status st = check_attn_args(q, k, v, o, B, H, N, d, strides, &sb, &sh, &sn);
    if (st != DIT_OK) return st;
    if (!(scale == scale) || std::isinf(scale)) return DIT_ERR_INVALID_ARG;
    if ((st = check_q8_args(d, smooth_k, pv_mode, workspace, workspace_bytes, B, H, N)) != DIT_OK) return st;
    const int pv_fp8 = pv_mode == DIT_PV_FP8_E4M3;
    const Q8Layout L = q8_layout(B, H, N, d, pv_fp8);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    // The workspace must not overlap the inputs or the output.
    const int64_t span = ((B - 1) * sb + (H - 1) * sh + (N - 1) * sn + d) * 2;
    const int64_t wsz = static_cast<int64_t>(L.total);
    for (const void* t : {q, k, v, static_cast<const void*>(o)}) {
        const uintptr_t x = reinterpret_cast<uintptr_t>(t), y = reinterpret_cast<uintptr_t>(ws);
        if (x < y + wsz && y < x + span) return DIT_ERR_WORKSPACE;
    }
    DeviceState* ds = device_state(&st);
    if (!ds) return st;
    CUtensorMap tq8, tk8, tv;
    if ((st = encode_u8_map(&tq8, ws + L.q_codes, B, H, N, d)) != DIT_OK) return st;
    if ((st = encode_u8_map(&tk8, ws + L.k_codes, B, H, N, d)) != DIT_OK) return st;
    if (pv_fp8)
        st = encode_u8_map(&tv, ws + L.v_codes, B, H, N, d);
    else
        st = encode_bf16_map(&tv, v, B, H, N, d, sb, sh, sn);
    if (st != DIT_OK) return st;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_q8_prepass(q, k, v, sb, sh, sn, B, H, N, d, smooth_k, pv_fp8, ws, s);
    if (e != cudaSuccess) return DIT_ERR_CUDA;
    const float sc = scale > 0.f ? scale : default_scale(d);
    const float scale_log2 = static_cast<float>(static_cast<double>(sc) * 1.4426950408889634);
    e = launch_attn_q8(tq8, tk8, tv, pv_fp8, ws, L, o, sb, sh, sn, B, H, N, d, scale_log2, ds->err_word, s);
    return e == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

size_t fbc_rel_l1_workspace_bytes(int64_t n) { return n < 1 ? 0 : fbc_workspace_bytes(n); }

dit_status fbc_rel_l1(const void* r_cur, const void* r_prev, int64_t n, int dtype, float threshold, double* out_rel,
                      int32_t* out_skip, void* workspace, size_t workspace_bytes, void* stream) {
    if (!r_cur || !r_prev || !out_rel || !out_skip || n < 1) return DIT_ERR_INVALID_ARG;
    if (dtype != DIT_DTYPE_F32 && dtype != DIT_DTYPE_BF16) return DIT_ERR_INVALID_ARG;
    if (!aligned16(r_cur) || !aligned16(r_prev)) return DIT_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(out_rel) & 7u) != 0 || (reinterpret_cast<uintptr_t>(out_skip) & 3u) != 0)
        return DIT_ERR_INVALID_ARG;
    if (!(threshold == threshold)) return DIT_ERR_INVALID_ARG;
    if (!workspace || !aligned16(workspace) || workspace_bytes < fbc_workspace_bytes(n)) return DIT_ERR_WORKSPACE;
    dit_status st;
    if (!device_state(&st)) return st;
    cudaError_t e = launch_fbc_rel_l1(r_cur, r_prev, n, dtype, threshold, out_rel, out_skip, workspace,
                                      static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

dit_status fbc_rel_l1_sums(const void* r_cur, const void* r_prev, int64_t n, int dtype, double* out_sums,
                           void* workspace, size_t workspace_bytes, void* stream) {
    if (!r_cur || !r_prev || !out_sums || n < 1) return DIT_ERR_INVALID_ARG;
    if (dtype != DIT_DTYPE_F32 && dtype != DIT_DTYPE_BF16) return DIT_ERR_INVALID_ARG;
    if (!aligned16(r_cur) || !aligned16(r_prev) || (reinterpret_cast<uintptr_t>(out_sums) & 7u) != 0)
        return DIT_ERR_INVALID_ARG;
    if (!workspace || !aligned16(workspace) || workspace_bytes < fbc_workspace_bytes(n)) return DIT_ERR_WORKSPACE;
    dit_status st;
    if (!device_state(&st)) return st;
    cudaError_t e = launch_fbc_sums(r_cur, r_prev, n, dtype, out_sums, workspace, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

dit_status fbc_rel_l1_finish(const double* sums, float threshold, double* out_rel, int32_t* out_skip,
                             void* stream) {
    if (!sums || !out_rel || !out_skip) return DIT_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(sums) & 7u) != 0 || (reinterpret_cast<uintptr_t>(out_rel) & 7u) != 0 ||
        (reinterpret_cast<uintptr_t>(out_skip) & 3u) != 0)
        return DIT_ERR_INVALID_ARG;
    if (!(threshold == threshold)) return DIT_ERR_INVALID_ARG;
    dit_status st;
    if (!device_state(&st)) return st;
    cudaError_t e = launch_fbc_finish(sums, threshold, out_rel, out_skip, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

dit_status dit_wait_selftest(int32_t* out_completed, void* stream) {
    if (out_completed == nullptr) return DIT_ERR_INVALID_ARG;
    dit_status st;
    DeviceState* ds = device_state(&st);
    if (!ds) return st;
    const cudaError_t e = launch_wait_selftest(ds->err_word, out_completed, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

dit_status dit_get_device_status(void* stream) {
    dit_status st;
    DeviceState* ds = device_state(&st);
    if (!ds) return st;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DIT_ERR_CUDA;
    int word = 0;
    if (cudaMemcpyFromSymbol(&word, g_dit_error, sizeof(int)) != cudaSuccess) return DIT_ERR_CUDA;
    if (word != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_dit_error, &zero, sizeof(int)) != cudaSuccess) return DIT_ERR_CUDA;
        return static_cast<dit_status>(word);
    }
    return DIT_OK;
}

const char* dit_status_string(int status) {
    switch (status) {
        case DIT_OK: return "DIT_OK";
        case DIT_ERR_INVALID_ARG: return "DIT_ERR_INVALID_ARG";
        case DIT_ERR_UNSUPPORTED: return "DIT_ERR_UNSUPPORTED";
        case DIT_ERR_WORKSPACE: return "DIT_ERR_WORKSPACE";
        case DIT_ERR_CUDA: return "DIT_ERR_CUDA";
        case DIT_ERR_TIMEOUT: return "DIT_ERR_TIMEOUT";
        default: return "DIT_ERR_UNKNOWN";
    }
}

}  // extern "C"
