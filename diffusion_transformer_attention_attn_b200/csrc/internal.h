// Host-side launchers shared between the C ABI (api.cu) and the kernel files.
// Arguments are validated by the caller; these only encode and launch.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "dit_attn.h"

namespace ditk {

// Softmax attention, bf16 in/out.  tq/tk/tv: 4-D tensor maps {d, N, H, B} with
// a {64, 128, 1, 1} box and 128-byte swizzle.  o: output base; s*: element
// strides of (b, h, n).  scale_log2 = scale * log2(e).  err: device error word.
// Nq query rows attend to Nkv keys (tq has Nq rows, tk/tv Nkv).  lse: NULL or
// fp32 [B, H, Nq] contiguous, the natural-log log-sum-exp of each row.
cudaError_t launch_attn_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, void* o,
                             int64_t sb, int64_t sh, int64_t sn, int B, int H, int Nq, int Nkv, int d,
                             float scale_log2, float* lse, int* err, cudaStream_t stream);

// Bounded-wait self-test (selftest.cu): one warp waits on an mbarrier that is
// never arrived on, gives up after the wait limit and records DIT_ERR_TIMEOUT
// in *err; *completed gets 0 (1 would mean the wait ended normally).
cudaError_t launch_wait_selftest(int* err, int32_t* completed, cudaStream_t stream);

// Merge of per-key-chunk outputs (see dit_attn_merge in dit_attn.h).
constexpr int kMaxMergeParts = 16;
cudaError_t launch_attn_merge(const void* const* o_parts, const float* const* lse_parts, int n_parts, int B, int H,
                              int N, int d, int64_t sb, int64_t sh, int64_t sn, void* o, float* lse,
                              cudaStream_t stream);

// ---- 8-bit path (d = 64 or 128) ---------------------------------------
// Tokens per statistics chunk of the pre-pass.
constexpr int kQ8StatChunk = 256;

// Byte offsets of the pre-pass products inside the caller's workspace (each
// 256-byte aligned).  Codes are [B, H, N, d] contiguous; q_scale is
// [B, H, ceil(N/128)], k_scale [B, H, ceil(N/64)], k_mean / v_scale / v_inv
// [B, H, d]; psum / pmax are the statistics partials [B, H, n_chunks, d].
struct Q8Layout {
    size_t q_codes, k_codes, v_codes, q_scale, k_scale, k_mean, v_scale, v_inv, psum, pmax, total;
    int n_chunks;
};
Q8Layout q8_layout(int B, int H, int N, int d, int pv_fp8);

// Statistics and quantisation of Q, K (and V when pv_fp8) into `ws`.
cudaError_t launch_q8_prepass(const void* q, const void* k, const void* v, int64_t sb, int64_t sh, int64_t sn, int B,
                              int H, int N, int d, int smooth_k, int pv_fp8, uint8_t* ws, cudaStream_t stream);

// The quantisation launches of the pre-pass alone (K mean and V scales
// already in `ws`).
cudaError_t launch_q8_codes(const void* q, const void* k, const void* v, int64_t sb, int64_t sh, int64_t sn, int B,
                            int H, int N, int d, int smooth_k, int pv_fp8, uint8_t* ws, cudaStream_t stream);
// Token-sharded pre-pass: the slice's per-channel K sums (fp64) and V maxima,
// then quantisation with the statistics combined over n_total tokens.
cudaError_t launch_q8_slice_stats(const void* k, const void* v, int64_t sb, int64_t sh, int64_t sn, int B, int H,
                                  int N, int d, int smooth_k, int pv_fp8, uint8_t* ws, double* k_sum, float* v_amax,
                                  cudaStream_t stream);
cudaError_t launch_q8_quantize_global(const void* q, const void* k, const void* v, int64_t sb, int64_t sh,
                                      int64_t sn, int B, int H, int N, int d, int smooth_k, int pv_fp8,
                                      const double* k_sum, const float* v_amax, int64_t n_total, uint8_t* ws,
                                      cudaStream_t stream);

// Fused quantise-and-scatter of a Ulysses group (`world` ranks, this one
// `rank`): this slice's codes and block scales go straight into the
// workspaces dst[0..world) of the head-sharded layout (B, H/world heads,
// world·N tokens), this rank's own V scales into dst[rank]; `ws` holds the
// slice's statistics.  At most kQ8MaxRanks ranks.
constexpr int kQ8MaxRanks = 16;
cudaError_t launch_q8_quantize_scatter(const void* q, const void* k, const void* v, int64_t sb, int64_t sh,
                                       int64_t sn, int B, int H, int N, int d, int smooth_k, int pv_fp8,
                                       const double* k_sum, const float* v_amax, int rank, int world,
                                       uint8_t* const* dst, uint8_t* ws, cudaStream_t stream);

// 8-bit attention over the pre-pass products.  tq8/tk8: 4-D maps over the
// INT8 codes {d, N, H, B}, box {d, 128, 1, 1} (128-byte swizzle at d = 128,
// 64-byte at d = 64); tv: e4m3 codes (same box and swizzle, pv_fp8) or the
// caller's bf16 V (box {64, 128, 1, 1}, 128-byte swizzle).
cudaError_t launch_attn_q8(const CUtensorMap& tq8, const CUtensorMap& tk8, const CUtensorMap& tv, int pv_fp8,
                           const uint8_t* ws, const Q8Layout& L, void* o, int64_t sb, int64_t sh, int64_t sn, int B,
                           int H, int N, int d, float scale_log2, int* err, cudaStream_t stream);

// DIT_OK when the current device is an sm_100 part (its one-time set-up done),
// else DIT_ERR_UNSUPPORTED or DIT_ERR_CUDA.
dit_status check_device();

// First-block-cache residual difference (see fbc_rel_l1 in dit_attn.h).
size_t fbc_workspace_bytes(int64_t n);
cudaError_t launch_fbc_rel_l1(const void* cur, const void* prev, int64_t n, int dtype, float threshold,
                              double* out_rel, int32_t* out_skip, void* workspace, cudaStream_t stream);
cudaError_t launch_fbc_sums(const void* cur, const void* prev, int64_t n, int dtype, double* out_sums,
                            void* workspace, cudaStream_t stream);
cudaError_t launch_fbc_finish(const double* sums, float threshold, double* out_rel, int32_t* out_skip,
                              cudaStream_t stream);

}  // namespace ditk
