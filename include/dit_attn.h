/*
 * dit_attn.h — C ABI of the B200 (sm_100a) diffusion-transformer attention
 * library (libditattn.so).
 *
 * The library holds the hot path of image and video diffusion transformers:
 * full bidirectional multi-head self-attention over one joint token stream
 * (bf16, and 8-bit with INT8 QKᵀ and FP8 or bf16 PV), and the first-block-cache
 * residual difference that decides whether a denoising step may reuse its
 * cached residual.  Around them: attention over a chunk of the keys with its
 * log-sum-exp and the merge of chunks, the 8-bit pre-pass split for a
 * token-sharded sequence (with a fused quantise-and-scatter for the Ulysses
 * all-to-all), the error of one output against another, and (in dit_cache.h)
 * step-cache policies whose decisions stay on the device.
 *
 * Conventions shared by every entry point
 *   - Every buffer is caller-owned device memory.  The library allocates no
 *     device memory on any call; where a kernel needs scratch, the caller
 *     passes a workspace whose size the matching *_workspace_bytes call gives.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL
 *     is the legacy default stream).  Argument errors are reported before any
 *     launch and leave every output untouched.
 *   - A launch failure returns DIT_ERR_CUDA.  Every wait inside a kernel is
 *     bounded in time: a wait that runs out records DIT_ERR_TIMEOUT in a
 *     device-side error word instead of hanging, and dit_get_device_status
 *     reports (and clears) it.
 *   - NaN or Inf inputs are outside the contract.
 */
#ifndef DIT_ATTN_H
#define DIT_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DIT_OK = 0,
    DIT_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size or stride */
    DIT_ERR_UNSUPPORTED = 2, /* valid request this build does not serve (e.g. d = 96) */
    DIT_ERR_WORKSPACE = 3,   /* workspace missing, misaligned or too small */
    DIT_ERR_CUDA = 4,        /* a CUDA runtime/driver call or launch failed */
    DIT_ERR_TIMEOUT = 5      /* a device-side wait ran out (see dit_get_device_status) */
} dit_status;

typedef enum { DIT_DTYPE_F32 = 0, DIT_DTYPE_BF16 = 1 } dit_dtype;

/* Precision of the P·V contraction of the 8-bit path. */
typedef enum { DIT_PV_FP8_E4M3 = 0, DIT_PV_BF16 = 1 } dit_pv_mode;

/*
 * dit_attn_fwd — softmax attention O = softmax(scale · Q Kᵀ) V, per (b, h),
 * over all N keys (no mask: the text and visual tokens form one joint,
 * bidirectional stream).
 *
 * Defined by: "Flash Attention 2 accelerates Z-Image S3-DiT 6B" (hotdry.top),
 * opening section (text, visual and VAE tokens concatenated into a single
 * stream; attention computed as QKᵀ, softmax, V in on-chip tiles), and by the
 * FLOP table of "TMAP image-to-video inference acceleration" (joto.ai),
 * section on hiding communication, where this operator
 * (aten._scaled_dot_product_flash_attention) is about 74% of all FLOPs.
 *
 *   q, k, v  device bf16, logical shape [B, H, N, d], d contiguous (stride 1).
 *   o        device bf16 output, same shape; its strides are `strides` too.
 *   strides  element strides of dimensions (b, h, n), shared by q, k, v, o;
 *            NULL means contiguous [B, H, N, d].  Each stride × 2 bytes must
 *            be a multiple of 16.
 *   d        64 or 128 (others: DIT_ERR_UNSUPPORTED).
 *   scale    logit scale; scale <= 0 means 1/sqrt(d) (computed in fp32).
 *   Pointers must be 16-byte aligned.  B, H, N >= 1.
 *   o must not overlap q, k or v.  Accumulation is fp32; O is rounded to
 *   bf16 (round to nearest even).
 */
dit_status dit_attn_fwd(const void* q, const void* k, const void* v, void* o,
                        int B, int H, int N, int d, const int64_t* strides,
                        float scale, void* stream);

/*
 * dit_attn_fwd_ex — dit_attn_fwd with separate query and key lengths and an
 * optional log-sum-exp output: Nq query rows attend to Nkv keys, and
 *   lse[b,h,i] = ln Σ_j exp(scale · q_i·k_j)        (fp32, natural log)
 *
 * Defined by: "ParaAttention" (diffusers docs), section "Context Parallelism",
 * and the TMAP image-to-video blog, section on sequence parallelism: the keys
 * of one attention may be split into chunks (one per device in ring-style
 * context parallelism).  Each chunk's normalised output and log-sum-exp are
 * what dit_attn_merge combines into the attention over all keys.
 *
 *   q, o        bf16 [B, H, Nq, d], strides q_strides (elements; NULL:
 *               contiguous); o must not overlap any input.
 *   k, v        bf16 [B, H, Nkv, d], strides kv_strides (NULL: contiguous).
 *               A chunk of a longer K/V is addressed by offsetting the base
 *               pointers by (start · sn) elements and passing its length.
 *   lse         device fp32 [B, H, Nq] contiguous, or NULL.
 *   Nq, Nkv >= 1; d in {64, 128}; alignment and stride rules as dit_attn_fwd.
 */
dit_status dit_attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                           int B, int H, int Nq, int Nkv, int d,
                           const int64_t* q_strides, const int64_t* kv_strides,
                           float scale, void* stream);

/*
 * dit_attn_merge — the attention over the union of key chunks, from the
 * chunks' outputs and log-sum-exps:
 *   lse = ln Σ_c exp(lse_c),   o = Σ_c exp(lse_c − lse) · o_c
 * (same passages as dit_attn_fwd_ex).
 *
 *   o_parts     host array of n_parts (1..16) device pointers, bf16
 *               [B, H, N, d] with `strides` (NULL: contiguous), 16-byte aligned.
 *   lse_parts   host array of n_parts device pointers, fp32 [B, H, N].
 *   o           bf16 output with the same strides; lse: fp32 [B, H, N] or NULL.
 *               Neither may overlap an input.
 *   d a multiple of 8 up to 256.  A row whose every lse_c is −inf gets o = 0
 *   and lse = −inf.  Weights use the largest lse_c as the shift (fp32).
 */
dit_status dit_attn_merge(const void* const* o_parts, const float* const* lse_parts, int n_parts,
                          int B, int H, int N, int d, const int64_t* strides,
                          void* o, float* lse, void* stream);

/*
 * dit_attn_fwd_q8 — the same attention with 8-bit operands.
 *
 * Defined by: "TMAP image-to-video inference acceleration" (joto.ai), section
 * on optimising operator details: 8-bit SageAttention-style attention with
 * per-block quantisation.  An all-zero channel made the quantisation scale 0
 * and the division by it turned the video black (NaN); the scale here is
 * guarded.  Recipe:
 *   Q  -> INT8 per block of 128 tokens (all d channels);
 *   K  -> optionally minus its per-channel mean over the N tokens (smooth_k;
 *         a per-row logit shift, so the softmax is unchanged), then INT8 per
 *         block of 64 tokens;
 *   INT8 scales: amax over the block's valid tokens, scale = amax/127,
 *         codes = round-half-even(x·127/amax) in [-127, 127]; amax = 0, or an
 *         amax so small that 127/amax overflows fp32, gives scale 0 and
 *         zero codes (V likewise with 448/amax);
 *   S = Q8·K8ᵀ in int32, dequantised by q_scale·k_scale;
 *   P·V in FP8 e4m3 (pv_mode DIT_PV_FP8_E4M3: V per channel, scale
 *         amax/448; P scaled by 2^6.5 before e4m3) or in bf16 (DIT_PV_BF16:
 *         P bf16, V as given).
 *
 *   Arguments as dit_attn_fwd, plus:
 *   smooth_k        0 or 1.
 *   pv_mode         a dit_pv_mode.
 *   workspace       device memory of dit_attn_q8_workspace_bytes(...) bytes,
 *                   256-byte aligned, not overlapping q, k, v or o; no
 *                   initialisation needed.  It receives the codes and scales
 *                   (layout: dit_attn_q8_workspace_layout).
 *   d               64 or 128 (others: DIT_ERR_UNSUPPORTED).
 *   Launches the pre-pass (3-5 kernels) and the attention kernel on `stream`.
 */
size_t dit_attn_q8_workspace_bytes(int B, int H, int N, int d, int pv_mode);
dit_status dit_attn_fwd_q8(const void* q, const void* k, const void* v, void* o,
                           int B, int H, int N, int d, const int64_t* strides,
                           float scale, int smooth_k, int pv_mode,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * dit_attn_q8_quantize — only the pre-pass of dit_attn_fwd_q8: writes the
 * codes and scales into `workspace` (arguments as dit_attn_fwd_q8, no o).
 *
 * dit_attn_q8_workspace_layout — byte offsets inside the workspace, in this
 * order: Q codes (int8 [B,H,N,d]), K codes (int8 [B,H,N,d]), V codes (e4m3
 * [B,H,N,d], FP8 mode only), Q scales (fp32 [B,H,ceil(N/128)]), K scales
 * (fp32 [B,H,ceil(N/64)]), K channel means (fp32 [B,H,d]; zeros when
 * smooth_k = 0), V scales (fp32 [B,H,d]), V inverse scales (fp32 [B,H,d]).
 * offsets: host array of 8 size_t.
 */
dit_status dit_attn_q8_quantize(const void* q, const void* k, const void* v,
                                int B, int H, int N, int d, const int64_t* strides,
                                int smooth_k, int pv_mode,
                                void* workspace, size_t workspace_bytes, void* stream);
dit_status dit_attn_q8_workspace_layout(int B, int H, int N, int d, int pv_mode, size_t* offsets);

/*
 * Token-sharded 8-bit path (Ulysses context parallelism with 8-bit attention).
 *
 * Defined by: "ParaAttention" (diffusers docs), section "Context Parallelism",
 * and the TMAP image-to-video blog, where sequence parallelism (Ulysses, the
 * all-to-all overlapped with computation) is combined with 8-bit attention.
 * Each device holds a slice of the tokens of every head.  The K channel mean
 * and the V channel maxima span all tokens, so:
 *   1. dit_attn_q8_channel_stats: this slice's per-channel K sums (fp64,
 *      zero when smooth_k = 0) and V maxima (fp32, zero in bf16-PV mode),
 *      both [B, H, d] device arrays; the devices then add the sums and take
 *      the maximum of the maxima (e.g. two all-reduces);
 *   2. dit_attn_q8_quantize_global: writes this slice's codes and scales into
 *      the workspace (layout of dit_attn_q8_workspace_layout for the slice's N
 *      tokens) with the K mean = k_sum / n_total and V scales = v_amax / 448;
 *   3. the caller moves codes and scales in the all-to-all (1 byte per value
 *      instead of 2) into a workspace laid out for H' heads and all N tokens,
 *      with the V scales of those heads;
 *   4. dit_attn_fwd_q8_prequantized: the attention kernel alone on that
 *      workspace (v: the bf16 V [B, H', N, d] in bf16-PV mode, else unused
 *      and may be NULL; o and v share `strides`).
 * When every slice holds whole 128-token blocks, the codes equal those that
 * dit_attn_fwd_q8 writes for the whole sequence, and so does the output.
 * Arguments, alignment and errors as dit_attn_q8_quantize / dit_attn_fwd_q8;
 * n_total >= N.
 */
dit_status dit_attn_q8_channel_stats(const void* k, const void* v, int B, int H, int N, int d,
                                     const int64_t* strides, int smooth_k, int pv_mode,
                                     double* k_sum, float* v_amax,
                                     void* workspace, size_t workspace_bytes, void* stream);
dit_status dit_attn_q8_quantize_global(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                                       const int64_t* strides, int smooth_k, int pv_mode,
                                       const double* k_sum, const float* v_amax, int64_t n_total,
                                       void* workspace, size_t workspace_bytes, void* stream);
dit_status dit_attn_fwd_q8_prequantized(const void* workspace, size_t workspace_bytes, const void* v, void* o,
                                        int B, int H, int N, int d, const int64_t* strides, float scale,
                                        int pv_mode, void* stream);

/*
 * dit_attn_q8_quantize_scatter — steps 2 and 3 above in one launch sequence:
 * the quantisers of dit_attn_q8_quantize_global store every code and block
 * scale of this rank's slice straight into the workspace of the rank that
 * owns its head after the all-to-all, so no separate exchange of the codes
 * runs.  Same sources: ParaAttention, "Context Parallelism"; the TMAP
 * image-to-video blog's sequence parallelism with 8-bit attention.
 *
 *   q, k, v, B, H, N, d, strides, smooth_k, pv_mode, k_sum, v_amax
 *                  as dit_attn_q8_quantize_global, for this rank's slice of N
 *                  tokens (the combined statistics of all world·N tokens).
 *   rank, world    this rank and the group size, 1 <= world <= 16; H must be
 *                  a multiple of world and, when world > 1, N of 128.
 *   dst_workspaces host array of `world` device pointers: the workspace of
 *                  each rank for the head-sharded problem (B, H/world heads,
 *                  world·N tokens), dit_attn_q8_workspace_bytes of it, 256-byte
 *                  aligned, pairwise disjoint.  Entry r receives this slice's
 *                  codes and scales of heads [r·H/world, (r+1)·H/world) at
 *                  token offset rank·N; entry `rank` also receives this rank's
 *                  heads' V scales (FP8 mode).  On a multi-GPU node the other
 *                  entries are peer-mapped device memory (P2P stores over
 *                  NVLink); the caller makes every rank's stores complete
 *                  (stream synchronisation and a group barrier) before any
 *                  rank runs dit_attn_fwd_q8_prequantized on its entry.
 *   workspace      this rank's slice workspace (dit_attn_q8_workspace_bytes for
 *                  B, H, N): receives the K mean and V scales.
 * Errors as dit_attn_q8_quantize_global; DIT_ERR_WORKSPACE for a destination
 * that is too small, misaligned or overlapping another buffer.
 */
dit_status dit_attn_q8_quantize_scatter(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                                        const int64_t* strides, int smooth_k, int pv_mode, const double* k_sum,
                                        const float* v_amax, int rank, int world, void* const* dst_workspaces,
                                        size_t dst_workspace_bytes, void* workspace, size_t workspace_bytes,
                                        void* stream);

/*
 * fbc_rel_l1 — first-block-cache residual difference and decision:
 *   rel  = Σ|r_cur − r_prev| / Σ|r_prev|   (over all n elements)
 *   skip = rel < threshold                 (1: reuse the cached residual)
 *
 * Defined by: "ParaAttention" (diffusers docs), section "First Block Cache":
 * the residual of the first transformer block between consecutive steps
 * approximates the change of the model output; when it is small enough
 * (0.08 for FLUX), the remaining blocks are skipped and the cache is reused.
 * Readings where the page is silent: the comparison is strict (at equality
 * the step is computed); Σ|r_prev| = 0 gives rel = 0 when the numerator is 0
 * too, else +inf.
 *
 *   r_cur, r_prev  device arrays of n elements of `dtype` (fp32 or bf16),
 *                  16-byte aligned.  n >= 1.
 *   out_rel        device double[1];  out_skip  device int32[1].
 *   workspace      device memory of fbc_rel_l1_workspace_bytes(n) bytes,
 *                  16-byte aligned, zero-filled before its first use; each
 *                  call leaves it zero-filled again.  Calls that share one
 *                  workspace must be ordered (same stream, or synchronised).
 *   Partial sums are fp32 per thread and fp64 across threads and blocks, in a
 *   fixed order: the result is deterministic for a given n on a given GPU model
 *   (the grid, at most one wave of resident blocks, follows the SM count).
 */
size_t fbc_rel_l1_workspace_bytes(int64_t n);
dit_status fbc_rel_l1(const void* r_cur, const void* r_prev, int64_t n, int dtype,
                      float threshold, double* out_rel, int32_t* out_skip,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * fbc_rel_l1_sums / fbc_rel_l1_finish — fbc_rel_l1 in two halves, for a
 * residual sharded across devices (as the token sequence is under the context
 * parallelism of the ParaAttention page, section "Context Parallelism"):
 *   fbc_rel_l1_sums   out_sums[0] = Σ|r_cur − r_prev|, out_sums[1] = Σ|r_prev|
 *                     over this device's n elements (device double[2], 8-byte
 *                     aligned); arguments and workspace rules as fbc_rel_l1.
 *   (the caller all-reduces the two doubles, e.g. one NCCL sum)
 *   fbc_rel_l1_finish rel and skip from the (reduced) sums, with fbc_rel_l1's
 *                     conventions; sums: device double[2].  One tiny launch.
 * With one device, sums then finish gives exactly fbc_rel_l1's result.
 */
dit_status fbc_rel_l1_sums(const void* r_cur, const void* r_prev, int64_t n, int dtype,
                           double* out_sums, void* workspace, size_t workspace_bytes, void* stream);
dit_status fbc_rel_l1_finish(const double* sums, float threshold, double* out_rel, int32_t* out_skip,
                             void* stream);

/*
 * fbc_rel_l1_noalloc — fbc_rel_l1 without a caller-provided workspace, for
 * callers that cannot allocate device memory.  Such a caller holds only its
 * input and output pointers: a plugin inside an inference engine, or a module
 * in a framework whose caching allocator owns all device memory.  For it,
 * cudaMalloc is either unavailable or an implicit device-wide synchronisation
 * it cannot afford inside a denoising step.  No page describes this call: it is
 * a deployment variant of fbc_rel_l1.
 *
 *   Arguments, result and determinism are those of fbc_rel_l1.  The call
 *   allocates nothing.  Its scratch (a 16 B finishing ticket plus one fp64
 *   partial pair per block, at most 1024 blocks: 16,400 B in all) is a fixed
 *   array inside the library.  Every GPU that loads the library holds it until
 *   the process exits.  A request whose scratch need exceeds that size returns
 *   DIT_ERR_WORKSPACE.  With the current kernel the need is the same for every
 *   n, so every n >= 1 fits.
 *   The first call on each device does a one-time set-up: it looks up the
 *   array's device address with that device current.  Make that first call
 *   before any stream capture.
 *   Every call clears the ticket (an asynchronous memset on `stream`) before
 *   its launch.  All calls share one array, which keeps the last call's
 *   partial sums, so calls that may overlap on the GPU race: calls on
 *   different streams without ordering, or concurrent calls from several host
 *   threads.  Order such calls, or use fbc_rel_l1 with one workspace each.
 */
dit_status fbc_rel_l1_noalloc(const void* r_cur, const void* r_prev, int64_t n, int dtype,
                              float threshold, double* out_rel, int32_t* out_skip, void* stream);

/*
 * dit_compare_stats — error of an output against a reference, per segment.
 *
 * Defined by: TMAP image-to-video blog, "keeping video quality": the error of
 * each attention layer's 8-bit output over the denoising steps is what picks
 * the layers that go back to 16-bit attention.  For each of n_segments
 * contiguous segments of segment_len elements:
 *   out[3s+0] = Σ|test − ref| / Σ|ref|              (relative L1)
 *   out[3s+1] = Σ ref·test / sqrt(Σ ref² · Σ test²)  (cosine similarity)
 *   out[3s+2] = max |test − ref|
 * Empty norms: relative L1 is 0 when both sums are 0 and +inf when only Σ|ref|
 * is; the cosine is 1 when both segments are all zero and 0 when one is.
 *
 *   ref, test   device arrays of n_segments * segment_len elements of
 *               `dtype` (fp32 or bf16), aligned to the element size.  With
 *               16-byte aligned bases and segments of whole 16-byte vectors
 *               the kernel reads 16-byte vectors, else single elements.
 *   n_segments  1..65535 (e.g. B*H for per-head errors of a [B,H,N,d] output).
 *   out         device double[3 * n_segments].
 *   workspace   device memory of dit_compare_workspace_bytes(...) bytes,
 *               16-byte aligned, zero-filled before its first use; each call
 *               leaves it zero-filled again.  Calls sharing it must be ordered.
 *   Sums are fp32 over one 16-byte vector, fp64 beyond, in a fixed order:
 *   deterministic for a given shape.
 * Returns 0 from dit_compare_workspace_bytes for invalid shapes.
 */
size_t dit_compare_workspace_bytes(int64_t n_segments, int64_t segment_len, int dtype);
dit_status dit_compare_stats(const void* ref, const void* test, int64_t n_segments, int64_t segment_len,
                             int dtype, double* out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * dit_get_device_status — synchronises `stream`, then returns and clears the
 * device-side error word of the current device (DIT_ERR_TIMEOUT if a bounded
 * wait inside a kernel ran out since the last call), or DIT_ERR_CUDA if the
 * synchronisation itself failed.
 */
dit_status dit_get_device_status(void* stream);

/*
 * dit_wait_selftest — exercises the bounded wait that every kernel of this
 * library uses (no page counterpart: it tests the library's own failure
 * detection).  One warp waits on an mbarrier that nothing arrives on, gives
 * up after the wait limit (1 s), records DIT_ERR_TIMEOUT in the device error
 * word and returns, leaving the GPU context usable.
 *   out_completed  device int32 [1]; set to 0 when the wait gave up (1 would
 *                  mean the barrier completed, which cannot happen).
 * Asynchronous on `stream` (it occupies the stream for about 1 s); read the
 * outcome with dit_get_device_status, which then returns DIT_ERR_TIMEOUT.
 * Returns DIT_ERR_INVALID_ARG for a NULL out_completed, DIT_ERR_CUDA if the
 * launch fails.
 */
dit_status dit_wait_selftest(int32_t* out_completed, void* stream);

/* Human-readable name of a status code (static string, never NULL). */
const char* dit_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* DIT_ATTN_H */
