/*
 * dit_cache.h — step-caching decisions kept on the device, and the CUDA-graph
 * plumbing that lets a decision skip work without a host round trip.
 *
 * A diffusion transformer runs the same network once per denoising step.  The
 * step caches below decide, on the device, whether a step runs the expensive
 * part of the network ("compute") or reuses what an earlier step produced
 * ("use cache").  The decision is written to a device-resident state and can
 * set a CUDA-graph conditional, so a captured step graph branches on it by
 * itself: no copy to the host and no synchronisation per step.
 *
 * Two policies:
 *   fbcache_step   first-block / dual-block cache.  "ParaAttention" (diffusers
 *                  docs), section "First Block Cache": the relative L1 change
 *                  of the residual of the first block(s) decides.  vLLM-Omni
 *                  cache-dit guide, section "DBCache" (key parameters) and the
 *                  "DiffusionCacheConfig" parameter table: warm-up steps,
 *                  a limit on cached steps in all and in a row, a threshold.
 *   teacache_step  TeaCache.  TMAP image-to-video blog, "TeaCache" (difference
 *                  estimation and rescaling; inference flow): the relative L1
 *                  distance of the timestep-modulated input between adjacent
 *                  steps, mapped through a calibrated polynomial, is summed
 *                  while the cache is reused and restarts when a step
 *                  computes.
 *
 * Both reduce their two inputs in one HBM-bound launch with the fixed-order
 * fp64 summation of fbc_rel_l1 (same workspace size and rules) and finish in
 * the last block.  Calls that share a state or a workspace must be ordered.
 *
 * Readings where the pages leave a step open: a step with no stored residual
 * computes; the stored residual is the one of the last computed step (the
 * caller refreshes it when the step computes, e.g. inside the conditional
 * body); the comparison is strict and takes the threshold as the float given;
 * a negative max_continuous_cached_steps means no limit, like -1 for
 * max_cached_steps; the difference is not evaluated during warm-up or with no
 * stored residual (reported as NaN); the TeaCache sum restarts at zero on
 * every computed step; polynomial coefficients are in ascending powers.
 */
#ifndef DIT_CACHE_H
#define DIT_CACHE_H

#include <stddef.h>
#include <stdint.h>

#include "dit_attn.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Decision codes: 0 reuses the cache, every other value computes (and says why). */
typedef enum dit_cache_decision {
    DIT_CACHE_USE = 0,            /* reuse the cached result */
    DIT_CACHE_WARMUP = 1,         /* step < max_warmup_steps */
    DIT_CACHE_NO_PREV = 2,        /* nothing stored to compare with */
    DIT_CACHE_ABOVE_THRESHOLD = 3,/* difference (or TeaCache sum) >= threshold */
    DIT_CACHE_MAX_CACHED = 4,     /* max_cached_steps reached */
    DIT_CACHE_MAX_CONTINUOUS = 5  /* max_continuous_cached_steps reached */
} dit_cache_decision;

/* Policy of fbcache_step (host memory; read during the call, so a captured
 * graph keeps the values it was captured with).  Defaults of the
 * DiffusionCacheConfig table: 4, -1, 3, 0.24. */
typedef struct dit_cache_policy {
    int32_t max_warmup_steps;            /* >= 0 */
    int32_t max_cached_steps;            /* -1 (or any negative): no limit */
    int32_t max_continuous_cached_steps; /* negative: no limit */
    float residual_diff_threshold;       /* finite */
} dit_cache_policy;

/* Device-resident state (40 bytes, 8-byte aligned).  All zero = a fresh run:
 * clear it with dit_cache_state_reset before the first step of each run. */
typedef struct dit_cache_state {
    int32_t step;              /* steps decided so far */
    int32_t cached_steps;      /* of which reused the cache */
    int32_t continuous_cached; /* length of the current run of cached steps */
    int32_t has_prev;          /* a residual / input is stored */
    int32_t last_decision;     /* dit_cache_decision of the last step */
    int32_t reserved;
    double last_rel;           /* difference of the last step (NaN if not evaluated) */
    double acc;                /* TeaCache running sum (0 for fbcache_step) */
} dit_cache_state;

/* One entry per step (24 bytes), written at index state.step when a trace is given. */
typedef struct dit_cache_trace {
    double rel;        /* difference evaluated at the step (NaN if none) */
    double acc;        /* TeaCache sum after the step (0 for fbcache_step) */
    int32_t decision;  /* dit_cache_decision */
    int32_t reserved;
} dit_cache_trace;

/* Zero the state on `stream` (asynchronous). state: device, 8-byte aligned. */
dit_status dit_cache_state_reset(dit_cache_state* state, void* stream);

/* Workspace bytes of fbcache_step / teacache_step for n elements (0 if n < 1). */
size_t dit_cache_workspace_bytes(int64_t n);

/*
 * fbcache_step — one decision of the first-block cache.
 *
 *   r_cur     device array of n elements of `dtype` (DIT_DTYPE_F32 or BF16):
 *             the residual of the first Fn blocks at this step.
 *   r_prev    device array, same shape: the stored residual.  Not read when
 *             the difference is not evaluated (warm-up, or has_prev == 0).
 *             Both 16-byte aligned.
 *   policy    host pointer, see dit_cache_policy.
 *   state     device dit_cache_state, updated in place.
 *   trace     device array of trace_capacity entries or NULL; entry
 *             state.step is written when state.step < trace_capacity.
 *   use_cond  0: no graph conditional.  1: the last block sets the
 *             conditional `cond_handle` to 1 when the step computes and 0 when
 *             it reuses the cache.  The handle must come from
 *             dit_graph_cond_create on the same, still capturing, stream
 *             (checked: otherwise DIT_ERR_INVALID_ARG, nothing launched).
 *   workspace as fbc_rel_l1 (dit_cache_workspace_bytes(n) bytes, 16-byte
 *             aligned, zero before first use, left zero by every call).
 *
 * After the call (in stream order) state.last_decision holds the decision.
 * The caller stores r_cur as the new r_prev when the step computes: inside
 * the conditional body, or conditioned on last_decision != 0.
 * Fn and Bn (the numbers of leading and trailing blocks that always run) are
 * the caller's split of the network around this call; the call itself only
 * sees the residual it is given.
 */
dit_status fbcache_step(const void* r_cur, const void* r_prev, int64_t n, int dtype,
                        const dit_cache_policy* policy, dit_cache_state* state,
                        dit_cache_trace* trace, int32_t trace_capacity,
                        int use_cond, unsigned long long cond_handle,
                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * teacache_step — one decision of the TeaCache accumulator, and the update of
 * the stored input in the same pass.
 *
 *   x_cur     device array of n elements of `dtype`: the timestep-modulated
 *             input of this step.
 *   x_prev    device array, same shape, 16-byte aligned, not overlapping
 *             x_cur: the previous step's input on entry, x_cur's values on
 *             exit (every step, cached or not).
 *   coeffs    host array of n_coeffs doubles (1..8), ascending powers:
 *             rescaled = c[0] + c[1] rel + c[2] rel^2 + ...
 *   threshold the sum below which the cache is reused (finite).
 *   state, trace, use_cond, cond_handle, workspace: as fbcache_step.
 *
 * Step with has_prev == 0: computes, sum reset to 0.  Otherwise
 * acc += rescaled(rel); acc < threshold reuses the cache, else the step
 * computes and acc restarts at 0.
 */
dit_status teacache_step(const void* x_cur, void* x_prev, int64_t n, int dtype,
                         const double* coeffs, int32_t n_coeffs, float threshold,
                         dit_cache_state* state, dit_cache_trace* trace, int32_t trace_capacity,
                         int use_cond, unsigned long long cond_handle,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * CUDA-graph plumbing for a step graph that branches on the decision.
 *
 *   dit_graph_capture_begin(s)      begin capturing `s` (relaxed mode).
 *   ... enqueue the first Fn blocks on s ...
 *   dit_graph_cond_create(s, &h)    create a conditional handle on the graph
 *                                   being captured on s (default value 1).
 *   fbcache_step(..., use_cond=1, h, ..., s)
 *   dit_graph_cond_body_begin(s, h, body)
 *                                   add an IF node after everything captured
 *                                   on s so far and start capturing `body`
 *                                   (another stream) into its body graph.
 *   ... enqueue the skippable blocks, and r_prev <- r_cur, on body ...
 *   dit_graph_cond_body_end(body)   end the body capture.
 *   ... enqueue the trailing Bn blocks on s ...
 *   dit_graph_capture_end(s, &exec) end the capture and instantiate; the
 *                                   executable graph is returned as an opaque
 *                                   handle.
 *   dit_graph_launch(exec, s) per step; dit_graph_destroy(exec) at the end.
 *
 * Every call returns DIT_ERR_INVALID_ARG for a stream in the wrong capture
 * state and DIT_ERR_CUDA when a CUDA call fails; a failed
 * dit_graph_capture_end still ends the capture.  Only operations allowed in
 * a conditional body (kernels, memcpy, memset, nested conditionals) may be
 * captured on `body`; nothing may allocate device memory during the capture.
 */
dit_status dit_graph_capture_begin(void* stream);
dit_status dit_graph_cond_create(void* stream, unsigned long long* cond_handle);
dit_status dit_graph_cond_body_begin(void* stream, unsigned long long cond_handle, void* body_stream);
dit_status dit_graph_cond_body_end(void* body_stream);
dit_status dit_graph_capture_end(void* stream, void** graph_exec);
dit_status dit_graph_launch(void* graph_exec, void* stream);
dit_status dit_graph_destroy(void* graph_exec);

#ifdef __cplusplus
}
#endif

#endif /* DIT_CACHE_H */
