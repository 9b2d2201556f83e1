// Step-caching decisions on the device (declared in include/dit_cache.h).
//
// fbcache_step: first-block / dual-block cache.  "ParaAttention" (diffusers
// docs), section "First Block Cache", and the vLLM-Omni cache-dit guide,
// section "DBCache" and the "DiffusionCacheConfig" table: the relative L1
// change of the first blocks' residual against the stored one decides, under
// a warm-up, a limit on cached steps in all and one on cached steps in a row.
//
// teacache_step: TMAP image-to-video blog, "TeaCache": the relative L1
// distance of the modulated input between adjacent steps, rescaled by a
// calibrated polynomial, is summed; the cache is reused while the sum stays
// below the threshold.
//
// Both run the shared one-pass reduction (rel_l1_reduce.cuh); the policy is
// the epilogue of its last block, which updates the device-resident state,
// appends the trace entry and, inside a captured graph, sets the conditional
// that gates the skippable work.  The host never sees the decision.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <iterator>
#include <mutex>
#include <unordered_map>

#include "dit_cache.h"
#include "internal.h"
#include "rel_l1_reduce.cuh"

namespace ditk {
namespace {

constexpr int kMaxCoeffs = 8;

__device__ __forceinline__ double quiet_nan() { return __longlong_as_double(0x7ff8000000000000LL); }

__device__ __forceinline__ void record(dit_cache_trace* trace, int32_t cap, int step, double rel, double acc,
                                       int d) {
    if (trace != nullptr && step < cap) {
        dit_cache_trace e;
        e.rel = rel;
        e.acc = acc;
        e.decision = d;
        e.reserved = 0;
        trace[step] = e;
    }
}

struct EpiFbcPolicy {
    static constexpr bool kProgrammatic = false;  // reads the state the previous step wrote first
    int32_t warmup, max_cached, max_cont;
    float threshold;
    dit_cache_state* st;
    dit_cache_trace* trace;
    int32_t trace_cap;
    int32_t use_cond;
    cudaGraphConditionalHandle cond;

    // The sums are needed only once warm-up is over and a residual is stored.
    __device__ bool evaluate() const { return __ldcg(&st->step) >= warmup && __ldcg(&st->has_prev) != 0; }

    __device__ void finish(double num, double den, bool eval) const {
        const int step = st->step, cached = st->cached_steps, cont = st->continuous_cached;
        const bool has_prev = st->has_prev != 0;
        const double rel = eval ? rl1_ratio(num, den) : quiet_nan();
        int d;
        if (step < warmup)
            d = DIT_CACHE_WARMUP;
        else if (!has_prev)
            d = DIT_CACHE_NO_PREV;
        else if (!(rel < static_cast<double>(threshold)))
            d = DIT_CACHE_ABOVE_THRESHOLD;
        else if (max_cached >= 0 && cached >= max_cached)
            d = DIT_CACHE_MAX_CACHED;
        else if (max_cont >= 0 && cont >= max_cont)
            d = DIT_CACHE_MAX_CONTINUOUS;
        else
            d = DIT_CACHE_USE;
        st->step = step + 1;
        if (d == DIT_CACHE_USE) {
            st->cached_steps = cached + 1;
            st->continuous_cached = cont + 1;
        } else {
            st->continuous_cached = 0;
            st->has_prev = 1;  // the computing step stores its residual
        }
        st->last_decision = d;
        st->last_rel = rel;
        st->acc = 0.0;
        record(trace, trace_cap, step, rel, 0.0, d);
        if (use_cond) cudaGraphSetConditional(cond, d != DIT_CACHE_USE ? 1u : 0u);
    }
};

struct EpiTeaCache {
    static constexpr bool kProgrammatic = false;
    double coeffs[kMaxCoeffs];
    int32_t n_coeffs;
    float threshold;
    dit_cache_state* st;
    dit_cache_trace* trace;
    int32_t trace_cap;
    int32_t use_cond;
    cudaGraphConditionalHandle cond;

    // The kernel streams both inputs on every step anyway (it stores x_cur);
    // the sums mean something only when an input was stored before.
    __device__ bool evaluate() const { return __ldcg(&st->has_prev) != 0; }

    __device__ void finish(double num, double den, bool eval) const {
        const int step = st->step, cached = st->cached_steps, cont = st->continuous_cached;
        double rel, acc;
        int d;
        if (!eval) {
            rel = quiet_nan();
            acc = 0.0;
            d = DIT_CACHE_NO_PREV;
        } else {
            rel = rl1_ratio(num, den);
            // Horner's scheme, ascending powers, no fused multiply-add.
            double r = 0.0;
            for (int k = n_coeffs - 1; k >= 0; --k) r = __dadd_rn(__dmul_rn(r, rel), coeffs[k]);
            acc = st->acc + r;
            if (acc < static_cast<double>(threshold)) {
                d = DIT_CACHE_USE;
            } else {
                d = DIT_CACHE_ABOVE_THRESHOLD;
                acc = 0.0;
            }
        }
        st->step = step + 1;
        st->has_prev = 1;
        if (d == DIT_CACHE_USE) {
            st->cached_steps = cached + 1;
            st->continuous_cached = cont + 1;
        } else {
            st->continuous_cached = 0;
        }
        st->last_decision = d;
        st->last_rel = rel;
        st->acc = acc;
        record(trace, trace_cap, step, rel, acc, d);
        if (use_cond) cudaGraphSetConditional(cond, d != DIT_CACHE_USE ? 1u : 0u);
    }
};

// ---- conditional handles -------------------------------------------------
// A kernel may set a conditional only inside the graph that owns the handle.
// Every handle made by dit_graph_cond_create is recorded with the id of the
// capture it belongs to, and a step asked to set it must be launched into
// that same capture.
std::mutex g_cond_mu;
std::unordered_map<unsigned long long, unsigned long long> g_cond_capture;

bool capture_info(cudaStream_t s, unsigned long long* id, cudaGraph_t* graph, const cudaGraphNode_t** deps,
                  size_t* ndeps) {
    cudaStreamCaptureStatus status = cudaStreamCaptureStatusNone;
    if (cudaStreamGetCaptureInfo(s, &status, id, graph, deps, ndeps) != cudaSuccess) return false;
    return status == cudaStreamCaptureStatusActive;
}

bool cond_belongs_to(cudaStream_t s, unsigned long long handle) {
    unsigned long long id = 0;
    if (!capture_info(s, &id, nullptr, nullptr, nullptr)) return false;
    std::lock_guard<std::mutex> lk(g_cond_mu);
    auto it = g_cond_capture.find(handle);
    return it != g_cond_capture.end() && it->second == id;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

dit_status check_step_common(const void* cur, const void* prev, int64_t n, int dtype, const dit_cache_state* state,
                             const dit_cache_trace* trace, int32_t trace_capacity, int use_cond,
                             unsigned long long cond, const void* ws, size_t ws_bytes, cudaStream_t s) {
    if (!cur || !prev || !state || n < 1) return DIT_ERR_INVALID_ARG;
    if (dtype != DIT_DTYPE_F32 && dtype != DIT_DTYPE_BF16) return DIT_ERR_INVALID_ARG;
    if (!aligned(cur, 16) || !aligned(prev, 16) || !aligned(state, 8)) return DIT_ERR_INVALID_ARG;
    if (trace && (!aligned(trace, 8) || trace_capacity < 0)) return DIT_ERR_INVALID_ARG;
    if (use_cond != 0 && use_cond != 1) return DIT_ERR_INVALID_ARG;
    if (!ws || !aligned(ws, 16) || ws_bytes < fbc_workspace_bytes(n)) return DIT_ERR_WORKSPACE;
    if (use_cond && !cond_belongs_to(s, cond)) return DIT_ERR_INVALID_ARG;
    return DIT_OK;
}

}  // namespace
}  // namespace ditk

using namespace ditk;

extern "C" {

dit_status dit_cache_state_reset(dit_cache_state* state, void* stream) {
    if (!state || !aligned(state, 8)) return DIT_ERR_INVALID_ARG;
    const dit_status st = check_device();
    if (st != DIT_OK) return st;
    return cudaMemsetAsync(state, 0, sizeof(dit_cache_state), static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? DIT_OK
               : DIT_ERR_CUDA;
}

size_t dit_cache_workspace_bytes(int64_t n) { return n < 1 ? 0 : fbc_workspace_bytes(n); }

dit_status fbcache_step(const void* r_cur, const void* r_prev, int64_t n, int dtype, const dit_cache_policy* policy,
                        dit_cache_state* state, dit_cache_trace* trace, int32_t trace_capacity, int use_cond,
                        unsigned long long cond_handle, void* workspace, size_t workspace_bytes, void* stream) {
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (!policy || policy->max_warmup_steps < 0 || !std::isfinite(policy->residual_diff_threshold))
        return DIT_ERR_INVALID_ARG;
    dit_status st = check_step_common(r_cur, r_prev, n, dtype, state, trace, trace_capacity, use_cond, cond_handle,
                                      workspace, workspace_bytes, s);
    if (st != DIT_OK) return st;
    if ((st = check_device()) != DIT_OK) return st;
    EpiFbcPolicy epi;
    epi.warmup = policy->max_warmup_steps;
    epi.max_cached = policy->max_cached_steps;
    epi.max_cont = policy->max_continuous_cached_steps;
    epi.threshold = policy->residual_diff_threshold;
    epi.st = state;
    epi.trace = trace;
    epi.trace_cap = trace ? trace_capacity : 0;
    epi.use_cond = use_cond;
    epi.cond = use_cond ? cond_handle : 0ull;
    const cudaError_t e = launch_rel_l1<false>(r_cur, r_prev, n, dtype, epi, workspace, s);
    return e == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

dit_status teacache_step(const void* x_cur, void* x_prev, int64_t n, int dtype, const double* coeffs,
                         int32_t n_coeffs, float threshold, dit_cache_state* state, dit_cache_trace* trace,
                         int32_t trace_capacity, int use_cond, unsigned long long cond_handle, void* workspace,
                         size_t workspace_bytes, void* stream) {
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (!coeffs || n_coeffs < 1 || n_coeffs > kMaxCoeffs || !std::isfinite(threshold)) return DIT_ERR_INVALID_ARG;
    for (int k = 0; k < n_coeffs; ++k)
        if (!std::isfinite(coeffs[k])) return DIT_ERR_INVALID_ARG;
    dit_status st = check_step_common(x_cur, x_prev, n, dtype, state, trace, trace_capacity, use_cond, cond_handle,
                                      workspace, workspace_bytes, s);
    if (st != DIT_OK) return st;
    // The pass stores x_cur into x_prev while reading both: they must not overlap.
    const int64_t bytes = n * (dtype == DIT_DTYPE_F32 ? 4 : 2);
    const uintptr_t a = reinterpret_cast<uintptr_t>(x_cur), b = reinterpret_cast<uintptr_t>(x_prev);
    if (a < b + static_cast<uintptr_t>(bytes) && b < a + static_cast<uintptr_t>(bytes)) return DIT_ERR_INVALID_ARG;
    if ((st = check_device()) != DIT_OK) return st;
    EpiTeaCache epi;
    for (int k = 0; k < kMaxCoeffs; ++k) epi.coeffs[k] = k < n_coeffs ? coeffs[k] : 0.0;
    epi.n_coeffs = n_coeffs;
    epi.threshold = threshold;
    epi.st = state;
    epi.trace = trace;
    epi.trace_cap = trace ? trace_capacity : 0;
    epi.use_cond = use_cond;
    epi.cond = use_cond ? cond_handle : 0ull;
    const cudaError_t e = launch_rel_l1<true>(x_cur, x_prev, n, dtype, epi, workspace, s);
    return e == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

// ---- graph plumbing ------------------------------------------------------

dit_status dit_graph_capture_begin(void* stream) {
    if (!stream) return DIT_ERR_INVALID_ARG;  // the legacy default stream cannot be captured
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaStreamCaptureStatus status;
    if (cudaStreamIsCapturing(s, &status) != cudaSuccess) return DIT_ERR_CUDA;
    if (status != cudaStreamCaptureStatusNone) return DIT_ERR_INVALID_ARG;
    return cudaStreamBeginCapture(s, cudaStreamCaptureModeRelaxed) == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

dit_status dit_graph_cond_create(void* stream, unsigned long long* cond_handle) {
    if (!stream || !cond_handle) return DIT_ERR_INVALID_ARG;
    unsigned long long id = 0;
    cudaGraph_t graph = nullptr;
    if (!capture_info(static_cast<cudaStream_t>(stream), &id, &graph, nullptr, nullptr) || !graph)
        return DIT_ERR_INVALID_ARG;
    cudaGraphConditionalHandle h = 0;
    // Default 1 (compute), re-applied at every launch of the graph.
    if (cudaGraphConditionalHandleCreate(&h, graph, 1u, cudaGraphCondAssignDefault) != cudaSuccess)
        return DIT_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lk(g_cond_mu);
        g_cond_capture[h] = id;
    }
    *cond_handle = h;
    return DIT_OK;
}

dit_status dit_graph_cond_body_begin(void* stream, unsigned long long cond_handle, void* body_stream) {
    if (!stream || !body_stream || stream == body_stream) return DIT_ERR_INVALID_ARG;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const cudaStream_t body = static_cast<cudaStream_t>(body_stream);
    cudaStreamCaptureStatus bs;
    if (cudaStreamIsCapturing(body, &bs) != cudaSuccess) return DIT_ERR_CUDA;
    if (bs != cudaStreamCaptureStatusNone) return DIT_ERR_INVALID_ARG;
    if (!cond_belongs_to(s, cond_handle)) return DIT_ERR_INVALID_ARG;
    unsigned long long id = 0;
    cudaGraph_t graph = nullptr;
    const cudaGraphNode_t* deps = nullptr;
    size_t ndeps = 0;
    if (!capture_info(s, &id, &graph, &deps, &ndeps) || !graph) return DIT_ERR_INVALID_ARG;
    cudaGraphNodeParams p = {};
    p.type = cudaGraphNodeTypeConditional;
    p.conditional.handle = cond_handle;
    p.conditional.type = cudaGraphCondTypeIf;
    p.conditional.size = 1;
    cudaGraphNode_t node = nullptr;
    if (cudaGraphAddNode(&node, graph, deps, ndeps, &p) != cudaSuccess) return DIT_ERR_CUDA;
    if (cudaStreamUpdateCaptureDependencies(s, &node, 1, cudaStreamSetCaptureDependencies) != cudaSuccess)
        return DIT_ERR_CUDA;
    cudaGraph_t body_graph = p.conditional.phGraph_out[0];
    if (cudaStreamBeginCaptureToGraph(body, body_graph, nullptr, nullptr, 0, cudaStreamCaptureModeRelaxed) !=
        cudaSuccess)
        return DIT_ERR_CUDA;
    return DIT_OK;
}

dit_status dit_graph_cond_body_end(void* body_stream) {
    if (!body_stream) return DIT_ERR_INVALID_ARG;
    const cudaStream_t body = static_cast<cudaStream_t>(body_stream);
    cudaStreamCaptureStatus bs;
    if (cudaStreamIsCapturing(body, &bs) != cudaSuccess) return DIT_ERR_CUDA;
    if (bs == cudaStreamCaptureStatusNone) return DIT_ERR_INVALID_ARG;
    cudaGraph_t g = nullptr;  // the body graph, owned by its conditional node
    return cudaStreamEndCapture(body, &g) == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

dit_status dit_graph_capture_end(void* stream, void** graph_exec) {
    if (!stream || !graph_exec) return DIT_ERR_INVALID_ARG;
    *graph_exec = nullptr;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaStreamCaptureStatus status;
    unsigned long long id = 0;
    if (cudaStreamGetCaptureInfo(s, &status, &id, nullptr, nullptr, nullptr) != cudaSuccess) return DIT_ERR_CUDA;
    if (status == cudaStreamCaptureStatusNone) return DIT_ERR_INVALID_ARG;
    {
        std::lock_guard<std::mutex> lk(g_cond_mu);
        for (auto it = g_cond_capture.begin(); it != g_cond_capture.end();)
            it = it->second == id ? g_cond_capture.erase(it) : std::next(it);
    }
    cudaGraph_t graph = nullptr;
    const cudaError_t e = cudaStreamEndCapture(s, &graph);
    if (e != cudaSuccess || !graph) {
        if (graph) cudaGraphDestroy(graph);
        return DIT_ERR_CUDA;
    }
    cudaGraphExec_t exec = nullptr;
    const cudaError_t ei = cudaGraphInstantiate(&exec, graph, 0ull);
    cudaGraphDestroy(graph);
    if (ei != cudaSuccess) return DIT_ERR_CUDA;
    *graph_exec = exec;
    return DIT_OK;
}

dit_status dit_graph_launch(void* graph_exec, void* stream) {
    if (!graph_exec) return DIT_ERR_INVALID_ARG;
    return cudaGraphLaunch(static_cast<cudaGraphExec_t>(graph_exec), static_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? DIT_OK
               : DIT_ERR_CUDA;
}

dit_status dit_graph_destroy(void* graph_exec) {
    if (!graph_exec) return DIT_ERR_INVALID_ARG;
    return cudaGraphExecDestroy(static_cast<cudaGraphExec_t>(graph_exec)) == cudaSuccess ? DIT_OK : DIT_ERR_CUDA;
}

}  // extern "C"
