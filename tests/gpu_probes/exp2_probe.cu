// Test probe: evaluates the library's FMA-pipe 2^x (ditk::exp2_poly2 in
// sm100_ptx.cuh, the exponential the attention kernels run for a share of
// their softmax elements), or its quadratic form exp2_poly2q, on a caller-given
// grid of arguments, so a test can hold each to its stated error bound.  Built
// and loaded only by the tests.
#include <cuda_runtime.h>

#include "sm100_ptx.cuh"

namespace {

// Thread i evaluates the pair (x[2i], x[2i+1]); n_pairs pairs in all.
// quadratic != 0 selects exp2_poly2q (the e4m3-P form), else exp2_poly2.
__global__ void exp2_poly_probe_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n_pairs,
                                       int quadratic) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= n_pairs) return;
    const float2 in = make_float2(x[2 * i], x[2 * i + 1]);
    const float2 r = quadratic ? ditk::exp2_poly2q(in) : ditk::exp2_poly2(in);
    y[2 * i] = r.x;
    y[2 * i + 1] = r.y;
}

}  // namespace

// x, y: device float arrays of 2·n_pairs elements.  Returns a cudaError_t.
extern "C" int exp2_poly_probe(const float* x, float* y, int64_t n_pairs, int quadratic, void* stream) {
    if (n_pairs <= 0) return 0;
    const int threads = 256;
    const int64_t blocks = (n_pairs + threads - 1) / threads;
    if (blocks > 0x7FFFFFFF) return static_cast<int>(cudaErrorInvalidValue);
    exp2_poly_probe_kernel<<<static_cast<unsigned>(blocks), threads, 0, static_cast<cudaStream_t>(stream)>>>(x, y,
                                                                                                          n_pairs, quadratic);
    return static_cast<int>(cudaGetLastError());
}
