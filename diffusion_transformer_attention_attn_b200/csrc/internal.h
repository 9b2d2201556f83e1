// Host-side launchers shared between the C ABI (api.cu) and the kernel files.
// Arguments are validated by the caller; these only encode and launch.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace ditk {

// Softmax attention, bf16 in/out.  tq/tk/tv: 4-D tensor maps {d, N, H, B} with
// a {64, 128, 1, 1} box and 128-byte swizzle.  o: output base; s*: element
// strides of (b, h, n).  scale_log2 = scale * log2(e).  err: device error word.
cudaError_t launch_attn_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, void* o,
                             int64_t sb, int64_t sh, int64_t sn, int B, int H, int N, int d, float scale_log2,
                             int* err, cudaStream_t stream);

// First-block-cache residual difference (see fbc_rel_l1 in dit_attn.h).
size_t fbc_workspace_bytes(int64_t n);
cudaError_t launch_fbc_rel_l1(const void* cur, const void* prev, int64_t n, int dtype, float threshold,
                              double* out_rel, int32_t* out_skip, void* workspace, cudaStream_t stream);

}  // namespace ditk
