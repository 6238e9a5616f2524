// backward.h -- launchers of the backward-pass kernels (backward.cu).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace moe {

// Adjoint of the combine: for every (t, j) with r = row_of[t*k + j] >= 0,
// dO_perm[r] = bf16(topk_w[t, j] * dy[t]) and dw[t, j] = dy[t] . Y_perm[r]
// (fp32; 0 where r < 0).  dy fp32 [T, d]; Y_perm, dO_perm bf16 [T*k, d].
cudaError_t launch_combine_backward(const float* dy, const void* Y_perm, const int32_t* row_of, const float* topk_w,
                                    int64_t T, int k, int d, void* dO_perm, float* dw, cudaStream_t stream);

// Gradient of the k selected logits of every token from dw, the selection held
// fixed; dlogits [T, E] fp32, zero outside the selection.  route 0: softmax
// over the selected logits; route 1: route_scale * s / sum(s), s = sigmoid.
cudaError_t launch_router_backward(const float* logits, const int32_t* topk_idx, const float* topk_w,
                                   const float* dw, int64_t T, int E, int k, int route, float route_scale,
                                   float* dlogits, cudaStream_t stream);

}  // namespace moe
