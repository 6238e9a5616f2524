// backward.cu -- the routing and combine steps of the layer's backward pass.
//
// The pages define the forward pass only (n4n.ai page "DeepSeek-V3's
// mixture-of-experts architecture explained", "The architecture in one
// diagram"; atlas page "DeepSeek-V3.2-Exp / Mixture of experts / Shared
// expert", "All 5 steps" and the MoE forward block of its "Code" section).
// These kernels are the derivative of its last two steps, with the expert
// selection held fixed (it is piecewise constant in the inputs):
//   y[t] = sum_j w[t, j] o[t, j] + shared(x[t])
//     -> dO[t, j] = w[t, j] dy[t],  dw[t, j] = dy[t] . o[t, j];
//   w = softmax over the selected logits
//     -> dl_j = w_j (dw_j - sum_i w_i dw_i);
//   w_j = rs s_j / Z, s = sigmoid(l), Z = sum of the selected s
//     -> dl_j = rs (dw_j / Z - sum_i dw_i s_i / Z^2) s_j (1 - s_j).
// Both are bandwidth-bound: the combine backward reads dy once per token (the
// k passes hit L1) and each selected row of Y_perm once, and writes each row of
// dO_perm once; reductions run in a fixed order (deterministic results).
#include <cstdint>

#include "backward.h"
#include "common.cuh"

namespace moe {

namespace {

constexpr int kCombineBwdThreads = 256;

__device__ __forceinline__ float warp_sum(float v) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// One CTA per token; each thread owns 16-byte vectors (8 features) of the row.
__global__ void __launch_bounds__(kCombineBwdThreads)
    combine_backward_kernel(const float4* __restrict__ dy, const uint4* __restrict__ Y_perm,
                            const int32_t* __restrict__ row_of, const float* __restrict__ topk_w, int k, int d,
                            uint4* __restrict__ dO_perm, float* __restrict__ dw) {
  __shared__ float partial[kCombineBwdThreads / 32];
  const int64_t t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  grid_dependency_wait();
  const int nv = d / 8;
  for (int j = 0; j < k; ++j) {
    const int32_t r = row_of[t * k + j];
    const float w = topk_w[t * k + j];
    float acc = 0.0f;
    if (r >= 0) {
      for (int v = threadIdx.x; v < nv; v += kCombineBwdThreads) {
        const float4 a = dy[(t * d) / 4 + 2 * v];
        const float4 b = dy[(t * d) / 4 + 2 * v + 1];
        const uint4 q = Y_perm[(int64_t)r * nv + v];
        acc = fmaf(a.x, ptx::bf16_lo(q.x), acc);
        acc = fmaf(a.y, ptx::bf16_hi(q.x), acc);
        acc = fmaf(a.z, ptx::bf16_lo(q.y), acc);
        acc = fmaf(a.w, ptx::bf16_hi(q.y), acc);
        acc = fmaf(b.x, ptx::bf16_lo(q.z), acc);
        acc = fmaf(b.y, ptx::bf16_hi(q.z), acc);
        acc = fmaf(b.z, ptx::bf16_lo(q.w), acc);
        acc = fmaf(b.w, ptx::bf16_hi(q.w), acc);
        dO_perm[(int64_t)r * nv + v] =
            make_uint4(ptx::pack_bf16x2(w * a.x, w * a.y), ptx::pack_bf16x2(w * a.z, w * a.w),
                       ptx::pack_bf16x2(w * b.x, w * b.y), ptx::pack_bf16x2(w * b.z, w * b.w));
      }
    }
    acc = warp_sum(acc);
    if (lane == 0) partial[warp] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
      float s = 0.0f;
      for (int i = 0; i < kCombineBwdThreads / 32; ++i) s += partial[i];
      dw[t * k + j] = r >= 0 ? s : 0.0f;
    }
    __syncthreads();
  }
}

// One warp per token: lane j < k holds slot j.  Every lane then writes its
// share of the token's dlogits row (the selected experts' values, zeros
// elsewhere), looking the slots up by shuffles.
__global__ void __launch_bounds__(256)
    router_backward_kernel(const float* __restrict__ logits, const int32_t* __restrict__ topk_idx,
                           const float* __restrict__ topk_w, const float* __restrict__ dw, int64_t T, int E, int k,
                           int route, float route_scale, float* __restrict__ dlogits) {
  grid_dependency_wait();
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  const bool mine = lane < k;
  int32_t e = mine ? topk_idx[t * k + lane] : -1;
  if (e < 0 || e >= E) e = -1;  // out-of-range index: no gradient
  const float w = mine ? topk_w[t * k + lane] : 0.0f;
  const float g = mine ? dw[t * k + lane] : 0.0f;
  const float l = e >= 0 ? logits[t * E + e] : 0.0f;
  float dl;
  if (route == 0) {
    const float wg = warp_sum(mine ? w * g : 0.0f);
    dl = w * (g - wg);
  } else {
    const float s = e >= 0 ? 1.0f / (1.0f + expf(-l)) : 0.0f;
    const float Z = warp_sum(s);
    const float gs = warp_sum(g * s);
    const float ds = route_scale * (g / Z - gs / (Z * Z));
    dl = ds * s * (1.0f - s);
  }
  for (int c = lane; c < E; c += 32) {
    float v = 0.0f;
    for (int j = 0; j < k; ++j) {
      const int32_t ej = __shfl_sync(0xffffffffu, e, j);
      const float dj = __shfl_sync(0xffffffffu, dl, j);
      if (ej == c) v = dj;
    }
    dlogits[t * E + c] = v;
  }
}

}  // namespace

cudaError_t launch_combine_backward(const float* dy, const void* Y_perm, const int32_t* row_of, const float* topk_w,
                                    int64_t T, int k, int d, void* dO_perm, float* dw, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const cudaError_t err = launch_chained(combine_backward_kernel, dim3((unsigned)T), dim3(kCombineBwdThreads), 0,
                                         stream, reinterpret_cast<const float4*>(dy),
                                         static_cast<const uint4*>(Y_perm), row_of, topk_w, k, d,
                                         static_cast<uint4*>(dO_perm), dw);
  return err != cudaSuccess ? err : cudaGetLastError();
}

cudaError_t launch_router_backward(const float* logits, const int32_t* topk_idx, const float* topk_w,
                                   const float* dw, int64_t T, int E, int k, int route, float route_scale,
                                   float* dlogits, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const unsigned blocks = (unsigned)((T + 7) / 8);
  const cudaError_t err = launch_chained(router_backward_kernel, dim3(blocks), dim3(256), 0, stream, logits,
                                         topk_idx, topk_w, dw, T, E, k, route, route_scale, dlogits);
  return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace moe
