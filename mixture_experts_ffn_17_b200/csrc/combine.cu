// combine.cu -- weighted sum of each token's expert outputs back in token order.
//
// The atlas page's MoE forward ("Code" section, MoE forward block) accumulates
// y[idx] += expert(x[idx]) * weights[idx, top] into an fp32 buffer, then adds
// the shared expert.  Here every token gathers its k routed rows (bf16, in
// permuted order, located through row_of) and its shared-expert row (fp32),
// and sums them in fp32 with no atomics, so the result is deterministic:
//   y[t] = Y_shared[t] + sum_j w[t, j] * Y_perm[row_of[t*k + j]].
// One CTA per token (per token and slice of the features when there are
// few tokens, so that small batches still spread over the SMs); each thread
// owns 8 consecutive features (one 16-byte vector of each routed row), so
// every row read is coalesced.
#include <algorithm>
#include <cstdint>

#include "common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

template <bool OUT_BF16>
__global__ void __launch_bounds__(128)
    combine_kernel(const uint4* __restrict__ Y_perm, const float4* __restrict__ Y_shared,
                   const int32_t* __restrict__ row_of, const float* __restrict__ topk_w, int k, int d,
                   void* __restrict__ y, const int32_t* __restrict__ offsets, int e_lo, int e_hi) {
  __shared__ int32_t rows[32];
  __shared__ float ws[32];
  const int64_t t = blockIdx.x;
  grid_dependency_wait();
  if (threadIdx.x < k) {
    int32_t r = row_of[t * k + threadIdx.x];
    // a shard adds only the rows of its own experts
    if (offsets && (r < offsets[e_lo] || r >= offsets[e_hi])) r = -1;
    rows[threadIdx.x] = r;
    ws[threadIdx.x] = topk_w ? topk_w[t * k + threadIdx.x] : 1.0f;  // no weights: a plain sum
  }
  __syncthreads();
  const int nv = d / 8;
  // this CTA's slice of the row's 16-byte vectors
  const int per = (nv + gridDim.y - 1) / gridDim.y;
  const int v_end = min(nv, (int)(blockIdx.y + 1) * per);
  for (int v = blockIdx.y * per + threadIdx.x; v < v_end; v += blockDim.x) {
    float acc[8];
    if (Y_shared) {
      const float4 a = Y_shared[(t * d) / 4 + 2 * v];
      const float4 b = Y_shared[(t * d) / 4 + 2 * v + 1];
      acc[0] = a.x; acc[1] = a.y; acc[2] = a.z; acc[3] = a.w;
      acc[4] = b.x; acc[5] = b.y; acc[6] = b.z; acc[7] = b.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    }
    for (int j = 0; j < k; ++j) {
      const int32_t r = rows[j];
      if (r < 0) continue;
      const uint4 q = Y_perm[(int64_t)r * nv + v];
      const float w = ws[j];
      acc[0] = fmaf(w, ptx::bf16_lo(q.x), acc[0]);
      acc[1] = fmaf(w, ptx::bf16_hi(q.x), acc[1]);
      acc[2] = fmaf(w, ptx::bf16_lo(q.y), acc[2]);
      acc[3] = fmaf(w, ptx::bf16_hi(q.y), acc[3]);
      acc[4] = fmaf(w, ptx::bf16_lo(q.z), acc[4]);
      acc[5] = fmaf(w, ptx::bf16_hi(q.z), acc[5]);
      acc[6] = fmaf(w, ptx::bf16_lo(q.w), acc[6]);
      acc[7] = fmaf(w, ptx::bf16_hi(q.w), acc[7]);
    }
    if (OUT_BF16) {
      uint4* out = static_cast<uint4*>(y);
      out[t * nv + v] = make_uint4(ptx::pack_bf16x2(acc[0], acc[1]), ptx::pack_bf16x2(acc[2], acc[3]),
                                   ptx::pack_bf16x2(acc[4], acc[5]), ptx::pack_bf16x2(acc[6], acc[7]));
    } else {
      float4* out = static_cast<float4*>(y);
      out[(t * d) / 4 + 2 * v] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      out[(t * d) / 4 + 2 * v + 1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
  }
}

}  // namespace

cudaError_t launch_combine(const void* Y_perm, const float* Y_shared, const int32_t* row_of, const float* topk_w,
                           int64_t T, int k, int d, void* y, bool y_bf16, cudaStream_t stream,
                           const int32_t* offsets, const Shard* shard) {
  if (T == 0) return cudaSuccess;
  const uint4* yp = static_cast<const uint4*>(Y_perm);
  const float4* ys = reinterpret_cast<const float4*>(Y_shared);
  const int e_lo = shard ? shard->e_lo : 0, e_hi = shard ? shard->e_hi : 0;
  if (!shard) offsets = nullptr;
  // feature slices per token: enough CTAs for about four per SM
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = ((int64_t)4 * sms + T - 1) / T;
  const unsigned slices = (unsigned)std::max<int64_t>(1, std::min<int64_t>(want, std::max(1, d / 8 / 128)));
  const dim3 grid((unsigned)T, slices);
  const cudaError_t err =
      y_bf16 ? launch_chained(combine_kernel<true>, grid, dim3(128), 0, stream, yp, ys, row_of, topk_w, k, d, y,
                              offsets, e_lo, e_hi)
             : launch_chained(combine_kernel<false>, grid, dim3(128), 0, stream, yp, ys, row_of, topk_w, k, d, y,
                              offsets, e_lo, e_hi);
  return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace moe
