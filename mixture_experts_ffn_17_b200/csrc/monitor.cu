// monitor.cu -- expert-utilisation monitor on the device.
//
// The n4n page's "Where the architecture struggles" section monitors router
// health with bincount(indices) normalised to fractions and an alert when an
// expert carries more than 2x or less than 0.1x the mean load.  Given the
// per-expert counts the dispatch already produces, one CTA computes
//   util[e] = counts[e] / total
//   flags[e] = +1 if counts[e] * E > 2 * total   (more than twice the mean)
//              -1 if 10 * counts[e] * E < total  (less than a tenth of the mean)
//               0 otherwise
// with exact integer tests.
#include <cstdint>

#include "common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

__global__ void expert_utilisation_kernel(const int32_t* __restrict__ counts, int E, float* __restrict__ util,
                                          int32_t* __restrict__ flags) {
  __shared__ long long partial[32];
  long long mine = 0;
  grid_dependency_wait();
  for (int e = threadIdx.x; e < E; e += blockDim.x) mine += counts[e];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, o);
  if ((threadIdx.x & 31) == 0) partial[threadIdx.x >> 5] = mine;
  __syncthreads();
  long long total = 0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) total += partial[w];
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const long long c = counts[e];
    if (util) util[e] = total > 0 ? (float)((double)c / (double)total) : 0.0f;
    if (flags) flags[e] = (c * E > 2 * total) ? 1 : ((10 * c * E < total) ? -1 : 0);
  }
}

}  // namespace

cudaError_t launch_expert_utilisation(const int32_t* counts, int E, float* util, int32_t* flags,
                                      cudaStream_t stream) {
  const cudaError_t err =
      launch_chained(expert_utilisation_kernel, dim3(1), dim3(256), 0, stream, counts, E, util, flags);
  return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace moe
