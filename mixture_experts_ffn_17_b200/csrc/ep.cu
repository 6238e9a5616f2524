// ep.cu -- the regrouping step of the all-to-all flavour of expert
// parallelism.
//
// With the experts split over ranks, each rank sends the rows routed to
// another rank's experts there (n4n.ai page, "Why 256 experts with top-8
// routing?": the tokens' hidden states travel to the devices that hold their
// experts; "Training infrastructure that made this possible": that
// all-to-all is overlapped with computation).  A rank receives, from every
// source rank in turn, that source's rows for each of its E_local experts in
// expert order (the source's own expert-major permutation), so the received
// buffer is source-major.  The grouped GEMMs want each expert's rows
// contiguous; this kernel computes the expert-major order of the received
// rows (stable: source, then the source's order) and the maps between the two
// orders:
//   offsets_local[e]      first expert-major row of local expert e (E_local+1)
//   to_expert_major[p]    the received row at expert-major position p
//   to_source_major[r]    the expert-major position of received row r
// so that gathers through them move rows either way.
#include <algorithm>
#include <cstdint>

#include "common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kEpThreads = 1024;

// exclusive scan of one value per thread over the block (blockDim.x = 1024)
__device__ int32_t block_exclusive_scan(int32_t v, int32_t* warp_tot, int32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int32_t t = warp_tot[lane];
    int32_t ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += y;
    }
    warp_tot[lane] = ti - t;  // exclusive prefix of the warp totals
    if (lane == 31) *total = ti;
  }
  __syncthreads();
  const int32_t r = warp_tot[warp] + incl - v;
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kEpThreads)
    ep_regroup_kernel(const int32_t* __restrict__ cnt, int n_src, int E_local, int32_t* __restrict__ offsets_local,
                      int32_t* __restrict__ to_em, int32_t* __restrict__ to_sm) {
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t total;
  __shared__ int32_t src_start[kEpThreads];  // source-major start of segment (s, e) at s * E_local + e
  __shared__ int32_t em_start[kEpThreads];   // expert-major start of the same segment
  grid_dependency_wait();
  const int i = threadIdx.x;
  const int nseg = n_src * E_local;
  // source-major segment starts: a scan over the flat [n_src, E_local] counts
  const int32_t c = i < nseg ? max(cnt[i], 0) : 0;
  const int32_t ss = block_exclusive_scan(c, warp_tot, &total);
  if (i < nseg) src_start[i] = ss;
  // expert totals and their scan
  int32_t te = 0;
  if (i < E_local)
    for (int s = 0; s < n_src; ++s) te += max(cnt[s * E_local + i], 0);
  const int32_t es = block_exclusive_scan(te, warp_tot, &total);
  if (i < E_local) {
    offsets_local[i] = es;
    int32_t run = es;
    for (int s = 0; s < n_src; ++s) {
      em_start[s * E_local + i] = run;
      run += max(cnt[s * E_local + i], 0);
    }
  }
  if (i == 0) offsets_local[E_local] = total;
  __syncthreads();
  // every row of every segment: one warp per segment
  const int warp = i >> 5, lane = i & 31;
  for (int g = warp; g < nseg; g += kEpThreads / 32) {
    const int32_t n = max(cnt[g], 0), a = src_start[g], b = em_start[g];
    for (int j = lane; j < n; j += 32) {
      to_sm[a + j] = b + j;
      to_em[b + j] = a + j;
    }
  }
}

}  // namespace

cudaError_t launch_ep_regroup(const int32_t* recv_counts, int n_src, int E_local, int32_t* offsets_local,
                              int32_t* to_expert_major, int32_t* to_source_major, cudaStream_t stream) {
  const cudaError_t err = launch_chained(ep_regroup_kernel, dim3(1), dim3(kEpThreads), 0, stream, recv_counts, n_src,
                                         E_local, offsets_local, to_expert_major, to_source_major);
  return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace moe
