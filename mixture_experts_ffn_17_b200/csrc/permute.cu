// permute.cu -- token-to-expert dispatch without a host round trip.
//
// The atlas page's MoE forward ("DeepSeek-V3.2-Exp / Mixture of experts",
// "Code" section, MoE forward block) counts assignments with bincount(indices,
// minlength=E), copies the counts to the host and, for each expert, gathers
// the tokens that chose it with torch.where(indices == e), i.e. in ascending
// (token, slot) order.  Here the same order is built on the device as a stable
// counting sort in three launches:
//   1. hist    : per block of 256 tokens, a shared-memory histogram over E;
//   2. scan    : one CTA; per expert the running sum over blocks (each block's
//                base), counts[e], and the exclusive prefix sum offsets[E+1];
//   3. scatter : each warp ranks its 32 tokens' k entries per expert with
//                __match_any_sync, warps are ordered by a per-warp histogram,
//                and entry (t, j) lands at offsets-based position r:
//                perm_token[r] = t, row_of[t*k + j] = r.
// A separate gather copies x rows into permuted order (x_perm), and the tile
// builder lists the 256-row tiles of every expert segment (plus the shared
// expert's tiles over all T tokens) for the grouped GEMMs.
#include <algorithm>
#include <cstdint>

#include "common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kPermTokens = 256;  // tokens per block in hist / scatter
constexpr int kPermThreads = 256;

__global__ void __launch_bounds__(kPermThreads)
    hist_kernel(const int32_t* __restrict__ idx, int T, int k, int E, int32_t* __restrict__ hist,
                uint32_t* __restrict__ status) {
  extern __shared__ int32_t h[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
  __syncthreads();
  grid_dependency_wait();
  const int64_t begin = (int64_t)blockIdx.x * kPermTokens * k;
  const int64_t end = ::min((long long)T * k, (long long)(begin + (int64_t)kPermTokens * k));
  for (int64_t i = begin + threadIdx.x; i < end; i += blockDim.x) {
    const int e = idx[i];
    if (e < 0 || e >= E) {
      atomicOr(status, kStatusBounds);
      continue;
    }
    atomicAdd(&h[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(size_t)blockIdx.x * E + e] = h[e];
}

// One CTA of >= E threads (a multiple of 32, <= 1024).
__global__ void scan_kernel(const int32_t* __restrict__ hist, int nb, int E, int32_t* __restrict__ base,
                            int32_t* __restrict__ counts, int32_t* __restrict__ offsets) {
  __shared__ int32_t warp_sums[32];
  const int e = threadIdx.x;
  int32_t run = 0;
  grid_dependency_wait();
  if (e < E)
    for (int b = 0; b < nb; ++b) {
      const int32_t v = hist[(size_t)b * E + e];
      base[(size_t)b * E + e] = run;
      run += v;
    }
  const int32_t c = (e < E) ? run : 0;
  // block exclusive scan of c
  const int lane = e & 31, warp = e >> 5;
  int32_t incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int32_t v = (lane < nw) ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (lane < nw) warp_sums[lane] = v - ((lane < nw) ? warp_sums[lane] : 0);  // exclusive per warp
  }
  __syncthreads();
  const int32_t excl = warp_sums[warp] + incl - c;
  if (e < E) {
    counts[e] = c;
    offsets[e] = excl;
    if (e == E - 1) offsets[E] = excl + c;
    for (int b = 0; b < nb; ++b) base[(size_t)b * E + e] += excl;
  }
}

// Stable scatter.  Block = 8 warps x 32 tokens; a warp walks its tokens' k*32
// entries in (token, slot) order, 32 entries per step.
__global__ void __launch_bounds__(kPermThreads)
    scatter_kernel(const int32_t* __restrict__ idx, int T, int k, int E, const int32_t* __restrict__ base,
                   int32_t* __restrict__ perm_token, int32_t* __restrict__ row_of) {
  extern __shared__ int32_t wh[];  // [8][E] per-warp counts, then exclusive per-warp bases
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = kPermThreads / 32;
  for (int i = threadIdx.x; i < nwarps * E; i += blockDim.x) wh[i] = 0;
  __syncthreads();
  grid_dependency_wait();

  const int64_t tok0 = (int64_t)blockIdx.x * kPermTokens + warp * 32;
  const int64_t ent0 = tok0 * k;
  const int64_t ent_end = ::min((long long)T * k, (long long)(ent0 + 32LL * k));
  int32_t* my = wh + warp * E;
  // pass 1: per-warp counts (entries in order, so ranks within the warp are
  // the running count before each entry)
  for (int64_t i0 = ent0; i0 < ent_end; i0 += 32) {
    const int64_t i = i0 + lane;
    const bool valid = i < ent_end;
    const int e = valid ? idx[i] : -1;
    const bool inrange = valid && e >= 0 && e < E;
    const uint32_t peers = __match_any_sync(0xffffffffu, inrange ? e : -1);
    if (inrange) {
      const int leader = __ffs(peers) - 1;
      if (lane == leader) my[e] += __popc(peers);
    }
    __syncwarp();
  }
  __syncthreads();
  // exclusive scan over warps per expert
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int32_t run = 0;
    for (int w = 0; w < nwarps; ++w) {
      const int32_t v = wh[w * E + e];
      wh[w * E + e] = run;
      run += v;
    }
  }
  __syncthreads();
  // pass 2: positions
  const int32_t* bb = base + (size_t)blockIdx.x * E;
  for (int64_t i0 = ent0; i0 < ent_end; i0 += 32) {
    const int64_t i = i0 + lane;
    const bool valid = i < ent_end;
    const int e = valid ? idx[i] : -1;
    const bool inrange = valid && e >= 0 && e < E;
    const uint32_t peers = __match_any_sync(0xffffffffu, inrange ? e : -1);
    if (inrange) {
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int32_t r = bb[e] + my[e] + rank;
      perm_token[r] = (int32_t)(i / k);
      row_of[i] = r;
    } else if (valid) {
      row_of[i] = -1;
    }
    __syncwarp();
    if (inrange) {
      const int leader = __ffs(peers) - 1;
      if (lane == leader) my[e] += __popc(peers);
    }
    __syncwarp();
  }
}

// x_perm[r, :] = x[perm_token[r], :]; rows of d bf16 (d % 8 == 0), 16-byte
// vectors, one CTA per row at a time.  Each thread issues kGatherUnroll loads
// before its stores, so an SM keeps enough bytes in flight to cover HBM
// latency; the next row's token index is fetched while this row is copied.
constexpr int kGatherUnroll = 4;

__global__ void __launch_bounds__(256)
    gather_rows_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ perm_token, int64_t rows,
                       int vec_per_row, uint4* __restrict__ x_perm, const int32_t* __restrict__ offsets, int e_lo,
                       int e_hi) {
  grid_dependency_wait();
  // rows [r_lo, r_hi) of the permuted order: all of them, or one expert slice
  const int64_t r_lo = offsets ? offsets[e_lo] : 0;
  if (offsets) rows = offsets[e_hi];
  int64_t r = r_lo + blockIdx.x;
  if (r >= rows) return;
  int32_t t = perm_token[r];
  for (; r < rows; r += gridDim.x) {
    const int64_t rn = r + gridDim.x;
    const int32_t tn = rn < rows ? perm_token[rn] : 0;
    const uint4* src = x + (size_t)t * vec_per_row;
    uint4* dst = x_perm + (size_t)r * vec_per_row;
    for (int v0 = threadIdx.x; v0 < vec_per_row; v0 += kGatherUnroll * blockDim.x) {
      uint4 buf[kGatherUnroll];
#pragma unroll
      for (int u = 0; u < kGatherUnroll; ++u) {
        const int v = v0 + u * blockDim.x;
        if (v < vec_per_row) buf[u] = __ldg(src + v);
      }
#pragma unroll
      for (int u = 0; u < kGatherUnroll; ++u) {
        const int v = v0 + u * blockDim.x;
        if (v < vec_per_row) dst[v] = buf[u];
      }
    }
    t = tn;
  }
}

// MOE_PAIR_LAST_ALL=1: a segment with full 256-row tiles also puts its last
// tile, however short, on the pair list (right after its full tiles, while
// its weights are still in L2) instead of the one-CTA list.
#ifndef MOE_PAIR_LAST_ALL
#define MOE_PAIR_LAST_ALL 0
#endif

// The same copy in token order: x_perm[row_of[t*k + j], :] = x[t, :] for the
// rows of [offsets[e_lo], offsets[e_hi]) (every row when e_lo = 0, e_hi = E;
// an entry with an out-of-range expert has row_of = -1 and is skipped).  Each
// x row is read once and written k times, where the permuted-order gather
// reads it k times far apart (x no longer in L2 by then).  A work item is
// one token's row, or a column part of it when there are few tokens.
__global__ void __launch_bounds__(256)
    scatter_rows_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ row_of, int T, int k,
                        int vec_per_row, int parts, uint4* __restrict__ x_perm, const int32_t* __restrict__ offsets,
                        int e_lo, int e_hi) {
  grid_dependency_wait();
  const int64_t r_lo = offsets[e_lo], r_hi = offsets[e_hi];
  const int vpp = (vec_per_row + parts - 1) / parts;
  const int64_t items = (int64_t)T * parts;
  for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
    const int t = (int)(it / parts);
    const int v_begin = (int)(it - (int64_t)t * parts) * vpp;
    const int v_end = min(vec_per_row, v_begin + vpp);
    const uint4* src = x + (size_t)t * vec_per_row;
    const int32_t* rows = row_of + (size_t)t * k;
    for (int v0 = v_begin + threadIdx.x; v0 < v_end; v0 += kGatherUnroll * blockDim.x) {
      uint4 buf[kGatherUnroll];
#pragma unroll
      for (int u = 0; u < kGatherUnroll; ++u) {
        const int v = v0 + u * blockDim.x;
        if (v < v_end) buf[u] = __ldg(src + v);
      }
      for (int j = 0; j < k; ++j) {
        const int64_t r = __ldg(rows + j);
        if (r < r_lo || r >= r_hi) continue;
        uint4* dst = x_perm + (size_t)r * vec_per_row;
#pragma unroll
        for (int u = 0; u < kGatherUnroll; ++u) {
          const int v = v0 + u * blockDim.x;
          if (v < v_end) dst[v] = buf[u];
        }
      }
    }
  }
}

// Tile lists for the grouped GEMMs: one int4 {group, row_start, rows,
// row tiles of the group's segment} per
// 256-row tile of each expert segment of [e_lo, e_hi) (group e, rows in
// permuted order), then the shared expert's tiles (group E, rows in token
// order).  Without a pair list every tile goes to `tiles` (ntiles[0] = all,
// ntiles[1] = routed).  With one (tiles_pair != nullptr) the full 256-row
// tiles, and a segment's last tile when it holds more than kPairMinRows rows,
// go to `tiles_pair` (ntiles[2] = all, ntiles[3] = routed); the other partial
// tiles to `tiles`.
__global__ void build_tiles_kernel(const int32_t* __restrict__ offsets, int E, int e_lo, int e_hi, int T,
                                   int with_shared, int4* __restrict__ tiles, int4* __restrict__ tiles_pair,
                                   int32_t* __restrict__ ntiles, int* __restrict__ sched_counters) {
  __shared__ long long warp_sums[32];
  __shared__ long long total;
  const int e = threadIdx.x;
  const int lane = e & 31, warp = e >> 5;
  const bool split = tiles_pair != nullptr;
  int32_t start = 0, cnt = 0, mt_full = 0, mt_part = 0;
  grid_dependency_wait();
  if (e >= e_lo && e < e_hi) {
    start = offsets[e];
    cnt = offsets[e + 1] - start;
    const int rem = cnt % kTileRows;
    // a segment's last tile goes on the pair list when it is nearly full, or
    // (MOE_PAIR_LAST_ALL) whenever the segment also has full tiles there
    const bool last_pair = rem > kPairMinRows || (MOE_PAIR_LAST_ALL && rem > 0 && cnt >= kTileRows);
    mt_full = split ? cnt / kTileRows + last_pair : 0;
    mt_part = split ? (rem != 0 && !last_pair) : (cnt + kTileRows - 1) / kTileRows;
  }
  // one scan of both counts: full tiles in the high word, partial in the low
  const long long mine_t = ((long long)mt_full << 32) | (unsigned)mt_part;
  long long incl = mine_t;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    const long long mine = (lane < nw) ? warp_sums[lane] : 0;
    long long v = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (lane < nw) warp_sums[lane] = v - mine;
    if (lane == nw - 1) total = v;
  }
  __syncthreads();
  const long long first = warp_sums[warp] + incl - mine_t;
  const int32_t first_full = (int32_t)(first >> 32), first_part = (int32_t)(first & 0xffffffffll);
  for (int m = 0; m < mt_full; ++m)
    tiles_pair[first_full + m] =
        make_int4(e, start + m * kTileRows, min(kTileRows, cnt - m * kTileRows), mt_full + mt_part);
  for (int m = 0; m < mt_part; ++m) {
    const int32_t r0 = (mt_full + m) * kTileRows;
    tiles[first_part + m] = make_int4(e, start + r0, min(kTileRows, cnt - r0), mt_full + mt_part);
  }
  const int32_t routed_full = (int32_t)(total >> 32), routed_part = (int32_t)(total & 0xffffffffll);
  const int t_rem = T % kTileRows;
  const int32_t shared_full = with_shared && split ? T / kTileRows + (t_rem > kPairMinRows) : 0;
  const int32_t shared_part =
      with_shared ? (split ? (t_rem != 0 && t_rem <= kPairMinRows) : (T + kTileRows - 1) / kTileRows) : 0;
  for (int m = threadIdx.x; m < shared_full; m += blockDim.x)
    tiles_pair[routed_full + m] = make_int4(E, m * kTileRows, min(kTileRows, T - m * kTileRows), 0);  // shared
  for (int m = threadIdx.x; m < shared_part; m += blockDim.x) {
    const int32_t r0 = (shared_full + m) * kTileRows;
    tiles[routed_part + m] = make_int4(E, r0, min(kTileRows, T - r0), 0);
  }
  if (threadIdx.x == 0) {
    ntiles[0] = routed_part + shared_part;
    ntiles[1] = routed_part;
    if (split) {
      ntiles[2] = routed_full + shared_full;
      ntiles[3] = routed_full;
    }
  }
  if (threadIdx.x < kNumSchedCounters) sched_counters[threadIdx.x] = 0;
}

}  // namespace

int permute_blocks(int64_t T) { return (int)((T + kPermTokens - 1) / kPermTokens); }

cudaError_t launch_permute(const int32_t* idx, int64_t T, int k, int E, int32_t* hist, int32_t* base,
                           int32_t* counts, int32_t* offsets, int32_t* perm_token, int32_t* row_of,
                           uint32_t* status, cudaStream_t stream) {
  const int nb = permute_blocks(T);
  cudaError_t err = launch_chained(hist_kernel, dim3(nb), dim3(kPermThreads), E * sizeof(int32_t), stream, idx,
                                   (int)T, k, E, hist, status);
  if (err != cudaSuccess) return err;
  const int st = ((E + 31) / 32) * 32;
  err = launch_chained(scan_kernel, dim3(1), dim3(st), 0, stream, hist, nb, E, base, counts, offsets);
  if (err != cudaSuccess) return err;
  const size_t sm = (size_t)(kPermThreads / 32) * E * sizeof(int32_t);
  if (sm > 48 * 1024) {
    err = cudaFuncSetAttribute(scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (err != cudaSuccess) return err;
  }
  err = launch_chained(scatter_kernel, dim3(nb), dim3(kPermThreads), sm, stream, idx, (int)T, k, E, base, perm_token,
                       row_of);
  return err != cudaSuccess ? err : cudaGetLastError();
}

cudaError_t launch_gather_rows(const void* x, const int32_t* perm_token, int64_t rows, int d, void* x_perm,
                               int num_sms, cudaStream_t stream, const int32_t* offsets, int e_lo, int e_hi) {
  if (rows == 0) return cudaSuccess;
  const int64_t g = std::min<int64_t>(rows, (int64_t)num_sms * 16);
  const cudaError_t err = launch_chained(gather_rows_kernel, dim3((unsigned)g), dim3(256), 0, stream,
                                         static_cast<const uint4*>(x), perm_token, rows, d / 8,
                                         static_cast<uint4*>(x_perm), offsets, e_lo, e_hi);
  return err != cudaSuccess ? err : cudaGetLastError();
}

cudaError_t launch_scatter_rows(const void* x, const int32_t* row_of, int64_t T, int k, int d, void* x_perm,
                                int num_sms, cudaStream_t stream, const int32_t* offsets, int e_lo, int e_hi) {
  if (T == 0) return cudaSuccess;
  const int vec = d / 8;
  // enough work items to cover the device: split rows into column parts when
  // tokens are few (at least 32 vectors per part)
  const int64_t want = (int64_t)num_sms * 4;
  int parts = (int)std::min<int64_t>((want + T - 1) / T, std::max(1, vec / 32));
  if (parts < 1) parts = 1;
  const int64_t items = T * parts;
  const int64_t g = std::min<int64_t>(items, (int64_t)num_sms * 16);
  const cudaError_t err = launch_chained(scatter_rows_kernel, dim3((unsigned)g), dim3(256), 0, stream,
                                         static_cast<const uint4*>(x), row_of, (int)T, k, vec, parts,
                                         static_cast<uint4*>(x_perm), offsets, e_lo, e_hi);
  return err != cudaSuccess ? err : cudaGetLastError();
}

cudaError_t launch_build_tiles(const int32_t* offsets, int E, int64_t T, const Shard& shard, bool with_shared,
                               int4* tiles, int32_t* ntiles, int* sched_counters, cudaStream_t stream,
                               int4* tiles_pair) {
  const int threads = ((E + 31) / 32) * 32;
  const cudaError_t err = launch_chained(build_tiles_kernel, dim3(1), dim3(threads < 32 ? 32 : threads), 0, stream,
                                         offsets, E, shard.e_lo, shard.e_hi, (int)T, with_shared ? 1 : 0, tiles,
                                         tiles_pair, ntiles, sched_counters);
  return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace moe
