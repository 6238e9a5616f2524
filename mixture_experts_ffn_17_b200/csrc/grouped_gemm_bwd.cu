// grouped_gemm_bwd.cu -- the expert contractions of the layer's backward pass
// on the 5th-generation tensor cores.
//
// The pages define the forward pass only (atlas page "DeepSeek-V3.2-Exp /
// Mixture of experts / Shared expert", "All 5 steps": g = x W1, u = x W3,
// h = silu(g) u, o = h W2; n4n.ai page, "The architecture in one diagram").
// These are the derivative of those steps for every expert's rows, the
// expert selection held fixed (it is piecewise constant in the inputs):
//   dH = dO W2^T,  dG = dH u silu'(g),  dU = dH silu(g),
//   dX = dG W1^T + dU W3^T                                  (dgrad_kernel)
//   dW1 = X^T dG,  dW3 = X^T dU,  dW2 = H^T dO,  dWg = dl^T x (wgrad_kernel)
// with silu'(g) = sigmoid(g) (1 + g (1 - sigmoid(g))).
//
// dgrad_kernel: persistent, one CTA per SM, over the forward's tile list (256
// rows of an expert segment per tile, one or two 128-row halves; the shared
// expert is group E over all T tokens).  Warp 0 is the TMA producer, warp 1's
// lane 0 issues tcgen05.mma (M=128, N=256, K=16; fp32 accumulators in two
// 256-column TMEM slots), warps 2-9 drain the accumulator (drain-first, as in
// the forward kernels) and run the epilogue.  A (the row operand) is K-major
// as in the forward; B is the weight read K-major, [256 N rows x 64 K] boxes
// straight from the weights' row-major layout (W2 [I, d] for dH, W1 / W3
// [d, I] for dX): no transposed copy.  K is a list of parts, each its own
// (A, B) pair: dX's routed tiles contract [dG | dU] with [W1 ; W3], and the
// shared expert's tiles add a third part, dl Wg (the router's contribution to
// the input gradient), so dX_shared + dl Wg come out of one accumulator.
//
// wgrad_kernel: the weight gradients contract over each expert's rows, a
// count known only on the device.  Tile = (group, 128 output rows, 256 output
// columns); K runs over the group's rows in steps of 64, both operands
// MN-major ([64 rows x 64 features] boxes of the row-major activations).  The
// last K step of a group usually holds rows of the next expert: only its
// 16-row MMA slices with rows of the group are issued, and warp 1 zeroes the
// rest of the last one in the A operand before the MMA reads it.  A
// group without rows writes zeros.  bf16 gradients leave through shared
// memory in TMA stores (a lane holds one output row, so direct stores would
// touch 32 lines per warp instruction); fp32 gradients are stored directly.  Each output element is produced by one
// CTA, in a fixed order: the results are deterministic, with no atomics.
#include <algorithm>
#include <cstdint>

#include "backward.h"
#include "common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kBK = 64;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSlotCols = 256;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;

// ------------------------------------------------------------------ dgrad
constexpr int kDgStages = 3;
constexpr uint32_t kDgABytes = kTileM * kBK * 2;  // one 128-row half, 16 KB
constexpr uint32_t kDgBBytes = 256 * kBK * 2;     // 256 N rows x 64 K, 32 KB
constexpr uint32_t kDgStageBytes = 2 * kDgABytes + kDgBBytes;
constexpr size_t dgrad_smem_bytes() { return 1024 + kDgStages * kDgStageBytes + 256; }
static_assert(dgrad_smem_bytes() <= 232448, "shared memory budget (dgrad)");

__device__ __forceinline__ const CUtensorMap* pick_map(const DgradMaps& m, int i) {
  switch (i) {
    case kMapA0: return &m.a[0];
    case kMapA1: return &m.a[1];
    case kMapA2: return &m.a[2];
    case kMapB0: return &m.b[0];
    case kMapB1: return &m.b[1];
    case kMapB2: return &m.b[2];
    case kMapB3: return &m.b[3];
    default: return &m.b[4];
  }
}

struct DgTile {
  int group, row0, rows, nb, halves;
  bool shared;
};

__device__ __forceinline__ bool dg_tile_at(const DgradParams& p, int tile, DgTile& ti) {
  const int q = tile / p.n_nb;
  ti.nb = tile - q * p.n_nb;
  const int4 e = p.tiles[q];
  ti.group = e.x;
  ti.row0 = e.y;
  ti.rows = e.z;
  ti.halves = e.z > kTileM ? 2 : 1;
  ti.shared = e.x == p.E;
  const int N = ti.shared ? p.N_shared : p.N_routed;
  return ti.nb * 256 < N;
}

__device__ __forceinline__ int dg_nk(const DgradParams& p, bool shared) {
  int nk = 0;
  const int n = shared ? p.n_parts_shared : p.n_parts_routed;
  for (int i = 0; i < n; ++i) nk += shared ? p.parts_shared[i].nk : p.parts_routed[i].nk;
  return nk;
}

__device__ __forceinline__ float sigmoidf_(float g) { return 1.0f / (1.0f + __expf(-g)); }

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) dgrad_kernel(const __grid_constant__ DgradMaps maps, const DgradParams p) {
  constexpr int S = kDgStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stage0 = align_1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(stage0 + S * kDgStageBytes);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  __shared__ uint32_t never;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&tfull[b], 1);
      ptx::mbar_init(&tempty[b], 32 * kEpiWarps);
    }
    ptx::mbar_init(done, 1);
    *abort_flag = 0u;
    never = 0u;
    ptx::fence_barrier_init();
    ptx::fence_proxy_async();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dependency_wait();

  const int mtiles = min(p.ntiles[0], p.max_mtiles);
  const int total = mtiles * p.n_nb;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_a = ptx::policy_evict_normal();  // rows reused by the tile row's column blocks
      const uint64_t pol_w = ptx::policy_evict_normal();
      int kg = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        DgTile ti;
        if (!dg_tile_at(p, tile, ti)) continue;
        const int np = ti.shared ? p.n_parts_shared : p.n_parts_routed;
        const int n0 = ti.nb * 256;
        const uint32_t bytes = ti.halves * kDgABytes + kDgBBytes;
        for (int pi = 0; ok && pi < np; ++pi) {
          const KPart part = ti.shared ? p.parts_shared[pi] : p.parts_routed[pi];
          const CUtensorMap* mA = pick_map(maps, part.a_map);
          const CUtensorMap* mB = pick_map(maps, part.b_map);
          const int arow = ti.row0 + part.a_row_off;
          const int e3 = ti.shared ? 0 : ti.group;
          for (int kb = 0; kb < part.nk; ++kb, ++kg) {
            const int s = kg % S;
            if (!ptx::wait_bounded(&empty[s], ((kg / S) & 1) ^ 1, abort_flag)) {
              raise_status(p.status, abort_flag, kStatusTimeout);
              ok = false;
              break;
            }
            uint8_t* st = stage0 + s * kDgStageBytes;
            ptx::mbar_arrive_expect_tx(&full[s], bytes);
            const int kc = part.a_col + kb * kBK;
            ptx::tma_load_2d(st, mA, &full[s], kc, arow, pol_a);
            if (ti.halves == 2) ptx::tma_load_2d(st + kDgABytes, mA, &full[s], kc, arow + kTileM, pol_a);
            ptx::tma_load_3d(st + 2 * kDgABytes, mB, &full[s], kb * kBK, n0, e3, pol_w);
          }
        }
      }
      for (int j = (kg > S ? kg - S : 0); j < kg; ++j)
        if (!ptx::wait_bounded(&full[j % S], (j / S) & 1, &never)) raise_status(p.status, abort_flag, kStatusTimeout);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_bf16(kTileM, 256, false, false);
      int kg = 0;
      uint32_t use[2] = {0u, 0u};
      int next = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        DgTile ti;
        if (!dg_tile_at(p, tile, ti)) continue;
        const int nk = dg_nk(p, ti.shared);
        for (int h = 0; h < ti.halves; ++h) {
          const int sl = (next + h) & 1;
          if (!ptx::wait_bounded(&tempty[sl], (use[sl] & 1) ^ 1, abort_flag)) {
            raise_status(p.status, abort_flag, kStatusTimeout);
            ok = false;
          }
        }
        if (!ok) break;
        ptx::tc_fence_after();
        for (int kb = 0; kb < nk; ++kb, ++kg) {
          const int s = kg % S;
          if (!ptx::wait_bounded(&full[s], (kg / S) & 1, abort_flag)) {
            raise_status(p.status, abort_flag, kStatusTimeout);
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a0 = ptx::smem_u32(stage0 + s * kDgStageBytes);
          const uint32_t b0 = a0 + 2 * kDgABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t bd = ptx::sdesc_sw128(b0 + kk * 32, 16, 1024);
            for (int h = 0; h < ti.halves; ++h)
              ptx::mma_bf16(tmem + ((next + h) & 1) * kSlotCols, ptx::sdesc_sw128(a0 + h * kDgABytes + kk * 32, 16, 1024),
                            bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          ptx::mma_commit(&empty[s]);
        }
        if (!ok) break;
        for (int h = 0; h < ti.halves; ++h) {
          const int sl = (next + h) & 1;
          ptx::mma_commit(&tfull[sl]);
          ++use[sl];
        }
        next = (next + ti.halves) & 1;
      }
      ptx::mma_commit(done);
      if (!ptx::wait_bounded(done, 0, &never)) raise_status(p.status, abort_flag, kStatusTimeout);
    }
  } else {
    // epilogue: lane quarter q of TMEM, part = which 128 of the 256 columns
    const int q = warp & 3;
    const int part = (warp - 2) / 4;
    const int row = q * 32 + lane;
    uint32_t use[2] = {0u, 0u};
    int next = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
      DgTile ti;
      if (!dg_tile_at(p, tile, ti)) continue;
      const int n0 = ti.nb * 256;
      const int N = ti.shared ? p.N_shared : p.N_routed;
      for (int h = 0; h < ti.halves; ++h) {
        const int sl = (next + h) & 1;
        if (!ptx::wait_bounded(&tfull[sl], use[sl] & 1, abort_flag)) {
          raise_status(p.status, abort_flag, kStatusTimeout);
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + sl * kSlotCols;
        uint32_t buf[4][32];
#pragma unroll
        for (int i = 0; i < 4; ++i) ptx::tmem_ld32(tbase + part * 128 + i * 32, buf[i]);
        ptx::tmem_ld_wait(buf[0]);
        ptx::tmem_ld_keep(buf[1]);
        ptx::tmem_ld_keep(buf[2]);
        ptx::tmem_ld_keep(buf[3]);
        ptx::tc_fence_before();
        ptx::mbar_arrive(&tempty[sl]);
        ++use[sl];
        const int r = h * kTileM + row;
        if (r >= ti.rows) continue;
        if (MODE == kDgradH) {
          // dG = dH u silu'(g), dU = dH silu(g); g and u (bf16) from the forward
          const int64_t grow = (int64_t)ti.row0 + r + (ti.shared ? p.shared_row_off : 0);
          const uint16_t* gu = static_cast<const uint16_t*>(p.gu) + grow * p.ld_gu;
          uint16_t* dgu = static_cast<uint16_t*>(p.out_routed) + grow * p.ld_gu;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int col = n0 + part * 128 + i * 32;
            if (col >= N) continue;
            const uint4* gp = reinterpret_cast<const uint4*>(gu + col);
            const uint4* up = reinterpret_cast<const uint4*>(gu + p.u_off + col);
            uint4* dgp = reinterpret_cast<uint4*>(dgu + col);
            uint4* dup = reinterpret_cast<uint4*>(dgu + p.u_off + col);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const uint4 gv = gp[v], uv = up[v];
              const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w}, uw[4] = {uv.x, uv.y, uv.z, uv.w};
              uint32_t og[4], ou[4];
#pragma unroll
              for (int z = 0; z < 4; ++z) {
                const float g0 = ptx::bf16_lo(gw[z]), g1 = ptx::bf16_hi(gw[z]);
                const float u0 = ptx::bf16_lo(uw[z]), u1 = ptx::bf16_hi(uw[z]);
                const float d0 = __uint_as_float(buf[i][8 * v + 2 * z]), d1 = __uint_as_float(buf[i][8 * v + 2 * z + 1]);
                const float s0 = sigmoidf_(g0), s1 = sigmoidf_(g1);
                og[z] = ptx::pack_bf16x2(d0 * u0 * (s0 * (1.0f + g0 * (1.0f - s0))),
                                         d1 * u1 * (s1 * (1.0f + g1 * (1.0f - s1))));
                ou[z] = ptx::pack_bf16x2(d0 * g0 * s0, d1 * g1 * s1);
              }
              dgp[v] = make_uint4(og[0], og[1], og[2], og[3]);
              dup[v] = make_uint4(ou[0], ou[1], ou[2], ou[3]);
            }
          }
        } else {
          // dX rows: routed rows bf16 (permuted order), shared rows fp32
          const int64_t orow = (int64_t)ti.row0 + r;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int col = n0 + part * 128 + i * 32;
            if (col >= N) continue;
            const uint32_t* v32 = buf[i];
            if (ti.shared) {
              float4* out = reinterpret_cast<float4*>(static_cast<float*>(p.out_shared) + orow * p.ld_out + col);
#pragma unroll
              for (int v = 0; v < 8; ++v)
                out[v] = make_float4(__uint_as_float(v32[4 * v]), __uint_as_float(v32[4 * v + 1]),
                                     __uint_as_float(v32[4 * v + 2]), __uint_as_float(v32[4 * v + 3]));
            } else {
              uint4* out = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out_routed) + orow * p.ld_out + col);
#pragma unroll
              for (int v = 0; v < 4; ++v)
                out[v] = make_uint4(ptx::pack_bf16x2(__uint_as_float(v32[8 * v + 0]), __uint_as_float(v32[8 * v + 1])),
                                    ptx::pack_bf16x2(__uint_as_float(v32[8 * v + 2]), __uint_as_float(v32[8 * v + 3])),
                                    ptx::pack_bf16x2(__uint_as_float(v32[8 * v + 4]), __uint_as_float(v32[8 * v + 5])),
                                    ptx::pack_bf16x2(__uint_as_float(v32[8 * v + 6]), __uint_as_float(v32[8 * v + 7])));
            }
          }
        }
      }
      next = (next + ti.halves) & 1;
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ wgrad
// operand ring depth and output staging buffers (build knobs): the short K
// loops of the weight gradients (2-3 steps per tile at prefill) wait on L2
// latency unless enough stages are in flight
#ifndef MOE_WGRAD_STAGES
#define MOE_WGRAD_STAGES 3
#endif
#ifndef MOE_WGRAD_OUT_BUFS
#define MOE_WGRAD_OUT_BUFS 1
#endif
constexpr int kWgStages = MOE_WGRAD_STAGES;
// 2: two whole-tile buffers (one tile's stores overlap the next tile's
// staging); 1: one whole-tile buffer; 0: one half-tile buffer that the tile's
// two 128-column halves take in turn (frees 32 KB for the operand ring)
constexpr int kWgOutBufs = MOE_WGRAD_OUT_BUFS;
static_assert(kWgOutBufs >= 0 && kWgOutBufs <= 2, "output staging: 0 (half tile), 1 or 2 tiles");
constexpr uint32_t kWgBox = 64 * 64 * 2;            // [64 K rows x 64 features] bf16, 8 KB
constexpr uint32_t kWgABytes = 2 * kWgBox;          // 128 output rows
constexpr uint32_t kWgBBytes = 4 * kWgBox;          // 256 output columns
constexpr uint32_t kWgStageBytes = kWgABytes + kWgBBytes;
// bf16 output tile staged for the TMA stores: four [128 rows x 64 columns]
// boxes, 128-byte swizzled like the output tensor maps; two such buffers, so
// one tile's stores overlap the next tile's staging
constexpr uint32_t kWgOutBox = 128 * 64 * 2;
constexpr uint32_t kWgOutTile = 4 * kWgOutBox;
constexpr uint32_t kWgOutBytes = kWgOutBufs == 0 ? kWgOutTile / 2 : kWgOutBufs * kWgOutTile;
constexpr size_t wgrad_smem_bytes() { return 1024 + kWgStages * kWgStageBytes + kWgOutBytes + 256; }
static_assert(wgrad_smem_bytes() <= 232448, "shared memory budget (wgrad)");

struct WgTile {
  int group;      // < n_routed: routed expert; == n_routed: the shared (or only) group
  int mb, nb;
  int a_row, b_row, rows;
  bool shared;
};

__device__ __forceinline__ void wg_tile_at(const WgradParams& p, int tile, WgTile& t) {
  const int per_r = p.mb_routed * p.nb_routed;
  if (tile < p.n_routed * per_r) {
    t.group = tile / per_r;
    const int rem = tile - t.group * per_r;
    t.mb = rem / p.nb_routed;
    t.nb = rem - t.mb * p.nb_routed;
    t.a_row = p.offsets[t.group];
    t.b_row = t.a_row;
    t.rows = p.offsets[t.group + 1] - t.a_row;
    t.shared = false;
  } else {
    const int rem = tile - p.n_routed * per_r;
    t.group = p.n_routed;
    t.mb = rem / p.nb_shared;
    t.nb = rem - t.mb * p.nb_shared;
    t.a_row = p.a_shared_row0;
    t.b_row = p.b_shared_row0;
    t.rows = p.shared_rows;
    t.shared = true;
  }
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) wgrad_kernel(const __grid_constant__ CUtensorMap tmA_r,
                                                            const __grid_constant__ CUtensorMap tmA_s,
                                                            const __grid_constant__ CUtensorMap tmB_r,
                                                            const __grid_constant__ CUtensorMap tmB_s,
                                                            const __grid_constant__ WgradOutMaps om,
                                                            const WgradParams p) {
  constexpr int S = kWgStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stage0 = align_1024(smem_raw);
  uint8_t* stg = stage0 + S * kWgStageBytes;  // staged bf16 output tile
  uint64_t* full = reinterpret_cast<uint64_t*>(stg + kWgOutBytes);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  __shared__ uint32_t never;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&tfull[b], 1);
      ptx::mbar_init(&tempty[b], 32 * kEpiWarps);
    }
    ptx::mbar_init(done, 1);
    *abort_flag = 0u;
    never = 0u;
    ptx::fence_barrier_init();
    ptx::fence_proxy_async();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dependency_wait();

  const int total = p.n_routed * p.mb_routed * p.nb_routed + (p.has_shared ? p.mb_shared * p.nb_shared : 0);

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol = ptx::policy_evict_normal();  // a group's rows serve all its tiles
      int kg = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        WgTile t;
        wg_tile_at(p, tile, t);
        const CUtensorMap* mA = t.shared ? &tmA_s : &tmA_r;
        const CUtensorMap* mB = t.shared ? &tmB_s : &tmB_r;
        const int m0 = t.mb * 128;
        const int nk = (t.rows + kBK - 1) / kBK;
        for (int kb = 0; kb < nk; ++kb, ++kg) {
          const int s = kg % S;
          if (!ptx::wait_bounded(&empty[s], ((kg / S) & 1) ^ 1, abort_flag)) {
            raise_status(p.status, abort_flag, kStatusTimeout);
            ok = false;
            break;
          }
          uint8_t* st = stage0 + s * kWgStageBytes;
          ptx::mbar_arrive_expect_tx(&full[s], kWgStageBytes);
          const int ra = t.a_row + kb * kBK, rb = t.b_row + kb * kBK;
          ptx::tma_load_2d(st, mA, &full[s], m0, ra, pol);
          ptx::tma_load_2d(st + kWgBox, mA, &full[s], m0 + 64, ra, pol);
          uint8_t* sb = st + kWgABytes;
          if (MODE == kWgradW13) {
            // [dG columns n0..n0+127 | dU columns n0..n0+127]
            const int n0 = t.nb * 128;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              ptx::tma_load_2d(sb + h * kWgBox, mB, &full[s], n0 + 64 * h, rb, pol);
              ptx::tma_load_2d(sb + (2 + h) * kWgBox, mB, &full[s], p.u_off + n0 + 64 * h, rb, pol);
            }
          } else {
            const int n0 = t.nb * 256;
#pragma unroll
            for (int h = 0; h < 4; ++h) ptx::tma_load_2d(sb + h * kWgBox, mB, &full[s], n0 + 64 * h, rb, pol);
          }
        }
      }
      for (int j = (kg > S ? kg - S : 0); j < kg; ++j)
        if (!ptx::wait_bounded(&full[j % S], (j / S) & 1, &never)) raise_status(p.status, abort_flag, kStatusTimeout);
    }
  } else if (warp == 1) {
    // the whole warp waits for each stage; on a group's last, partial K step
    // it zeroes the rows past the group's end (they belong to the next group)
    // in both operands, then lane 0 issues the MMAs
    constexpr uint32_t idesc = ptx::idesc_bf16(128, 256, true, true);
    int kg = 0;
    uint32_t use[2] = {0u, 0u};
    int tl = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
      WgTile t;
      wg_tile_at(p, tile, t);
      const int nk = (t.rows + kBK - 1) / kBK;
      const int sl = tl & 1;
      if (lane == 0 && !ptx::wait_bounded(&tempty[sl], (use[sl] & 1) ^ 1, abort_flag)) {
        raise_status(p.status, abort_flag, kStatusTimeout);
        ok = false;
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      ptx::tc_fence_after();
      for (int kb = 0; kb < nk; ++kb, ++kg) {
        const int s = kg % S;
        const bool landed = ptx::wait_bounded(&full[s], (kg / S) & 1, abort_flag);
        if (!__all_sync(0xffffffffu, landed)) {
          if (lane == 0) raise_status(p.status, abort_flag, kStatusTimeout);
          ok = false;
          break;
        }
        uint8_t* st = stage0 + s * kWgStageBytes;
        // rows of this K step inside the group: only the 16-row MMA slices
        // that hold some are issued; the rest of the last such slice (rows
        // of the next group) is zeroed in A, which the MMA multiplies with B
        // (every B row a slice can reach holds finite values: written rows,
        // or zero fill past the end of the tensor)
        const int valid = t.rows - kb * kBK;
        const int n_mma = valid < kBK ? (valid + 15) / 16 : kBK / 16;
        const int zend = n_mma * 16;
        if (valid < zend) {
          // 2 A boxes x (zend - valid) rows x 8 16-byte chunks; a whole
          // 128-byte row is zeroed, so the swizzle of its chunks does not matter
          const int zr = zend - valid;
          for (int i = lane; i < 2 * zr * 8; i += 32) {
            const int box = i / (zr * 8);
            const int rem = i - box * zr * 8;
            const int rr = valid + rem / 8, ch = rem & 7;
            *reinterpret_cast<uint4*>(st + box * kWgBox + rr * 128 + ch * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
          ptx::fence_proxy_async();
          __syncwarp();
        }
        if (lane == 0) {
          ptx::tc_fence_after();
          const uint32_t a0 = ptx::smem_u32(st);
          const uint32_t b0 = a0 + kWgABytes;
          for (int kk = 0; kk < n_mma; ++kk)
            ptx::mma_bf16(tmem + sl * kSlotCols, ptx::sdesc_sw128(a0 + kk * 2048, kWgBox, 1024),
                          ptx::sdesc_sw128(b0 + kk * 2048, kWgBox, 1024), idesc, (kb | kk) != 0 ? 1u : 0u);
          ptx::mma_commit(&empty[s]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) ptx::mma_commit(&tfull[sl]);
      ++use[sl];
      ++tl;
    }
    if (lane == 0) {
      ptx::mma_commit(done);
      if (!ptx::wait_bounded(done, 0, &never)) raise_status(p.status, abort_flag, kStatusTimeout);
    }
  } else {
    const int q = warp & 3;
    const int part = (warp - 2) / 4;
    const int row = q * 32 + lane;  // output row within the tile (TMEM lane)
    uint32_t use[2] = {0u, 0u};
    int tl = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
      WgTile t;
      wg_tile_at(p, tile, t);
      const int sl = tl & 1;
      const bool got = ptx::wait_bounded(&tfull[sl], use[sl] & 1, abort_flag);
      if (!got) raise_status(p.status, abort_flag, kStatusTimeout);
      if (p.out_bf16) {
        // the epilogue warps meet on a named barrier below, so they leave the
        // loop together or not at all; this barrier is also where the stores
        // of two tiles ago are known to have read this tile's staging buffer
        // (the previous tile's may still be in flight from the other one)
        if (threadIdx.x == 64) {
          if (kWgOutBufs == 2)
            ptx::bulk_wait_read_one_pending();
          else
            ptx::bulk_wait_read_all();  // 0 or 1 buffer: the previous stores must have read it
        }
        if (!ptx::named_barrier_and(1, 32 * kEpiWarps, got)) break;
      } else if (!got) {
        break;
      }
      ptx::tc_fence_after();
      uint32_t buf[4][32];
      const bool any = t.rows > 0;
      if (any) {
        const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + sl * kSlotCols;
#pragma unroll
        for (int i = 0; i < 4; ++i) ptx::tmem_ld32(tbase + part * 128 + i * 32, buf[i]);
        ptx::tmem_ld_wait(buf[0]);
        ptx::tmem_ld_keep(buf[1]);
        ptx::tmem_ld_keep(buf[2]);
        ptx::tmem_ld_keep(buf[3]);
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 32; ++j) buf[i][j] = 0u;  // a group without rows: zero gradient
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(&tempty[sl]);
      ++use[sl];
      ++tl;
      if (p.out_bf16) {
        // bf16 gradients: the tile goes through shared memory and leaves in
        // four TMA stores (full lines, rows past the matrix clipped by the
        // tensor map)
        const bool issuer = threadIdx.x == 64;
        const int m0 = t.mb * 128, g = t.shared ? 0 : t.group;
        const int ncols = t.shared ? p.ncols_shared : p.ncols_routed;
        // output box b (64 columns of the tile) -> tensor map index and column
        auto box_target = [&](int b, int& mi, int& col) {
          if (MODE == kWgradW13) {
            mi = (t.shared ? 2 : 0) + (b >> 1);  // boxes 0-1: dW1, 2-3: dW3
            col = t.nb * 128 + 64 * (b & 1);
          } else {
            mi = t.shared ? 2 : 0;
            col = t.nb * 256 + 64 * b;
          }
        };
        // this thread's 128 columns (its part) as 16-byte bf16 chunks into the
        // staging boxes at `dst` (box index relative to the part's first box)
        auto stage_part = [&](uint8_t* dst) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint8_t* box = dst + (i / 2) * kWgOutBox + row * 128;
            const int j0 = (i & 1) * 4;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const uint32_t* w8 = buf[i] + 8 * v;
              *reinterpret_cast<uint4*>(box + (((j0 + v) ^ (row & 7)) << 4)) =
                  make_uint4(ptx::pack_bf16x2(__uint_as_float(w8[0]), __uint_as_float(w8[1])),
                             ptx::pack_bf16x2(__uint_as_float(w8[2]), __uint_as_float(w8[3])),
                             ptx::pack_bf16x2(__uint_as_float(w8[4]), __uint_as_float(w8[5])),
                             ptx::pack_bf16x2(__uint_as_float(w8[6]), __uint_as_float(w8[7])));
            }
          }
        };
        if (kWgOutBufs > 0) {
          uint8_t* tile_buf = stg + (tl % (kWgOutBufs > 0 ? kWgOutBufs : 1)) * kWgOutTile;
          stage_part(tile_buf + part * 2 * kWgOutBox);
          ptx::fence_proxy_async();
          ptx::named_barrier(1, 32 * kEpiWarps);
          if (issuer) {
#pragma unroll
            for (int b = 0; b < 4; ++b) {
              int mi, col;
              box_target(b, mi, col);
              if (col < ncols) ptx::tma_store_3d(&om.m[mi], tile_buf + b * kWgOutBox, col, m0, g);
            }
            ptx::bulk_commit_group();
          }
        } else {
          // the two halves of the tile through one half-tile buffer in turn
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (part == h) stage_part(stg);
            ptx::fence_proxy_async();
            ptx::named_barrier(1, 32 * kEpiWarps);
            if (issuer) {
#pragma unroll
              for (int b = 0; b < 2; ++b) {
                int mi, col;
                box_target(2 * h + b, mi, col);
                if (col < ncols) ptx::tma_store_3d(&om.m[mi], stg + b * kWgOutBox, col, m0, g);
              }
              ptx::bulk_commit_group();
              if (h == 0) ptx::bulk_wait_read_all();
            }
            if (h == 0) ptx::named_barrier(1, 32 * kEpiWarps);
          }
        }
        continue;
      }
      const int M = t.shared ? p.M_shared : p.M_routed;
      const int m = t.mb * 128 + row;
      if (m >= M) continue;
      const int ncols = t.shared ? p.ncols_shared : p.ncols_routed;  // row length of the output matrix
      // output matrix and its first column for this thread's 128 columns
      void* base;
      int c0;
      if (MODE == kWgradW13) {
        base = part == 0 ? (t.shared ? p.out1_shared : p.out1) : (t.shared ? p.out2_shared : p.out2);
        c0 = t.nb * 128;
      } else {
        base = t.shared ? p.out1_shared : p.out1;
        c0 = t.nb * 256 + part * 128;
      }
      const int64_t mat = t.shared ? 0 : (int64_t)t.group * M * ncols;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int col = c0 + i * 32;
        if (col >= ncols) continue;
        const uint32_t* v32 = buf[i];
        const int64_t off = mat + (int64_t)m * ncols + col;
        float4* out = reinterpret_cast<float4*>(static_cast<float*>(base) + off);
#pragma unroll
        for (int v = 0; v < 8; ++v)
          out[v] = make_float4(__uint_as_float(v32[4 * v]), __uint_as_float(v32[4 * v + 1]),
                               __uint_as_float(v32[4 * v + 2]), __uint_as_float(v32[4 * v + 3]));
      }
    }
    // the last tile's stores complete before the CTA exits
    if (p.out_bf16 && threadIdx.x == 64) ptx::bulk_wait_all();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------ small kernels
// out[i] = bf16(in[i]) for a row-major [rows, cols] fp32 matrix, written into
// rows of ld_out >= cols elements whose columns cols..ld_out-1 are zeroed.
__global__ void cast_pad_bf16_kernel(const float* __restrict__ in, int64_t rows, int cols, int ld_out,
                                     uint16_t* __restrict__ out) {
  grid_dependency_wait();
  const int64_t n = rows * ld_out;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / ld_out;
    const int c = (int)(i - r * ld_out);
    const float v = c < cols ? in[r * cols + c] : 0.0f;
    out[i] = (uint16_t)(ptx::pack_bf16x2(v, 0.0f) & 0xFFFFu);
  }
}

// out[c, e] = in[e, c] for bf16 in [E, d]; out [d, ld_out], columns E..ld_out-1
// zero.  32 x 32 tiles through shared memory.
__global__ void transpose_pad_bf16_kernel(const uint16_t* __restrict__ in, int E, int d, int ld_out,
                                          uint16_t* __restrict__ out) {
  __shared__ uint16_t tile[32][33];
  grid_dependency_wait();
  const int e0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int e = e0 + i, c = c0 + threadIdx.x;
    tile[i][threadIdx.x] = (e < E && c < d) ? in[(int64_t)e * d + c] : (uint16_t)0;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i, e = e0 + threadIdx.x;
    if (c < d && e < ld_out) out[(int64_t)c * ld_out + e] = tile[threadIdx.x][i];
  }
}

}  // namespace

cudaError_t launch_dgrad(int mode, const DgradMaps& maps, const DgradParams& p, int grid, cudaStream_t stream) {
  const size_t smem = dgrad_smem_bytes();
  auto kernel = mode == kDgradH ? dgrad_kernel<kDgradH> : dgrad_kernel<kDgradX>;
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  if (grid <= 0) return cudaSuccess;
  err = launch_chained(kernel, dim3(grid), dim3(kThreads), smem, stream, maps, p);
  return err != cudaSuccess ? err : cudaGetLastError();
}

cudaError_t launch_wgrad(int mode, const CUtensorMap& tmA_r, const CUtensorMap& tmA_s, const CUtensorMap& tmB_r,
                         const CUtensorMap& tmB_s, const WgradOutMaps& om, const WgradParams& p, int grid,
                         cudaStream_t stream) {
  const size_t smem = wgrad_smem_bytes();
  auto kernel = mode == kWgradW13 ? wgrad_kernel<kWgradW13> : wgrad_kernel<kWgradPlain>;
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const int total = p.n_routed * p.mb_routed * p.nb_routed + (p.has_shared ? p.mb_shared * p.nb_shared : 0);
  grid = std::min(grid, total);
  if (grid <= 0) return cudaSuccess;
  err = launch_chained(kernel, dim3(grid), dim3(kThreads), smem, stream, tmA_r, tmA_s, tmB_r, tmB_s, om, p);
  return err != cudaSuccess ? err : cudaGetLastError();
}

cudaError_t launch_cast_pad_bf16(const float* in, int64_t rows, int cols, int ld_out, void* out, int num_sms,
                                 cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const int64_t n = rows * ld_out;
  const unsigned g = (unsigned)std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, (int64_t)num_sms * 8));
  const cudaError_t err = launch_chained(cast_pad_bf16_kernel, dim3(g), dim3(256), 0, stream, in, rows, cols, ld_out,
                                         static_cast<uint16_t*>(out));
  return err != cudaSuccess ? err : cudaGetLastError();
}

cudaError_t launch_transpose_pad_bf16(const void* in, int E, int d, int ld_out, void* out, cudaStream_t stream) {
  const dim3 grid((unsigned)((d + 31) / 32), (unsigned)((ld_out + 31) / 32));
  const cudaError_t err = launch_chained(transpose_pad_bf16_kernel, grid, dim3(32, 8), 0, stream,
                                         static_cast<const uint16_t*>(in), E, d, ld_out, static_cast<uint16_t*>(out));
  return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace moe
