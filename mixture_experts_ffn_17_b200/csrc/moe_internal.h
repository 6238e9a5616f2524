// moe_internal.h -- host-side declarations shared by the library's .cu files.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace moe {

constexpr int kTileM = 128;     // rows per MMA (tcgen05 M) and per A box
constexpr int kTileRows = 256;  // rows per grouped-GEMM tile list entry (two M halves)
// A segment's last, partial tile runs on a CTA pair (as an M=256 MMA) when it
// holds more than this many rows, else on one CTA.
constexpr int kPairMinRows = 192;

// K depth of one grouped-GEMM pipeline stage (32: A halves use a 64-byte
// swizzle; 64: a 128-byte swizzle) and the number of stages.
#ifndef MOE_GEMM_BK
#define MOE_GEMM_BK 64
#endif
#ifndef MOE_GEMM_STAGES
#define MOE_GEMM_STAGES 3
#endif
// Weight boxes are prefetched into L2 this many K stages ahead of their load
// (0 = off).
#ifndef MOE_GEMM_L2_PREFETCH
#define MOE_GEMM_L2_PREFETCH 0
#endif
constexpr int kGemmL2Prefetch = MOE_GEMM_L2_PREFETCH;
constexpr int kGemmBK = MOE_GEMM_BK;
constexpr int kGemmStages = MOE_GEMM_STAGES;
static_assert(kGemmBK == 32 || kGemmBK == 64, "stage K depth must be 32 or 64");

// Device status bits OR-ed into the status word at the head of the workspace.
enum : uint32_t {
  kStatusTimeout = 1u,  // a bounded wait gave up
  kStatusBounds = 2u,   // an index outside its range was seen and skipped
};

// A wait longer than this is a fault (a wait in a healthy launch lasts
// microseconds).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

struct RouteParams {
  int route;        // 0: top-k then softmax; 1: sigmoid group-limited
  int n_group;
  int topk_group;
  int group_topn;
  float route_scale;
};

// router.cu
int router_expert_block(int E);
// Number of K splits of the gate GEMM on a device with `sms` SMs (1 when the
// (128-token, expert-block) tiles alone fill half the device); non-decreasing
// in sms.  Split partial sums are fp64 [splits, T, E].
int router_splits(int64_t T, int d, int E, int sms);
constexpr int kRouterMaxSms = 256;  // workspace is sized for router_splits(.., kRouterMaxSms)
// splits == 1: fp32 logits written directly; splits > 1: fp64 partials to
// `part`, summed in split order by the top-k launch.
cudaError_t launch_router_logits(const CUtensorMap& tm_x, const CUtensorMap& tm_wg, int T, int d, int E, int splits,
                                 float* logits, double* part, uint32_t* status, cudaStream_t stream);
// splits > 1: logits[t][e] = (float) sum_s part[s][t][e] is computed (and
// stored to `logits`) first, by one more launch; otherwise logits are read.
cudaError_t launch_router_topk(float* logits, const double* part, int splits, const float* bias,
                               const uint8_t* allowed, const RouteParams& rp, int T, int E, int k, int32_t* idx,
                               float* w, cudaStream_t stream);

// monitor.cu
cudaError_t launch_expert_utilisation(const int32_t* counts, int E, float* util, int32_t* flags,
                                      cudaStream_t stream);

// The routed experts one call computes: [e_lo, e_hi), on every token routed
// to them.  The whole layer is {0, E}; an expert-parallel rank takes its slice.
struct Shard {
  int e_lo, e_hi;
};

// permute.cu
int permute_blocks(int64_t T);
cudaError_t launch_permute(const int32_t* idx, int64_t T, int k, int E, int32_t* hist, int32_t* base,
                           int32_t* counts, int32_t* offsets, int32_t* perm_token, int32_t* row_of,
                           uint32_t* status, cudaStream_t stream);
// offsets != nullptr: only permuted rows of experts [e_lo, e_hi) are copied.
cudaError_t launch_gather_rows(const void* x, const int32_t* perm_token, int64_t rows, int d, void* x_perm,
                               int num_sms, cudaStream_t stream, const int32_t* offsets = nullptr, int e_lo = 0,
                               int e_hi = 0);
// x_perm[row_of[t*k + j]] = x[t] in token order (each x row read once) for the
// rows [offsets[e_lo], offsets[e_hi]); the same rows and values as
// launch_gather_rows over that range.
cudaError_t launch_scatter_rows(const void* x, const int32_t* row_of, int64_t T, int k, int d, void* x_perm,
                                int num_sms, cudaStream_t stream, const int32_t* offsets, int e_lo, int e_hi);
// Also zeroes the grouped GEMMs' tile counters (kNumSchedCounters ints).
constexpr int kNumSchedCounters = 4;
// tiles_pair != nullptr: full 256-row tiles go to that list (ntiles[2], [3])
// and only partial tiles to `tiles` (ntiles[0], [1]).
cudaError_t launch_build_tiles(const int32_t* offsets, int E, int64_t T, const Shard& shard, bool with_shared,
                               int4* tiles, int32_t* ntiles, int* sched_counters, cudaStream_t stream,
                               int4* tiles_pair = nullptr);

// grouped_gemm.cu
// Which part of the tile list a grouped-GEMM launch walks.
enum TileSet : int { kTilesAll = 0, kTilesRouted = 1, kTilesShared = 2 };

struct GemmParams {
  const int4* tiles;
  const int32_t* ntiles;  // [0] = all tiles, [1] = routed tiles (the shared expert's follow)
  int max_mtiles;         // capacity of the tile list (clamps the device counts)
  int tile_set;           // TileSet
  int E;                  // group index E = shared expert
  int group_base;         // routed group g uses weight (and scale) slice g - group_base
  int n_nb;               // N blocks per tile row (max over routed / shared)
  int K_routed, K_shared;
  int N_routed, N_shared;
  int a_shared_row_offset;  // row of the shared expert's first A row in its map
  void* out_routed;       // bf16 rows
  void* out_shared;       // SwiGLU: bf16 rows; down: fp32 rows
  int64_t out_shared_row_offset;  // rows to skip in out_shared
  int ld_out;             // output row stride (elements)
  // FP8 routed weights: fp32 block scales [E, K/128, N/128] of the B (and,
  // SwiGLU, C = W3) operand
  const float* scale_b;
  const float* scale_c;
  uint32_t* status;
  int* sched_counter;     // tiles claimed so far (zeroed by the tile-list kernel)
  // Failure-path testing: when nonzero the producer issues no loads, so the
  // MMA issuer's bounded wait runs out and the launch reports a timeout.
  int debug_withhold_loads;
  // SwiGLU, bf16 weights, one-CTA kernel (the backward pass keeps the
  // forward's g and u): when non-null, g and u are also stored bf16 in rows of
  // 2 * ld_out elements, g at column n and u at column ld_out + n, on the same
  // rows as H.
  void* out_gu;
};

int gemm_block_n_swiglu();
int gemm_block_n_down();
cudaError_t launch_grouped_swiglu(const CUtensorMap& tmA_r, const CUtensorMap& tmA_s, const CUtensorMap& tmW1_r,
                                  const CUtensorMap& tmW1_s, const CUtensorMap& tmW3_r, const CUtensorMap& tmW3_s,
                                  const GemmParams& p, int grid, cudaStream_t stream);
// Full 256-row tiles of bf16 experts on 2-CTA clusters (tcgen05.mma
// .cta_group::2, M=256): the pair tile list (full tiles and long last tiles); grid is
// rounded down to whole clusters.
cudaError_t launch_grouped_swiglu_pair(const CUtensorMap& tmA_r, const CUtensorMap& tmA_s, const CUtensorMap& tmW1_r,
                                       const CUtensorMap& tmW1_s, const CUtensorMap& tmW3_r, const CUtensorMap& tmW3_s,
                                       const GemmParams& p, int grid, cudaStream_t stream);
cudaError_t launch_grouped_down_pair(const CUtensorMap& tmA, const CUtensorMap& tmW2_r, const CUtensorMap& tmW2_s,
                                     const GemmParams& p, int grid, cudaStream_t stream);
// FP8 routed tiles of the pair list on 2-CTA clusters (tile_set must be
// kTilesRouted: the shared expert is bf16).
cudaError_t launch_grouped_swiglu_pair_fp8(const CUtensorMap& tmA_r, const CUtensorMap& tmW1_r,
                                           const CUtensorMap& tmW3_r, const GemmParams& p, int grid,
                                           cudaStream_t stream);
cudaError_t launch_grouped_down_pair_fp8(const CUtensorMap& tmA, const CUtensorMap& tmW2_r, const GemmParams& p,
                                         int grid, cudaStream_t stream);
cudaError_t launch_grouped_down(const CUtensorMap& tmA, const CUtensorMap& tmW2_r, const CUtensorMap& tmW2_s,
                                const GemmParams& p, int grid, cudaStream_t stream);
// FP8 (e4m3 + 128x128 block scales) routed experts; the tensor maps of W are
// uint8 [E, K, N] with [1 x 64 x 128] boxes and no swizzle.  short_rows: 1
// when every routed tile holds at most 128 rows, 2 when at most 64 (the caller
// knows it, e.g. T <= 128 or 64 with distinct experts per token): the kernel's
// stages then hold one 128-row A half, or one 64-row A box (tmA's boxes must
// be 64 rows then), and its rings are deeper; a longer tile is skipped and
// raises kStatusBounds.  0: the general layout.
cudaError_t launch_grouped_swiglu_fp8(const CUtensorMap& tmA_r, const CUtensorMap& tmW1_r,
                                      const CUtensorMap& tmW3_r, const GemmParams& p, int grid,
                                      cudaStream_t stream, int short_rows);
cudaError_t launch_grouped_down_fp8(const CUtensorMap& tmA, const CUtensorMap& tmW2_r, const GemmParams& p, int grid,
                                    cudaStream_t stream, int short_rows);

// ep.cu: expert-major order of rows received from n_src ranks (source-major,
// each source's rows in expert order); n_src * E_local <= 1024.
cudaError_t launch_ep_regroup(const int32_t* recv_counts, int n_src, int E_local, int32_t* offsets_local,
                              int32_t* to_expert_major, int32_t* to_source_major, cudaStream_t stream);

// combine.cu
// offsets != nullptr: only permuted rows of experts [shard.e_lo, shard.e_hi)
// are added.  topk_w == nullptr: every row has weight 1.
cudaError_t launch_combine(const void* Y_perm, const float* Y_shared, const int32_t* row_of, const float* topk_w,
                           int64_t T, int k, int d, void* y, bool y_bf16, cudaStream_t stream,
                           const int32_t* offsets = nullptr, const Shard* shard = nullptr);

}  // namespace moe
