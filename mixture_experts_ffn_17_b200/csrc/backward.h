// backward.h -- launchers of the backward-pass kernels (backward.cu).
#pragma once

#include <cstdint>
#include <cuda.h>
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

// ---------------------------------------------------- expert contractions
// (grouped_gemm_bwd.cu)

// dgrad kernel modes: dH = dO W2^T with the SwiGLU derivative in the epilogue
// (writes dG | dU), and dX = [dG | dU] [W1 ; W3]^T (+ dl Wg for the shared
// expert's tiles).
enum : int { kDgradH = 0, kDgradX = 1 };

// Tensor maps of one dgrad launch: A maps are 2D bf16 [rows, K] with
// [128 rows x 64 K] boxes; B maps are 3D bf16 [groups, N, K] with [1 x 256 x 64]
// boxes (the weights read K-major).  Both use a 128-byte swizzle.
enum : int { kMapA0 = 0, kMapA1 = 1, kMapA2 = 2, kMapB0 = 3, kMapB1 = 4, kMapB2 = 5, kMapB3 = 6, kMapB4 = 7 };
struct DgradMaps {
  CUtensorMap a[3];
  CUtensorMap b[5];
};

// One part of a tile's K range: nk steps of 64, A columns from a_col on (rows
// shifted by a_row_off), B (K columns from 0, N rows of the tile's column
// block, group = the tile's expert, or 0 for the shared expert's tiles).
struct KPart {
  int nk, a_map, a_col, a_row_off, b_map;
};

struct DgradParams {
  const int4* tiles;        // the forward's one-CTA tile list (shared expert = group E, after the routed tiles)
  const int32_t* ntiles;    // [0] = tiles in the list
  int max_mtiles;
  int E;
  int n_nb;                 // 256-column blocks per tile row
  int N_routed, N_shared;   // output columns
  KPart parts_routed[2];
  int n_parts_routed;
  KPart parts_shared[3];
  int n_parts_shared;
  // kDgradH: g | u of the forward (bf16 rows, u at column u_off, row stride
  // ld_gu; shared rows from shared_row_off on) and dG | dU written in the same
  // layout to out_routed.  kDgradX: routed rows bf16 to out_routed, shared rows
  // fp32 to out_shared, row stride ld_out.
  const void* gu;
  int64_t ld_gu;
  int u_off;
  int64_t shared_row_off;
  void* out_routed;
  void* out_shared;
  int64_t ld_out;
  uint32_t* status;
};

cudaError_t launch_dgrad(int mode, const DgradMaps& maps, const DgradParams& p, int grid, cudaStream_t stream);

// wgrad kernel modes: out1 / out2 = A^T [dG | dU] (dW1 and dW3), or out1 = A^T B.
enum : int { kWgradW13 = 0, kWgradPlain = 1 };

// Tiles: (group, 128 output rows, 256 output columns -- W13: 128 columns of
// dW1 and the same 128 of dW3); routed group g contracts rows
// offsets[g] .. offsets[g+1] of A and B, the shared (or only) group
// shared_rows rows from a_shared_row0 / b_shared_row0.  A and B maps are 2D
// bf16 [rows, features] with [64 rows x 64 features] boxes, 128-byte swizzle.
// Outputs are row-major [groups, M, ncols] (routed) and [M, ncols] (shared),
// fp32 or bf16.
struct WgradParams {
  const int32_t* offsets;
  int n_routed;             // routed groups (0: only the shared group)
  int has_shared;
  int mb_routed, nb_routed, mb_shared, nb_shared;
  int M_routed, M_shared;   // output rows
  int ncols_routed, ncols_shared;
  int a_shared_row0, b_shared_row0, shared_rows;
  int u_off;                // W13: column of dU in the B rows
  void* out1;
  void* out2;
  void* out1_shared;
  void* out2_shared;
  int out_bf16;
  uint32_t* status;
};

// bf16 outputs (out_bf16): 3D bf16 maps [groups, M, ncols] with [1 x 128 x 64]
// boxes, 128-byte swizzle, of out1, out2 (routed) and out1_shared,
// out2_shared (groups = 1); the pointers in WgradParams then go unused.
struct WgradOutMaps {
  CUtensorMap m[4];
};

cudaError_t launch_wgrad(int mode, const CUtensorMap& tmA_r, const CUtensorMap& tmA_s, const CUtensorMap& tmB_r,
                         const CUtensorMap& tmB_s, const WgradOutMaps& om, const WgradParams& p, int grid,
                         cudaStream_t stream);

// bf16 copy of a row-major fp32 [rows, cols] matrix into rows of ld_out
// elements, the columns past cols zeroed.
cudaError_t launch_cast_pad_bf16(const float* in, int64_t rows, int cols, int ld_out, void* out, int num_sms,
                                 cudaStream_t stream);
// out [d, ld_out] = transpose of the bf16 [E, d] matrix `in`, columns past E zeroed.
cudaError_t launch_transpose_pad_bf16(const void* in, int E, int d, int ld_out, void* out, cudaStream_t stream);

}  // namespace moe
