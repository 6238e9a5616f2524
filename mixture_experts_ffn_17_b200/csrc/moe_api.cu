// moe_api.cu -- host side of the C ABI declared in include/moe.h: argument
// validation, workspace layout, TMA tensor maps and the launch sequences.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "moe.h"
#include "backward.h"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status validate_shape(const moe_shape* s) {
  if (!s) return MOE_ERR_INVALID_ARG;
  if (s->T < 0 || s->d <= 0 || s->E <= 0 || s->k <= 0 || s->inter <= 0 || s->shared_inter < 0)
    return MOE_ERR_INVALID_ARG;
  if (s->k > s->E) return MOE_ERR_INVALID_ARG;
  if (s->route != MOE_ROUTE_TOPK_SOFTMAX && s->route != MOE_ROUTE_SIGMOID_GROUP) return MOE_ERR_INVALID_ARG;
  if (s->w_dtype != MOE_BF16 && s->w_dtype != MOE_E4M3) return MOE_ERR_INVALID_ARG;
  if (s->y_dtype != MOE_F32 && s->y_dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (s->route == MOE_ROUTE_SIGMOID_GROUP) {
    if (s->n_group <= 0 || s->E % s->n_group != 0) return MOE_ERR_INVALID_ARG;
    const int gsize = s->E / s->n_group;
    if (s->topk_group <= 0 || s->topk_group > s->n_group) return MOE_ERR_INVALID_ARG;
    if (s->group_topn <= 0 || s->group_topn > gsize) return MOE_ERR_INVALID_ARG;
    if ((int64_t)s->topk_group * gsize < s->k) return MOE_ERR_INVALID_ARG;
    if (s->n_group > 32 || gsize > 64) return MOE_ERR_UNSUPPORTED;
  }
  if (s->d % 128 != 0 || s->inter % 128 != 0 || s->shared_inter % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (s->E % 32 != 0 || s->E > 1024 || s->k > 32) return MOE_ERR_UNSUPPORTED;
  if (s->T * (int64_t)s->k + s->T >= (int64_t)1 << 31) return MOE_ERR_UNSUPPORTED;
  if (s->d > (1 << 20) || s->inter > (1 << 20) || s->shared_inter > (1 << 20)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

struct Layout {
  size_t status, logits, rpart, idx, w, hist, base, counts, offsets, perm, row_of, tiles, tiles_pair, ntiles, sched, x_perm, H, Y_perm,
      Y_shared, total;
  int nb, max_mtiles, Hld;
  int64_t Hrows;
};

Layout make_layout(const moe_shape& s) {
  Layout L{};
  const int64_t T = s.T, Tk = s.T * s.k;
  const bool sh = s.shared_inter > 0;
  L.nb = permute_blocks(T);
  L.max_mtiles = (int)((Tk + kTileRows - 1) / kTileRows + s.E + (sh ? (T + kTileRows - 1) / kTileRows : 0));
  L.Hld = std::max(s.inter, s.shared_inter);
  L.Hrows = Tk + (sh ? T : 0);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off += align_up(std::max<size_t>(bytes, 1));
    return at;
  };
  L.status = take(64);
  L.logits = take((size_t)T * s.E * 4);
  const int rsplits = router_splits(T, s.d, s.E, kRouterMaxSms);
  L.rpart = take(rsplits > 1 ? (size_t)rsplits * T * s.E * 8 : 0);
  L.idx = take((size_t)Tk * 4);
  L.w = take((size_t)Tk * 4);
  L.hist = take((size_t)L.nb * s.E * 4);
  L.base = take((size_t)L.nb * s.E * 4);
  L.counts = take((size_t)s.E * 4);
  L.offsets = take((size_t)(s.E + 1) * 4);
  L.perm = take((size_t)Tk * 4);
  L.row_of = take((size_t)Tk * 4);
  L.tiles = take((size_t)L.max_mtiles * 16);
  L.tiles_pair = take((size_t)L.max_mtiles * 16);
  L.ntiles = take(16);
  L.sched = take(kNumSchedCounters * 4);
  L.x_perm = take((size_t)Tk * s.d * 2);
  L.H = take((size_t)L.Hrows * L.Hld * 2);
  L.Y_perm = take((size_t)Tk * s.d * 2);
  L.Y_shared = take(sh ? (size_t)T * s.d * 4 : 0);
  L.total = off;
  return L;
}

template <typename P>
P* at(void* ws, size_t off) {
  return reinterpret_cast<P*>(static_cast<uint8_t*>(ws) + off);
}

// ------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// bf16 row-major [outer, inner]; box [box_outer rows x box_inner elements];
// the swizzle span equals the box row (64 or 128 bytes).
bool map_2d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_inner,
            uint32_t box_outer) {
  const CUtensorMapSwizzle swz = box_inner * 2 == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 row-major [outer, mid, inner]; box [1 x box_mid x 64], 128-byte swizzle.
bool map_3d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t mid, uint64_t outer, uint32_t box_mid) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, mid, outer};
  cuuint64_t strides[2] = {inner * 2, inner * mid * 2};
  cuuint32_t box[3] = {64, box_mid, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// uint8 (e4m3 codes) row-major [outer, mid, inner]; box [1 x 64 x 128], no
// swizzle (the converter warps read the codes row by row).
bool map_3d_u8(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t mid, uint64_t outer) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, mid, outer};
  cuuint64_t strides[2] = {inner, inner * mid};
  cuuint32_t box[3] = {128, 64, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// MOE_DEBUG_WITHHOLD_LOADS=1 in the environment makes the grouped-GEMM
// producers issue no loads (failure-path testing: their consumers' bounded
// waits run out and the call reports MOE_ERR_DEVICE_TIMEOUT).
bool debug_withhold_loads() {
  const char* v = std::getenv("MOE_DEBUG_WITHHOLD_LOADS");
  return v && v[0] == '1';
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

#define MOE_CUDA(call)                          \
  do {                                          \
    if ((call) != cudaSuccess) return MOE_ERR_CUDA; \
  } while (0)

// Full 256-row tiles (and last tiles of more than 192 rows) run on CTA pairs
// (one tcgen05.mma.cta_group::2 M=256 per K step, B read from shared memory
// once per 256 rows; FP8 weights also converted once per 256 rows) when
// segments are long enough for most rows to sit in such tiles: on average at
// least 384 rows per expert, bf16 weights.  With FP8 weights the pair kernels
// measured no faster than the one-CTA path (T=8192 layer: 9.53 vs 9.61 ms), so
// they run only when forced.  MOE_PAIR_TILES=1 / 0 in the environment forces
// pairs on / off.
// FP8 batches whose segments all fit one 128-row half (T <= 128) launch the
// FP8 kernels with one-A-half stages and deeper rings; with 2, those whose
// segments fit 64 rows (T <= 64) use 64-row A boxes and deeper rings still
// (1: only the first; 0: the general layout)
#ifndef MOE_F8_ONE_HALF_STAGES
#define MOE_F8_ONE_HALF_STAGES 2
#endif

bool use_pair_tiles(const moe_shape& s) {
  const char* v = std::getenv("MOE_PAIR_TILES");
  if (v && v[0] == '1') return true;
  if (v && v[0] == '0') return false;
  if (s.w_dtype == MOE_E4M3) return false;
  return s.T * (int64_t)s.k >= (int64_t)384 * s.E;
}

// ------------------------------------------------------------ stages
moe_status run_router(const moe_shape& s, const void* x, const void* Wg, const float* bias, int32_t* idx, float* w,
                      float* logits, double* part, uint32_t* status, cudaStream_t st,
                      const uint8_t* allowed = nullptr) {
  CUtensorMap tm_x, tm_wg;
  const int eb = router_expert_block(s.E);
  if (!map_2d(&tm_x, x, s.d, s.T, 64, 128) || !map_2d(&tm_wg, Wg, s.d, s.E, 64, eb)) return MOE_ERR_CUDA;
  // small batches split the gate GEMM's K so that the grid covers the device
  const int splits = router_splits(s.T, s.d, s.E, std::min(num_sms(), kRouterMaxSms));
  MOE_CUDA(launch_router_logits(tm_x, tm_wg, (int)s.T, s.d, s.E, splits, logits, part, status, st));
  RouteParams rp{s.route, s.n_group, s.topk_group, s.group_topn, s.route_scale};
  MOE_CUDA(launch_router_topk(logits, part, splits, s.route == MOE_ROUTE_SIGMOID_GROUP ? bias : nullptr, allowed, rp,
                              (int)s.T, s.E, s.k, idx, w, st));
  return MOE_OK;
}

Shard whole_layer(const moe_shape& s) { return Shard{0, s.E}; }

// Routed weights (and FP8 scales) hold the experts [shard.e_lo, shard.e_hi)
// only: slice 0 is expert shard.e_lo.
moe_status run_experts(const moe_shape& s, const Layout& L, void* ws, const void* x, const void* x_perm,
                       const int32_t* offsets, const void* W1, const void* W3, const void* W2, const float* s1,
                       const float* s3, const float* s2, const void* W1s, const void* W3s, const void* W2s,
                       void* Y_perm, float* Y_shared, uint32_t* status, cudaStream_t st, const Shard& shard,
                       const cudaEvent_t* ev = nullptr, int64_t max_segment = -1) {
  const bool f8 = s.w_dtype == MOE_E4M3;
  // FP8 launches with short stages and deeper rings when no segment can
  // exceed one 128-row half, or 64 rows (see launch_grouped_swiglu_fp8);
  // max_segment < 0: unknown
  const int f8_short = !f8 || max_segment < 0 || !MOE_F8_ONE_HALF_STAGES || use_pair_tiles(s) ? 0
                       : max_segment <= kTileM / 2 && MOE_F8_ONE_HALF_STAGES >= 2 ? 2
                       : max_segment <= kTileM                                      ? 1
                                                                                    : 0;
  const int a8_rows = f8_short == 2 ? kTileM / 2 : kTileM;  // rows of the FP8 launches' A boxes
  const bool sh = s.shared_inter > 0;
  const int64_t Tk = s.T * s.k;
  int4* tiles = at<int4>(ws, L.tiles);
  int32_t* ntiles = at<int32_t>(ws, L.ntiles);
  uint16_t* H = at<uint16_t>(ws, L.H);
  int* sched = at<int>(ws, L.sched);
  const bool pair = use_pair_tiles(s);
  int4* tiles_pair = pair ? at<int4>(ws, L.tiles_pair) : nullptr;
  MOE_CUDA(launch_build_tiles(offsets, s.E, s.T, shard, sh, tiles, ntiles, sched, st, tiles_pair));
  const int E_w = shard.e_hi - shard.e_lo;  // expert slices held by the weight tensors
  if (ev) MOE_CUDA(cudaEventRecord(ev[0], st));

  const int sms = num_sms();
  // SwiGLU: A = gathered rows (routed) or x (shared); B = W1 | W3 column blocks
  CUtensorMap a_r, a_s, w1_r, w1_s, w3_r, w3_s, a8_r, w18_r, w38_r;
  if (!map_2d(&a_r, x_perm, s.d, Tk, kGemmBK, kTileM) || !map_2d(&a_s, x, s.d, s.T, kGemmBK, kTileM))
    return MOE_ERR_CUDA;
  if (f8) {
    // FP8 launches use a 64-deep K stage whatever the bf16 kernel's depth
    if (!map_2d(&a8_r, x_perm, s.d, Tk, 64, a8_rows) || !map_3d_u8(&w18_r, W1, s.inter, s.d, E_w) ||
        !map_3d_u8(&w38_r, W3, s.inter, s.d, E_w))
      return MOE_ERR_CUDA;
    w1_r = a_r;  // placeholders: the bf16 launch below only walks the shared expert's tiles
    w3_r = a_r;
  } else if (!map_3d(&w1_r, W1, s.inter, s.d, E_w, kGemmBK) || !map_3d(&w3_r, W3, s.inter, s.d, E_w, kGemmBK)) {
    return MOE_ERR_CUDA;
  }
  if (sh) {
    if (!map_3d(&w1_s, W1s, s.shared_inter, s.d, 1, kGemmBK) || !map_3d(&w3_s, W3s, s.shared_inter, s.d, 1, kGemmBK))
      return MOE_ERR_CUDA;
  } else {
    w1_s = w1_r;
    w3_s = w3_r;
  }
  GemmParams p1{};
  p1.tiles = tiles;
  p1.ntiles = ntiles;
  p1.max_mtiles = L.max_mtiles;
  p1.E = s.E;
  p1.group_base = shard.e_lo;
  const int bn1 = gemm_block_n_swiglu();
  p1.n_nb = (L.Hld + bn1 - 1) / bn1;
  p1.K_routed = s.d;
  p1.K_shared = s.d;
  p1.N_routed = s.inter;
  p1.N_shared = s.shared_inter;
  p1.a_shared_row_offset = 0;
  p1.out_routed = H;
  p1.out_shared = H;
  p1.out_shared_row_offset = Tk;
  p1.ld_out = L.Hld;
  p1.status = status;
  p1.tile_set = kTilesAll;
  p1.debug_withhold_loads = debug_withhold_loads() ? 1 : 0;
  p1.sched_counter = sched + 0;
  const int grid1 = (int)std::min<int64_t>(sms, (int64_t)L.max_mtiles * p1.n_nb);
  if (f8) {
    GemmParams q = p1;
    q.tile_set = kTilesRouted;
    q.scale_b = s1;
    q.scale_c = s3;
    if (pair) {
      GemmParams qp = q;
      qp.tiles = tiles_pair;
      qp.ntiles = ntiles + 2;
      MOE_CUDA(launch_grouped_swiglu_pair_fp8(a8_r, w18_r, w38_r, qp, sms, st));
    }
    MOE_CUDA(launch_grouped_swiglu_fp8(a8_r, w18_r, w38_r, q, grid1, st, f8_short));
    if (sh) {
      q = p1;
      q.tile_set = kTilesShared;
      if (pair) {
        GemmParams qp = q;
        qp.tiles = tiles_pair;
        qp.ntiles = ntiles + 2;
        MOE_CUDA(launch_grouped_swiglu_pair(a_r, a_s, w1_r, w1_s, w3_r, w3_s, qp, sms, st));
      }
      q.sched_counter = sched + 1;
      MOE_CUDA(launch_grouped_swiglu(a_r, a_s, w1_r, w1_s, w3_r, w3_s, q, grid1, st));
    }
  } else {
    if (pair) {
      GemmParams q = p1;  // full tiles on CTA pairs, then the partial tiles
      q.tiles = tiles_pair;
      q.ntiles = ntiles + 2;
      MOE_CUDA(launch_grouped_swiglu_pair(a_r, a_s, w1_r, w1_s, w3_r, w3_s, q, sms, st));
    }
    MOE_CUDA(launch_grouped_swiglu(a_r, a_s, w1_r, w1_s, w3_r, w3_s, p1, grid1, st));
  }
  if (ev) MOE_CUDA(cudaEventRecord(ev[1], st));

  // down projection: A = H (routed rows, then shared rows); B = W2 column blocks
  CUtensorMap h_map, w2_r, w2_s, h8_map, w28_r;
  if (!map_2d(&h_map, H, L.Hld, L.Hrows, kGemmBK, kTileM)) return MOE_ERR_CUDA;
  if (f8) {
    if (!map_2d(&h8_map, H, L.Hld, L.Hrows, 64, a8_rows) || !map_3d_u8(&w28_r, W2, s.d, s.inter, E_w))
      return MOE_ERR_CUDA;
    w2_r = h_map;  // placeholder: the bf16 launch below only walks the shared expert's tiles
  } else if (!map_3d(&w2_r, W2, s.d, s.inter, E_w, kGemmBK)) {
    return MOE_ERR_CUDA;
  }
  if (sh) {
    if (!map_3d(&w2_s, W2s, s.d, s.shared_inter, 1, kGemmBK)) return MOE_ERR_CUDA;
  } else {
    w2_s = w2_r;
  }
  GemmParams p2 = p1;
  p2.sched_counter = sched + 2;
  const int bn2 = gemm_block_n_down();
  p2.n_nb = (s.d + bn2 - 1) / bn2;
  p2.K_routed = s.inter;
  p2.K_shared = s.shared_inter;
  p2.N_routed = s.d;
  p2.N_shared = s.d;
  p2.a_shared_row_offset = (int)Tk;
  p2.out_routed = Y_perm;
  p2.out_shared = Y_shared;
  p2.out_shared_row_offset = 0;
  p2.ld_out = s.d;
  const int grid2 = (int)std::min<int64_t>(sms, (int64_t)L.max_mtiles * p2.n_nb);
  if (f8) {
    GemmParams q = p2;
    q.tile_set = kTilesRouted;
    q.scale_b = s2;
    q.scale_c = s2;
    if (pair) {
      GemmParams qp = q;
      qp.tiles = tiles_pair;
      qp.ntiles = ntiles + 2;
      MOE_CUDA(launch_grouped_down_pair_fp8(h8_map, w28_r, qp, sms, st));
    }
    MOE_CUDA(launch_grouped_down_fp8(h8_map, w28_r, q, grid2, st, f8_short));
    if (sh) {
      q = p2;
      q.tile_set = kTilesShared;
      if (pair) {
        GemmParams qp = q;
        qp.tiles = tiles_pair;
        qp.ntiles = ntiles + 2;
        MOE_CUDA(launch_grouped_down_pair(h_map, w2_r, w2_s, qp, sms, st));
      }
      q.sched_counter = sched + 3;
      MOE_CUDA(launch_grouped_down(h_map, w2_r, w2_s, q, grid2, st));
    }
  } else {
    if (pair) {
      GemmParams q = p2;
      q.tiles = tiles_pair;
      q.ntiles = ntiles + 2;
      MOE_CUDA(launch_grouped_down_pair(h_map, w2_r, w2_s, q, sms, st));
    }
    MOE_CUDA(launch_grouped_down(h_map, w2_r, w2_s, p2, grid2, st));
  }
  if (ev) MOE_CUDA(cudaEventRecord(ev[2], st));
  return MOE_OK;
}

bool ws_ok(const void* ws, size_t ws_bytes, size_t need) {
  return ws && ws_bytes >= need && (reinterpret_cast<uintptr_t>(ws) % kAlign) == 0;
}

moe_status forward_impl(const moe_shape* shape, const void* x, const void* Wg, const float* bias, const void* W1,
                        const void* W3, const void* W2, const float* s1, const float* s3, const float* s2,
                        const void* W1s, const void* W3s, const void* W2s, void* y, int32_t* topk_idx_out,
                        float* topk_w_out, int32_t* counts_out, void* ws, size_t ws_bytes, void* stream,
                        const cudaEvent_t* ev, int ep_rank = 0, int ep_size = 1) {
  moe_status v = validate_shape(shape);
  if (v != MOE_OK) return v;
  const moe_shape& s = *shape;
  if (ep_size < 1 || ep_rank < 0 || ep_rank >= ep_size) return MOE_ERR_INVALID_ARG;
  // expert-parallel share (atlas page, "Code" section, the MoE constructor and
  // forward blocks): an even slice of the routed experts, and the shared
  // expert's slice of hidden features (its W1/W3 columns, W2 rows), so that
  // the sum over ranks is the layer
  if (s.E % ep_size != 0 || s.shared_inter % ep_size != 0 || (s.shared_inter / ep_size) % 128 != 0)
    return MOE_ERR_UNSUPPORTED;
  const int e_per = s.E / ep_size;
  const Shard shard{ep_rank * e_per, (ep_rank + 1) * e_per};
  const bool whole = ep_size == 1;
  moe_shape sl = s;  // this rank's experts: shared expert of shared_inter / ep_size features
  sl.shared_inter = s.shared_inter / ep_size;
  const bool sh = s.shared_inter > 0;
  if (!x || !Wg || !W1 || !W3 || !W2 || !y) return MOE_ERR_INVALID_ARG;
  if (sh && (!W1s || !W3s || !W2s)) return MOE_ERR_INVALID_ARG;
  if (s.w_dtype == MOE_E4M3 && (!s1 || !s3 || !s2)) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {x, Wg, bias, W1, W3, W2, s1, s3, s2, W1s, W3s, W2s, y, topk_idx_out, topk_w_out, counts_out};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
  const Layout L = make_layout(s);
  if (!ws_ok(ws, ws_bytes, L.total)) return MOE_ERR_WORKSPACE;
  if (s.T == 0) return MOE_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* status = at<uint32_t>(ws, L.status);
  MOE_CUDA(cudaMemsetAsync(status, 0, 4, st));
  if (ev) MOE_CUDA(cudaEventRecord(ev[0], st));

  int32_t* idx = topk_idx_out ? topk_idx_out : at<int32_t>(ws, L.idx);
  float* w = topk_w_out ? topk_w_out : at<float>(ws, L.w);
  int32_t* counts = counts_out ? counts_out : at<int32_t>(ws, L.counts);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* perm = at<int32_t>(ws, L.perm);
  int32_t* row_of = at<int32_t>(ws, L.row_of);
  void* x_perm = at<void>(ws, L.x_perm);
  void* Y_perm = at<void>(ws, L.Y_perm);
  float* Y_shared = sh ? at<float>(ws, L.Y_shared) : nullptr;

  moe_status r = run_router(s, x, Wg, bias, idx, w, at<float>(ws, L.logits), at<double>(ws, L.rpart), status, st);
  if (r != MOE_OK) return r;
  if (ev) MOE_CUDA(cudaEventRecord(ev[1], st));
  MOE_CUDA(launch_permute(idx, s.T, s.k, s.E, at<int32_t>(ws, L.hist), at<int32_t>(ws, L.base), counts, offsets,
                          perm, row_of, status, st));
  MOE_CUDA(launch_scatter_rows(x, row_of, s.T, s.k, s.d, x_perm, num_sms(), st, offsets, shard.e_lo, shard.e_hi));
  // the router picks k distinct experts per token, so no segment exceeds T rows
  r = run_experts(sl, L, ws, x, x_perm, offsets, W1, W3, W2, s1, s3, s2, W1s, W3s, W2s, Y_perm, Y_shared, status, st,
                  shard, ev ? ev + 2 : nullptr, s.T);
  if (r != MOE_OK) return r;
  MOE_CUDA(launch_combine(Y_perm, Y_shared, row_of, w, s.T, s.k, s.d, y, s.y_dtype == MOE_BF16, st,
                          whole ? nullptr : offsets, whole ? nullptr : &shard));
  if (ev) MOE_CUDA(cudaEventRecord(ev[5], st));
  return MOE_OK;
}

// The shared expert alone over the T tokens of x (no routed rows): the tile
// list holds only its tiles, and both grouped GEMMs walk them.
moe_status run_shared_only(const moe_shape& s, const Layout& L, void* ws, const void* x, const void* W1s,
                           const void* W3s, const void* W2s, float* Y_shared, uint32_t* status, cudaStream_t st) {
  int4* tiles = at<int4>(ws, L.tiles);
  int32_t* ntiles = at<int32_t>(ws, L.ntiles);
  int* sched = at<int>(ws, L.sched);
  uint16_t* H = at<uint16_t>(ws, L.H);
  const int64_t Tk = s.T * s.k;
  MOE_CUDA(launch_build_tiles(at<int32_t>(ws, L.offsets), s.E, s.T, Shard{0, 0}, true, tiles, ntiles, sched, st,
                              nullptr));
  const int sms = num_sms();
  CUtensorMap a_s, w1_s, w3_s, h_map, w2_s;
  if (!map_2d(&a_s, x, s.d, s.T, kGemmBK, kTileM) || !map_3d(&w1_s, W1s, s.shared_inter, s.d, 1, kGemmBK) ||
      !map_3d(&w3_s, W3s, s.shared_inter, s.d, 1, kGemmBK) || !map_2d(&h_map, H, L.Hld, L.Hrows, kGemmBK, kTileM) ||
      !map_3d(&w2_s, W2s, s.d, s.shared_inter, 1, kGemmBK))
    return MOE_ERR_CUDA;
  GemmParams p1{};
  p1.tiles = tiles;
  p1.ntiles = ntiles;
  p1.max_mtiles = L.max_mtiles;
  p1.tile_set = kTilesShared;
  p1.E = s.E;
  p1.n_nb = (L.Hld + gemm_block_n_swiglu() - 1) / gemm_block_n_swiglu();
  p1.K_routed = p1.K_shared = s.d;
  p1.N_routed = 0;
  p1.N_shared = s.shared_inter;
  p1.out_routed = p1.out_shared = H;
  p1.out_shared_row_offset = Tk;
  p1.ld_out = L.Hld;
  p1.status = status;
  p1.sched_counter = sched + 1;
  MOE_CUDA(launch_grouped_swiglu(a_s, a_s, w1_s, w1_s, w3_s, w3_s, p1,
                                 (int)std::min<int64_t>(sms, (int64_t)L.max_mtiles * p1.n_nb), st));
  GemmParams p2 = p1;
  p2.sched_counter = sched + 3;
  p2.n_nb = (s.d + gemm_block_n_down() - 1) / gemm_block_n_down();
  p2.K_routed = p2.K_shared = s.shared_inter;
  p2.N_routed = 0;
  p2.N_shared = s.d;
  p2.a_shared_row_offset = (int)Tk;
  p2.out_routed = nullptr;
  p2.out_shared = Y_shared;
  p2.out_shared_row_offset = 0;
  p2.ld_out = s.d;
  MOE_CUDA(launch_grouped_down(h_map, w2_s, w2_s, p2, (int)std::min<int64_t>(sms, (int64_t)L.max_mtiles * p2.n_nb),
                               st));
  return MOE_OK;
}

// ------------------------------------------------------------ backward pass
// Workspace of moe_backward: the forward's layout (routing, dispatch, x_perm,
// H, Y_perm) and the backward's own buffers after it.
struct BwdLayout {
  Layout f;
  size_t tiles, gu, dgu, dO, dy_b, dw, dl, dl_b, wgT, dX, dXs, total;
  int max_mtiles, Ep;
  int64_t rows;  // T*k routed rows + T shared rows of gu / dgu
};

BwdLayout make_bwd_layout(const moe_shape& s) {
  BwdLayout B{};
  B.f = make_layout(s);
  const int64_t T = s.T, Tk = s.T * s.k;
  size_t off = B.f.total;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off += align_up(std::max<size_t>(bytes, 1));
    return at;
  };
  // the shared expert's tiles are always listed: with no shared expert they
  // still carry the router's part of the input gradient (dl Wg)
  B.max_mtiles = (int)((Tk + kTileRows - 1) / kTileRows + s.E + (T + kTileRows - 1) / kTileRows);
  B.Ep = (s.E + 63) / 64 * 64;
  B.rows = Tk + T;
  const int64_t Hld = B.f.Hld;
  B.tiles = take((size_t)B.max_mtiles * 16);
  B.gu = take((size_t)B.rows * 2 * Hld * 2);
  B.dgu = take((size_t)B.rows * 2 * Hld * 2);
  B.dO = take((size_t)Tk * s.d * 2);
  B.dy_b = take((size_t)T * s.d * 2);
  B.dw = take((size_t)Tk * 4);
  B.dl = take((size_t)T * s.E * 4);
  B.dl_b = take((size_t)T * B.Ep * 2);
  B.wgT = take((size_t)s.d * B.Ep * 2);
  B.dX = take((size_t)Tk * s.d * 2);
  B.dXs = take((size_t)T * s.d * 4);
  B.total = off;
  return B;
}

moe_status validate_backward(const moe_shape* s) {
  moe_status v = validate_shape(s);
  if (v != MOE_OK) return v;
  if (s->w_dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;  // bf16 experts only
  return MOE_OK;
}

// bf16 row-major [outer, inner] map with [box_outer rows x 64] boxes
bool map_rows(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_outer) {
  return map_2d(m, ptr, inner, outer, 64, box_outer);
}

// The forward of the training pass: routing, dispatch and both expert GEMMs,
// keeping in the backward workspace what the gradient needs (logits, routing,
// x_perm, g and u in bf16, H, the routed expert outputs Y_perm).  y != nullptr:
// the shared expert's output too, and the combine into y (shape.y_dtype).
moe_status train_forward(const moe_shape& s, const void* x, const void* Wg, const float* bias, const void* W1,
                         const void* W3, const void* W2, const void* W1s, const void* W3s, const void* W2s, void* y,
                         void* ws, cudaStream_t st) {
  const BwdLayout B = make_bwd_layout(s);
  const Layout& L = B.f;
  const bool sh = s.shared_inter > 0;
  const int64_t Tk = s.T * s.k;
  const int Hld = L.Hld;
  const int sms = num_sms();
  uint32_t* status = at<uint32_t>(ws, L.status);
  int32_t* idx = at<int32_t>(ws, L.idx);
  float* w = at<float>(ws, L.w);
  float* logits = at<float>(ws, L.logits);
  int32_t* counts = at<int32_t>(ws, L.counts);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* perm = at<int32_t>(ws, L.perm);
  int32_t* row_of = at<int32_t>(ws, L.row_of);
  void* x_perm = at<void>(ws, L.x_perm);
  uint16_t* H = at<uint16_t>(ws, L.H);
  void* Y_perm = at<void>(ws, L.Y_perm);
  int4* tiles = at<int4>(ws, B.tiles);
  int32_t* ntiles = at<int32_t>(ws, L.ntiles);
  int* sched = at<int>(ws, L.sched);
  void* GU = at<void>(ws, B.gu);

  moe_status r = run_router(s, x, Wg, bias, idx, w, logits, at<double>(ws, L.rpart), status, st);
  if (r != MOE_OK) return r;
  MOE_CUDA(launch_permute(idx, s.T, s.k, s.E, at<int32_t>(ws, L.hist), at<int32_t>(ws, L.base), counts, offsets,
                          perm, row_of, status, st));
  MOE_CUDA(launch_scatter_rows(x, row_of, s.T, s.k, s.d, x_perm, sms, st, offsets, 0, s.E));
  MOE_CUDA(launch_build_tiles(offsets, s.E, s.T, whole_layer(s), true, tiles, ntiles, sched, st, nullptr));

  CUtensorMap a_r, a_s, w1_r, w1_s, w3_r, w3_s;
  if (!map_2d(&a_r, x_perm, s.d, Tk, kGemmBK, kTileM) || !map_2d(&a_s, x, s.d, s.T, kGemmBK, kTileM) ||
      !map_3d(&w1_r, W1, s.inter, s.d, s.E, kGemmBK) || !map_3d(&w3_r, W3, s.inter, s.d, s.E, kGemmBK))
    return MOE_ERR_CUDA;
  if (sh) {
    if (!map_3d(&w1_s, W1s, s.shared_inter, s.d, 1, kGemmBK) || !map_3d(&w3_s, W3s, s.shared_inter, s.d, 1, kGemmBK))
      return MOE_ERR_CUDA;
  } else {
    w1_s = w1_r;  // placeholders: shared tiles have no columns without a shared expert
    w3_s = w3_r;
  }
  GemmParams p1{};
  p1.tiles = tiles;
  p1.ntiles = ntiles;
  p1.max_mtiles = B.max_mtiles;
  p1.tile_set = kTilesAll;
  p1.E = s.E;
  p1.group_base = 0;
  p1.n_nb = (Hld + gemm_block_n_swiglu() - 1) / gemm_block_n_swiglu();
  p1.K_routed = s.d;
  p1.K_shared = s.d;
  p1.N_routed = s.inter;
  p1.N_shared = s.shared_inter;
  p1.out_routed = H;
  p1.out_shared = H;
  p1.out_shared_row_offset = Tk;
  p1.ld_out = Hld;
  p1.status = status;
  p1.sched_counter = sched + 0;
  p1.out_gu = GU;
  const int grid1 = (int)std::min<int64_t>(sms, (int64_t)B.max_mtiles * p1.n_nb);
  MOE_CUDA(launch_grouped_swiglu(a_r, a_s, w1_r, w1_s, w3_r, w3_s, p1, grid1, st));

  CUtensorMap h_map, w2_r, w2_s;
  if (!map_2d(&h_map, H, Hld, L.Hrows, kGemmBK, kTileM) || !map_3d(&w2_r, W2, s.d, s.inter, s.E, kGemmBK))
    return MOE_ERR_CUDA;
  if (sh && y) {
    if (!map_3d(&w2_s, W2s, s.d, s.shared_inter, 1, kGemmBK)) return MOE_ERR_CUDA;
  } else {
    w2_s = w2_r;
  }
  GemmParams p2 = p1;
  p2.out_gu = nullptr;
  // the gradient needs Y_perm only; the shared expert's output only for y
  p2.tile_set = y && sh ? kTilesAll : kTilesRouted;
  p2.sched_counter = sched + 2;
  p2.n_nb = (s.d + gemm_block_n_down() - 1) / gemm_block_n_down();
  p2.K_routed = s.inter;
  p2.K_shared = s.shared_inter;
  p2.N_routed = s.d;
  p2.N_shared = s.d;
  p2.a_shared_row_offset = (int)Tk;
  p2.out_routed = Y_perm;
  p2.out_shared = y && sh ? at<float>(ws, L.Y_shared) : nullptr;
  p2.out_shared_row_offset = 0;
  p2.ld_out = s.d;
  const int grid2 = (int)std::min<int64_t>(sms, (int64_t)B.max_mtiles * p2.n_nb);
  MOE_CUDA(launch_grouped_down(h_map, w2_r, w2_s, p2, grid2, st));
  if (y)
    MOE_CUDA(launch_combine(Y_perm, sh ? at<float>(ws, L.Y_shared) : nullptr, row_of, w, s.T, s.k, s.d, y,
                            s.y_dtype == MOE_BF16, st));
  return MOE_OK;
}


// The gradient from the state train_forward left in the workspace.
moe_status train_backward(const moe_shape& s, const void* x, const void* Wg, const void* W1, const void* W3,
                          const void* W2, const void* W1s, const void* W3s, const void* W2s, const float* dy, void* dx,
                          void* dWg, void* dW1, void* dW3, void* dW2, void* dW1s, void* dW3s, void* dW2s, void* ws,
                          cudaStream_t st) {
  const BwdLayout B = make_bwd_layout(s);
  const Layout& L = B.f;
  const bool sh = s.shared_inter > 0;
  const int64_t T = s.T, Tk = s.T * s.k;
  const int Hld = L.Hld;
  const int sms = num_sms();
  const bool gbf16 = s.y_dtype == MOE_BF16;
  uint32_t* status = at<uint32_t>(ws, L.status);
  int32_t* idx = at<int32_t>(ws, L.idx);
  float* w = at<float>(ws, L.w);
  float* logits = at<float>(ws, L.logits);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* row_of = at<int32_t>(ws, L.row_of);
  void* x_perm = at<void>(ws, L.x_perm);
  uint16_t* H = at<uint16_t>(ws, L.H);
  void* Y_perm = at<void>(ws, L.Y_perm);
  int4* tiles = at<int4>(ws, B.tiles);
  int32_t* ntiles = at<int32_t>(ws, L.ntiles);
  void* GU = at<void>(ws, B.gu);
  void* dGU = at<void>(ws, B.dgu);
  void* dO = at<void>(ws, B.dO);
  void* dy_b = at<void>(ws, B.dy_b);
  float* dw = at<float>(ws, B.dw);
  float* dl = at<float>(ws, B.dl);
  void* dl_b = at<void>(ws, B.dl_b);
  void* wgT = at<void>(ws, B.wgT);
  void* dX = at<void>(ws, B.dX);
  float* dXs = at<float>(ws, B.dXs);

  // ---- combine and routing steps
  MOE_CUDA(launch_combine_backward(dy, Y_perm, row_of, w, s.T, s.k, s.d, dO, dw, st));
  MOE_CUDA(launch_router_backward(logits, idx, w, dw, s.T, s.E, s.k, s.route == MOE_ROUTE_SIGMOID_GROUP ? 1 : 0,
                                  s.route_scale, dl, st));
  MOE_CUDA(launch_cast_pad_bf16(dl, T, s.E, B.Ep, dl_b, sms, st));
  MOE_CUDA(launch_cast_pad_bf16(dy, T, s.d, s.d, dy_b, sms, st));
  MOE_CUDA(launch_transpose_pad_bf16(Wg, s.E, s.d, B.Ep, wgT, st));

  // ---- dH = dO W2^T (routed), dy W2s^T (shared) -> dG | dU
  {
    DgradMaps m{};
    if (!map_rows(&m.a[0], dO, s.d, Tk, kTileM) || !map_rows(&m.a[1], dy_b, s.d, T, kTileM) ||
        !map_3d(&m.b[0], W2, s.d, s.inter, s.E, 256))
      return MOE_ERR_CUDA;
    if (sh) {
      if (!map_3d(&m.b[1], W2s, s.d, s.shared_inter, 1, 256)) return MOE_ERR_CUDA;
    } else {
      m.b[1] = m.b[0];
    }
    m.a[2] = m.a[0];
    m.b[2] = m.b[3] = m.b[4] = m.b[0];
    DgradParams q{};
    q.tiles = tiles;
    q.ntiles = ntiles;
    q.max_mtiles = B.max_mtiles;
    q.E = s.E;
    q.n_nb = (Hld + 255) / 256;
    q.N_routed = s.inter;
    q.N_shared = s.shared_inter;  // 0: the shared tiles are skipped
    q.parts_routed[0] = KPart{s.d / 64, kMapA0, 0, 0, kMapB0};
    q.n_parts_routed = 1;
    q.parts_shared[0] = KPart{s.d / 64, kMapA1, 0, 0, kMapB1};
    q.n_parts_shared = 1;
    q.gu = GU;
    q.ld_gu = 2 * (int64_t)Hld;
    q.u_off = Hld;
    q.shared_row_off = Tk;
    q.out_routed = dGU;
    q.status = status;
    MOE_CUDA(launch_dgrad(kDgradH, m, q, (int)std::min<int64_t>(sms, (int64_t)B.max_mtiles * q.n_nb), st));
  }
  // ---- dX = [dG | dU] [W1 ; W3]^T (routed rows), and for the shared expert's
  // tiles [dGs | dUs] [W1s ; W3s]^T + dl Wg
  {
    DgradMaps m{};
    if (!map_rows(&m.a[0], dGU, 2 * (uint64_t)Hld, B.rows, kTileM) || !map_rows(&m.a[1], dl_b, B.Ep, T, kTileM) ||
        !map_3d(&m.b[0], W1, s.inter, s.d, s.E, 256) || !map_3d(&m.b[1], W3, s.inter, s.d, s.E, 256) ||
        !map_3d(&m.b[4], wgT, B.Ep, s.d, 1, 256))
      return MOE_ERR_CUDA;
    if (sh) {
      if (!map_3d(&m.b[2], W1s, s.shared_inter, s.d, 1, 256) || !map_3d(&m.b[3], W3s, s.shared_inter, s.d, 1, 256))
        return MOE_ERR_CUDA;
    } else {
      m.b[2] = m.b[3] = m.b[0];
    }
    m.a[2] = m.a[0];
    DgradParams q{};
    q.tiles = tiles;
    q.ntiles = ntiles;
    q.max_mtiles = B.max_mtiles;
    q.E = s.E;
    q.n_nb = (s.d + 255) / 256;
    q.N_routed = s.d;
    q.N_shared = s.d;
    q.parts_routed[0] = KPart{s.inter / 64, kMapA0, 0, 0, kMapB0};
    q.parts_routed[1] = KPart{s.inter / 64, kMapA0, Hld, 0, kMapB1};
    q.n_parts_routed = 2;
    int np = 0;
    if (sh) {
      q.parts_shared[np++] = KPart{s.shared_inter / 64, kMapA0, 0, (int)Tk, kMapB2};
      q.parts_shared[np++] = KPart{s.shared_inter / 64, kMapA0, Hld, (int)Tk, kMapB3};
    }
    q.parts_shared[np++] = KPart{B.Ep / 64, kMapA1, 0, 0, kMapB4};
    q.n_parts_shared = np;
    q.out_routed = dX;
    q.out_shared = dXs;
    q.ld_out = s.d;
    q.status = status;
    MOE_CUDA(launch_dgrad(kDgradX, m, q, (int)std::min<int64_t>(sms, (int64_t)B.max_mtiles * q.n_nb), st));
  }
  // ---- dx[t] = sum_j dX[row_of[t, j]] + dX_shared[t] (which holds dl Wg)
  MOE_CUDA(launch_combine(dX, dXs, row_of, nullptr, s.T, s.k, s.d, dx, gbf16, st));

  // ---- weight gradients
  {
    // the routed dG | dU rows and the shared expert's get maps of their own,
    // each ending at its last row: the last MMA slice of a group reads zero
    // fill past it, never another region's rows (whose columns past its own
    // width are not written)
    CUtensorMap ax_r, ax_s, bg_r, bg_s;
    if (!map_rows(&ax_r, x_perm, s.d, Tk, 64) || !map_rows(&ax_s, x, s.d, T, 64) ||
        !map_rows(&bg_r, dGU, 2 * (uint64_t)Hld, Tk, 64))
      return MOE_ERR_CUDA;
    if (sh) {
      const uint16_t* dgu_shared = static_cast<const uint16_t*>(dGU) + Tk * 2 * (int64_t)Hld;
      if (!map_rows(&bg_s, dgu_shared, 2 * (uint64_t)Hld, T, 64)) return MOE_ERR_CUDA;
    } else {
      bg_s = bg_r;
    }
    WgradParams q{};
    q.offsets = offsets;
    q.n_routed = s.E;
    q.has_shared = sh ? 1 : 0;
    q.mb_routed = s.d / 128;
    q.nb_routed = s.inter / 128;
    q.mb_shared = s.d / 128;
    q.nb_shared = s.shared_inter / 128;
    q.M_routed = q.M_shared = s.d;
    q.ncols_routed = s.inter;
    q.ncols_shared = s.shared_inter;
    q.a_shared_row0 = 0;
    q.b_shared_row0 = 0;
    q.shared_rows = s.T;
    q.u_off = Hld;
    q.out1 = dW1;
    q.out2 = dW3;
    q.out1_shared = dW1s;
    q.out2_shared = dW3s;
    q.out_bf16 = gbf16 ? 1 : 0;
    q.status = status;
    WgradOutMaps om{};
    om.m[0] = om.m[1] = om.m[2] = om.m[3] = ax_r;  // placeholders for fp32 gradients (stored directly)
    if (gbf16) {
      if (!map_3d(&om.m[0], dW1, s.inter, s.d, s.E, 128) || !map_3d(&om.m[1], dW3, s.inter, s.d, s.E, 128))
        return MOE_ERR_CUDA;
      if (sh && (!map_3d(&om.m[2], dW1s, s.shared_inter, s.d, 1, 128) ||
                 !map_3d(&om.m[3], dW3s, s.shared_inter, s.d, 1, 128)))
        return MOE_ERR_CUDA;
    }
    MOE_CUDA(launch_wgrad(kWgradW13, ax_r, ax_s, bg_r, bg_s, om, q, sms, st));
  }
  {
    CUtensorMap ah, bo_r, bo_s;
    if (!map_rows(&ah, H, Hld, L.Hrows, 64) || !map_rows(&bo_r, dO, s.d, Tk, 64) ||
        !map_rows(&bo_s, dy_b, s.d, T, 64))
      return MOE_ERR_CUDA;
    WgradParams q{};
    q.offsets = offsets;
    q.n_routed = s.E;
    q.has_shared = sh ? 1 : 0;
    q.mb_routed = s.inter / 128;
    q.nb_routed = (s.d + 255) / 256;
    q.mb_shared = s.shared_inter / 128;
    q.nb_shared = (s.d + 255) / 256;
    q.M_routed = s.inter;
    q.M_shared = s.shared_inter;
    q.ncols_routed = q.ncols_shared = s.d;
    q.a_shared_row0 = (int)Tk;
    q.b_shared_row0 = 0;
    q.shared_rows = s.T;
    q.out1 = dW2;
    q.out1_shared = dW2s;
    q.out_bf16 = gbf16 ? 1 : 0;
    q.status = status;
    WgradOutMaps om{};
    om.m[0] = om.m[1] = om.m[2] = om.m[3] = ah;
    if (gbf16) {
      if (!map_3d(&om.m[0], dW2, s.d, s.inter, s.E, 128)) return MOE_ERR_CUDA;
      if (sh && !map_3d(&om.m[2], dW2s, s.d, s.shared_inter, 1, 128)) return MOE_ERR_CUDA;
    }
    MOE_CUDA(launch_wgrad(kWgradPlain, ah, ah, bo_r, bo_s, om, q, sms, st));
  }
  {
    CUtensorMap al, bx;
    if (!map_rows(&al, dl_b, B.Ep, T, 64) || !map_rows(&bx, x, s.d, T, 64)) return MOE_ERR_CUDA;
    WgradParams q{};
    q.offsets = offsets;
    q.n_routed = 0;
    q.has_shared = 1;
    q.mb_shared = (s.E + 127) / 128;
    q.nb_shared = (s.d + 255) / 256;
    q.M_shared = s.E;
    q.ncols_shared = s.d;
    q.shared_rows = s.T;
    q.out1_shared = dWg;
    q.out_bf16 = gbf16 ? 1 : 0;
    q.status = status;
    WgradOutMaps om{};
    om.m[0] = om.m[1] = om.m[2] = om.m[3] = al;
    if (gbf16 && !map_3d(&om.m[2], dWg, s.d, s.E, 1, 128)) return MOE_ERR_CUDA;
    MOE_CUDA(launch_wgrad(kWgradPlain, al, al, bx, bx, om, q, sms, st));
  }
  return MOE_OK;
}

moe_status backward_impl(const moe_shape& s, const void* x, const void* Wg, const float* bias, const void* W1,
                         const void* W3, const void* W2, const void* W1s, const void* W3s, const void* W2s,
                         const float* dy, void* dx, void* dWg, void* dW1, void* dW3, void* dW2, void* dW1s, void* dW3s,
                         void* dW2s, void* ws, cudaStream_t st) {
  moe_status r = train_forward(s, x, Wg, bias, W1, W3, W2, W1s, W3s, W2s, nullptr, ws, st);
  if (r != MOE_OK) return r;
  return train_backward(s, x, Wg, W1, W3, W2, W1s, W3s, W2s, dy, dx, dWg, dW1, dW3, dW2, dW1s, dW3s, dW2s, ws, st);
}

// Arguments of the training calls (moe_backward, moe_forward_train,
// moe_backward_saved): bf16 experts, the pointers each needs, alignment and
// workspace.
moe_status check_train_args(const moe_shape* shape, const void* const* need, int n_need, const void* const* opt,
                            int n_opt, const void* ws, size_t ws_bytes) {
  moe_status v = validate_backward(shape);
  if (v != MOE_OK) return v;
  for (int i = 0; i < n_need; ++i)
    if (!need[i] || !aligned16(need[i])) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < n_opt; ++i)
    if (opt[i] && !aligned16(opt[i])) return MOE_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, make_bwd_layout(*shape).total)) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

// Every weight gradient of an empty batch is zero.
moe_status zero_weight_grads(const moe_shape& s, void* dWg, void* dW1, void* dW3, void* dW2, void* dW1s, void* dW3s,
                             void* dW2s, cudaStream_t st) {
  const size_t gb = s.y_dtype == MOE_BF16 ? 2 : 4;
  const size_t eI = (size_t)s.E * s.d * s.inter * gb, sI = (size_t)s.d * s.shared_inter * gb;
  MOE_CUDA(cudaMemsetAsync(dWg, 0, (size_t)s.E * s.d * gb, st));
  MOE_CUDA(cudaMemsetAsync(dW1, 0, eI, st));
  MOE_CUDA(cudaMemsetAsync(dW3, 0, eI, st));
  MOE_CUDA(cudaMemsetAsync(dW2, 0, eI, st));
  if (s.shared_inter > 0) {
    MOE_CUDA(cudaMemsetAsync(dW1s, 0, sI, st));
    MOE_CUDA(cudaMemsetAsync(dW3s, 0, sI, st));
    MOE_CUDA(cudaMemsetAsync(dW2s, 0, sI, st));
  }
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_workspace_size(const moe_shape* shape) {
  if (validate_shape(shape) != MOE_OK) return 0;
  return make_layout(*shape).total;
}

moe_status moe_router_topk(const moe_shape* shape, const void* x, const void* Wg, const float* bias,
                           int32_t* topk_idx, float* topk_w, float* logits, void* ws, size_t ws_bytes,
                           void* stream) {
  moe_status v = validate_shape(shape);
  if (v != MOE_OK) return v;
  const moe_shape& s = *shape;
  if (!x || !Wg || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(Wg) || !aligned16(topk_idx) || !aligned16(topk_w) ||
      (logits && !aligned16(logits)) || (bias && !aligned16(bias)))
    return MOE_ERR_INVALID_ARG;
  const Layout L = make_layout(s);
  if (!ws_ok(ws, ws_bytes, L.total)) return MOE_ERR_WORKSPACE;
  if (s.T == 0) return MOE_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* status = at<uint32_t>(ws, L.status);
  MOE_CUDA(cudaMemsetAsync(status, 0, 4, st));
  return run_router(s, x, Wg, bias, topk_idx, topk_w, logits ? logits : at<float>(ws, L.logits),
                    at<double>(ws, L.rpart), status, st);
}

moe_status moe_router_topk_limited(const moe_shape* shape, const void* x, const void* Wg, const uint8_t* allowed,
                                   int32_t* topk_idx, float* topk_w, float* logits, void* ws, size_t ws_bytes,
                                   void* stream) {
  moe_status v = validate_shape(shape);
  if (v != MOE_OK) return v;
  const moe_shape& s = *shape;
  if (s.route != MOE_ROUTE_TOPK_SOFTMAX) return MOE_ERR_UNSUPPORTED;
  if (!x || !Wg || !allowed || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(Wg) || !aligned16(topk_idx) || !aligned16(topk_w) ||
      (logits && !aligned16(logits)))
    return MOE_ERR_INVALID_ARG;
  const Layout L = make_layout(s);
  if (!ws_ok(ws, ws_bytes, L.total)) return MOE_ERR_WORKSPACE;
  if (s.T == 0) return MOE_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* status = at<uint32_t>(ws, L.status);
  MOE_CUDA(cudaMemsetAsync(status, 0, 4, st));
  return run_router(s, x, Wg, nullptr, topk_idx, topk_w, logits ? logits : at<float>(ws, L.logits),
                    at<double>(ws, L.rpart), status, st, allowed);
}

moe_status moe_expert_utilisation(const moe_shape* shape, const int32_t* counts, float* utilisation, int32_t* flags,
                                  void* stream) {
  moe_status v = validate_shape(shape);
  if (v != MOE_OK) return v;
  if (!counts || (!utilisation && !flags)) return MOE_ERR_INVALID_ARG;
  MOE_CUDA(launch_expert_utilisation(counts, shape->E, utilisation, flags, static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_permute(const moe_shape* shape, const int32_t* topk_idx, int32_t* counts, int32_t* offsets,
                       int32_t* perm_token, int32_t* row_of, const void* x, void* x_perm, void* ws,
                       size_t ws_bytes, void* stream) {
  moe_status v = validate_shape(shape);
  if (v != MOE_OK) return v;
  const moe_shape& s = *shape;
  if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
  // an empty batch writes counts and offsets only: its [T*k] arrays may be NULL
  if (s.T > 0 && (!topk_idx || !perm_token || !row_of)) return MOE_ERR_INVALID_ARG;
  if (s.T > 0 && (x == nullptr) != (x_perm == nullptr)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(topk_idx) || !aligned16(counts) || !aligned16(offsets) || !aligned16(perm_token) ||
      !aligned16(row_of) || (x && !aligned16(x)) || (x_perm && !aligned16(x_perm)))
    return MOE_ERR_INVALID_ARG;
  const Layout L = make_layout(s);
  if (!ws_ok(ws, ws_bytes, L.total)) return MOE_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* status = at<uint32_t>(ws, L.status);
  MOE_CUDA(cudaMemsetAsync(status, 0, 4, st));
  if (s.T == 0) {
    MOE_CUDA(cudaMemsetAsync(counts, 0, (size_t)s.E * 4, st));
    MOE_CUDA(cudaMemsetAsync(offsets, 0, (size_t)(s.E + 1) * 4, st));
    return MOE_OK;
  }
  MOE_CUDA(launch_permute(topk_idx, s.T, s.k, s.E, at<int32_t>(ws, L.hist), at<int32_t>(ws, L.base), counts, offsets,
                          perm_token, row_of, status, st));
  // only the rows the scatter wrote: entries with an out-of-range index are
  // skipped (row_of = -1), so offsets[E] <= T*k rows are filled
  if (x) MOE_CUDA(launch_scatter_rows(x, row_of, s.T, s.k, s.d, x_perm, num_sms(), st, offsets, 0, s.E));
  return MOE_OK;
}

moe_status moe_grouped_swiglu(const moe_shape* shape, const void* x, const void* x_perm, const int32_t* offsets,
                              const void* W1, const void* W3, const void* W2, const float* s1, const float* s3,
                              const float* s2, const void* W1s, const void* W3s, const void* W2s, void* Y_perm,
                              float* Y_shared, void* ws, size_t ws_bytes, void* stream) {
  moe_status v = validate_shape(shape);
  if (v != MOE_OK) return v;
  const moe_shape& s = *shape;
  const bool sh = s.shared_inter > 0;
  if (!x || !x_perm || !offsets || !W1 || !W3 || !W2 || !Y_perm) return MOE_ERR_INVALID_ARG;
  if (sh && (!W1s || !W3s || !W2s || !Y_shared)) return MOE_ERR_INVALID_ARG;
  if (s.w_dtype == MOE_E4M3 && (!s1 || !s3 || !s2)) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {x, x_perm, offsets, W1, W3, W2, s1, s3, s2, W1s, W3s, W2s, Y_perm, Y_shared};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
  const Layout L = make_layout(s);
  if (!ws_ok(ws, ws_bytes, L.total)) return MOE_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* status = at<uint32_t>(ws, L.status);
  MOE_CUDA(cudaMemsetAsync(status, 0, 4, st));
  if (s.T == 0) return MOE_OK;
  // caller-given offsets: segments are bounded only by the T*k rows
  return run_experts(s, L, ws, x, x_perm, offsets, W1, W3, W2, s1, s3, s2, W1s, W3s, W2s, Y_perm,
                     sh ? Y_shared : nullptr, status, st, whole_layer(s), nullptr, s.T * s.k);
}

moe_status moe_combine(const moe_shape* shape, const void* Y_perm, const float* Y_shared, const int32_t* row_of,
                       const float* topk_w, void* y, void* stream) {
  moe_status v = validate_shape(shape);
  if (v != MOE_OK) return v;
  const moe_shape& s = *shape;
  if (!Y_perm || !row_of || !topk_w || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned16(Y_perm) || !aligned16(row_of) || !aligned16(topk_w) || !aligned16(y) ||
      (Y_shared && !aligned16(Y_shared)))
    return MOE_ERR_INVALID_ARG;
  if (s.T == 0) return MOE_OK;
  MOE_CUDA(launch_combine(Y_perm, Y_shared, row_of, topk_w, s.T, s.k, s.d, y, s.y_dtype == MOE_BF16,
                          static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_combine_backward(const moe_shape* shape, const float* dy, const void* Y_perm, const int32_t* row_of,
                                const float* topk_w, void* dO_perm, float* dw, void* stream) {
  moe_status v = validate_shape(shape);
  if (v != MOE_OK) return v;
  const moe_shape& s = *shape;
  if (!dy || !Y_perm || !row_of || !topk_w || !dO_perm || !dw) return MOE_ERR_INVALID_ARG;
  if (!aligned16(dy) || !aligned16(Y_perm) || !aligned16(row_of) || !aligned16(topk_w) || !aligned16(dO_perm) ||
      !aligned16(dw))
    return MOE_ERR_INVALID_ARG;
  if (s.T == 0) return MOE_OK;
  MOE_CUDA(launch_combine_backward(dy, Y_perm, row_of, topk_w, s.T, s.k, s.d, dO_perm, dw,
                                   static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_router_backward(const moe_shape* shape, const float* logits, const int32_t* topk_idx,
                               const float* topk_w, const float* dw, float* dlogits, void* stream) {
  moe_status v = validate_shape(shape);
  if (v != MOE_OK) return v;
  const moe_shape& s = *shape;
  if (!logits || !topk_idx || !topk_w || !dw || !dlogits) return MOE_ERR_INVALID_ARG;
  if (!aligned16(logits) || !aligned16(topk_idx) || !aligned16(topk_w) || !aligned16(dw) || !aligned16(dlogits))
    return MOE_ERR_INVALID_ARG;
  if (s.T == 0) return MOE_OK;
  MOE_CUDA(launch_router_backward(logits, topk_idx, topk_w, dw, s.T, s.E, s.k,
                                  s.route == MOE_ROUTE_SIGMOID_GROUP ? 1 : 0, s.route_scale, dlogits,
                                  static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_forward(const moe_shape* shape, const void* x, const void* Wg, const float* bias, const void* W1,
                       const void* W3, const void* W2, const float* s1, const float* s3, const float* s2,
                       const void* W1s, const void* W3s, const void* W2s, void* y, int32_t* topk_idx_out,
                       float* topk_w_out, int32_t* counts_out, void* ws, size_t ws_bytes, void* stream) {
  return forward_impl(shape, x, Wg, bias, W1, W3, W2, s1, s3, s2, W1s, W3s, W2s, y, topk_idx_out, topk_w_out,
                      counts_out, ws, ws_bytes, stream, nullptr);
}

moe_status moe_forward_profiled(const moe_shape* shape, const void* x, const void* Wg, const float* bias,
                                const void* W1, const void* W3, const void* W2, const float* s1, const float* s3,
                                const float* s2, const void* W1s, const void* W3s, const void* W2s, void* y,
                                int32_t* topk_idx_out, float* topk_w_out, int32_t* counts_out, void* ws,
                                size_t ws_bytes, void* stream, void* const* stage_events) {
  if (!stage_events) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < MOE_NUM_STAGE_EVENTS; ++i)
    if (!stage_events[i]) return MOE_ERR_INVALID_ARG;
  return forward_impl(shape, x, Wg, bias, W1, W3, W2, s1, s3, s2, W1s, W3s, W2s, y, topk_idx_out, topk_w_out,
                      counts_out, ws, ws_bytes, stream, reinterpret_cast<const cudaEvent_t*>(stage_events));
}

int moe_forward_launches(const moe_shape* shape) {
  if (validate_shape(shape) != MOE_OK) return -1;
  const moe_shape& s = *shape;
  if (s.T == 0) return 0;
  const int splits = router_splits(s.T, s.d, s.E, std::min(num_sms(), kRouterMaxSms));
  // per grouped GEMM: the routed tiles (CTA-pair launch + one-CTA launch with
  // pairs), and with FP8 experts the bf16 shared expert's launches as well
  const bool pair = use_pair_tiles(s);
  int gemm_launches = pair ? 2 : 1;
  if (s.w_dtype == MOE_E4M3 && s.shared_inter > 0) gemm_launches += pair ? 2 : 1;
  // router (+ split sum) + top-k, hist + scan + scatter, gather, tile list, two grouped GEMMs, combine
  return 1 + (splits > 1 ? 1 : 0) + 1 + 3 + 1 + 1 + 2 * gemm_launches + 1;
}

moe_status moe_forward_ep(const moe_shape* shape, int ep_rank, int ep_size, const void* x, const void* Wg,
                          const float* bias, const void* W1, const void* W3, const void* W2, const float* s1,
                          const float* s3, const float* s2, const void* W1s, const void* W3s, const void* W2s, void* y,
                          int32_t* topk_idx_out, float* topk_w_out, int32_t* counts_out, void* ws, size_t ws_bytes,
                          void* stream) {
  return forward_impl(shape, x, Wg, bias, W1, W3, W2, s1, s3, s2, W1s, W3s, W2s, y, topk_idx_out, topk_w_out,
                      counts_out, ws, ws_bytes, stream, nullptr, ep_rank, ep_size);
}

moe_status moe_shared_expert(const moe_shape* shape, const void* x, const void* W1s, const void* W3s,
                             const void* W2s, float* Y_shared, void* ws, size_t ws_bytes, void* stream) {
  moe_status v = validate_shape(shape);
  if (v != MOE_OK) return v;
  const moe_shape& s = *shape;
  if (s.shared_inter <= 0) return MOE_ERR_INVALID_ARG;
  if (!x || !W1s || !W3s || !W2s || !Y_shared) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {x, W1s, W3s, W2s, Y_shared};
  for (const void* p : ptrs)
    if (!aligned16(p)) return MOE_ERR_INVALID_ARG;
  const Layout L = make_layout(s);
  if (!ws_ok(ws, ws_bytes, L.total)) return MOE_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* status = at<uint32_t>(ws, L.status);
  MOE_CUDA(cudaMemsetAsync(status, 0, 4, st));
  if (s.T == 0) return MOE_OK;
  return run_shared_only(s, L, ws, x, W1s, W3s, W2s, Y_shared, status, st);
}

moe_status moe_ep_regroup_layout(int n_src, int E_local, const int32_t* recv_counts, int32_t* offsets_local,
                                 int32_t* to_expert_major, int32_t* to_source_major, void* stream) {
  if (n_src < 1 || E_local < 1 || (int64_t)n_src * E_local > 1024) return MOE_ERR_INVALID_ARG;
  if (!recv_counts || !offsets_local || !to_expert_major || !to_source_major) return MOE_ERR_INVALID_ARG;
  if (!aligned16(recv_counts) || !aligned16(offsets_local) || !aligned16(to_expert_major) ||
      !aligned16(to_source_major))
    return MOE_ERR_INVALID_ARG;
  MOE_CUDA(launch_ep_regroup(recv_counts, n_src, E_local, offsets_local, to_expert_major, to_source_major,
                             static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_gather_rows(const void* src, const int32_t* index, int64_t rows, int d, void* dst, void* stream) {
  if (rows < 0 || d <= 0 || d % 8 != 0) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (!src || !index || !dst || !aligned16(src) || !aligned16(index) || !aligned16(dst)) return MOE_ERR_INVALID_ARG;
  MOE_CUDA(launch_gather_rows(src, index, rows, d, dst, num_sms(), static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

size_t moe_backward_workspace_size(const moe_shape* shape) {
  if (validate_backward(shape) != MOE_OK) return 0;
  return make_bwd_layout(*shape).total;
}

moe_status moe_forward_train(const moe_shape* shape, const void* x, const void* Wg, const float* bias,
                                        const void* W1, const void* W3, const void* W2, const void* W1s,
                                        const void* W3s, const void* W2s, void* y, void* ws, size_t ws_bytes,
                                        void* stream) {
  if (!shape) return MOE_ERR_INVALID_ARG;
  const bool sh = shape->shared_inter > 0;
  const void* need[] = {x, Wg, W1, W3, W2, y, sh ? W1s : x, sh ? W3s : x, sh ? W2s : x};
  const void* opt[] = {bias};
  moe_status v = check_train_args(shape, need, 9, opt, 1, ws, ws_bytes);
  if (v != MOE_OK) return v;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MOE_CUDA(cudaMemsetAsync(at<uint32_t>(ws, make_bwd_layout(*shape).f.status), 0, 4, st));
  if (shape->T == 0) return MOE_OK;
  return train_forward(*shape, x, Wg, bias, W1, W3, W2, W1s, W3s, W2s, y, ws, st);
}

moe_status moe_backward_saved(const moe_shape* shape, const void* x, const void* Wg, const void* W1,
                                         const void* W3, const void* W2, const void* W1s, const void* W3s,
                                         const void* W2s, const float* dy, void* dx, void* dWg, void* dW1, void* dW3,
                                         void* dW2, void* dW1s, void* dW3s, void* dW2s, void* ws, size_t ws_bytes,
                                         void* stream) {
  if (!shape) return MOE_ERR_INVALID_ARG;
  const bool sh = shape->shared_inter > 0;
  const void* need[] = {x, Wg, W1, W3, W2, dy, dx, dWg, dW1, dW3, dW2, sh ? W1s : x, sh ? W3s : x, sh ? W2s : x,
                        sh ? dW1s : x, sh ? dW3s : x, sh ? dW2s : x};
  moe_status v = check_train_args(shape, need, 17, nullptr, 0, ws, ws_bytes);
  if (v != MOE_OK) return v;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the status word keeps what moe_forward_train raised
  if (shape->T == 0) return zero_weight_grads(*shape, dWg, dW1, dW3, dW2, dW1s, dW3s, dW2s, st);
  return train_backward(*shape, x, Wg, W1, W3, W2, W1s, W3s, W2s, dy, dx, dWg, dW1, dW3, dW2, dW1s, dW3s, dW2s, ws,
                        st);
}

moe_status moe_backward(const moe_shape* shape, const void* x, const void* Wg, const float* bias, const void* W1,
                        const void* W3, const void* W2, const void* W1s, const void* W3s, const void* W2s,
                        const float* dy, void* dx, void* dWg, void* dW1, void* dW3, void* dW2, void* dW1s, void* dW3s,
                        void* dW2s, void* ws, size_t ws_bytes, void* stream) {
  moe_status v = validate_backward(shape);
  if (v != MOE_OK) return v;
  const moe_shape& s = *shape;
  const bool sh = s.shared_inter > 0;
  if (!x || !Wg || !W1 || !W3 || !W2 || !dy || !dx || !dWg || !dW1 || !dW3 || !dW2) return MOE_ERR_INVALID_ARG;
  if (sh && (!W1s || !W3s || !W2s || !dW1s || !dW3s || !dW2s)) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {x, Wg, bias, W1, W3, W2, W1s, W3s, W2s, dy, dx, dWg, dW1, dW3, dW2, dW1s, dW3s, dW2s};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
  const BwdLayout B = make_bwd_layout(s);
  if (!ws_ok(ws, ws_bytes, B.total)) return MOE_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MOE_CUDA(cudaMemsetAsync(at<uint32_t>(ws, B.f.status), 0, 4, st));
  if (s.T == 0) return zero_weight_grads(s, dWg, dW1, dW3, dW2, dW1s, dW3s, dW2s, st);  // no tokens
  return backward_impl(s, x, Wg, bias, W1, W3, W2, W1s, W3s, W2s, dy, dx, dWg, dW1, dW3, dW2, dW1s, dW3s, dW2s, ws,
                       st);
}

moe_status moe_check_device_status(const void* ws, void* stream, uint32_t* raw) {
  if (!ws) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpy(&v, ws, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (raw) *raw = v;
  if (v & kStatusTimeout) return MOE_ERR_DEVICE_TIMEOUT;
  if (v & kStatusBounds) return MOE_ERR_DEVICE_BOUNDS;
  return MOE_OK;
}

const char* moe_status_string(moe_status status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case MOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case MOE_ERR_CUDA: return "CUDA call or kernel launch failed";
    case MOE_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait timed out";
    case MOE_ERR_DEVICE_BOUNDS: return "expert index out of range (skipped)";
  }
  return "unknown status";
}

const char* moe_version(void) { return "moe-b200 0.1 (sm_100a)"; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free dispatch (moe_permute_noalloc).
//
// Some callers cannot allocate device memory at all: a plugin running inside
// another runtime that hands it only its input and output buffers, or an
// embedding whose allocator is owned elsewhere.  For them the dispatch step
// keeps its scratch (the per-block histograms and bases, and a status word) in
// this file-scope device array instead of a caller workspace.  Every GPU that
// loads the library holds the array (512 KiB) until the process exits.
//
// In host code `g_noalloc_scratch` names a host-side stand-in, not a device
// address, so its device address is fetched with cudaGetSymbolAddress in the
// caller's current context (the current device's) and passed to the kernels.
// ---------------------------------------------------------------------------
namespace moe {
namespace {

constexpr int64_t kNoallocScratchInts = 1 << 17;  // 512 KiB of int32
constexpr int64_t kNoallocStatusInts = 64;        // status word, padded to 256 bytes

static __device__ __align__(256) int32_t g_noalloc_scratch[kNoallocScratchInts];

// Device address of the static scratch in the calling thread's current
// context.  A __device__ array has one copy per context that loads this
// library's device code (the primary context of each device, and any context
// a host runtime creates itself), and a context destroyed by cudaDeviceReset
// takes its copy with it, so the address is looked up on every call rather
// than cached.  The lookup allocates nothing; in a context where the library's
// device code is not loaded yet (lazy module loading) it loads it first.
moe_status noalloc_scratch(int32_t** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
  *out = static_cast<int32_t*>(p);
  return MOE_OK;
}

int64_t round64(int64_t v) { return (v + 63) / 64 * 64; }

}  // namespace
}  // namespace moe

extern "C" moe_status moe_permute_noalloc(const moe_shape* shape, const int32_t* topk_idx, int32_t* counts,
                                          int32_t* offsets, int32_t* perm_token, int32_t* row_of, const void* x,
                                          void* x_perm, void* stream) {
  moe_status v = validate_shape(shape);
  if (v != MOE_OK) return v;
  const moe_shape& s = *shape;
  if (!counts || !offsets) return MOE_ERR_INVALID_ARG;
  // an empty batch writes counts and offsets only: its [T*k] arrays may be NULL
  if (s.T > 0 && (!topk_idx || !perm_token || !row_of)) return MOE_ERR_INVALID_ARG;
  if (s.T > 0 && (x == nullptr) != (x_perm == nullptr)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(topk_idx) || !aligned16(counts) || !aligned16(offsets) || !aligned16(perm_token) ||
      !aligned16(row_of) || (x && !aligned16(x)) || (x_perm && !aligned16(x_perm)))
    return MOE_ERR_INVALID_ARG;
  const int64_t per = round64((int64_t)permute_blocks(s.T) * s.E);  // histogram (and base) entries
  if (kNoallocStatusInts + 2 * per > kNoallocScratchInts) return MOE_ERR_UNSUPPORTED;
  int32_t* scratch = nullptr;
  moe_status r = noalloc_scratch(&scratch);
  if (r != MOE_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* status = reinterpret_cast<uint32_t*>(scratch);
  // the array keeps the previous call's contents: the status word must start
  // at zero; the histograms and bases are fully rewritten by the kernels
  MOE_CUDA(cudaMemsetAsync(status, 0, 4, st));
  if (s.T == 0) {
    MOE_CUDA(cudaMemsetAsync(counts, 0, (size_t)s.E * 4, st));
    MOE_CUDA(cudaMemsetAsync(offsets, 0, (size_t)(s.E + 1) * 4, st));
    return MOE_OK;
  }
  int32_t* hist = scratch + kNoallocStatusInts;
  int32_t* base = hist + per;
  MOE_CUDA(launch_permute(topk_idx, s.T, s.k, s.E, hist, base, counts, offsets, perm_token, row_of, status, st));
  // only the rows the scatter wrote: entries with an out-of-range index are
  // skipped (row_of = -1), so offsets[E] <= T*k rows are filled
  if (x) MOE_CUDA(launch_scatter_rows(x, row_of, s.T, s.k, s.d, x_perm, num_sms(), st, offsets, 0, s.E));
  return MOE_OK;
}
