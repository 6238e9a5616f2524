// grouped_gemm.cu -- the expert contractions on the 5th-generation tensor cores.
//
// SwiGLU expert ("DeepSeek-V3.2-Exp / Mixture of experts / Shared expert",
// "All 5 steps"): g = x W1, u = x W3, a = g sigmoid(g), h = a * u, y = h W2.
// The page's code applies silu and the product in fp32 and casts h to the
// activation dtype before W2 (the expert forward block of its "Code" section); h is stored bf16.
//
// Both kernels are persistent (one CTA per SM) and walk a device-side tile
// list: one entry per 256-row slice of an expert's segment of permuted rows,
// plus the shared expert (group E) over all T tokens.  Tile t -> (row tile
// t / n_nb, column block t % n_nb).  A tile is one or two 128-row halves that
// share every weight stage loaded into shared memory, so each weight byte
// crosses HBM once for up to 256 rows (an expert's segment at V3 prefill
// shapes is about 128 +- 11 rows); a half with no rows is never computed.
// Warp roles:
//   warp 0    TMA producer: A halves [128 rows x 64 K] (K-major, 128B
//             swizzle) and B tiles as [64 K x 64 N] boxes (N-major, 128B
//             swizzle: the weights' natural [K, N] row-major layout) into a
//             3-stage ring (the K depth and stage count are build-time knobs,
//             MOE_GEMM_BK / MOE_GEMM_STAGES; 64 x 3 measured fastest);
//   warp 1    single-thread tcgen05.mma issuer, M=128 (a half of at most
//             64 rows: transposed, the weights as an M=128 operand and the
//             rows as an N=16-64 operand; M=64 with FP8 weights), K=16 per
//             instruction, fp32 accumulators in
//             TMEM: two 256-column slots handed out round-robin (a one-half
//             tile takes one, a two-half tile both), so one-half tiles overlap
//             their epilogue with the next main loop;
//   warps 2-9 epilogue (2-5 with FP8 weights): tcgen05.ld the accumulator
//             rows (one row per thread, two warps per TMEM lane quarter each
//             taking half of the columns; bf16: the whole share is read before
//             the slot is released), apply silu(g)*u (SwiGLU kernel) and store;
//   warps 6-13 (FP8 weights only) converters: the producer brings raw e4m3
//             weight tiles [64 K x 128 N] into the stage; these warps turn
//             them into bf16 (code * the tile's 128 x 128 block scale) in the
//             swizzled N-major layout the MMA reads, through a 2-deep ring.
//             The tensor cores take A and B of one type and the activations
//             stay bf16, so the weights are widened in shared memory and the
//             MMA runs kind::f16.  When no tile can hold more than one half
//             (batches of at most 128 tokens) the FP8 stages hold one A half,
//             and the rings are 4 raw + 3 converted stages deep; at most 64
//             rows (64 tokens): a 64-row A box and 5 + 3 stages.
//
// Kernel A (SwiGLU):  N = 128 columns of W1 and the same 128 of W3 per tile,
//                     one N=256 MMA per K step over [W1 | W3] (g and u side by
//                     side in the accumulator), H[row, n0:n0+128] =
//                     bf16(silu(g) * u).
// Kernel B (down):    N = 256 columns of W2 per tile; routed rows are stored
//                     bf16 into Y_perm, shared-expert rows fp32 into Y_shared.
//
// Long segments (the Zipf-skewed workload) also use the CTA-pair kernels at
// the end of this file: full 256-row tiles and last tiles of more than 192
// rows run on 2-CTA clusters with tcgen05.mma.cta_group::2 (M=256), so each
// weight byte is read from shared memory once per 256 rows.
#include <algorithm>
#include <cstdint>

#include "common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kBK = kGemmBK;
constexpr int kStages = kGemmStages;
constexpr uint32_t kABytes = kTileM * kBK * 2;  // one 128-row half of the A tile
constexpr uint32_t kBoxBytes = 64 * kBK * 2;    // one [kBK K x 64 N] bf16 box
constexpr uint32_t kBBytes = 4 * kBoxBytes;     // bf16 B part of a stage
constexpr uint32_t kStageBytes = 2 * kABytes + kBBytes;
// A halves: K-major rows of kBK bf16 (64 or 128 bytes), swizzled to match
// the tensor map; 8-row groups kBK*16 bytes apart.
constexpr uint32_t kASwizzle = kBK == 64 ? ptx::kSwizzle128B : ptx::kSwizzle64B;
constexpr uint32_t kASBO = 8 * kBK * 2;
constexpr uint32_t kTmemCols = 512;  // two 256-column accumulator slots
constexpr uint32_t kSlotCols = 256;

// FP8 weights: a stage holds the A halves and two raw e4m3 boxes
// [64 K x 128 N] (16 KB); converted bf16 B tiles live in their own ring.
constexpr int kF8BK = 64;
constexpr int kF8Stages = 3;
constexpr int kF8ConvStages = 2;
constexpr uint32_t kF8ABytes = kTileM * kF8BK * 2;      // 16 KB
constexpr uint32_t kF8RawBox = 64 * 128;                // 8 KB of codes
constexpr uint32_t kF8StageBytes = 2 * kF8ABytes + 2 * kF8RawBox;
constexpr uint32_t kF8BoxBytes = 64 * kF8BK * 2;        // bf16 [64 K x 64 N] box, 8 KB
constexpr uint32_t kF8ConvBytes = 4 * kF8BoxBytes;      // 32 KB
constexpr int kConvWarps = 8;
constexpr int kSchedDepth = 4;  // tile indices the producer may publish ahead

// FP8 weights at small batches (every routed tile one 128-row half, which
// the host knows when T <= 128): a stage holds one A half and the raw codes,
// so deeper rings fit -- each raw stage is held through the HBM latency and
// the widening, each converted buffer until its MMAs complete, and at such
// batches no MMA work hides them.  4 raw + 3 converted stages measured best
// (of 5 + 2, 4 + 3, 3 + 4, 2 + 5 in the same 224 KB).
constexpr int kF8NStages = 4;
constexpr int kF8NConvStages = 3;
constexpr uint32_t kF8NStageBytes = kF8ABytes + 2 * kF8RawBox;  // 32 KB
// ... and when no tile can hold more than 64 rows (batches of at most 64
// tokens) the A box is 64 rows, the stage 24 KB, and the ring 5 deep
#ifndef MOE_F8N2_STAGES
#define MOE_F8N2_STAGES 5
#endif
constexpr int kF8N2Stages = MOE_F8N2_STAGES;
constexpr uint32_t kF8N2ABytes = kF8ABytes / 2;
constexpr uint32_t kF8N2StageBytes = kF8N2ABytes + 2 * kF8RawBox;  // 24 KB

static_assert(kStages * kStageBytes + 1024 + 256 <= 232448, "shared memory budget");
static_assert(kF8Stages * kF8StageBytes + kF8ConvStages * kF8ConvBytes + 1024 + 256 <= 232448,
              "shared memory budget (FP8)");
static_assert(kF8NStages * kF8NStageBytes + kF8NConvStages * kF8ConvBytes + 1024 + 256 <= 232448,
              "shared memory budget (FP8, one-half stages)");
static_assert(kF8N2Stages * kF8N2StageBytes + kF8NConvStages * kF8ConvBytes + 1024 + 256 <= 232448,
              "shared memory budget (FP8, 64-row stages)");
static_assert(kF8N2StageBytes % 1024 == 0, "64-row stages keep the 1024-byte alignment of the A boxes");

enum class Mode { kSwiGLU, kDown };

template <Mode M>
struct Cfg;
template <>
struct Cfg<Mode::kSwiGLU> {
  static constexpr int BN = 128;  // columns of W1 (and the same columns of W3) per tile
};
template <>
struct Cfg<Mode::kDown> {
  static constexpr int BN = 256;  // columns of W2 per tile
};

// N1 (FP8 only): 0 the general layout, 1 stages of one 128-row A half,
// 2 stages of one 64-row A box
template <bool F8, int N1 = 0>
constexpr size_t smem_bytes() {
  return F8 ? 1024 + (N1 == 2 ? kF8N2Stages * kF8N2StageBytes + kF8NConvStages * kF8ConvBytes
                     : N1 ? kF8NStages * kF8NStageBytes + kF8NConvStages * kF8ConvBytes
                         : kF8Stages * kF8StageBytes + kF8ConvStages * kF8ConvBytes) +
                  256
            : 1024 + kStages * kStageBytes + 256;
}

struct TileInfo {
  int group, row0, rows, nb, halves, k_routed;
  int seg_tiles;  // row tiles of the group's segment (its weights are read once per row tile)
  bool shared;
};

// A half with at most 64 rows runs as an M=64 MMA (half the tensor work of
// M=128).  Its accumulator holds row 16q + i in TMEM lane 32q + i (i < 16) of
// the slot: the half-subpartition layout of the 64-row tcgen05.mma.
__device__ __forceinline__ bool narrow_half(const TileInfo& ti, int h) { return ti.rows - h * kTileM <= kTileM / 2; }

// With bf16 weights a half of at most 64 rows is computed transposed instead:
// D^T = W^T x^T, the weight tile (already in shared memory as MN-major boxes)
// as the M=128 operand and the half's rows (its K-major A box) as an N operand
// of the rows rounded up to 16.  Per K=16 slice that is two M=128 MMAs of N
// 16-64 (one per 128 output columns) instead of one M=64 N=256 MMA: about an
// eighth of the tensor work for the 1-16 rows of a prefill segment's tail or a
// decode segment.  D^T sits in the half's slot: lane = output column, columns
// [0, N) for output columns 0-127 of the tile and [128, 128 + N) for 128-255.
__device__ __forceinline__ int transposed_cols(const TileInfo& ti, int h) {
  return ((ti.rows - h * kTileM + 15) / 16) * 16;
}

// With FP8 weights the narrow half stays an M=64 MMA: the converted B buffer
// has the bf16 boxes' layout, so the transposed MMA would apply, but it
// measured slower there (the four FP8 epilogue warps take both row chunks).
template <bool F8>
__device__ __forceinline__ bool transposed_half(const TileInfo& ti, int h) {
  return !F8 && narrow_half(ti, h);
}

// The part of the tile list this launch walks: `count` tile-list rows from
// `begin` (the whole list, the routed tiles only, or the shared expert's).
struct TileSpan {
  int begin, count, routed, shared;
};

__device__ __forceinline__ TileSpan tile_span(const GemmParams& p) {
  const int all = min(p.ntiles[0], p.max_mtiles);
  const int routed = min(p.ntiles[1], all);
  TileSpan t;
  t.routed = routed;
  t.shared = all - routed;
  t.begin = p.tile_set == kTilesShared ? routed : 0;
  t.count = p.tile_set == kTilesRouted ? routed : (p.tile_set == kTilesShared ? all - routed : all);
  return t;
}

// Work item `tile` = row tile q (in list order: the routed experts' tiles,
// then the shared expert's) x column block nb, column blocks of a row tile
// consecutive.  The shared expert's tiles run back to back at the end, so
// its weights stay in L2 across its row tiles without being held there for
// the whole launch.
__device__ __forceinline__ bool tile_at(const GemmParams& p, const TileSpan& sp, int tile, int BN, TileInfo& ti) {
  const int q = tile / p.n_nb;
  ti.nb = tile - q * p.n_nb;
  const int4 e = p.tiles[sp.begin + q];
  ti.group = e.x;
  ti.row0 = e.y;
  ti.rows = e.z;
  ti.seg_tiles = e.w;
  ti.halves = e.z > kTileM ? 2 : 1;
  ti.shared = (e.x == p.E);
  const int N = ti.shared ? p.N_shared : p.N_routed;
  return ti.nb * BN < N;  // false: this column block does not exist for the group
}

// Accumulator slots are handed out round-robin: a one-half tile takes the next
// slot, a two-half tile takes both.  MMA issuer and epilogue walk the same
// tile sequence, so they derive the same slot sequence.
struct SlotRing {
  int next = 0;
  uint32_t u0 = 0u, u1 = 0u;  // completed uses of slot 0 / slot 1
  __device__ __forceinline__ uint32_t use(int sl) const { return sl ? u1 : u0; }
  __device__ __forceinline__ void bump(int sl) {
    if (sl) ++u1; else ++u0;
  }
};

// One fp32 rounded to nearest-even bf16, as its 16 bits.
__device__ __forceinline__ uint16_t bf16_bits(float v) { return (uint16_t)(ptx::pack_bf16x2(v, 0.0f) & 0xFFFFu); }

// e4m3 codes (4 per word) * scale -> 4 bf16 (two packed words).  The e4m3 ->
// f16 widening is exact; the product is rounded once to bf16.
__device__ __forceinline__ uint2 e4m3x4_to_bf16x4(uint32_t q, float scale) {
  uint32_t h01, h23;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "mov.b32 {lo, hi}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, lo;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, hi;\n\t}\n"
      : "=r"(h01), "=r"(h23)
      : "r"(q));
  float a0, a1, b0, b1;
  asm("{\n\t.reg .b16 l0, h0, l1, h1;\n\t"
      "mov.b32 {l0, h0}, %4;\n\t"
      "mov.b32 {l1, h1}, %5;\n\t"
      "cvt.f32.f16 %0, l0;\n\t"
      "cvt.f32.f16 %1, h0;\n\t"
      "cvt.f32.f16 %2, l1;\n\t"
      "cvt.f32.f16 %3, h1;\n\t}\n"
      : "=f"(a0), "=f"(a1), "=f"(b0), "=f"(b1)
      : "r"(h01), "r"(h23));
  // the products of a pair in one packed multiply (the same rounding as two)
  float p0, p1, p2, p3;
  asm("{\n\t.reg .b64 a, b, s, pa, pb;\n\t"
      "mov.b64 a, {%4, %5};\n\t"
      "mov.b64 b, {%6, %7};\n\t"
      "mov.b64 s, {%8, %8};\n\t"
      "mul.rn.f32x2 pa, a, s;\n\t"
      "mul.rn.f32x2 pb, b, s;\n\t"
      "mov.b64 {%0, %1}, pa;\n\t"
      "mov.b64 {%2, %3}, pb;\n\t}\n"
      : "=f"(p0), "=f"(p1), "=f"(p2), "=f"(p3)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(scale));
  return make_uint2(ptx::pack_bf16x2(p0, p1), ptx::pack_bf16x2(p2, p3));
}

// Epilogue warps: two per TMEM lane quarter with bf16 weights (each drains
// half of the columns), one per quarter with FP8 weights (whose converter
// warps take the rest of the thread budget).
template <bool F8>
constexpr int epi_warps() {
  return F8 ? 4 : 8;
}
template <bool F8>
constexpr int kernel_threads() {
  return 64 + 32 * epi_warps<F8>() + (F8 ? 32 * kConvWarps : 0);
}

template <Mode M, bool F8, int N1 = 0>
__global__ void __launch_bounds__(kernel_threads<F8>(), 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA_r, const __grid_constant__ CUtensorMap tmA_s,
                        const __grid_constant__ CUtensorMap tmB_r, const __grid_constant__ CUtensorMap tmB_s,
                        const __grid_constant__ CUtensorMap tmC_r, const __grid_constant__ CUtensorMap tmC_s,
                        const GemmParams p) {
  static_assert(!N1 || F8, "one-half stages are an FP8 layout");
  constexpr int S = F8 ? (N1 == 2 ? kF8N2Stages : N1 ? kF8NStages : kF8Stages) : kStages;
  constexpr int BK = F8 ? kF8BK : kBK;
  constexpr uint32_t ABytes = F8 ? (N1 == 2 ? kF8N2ABytes : kF8ABytes) : kABytes;
  constexpr uint32_t StageBytes =
      F8 ? (N1 == 2 ? kF8N2StageBytes : N1 ? kF8NStageBytes : kF8StageBytes) : kStageBytes;
  constexpr int AHalves = N1 ? 1 : 2;  // A halves a stage has room for
  constexpr uint32_t BoxBytes = F8 ? kF8BoxBytes : kBoxBytes;
  constexpr uint32_t ASwz = F8 ? ptx::kSwizzle128B : kASwizzle;
  constexpr uint32_t ASBO = F8 ? 1024 : kASBO;
  constexpr int BN = Cfg<M>::BN;
  constexpr int CS = N1 ? kF8NConvStages : kF8ConvStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stage0 = align_1024(smem_raw);
  uint8_t* conv0 = stage0 + S * StageBytes;  // FP8: converted bf16 B ring
  uint64_t* full = reinterpret_cast<uint64_t*>(conv0 + (F8 ? CS * kF8ConvBytes : 0));
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* cfull = tempty + 2;
  uint64_t* cempty = cfull + CS;
  uint64_t* sfull = cempty + CS;  // tile-index ring: producer -> other roles
  uint64_t* sempty = sfull + kSchedDepth;
  uint64_t* done = sempty + kSchedDepth;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile int* sched_tile = reinterpret_cast<volatile int*>(tmem_slot + 2);
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
      ptx::mbar_init(&tempty[b], 32 * epi_warps<F8>());
    }
    for (int c = 0; c < CS; ++c) {
      ptx::mbar_init(&cfull[c], kConvWarps * 32);
      ptx::mbar_init(&cempty[c], 1);
    }
    for (int i = 0; i < kSchedDepth; ++i) {
      ptx::mbar_init(&sfull[i], 1);
      ptx::mbar_init(&sempty[i], 1 + 32 * epi_warps<F8>() + (F8 ? kConvWarps * 32 : 0));
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
  grid_dependency_wait();  // tile list, counters and A rows come from earlier kernels

  const TileSpan span = tile_span(p);
  const int total = span.count * p.n_nb;

  // Consumers take tile indices from the ring in the order the producer
  // claimed them; -1 ends the sequence.
  auto next_tile = [&](int& n, bool& ok) -> int {
    const int sd = n % kSchedDepth;
    if (!ptx::wait_bounded(&sfull[sd], (n / kSchedDepth) & 1, abort_flag)) {
      raise_status(p.status, abort_flag, kStatusTimeout);
      ok = false;
      return -1;
    }
    const int t = sched_tile[sd];
    ptx::mbar_arrive(&sempty[sd]);
    ++n;
    return t;
  };

  if (warp == 0) {
    if (lane == 0) {
      ptx::prefetch_tmap(&tmA_r);
      ptx::prefetch_tmap(&tmB_r);
      if (!F8) {
        ptx::prefetch_tmap(&tmA_s);
        ptx::prefetch_tmap(&tmB_s);
      }
      if (M == Mode::kSwiGLU) {
        ptx::prefetch_tmap(&tmC_r);
        if (!F8) ptx::prefetch_tmap(&tmC_s);
      }
#ifndef MOE_GEMM_A_POLICY
#define MOE_GEMM_A_POLICY 1
#endif
      // A rows are reused by the column blocks of their row tile, which run at
      // about the same time
      const uint64_t pol_a = MOE_GEMM_A_POLICY == 0 ? ptx::policy_evict_first()
                             : MOE_GEMM_A_POLICY == 1 ? ptx::policy_evict_normal()
                                                      : ptx::policy_evict_last();
      const uint64_t pol_w = ptx::policy_evict_first();  // each weight tile is read once

      int kg = 0, ns = 0;
      bool ok = !p.debug_withhold_loads;
      while (ok) {
        // claim the next tile and publish it to the other roles
        int tile = atomicAdd(p.sched_counter, 1);
        if (tile >= total) tile = -1;
        const int sd = ns % kSchedDepth;
        if (!ptx::wait_bounded(&sempty[sd], ((ns / kSchedDepth) & 1) ^ 1, abort_flag)) {
          raise_status(p.status, abort_flag, kStatusTimeout);
          ok = false;
          break;
        }
        sched_tile[sd] = tile;
        ptx::mbar_arrive(&sfull[sd]);
        ++ns;
        if (tile < 0) break;
        TileInfo ti;
        if (!tile_at(p, span, tile, BN, ti)) continue;
        if (N1 && ti.rows > (N1 == 2 ? kTileM / 2 : kTileM)) {  // longer than the stages hold: not computed
          raise_status(p.status, abort_flag, kStatusBounds);
          continue;
        }
        // weights of a group with several row tiles (the shared expert, an
        // expert with many rows) are read again by each of them: keep them in
        // L2 (evict-normal) instead of streaming them (evict-first); evict-last
        // would keep them past their last row tile, at the expense of the
        // weights that stream after them
        const uint64_t pol_b = (ti.shared || ti.seg_tiles > 1) ? pol_a : pol_w;
        const CUtensorMap* mA = ti.shared ? &tmA_s : &tmA_r;
        const CUtensorMap* mB = ti.shared ? &tmB_s : &tmB_r;
        const CUtensorMap* mC = ti.shared ? &tmC_s : &tmC_r;
        const int arow = ti.row0 + (ti.shared ? p.a_shared_row_offset : 0);
        const int e3 = ti.shared ? 0 : ti.group - p.group_base;
        const int nk = (ti.shared ? p.K_shared : p.K_routed) / BK;
        const int n0 = ti.nb * BN;
        const uint32_t bytes = ti.halves * ABytes + (F8 ? 2 * kF8RawBox : kBBytes);
        for (int kb = 0; kb < nk; ++kb, ++kg) {
          const int s = kg % S;
          const uint32_t ph = (kg / S) & 1;
          if (!ptx::wait_bounded(&empty[s], ph ^ 1, abort_flag)) {
            raise_status(p.status, abort_flag, kStatusTimeout);
            ok = false;
            break;
          }
          if (kGemmL2Prefetch > 0 && !F8 && kb + kGemmL2Prefetch < nk) {
            const int kp = (kb + kGemmL2Prefetch) * BK;
            if (M == Mode::kSwiGLU) {
              ptx::tma_prefetch_3d(mB, n0, kp, e3);
              ptx::tma_prefetch_3d(mB, n0 + 64, kp, e3);
              ptx::tma_prefetch_3d(mC, n0, kp, e3);
              ptx::tma_prefetch_3d(mC, n0 + 64, kp, e3);
            } else {
#pragma unroll
              for (int h = 0; h < 4; ++h) ptx::tma_prefetch_3d(mB, n0 + 64 * h, kp, e3);
            }
          }
          uint8_t* st = stage0 + s * StageBytes;
          ptx::mbar_arrive_expect_tx(&full[s], bytes);
          ptx::tma_load_2d(st, mA, &full[s], kb * BK, arow, pol_a);
          if (ti.halves == 2) ptx::tma_load_2d(st + ABytes, mA, &full[s], kb * BK, arow + kTileM, pol_a);
          uint8_t* sb = st + AHalves * ABytes;
          if (F8) {
            // raw codes: box 0 = W1 (or W2 columns n0..n0+127), box 1 = W3 (or W2 n0+128..)
            if (M == Mode::kSwiGLU) {
              ptx::tma_load_3d(sb, mB, &full[s], n0, kb * BK, e3, pol_b);
              ptx::tma_load_3d(sb + kF8RawBox, mC, &full[s], n0, kb * BK, e3, pol_b);
            } else {
              ptx::tma_load_3d(sb, mB, &full[s], n0, kb * BK, e3, pol_b);
              ptx::tma_load_3d(sb + kF8RawBox, mB, &full[s], n0 + 128, kb * BK, e3, pol_b);
            }
          } else if (M == Mode::kSwiGLU) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              ptx::tma_load_3d(sb + h * kBoxBytes, mB, &full[s], n0 + 64 * h, kb * BK, e3, pol_b);
              ptx::tma_load_3d(sb + (2 + h) * kBoxBytes, mC, &full[s], n0 + 64 * h, kb * BK, e3, pol_b);
            }
          } else {
#pragma unroll
            for (int h = 0; h < 4; ++h)
              ptx::tma_load_3d(sb + h * kBoxBytes, mB, &full[s], n0 + 64 * h, kb * BK, e3, pol_b);
          }
        }
      }
      // every issued copy must land before the CTA may exit
      for (int j = (kg > S ? kg - S : 0); j < kg; ++j)
        if (!ptx::wait_bounded(&full[j % S], (j / S) & 1, &never)) raise_status(p.status, abort_flag, kStatusTimeout);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // One N=256 MMA per half and K step.  SwiGLU: the stage holds W1's two
      // 64-column boxes followed by W3's, one box stride apart, so columns
      // 0-127 of the accumulator are g = x W1 and 128-255 are u = x W3 (A is
      // read once for both).  Down: 256 columns of W2.
      constexpr uint32_t idesc = ptx::idesc_bf16(kTileM, 256, false, true);
      constexpr uint32_t idesc_narrow = ptx::idesc_bf16(kTileM / 2, 256, false, true);
      int kg = 0, ns = 0;
      SlotRing ring;
      bool ok = true;
      while (ok) {
        const int tile = next_tile(ns, ok);
        if (tile < 0) break;
        TileInfo ti;
        if (!tile_at(p, span, tile, BN, ti) || (N1 && ti.rows > (N1 == 2 ? kTileM / 2 : kTileM))) continue;
        const int nk = (ti.shared ? p.K_shared : p.K_routed) / BK;
        for (int h = 0; h < ti.halves; ++h) {
          const int sl = (ring.next + h) & 1;
          if (!ptx::wait_bounded(&tempty[sl], (ring.use(sl) & 1) ^ 1, abort_flag)) {
            raise_status(p.status, abort_flag, kStatusTimeout);
            ok = false;
          }
        }
        if (!ok) break;
        ptx::tc_fence_after();
        for (int kb = 0; kb < nk; ++kb, ++kg) {
          const int s = kg % S;
          const uint32_t ph = (kg / S) & 1;
          const int c = kg % CS;
          if (!ptx::wait_bounded(&full[s], ph, abort_flag) ||
              (F8 && !ptx::wait_bounded(&cfull[c], (kg / CS) & 1, abort_flag))) {
            raise_status(p.status, abort_flag, kStatusTimeout);
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a0 = ptx::smem_u32(stage0 + s * StageBytes);
          const uint32_t b0 = F8 ? ptx::smem_u32(conv0 + c * kF8ConvBytes) : a0 + 2 * ABytes;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
            const uint64_t bd = ptx::sdesc_sw128(b0 + kk * 2048, BoxBytes, 1024);
            for (int h = 0; h < ti.halves; ++h) {
              const uint64_t ad = ptx::sdesc(a0 + h * ABytes + kk * 32, 16, ASBO, ASwz);
              const uint32_t dslot = tmem + ((ring.next + h) & 1) * kSlotCols;
              if (transposed_half<F8>(ti, h)) {
                // transposed: the weight boxes 0-1 and 2-3 (MN-major) as M=128
                // operands, the half's rows (K-major) as the N operand
                const uint32_t idt = ptx::idesc_bf16(kTileM, transposed_cols(ti, h), true, false);
                ptx::mma_bf16(dslot, bd, ad, idt, acc);
                ptx::mma_bf16(dslot + 128, ptx::sdesc_sw128(b0 + 2 * BoxBytes + kk * 2048, BoxBytes, 1024), ad, idt,
                              acc);
              } else {
                ptx::mma_bf16(dslot, ad, bd, narrow_half(ti, h) ? idesc_narrow : idesc, acc);
              }
            }
          }
          ptx::mma_commit(&empty[s]);
          if (F8) ptx::mma_commit(&cempty[c]);
        }
        if (!ok) break;
        for (int h = 0; h < ti.halves; ++h) {
          const int sl = (ring.next + h) & 1;
          ptx::mma_commit(&tfull[sl]);
          ring.bump(sl);
        }
        ring.next = (ring.next + ti.halves) & 1;
      }
      ptx::mma_commit(done);
      if (!ptx::wait_bounded(done, 0, &never)) raise_status(p.status, abort_flag, kStatusTimeout);
    }
  } else if (warp < 2 + epi_warps<F8>()) {
    constexpr int kParts = epi_warps<F8>() / 4;           // column parts per lane quarter
    constexpr int kChunks = BN / 32 / kParts;             // 32-column chunks per part
    const int q = warp & 3;                               // TMEM lane quarter this warp may access
    const int part = (warp - 2) / 4;
    const int row = q * 32 + lane;
    SlotRing ring;
    bool ok = true;
    int ns = 0;
    while (ok) {
      const int tile = next_tile(ns, ok);
      if (tile < 0) break;
      TileInfo ti;
      if (!tile_at(p, span, tile, BN, ti) || (N1 && ti.rows > (N1 == 2 ? kTileM / 2 : kTileM))) continue;
      const int n0 = ti.nb * BN;
      for (int h = 0; h < ti.halves; ++h) {
        const int sl = (ring.next + h) & 1;
        if (!ptx::wait_bounded(&tfull[sl], ring.use(sl) & 1, abort_flag)) {
          raise_status(p.status, abort_flag, kStatusTimeout);
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + sl * kSlotCols;
        const bool narrow = narrow_half(ti, h);
        const int r = h * kTileM + (narrow ? (lane < 16 ? q * 16 + lane : kTileM) : row);  // row within the tile
        const bool valid = r < ti.rows && (!narrow || lane < 16);
        if (transposed_half<F8>(ti, h)) {
          // transposed half: this lane holds output column f (and f + 128) of
          // the tile for the half's rows; each part takes 32 of its <= 64 rows
          const int f = q * 32 + lane;
          const int r0 = part * 32;
          uint32_t da[32], db[32];
          ptx::tmem_ld32(tbase + r0, da);
          ptx::tmem_ld32(tbase + 128 + r0, db);
          ptx::tmem_ld_wait2(da, db);
          ptx::tc_fence_before();
          ptx::mbar_arrive(&tempty[sl]);
          const int nr = ti.rows - h * kTileM - r0;  // rows of this part (may be <= 0)
          const int64_t grow0 = (int64_t)ti.row0 + h * kTileM + r0 + (ti.shared ? p.out_shared_row_offset : 0);
          if (M == Mode::kSwiGLU) {
            uint16_t* base = static_cast<uint16_t*>(ti.shared ? p.out_shared : p.out_routed);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (j < nr) {
                const float g = __uint_as_float(da[j]), u = __uint_as_float(db[j]);
                const int64_t hrow = grow0 + j;
                base[hrow * p.ld_out + n0 + f] = bf16_bits(g / (1.0f + __expf(-g)) * u);
                if (p.out_gu) {
                  uint16_t* gu_row = static_cast<uint16_t*>(p.out_gu) + hrow * 2 * p.ld_out + n0 + f;
                  gu_row[0] = bf16_bits(g);
                  gu_row[p.ld_out] = bf16_bits(u);
                }
              }
            }
          } else {
            const int N = ti.shared ? p.N_shared : p.N_routed;
            const bool c0ok = n0 + f < N, c1ok = n0 + 128 + f < N;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (j < nr) {
                const int64_t orow = grow0 + j;
                if (ti.shared) {
                  float* out = static_cast<float*>(p.out_shared) + orow * p.ld_out + n0 + f;
                  if (c0ok) out[0] = __uint_as_float(da[j]);
                  if (c1ok) out[128] = __uint_as_float(db[j]);
                } else {
                  uint16_t* out = static_cast<uint16_t*>(p.out_routed) + orow * p.ld_out + n0 + f;
                  if (c0ok) out[0] = bf16_bits(__uint_as_float(da[j]));
                  if (c1ok) out[128] = bf16_bits(__uint_as_float(db[j]));
                }
              }
            }
          }
          ring.bump(sl);
          continue;
        }
        if constexpr (!F8) {
          // Drain first: this warp's whole share of the slot (128 fp32 per
          // lane: g and u of two 32-column chunks, or four W2 chunks) is read
          // before the slot is released, so the MMA can reuse it while the
          // stores below are still in flight.
          static_assert(kChunks * 32 * (M == Mode::kSwiGLU ? 2 : 1) == 128, "drain-first share is 128 columns");
          uint32_t buf[4][32];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int col = M == Mode::kSwiGLU ? (i >= 2 ? 128 : 0) + (part * kChunks + (i & 1)) * 32
                                               : (part * kChunks + i) * 32;
            ptx::tmem_ld32(tbase + col, buf[i]);
          }
          ptx::tmem_ld_wait(buf[0]);
          ptx::tmem_ld_keep(buf[1]);
          ptx::tmem_ld_keep(buf[2]);
          ptx::tmem_ld_keep(buf[3]);
          ptx::tc_fence_before();
          ptx::mbar_arrive(&tempty[sl]);
          if (valid) {
            if (M == Mode::kSwiGLU) {
              const int64_t hrow = (int64_t)ti.row0 + r + (ti.shared ? p.out_shared_row_offset : 0);
              uint16_t* base = static_cast<uint16_t*>(ti.shared ? p.out_shared : p.out_routed);
              uint4* out = reinterpret_cast<uint4*>(base + hrow * p.ld_out + n0);
#pragma unroll
              for (int cc = 0; cc < 2; ++cc) {
                const uint32_t* g = buf[cc];
                const uint32_t* u = buf[2 + cc];
                uint32_t hp[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                  const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
                  const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
                  const float h0 = g0 / (1.0f + __expf(-g0)) * u0;
                  const float h1 = g1 / (1.0f + __expf(-g1)) * u1;
                  hp[i] = ptx::pack_bf16x2(h0, h1);
                }
                const int c = part * kChunks + cc;
#pragma unroll
                for (int v = 0; v < 4; ++v)
                  out[c * 4 + v] = make_uint4(hp[4 * v], hp[4 * v + 1], hp[4 * v + 2], hp[4 * v + 3]);
                if (p.out_gu) {
                  // the backward pass's copy of g and u (bf16, same row as H)
                  uint16_t* gu_row = static_cast<uint16_t*>(p.out_gu) + hrow * 2 * p.ld_out + n0 + c * 32;
                  uint4* og = reinterpret_cast<uint4*>(gu_row);
                  uint4* ou = reinterpret_cast<uint4*>(gu_row + p.ld_out);
#pragma unroll
                  for (int v = 0; v < 4; ++v) {
                    og[v] = make_uint4(ptx::pack_bf16x2(__uint_as_float(g[8 * v]), __uint_as_float(g[8 * v + 1])),
                                       ptx::pack_bf16x2(__uint_as_float(g[8 * v + 2]), __uint_as_float(g[8 * v + 3])),
                                       ptx::pack_bf16x2(__uint_as_float(g[8 * v + 4]), __uint_as_float(g[8 * v + 5])),
                                       ptx::pack_bf16x2(__uint_as_float(g[8 * v + 6]), __uint_as_float(g[8 * v + 7])));
                    ou[v] = make_uint4(ptx::pack_bf16x2(__uint_as_float(u[8 * v]), __uint_as_float(u[8 * v + 1])),
                                       ptx::pack_bf16x2(__uint_as_float(u[8 * v + 2]), __uint_as_float(u[8 * v + 3])),
                                       ptx::pack_bf16x2(__uint_as_float(u[8 * v + 4]), __uint_as_float(u[8 * v + 5])),
                                       ptx::pack_bf16x2(__uint_as_float(u[8 * v + 6]), __uint_as_float(u[8 * v + 7])));
                  }
                }
              }
            } else {
              const int64_t orow = (int64_t)ti.row0 + r + (ti.shared ? p.out_shared_row_offset : 0);
              const int N = ti.shared ? p.N_shared : p.N_routed;
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const uint32_t* v32 = buf[i];
                const int col = n0 + (part * kChunks + i) * 32;
                if (col >= N) continue;
                if (ti.shared) {
                  float4* out = reinterpret_cast<float4*>(static_cast<float*>(p.out_shared) + orow * p.ld_out + col);
#pragma unroll
                  for (int v = 0; v < 8; ++v)
                    out[v] = make_float4(__uint_as_float(v32[4 * v]), __uint_as_float(v32[4 * v + 1]),
                                         __uint_as_float(v32[4 * v + 2]), __uint_as_float(v32[4 * v + 3]));
                } else {
                  uint4* out =
                      reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out_routed) + orow * p.ld_out + col);
#pragma unroll
                  for (int v = 0; v < 4; ++v)
                    out[v] = make_uint4(
                        ptx::pack_bf16x2(__uint_as_float(v32[8 * v + 0]), __uint_as_float(v32[8 * v + 1])),
                        ptx::pack_bf16x2(__uint_as_float(v32[8 * v + 2]), __uint_as_float(v32[8 * v + 3])),
                        ptx::pack_bf16x2(__uint_as_float(v32[8 * v + 4]), __uint_as_float(v32[8 * v + 5])),
                        ptx::pack_bf16x2(__uint_as_float(v32[8 * v + 6]), __uint_as_float(v32[8 * v + 7])));
                }
              }
            }
          }
        } else if (M == Mode::kSwiGLU) {
          const int64_t hrow = (int64_t)ti.row0 + r + (ti.shared ? p.out_shared_row_offset : 0);
          uint16_t* base = static_cast<uint16_t*>(ti.shared ? p.out_shared : p.out_routed);
          uint4* out = reinterpret_cast<uint4*>(base + hrow * p.ld_out + n0);
#pragma unroll 1
          for (int cc = 0; cc < kChunks; ++cc) {
            const int c = part * kChunks + cc;
            uint32_t g[32], u[32];
            ptx::tmem_ld32(tbase + c * 32, g);
            ptx::tmem_ld32(tbase + 128 + c * 32, u);
            ptx::tmem_ld_wait2(g, u);
            if (cc == kChunks - 1) {
              ptx::tc_fence_before();
              ptx::mbar_arrive(&tempty[sl]);
            }
            if (valid) {
              uint32_t hp[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
                const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
                const float h0 = g0 / (1.0f + __expf(-g0)) * u0;
                const float h1 = g1 / (1.0f + __expf(-g1)) * u1;
                hp[i] = ptx::pack_bf16x2(h0, h1);
              }
#pragma unroll
              for (int v = 0; v < 4; ++v)
                out[c * 4 + v] = make_uint4(hp[4 * v], hp[4 * v + 1], hp[4 * v + 2], hp[4 * v + 3]);
            }
          }
        } else {
          const int64_t orow = (int64_t)ti.row0 + r + (ti.shared ? p.out_shared_row_offset : 0);
          const int N = ti.shared ? p.N_shared : p.N_routed;
#pragma unroll 1
          for (int cc = 0; cc < kChunks; cc += 2) {
            // two 32-column chunks in flight before one wait
            const int c = part * kChunks + cc;
            uint32_t va[32], vb[32];
            ptx::tmem_ld32(tbase + c * 32, va);
            ptx::tmem_ld32(tbase + (c + 1) * 32, vb);
            ptx::tmem_ld_wait2(va, vb);
            if (cc + 2 >= kChunks) {
              ptx::tc_fence_before();
              ptx::mbar_arrive(&tempty[sl]);
            }
#pragma unroll
            for (int z = 0; z < 2; ++z) {
              const uint32_t* v32 = z ? vb : va;
              const int col = n0 + (c + z) * 32;
              if (!valid || col >= N) continue;
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
                  out[v] = make_uint4(
                      ptx::pack_bf16x2(__uint_as_float(v32[8 * v + 0]), __uint_as_float(v32[8 * v + 1])),
                      ptx::pack_bf16x2(__uint_as_float(v32[8 * v + 2]), __uint_as_float(v32[8 * v + 3])),
                      ptx::pack_bf16x2(__uint_as_float(v32[8 * v + 4]), __uint_as_float(v32[8 * v + 5])),
                      ptx::pack_bf16x2(__uint_as_float(v32[8 * v + 6]), __uint_as_float(v32[8 * v + 7])));
              }
            }
          }
        }
        ring.bump(sl);
      }
      ring.next = (ring.next + ti.halves) & 1;
    }
  } else if (F8) {
    // converters: kConvWarps warps.  A raw stage is 2 boxes x 64 K rows of 128
    // codes = 128 rows; a warp step covers 4 rows, a lane 16 codes (one
    // 16-byte load, two 16-byte stores of bf16).
    const int cw = warp - 2 - epi_warps<F8>();
    const int sub_row = lane >> 3;          // row within the 4-row step
    const int col16 = lane & 7;             // 16-code column group within the row
    int kg = 0, ns = 0;
    bool ok = true;
    while (ok) {
      const int tile = next_tile(ns, ok);
      if (tile < 0) break;
      TileInfo ti;
      if (!tile_at(p, span, tile, BN, ti) || (N1 && ti.rows > (N1 == 2 ? kTileM / 2 : kTileM))) continue;
      const int nk = p.K_routed / BK;
      const int n0 = ti.nb * BN;
      const int ksb = p.K_routed / 128, nsb = p.N_routed / 128;  // scale blocks per expert
      // the block scales of K step kb (one 128 x 128 block per box)
      auto load_scales = [&](int kb, float* sc) {
        const int kblk = (kb * BK) / 128;
        const int64_t sbase = ((int64_t)(ti.group - p.group_base) * ksb + kblk) * nsb;
        if (M == Mode::kSwiGLU) {
          sc[0] = p.scale_b[sbase + n0 / 128];
          sc[1] = p.scale_c[sbase + n0 / 128];
        } else {
          sc[0] = p.scale_b[sbase + n0 / 128];
          sc[1] = n0 + 128 < p.N_routed ? p.scale_b[sbase + n0 / 128 + 1] : 0.0f;  // past the last column
        }
      };
      float sc_next[2];
      load_scales(0, sc_next);
      for (int kb = 0; kb < nk; ++kb, ++kg) {
        const int s = kg % S;
        const int c = kg % CS;
        // this step's scales were loaded one step ahead; the next step's load
        // is issued before the waits, so its latency overlaps them
        const float sc[2] = {sc_next[0], sc_next[1]};
        if (kb + 1 < nk) load_scales(kb + 1, sc_next);
        if (!ptx::wait_bounded(&full[s], (kg / S) & 1, abort_flag) ||
            !ptx::wait_bounded(&cempty[c], ((kg / CS) & 1) ^ 1, abort_flag)) {
          raise_status(p.status, abort_flag, kStatusTimeout);
          ok = false;
          break;
        }
        const uint8_t* raw = stage0 + s * StageBytes + AHalves * ABytes;
        uint8_t* conv = conv0 + c * kF8ConvBytes;
#pragma unroll
        for (int i = 0; i < 128 / (4 * kConvWarps); ++i) {
          const int rr = (cw * (128 / kConvWarps)) + i * 4 + sub_row;  // 0..127
          const int box = rr >> 6, k = rr & 63;
          const uint4 q = *reinterpret_cast<const uint4*>(raw + box * kF8RawBox + k * 128 + col16 * 16);
          const float scale = box ? sc[1] : sc[0];
          const uint2 v0 = e4m3x4_to_bf16x4(q.x, scale), v1 = e4m3x4_to_bf16x4(q.y, scale);
          const uint2 v2 = e4m3x4_to_bf16x4(q.z, scale), v3 = e4m3x4_to_bf16x4(q.w, scale);
          // codes col16*16 .. +15 of box `box` = bf16 sub-box 2*box + col16/4,
          // 16-byte chunks 2*(col16%4) and 2*(col16%4)+1 of row k (swizzled)
          uint8_t* dst = conv + (2 * box + (col16 >> 2)) * kF8BoxBytes + k * 128;
          const int ch = 2 * (col16 & 3);
          *reinterpret_cast<uint4*>(dst + ((ch ^ (k & 7)) << 4)) = make_uint4(v0.x, v0.y, v1.x, v1.y);
          *reinterpret_cast<uint4*>(dst + (((ch + 1) ^ (k & 7)) << 4)) = make_uint4(v2.x, v2.y, v3.x, v3.y);
        }
        ptx::fence_proxy_async();
        ptx::mbar_arrive(&cfull[c]);
      }
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

// ------------------------------------------------------------ CTA pairs
// Full 256-row tiles, and last tiles of more than kPairMinRows rows (bf16
// weights), on a 2-CTA cluster: CTA r holds rows
// 128r..128r+127 of the tile (A) and half of its B columns (SwiGLU: CTA 0 the
// 128 W1 columns, CTA 1 the same 128 W3 columns; down: 128 of the 256 W2
// columns each).  CTA 0's thread issues tcgen05.mma.cta_group::2 with M=256,
// N=256, so each weight byte is read from shared memory once per 256 rows
// (the one-CTA kernel reads it once per 128-row half); each CTA's TMEM gets
// its 128 rows x 256 columns, in the same column order as the one-CTA kernel
// (SwiGLU: g then u), and each CTA's epilogue stores its own rows.  Tiles are
// taken in a fixed order: cluster c takes tiles c, c + clusters, ...
constexpr int kPairStages = 6;
constexpr uint32_t kPairABytes = kTileM * kBK * 2;  // this CTA's 128 rows
constexpr uint32_t kPairBBytes = 2 * kBoxBytes;     // this CTA's 128 columns
constexpr uint32_t kPairStageBytes = kPairABytes + kPairBBytes;
constexpr int kPairEpiWarps = 8;
constexpr int kPairThreads = 64 + 32 * kPairEpiWarps;
static_assert(kBK == 64, "the pair kernel uses 64-deep K steps");
static_assert(kPairStages * kPairStageBytes + 1024 + 256 <= 232448, "shared memory budget (pair)");

constexpr size_t pair_smem_bytes() { return 1024 + kPairStages * kPairStageBytes + 256; }

template <Mode M>
__global__ void __launch_bounds__(kPairThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA_r, const __grid_constant__ CUtensorMap tmA_s,
                             const __grid_constant__ CUtensorMap tmB_r, const __grid_constant__ CUtensorMap tmB_s,
                             const __grid_constant__ CUtensorMap tmC_r, const __grid_constant__ CUtensorMap tmC_s,
                             const GemmParams p) {
  constexpr int S = kPairStages;
  constexpr int BN = Cfg<M>::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stage0 = align_1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(stage0 + S * kPairStageBytes);  // used on CTA 0
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;  // used on CTA 0: both CTAs' epilogues arrive
  uint64_t* done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  __shared__ uint32_t never;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();  // 0: issues the MMA
  const bool lead = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&tfull[b], 1);
      ptx::mbar_init(&tempty[b], 2 * 32 * kPairEpiWarps);
    }
    ptx::mbar_init(done, 1);
    *abort_flag = 0u;
    never = 0u;
    ptx::fence_barrier_init();
    ptx::fence_proxy_async();
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(tmem_slot, kTmemCols);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // both CTAs' barriers exist before any cross-CTA arrival
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dependency_wait();

  const TileSpan span = tile_span(p);
  const int total = span.count * p.n_nb;
  const int cluster = blockIdx.x >> 1, clusters = gridDim.x >> 1;

  if (warp == 0) {
    if (lane == 0) {
      ptx::prefetch_tmap(&tmA_r);
      ptx::prefetch_tmap(&tmB_r);
      ptx::prefetch_tmap(&tmA_s);
      ptx::prefetch_tmap(&tmB_s);
      if (M == Mode::kSwiGLU) {
        ptx::prefetch_tmap(&tmC_r);
        ptx::prefetch_tmap(&tmC_s);
      }
      const uint64_t pol_a = ptx::policy_evict_normal();
      const uint64_t pol_w = ptx::policy_evict_first();
      int kg = 0;
      bool ok = !p.debug_withhold_loads;
      for (int tile = cluster; ok && tile < total; tile += clusters) {
        TileInfo ti;
        if (!tile_at(p, span, tile, BN, ti)) continue;
        // weights read again by later row tiles stay in L2 (as above)
        const uint64_t pol_b = (ti.shared || ti.seg_tiles > 1) ? pol_a : pol_w;
        const CUtensorMap* mA = ti.shared ? &tmA_s : &tmA_r;
        // SwiGLU: CTA 0 loads W1's columns, CTA 1 the same columns of W3
        const CUtensorMap* mB = (M == Mode::kSwiGLU && rank == 1) ? (ti.shared ? &tmC_s : &tmC_r)
                                                                   : (ti.shared ? &tmB_s : &tmB_r);
        const int arow = ti.row0 + (ti.shared ? p.a_shared_row_offset : 0) + (int)rank * kTileM;
        const int e3 = ti.shared ? 0 : ti.group - p.group_base;
        const int nk = (ti.shared ? p.K_shared : p.K_routed) / kBK;
        const int nb0 = ti.nb * BN + (M == Mode::kSwiGLU ? 0 : (int)rank * 128);  // this CTA's first B column
        for (int kb = 0; kb < nk; ++kb, ++kg) {
          const int s = kg % S;
          if (!ptx::wait_bounded(&empty[s], ((kg / S) & 1) ^ 1, abort_flag)) {
            raise_status(p.status, abort_flag, kStatusTimeout);
            ok = false;
            break;
          }
          const uint32_t bar = ptx::mapa(&full[s], 0);
          if (lead) ptx::mbar_arrive_expect_tx(&full[s], 2 * kPairStageBytes);  // both CTAs' bytes
          uint8_t* st = stage0 + s * kPairStageBytes;
          ptx::tma_load_2d_pair(st, mA, bar, kb * kBK, arow, pol_a);
#pragma unroll
          for (int h = 0; h < 2; ++h)
            ptx::tma_load_3d_pair(st + kPairABytes + h * kBoxBytes, mB, bar, nb0 + 64 * h, kb * kBK, e3, pol_b);
        }
      }
      // CTA 0 sees every copy of both CTAs land before the pair may exit (the
      // final cluster barrier holds CTA 1 until then)
      if (lead)
        for (int j = (kg > S ? kg - S : 0); j < kg; ++j)
          if (!ptx::wait_bounded(&full[j % S], (j / S) & 1, &never)) raise_status(p.status, abort_flag, kStatusTimeout);
    }
  } else if (warp == 1) {
    if (lane == 0 && lead) {
      constexpr uint32_t idesc = ptx::idesc_bf16(2 * kTileM, 256, false, true);
      int kg = 0, tl = 0;
      bool ok = true;
      for (int tile = cluster; ok && tile < total; tile += clusters) {
        TileInfo ti;
        if (!tile_at(p, span, tile, BN, ti)) continue;
        const int nk = (ti.shared ? p.K_shared : p.K_routed) / kBK;
        const int sl = tl & 1;
        if (!ptx::wait_bounded(&tempty[sl], ((tl >> 1) & 1) ^ 1, abort_flag)) {
          raise_status(p.status, abort_flag, kStatusTimeout);
          break;
        }
        ptx::tc_fence_after();
        for (int kb = 0; kb < nk; ++kb, ++kg) {
          const int s = kg % S;
          if (!ptx::wait_bounded(&full[s], (kg / S) & 1, abort_flag)) {
            raise_status(p.status, abort_flag, kStatusTimeout);
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a0 = ptx::smem_u32(stage0 + s * kPairStageBytes);
          const uint32_t b0 = a0 + kPairABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            ptx::mma_bf16_pair(tmem + sl * kSlotCols, ptx::sdesc(a0 + kk * 32, 16, kASBO, kASwizzle),
                               ptx::sdesc_sw128(b0 + kk * 2048, kBoxBytes, 1024), idesc, (kb | kk) != 0 ? 1u : 0u);
          ptx::mma_commit_pair(&empty[s], 0x3);
        }
        if (!ok) break;
        ptx::mma_commit_pair(&tfull[sl], 0x3);
        ++tl;
      }
      ptx::mma_commit_pair(done, 0x1);
      if (!ptx::wait_bounded(done, 0, &never)) raise_status(p.status, abort_flag, kStatusTimeout);
    }
  } else {
    // epilogue: this CTA's 128 rows; each lane drains its 128 columns, frees
    // the slot on CTA 0's barrier, then computes and stores
    constexpr int kChunks = BN / 32 / 2;  // 32-column chunks per part (two parts per lane quarter)
    const int q = warp & 3;
    const int part = (warp - 2) / 4;
    const int row = (int)rank * kTileM + q * 32 + lane;  // row within the tile
    const uint32_t tempty_lead0 = ptx::mapa(&tempty[0], 0), tempty_lead1 = ptx::mapa(&tempty[1], 0);
    int tl = 0;
    for (int tile = cluster; tile < total; tile += clusters) {
      TileInfo ti;
      if (!tile_at(p, span, tile, BN, ti)) continue;
      const int sl = tl & 1;
      if (!ptx::wait_bounded(&tfull[sl], (tl >> 1) & 1, abort_flag)) {
        raise_status(p.status, abort_flag, kStatusTimeout);
        break;
      }
      ptx::tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + sl * kSlotCols;
      uint32_t buf[4][32];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int col = M == Mode::kSwiGLU ? (i >= 2 ? 128 : 0) + (part * kChunks + (i & 1)) * 32
                                           : (part * kChunks + i) * 32;
        ptx::tmem_ld32(tbase + col, buf[i]);
      }
      ptx::tmem_ld_wait(buf[0]);
      ptx::tmem_ld_keep(buf[1]);
      ptx::tmem_ld_keep(buf[2]);
      ptx::tmem_ld_keep(buf[3]);
      ptx::tc_fence_before();
      ptx::mbar_arrive_cluster(sl ? tempty_lead1 : tempty_lead0);
      ++tl;
      if (row >= ti.rows) continue;
      const int n0 = ti.nb * BN;
      if (M == Mode::kSwiGLU) {
        const int64_t hrow = (int64_t)ti.row0 + row + (ti.shared ? p.out_shared_row_offset : 0);
        uint16_t* base = static_cast<uint16_t*>(ti.shared ? p.out_shared : p.out_routed);
        uint4* out = reinterpret_cast<uint4*>(base + hrow * p.ld_out + n0);
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const uint32_t* g = buf[cc];
          const uint32_t* u = buf[2 + cc];
          uint32_t hp[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
            const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
            hp[i] = ptx::pack_bf16x2(g0 / (1.0f + __expf(-g0)) * u0, g1 / (1.0f + __expf(-g1)) * u1);
          }
          const int c = part * kChunks + cc;
#pragma unroll
          for (int v = 0; v < 4; ++v)
            out[c * 4 + v] = make_uint4(hp[4 * v], hp[4 * v + 1], hp[4 * v + 2], hp[4 * v + 3]);
        }
      } else {
        const int64_t orow = (int64_t)ti.row0 + row + (ti.shared ? p.out_shared_row_offset : 0);
        const int N = ti.shared ? p.N_shared : p.N_routed;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t* v32 = buf[i];
          const int col = n0 + (part * kChunks + i) * 32;
          if (col >= N) continue;
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
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();  // no cross-CTA arrival or MMA operand read is still pending
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// FP8 weights on CTA pairs: per K step each CTA brings its 128 rows of A
// (counted on CTA 0's barrier) and the raw e4m3 codes of its half of B
// ([64 K x 128 N], counted on its own barrier); its converter warps widen them
// (code x block scale -> bf16) into its own converted ring and arrive on CTA
// 0's barrier; CTA 0 issues the M=256 pair MMA once both CTAs' A and both
// conversions are in.  Routed tiles only (the shared expert is bf16).
#ifndef MOE_PAIR_F8_STAGES
#define MOE_PAIR_F8_STAGES 5
#endif
#ifndef MOE_PAIR_F8_CONV_STAGES
#define MOE_PAIR_F8_CONV_STAGES 5
#endif
// The converted ring is as deep as the operand ring: its hand-off (MMA done on
// CTA 0 -> commit to CTA 1 -> CTA 1 converts -> arrival on CTA 0) crosses the
// pair twice per K step.
constexpr int kPairF8Stages = MOE_PAIR_F8_STAGES;
constexpr uint32_t kPairF8RawBytes = 64 * 128;                         // one raw box
constexpr uint32_t kPairF8StageBytes = kPairABytes + kPairF8RawBytes;  // 24 KB
constexpr int kPairF8ConvStages = MOE_PAIR_F8_CONV_STAGES;
// Converted buffer c = K step % kPairF8ConvStages is free once the MMA that
// read it kPairF8ConvStages steps earlier has completed.  With both rings of
// one depth that MMA's commit to the stage's `empty` barrier is what lets the
// producer reload stage s, and the converters start on step kg only after its
// raw codes landed in stage s, i.e. after that commit: the separate `cempty`
// hand-off is then redundant.
#ifndef MOE_PAIR_F8_ONE_COMMIT
#define MOE_PAIR_F8_ONE_COMMIT 1
#endif
constexpr bool kPairF8OneCommit = MOE_PAIR_F8_ONE_COMMIT && kPairF8ConvStages == kPairF8Stages;
constexpr uint32_t kPairF8ConvBytes = 2 * kF8BoxBytes;  // 16 KB: two bf16 [64 K x 64 N] boxes
constexpr int kPairF8EpiWarps = 4;
constexpr int kPairF8Threads = 64 + 32 * kPairF8EpiWarps + 32 * kConvWarps;
constexpr size_t pair_f8_smem_bytes() {
  return 1024 + kPairF8Stages * kPairF8StageBytes + kPairF8ConvStages * kPairF8ConvBytes + 512;
}
static_assert(pair_f8_smem_bytes() <= 232448, "shared memory budget (FP8 pair)");

template <Mode M>
__global__ void __launch_bounds__(kPairF8Threads, 1)
    grouped_gemm_pair_f8_kernel(const __grid_constant__ CUtensorMap tmA_r, const __grid_constant__ CUtensorMap tmB_r,
                                const __grid_constant__ CUtensorMap tmC_r, const GemmParams p) {
  constexpr int S = kPairF8Stages;
  constexpr int CS = kPairF8ConvStages;
  constexpr int BN = Cfg<M>::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* stage0 = align_1024(smem_raw);
  uint8_t* conv0 = stage0 + S * kPairF8StageBytes;
  uint64_t* afull = reinterpret_cast<uint64_t*>(conv0 + CS * kPairF8ConvBytes);  // CTA 0: both CTAs' A
  uint64_t* rfull = afull + S;   // each CTA: its raw codes
  uint64_t* empty = rfull + S;   // each CTA: stage free (MMA commit)
  uint64_t* cfull = empty + S;   // CTA 0: both CTAs' conversions
  uint64_t* cempty = cfull + CS; // each CTA: converted buffer free (MMA commit)
  uint64_t* tfull = cempty + CS;
  uint64_t* tempty = tfull + 2;  // CTA 0: both CTAs' epilogues
  uint64_t* done = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  __shared__ uint32_t never;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const bool lead = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(&afull[s], 1);
      ptx::mbar_init(&rfull[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int c = 0; c < CS; ++c) {
      ptx::mbar_init(&cfull[c], 2 * kConvWarps);  // one arrival per converter warp of either CTA
      ptx::mbar_init(&cempty[c], 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&tfull[b], 1);
      ptx::mbar_init(&tempty[b], 2 * 32 * kPairF8EpiWarps);
    }
    ptx::mbar_init(done, 1);
    *abort_flag = 0u;
    never = 0u;
    ptx::fence_barrier_init();
    ptx::fence_proxy_async();
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(tmem_slot, kTmemCols);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dependency_wait();

  const TileSpan span = tile_span(p);
  const int total = span.count * p.n_nb;
  const int cluster = blockIdx.x >> 1, clusters = gridDim.x >> 1;

  if (warp == 0) {
    if (lane == 0) {
      ptx::prefetch_tmap(&tmA_r);
      ptx::prefetch_tmap(&tmB_r);
      if (M == Mode::kSwiGLU) ptx::prefetch_tmap(&tmC_r);
      const uint64_t pol_a = ptx::policy_evict_normal();
      const uint64_t pol_w = ptx::policy_evict_first();
      int kg = 0;
      bool ok = !p.debug_withhold_loads;
      for (int tile = cluster; ok && tile < total; tile += clusters) {
        TileInfo ti;
        if (!tile_at(p, span, tile, BN, ti)) continue;
        const uint64_t pol_b = ti.seg_tiles > 1 ? pol_a : pol_w;
        // raw codes: SwiGLU CTA 0 W1 / CTA 1 W3 at columns n0; down W2 at n0 + 128r
        const CUtensorMap* mR = (M == Mode::kSwiGLU && rank == 1) ? &tmC_r : &tmB_r;
        const int rcol = ti.nb * BN + (M == Mode::kSwiGLU ? 0 : (int)rank * 128);
        const int arow = ti.row0 + (int)rank * kTileM;
        const int e3 = ti.group - p.group_base;
        const int nk = p.K_routed / kF8BK;
        for (int kb = 0; kb < nk; ++kb, ++kg) {
          const int s = kg % S;
          if (!ptx::wait_bounded(&empty[s], ((kg / S) & 1) ^ 1, abort_flag)) {
            raise_status(p.status, abort_flag, kStatusTimeout);
            ok = false;
            break;
          }
          if (lead) ptx::mbar_arrive_expect_tx(&afull[s], 2 * kPairABytes);
          ptx::mbar_arrive_expect_tx(&rfull[s], kPairF8RawBytes);
          uint8_t* st = stage0 + s * kPairF8StageBytes;
          ptx::tma_load_2d_pair(st, &tmA_r, ptx::mapa(&afull[s], 0), kb * kF8BK, arow, pol_a);
          ptx::tma_load_3d(st + kPairABytes, mR, &rfull[s], rcol, kb * kF8BK, e3, pol_b);
        }
      }
      // every copy of both CTAs lands before the pair may exit
      for (int j = (kg > S ? kg - S : 0); j < kg; ++j) {
        if (!ptx::wait_bounded(&rfull[j % S], (j / S) & 1, &never)) raise_status(p.status, abort_flag, kStatusTimeout);
        if (lead && !ptx::wait_bounded(&afull[j % S], (j / S) & 1, &never))
          raise_status(p.status, abort_flag, kStatusTimeout);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && lead) {
      constexpr uint32_t idesc = ptx::idesc_bf16(2 * kTileM, 256, false, true);
      int kg = 0, tl = 0;
      bool ok = true;
      for (int tile = cluster; ok && tile < total; tile += clusters) {
        TileInfo ti;
        if (!tile_at(p, span, tile, BN, ti)) continue;
        const int nk = p.K_routed / kF8BK;
        const int sl = tl & 1;
        if (!ptx::wait_bounded(&tempty[sl], ((tl >> 1) & 1) ^ 1, abort_flag)) {
          raise_status(p.status, abort_flag, kStatusTimeout);
          break;
        }
        ptx::tc_fence_after();
        for (int kb = 0; kb < nk; ++kb, ++kg) {
          const int s = kg % S;
          const int c = kg % CS;
          if (!ptx::wait_bounded(&afull[s], (kg / S) & 1, abort_flag) ||
              !ptx::wait_bounded(&cfull[c], (kg / CS) & 1, abort_flag)) {
            raise_status(p.status, abort_flag, kStatusTimeout);
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t a0 = ptx::smem_u32(stage0 + s * kPairF8StageBytes);
          const uint32_t b0 = ptx::smem_u32(conv0 + c * kPairF8ConvBytes);
#pragma unroll
          for (int kk = 0; kk < kF8BK / 16; ++kk)
            ptx::mma_bf16_pair(tmem + sl * kSlotCols, ptx::sdesc_sw128(a0 + kk * 32, 16, 1024),
                               ptx::sdesc_sw128(b0 + kk * 2048, kF8BoxBytes, 1024), idesc, (kb | kk) != 0 ? 1u : 0u);
          ptx::mma_commit_pair(&empty[s], 0x3);
          // with rings of one depth, converted buffer c is stage s: the
          // converters' wait for the stage's raw codes already orders them
          // after this commit, so no second commit is needed
          if (!kPairF8OneCommit) ptx::mma_commit_pair(&cempty[c], 0x3);
        }
        if (!ok) break;
        ptx::mma_commit_pair(&tfull[sl], 0x3);
        ++tl;
      }
      ptx::mma_commit_pair(done, 0x1);
      if (!ptx::wait_bounded(done, 0, &never)) raise_status(p.status, abort_flag, kStatusTimeout);
    }
  } else if (warp < 2 + kPairF8EpiWarps) {
    // epilogue: one warp per TMEM lane quarter, streaming 32-column chunks
    const int q = warp & 3;
    const int row = (int)rank * kTileM + q * 32 + lane;
    const uint32_t tempty_lead0 = ptx::mapa(&tempty[0], 0), tempty_lead1 = ptx::mapa(&tempty[1], 0);
    int tl = 0;
    for (int tile = cluster; tile < total; tile += clusters) {
      TileInfo ti;
      if (!tile_at(p, span, tile, BN, ti)) continue;
      const int sl = tl & 1;
      if (!ptx::wait_bounded(&tfull[sl], (tl >> 1) & 1, abort_flag)) {
        raise_status(p.status, abort_flag, kStatusTimeout);
        break;
      }
      ptx::tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + sl * kSlotCols;
      const bool valid = row < ti.rows;
      const int n0 = ti.nb * BN;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t va[32], vb[32];
        // SwiGLU: g and u of outputs n0 + 32c; down: W2 columns n0 + 64c, +32
        ptx::tmem_ld32(tbase + (M == Mode::kSwiGLU ? c * 32 : c * 64), va);
        ptx::tmem_ld32(tbase + (M == Mode::kSwiGLU ? 128 + c * 32 : c * 64 + 32), vb);
        ptx::tmem_ld_wait2(va, vb);
        if (c == 3) {
          ptx::tc_fence_before();
          ptx::mbar_arrive_cluster(sl ? tempty_lead1 : tempty_lead0);
        }
        if (!valid) continue;
        if (M == Mode::kSwiGLU) {
          uint16_t* base = static_cast<uint16_t*>(p.out_routed);
          uint4* out = reinterpret_cast<uint4*>(base + ((int64_t)ti.row0 + row) * p.ld_out + n0 + c * 32);
          uint32_t hp[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float g0 = __uint_as_float(va[2 * i]), g1 = __uint_as_float(va[2 * i + 1]);
            const float u0 = __uint_as_float(vb[2 * i]), u1 = __uint_as_float(vb[2 * i + 1]);
            hp[i] = ptx::pack_bf16x2(g0 / (1.0f + __expf(-g0)) * u0, g1 / (1.0f + __expf(-g1)) * u1);
          }
#pragma unroll
          for (int v = 0; v < 4; ++v) out[v] = make_uint4(hp[4 * v], hp[4 * v + 1], hp[4 * v + 2], hp[4 * v + 3]);
        } else {
#pragma unroll
          for (int z = 0; z < 2; ++z) {
            const uint32_t* v32 = z ? vb : va;
            const int col = n0 + c * 64 + z * 32;
            if (col >= p.N_routed) continue;
            uint4* out =
                reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out_routed) + ((int64_t)ti.row0 + row) * p.ld_out + col);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              out[v] = make_uint4(ptx::pack_bf16x2(__uint_as_float(v32[8 * v + 0]), __uint_as_float(v32[8 * v + 1])),
                                  ptx::pack_bf16x2(__uint_as_float(v32[8 * v + 2]), __uint_as_float(v32[8 * v + 3])),
                                  ptx::pack_bf16x2(__uint_as_float(v32[8 * v + 4]), __uint_as_float(v32[8 * v + 5])),
                                  ptx::pack_bf16x2(__uint_as_float(v32[8 * v + 6]), __uint_as_float(v32[8 * v + 7])));
          }
        }
      }
      ++tl;
    }
  } else {
    // converters: this CTA's raw box [64 K x 128 N] -> two bf16 [64 K x 64 N]
    // boxes (128-byte swizzle, N-major); a warp step is 4 rows, a lane 16 codes
    const int cw = warp - 2 - kPairF8EpiWarps;
    const int sub_row = lane >> 3;
    const int col16 = lane & 7;
    int kg = 0;
    bool ok = true;
    for (int tile = cluster; ok && tile < total; tile += clusters) {
      TileInfo ti;
      if (!tile_at(p, span, tile, BN, ti)) continue;
      const int nk = p.K_routed / kF8BK;
      const int ncol = ti.nb * BN + (M == Mode::kSwiGLU ? 0 : (int)rank * 128);  // first raw column
      const int ksb = p.K_routed / 128, nsb = p.N_routed / 128;
      const float* scales = (M == Mode::kSwiGLU && rank == 1) ? p.scale_c : p.scale_b;
      for (int kb = 0; kb < nk; ++kb, ++kg) {
        const int s = kg % S;
        const int c = kg % CS;
        if (!ptx::wait_bounded(&rfull[s], (kg / S) & 1, abort_flag) ||
            (!kPairF8OneCommit && !ptx::wait_bounded(&cempty[c], ((kg / CS) & 1) ^ 1, abort_flag))) {
          raise_status(p.status, abort_flag, kStatusTimeout);
          ok = false;
          break;
        }
        const uint8_t* raw = stage0 + s * kPairF8StageBytes + kPairABytes;
        uint8_t* conv = conv0 + c * kPairF8ConvBytes;
        const float scale =
            scales[((int64_t)(ti.group - p.group_base) * ksb + (kb * kF8BK) / 128) * nsb + ncol / 128];
#pragma unroll
        for (int i = 0; i < 64 / (4 * kConvWarps); ++i) {
          const int k = cw * (64 / kConvWarps) + i * 4 + sub_row;  // 0..63
          const uint4 qv = *reinterpret_cast<const uint4*>(raw + k * 128 + col16 * 16);
          const uint2 v0 = e4m3x4_to_bf16x4(qv.x, scale), v1 = e4m3x4_to_bf16x4(qv.y, scale);
          const uint2 v2 = e4m3x4_to_bf16x4(qv.z, scale), v3 = e4m3x4_to_bf16x4(qv.w, scale);
          uint8_t* dst = conv + (col16 >> 2) * kF8BoxBytes + k * 128;
          const int ch = 2 * (col16 & 3);
          *reinterpret_cast<uint4*>(dst + ((ch ^ (k & 7)) << 4)) = make_uint4(v0.x, v0.y, v1.x, v1.y);
          *reinterpret_cast<uint4*>(dst + (((ch + 1) ^ (k & 7)) << 4)) = make_uint4(v2.x, v2.y, v3.x, v3.y);
        }
        // every lane's stores are made visible to the tensor cores' proxy, then
        // one arrival per warp (a remote arrival per lane would cost a cluster
        // transaction each)
        ptx::fence_proxy_async();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(ptx::mapa(&cfull[c], 0));
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem, kTmemCols);
  }
}

template <Mode M>
cudaError_t launch_pair_f8(const CUtensorMap& a_r, const CUtensorMap& b_r, const CUtensorMap& c_r,
                           const GemmParams& p, int grid, cudaStream_t stream) {
  const size_t smem = pair_f8_smem_bytes();
  cudaError_t err =
      cudaFuncSetAttribute(grouped_gemm_pair_f8_kernel<M>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  grid &= ~1;
  if (grid <= 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kPairF8Threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = MOE_PDL ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  err = cudaLaunchKernelEx(&cfg, grouped_gemm_pair_f8_kernel<M>, a_r, b_r, c_r, p);
  return err != cudaSuccess ? err : cudaGetLastError();
}

template <Mode M>
cudaError_t launch_pair(const CUtensorMap& a_r, const CUtensorMap& a_s, const CUtensorMap& b_r,
                        const CUtensorMap& b_s, const CUtensorMap& c_r, const CUtensorMap& c_s, const GemmParams& p,
                        int grid, cudaStream_t stream) {
  const size_t smem = pair_smem_bytes();
  cudaError_t err =
      cudaFuncSetAttribute(grouped_gemm_pair_kernel<M>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  grid &= ~1;  // whole clusters
  if (grid <= 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kPairThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = MOE_PDL ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  err = cudaLaunchKernelEx(&cfg, grouped_gemm_pair_kernel<M>, a_r, a_s, b_r, b_s, c_r, c_s, p);
  return err != cudaSuccess ? err : cudaGetLastError();
}

template <Mode M, bool F8, int N1 = 0>
cudaError_t launch(const CUtensorMap& a_r, const CUtensorMap& a_s, const CUtensorMap& b_r, const CUtensorMap& b_s,
                   const CUtensorMap& c_r, const CUtensorMap& c_s, const GemmParams& p, int grid,
                   cudaStream_t stream) {
  const size_t smem = smem_bytes<F8, N1>();
  cudaError_t err =
      cudaFuncSetAttribute(grouped_gemm_kernel<M, F8, N1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  if (grid <= 0) return cudaSuccess;
  cudaError_t e = launch_chained(grouped_gemm_kernel<M, F8, N1>, grid, dim3(kernel_threads<F8>()), smem, stream,
                                 a_r, a_s, b_r, b_s, c_r, c_s, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

int gemm_block_n_swiglu() { return Cfg<Mode::kSwiGLU>::BN; }
int gemm_block_n_down() { return Cfg<Mode::kDown>::BN; }

cudaError_t launch_grouped_swiglu(const CUtensorMap& tmA_r, const CUtensorMap& tmA_s, const CUtensorMap& tmW1_r,
                                  const CUtensorMap& tmW1_s, const CUtensorMap& tmW3_r, const CUtensorMap& tmW3_s,
                                  const GemmParams& p, int grid, cudaStream_t stream) {
  return launch<Mode::kSwiGLU, false>(tmA_r, tmA_s, tmW1_r, tmW1_s, tmW3_r, tmW3_s, p, grid, stream);
}

cudaError_t launch_grouped_down(const CUtensorMap& tmA, const CUtensorMap& tmW2_r, const CUtensorMap& tmW2_s,
                                const GemmParams& p, int grid, cudaStream_t stream) {
  return launch<Mode::kDown, false>(tmA, tmA, tmW2_r, tmW2_s, tmW2_r, tmW2_s, p, grid, stream);
}

cudaError_t launch_grouped_swiglu_pair(const CUtensorMap& tmA_r, const CUtensorMap& tmA_s, const CUtensorMap& tmW1_r,
                                       const CUtensorMap& tmW1_s, const CUtensorMap& tmW3_r, const CUtensorMap& tmW3_s,
                                       const GemmParams& p, int grid, cudaStream_t stream) {
  return launch_pair<Mode::kSwiGLU>(tmA_r, tmA_s, tmW1_r, tmW1_s, tmW3_r, tmW3_s, p, grid, stream);
}

cudaError_t launch_grouped_down_pair(const CUtensorMap& tmA, const CUtensorMap& tmW2_r, const CUtensorMap& tmW2_s,
                                     const GemmParams& p, int grid, cudaStream_t stream) {
  return launch_pair<Mode::kDown>(tmA, tmA, tmW2_r, tmW2_s, tmW2_r, tmW2_s, p, grid, stream);
}

cudaError_t launch_grouped_swiglu_pair_fp8(const CUtensorMap& tmA_r, const CUtensorMap& tmW1_r,
                                           const CUtensorMap& tmW3_r, const GemmParams& p, int grid,
                                           cudaStream_t stream) {
  return launch_pair_f8<Mode::kSwiGLU>(tmA_r, tmW1_r, tmW3_r, p, grid, stream);
}

cudaError_t launch_grouped_down_pair_fp8(const CUtensorMap& tmA, const CUtensorMap& tmW2_r, const GemmParams& p,
                                         int grid, cudaStream_t stream) {
  return launch_pair_f8<Mode::kDown>(tmA, tmW2_r, tmW2_r, p, grid, stream);
}

cudaError_t launch_grouped_swiglu_fp8(const CUtensorMap& tmA_r, const CUtensorMap& tmW1_r,
                                      const CUtensorMap& tmW3_r, const GemmParams& p, int grid,
                                      cudaStream_t stream, int short_rows) {
  if (short_rows == 2)
    return launch<Mode::kSwiGLU, true, 2>(tmA_r, tmA_r, tmW1_r, tmW1_r, tmW3_r, tmW3_r, p, grid, stream);
  if (short_rows == 1)
    return launch<Mode::kSwiGLU, true, 1>(tmA_r, tmA_r, tmW1_r, tmW1_r, tmW3_r, tmW3_r, p, grid, stream);
  return launch<Mode::kSwiGLU, true>(tmA_r, tmA_r, tmW1_r, tmW1_r, tmW3_r, tmW3_r, p, grid, stream);
}

cudaError_t launch_grouped_down_fp8(const CUtensorMap& tmA, const CUtensorMap& tmW2_r, const GemmParams& p, int grid,
                                    cudaStream_t stream, int short_rows) {
  if (short_rows == 2) return launch<Mode::kDown, true, 2>(tmA, tmA, tmW2_r, tmW2_r, tmW2_r, tmW2_r, p, grid, stream);
  if (short_rows == 1) return launch<Mode::kDown, true, 1>(tmA, tmA, tmW2_r, tmW2_r, tmW2_r, tmW2_r, p, grid, stream);
  return launch<Mode::kDown, true>(tmA, tmA, tmW2_r, tmW2_r, tmW2_r, tmW2_r, p, grid, stream);
}

}  // namespace moe
