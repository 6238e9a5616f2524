// router.cu -- gate GEMM on the tensor cores and the per-token top-k.
//
// Gate ("DeepSeek-V3's mixture-of-experts architecture explained", section
// "The architecture in one diagram"): logits = x Wg^T, a bias-free linear,
// x [T, d] bf16, Wg [E, d] bf16.  Selection: top-k of the logits then a
// softmax over the k; or, in group mode, sigmoid scores with a selection bias,
// 8 contiguous groups, group score = sum of the group's top-2, keep the top-4
// groups, top-k inside them, weights = 2.5 * s / sum(s).
//
// Kernel 1 (router_logits_kernel): one CTA per (128 tokens, EB experts, K
// split).
//   warp 0 : TMA producer (x tile [128 x 64] and Wg tile [EB x 64] per stage,
//            128-byte swizzle, 4-stage ring)
//   warp 1 : tcgen05.mma issuer, M=128 N=EB K=16, fp32 accumulator in TMEM;
//            each 64-wide K chunk goes to the next of four TMEM buffers
//   warps 2..: EB/16 drain warps per TMEM lane quarter, 16 columns each: each
//            finished chunk is read from TMEM and added into fp64 registers,
//            so a logit carries one fp32 rounding per 64 terms.  Without a K
//            split the fp32 logits [T, E] are written at the end; with one,
//            the fp64 partial sums [split, T, E] are, and a small kernel
//            adds them in split order (one thread per logit).  Small batches split K so that the grid still
//            covers the device.
// Kernel 2 (router_topk_kernel): one warp per token, k rounds of a warp
//   arg-max on (value desc, index asc), then the weights.
#include <cstdint>

#include "common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kRouterBM = 128;
constexpr int kRouterBK = 64;
#ifndef MOE_ROUTER_STAGES
#define MOE_ROUTER_STAGES 4
#endif
constexpr int kRouterStages = MOE_ROUTER_STAGES;

constexpr int kRouterAccBufs = 4;    // TMEM buffers: the MMA may run this many K groups ahead of the drain
#ifndef MOE_ROUTER_DRAIN_COLS
#define MOE_ROUTER_DRAIN_COLS 16
#endif
constexpr int kRouterDrainCols = MOE_ROUTER_DRAIN_COLS;  // accumulator columns per drain warp
// K chunks (64 deep each) the tensor core accumulates into one TMEM buffer
// before the drain reads it (a K group).
#ifndef MOE_ROUTER_MMA_CHUNKS
#define MOE_ROUTER_MMA_CHUNKS 1
#endif
constexpr int kRouterMmaChunks = MOE_ROUTER_MMA_CHUNKS;
// K groups a drain lane sums in fp32 before widening the sum
// to fp64 once: the widening runs on the XU pipe (16 per clock per SM) and
// bounds the kernel when done for every chunk.
#ifndef MOE_ROUTER_FP32_CHUNKS
#define MOE_ROUTER_FP32_CHUNKS 4
#endif
constexpr int kRouterFp32Chunks = MOE_ROUTER_FP32_CHUNKS;

template <int EB>
struct RouterSmem {
  static constexpr int kDrainWarps = 4 * (EB / kRouterDrainCols);
  static constexpr int kThreads = 64 + 32 * kDrainWarps;
  static_assert(kThreads <= 1024, "too many drain warps for one CTA");
  static constexpr uint32_t kABytes = kRouterBM * kRouterBK * 2;
  static constexpr uint32_t kBBytes = EB * kRouterBK * 2;
  static constexpr uint32_t kAccCols = kRouterAccBufs * EB;
  static_assert(kAccCols <= 512, "TMEM holds 512 columns");
  static constexpr uint32_t kTmemCols = kAccCols <= 128 ? 128 : (kAccCols <= 256 ? 256 : 512);
  static constexpr size_t kBytes = 1024 + kRouterStages * (kABytes + kBBytes) + 256;
};

// A drain lane's columns of one finished K group, read from TMEM.
__device__ __forceinline__ void drain_load(uint32_t taddr, uint32_t (&r)[16]) {
  ptx::tmem_ld16(taddr, r);
  ptx::tmem_ld_wait(r);
}
__device__ __forceinline__ void drain_load(uint32_t taddr, uint32_t (&r)[32]) {
  ptx::tmem_ld32(taddr, r);
  ptx::tmem_ld_wait(r);
}

template <int EB>
__global__ void __launch_bounds__(RouterSmem<EB>::kThreads, 1)
    router_logits_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_wg,
                         int T, int d, int E, int chunks_per_split, float* __restrict__ logits,
                         double* __restrict__ part, uint32_t* __restrict__ status) {
  using L = RouterSmem<EB>;
  constexpr int S = kRouterStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align_1024(smem_raw);
  uint8_t* sA = base;
  uint8_t* sB = base + S * L::kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + S * L::kBBytes);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + kRouterAccBufs;
  uint64_t* done = tempty + kRouterAccBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  __shared__ uint32_t never;  // a flag nobody raises (drain waits)

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kRouterBM;
  const int e0 = blockIdx.y * EB;
  const int kc0 = blockIdx.z * chunks_per_split;  // first K chunk of this split
  const int nk = min(d / kRouterBK, kc0 + chunks_per_split) - kc0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < kRouterAccBufs; ++b) {
      ptx::mbar_init(&tfull[b], 1);
      ptx::mbar_init(&tempty[b], 32 * L::kDrainWarps);
    }
    ptx::mbar_init(done, 1);
    *abort_flag = 0u;
    never = 0u;
    ptx::fence_barrier_init();
    ptx::fence_proxy_async();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, L::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dependency_wait();

  if (warp == 0) {
    if (lane == 0) {
      ptx::prefetch_tmap(&tm_x);
      ptx::prefetch_tmap(&tm_wg);
      const uint64_t pol = ptx::policy_evict_last();
      int issued = 0;
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % S;
        const uint32_t ph = (kb / S) & 1;
        if (!ptx::wait_bounded(&empty[s], ph ^ 1, abort_flag)) {
          raise_status(status, abort_flag, kStatusTimeout);
          break;
        }
        ptx::mbar_arrive_expect_tx(&full[s], L::kABytes + L::kBBytes);
        ptx::tma_load_2d(sA + s * L::kABytes, &tm_x, &full[s], (kc0 + kb) * kRouterBK, m0, pol);
        ptx::tma_load_2d(sB + s * L::kBBytes, &tm_wg, &full[s], (kc0 + kb) * kRouterBK, e0, pol);
        issued = kb + 1;
      }
      // every issued copy must land before the CTA may exit
      for (int kb = (issued > S ? issued - S : 0); kb < issued; ++kb)
        if (!ptx::wait_bounded(&full[kb % S], (kb / S) & 1, &never)) raise_status(status, abort_flag, kStatusTimeout);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_bf16(128, EB, false, false);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % S;
        const uint32_t ph = (kb / S) & 1;
        const int gi = kb / kRouterMmaChunks;  // K group
        const bool first = kb % kRouterMmaChunks == 0;
        const bool last = (kb + 1) % kRouterMmaChunks == 0 || kb + 1 == nk;
        const int b = gi % kRouterAccBufs;
        const uint32_t use = gi / kRouterAccBufs;
        if ((first && !ptx::wait_bounded(&tempty[b], (use & 1) ^ 1, abort_flag)) ||
            !ptx::wait_bounded(&full[s], ph, abort_flag)) {
          raise_status(status, abort_flag, kStatusTimeout);
          break;
        }
        ptx::tc_fence_after();
        const uint32_t a0 = ptx::smem_u32(sA + s * L::kABytes);
        const uint32_t b0 = ptx::smem_u32(sB + s * L::kBBytes);
#pragma unroll
        for (int kk = 0; kk < kRouterBK / 16; ++kk)
          ptx::mma_bf16(tmem + b * EB, ptx::sdesc_sw128(a0 + kk * 32, 16, 1024),
                        ptx::sdesc_sw128(b0 + kk * 32, 16, 1024), idesc, (kk > 0 || !first) ? 1u : 0u);
        ptx::mma_commit(&empty[s]);
        if (last) ptx::mma_commit(&tfull[b]);
      }
      ptx::mma_commit(done);
      if (!ptx::wait_bounded(done, 0, &never)) raise_status(status, abort_flag, kStatusTimeout);
    }
  } else {
    const int q = warp & 3;                             // TMEM lane quarter this warp may access
    const int c0 = ((warp - 2) >> 2) * kRouterDrainCols;  // first accumulator column it drains
    const int row = q * 32 + lane;
    double acc[kRouterDrainCols];
    float part32[kRouterDrainCols];
#pragma unroll
    for (int j = 0; j < kRouterDrainCols; ++j) {
      acc[j] = 0.0;
      part32[j] = 0.0f;
    }
    bool ok = true;
    const int ng = (nk + kRouterMmaChunks - 1) / kRouterMmaChunks;  // K groups
    for (int kb = 0; kb < ng; ++kb) {
      const int b = kb % kRouterAccBufs;
      const uint32_t use = kb / kRouterAccBufs;
      if (!ptx::wait_bounded(&tfull[b], use & 1, abort_flag)) {
        raise_status(status, abort_flag, kStatusTimeout);
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      uint32_t r[kRouterDrainCols];
      drain_load(tmem + ((uint32_t)(q * 32) << 16) + b * EB + c0, r);
      ptx::tc_fence_before();
      ptx::mbar_arrive(&tempty[b]);
      if (kRouterFp32Chunks == 1) {
#pragma unroll
        for (int i = 0; i < kRouterDrainCols; ++i) acc[i] += (double)__uint_as_float(r[i]);
      } else {
#pragma unroll
        for (int i = 0; i < kRouterDrainCols; ++i) part32[i] += __uint_as_float(r[i]);
        if ((kb + 1) % kRouterFp32Chunks == 0 || kb + 1 == ng) {
#pragma unroll
          for (int i = 0; i < kRouterDrainCols; ++i) {
            acc[i] += (double)part32[i];
            part32[i] = 0.0f;
          }
        }
      }
    }
    if (ok && m0 + row < T) {
      if (part == nullptr) {
        float4* out = reinterpret_cast<float4*>(logits + (size_t)(m0 + row) * E + e0 + c0);
#pragma unroll
        for (int j = 0; j < kRouterDrainCols / 4; ++j)
          out[j] = make_float4((float)acc[4 * j], (float)acc[4 * j + 1], (float)acc[4 * j + 2], (float)acc[4 * j + 3]);
      } else {
        double2* out = reinterpret_cast<double2*>(part + ((size_t)blockIdx.z * T + m0 + row) * E + e0 + c0);
#pragma unroll
        for (int j = 0; j < kRouterDrainCols / 2; ++j) out[j] = make_double2(acc[2 * j], acc[2 * j + 1]);
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, L::kTmemCols);
  }
}

// K-split gate GEMM: logits[i] = (float) sum_s part[s][i] over the T*E
// logits, the splits added in order; one thread per logit, loads issued
// several splits ahead of the adds.
__global__ void __launch_bounds__(256)
    router_split_sum_kernel(const double* __restrict__ part, int splits, int64_t n, float* __restrict__ logits) {
  grid_dependency_wait();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  double a = 0.0;
#pragma unroll 8
  for (int sp = 0; sp < splits; ++sp) a += __ldg(part + sp * n + i);
  logits[i] = (float)a;
}

// ---------------------------------------------------------------- top-k
struct Cand {
  float key;   // selection score
  int idx;     // expert index (INT32_MAX when none)
  float aux;   // carried payload (sigmoid score in group mode)
};

__device__ __forceinline__ Cand warp_best(Cand c) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    Cand x;
    x.key = __shfl_xor_sync(0xffffffffu, c.key, o);
    x.idx = __shfl_xor_sync(0xffffffffu, c.idx, o);
    x.aux = __shfl_xor_sync(0xffffffffu, c.aux, o);
    if (key_before(x.key, x.idx, c.key, c.idx)) c = x;
  }
  return c;
}

// NV = values per lane (expert e lives in lane e % 32, slot e / 32).
template <int NV>
__global__ void __launch_bounds__(128)
    router_topk_kernel(const float* __restrict__ logits, const float* __restrict__ bias, const uint8_t* __restrict__ allowed, int T, int E, int k,
                       int route, int n_group,
                       int topk_group, int group_topn, float route_scale, int32_t* __restrict__ topk_idx,
                       float* __restrict__ topk_w) {
  __shared__ float sel_sh[4][NV * 32];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 4 + warp;
  grid_dependency_wait();
  if (t >= T) return;
  const float NEG = -__int_as_float(0x7f800000);  // -inf

  float key[NV], aux[NV];
  uint32_t taken = 0;  // bit v: slot v of this lane is out of the running
  const float* lrow = logits + (size_t)t * E;
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    const int e = v * 32 + lane;
    if (e < E) {
      // device-limited routing: experts this device does not hold get -inf
      const float l = (allowed && !allowed[e]) ? NEG : lrow[e];
      if (route == 0) {
        key[v] = l;
        aux[v] = l;
      } else {
        const float s = 1.0f / (1.0f + expf(-l));
        aux[v] = s;
        key[v] = s + (bias ? bias[e] : 0.0f);
      }
    } else {
      key[v] = NEG;
      aux[v] = 0.0f;
      taken |= 1u << v;
    }
  }

  if (route == 1) {
    // group scores: sum of the group's top `group_topn` selection scores
    float* sh = sel_sh[warp];
#pragma unroll
    for (int v = 0; v < NV; ++v)
      if (v * 32 + lane < E) sh[v * 32 + lane] = key[v];
    __syncwarp();
    const int gsize = E / n_group;
    float gscore = NEG;
    if (lane < n_group) {
      uint32_t used_lo = 0, used_hi = 0;  // up to 64 members tracked per pass
      float acc = 0.0f;
      for (int p = 0; p < group_topn; ++p) {
        float bv = NEG;
        int bi = -1;
        for (int i = 0; i < gsize; ++i) {
          const bool used = (i < 32) ? ((used_lo >> i) & 1u) : (i < 64 ? ((used_hi >> (i - 32)) & 1u) : 0u);
          if (used) continue;
          const float v = sh[lane * gsize + i];
          if (bi < 0 || v > bv) {
            bv = v;
            bi = i;
          }
        }
        if (bi < 32) used_lo |= 1u << bi; else used_hi |= 1u << (bi - 32);
        acc += bv;
      }
      gscore = acc;
    }
    // keep the best topk_group groups (score desc, group index asc)
    uint32_t kept = 0;
    Cand g{lane < n_group ? gscore : NEG, lane < n_group ? lane : 0x7fffffff, 0.0f};
    for (int r = 0; r < topk_group; ++r) {
      const Cand b = warp_best(g);
      kept |= 1u << b.idx;
      if (lane == b.idx) g = Cand{NEG, 0x7fffffff, 0.0f};
    }
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const int e = v * 32 + lane;
      if (e < E && !((kept >> (e / gsize)) & 1u)) taken |= 1u << v;
    }
  }

  // k rounds of warp arg-max; lane j keeps slot j
  float my_key = 0.0f, my_aux = 0.0f;
  int my_idx = 0;
  float top_key = 0.0f;
  for (int j = 0; j < k; ++j) {
    Cand c{NEG, 0x7fffffff, 0.0f};
#pragma unroll
    for (int v = 0; v < NV; ++v)
      if (!((taken >> v) & 1u) && key_before(key[v], v * 32 + lane, c.key, c.idx)) c = Cand{key[v], v * 32 + lane, aux[v]};
    const Cand b = warp_best(c);
    if (j == 0) top_key = b.key;
    if (lane == j) {
      my_key = b.key;
      my_idx = b.idx;
      my_aux = b.aux;
    }
    if ((b.idx & 31) == lane) taken |= 1u << (b.idx >> 5);
  }

  float num;
  if (route == 0)
    num = (lane < k) ? expf(my_key - top_key) : 0.0f;
  else
    num = (lane < k) ? my_aux : 0.0f;
  float den = num;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  if (lane < k) {
    topk_idx[(size_t)t * k + lane] = my_idx;
    topk_w[(size_t)t * k + lane] = (route == 0 ? 1.0f : route_scale) * (num / den);
  }
}

template <int EB>
cudaError_t launch_router_logits(const CUtensorMap& tm_x, const CUtensorMap& tm_wg, int T, int d, int E, int splits,
                                 float* logits, double* part, uint32_t* status, cudaStream_t stream) {
  const size_t smem = RouterSmem<EB>::kBytes;
  cudaError_t err = cudaFuncSetAttribute(router_logits_kernel<EB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
  if (err != cudaSuccess) return err;
  const int nk = d / kRouterBK;
  if (splits < 1 || splits > nk || (splits > 1 && part == nullptr)) return cudaErrorInvalidValue;
  const int cps = (nk + splits - 1) / splits;
  if ((nk + cps - 1) / cps != splits) return cudaErrorInvalidValue;  // a split would get no chunk
  dim3 grid((T + kRouterBM - 1) / kRouterBM, E / EB, splits);
  err = launch_chained(router_logits_kernel<EB>, grid, dim3(RouterSmem<EB>::kThreads), smem, stream, tm_x, tm_wg, T,
                       d, E, cps, logits, splits > 1 ? part : nullptr, status);
  return err != cudaSuccess ? err : cudaGetLastError();
}

template <int NV>
cudaError_t launch_topk_nv(const float* logits, const float* bias, const uint8_t* allowed, const RouteParams& rp,
                           int T, int E, int k, int32_t* idx, float* w, cudaStream_t stream) {
  const cudaError_t err =
      launch_chained(router_topk_kernel<NV>, dim3((T + 3) / 4), dim3(128), 0, stream, logits, bias, allowed, T, E, k,
                     rp.route, rp.n_group, rp.topk_group, rp.group_topn, rp.route_scale, idx, w);
  return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace

#ifndef MOE_ROUTER_EB
#define MOE_ROUTER_EB 64
#endif

int router_expert_block(int E) {
  if (MOE_ROUTER_EB >= 128 && E % 128 == 0) return 128;
  if (E % 64 == 0) return 64;
  if (E % 32 == 0) return 32;
  return 0;
}

int router_splits(int64_t T, int d, int E, int sms) {
  const int eb = router_expert_block(E);
  const int nk = d / kRouterBK;
  if (eb == 0 || T <= 0 || nk <= 1) return 1;
  sms = sms < 1 ? 1 : (sms > kRouterMaxSms ? kRouterMaxSms : sms);
  const int64_t ctas = (T + kRouterBM - 1) / kRouterBM * (E / eb);
  if (ctas * 2 > sms) return 1;
  const int want = (int)(sms / ctas);
  const int cps = (nk + want - 1) / want;
  return (nk + cps - 1) / cps;
}

cudaError_t launch_router_logits(const CUtensorMap& tm_x, const CUtensorMap& tm_wg, int T, int d, int E, int splits,
                                 float* logits, double* part, uint32_t* status, cudaStream_t stream) {
  switch (router_expert_block(E)) {
#if MOE_ROUTER_EB >= 128
    case 128: return launch_router_logits<128>(tm_x, tm_wg, T, d, E, splits, logits, part, status, stream);
#endif
    case 64: return launch_router_logits<64>(tm_x, tm_wg, T, d, E, splits, logits, part, status, stream);
    case 32: return launch_router_logits<32>(tm_x, tm_wg, T, d, E, splits, logits, part, status, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_router_topk(float* logits, const double* part, int splits, const float* bias,
                               const uint8_t* allowed, const RouteParams& rp, int T, int E, int k, int32_t* idx,
                               float* w, cudaStream_t stream) {
  const int nv = (E + 31) / 32;
  if (splits > 1) {
    const int64_t n = (int64_t)T * E;
    const cudaError_t err = launch_chained(router_split_sum_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0,
                                           stream, part, splits, n, logits);
    if (err != cudaSuccess) return err;
  }
#define MOE_TOPK(N) return launch_topk_nv<N>(logits, bias, allowed, rp, T, E, k, idx, w, stream)
  if (nv <= 1) MOE_TOPK(1);
  if (nv <= 2) MOE_TOPK(2);
  if (nv <= 4) MOE_TOPK(4);
  if (nv <= 8) MOE_TOPK(8);
  if (nv <= 16) MOE_TOPK(16);
  if (nv <= 32) MOE_TOPK(32);
#undef MOE_TOPK
  return cudaErrorInvalidValue;
}

}  // namespace moe
