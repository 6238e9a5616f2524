/*
 * moe.h -- C ABI of libmoe: forward pass of one DeepSeek-V3-style
 * mixture-of-experts feed-forward layer on one NVIDIA B200 (sm_100a).
 *
 * What the layer computes (sources are the web pages this library follows):
 *   logits = x Wg^T                       gate, a linear layer without bias
 *       ("DeepSeek-V3's mixture-of-experts architecture explained", n4n.ai,
 *        section "The architecture in one diagram", simplified block code)
 *   idx, w = route(logits)                top-k then softmax over the k
 *       (same section), or the sigmoid group-limited rule with selection
 *       bias (MOE_ROUTE_SIGMOID_GROUP, below)
 *   expert(x) = W2^T (silu(x W1) * (x W3))   SwiGLU, "All 5 steps" of
 *       "DeepSeek-V3.2-Exp / Mixture of experts / Shared expert" (atlas page)
 *   y[t] = sum_j w[t,j] expert_{idx[t,j]}(x[t]) + shared(x[t])
 *       (atlas page, "Code" section, MoE forward block: per-expert token
 *        lists from bincount/where, an fp32 accumulator, then the shared
 *        expert added to every token)
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller, contiguous
 *    row-major, 16-byte aligned (the tensor-memory-accelerator copies require
 *    it).  The library never allocates, frees or keeps a pointer after a call
 *    returns.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; 0 = legacy default
 *    stream) and never synchronise the host, except moe_check_device_status.
 *    A moe_forward call on a capturing stream is recorded into the CUDA graph
 *    (kernels and memsets only); replays read whatever the captured buffers
 *    hold at replay time.
 *  - Arguments are validated on the host before any launch; an invalid call
 *    returns an error and launches nothing.  T == 0 is valid and does nothing.
 *  - Dtypes: x, Wg, the shared expert and bf16 routed weights are bfloat16.
 *    FP8 routed weights are OCP e4m3 codes (one byte) with one fp32 scale per
 *    128 x 128 block.  Logits, routing weights and the combine accumulate in
 *    fp32; all tensor-core contractions accumulate in fp32.
 *  - `ws` is a caller-allocated device workspace of at least
 *    moe_workspace_size(shape) bytes (256-byte aligned).  Its first 4 bytes
 *    are the device status word (see moe_check_device_status); the rest is
 *    scratch whose contents do not survive between calls.  Calls that overlap
 *    on the device must use different workspaces.
 *  - Identical inputs give bit-identical outputs (no floating-point atomics).
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,    /* null required pointer, misaligned pointer, bad size */
  MOE_ERR_UNSUPPORTED = 2,    /* shape/dtype combination this library does not implement */
  MOE_ERR_WORKSPACE = 3,      /* ws null or smaller than moe_workspace_size() */
  MOE_ERR_CUDA = 4,           /* a CUDA runtime/driver call or a launch failed */
  MOE_ERR_DEVICE_TIMEOUT = 5, /* a kernel's bounded wait gave up (reported by moe_check_device_status) */
  MOE_ERR_DEVICE_BOUNDS = 6   /* an expert index outside [0, E) was seen and skipped */
} moe_status;

typedef enum { MOE_BF16 = 0, MOE_E4M3 = 1, MOE_F32 = 2 } moe_dtype;

typedef enum {
  /* top-k of the logits (descending, lowest index first on ties), softmax
   * over the k selected logits (n4n.ai page, "The architecture in one
   * diagram"). */
  MOE_ROUTE_TOPK_SOFTMAX = 0,
  /* s = sigmoid(logit), sel = s + bias; experts form n_group contiguous
   * groups of E/n_group; a group's score is the sum of its group_topn best
   * sel; the topk_group best groups are kept; the k best sel among their
   * experts are chosen; w = route_scale * s / sum(s) over the chosen
   * (DeepSeek-V3 group-limited routing; the pages only outline it: Baidu
   * page "Hierarchical Dynamic Routing", freedom251 page "How V3 balances
   * expert traffic"). */
  MOE_ROUTE_SIGMOID_GROUP = 1
} moe_route;

typedef struct {
  int64_t T;            /* tokens (rows of x); 0 <= T, T*k < 2^31 */
  int32_t d;            /* model width (7168); multiple of 128 */
  int32_t E;            /* routed experts (256); multiple of 32, <= 1024 */
  int32_t k;            /* experts per token (8); 1 <= k <= min(E, 32) */
  int32_t inter;        /* routed expert width (moe_inter_dim, 2048); multiple of 128 */
  int32_t shared_inter; /* shared expert width (n_shared x moe_inter = 2048); 0 = none; multiple of 128 */
  int32_t route;        /* moe_route */
  int32_t n_group;      /* group mode: groups (8); divides E; E/n_group <= 64; n_group <= 32 */
  int32_t topk_group;   /* group mode: kept groups (4); topk_group*E/n_group >= k */
  int32_t group_topn;   /* group mode: experts summed per group score (2) */
  float route_scale;    /* group mode: weight scale (2.5); ignored in top-k/softmax mode */
  int32_t w_dtype;      /* routed expert weights: MOE_BF16 or MOE_E4M3 */
  int32_t y_dtype;      /* output y: MOE_F32 (the pages' fp32 accumulator) or MOE_BF16 */
} moe_shape;

/* Bytes of workspace every entry point below needs for `shape` (the maximum
 * over them).  Returns 0 when the shape is invalid or unsupported. */
size_t moe_workspace_size(const moe_shape* shape);

/* Router: logits = x Wg^T in fp32 (tensor cores; each 64-term partial sum is
 * accumulated in fp64), then the k experts per token and their weights.
 *   x        [T, d] bf16            Wg [E, d] bf16
 *   bias     [E] fp32 selection bias, group mode only (may be NULL = zeros)
 *   topk_idx [T, k] int32 out, slots in descending score order
 *   topk_w   [T, k] fp32 out
 *   logits   [T, E] fp32 out, optional (NULL: kept in the workspace)
 * Source: n4n.ai page "The architecture in one diagram" (gate, topk, softmax). */
moe_status moe_router_topk(const moe_shape* shape, const void* x, const void* Wg, const float* bias,
                           int32_t* topk_idx, float* topk_w, float* logits, void* ws, size_t ws_bytes,
                           void* stream);

/* Device-limited routing (n4n page, "Why 256 experts with top-8 routing?",
 * device-limited routing code): experts with allowed[e] == 0 (those not held
 * by this device) get -inf added to their logit before the top-k; then the
 * top-k / softmax rule of moe_router_topk.  allowed [E] uint8 device array.
 * Top-k/softmax mode only (MOE_ERR_UNSUPPORTED otherwise).  With fewer than k
 * allowed experts the remaining slots hold the lowest-index masked experts
 * with weight 0. */
moe_status moe_router_topk_limited(const moe_shape* shape, const void* x, const void* Wg, const uint8_t* allowed,
                                   int32_t* topk_idx, float* topk_w, float* logits, void* ws, size_t ws_bytes,
                                   void* stream);

/* Expert-utilisation monitor (n4n page, "Where the architecture struggles",
 * log_expert_utilization): from per-expert counts [E] (moe_permute,
 * moe_forward's counts_out) computes utilisation[e] = counts[e] / sum(counts)
 * (fp32) and flags[e] = +1 when counts[e] > 2x the mean count, -1 when below
 * 0.1x the mean, else 0 (decided exactly: counts*E > 2*total,
 * 10*counts*E < total).  Either output may be NULL (not both). */
moe_status moe_expert_utilisation(const moe_shape* shape, const int32_t* counts, float* utilisation, int32_t* flags,
                                  void* stream);

/* Dispatch: counts = bincount(topk_idx, minlength=E); offsets = exclusive
 * prefix sum (E+1 entries); the permuted order lists experts ascending and,
 * within an expert, its (token, slot) entries ascending -- the order of the
 * atlas page's torch.where(indices == i) ("Code" section, MoE forward block).
 *   perm_token [T*k] int32 out: token at permuted position r
 *   row_of     [T*k] int32 out: permuted position of entry (t, j) at t*k + j
 *   x, x_perm  optional pair: when both are non-NULL, x_perm [T*k, d] bf16
 *              receives x[perm_token[r]] at row r, for r < offsets[E].
 * An index outside [0, E) is skipped (its row_of is -1) and raises
 * MOE_ERR_DEVICE_BOUNDS in the workspace status word; the skipped entries
 * take no permuted position, so perm_token and x_perm hold offsets[E] < T*k
 * rows and their tails are left untouched.  With T == 0 only counts and
 * offsets are written (all zero) and the other pointers may be NULL. */
moe_status moe_permute(const moe_shape* shape, const int32_t* topk_idx, int32_t* counts, int32_t* offsets,
                       int32_t* perm_token, int32_t* row_of, const void* x, void* x_perm, void* ws,
                       size_t ws_bytes, void* stream);

/* moe_permute for callers that cannot allocate device memory -- for example a
 * plugin inside another runtime that is handed only its input and output
 * buffers.  Same arguments and results as moe_permute, minus the workspace:
 * the scratch (per-block histograms and bases, a status word) lives in a
 * 512 KiB array inside the library that every GPU loading the library holds
 * until the process exits.  No counterpart on the pages; it exists only for
 * such callers.
 *  - Limit: ceil(T / 256) * E <= 65472 (e.g. T <= 65280 with E = 256);
 *    larger shapes return MOE_ERR_UNSUPPORTED and launch nothing.
 *  - Every call looks up the array's device address in the calling thread's
 *    current context (the array has one copy per context that loads the
 *    library: the device's primary context, or a context the host runtime
 *    made itself); the first call in a context may load the library's device
 *    code there, so make that first call before any stream capture.
 *  - Allocates nothing (no cudaMalloc/cudaFree, no allocating library call).
 *  - All calls share the one array and it keeps the last call's contents:
 *    calls that overlap on the GPU (other streams, other threads) race;
 *    serialise them.
 *  - Out-of-range indices are skipped (row_of = -1); there is no workspace,
 *    so no status word is reported to the caller. */
moe_status moe_permute_noalloc(const moe_shape* shape, const int32_t* topk_idx, int32_t* counts, int32_t* offsets,
                               int32_t* perm_token, int32_t* row_of, const void* x, void* x_perm, void* stream);

/* Grouped SwiGLU experts over the permuted rows plus the shared expert:
 *   for each expert e and each permuted row r in [offsets[e], offsets[e+1]):
 *     Y_perm[r] = bf16( (bf16(silu(x_perm[r] W1[e]) * (x_perm[r] W3[e]))) W2[e] )
 *   for each token t (shared expert, when shape->shared_inter > 0):
 *     Y_shared[t] = (bf16(silu(x[t] W1s) * (x[t] W3s))) W2s   in fp32
 *   x [T, d] bf16; x_perm [T*k, d] bf16 (from moe_permute); offsets [E+1]
 *   W1, W3 [E, d, inter], W2 [E, inter, d]: bf16, or e4m3 codes when
 *     w_dtype == MOE_E4M3 with fp32 block scales s1, s3 [E, d/128, inter/128]
 *     and s2 [E, inter/128, d/128] (dequantised value = code * scale)
 *   W1s, W3s [d, shared_inter], W2s [shared_inter, d] bf16 (NULL when none)
 *   Y_perm [T*k, d] bf16 out; Y_shared [T, d] fp32 out (NULL when none)
 * Source: atlas page "All 5 steps" and the expert forward block of its "Code"
 * section (silu and
 * product in fp32, h cast to the activation dtype before W2). */
moe_status moe_grouped_swiglu(const moe_shape* shape, const void* x, const void* x_perm, const int32_t* offsets,
                              const void* W1, const void* W3, const void* W2, const float* s1, const float* s3,
                              const float* s2, const void* W1s, const void* W3s, const void* W2s, void* Y_perm,
                              float* Y_shared, void* ws, size_t ws_bytes, void* stream);

/* Combine: y[t] = Y_shared[t] + sum_j topk_w[t,j] * Y_perm[row_of[t*k+j]],
 * summed in fp32 in slot order, written as shape->y_dtype.  Y_shared may be
 * NULL (no shared expert).  Source: atlas page, "Code" section, MoE forward
 * block. */
moe_status moe_combine(const moe_shape* shape, const void* Y_perm, const float* Y_shared, const int32_t* row_of,
                       const float* topk_w, void* y, void* stream);

/* Backward of the combine (first step of the layer's backward pass).  The
 * pages print no backward arithmetic; this is the derivative of the combine
 * above with the expert selection held fixed.  For every (t, j) with
 * r = row_of[t*k+j] >= 0:
 *   dO_perm[r] = bf16(topk_w[t,j] * dy[t])     (the gradient of the routed
 *                expert output, in the permuted row order of moe_permute)
 *   dw[t,j]    = dy[t] . Y_perm[r]             (fp32 sum, fixed order)
 * and dw[t,j] = 0 where r < 0.
 *   dy [T, d] fp32; Y_perm [T*k, d] bf16 (the forward's routed expert
 *   outputs, as moe_grouped_swiglu writes them); row_of [T*k], topk_w [T, k]
 *   as moe_permute / moe_router_topk return them; dO_perm [T*k, d] bf16 out
 *   (rows not addressed by row_of are not written); dw [T, k] fp32 out. */
moe_status moe_combine_backward(const moe_shape* shape, const float* dy, const void* Y_perm, const int32_t* row_of,
                                const float* topk_w, void* dO_perm, float* dw, void* stream);

/* Backward of the routing weights with the selection held fixed: dlogits
 * [T, E] fp32 out, zero outside each token's k selected experts.
 *   top-k/softmax mode:  dl_j = w_j (dw_j - sum_i w_i dw_i)
 *   group mode:          s = sigmoid(logit), Z = sum of the selected s,
 *                        dl_j = route_scale (dw_j / Z - sum_i dw_i s_i / Z^2) s_j (1 - s_j)
 * (derivatives of the weight rules of moe_route; the selection bias moves
 * only the selection and gets no gradient).  logits [T, E] fp32 and
 * topk_idx, topk_w [T, k] as moe_router_topk returns them; dw [T, k] fp32 as
 * moe_combine_backward returns it.  An index outside [0, E) gets no
 * gradient. */
moe_status moe_router_backward(const moe_shape* shape, const float* logits, const int32_t* topk_idx,
                               const float* topk_w, const float* dw, float* dlogits, void* stream);

/* The shared expert alone (atlas page, "Code" section, MoE forward block:
 * y += shared_experts(x)): Y_shared[t] = (bf16(silu(x[t] W1s) * (x[t] W3s)))
 * W2s in fp32 for the T tokens of x, with the grouped-GEMM kernels of
 * moe_grouped_swiglu.  Used by the all-to-all flavour of expert parallelism,
 * where each rank's routed rows run on other ranks and its shared expert on
 * its own tokens.  shape->shared_inter must be > 0; x [T, d] bf16; W1s, W3s
 * [d, shared_inter], W2s [shared_inter, d] bf16; Y_shared [T, d] fp32 out;
 * ws as for moe_forward (moe_workspace_size bytes). */
moe_status moe_shared_expert(const moe_shape* shape, const void* x, const void* W1s, const void* W3s,
                             const void* W2s, float* Y_shared, void* ws, size_t ws_bytes, void* stream);

/* All-to-all expert parallelism, the receiving side's regrouping (n4n page,
 * "Why 256 experts with top-8 routing?": hidden states travel to the devices
 * that hold their experts).  A rank holding E_local experts receives from each
 * of n_src source ranks, in source order, that source's rows for its experts
 * in expert order; recv_counts [n_src, E_local] int32 (device) gives how many
 * rows each source sends for each local expert.  Writes, for the R =
 * sum(recv_counts) received rows:
 *   offsets_local [E_local + 1]: expert-major segment starts (R at the end),
 *   to_expert_major [R]: the received (source-major) row at expert-major
 *                        position p,
 *   to_source_major [R]: the expert-major position of received row r
 * (expert-major order: experts ascending, then sources, then each source's
 * order), so that moe_gather_rows through them moves rows either way.
 * n_src * E_local <= 1024. */
moe_status moe_ep_regroup_layout(int n_src, int E_local, const int32_t* recv_counts, int32_t* offsets_local,
                                 int32_t* to_expert_major, int32_t* to_source_major, void* stream);

/* Row gather: dst[r] = src[index[r]] for r < rows, rows of d bf16 (d a
 * multiple of 8), 16-byte aligned device buffers.  Indices must address rows
 * of src (not checked). */
moe_status moe_gather_rows(const void* src, const int32_t* index, int64_t rows, int d, void* dst, void* stream);

/* Gradient of the whole layer (training): for the loss sum(dy * y) with
 * y = moe_forward(...), the gradients with respect to x, Wg, W1, W3, W2 and
 * the shared expert's weights, the expert selection held fixed (it is
 * piecewise constant in the inputs; the selection bias only moves it and gets
 * no gradient).  The pages print no backward arithmetic (the n4n page's
 * "Training infrastructure that made this possible" only names training);
 * this is the chain rule through the forward steps of the atlas page ("All 5
 * steps", and the MoE forward block of its "Code" section):
 *   dO = w dy (per routed slot),  dw = dy . o,  dl from dw through the weight
 *   rule (as moe_router_backward),
 *   dH = dO W2^T,  dG = dH u silu'(g),  dU = dH silu(g),
 *   dW2 = H^T dO,  dW1 = X^T dG,  dW3 = X^T dU   (each expert over its rows),
 *   dx = sum over slots of (dG W1^T + dU W3^T) + the shared expert's input
 *        gradient + dl Wg,   dWg = dl^T x,
 * with silu'(g) = sigmoid(g) (1 + g (1 - sigmoid(g))).  The call recomputes
 * the forward (routing, g, u, H and the expert outputs; they stay in the
 * workspace) and then runs the backward steps, all on the device, with no
 * host synchronisation and no atomics (deterministic results).
 *   x, Wg, bias, W1, W3, W2, W1s, W3s, W2s: as moe_forward (bf16 experts only:
 *     w_dtype must be MOE_BF16, else MOE_ERR_UNSUPPORTED)
 *   dy [T, d] fp32: gradient of the layer output
 *   outputs, all in shape->y_dtype (fp32 or bf16), row-major, every element
 *   written (experts no token chose get zero):
 *     dx [T, d]; dWg [E, d]; dW1, dW3 [E, d, inter]; dW2 [E, inter, d];
 *     dW1s, dW3s [d, shared_inter], dW2s [shared_inter, d] (NULL when there is
 *     no shared expert)
 *   ws: caller-owned device workspace of moe_backward_workspace_size(shape)
 *     bytes, 256-byte aligned (its head holds the status word that
 *     moe_check_device_status reads).
 * Errors as moe_forward. */
size_t moe_backward_workspace_size(const moe_shape* shape);
moe_status moe_backward(const moe_shape* shape, const void* x, const void* Wg, const float* bias, const void* W1,
                        const void* W3, const void* W2, const void* W1s, const void* W3s, const void* W2s,
                        const float* dy, void* dx, void* dWg, void* dW1, void* dW3, void* dW2, void* dW1s, void* dW3s,
                        void* dW2s, void* ws, size_t ws_bytes, void* stream);

/* The same gradient in two calls, for a training step that keeps the
 * forward's state instead of recomputing it (the HBM holds it easily):
 * moe_forward_train is moe_forward (y in shape->y_dtype, the same value)
 * that also leaves in `ws` -- a moe_backward_workspace_size workspace -- the
 * logits, the routing, the permuted rows, g and u (bf16), H and the routed
 * expert outputs; moe_backward_saved then computes every gradient from that
 * state (same results as moe_backward on the same inputs).  Between the two
 * calls the workspace must not be reused, and x, Wg, the weights and the
 * shape must be the ones the forward saw.  Arguments, layouts and errors as
 * moe_forward / moe_backward; moe_backward_saved takes no bias (the routing
 * is the saved one). */
moe_status moe_forward_train(const moe_shape* shape, const void* x, const void* Wg, const float* bias,
                             const void* W1, const void* W3, const void* W2, const void* W1s, const void* W3s,
                             const void* W2s, void* y, void* ws, size_t ws_bytes, void* stream);
moe_status moe_backward_saved(const moe_shape* shape, const void* x, const void* Wg, const void* W1, const void* W3,
                              const void* W2, const void* W1s, const void* W3s, const void* W2s, const float* dy,
                              void* dx, void* dWg, void* dW1, void* dW3, void* dW2, void* dW1s, void* dW3s,
                              void* dW2s, void* ws, size_t ws_bytes, void* stream);

/* The whole layer: router, dispatch, grouped experts, shared expert and
 * combine, with no host synchronisation.
 *   y [T, d] out (fp32 or bf16 per shape->y_dtype)
 *   topk_idx_out [T, k], topk_w_out [T, k], counts_out [E]: optional copies
 *   of the routing (NULL = not returned). */
moe_status moe_forward(const moe_shape* shape, const void* x, const void* Wg, const float* bias, const void* W1,
                       const void* W3, const void* W2, const float* s1, const float* s3, const float* s2,
                       const void* W1s, const void* W3s, const void* W2s, void* y, int32_t* topk_idx_out,
                       float* topk_w_out, int32_t* counts_out, void* ws, size_t ws_bytes, void* stream);

/* One rank's share of the expert-parallel layer (atlas page, "Code" section:
 * the MoE constructor block gives rank r the experts
 * [r*E/ep_size, (r+1)*E/ep_size) and a tensor-parallel shared expert; the MoE
 * forward block adds the local experts' weighted outputs and this rank's
 * shared-expert partial into y, then all-reduces y over the ranks):
 *   y[t] = sum over slots j with e = topk_idx[t,j] local of topk_w[t,j] * expert_e(x[t])
 *        + shared_r(x[t]),
 *   shared_r = the shared expert restricted to hidden features
 *              [r*Is/ep_size, (r+1)*Is/ep_size) (Is = shape->shared_inter).
 * Summing y over ep_rank = 0..ep_size-1 gives moe_forward's y; the caller does
 * that sum (the all-reduce, e.g. NCCL).  Routing runs over all E experts on
 * every rank (same inputs, same indices).
 *   shape: the whole layer's shape (E experts, shared_inter Is).
 *   W1, W3 [E/ep_size, d, inter], W2 [E/ep_size, inter, d] (and s1, s3, s2
 *     [E/ep_size, ...] for MOE_E4M3): this rank's experts only, slice 0 =
 *     expert r*E/ep_size.
 *   W1s, W3s [d, Is/ep_size], W2s [Is/ep_size, d]: this rank's columns of the
 *     shared W1/W3 and rows of W2 (NULL when Is = 0).
 *   Other arguments as moe_forward; topk_idx_out / topk_w_out / counts_out
 *   report the full routing.
 * Errors: MOE_ERR_INVALID_ARG for ep_size < 1 or ep_rank outside
 * [0, ep_size); MOE_ERR_UNSUPPORTED unless E and Is divide by ep_size and
 * Is/ep_size is a multiple of 128.  ep_size = 1 is moe_forward. */
moe_status moe_forward_ep(const moe_shape* shape, int ep_rank, int ep_size, const void* x, const void* Wg,
                          const float* bias, const void* W1, const void* W3, const void* W2, const float* s1,
                          const float* s3, const float* s2, const void* W1s, const void* W3s, const void* W2s, void* y,
                          int32_t* topk_idx_out, float* topk_w_out, int32_t* counts_out, void* ws, size_t ws_bytes,
                          void* stream);

/* Number of kernel launches moe_forward (and moe_forward_ep, moe_forward_profiled)
 * issues for this shape on the current device; -1 for an invalid shape.
 * Profiling aid; the pages have no counterpart. */
int moe_forward_launches(const moe_shape* shape);

/* moe_forward plus per-stage timing: records the caller's CUDA events
 * (cudaEvent_t handles, created with timing enabled) on `stream` at the stage
 * boundaries, without synchronising:
 *   [0] start  [1] after the router  [2] after dispatch (permutation, x rows
 *   copied into permuted order, tile list)  [3] after the grouped SwiGLU
 *   up-projection
 *   [4] after the grouped down-projection  [5] after the combine.
 * Same results and launches as moe_forward.  Profiling aid; the pages have no
 * counterpart. */
#define MOE_NUM_STAGE_EVENTS 6
moe_status moe_forward_profiled(const moe_shape* shape, const void* x, const void* Wg, const float* bias,
                                const void* W1, const void* W3, const void* W2, const float* s1, const float* s3,
                                const float* s2, const void* W1s, const void* W3s, const void* W2s, void* y,
                                int32_t* topk_idx_out, float* topk_w_out, int32_t* counts_out, void* ws,
                                size_t ws_bytes, void* stream, void* const* stage_events);

/* Synchronises `stream`, reads the status word of `ws` written by the last
 * call that used this workspace and returns MOE_OK, MOE_ERR_DEVICE_TIMEOUT or
 * MOE_ERR_DEVICE_BOUNDS (timeout wins when both are set); `raw` (optional)
 * receives the raw bits.  Returns MOE_ERR_CUDA when the stream itself reports
 * an error. */
moe_status moe_check_device_status(const void* ws, void* stream, uint32_t* raw);

/* Static description of a status code. */
const char* moe_status_string(moe_status status);

/* Library version string. */
const char* moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
