"""Expert-parallel plumbing around ``moe_forward_ep``: which experts and which
slice of the shared expert a rank holds, the rank's weight slices, and the
all-reduce that completes the layer.

Layout of the split (atlas page "DeepSeek-V3.2-Exp / Mixture of experts /
Shared expert", "Code" section): the MoE constructor block gives rank r of
``world`` ranks the routed experts ``[r*E/world, (r+1)*E/world)``, and its
shared-expert MLP has column-parallel W1/W3 and a row-parallel W2 whose output
is not reduced, i.e. rank r holds hidden features ``[r*Is/world,
(r+1)*Is/world)`` of it.  The MoE forward block adds the local experts'
weighted outputs and the shared MLP's partial output into ``y`` and then runs
one ``all_reduce`` of ``y`` over the ranks.  ``moe_forward_ep`` computes that
partial ``y`` on the GPU; the all-reduce is a plain ``torch.distributed``
collective (NCCL on GPUs).

The partition is computed here only to slice the weights a rank is given; the
library derives the same ranges from ``(ep_rank, ep_size)`` itself.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

from . import binding as B


@dataclasses.dataclass(frozen=True)
class EpSlice:
    e_lo: int  # first routed expert held
    e_hi: int  # one past the last
    i_lo: int  # first hidden feature of the shared expert held
    i_hi: int


def ep_slice(E: int, shared_inter: int, rank: int, world: int) -> EpSlice:
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of {world}")
    if E % world or shared_inter % world:
        raise ValueError(f"E={E} and shared_inter={shared_inter} must divide by the {world} ranks")
    el, il = E // world, shared_inter // world
    return EpSlice(rank * el, (rank + 1) * el, rank * il, (rank + 1) * il)


@dataclasses.dataclass
class EpWeights:
    """One rank's weights: routed experts [e_lo, e_hi) (and their FP8 scales)
    and its hidden-feature slice of the shared expert, each contiguous."""
    W1: torch.Tensor
    W3: torch.Tensor
    W2: torch.Tensor
    s1: Optional[torch.Tensor]
    s3: Optional[torch.Tensor]
    s2: Optional[torch.Tensor]
    W1s: Optional[torch.Tensor]
    W3s: Optional[torch.Tensor]
    W2s: Optional[torch.Tensor]


def shard_weights(W1, W3, W2, s1, s3, s2, W1s, W3s, W2s, rank: int, world: int) -> EpWeights:
    """Slice full-layer weights (W1, W3 [E, d, I], W2 [E, I, d], scales
    [E, ., .], shared W1s, W3s [d, Is], W2s [Is, d]) down to rank `rank`'s."""
    E = W1.shape[0]
    Is = 0 if W1s is None else W1s.shape[1]
    sl = ep_slice(E, Is, rank, world)
    ex = lambda t: None if t is None else t[sl.e_lo:sl.e_hi].contiguous()
    return EpWeights(ex(W1), ex(W3), ex(W2), ex(s1), ex(s3), ex(s2),
                     None if W1s is None else W1s[:, sl.i_lo:sl.i_hi].contiguous(),
                     None if W3s is None else W3s[:, sl.i_lo:sl.i_hi].contiguous(),
                     None if W2s is None else W2s[sl.i_lo:sl.i_hi].contiguous())


def all_reduce_partial(y: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the ranks' partial outputs in place (the MoE forward block's
    all-reduce); a no-op without an initialised process group of size > 1."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(y, op=dist.ReduceOp.SUM, group=group)
    return y


def forward(shape, rank: int, world: int, x, Wg, bias, w: EpWeights, y, ws, group=None, stream=None,
            topk_idx=None, topk_w=None, counts=None) -> torch.Tensor:
    """This rank's partial layer on its GPU, then the all-reduce over `group`
    (the layer's output, identical on every rank)."""
    B.forward_ep(shape, rank, world, x, Wg, bias, w.W1, w.W3, w.W2, w.s1, w.s3, w.s2, w.W1s, w.W3s, w.W2s, y, ws,
                 topk_idx=topk_idx, topk_w=topk_w, counts=counts, stream=stream)
    return all_reduce_partial(y, group)


# --------------------------------------------------------------------------
# All-to-all flavour.
#
# Here every rank holds its own batch of tokens and E/world routed experts;
# the shared expert is replicated and runs on each rank's own tokens.  A
# token's hidden state travels to the ranks that hold its selected experts
# and the expert outputs travel back (n4n.ai page, "Why 256 experts with top-8
# routing?", device-limited routing and the all-to-all it bounds; "Training
# infrastructure that made this possible": that all-to-all overlapped with
# computation).  Per rank:
#   1. route its tokens over all E experts and permute them (moe_router_topk,
#      moe_permute): the rows for rank q's experts form one contiguous block of
#      the expert-major x_perm;
#   2. exchange the per-expert row counts, then the rows (all-to-all);
#   3. regroup the received rows expert-major (moe_ep_regroup_layout,
#      moe_gather_rows), run the local experts (moe_grouped_swiglu), and put
#      the outputs back in the received order;
#   4. send them back (all-to-all); they arrive in the rank's own x_perm order,
#      i.e. as its Y_perm;
#   5. the shared expert on its own tokens (moe_shared_expert) and the combine
#      (moe_combine) give the rank's y.
# With several token chunks, chunk c+1's rows travel while chunk c's experts
# compute, and chunk c's outputs travel back while chunk c+1's compute.
# Every arithmetic step runs in the library's kernels; this module moves
# tensors between ranks.
# --------------------------------------------------------------------------

@dataclasses.dataclass
class A2AWeights:
    """One rank's weights in the all-to-all flavour: routed experts
    [e_lo, e_hi) (e4m3 codes with their 128 x 128 block scales s1, s3, s2, or
    bf16 with no scales) and the whole shared expert (replicated, bf16)."""
    W1: torch.Tensor
    W3: torch.Tensor
    W2: torch.Tensor
    W1s: Optional[torch.Tensor]
    W3s: Optional[torch.Tensor]
    W2s: Optional[torch.Tensor]
    s1: Optional[torch.Tensor] = None
    s3: Optional[torch.Tensor] = None
    s2: Optional[torch.Tensor] = None


def shard_weights_a2a(W1, W3, W2, W1s, W3s, W2s, rank: int, world: int, s1=None, s3=None, s2=None) -> A2AWeights:
    """Rank `rank`'s routed experts (and, for e4m3 experts, their block scales
    [E, ., .]) of the full layer's weights; the shared expert is kept whole."""
    E = W1.shape[0]
    if E % world or (E // world) % 32:
        raise ValueError(f"E={E} over {world} ranks: each rank's expert count must be a multiple of 32")
    if (s1 is None) != (s3 is None) or (s1 is None) != (s2 is None):
        raise ValueError("e4m3 experts need all three block-scale tensors")
    lo, hi = rank * (E // world), (rank + 1) * (E // world)
    ex = lambda t: None if t is None else t[lo:hi].contiguous()
    return A2AWeights(ex(W1), ex(W3), ex(W2), W1s, W3s, W2s, ex(s1), ex(s3), ex(s2))


class A2ARank:
    """One rank's steps of the all-to-all layer for one batch of its tokens.
    `shape` is the whole layer's shape for this batch (T = the rank's tokens,
    E = all experts)."""

    def __init__(self, shape, rank: int, world: int, w: A2AWeights, device, stream=None):
        self.shape, self.rank, self.world, self.w = shape, rank, world, w
        self.stream = stream
        T, d, E, k = shape.T, shape.d, shape.E, shape.k
        self.El = E // world
        dev = device
        self.ws = B.alloc_workspace(shape, dev)
        self.idx = torch.empty(T, k, dtype=torch.int32, device=dev)
        self.tw = torch.empty(T, k, dtype=torch.float32, device=dev)
        self.counts = torch.empty(E, dtype=torch.int32, device=dev)
        self.offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        self.perm = torch.empty(T * k, dtype=torch.int32, device=dev)
        self.row_of = torch.empty(T * k, dtype=torch.int32, device=dev)
        self.x_perm = torch.empty(T * k, d, dtype=torch.bfloat16, device=dev)
        self.Y_shared = (torch.empty(T, d, dtype=torch.float32, device=dev) if shape.shared_inter > 0 else None)

    # step 1
    def dispatch(self, x, Wg, bias) -> torch.Tensor:
        """Route and permute; returns the send counts [world, E_local] (device)."""
        s = self.shape
        B.router_topk(s, x, Wg, bias, self.idx, self.tw, None, self.ws, stream=self.stream)
        B.permute(s, self.idx, self.counts, self.offsets, self.perm, self.row_of, x, self.x_perm, self.ws,
                  stream=self.stream)
        return self.counts.view(self.world, self.El)

    # step 3
    def compute(self, x_recv: torch.Tensor, recv_counts: torch.Tensor) -> torch.Tensor:
        """Rows received from every rank (source-major) and their counts
        [world, E_local] -> this rank's expert outputs in the same order."""
        s = self.shape
        R = int(x_recv.shape[0])
        dev = x_recv.device
        y_send = torch.empty(R, s.d, dtype=torch.bfloat16, device=dev)
        if R == 0:
            return y_send
        offs = torch.empty(self.El + 1, dtype=torch.int32, device=dev)
        to_em = torch.empty(R, dtype=torch.int32, device=dev)
        to_sm = torch.empty(R, dtype=torch.int32, device=dev)
        B.ep_regroup_layout(self.world, self.El, recv_counts.contiguous(), offs, to_em, to_sm, stream=self.stream)
        x_loc = torch.empty(R, s.d, dtype=torch.bfloat16, device=dev)
        B.gather_rows(x_recv, to_em, x_loc, stream=self.stream)
        shape_loc = B.make_shape(T=R, d=s.d, E=self.El, k=1, inter=s.inter, shared_inter=0, w_dtype=s.w_dtype)
        ws_loc = B.alloc_workspace(shape_loc, dev)
        Y_loc = torch.empty(R, s.d, dtype=torch.bfloat16, device=dev)
        B.grouped_swiglu(shape_loc, x_loc, x_loc, offs, self.w.W1, self.w.W3, self.w.W2, self.w.s1, self.w.s3,
                         self.w.s2, None, None, None, Y_loc, None, ws_loc, stream=self.stream)
        B.gather_rows(Y_loc, to_sm, y_send, stream=self.stream)
        return y_send

    # step 5
    def combine(self, x, Y_perm: torch.Tensor, y: torch.Tensor):
        s = self.shape
        if self.Y_shared is not None:
            B.shared_expert(s, x, self.w.W1s, self.w.W3s, self.w.W2s, self.Y_shared, self.ws, stream=self.stream)
        B.combine(s, Y_perm, self.Y_shared, self.row_of, self.tw, y, stream=self.stream)
        return y


def _splits(counts_2d: torch.Tensor):
    return [int(v) for v in counts_2d.sum(dim=1).tolist()]


class ProcessGroupTransport:
    """all_to_all_single over a torch.distributed group (NCCL on GPUs, gloo on
    CPU).  Rows are dim 0; split sizes are host lists."""

    def __init__(self, group=None):
        self.group = group

    def all_to_all(self, send: torch.Tensor, send_splits, recv_splits, async_op: bool = False):
        import torch.distributed as dist
        out = send.new_empty((sum(recv_splits),) + tuple(send.shape[1:]))
        work = dist.all_to_all_single(out, send.contiguous(), list(recv_splits), list(send_splits), group=self.group,
                                      async_op=async_op)
        return out, work

    def exchange_counts(self, send_counts: torch.Tensor) -> torch.Tensor:
        """send_counts [world, E_local]: row q is what this rank sends to rank
        q; returns [world, E_local], row s is what rank s sends here."""
        n = send_counts.shape[0]
        out, _ = self.all_to_all(send_counts.contiguous(), [1] * n, [1] * n)
        return out


def forward_all_to_all(shape, rank: int, world: int, x, Wg, bias, w: A2AWeights, y, transport=None, chunks: int = 2,
                       stream=None) -> torch.Tensor:
    """This rank's y (its own tokens) through the all-to-all layer, with the
    tokens split into `chunks` batches whose exchanges overlap the other
    batches' expert GEMMs.  Every rank of the group calls it with the same
    `chunks` (the collectives run in the same order everywhere).  `stream`
    (default: the current one) orders the kernels and the collectives alike:
    torch.distributed enqueues its work after the current stream's."""
    if stream is not None:
        with torch.cuda.stream(stream):
            return forward_all_to_all(shape, rank, world, x, Wg, bias, w, y, transport, chunks, None)
    transport = transport or ProcessGroupTransport()
    T = shape.T
    bounds = [T * c // chunks for c in range(chunks + 1)]
    parts = []
    for c in range(chunks):
        sl = slice(bounds[c], bounds[c + 1])
        sh = B.make_shape(T=bounds[c + 1] - bounds[c], d=shape.d, E=shape.E, k=shape.k, inter=shape.inter,
                          shared_inter=shape.shared_inter, route=shape.route, n_group=shape.n_group,
                          topk_group=shape.topk_group, group_topn=shape.group_topn, route_scale=shape.route_scale,
                          w_dtype=shape.w_dtype, y_dtype=shape.y_dtype)
        parts.append((sl, A2ARank(sh, rank, world, w, x.device, stream)))
    sends, recvs, xs = [], [], []
    for sl, st in parts:
        sends.append(st.dispatch(x[sl], Wg, bias))
    for c, (sl, st) in enumerate(parts):
        recvs.append(transport.exchange_counts(sends[c]))
    for c, (sl, st) in enumerate(parts):
        xs.append(transport.all_to_all(st.x_perm, _splits(sends[c]), _splits(recvs[c]), async_op=True))
    rets = []
    for c, (sl, st) in enumerate(parts):
        x_recv, work = xs[c]
        if work is not None:
            work.wait()
        y_send = st.compute(x_recv, recvs[c])
        rets.append(transport.all_to_all(y_send, _splits(recvs[c]), _splits(sends[c]), async_op=True))
    for c, (sl, st) in enumerate(parts):
        Y_perm, work = rets[c]
        if work is not None:
            work.wait()
        st.combine(x[sl], Y_perm, y[sl])
    return y


def simulate_all_to_all(shape, xs, Wg, bias, weights, ys, stream=None):
    """All ranks of the all-to-all layer in one process (one GPU), the
    exchanges done by slicing: rank r's tokens xs[r] and weights weights[r]
    -> ys[r].  The same per-rank steps as forward_all_to_all, in lock step."""
    world = len(xs)
    states = [A2ARank(shape, r, world, weights[r], xs[r].device, stream) for r in range(world)]
    send = [st.dispatch(xs[r], Wg, bias) for r, st in enumerate(states)]
    recv = [torch.stack([send[s][r] for s in range(world)]) for r in range(world)]
    blocks = [list(torch.split(states[s].x_perm, _splits(send[s]))) for s in range(world)]
    x_recv = [torch.cat([blocks[s][r] for s in range(world)]) for r in range(world)]
    y_send = [st.compute(x_recv[r], recv[r]) for r, st in enumerate(states)]
    back = [list(torch.split(y_send[r], _splits(recv[r]))) for r in range(world)]
    for r, st in enumerate(states):
        st.combine(xs[r], torch.cat([back[q][r] for q in range(world)]), ys[r])
    return ys
