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
