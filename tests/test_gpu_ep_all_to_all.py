"""The all-to-all flavour of expert parallelism against the fp64 oracle.

Every rank holds its own tokens and E/world experts; rows travel to the rank
of their expert and back.  On one GPU the ranks run in lock step in one
process (simulate_all_to_all: the same per-rank steps, the exchanges done by
slicing); each rank's output must be the whole layer applied to its own
tokens.  The chunked driver with real collectives runs here on a one-rank
NCCL group (exchanges with itself); its multi-GPU run is not covered by these
tests (every call on this hardware has one GPU)."""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_ffn_17_b200 import binding as B
from mixture_experts_ffn_17_b200 import build as libbuild
from mixture_experts_ffn_17_b200 import expert_parallel as ep
from mixture_experts_ffn_17_b200 import workloads

from gpu_util import oracle_full, route_with_exemptions, run_forward, to_device
from parity import TOL_BF16, TOL_FP8, dec, max_rel_err, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    libbuild.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _rank_tokens(base, r):
    """Rank r's own batch: the base workload's weights, tokens from another seed."""
    w = workloads.make(base.cfg.replace(seed=base.cfg.seed + 101 * (r + 1)))
    return to_device(workloads.Workload(base.cfg, w.x, base.Wg, base.W1, base.W3, base.W2, base.W1s, base.W3s,
                                        base.W2s, bias=base.bias, s1=base.s1, s3=base.s3, s2=base.s2))


def _check(base, world, mutate=None, tol=TOL_BF16):
    cfg = base.cfg
    ranks = [_rank_tokens(base, r) for r in range(world)]
    wdev = to_device(base)
    if mutate:
        mutate(wdev, ranks)
    shape = B.shape_of(cfg)
    weights = [ep.shard_weights_a2a(wdev.W1, wdev.W3, wdev.W2, wdev.W1s, wdev.W3s, wdev.W2s, r, world,
                                    wdev.s1, wdev.s3, wdev.s2)
               for r in range(world)]
    ys = [torch.empty(cfg.T, cfg.d, dtype=torch.float32, device="cuda") for _ in range(world)]
    ep.simulate_all_to_all(shape, [w.x for w in ranks], wdev.Wg, wdev.bias, weights, ys)
    torch.cuda.synchronize()
    received = []
    for r, w in enumerate(ranks):
        y1, idx, _, counts, _ = run_forward(w)              # the whole layer on one GPU
        rms = float(y1.double().pow(2).mean().sqrt())
        assert float((ys[r] - y1).abs().max()) <= 1e-3 * rms, r
        y_o, _, _, lg = oracle_full(w)
        _, _, merged, report, n_near = route_with_exemptions(w, lg, to_np(idx))
        assert len(report) <= n_near
        if report:
            y_o, *_ = oracle_full(w, force_idx=merged)
        err = max_rel_err(to_np(ys[r]).astype(np.float64), y_o)
        assert err <= tol, (r, err)
        received.append(to_np(counts))
    return received


@pytest.mark.parametrize("world,E", [(2, 64), (4, 128)])
def test_all_to_all_ranks_match_the_layer(world, E):
    base = workloads.make_small("prefill", T=160, d=512, E=E, k=4, inter=256, shared_inter=256)
    _check(base, world)


def test_all_to_all_group_routing_with_bias():
    # sigmoid group-limited routing with the selection bias (8 groups of 16,
    # top-4 groups, x 2.5), bf16 experts, 2 ranks
    base = workloads.make_small("fp8", T=160, d=512, E=128, k=8, inter=256, shared_inter=256, fp8=False)
    _check(base, 2)


def test_all_to_all_fp8_experts_group_routing():
    # e4m3 routed experts with 128 x 128 block scales (each rank holds its
    # experts' codes and scales), bf16 shared expert, group routing, 2 ranks
    base = workloads.make_small("fp8", T=160, d=512, E=128, k=8, inter=256, shared_inter=256)
    assert base.cfg.fp8 and base.s1 is not None
    _check(base, 2, tol=TOL_FP8)


def test_all_to_all_fp8_small_batch():
    # 8 tokens per rank, top-4 of 64 experts over 2 ranks: each rank receives
    # at most 64 rows, so its local e4m3 GEMMs run the small-batch stage layout
    base = workloads.make_small("fp8", T=8, d=512, E=64, k=4, inter=256, shared_inter=256, n_group=8,
                                topk_group=2)
    _check(base, 2, tol=TOL_FP8)


def test_all_to_all_fp8_chunked_driver_on_a_one_rank_nccl_group():
    import torch.distributed as dist
    base = to_device(workloads.make_small("fp8", T=300, d=512, E=64, k=6, inter=256, shared_inter=256, n_group=8,
                                          topk_group=3))
    cfg = base.cfg
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        w = ep.shard_weights_a2a(base.W1, base.W3, base.W2, base.W1s, base.W3s, base.W2s, 0, 1,
                                 base.s1, base.s3, base.s2)
        y = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device="cuda")
        ep.forward_all_to_all(B.shape_of(cfg), 0, 1, base.x, base.Wg, base.bias, w, y, chunks=2)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    y1, *_ = run_forward(base)
    rms = float(y1.double().pow(2).mean().sqrt())
    assert float((y - y1).abs().max()) <= 1e-3 * rms


def test_all_to_all_rank_without_rows_and_no_shared_expert():
    # rank 1's experts (32..63) are never chosen: it receives no rows at all
    base = workloads.make_small("prefill", T=200, d=512, E=64, k=4, inter=256, shared_inter=0)

    def mutate(wdev, ranks):
        Wg = wdev.Wg.float()
        Wg[32:] = 0.0
        Wg[32:, 0] = -50.0
        wdev.Wg.copy_(Wg.to(torch.bfloat16))
        for w in ranks:
            x = w.x.float()
            x[:, 0] = 3.0
            w.x.copy_(x.to(torch.bfloat16))
            w.Wg = wdev.Wg

    counts = _check(base, 2, mutate)
    assert all(c[32:].sum() == 0 for c in counts)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_chunked_driver_on_a_one_rank_nccl_group():
    import torch.distributed as dist
    base = to_device(workloads.make_small("prefill", T=300, d=512, E=64, k=4, inter=256, shared_inter=256))
    cfg = base.cfg
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        w = ep.shard_weights_a2a(base.W1, base.W3, base.W2, base.W1s, base.W3s, base.W2s, 0, 1)
        y = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device="cuda")
        ep.forward_all_to_all(B.shape_of(cfg), 0, 1, base.x, base.Wg, None, w, y, chunks=3)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    y1, *_ = run_forward(base)
    rms = float(y1.double().pow(2).mean().sqrt())
    assert float((y - y1).abs().max()) <= 1e-3 * rms


def test_all_to_all_v3_decode_eight_ranks():
    # V3 shapes: 256 experts over 8 simulated ranks (32 each), each rank with
    # its own decode batch of 64 tokens; every rank's y against the whole layer
    # on one GPU, rank 0's against the fp64 oracle on all its tokens
    from gpu_util import oracle_sampled
    base_cfg = workloads.CONFIGS["decode"]
    world = 8
    base = workloads.make(base_cfg, device="cuda")
    ranks = []
    for r in range(world):
        g = torch.Generator(device="cuda").manual_seed(base_cfg.seed + 17 * (r + 1))
        z = torch.randn(base_cfg.T, base_cfg.d, generator=g, device="cuda")
        x = (z / z.pow(2).mean(dim=1, keepdim=True).sqrt()).to(torch.bfloat16)
        ranks.append(workloads.Workload(base_cfg, x, base.Wg, base.W1, base.W3, base.W2, base.W1s, base.W3s,
                                        base.W2s))
    shape = B.shape_of(base_cfg)
    weights = [ep.shard_weights_a2a(base.W1, base.W3, base.W2, base.W1s, base.W3s, base.W2s, r, world)
               for r in range(world)]
    ys = [torch.empty(base_cfg.T, base_cfg.d, dtype=torch.float32, device="cuda") for _ in range(world)]
    ep.simulate_all_to_all(shape, [w.x for w in ranks], base.Wg, None, weights, ys)
    torch.cuda.synchronize()
    for r, w in enumerate(ranks):
        y1, idx, _, _, _ = run_forward(w)
        rms = float(y1.double().pow(2).mean().sqrt())
        assert float((ys[r] - y1).abs().max()) <= 1e-3 * rms, r
    w = ranks[0]
    lg = oracle.logits(dec(w.x), dec(w.Wg))
    _, idx, _, _, _ = run_forward(w)
    _, _, merged, report, n_near = route_with_exemptions(w, lg, to_np(idx))
    assert len(report) <= n_near
    y_o = oracle_sampled(w, lg, merged, np.arange(base_cfg.T))
    err = max_rel_err(to_np(ys[0]).astype(np.float64), y_o)
    print(f"all-to-all, 8 ranks, V3 decode shapes: rank 0 max|err|/rms = {err:.2e}")
    assert err <= TOL_BF16, err
