"""Helpers shared by the GPU tests: move workloads to the device, run the
library through its C ABI, and run the oracle on the same stored values."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from mixture_experts_ffn_17_b200 import binding as B
from mixture_experts_ffn_17_b200 import workloads

from parity import dec, oracle_route


def to_device(w: workloads.Workload, device="cuda") -> workloads.Workload:
    mv = lambda t: None if t is None else t.to(device)
    return workloads.Workload(w.cfg, mv(w.x), mv(w.Wg), mv(w.W1), mv(w.W3), mv(w.W2), mv(w.W1s), mv(w.W3s),
                              mv(w.W2s), bias=mv(w.bias), s1=mv(w.s1), s3=mv(w.s3), s2=mv(w.s2))


def run_forward(w: workloads.Workload, y_dtype=B.MOE_F32, ws=None):
    cfg = w.cfg
    dev = w.x.device
    shape = B.shape_of(cfg, y_dtype)
    if ws is None:
        ws = B.alloc_workspace(shape, dev)
    y = torch.empty(cfg.T, cfg.d, dtype=torch.float32 if y_dtype == B.MOE_F32 else torch.bfloat16, device=dev)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=dev)
    tw = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=dev)
    counts = torch.empty(cfg.E, dtype=torch.int32, device=dev)
    B.forward(shape, w.x, w.Wg, w.bias, w.W1, w.W3, w.W2, w.s1, w.s3, w.s2, w.W1s, w.W3s, w.W2s, y, ws, idx, tw,
              counts)
    rc, raw = B.check_device_status(ws)
    assert rc == B.MOE_OK, (rc, raw)
    return y, idx, tw, counts, ws


def expert_weights_f64(w: workloads.Workload, e: int):
    """(W1[e], W3[e], W2[e]) of the stored weights, decoded to fp64 on the host."""
    if w.cfg.fp8:
        return (oracle.decode_e4m3_blocks(w.W1[e].cpu().numpy(), w.s1[e].cpu().numpy()),
                oracle.decode_e4m3_blocks(w.W3[e].cpu().numpy(), w.s3[e].cpu().numpy()),
                oracle.decode_e4m3_blocks(w.W2[e].cpu().numpy(), w.s2[e].cpu().numpy()))
    return dec(w.W1[e]), dec(w.W3[e]), dec(w.W2[e])


def oracle_full(w: workloads.Workload, force_idx=None):
    """Whole-layer oracle for workloads that fit in host memory (all experts)."""
    cfg = w.cfg
    if cfg.fp8:
        W = [expert_weights_f64(w, e) for e in range(cfg.E)]
        W1 = np.stack([a for a, _, _ in W]); W3 = np.stack([b for _, b, _ in W]); W2 = np.stack([c for _, _, c in W])
    else:
        W1, W3, W2 = dec(w.W1), dec(w.W3), dec(w.W2)
    bias = None if w.bias is None else dec(w.bias)
    shared = {} if cfg.shared_inter == 0 else dict(W1s=dec(w.W1s), W3s=dec(w.W3s), W2s=dec(w.W2s))
    return oracle.moe_forward(dec(w.x), dec(w.Wg), W1, W3, W2, k=cfg.k, route=cfg.route, bias=bias,
                              n_group=cfg.n_group, topk_group=cfg.topk_group, group_topn=cfg.group_topn,
                              route_scale=cfg.route_scale, force_idx=force_idx, **shared)


def oracle_sampled(w: workloads.Workload, lg: np.ndarray, idx: np.ndarray, tokens: np.ndarray, threads=None):
    """Oracle outputs for a sample of tokens, fetching one expert at a time.

    lg: fp64 logits [T, E]; idx: the routing to use [T, k] (the oracle's, with
    near-tie tokens replaced by the device's choice).  Experts run in a few
    host threads (each oracle call is independent)."""
    import concurrent.futures
    import os
    cfg = w.cfg
    x = dec(w.x[torch.as_tensor(tokens, device=w.x.device)])
    wts = oracle.weights_for(lg[tokens], idx[tokens], cfg.route, cfg.route_scale)
    sel = idx[tokens]

    def one(e):
        rows, slots = np.nonzero(sel == e)
        W1, W3, W2 = expert_weights_f64(w, int(e))
        return rows, wts[rows, slots][:, None] * oracle.swiglu_rows(x[rows], W1, W3, W2)

    y = np.zeros((len(tokens), cfg.d))
    n = threads or max(1, min(8, (os.cpu_count() or 2) // 2))
    with concurrent.futures.ThreadPoolExecutor(n) as ex:
        for rows, contrib in ex.map(one, [int(e) for e in np.unique(sel)]):
            np.add.at(y, rows, contrib)
    if cfg.shared_inter > 0:
        y += oracle.swiglu_rows(x, dec(w.W1s), dec(w.W3s), dec(w.W2s))
    return y


def choose_sample(idx: np.ndarray, counts: np.ndarray, near_tie_tokens, size: int, seed: int,
                  per_expert: int = 4) -> np.ndarray:
    """Sample of tokens for output checks at full size: every near-tie token,
    tokens on the 3 most- and 3 least-loaded non-empty experts (up to
    `per_expert` each), the first and last token, the rest seeded random, up
    to `size` tokens in all."""
    T = idx.shape[0]
    pick = set(int(t) for t in near_tie_tokens)
    pick.update((0, T - 1))
    nz = np.nonzero(counts > 0)[0]
    order = nz[np.argsort(counts[nz], kind="stable")]
    for e in list(order[:3]) + list(order[-3:]):
        toks = np.nonzero((idx == e).any(axis=1))[0]
        pick.update(int(t) for t in toks[:per_expert])
    rng = np.random.default_rng(seed)
    rest = [t for t in rng.permutation(T) if t not in pick]
    pick.update(int(t) for t in rest[:max(0, size - len(pick))])
    return np.array(sorted(pick), dtype=np.int64)


def oracle_logits(w: workloads.Workload) -> np.ndarray:
    return oracle.logits(dec(w.x), dec(w.Wg))


def route_with_exemptions(w, lg, idx_dev):
    """Oracle routing, the per-slot exemption check, and the merged index set
    (the oracle's, with exempted tokens replaced by the device's choice).

    Returns (idx_o, w_o, merged, report, n_near) where n_near counts the tokens
    whose oracle routing has a near-tie at all."""
    from parity import compare_indices, near_tie_tokens
    cfg = w.cfg
    bias = None if w.bias is None else dec(w.bias)
    idx_o, w_o, scores, gaps, ggap = oracle_route(cfg, lg, bias)
    group = (cfg.n_group, cfg.topk_group, cfg.group_topn) if cfg.route == 1 else None
    n_ex, report = compare_indices(idx_dev, idx_o, scores, gaps, ggap, cfg.E, group=group)
    merged = idx_o.copy()
    for t, _, _ in report:
        merged[t] = idx_dev[t]
    return idx_o, w_o, merged, report, len(near_tie_tokens(gaps, ggap))
