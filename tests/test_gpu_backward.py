"""Backward-pass kernels (moe_combine_backward, moe_router_backward) against
the fp64 gradient oracle (oracle/backward.py): per kernel on the device's own
inputs with tight tolerances, and chained after the forward stages of the tiny
workload against the oracle's gradient of the whole layer."""
import numpy as np
import pytest
import torch

from oracle import backward as obw
from mixture_experts_ffn_17_b200 import binding as B
from mixture_experts_ffn_17_b200 import build as libbuild
from mixture_experts_ffn_17_b200 import workloads

from gpu_util import to_device
from parity import TOL_BF16, dec, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    libbuild.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _route_and_permute(w):
    cfg = w.cfg
    shape = B.shape_of(cfg)
    ws = B.alloc_workspace(shape)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device="cuda")
    tw = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device="cuda")
    lg = torch.empty(cfg.T, cfg.E, dtype=torch.float32, device="cuda")
    B.router_topk(shape, w.x, w.Wg, w.bias, idx, tw, lg, ws)
    counts = torch.empty(cfg.E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(cfg.E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(cfg.T * cfg.k, dtype=torch.int32, device="cuda")
    row_of = torch.empty(cfg.T * cfg.k, dtype=torch.int32, device="cuda")
    x_perm = torch.empty(cfg.T * cfg.k, cfg.d, dtype=torch.bfloat16, device="cuda")
    B.permute(shape, idx, counts, offsets, perm, row_of, w.x, x_perm, ws)
    return shape, ws, idx, tw, lg, offsets, row_of, x_perm


CASES = {
    "topk_softmax": ("prefill", dict(T=700, d=1024, E=64, k=6, inter=256, shared_inter=0)),
    "sigmoid_group": ("fp8", dict(T=600, d=1024, E=64, k=8, inter=256, shared_inter=0, fp8=False)),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_combine_and_router_backward_match_oracle(case):
    name, kw = CASES[case]
    w = to_device(workloads.make_small(name, **kw))
    cfg = w.cfg
    shape, ws, idx, tw, lg, offsets, row_of, _ = _route_and_permute(w)
    g = torch.Generator(device="cuda").manual_seed(1234)
    Tk = cfg.T * cfg.k
    Y_perm = (torch.randn(Tk, cfg.d, generator=g, device="cuda") * 0.05).to(torch.bfloat16)
    dy = torch.randn(cfg.T, cfg.d, generator=g, device="cuda")
    dO = torch.zeros(Tk, cfg.d, dtype=torch.bfloat16, device="cuda")
    dw = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device="cuda")
    dl = torch.full((cfg.T, cfg.E), float("nan"), dtype=torch.float32, device="cuda")
    B.combine_backward(shape, dy, Y_perm, row_of, tw, dO, dw)
    B.router_backward(shape, lg, idx, tw, dw, dl)
    torch.cuda.synchronize()

    # combine backward on the same stored inputs
    dO_o, dw_o = obw.combine_backward(to_np(dy).astype(np.float64), dec(Y_perm), to_np(row_of),
                                      to_np(tw).astype(np.float64))
    dO_d = dec(dO)
    # bf16(fp32(w * dy)): within one bf16 unit in the last place of the exact product
    assert np.all(np.abs(dO_d - dO_o) <= 2.0 ** -7 * np.abs(dO_o) + 1e-30)
    scale = np.abs(to_np(dy)).astype(np.float64) @ np.ones(cfg.d) * np.abs(dec(Y_perm)).max()
    err = np.abs(to_np(dw).astype(np.float64) - dw_o)
    assert np.all(err <= 1e-5 * scale[:, None]), err.max()

    # router backward on the device's logits, weights and dw
    lg_d = to_np(lg).astype(np.float64)
    idx_d = to_np(idx)
    w_d = to_np(tw).astype(np.float64)
    dw_d = to_np(dw).astype(np.float64)
    dl_o = np.zeros((cfg.T, cfg.E))
    for t in range(cfg.T):
        dl_o[t, idx_d[t]] = obw.routing_backward(lg_d[t, idx_d[t]], w_d[t], dw_d[t], cfg.route, cfg.route_scale)
    dl_d = to_np(dl).astype(np.float64)
    assert np.isfinite(dl_d).all()
    mask = np.zeros((cfg.T, cfg.E), dtype=bool)
    np.put_along_axis(mask, idx_d.astype(np.int64), True, axis=1)
    assert not dl_d[~mask].any()  # zero outside the selection, every entry written
    tol = 1e-5 * (np.abs(w_d * dw_d).sum(axis=1, keepdims=True) * max(1.0, cfg.route_scale) + 1e-12)
    assert np.all(np.abs(dl_d - dl_o) <= tol), np.abs(dl_d - dl_o).max()


def test_backward_steps_after_the_forward_match_the_layer_gradient():
    # tiny workload: forward stages on the GPU (router, dispatch, grouped SwiGLU),
    # then the two backward steps; against the oracle's gradient of the layer
    w = to_device(workloads.make("tiny"))
    cfg = w.cfg
    shape, ws, idx, tw, lg, offsets, row_of, x_perm = _route_and_permute(w)
    Y_perm = torch.empty(cfg.T * cfg.k, cfg.d, dtype=torch.bfloat16, device="cuda")
    Y_shared = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device="cuda")
    B.grouped_swiglu(shape, w.x, x_perm, offsets, w.W1, w.W3, w.W2, None, None, None, w.W1s, w.W3s, w.W2s, Y_perm,
                     Y_shared, ws)
    dy = torch.randn(cfg.T, cfg.d, generator=torch.Generator(device="cuda").manual_seed(99), device="cuda")
    dO = torch.zeros_like(Y_perm)
    dw = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device="cuda")
    dl = torch.empty(cfg.T, cfg.E, dtype=torch.float32, device="cuda")
    B.combine_backward(shape, dy, Y_perm, row_of, tw, dO, dw)
    B.router_backward(shape, lg, idx, tw, dw, dl)
    rc, raw = B.check_device_status(ws)
    assert rc == B.MOE_OK, (rc, raw)

    g = obw.moe_backward(dec(w.x), dec(w.Wg), dec(w.W1), dec(w.W3), dec(w.W2), dec(w.W1s), dec(w.W3s), dec(w.W2s),
                         dy=to_np(dy).astype(np.float64), k=cfg.k)
    same = np.all(to_np(idx) == g["idx"], axis=1)
    assert same.mean() >= 0.99, "routing differs on more than near-tie tokens"
    dw_d = to_np(dw).astype(np.float64)[same]
    dw_o = g["dw"][same]
    assert np.max(np.abs(dw_d - dw_o)) <= TOL_BF16 * np.sqrt(np.mean(dw_o ** 2))
    # dl_j = w_j (dw_j - sum_i w_i dw_i), so an error of at most e in every dw
    # moves dl_j by at most 2 w_j e: allow what the dw check allows, carried
    # through the softmax Jacobian (dl is a difference of nearby numbers)
    e_dw = TOL_BF16 * np.sqrt(np.mean(dw_o ** 2))
    w_o = g["w"][same]
    dl_d = np.take_along_axis(to_np(dl).astype(np.float64)[same], g["idx"][same].astype(np.int64), axis=1)
    dl_o = np.take_along_axis(g["dl"][same], g["idx"][same].astype(np.int64), axis=1)
    assert np.all(np.abs(dl_d - dl_o) <= 2.0 * w_o * e_dw), np.max(np.abs(dl_d - dl_o) / (w_o * e_dw))
    # and nothing outside the selection
    dl_all = to_np(dl).astype(np.float64)
    mask = np.zeros_like(dl_all, dtype=bool)
    np.put_along_axis(mask, to_np(idx).astype(np.int64), True, axis=1)
    assert not dl_all[~mask].any()
    if same.all():
        # same selection everywhere: the permuted rows line up with the oracle's
        dO_d = dec(dO)
        assert np.max(np.abs(dO_d - g["dO_perm"])) <= 2.0 ** -8 * np.abs(g["dO_perm"]).max()
