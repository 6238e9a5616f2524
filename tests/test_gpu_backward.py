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

from gpu_util import run_forward, to_device
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


# ------------------------------------------------------ the whole backward pass
def _backward(w, dy, grad_bf16=False):
    """moe_backward on the device -> dict of gradients (torch tensors)."""
    cfg = w.cfg
    shape = B.shape_of(cfg, B.MOE_BF16 if grad_bf16 else B.MOE_F32)
    ws = B.alloc_backward_workspace(shape)
    dt = torch.bfloat16 if grad_bf16 else torch.float32
    z = lambda *s: torch.full(s, float("nan"), dtype=dt, device="cuda")   # every element must be written
    g = dict(dx=z(cfg.T, cfg.d), dWg=z(cfg.E, cfg.d), dW1=z(cfg.E, cfg.d, cfg.inter), dW3=z(cfg.E, cfg.d, cfg.inter),
             dW2=z(cfg.E, cfg.inter, cfg.d))
    sh = cfg.shared_inter > 0
    if sh:
        g.update(dW1s=z(cfg.d, cfg.shared_inter), dW3s=z(cfg.d, cfg.shared_inter), dW2s=z(cfg.shared_inter, cfg.d))
    B.backward(shape, w.x, w.Wg, w.bias, w.W1, w.W3, w.W2, w.W1s, w.W3s, w.W2s, dy, g["dx"], g["dWg"], g["dW1"],
               g["dW3"], g["dW2"], g.get("dW1s"), g.get("dW3s"), g.get("dW2s"), ws)
    rc, raw = B.check_device_status(ws)
    assert rc == B.MOE_OK, (rc, raw)
    return g, ws


def _oracle_backward(w, dy, force_idx=None):
    cfg = w.cfg
    sh = {} if cfg.shared_inter == 0 else dict(W1s=dec(w.W1s), W3s=dec(w.W3s), W2s=dec(w.W2s))
    return obw.moe_backward(dec(w.x), dec(w.Wg), dec(w.W1), dec(w.W3), dec(w.W2), dy=to_np(dy).astype(np.float64),
                            k=cfg.k, route=cfg.route, bias=None if w.bias is None else dec(w.bias),
                            n_group=cfg.n_group, topk_group=cfg.topk_group, group_topn=cfg.group_topn,
                            route_scale=cfg.route_scale, force_idx=force_idx, **sh)


GRADS = ("dx", "dWg", "dW1", "dW3", "dW2", "dW1s", "dW3s", "dW2s")
PER_EXPERT = ("dW1", "dW3", "dW2")
TOL_FRO = 1e-2   # relative Frobenius error of each gradient tensor
TOL_MAX = 2e-2   # max error over each tensor (each expert's block) / its largest entry


def _check_backward(w, seed=7, grad_bf16=False):
    """Every gradient against the fp64 oracle, element by element.

    The device keeps the forward's g and u, the output gradient w dy, dG and
    dU, and H in bf16 (each a rounding of at most 2^-9 relative), and sums in
    fp32: every gradient is then a sum of products carrying a relative error of
    a few 2^-9, about 0.3% in norm.  The bound is norm-wise, not the forward
    output's max-over-rms rule: an expert's weight gradient is a sum of outer
    products over its few rows, whose largest entries are 15-20x its rms, so
    a max-over-rms measure scales with that spread rather than with the
    arithmetic.  Per tensor: ||err||_F <= 1e-2 ||ref||_F; per tensor (per
    expert for the routed weight gradients): max|err| <= 2e-2 max|ref|; an
    expert no token chose has an exactly zero gradient."""
    from gpu_util import route_with_exemptions
    cfg = w.cfg
    dy = torch.randn(cfg.T, cfg.d, generator=torch.Generator(device="cuda").manual_seed(seed), device="cuda")
    g, ws = _backward(w, dy, grad_bf16)
    # the device's routing (for near-tie tokens the oracle follows it)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device="cuda")
    y = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device="cuda")
    fws = B.alloc_workspace(B.shape_of(cfg))
    B.forward(B.shape_of(cfg), w.x, w.Wg, w.bias, w.W1, w.W3, w.W2, None, None, None, w.W1s, w.W3s, w.W2s, y, fws,
              topk_idx=idx)
    lg = obw._logits(dec(w.x), dec(w.Wg))
    _, _, merged, report, n_near = route_with_exemptions(w, lg, to_np(idx))
    assert len(report) <= n_near, report
    ref = _oracle_backward(w, dy, force_idx=merged if report else None)
    stats = {}
    for name in GRADS:
        if name not in g:
            continue
        d = to_np(g[name].float()).astype(np.float64)
        o = ref[name]
        assert np.isfinite(d).all(), f"{name}: not every element written"
        fro = float(np.linalg.norm(d - o) / np.linalg.norm(o))
        blocks = [(d[e], o[e]) for e in range(d.shape[0])] if name in PER_EXPERT else [(d, o)]
        worst = 0.0
        for db, ob in blocks:
            m = float(np.abs(ob).max())
            if m == 0.0:
                assert not db.any(), f"{name}: an expert without rows has a nonzero gradient"
                continue
            worst = max(worst, float(np.abs(db - ob).max()) / m)
        stats[name] = (fro, worst)
    print({k: f"fro {a:.1e} max {b:.1e}" for k, (a, b) in stats.items()})
    for name, (fro, worst) in stats.items():
        assert fro <= TOL_FRO and worst <= TOL_MAX, (name, fro, worst)
    return g, ref


def _medium(**kw):
    shape = dict(T=1000, d=1024, E=64, k=6, inter=512, shared_inter=384)
    shape.update(kw)
    return to_device(workloads.make_small("prefill", **shape))


def test_backward_tiny():
    _check_backward(to_device(workloads.make("tiny")))


def test_backward_medium_ragged():
    # I != Is, a partial 256-column block of the shared expert, ragged segments
    _check_backward(_medium())


def test_backward_no_shared_expert():
    # the shared expert's tiles then carry only the router's dl Wg part of dx
    _check_backward(_medium(T=300, shared_inter=0))


def test_backward_group_routing():
    w = to_device(workloads.make_small("fp8", T=600, d=1024, E=64, k=8, inter=256, shared_inter=256, n_group=8,
                                       topk_group=4, fp8=False))
    _check_backward(w)


def test_backward_empty_and_oversize_segments():
    # a shared direction in x and gate rows aligned with it: expert 0 takes
    # nearly every token (a segment of several 256-row tiles), experts 1-3 most
    # second slots, and most other experts receive no row (zero weight gradient)
    w = workloads.make_small("prefill", T=700, d=512, E=64, k=2, inter=256, shared_inter=256)
    gen = torch.Generator().manual_seed(3)
    u = torch.randn(w.cfg.d, generator=gen)
    u = u / u.norm()
    x = w.x.float() + 3.0 * u
    x = x / x.pow(2).mean(dim=1, keepdim=True).sqrt()
    Wg = w.Wg.float()
    Wg[0] += 6.0 * u
    Wg[1:4] += 2.5 * u
    Wg[4:] -= 2.0 * u
    w.x, w.Wg = x.to(torch.bfloat16), Wg.to(torch.bfloat16)
    w = to_device(w)
    g, ref = _check_backward(w)
    c = np.bincount(ref["idx"].ravel(), minlength=w.cfg.E)
    assert c[0] > 512 and (c == 0).sum() >= 40, c      # several 256-row tiles; most experts empty
    empty = np.nonzero(c == 0)[0]
    assert not to_np(g["dW1"][torch.as_tensor(empty, device="cuda")]).any()
    assert not to_np(g["dW2"][torch.as_tensor(empty, device="cuda")]).any()


def test_backward_bf16_gradients_and_determinism():
    w = to_device(workloads.make("tiny"))
    g32, _ = _check_backward(w)
    dy = torch.randn(w.cfg.T, w.cfg.d, generator=torch.Generator(device="cuda").manual_seed(7), device="cuda")
    a, _ = _backward(w, dy)
    b, _ = _backward(w, dy)
    for name in a:
        assert torch.equal(a[name], b[name]), name        # bit-identical repeat
        assert torch.equal(a[name], g32[name]), name
    h, _ = _backward(w, dy, grad_bf16=True)
    for name in h:
        # the bf16 gradients are the fp32 ones rounded once
        assert torch.equal(h[name], g32[name].to(torch.bfloat16)), name


@pytest.mark.parametrize("shared", [384, 0])
def test_training_step_with_saved_state_matches_recomputing_calls(shared):
    # moe_forward_train + moe_backward_saved give moe_forward's y and
    # moe_backward's gradients, bit for bit (same kernels, same order)
    w = _medium(T=700, shared_inter=shared)
    cfg = w.cfg
    dy = torch.randn(cfg.T, cfg.d, generator=torch.Generator(device="cuda").manual_seed(11), device="cuda")
    ref, _ = _backward(w, dy)
    y_ref, *_ = run_forward(w)
    shape = B.shape_of(cfg, B.MOE_F32)
    ws = B.alloc_backward_workspace(shape)
    y = torch.empty_like(y_ref)
    B.forward_train(shape, w.x, w.Wg, w.bias, w.W1, w.W3, w.W2, w.W1s, w.W3s, w.W2s, y, ws)
    z = lambda *sz: torch.full(sz, float("nan"), dtype=torch.float32, device="cuda")
    g = {k: z(*v.shape) for k, v in ref.items()}
    B.backward_saved(shape, w.x, w.Wg, w.W1, w.W3, w.W2, w.W1s, w.W3s, w.W2s, dy, g["dx"], g["dWg"], g["dW1"],
                     g["dW3"], g["dW2"], g.get("dW1s"), g.get("dW3s"), g.get("dW2s"), ws)
    rc, raw = B.check_device_status(ws)
    assert rc == B.MOE_OK, (rc, raw)
    assert torch.equal(y, y_ref)
    for name in ref:
        assert torch.equal(g[name], ref[name]), name
