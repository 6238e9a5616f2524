"""moe_backward at the DeepSeek-V3 prefill shapes (T=4096, d=7168, 256 experts
top-8, inter 2048, shared expert 2048), in the configuration the benchmark
times (bf16 gradients), against the fp64 gradient oracle on outputs it can
compute piece by piece: the weight gradients of sampled experts (the most and
least loaded and a random one), the shared expert's weight gradients over all
tokens, and the input gradient of sampled tokens (their k experts, the shared
expert and the router's part).  The bounds are those of the small-size
backward tests: ||err||_F <= 1e-2 ||ref||_F and max|err| <= 2e-2 max|ref|."""
import numpy as np
import pytest
import torch

from oracle import backward as obw
import oracle
from mixture_experts_ffn_17_b200 import binding as B
from mixture_experts_ffn_17_b200 import build as libbuild
from mixture_experts_ffn_17_b200 import workloads

from gpu_util import expert_weights_f64, oracle_logits, route_with_exemptions, run_forward
from parity import dec, to_np

pytestmark = pytest.mark.gpu

TOL_FRO, TOL_MAX = 1e-2, 2e-2


@pytest.fixture(scope="module", autouse=True)
def built():
    libbuild.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _close(d, o, what):
    d = np.asarray(d, dtype=np.float64)
    fro = float(np.linalg.norm(d - o) / np.linalg.norm(o))
    mx = float(np.abs(d - o).max() / np.abs(o).max())
    print(f"{what}: fro {fro:.2e} max {mx:.2e}")
    assert fro <= TOL_FRO and mx <= TOL_MAX, (what, fro, mx)


def test_v3_prefill_backward_sampled():
    _check_backward_sampled(workloads.make(workloads.CONFIGS["prefill"], device="cuda"))


def test_large_batch_narrow_layer_skewed_backward():
    # 100,000 tokens of a narrow layer with Zipf routing: the weight gradients
    # of the hot experts contract over tens of thousands of rows (a K loop of
    # hundreds of 64-row steps per tile), far past the V3 prefill segments
    w = workloads.make_small("skewed", device="cuda", T=100_000, d=256, E=64, k=8, inter=128, shared_inter=128)
    c = _check_backward_sampled(w)
    assert c.max() > 20_000


def _check_backward_sampled(w):
    cfg = w.cfg
    dy = torch.randn(cfg.T, cfg.d, generator=torch.Generator(device="cuda").manual_seed(314), device="cuda")
    shape = B.shape_of(cfg, B.MOE_BF16)
    ws = B.alloc_backward_workspace(shape)
    e = lambda *sz: torch.empty(sz, dtype=torch.bfloat16, device="cuda")
    g = dict(dx=e(cfg.T, cfg.d), dWg=e(cfg.E, cfg.d), dW1=e(cfg.E, cfg.d, cfg.inter), dW3=e(cfg.E, cfg.d, cfg.inter),
             dW2=e(cfg.E, cfg.inter, cfg.d), dW1s=e(cfg.d, cfg.shared_inter), dW3s=e(cfg.d, cfg.shared_inter),
             dW2s=e(cfg.shared_inter, cfg.d))
    B.backward(shape, w.x, w.Wg, w.bias, w.W1, w.W3, w.W2, w.W1s, w.W3s, w.W2s, dy, *g.values(), ws)
    rc, raw = B.check_device_status(ws)
    assert rc == B.MOE_OK, (rc, raw)

    # the routing the gradient was taken at (the device's, exact up to reported near-ties)
    _, idx, _, counts, _ = run_forward(w)
    lg = oracle_logits(w)
    _, _, merged, report, n_near = route_with_exemptions(w, lg, to_np(idx))
    assert len(report) <= n_near
    wts = oracle.weights_for(lg, merged, cfg.route, cfg.route_scale)
    x = dec(w.x)
    dy64 = to_np(dy).astype(np.float64)
    c = np.bincount(merged.ravel(), minlength=cfg.E)

    # weight gradients of sampled experts: the expert's rows (tokens in order)
    # with output gradient w * dy
    order = np.argsort(c, kind="stable")
    rng = np.random.default_rng(cfg.seed)
    experts = [int(order[-1]), int(order[np.nonzero(c[order] > 0)[0][0]]), int(rng.integers(cfg.E))]
    for ex in experts:
        tok, slot = np.nonzero(merged == ex)
        W1, W3, W2 = expert_weights_f64(w, ex)
        _, dW1, dW3, dW2, _ = obw.swiglu_backward(x[tok], W1, W3, W2, wts[tok, slot][:, None] * dy64[tok])
        for name, ref in (("dW1", dW1), ("dW3", dW3), ("dW2", dW2)):
            _close(to_np(g[name][ex].float()), ref, f"{name}[{ex}] ({len(tok)} rows)")

    # the shared expert over every token
    dXs, dW1s, dW3s, dW2s, _ = obw.swiglu_backward(x, dec(w.W1s), dec(w.W3s), dec(w.W2s), dy64)
    for name, ref in (("dW1s", dW1s), ("dW3s", dW3s), ("dW2s", dW2s)):
        _close(to_np(g[name].float()), ref, name)

    # input gradient of sampled tokens: each selected expert's input gradient
    # and its output (for the routing weights' gradient), the shared expert's
    # input gradient, and dl Wg
    Wg = dec(w.Wg)
    for t in (0, 1234, cfg.T - 1):
        dx_t = dXs[t].copy()
        dw_t = np.zeros(cfg.k)
        for j, ex in enumerate(merged[t]):
            W1, W3, W2 = expert_weights_f64(w, int(ex))
            dX, _, _, _, o = obw.swiglu_backward(x[t:t + 1], W1, W3, W2, wts[t, j] * dy64[t:t + 1])
            dx_t += dX[0]
            dw_t[j] = float(dy64[t] @ o[0])
        dl = obw.routing_backward(lg[t, merged[t]], wts[t], dw_t, cfg.route, cfg.route_scale)
        dx_t += dl @ Wg[merged[t]]
        _close(to_np(g["dx"][t].float()), dx_t, f"dx[{t}]")
    return c
