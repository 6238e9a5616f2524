"""Pins of the fp64 gradient oracle (oracle/backward.py) on the CPU.

The gradient oracle is checked against things other than itself:
- central finite differences of sum(dy * y) through the forward oracle (the C
  library, pinned on its own in test_oracle_pins.py), for every entry of every
  input, in both routing modes, at points where the expert selection does not
  change within the step;
- the forward value it passes through equals the forward oracle's;
- the routing Jacobians' invariants (softmax weights sum to one, the group
  weights are scale-free in the sigmoid scores), which catch sign and
  normalisation mistakes;
- special cases with exact answers (zero down projection, one expert);
- planted mistakes in a patched copy of the oracle, which the finite
  differences must catch.
"""
import numpy as np
import pytest

import oracle
from oracle import backward as bw


def _instance(seed, route):
    rng = np.random.default_rng(seed)
    T, d, I, Is = 5, 6, 3, 2
    E, k = (5, 2) if route == 0 else (8, 2)
    p = dict(
        x=rng.normal(0, 1.0, (T, d)),
        Wg=rng.normal(0, 0.8, (E, d)),
        W1=rng.normal(0, 0.5, (E, d, I)),
        W3=rng.normal(0, 0.5, (E, d, I)),
        W2=rng.normal(0, 0.5, (E, I, d)),
        W1s=rng.normal(0, 0.5, (d, Is)),
        W3s=rng.normal(0, 0.5, (d, Is)),
        W2s=rng.normal(0, 0.5, (Is, d)),
    )
    kw = dict(k=k, route=route)
    if route == 1:
        kw.update(bias=rng.normal(0, 0.05, E), n_group=4, topk_group=2, group_topn=2, route_scale=2.5)
    dy = rng.normal(0, 1.0, (T, d))
    return p, kw, dy


def _forward(p, kw):
    y, idx, _, _ = oracle.moe_forward(p["x"], p["Wg"], p["W1"], p["W3"], p["W2"], p["W1s"], p["W3s"], p["W2s"], **kw)
    return y, idx


def _fd_max_rel_err(p, kw, dy, grads, h=1e-5):
    """max over all inputs of |fd - analytic| / (1 + |analytic|), with the
    selection checked to stay fixed for every perturbed evaluation."""
    _, idx0 = _forward(p, kw)
    names = {"x": "dx", "Wg": "dWg", "W1": "dW1", "W3": "dW3", "W2": "dW2", "W1s": "dW1s", "W3s": "dW3s",
             "W2s": "dW2s"}
    worst = 0.0
    for name, gname in names.items():
        a = p[name]
        g = grads[gname]
        for i in np.ndindex(a.shape):
            v = a[i]
            a[i] = v + h
            yp, ip = _forward(p, kw)
            a[i] = v - h
            ym, im = _forward(p, kw)
            a[i] = v
            assert np.array_equal(ip, idx0) and np.array_equal(im, idx0), "selection moved: pick another point"
            fd = (np.sum(dy * yp) - np.sum(dy * ym)) / (2 * h)
            worst = max(worst, abs(fd - g[i]) / (1.0 + abs(g[i])))
    return worst


def _grads(p, kw, dy):
    return bw.moe_backward(p["x"], p["Wg"], p["W1"], p["W3"], p["W2"], p["W1s"], p["W3s"], p["W2s"], dy=dy, **kw)


@pytest.mark.parametrize("route", [0, 1])
def test_gradient_matches_finite_differences(route):
    p, kw, dy = _instance(11 + route, route)
    g = _grads(p, kw, dy)
    assert _fd_max_rel_err(p, kw, dy, g) < 1e-6


@pytest.mark.parametrize("route", [0, 1])
def test_forward_value_matches_forward_oracle(route):
    p, kw, dy = _instance(21 + route, route)
    g = _grads(p, kw, dy)
    y, idx = _forward(p, kw)
    assert np.array_equal(g["idx"], idx)
    rms = np.sqrt(np.mean(y ** 2))
    assert np.max(np.abs(g["y"] - y)) <= 1e-12 * rms


def test_routing_jacobian_invariants():
    rng = np.random.default_rng(5)
    for _ in range(20):
        k = int(rng.integers(1, 6))
        lg = rng.normal(0, 2, k)
        dw = rng.normal(0, 1, k)
        # softmax weights sum to 1: shifting every selected logit changes nothing
        w = np.exp(lg - lg.max())
        w /= w.sum()
        dl = bw.routing_backward(lg, w, dw, 0, 1.0)
        assert abs(dl.sum()) < 1e-12
        # group weights rs * s / sum(s) are unchanged by scaling all s together:
        # sum_m ds_m s_m = 0, i.e. sum_m dl_m / (1 - s_m) = 0
        s = 1.0 / (1.0 + np.exp(-lg))
        dl = bw.routing_backward(lg, 2.5 * s / s.sum(), dw, 1, 2.5)
        assert abs(np.sum(dl / (1.0 - s))) < 1e-12


def test_zero_down_projection_leaves_only_the_shared_expert_and_dW2():
    p, kw, dy = _instance(31, 0)
    p["W2"][:] = 0.0
    g = _grads(p, kw, dy)
    assert not g["dW1"].any() and not g["dW3"].any() and not g["dWg"].any()
    assert np.abs(g["dW2"]).max() > 0
    # no routed expert contributes to y, so dx is the shared expert's alone:
    # compare with finite differences of the shared-only layer
    q = dict(p)
    q["W1"] = np.zeros_like(p["W1"])
    gq = _grads(q, kw, dy)
    assert np.allclose(g["dx"], gq["dx"], rtol=0, atol=1e-14)
    assert _fd_max_rel_err(p, kw, dy, g) < 1e-6


def test_single_expert_k1_has_no_routing_gradient():
    # E = k = 1: the softmax weight is identically 1, so the gate gets no gradient
    rng = np.random.default_rng(41)
    T, d, I = 4, 3, 2
    p = dict(x=rng.normal(size=(T, d)), Wg=rng.normal(size=(1, d)), W1=rng.normal(size=(1, d, I)),
             W3=rng.normal(size=(1, d, I)), W2=rng.normal(size=(1, I, d)), W1s=None, W3s=None, W2s=None)
    dy = rng.normal(size=(T, d))
    g = bw.moe_backward(p["x"], p["Wg"], p["W1"], p["W3"], p["W2"], dy=dy, k=1)
    assert not g["dWg"].any()
    assert np.all(g["w"] == 1.0)


def test_combine_backward_is_the_adjoint_of_the_combine():
    # <dy, combine(Yp, w)> = <dO, Yp> = <dw, w>, with the forward oracle's combine
    rng = np.random.default_rng(7)
    T, d, E, k = 40, 24, 9, 3
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    _, _, _, row_of = oracle.dispatch(idx, E)
    Yp = rng.normal(size=(T * k, d))
    w = rng.uniform(0.1, 1.0, size=(T, k))
    dy = rng.normal(size=(T, d))
    y = oracle.combine(Yp, None, row_of, w)
    dO, dw = bw.combine_backward(dy, Yp, row_of, w)
    lhs = np.sum(dy * y)
    assert abs(lhs - np.sum(dO * Yp)) <= 1e-12 * (1 + abs(lhs))
    assert abs(lhs - np.sum(dw * w)) <= 1e-12 * (1 + abs(lhs))


@pytest.mark.parametrize("route", [0, 1])
def test_routing_backward_matches_directional_differences_of_the_weight_rule(route):
    # d/dh sum(dw * w(l + h v)) at h = 0 equals sum(dl * v), with w from the
    # forward oracle's weight rule for a fixed selection
    rng = np.random.default_rng(17 + route)
    T, E, k = 30, 12, 4
    lg = rng.normal(0, 1.5, size=(T, E))
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    dw = rng.normal(size=(T, k))
    v = rng.normal(size=(T, E))
    w0 = oracle.weights_for(lg, idx, route, 2.5)
    dl = np.zeros((T, E))
    for t in range(T):
        dl[t, idx[t]] = bw.routing_backward(lg[t, idx[t]], w0[t], dw[t], route, 2.5)
    h = 1e-6
    fd = (np.sum(dw * oracle.weights_for(lg + h * v, idx, route, 2.5))
          - np.sum(dw * oracle.weights_for(lg - h * v, idx, route, 2.5))) / (2 * h)
    an = np.sum(dl * v)
    assert abs(fd - an) <= 1e-7 * (1 + abs(an))


# ------------------------------------------------------------ planted mistakes
_ROUTING = bw.routing_backward


def _bad_swiglu_no_gate_term(X, W1, W3, W2, dO):
    G, U = X @ W1, X @ W3
    sg = 1.0 / (1.0 + np.exp(-G))
    A = G * sg
    H = A * U
    dH = dO @ W2.T
    dG = dH * U * sg  # mistake: silu'(g) taken as sigmoid(g)
    dU = dH * A
    return dG @ W1.T + dU @ W3.T, X.T @ dG, X.T @ dU, H.T @ dO, H @ W2


def _bad_swiglu_up_uses_g(X, W1, W3, W2, dO):
    G, U = X @ W1, X @ W3
    sg = 1.0 / (1.0 + np.exp(-G))
    A = G * sg
    H = A * U
    dH = dO @ W2.T
    dG = dH * U * (sg * (1.0 + G * (1.0 - sg)))
    dU = dH * G  # mistake: du = dh * g instead of dh * silu(g)
    return dG @ W1.T + dU @ W3.T, X.T @ dG, X.T @ dU, H.T @ dO, H @ W2


def _bad_routing_no_centering(lg_sel, w, dw, route, route_scale):
    if route == 0:
        return w * dw  # mistake: softmax Jacobian without the -sum(w dw) term
    return _ROUTING(lg_sel, w, dw, route, route_scale)


def _bad_routing_no_sigmoid_slope(lg_sel, w, dw, route, route_scale):
    if route == 1:
        s = 1.0 / (1.0 + np.exp(-lg_sel))
        Z = s.sum()
        return route_scale * (dw / Z - np.dot(dw, s) / (Z * Z))  # mistake: missing s (1 - s)
    return _ROUTING(lg_sel, w, dw, route, route_scale)


@pytest.mark.parametrize("name,fn,route", [
    ("swiglu_backward", _bad_swiglu_no_gate_term, 0),
    ("swiglu_backward", _bad_swiglu_up_uses_g, 1),
    ("routing_backward", _bad_routing_no_centering, 0),
    ("routing_backward", _bad_routing_no_sigmoid_slope, 1),
])
def test_planted_mistakes_are_caught(monkeypatch, name, fn, route):
    p, kw, dy = _instance(11 + route, route)
    monkeypatch.setattr(bw, name, fn)
    g = _grads(p, kw, dy)
    assert _fd_max_rel_err(p, kw, dy, g) > 1e-3
