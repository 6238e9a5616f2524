"""fp64 gradient of the MoE feed-forward layer.

TEST INFRASTRUCTURE ONLY, like the rest of this package: only the tests may
import it.  The library's backward pass (moe_backward and its combine and
routing steps) is checked against it.

The pages define the forward pass only (n4n.ai page "DeepSeek-V3's
mixture-of-experts architecture explained", "The architecture in one diagram";
atlas page "DeepSeek-V3.2-Exp / Mixture of experts / Shared expert", "All 5
steps" and the MoE forward block of its "Code" section) and speak of training
(n4n page, "Training infrastructure that made this possible") without printing
its arithmetic.  The gradient here is the derivative of that forward
definition by the chain rule, step by step in reverse order:

  y_t = sum_j w_tj o_tj + shared(x_t),  o = h W2[e],  h = silu(g) * u,
  g = x W1[e],  u = x W3[e],  logits l = x Wg^T,
  page-1 routing w = softmax over the k selected logits,
  group routing  w_j = rs * s_j / sum_i s_i with s = sigmoid(l).

The expert selection is piecewise constant in the inputs, so it is held fixed
(taken from the forward oracle); the gradient is that of the layer on the
open set where the selection does not change.  The selection bias only moves
the selection and has no gradient.  Each expert's rows are processed with
numpy matrix products (library primitives for the sums over rows and
features); the routing Jacobians are written out per token.
"""
from __future__ import annotations

import numpy as np

from . import dispatch as _dispatch
from . import logits as _logits
from . import route_sigmoid_group as _route_group
from . import route_topk_softmax as _route_topk
from . import swiglu_rows as _swiglu_rows
from . import weights_for as _weights_for


def _sigmoid(z: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-z))


def swiglu_backward(X: np.ndarray, W1: np.ndarray, W3: np.ndarray, W2: np.ndarray, dO: np.ndarray):
    """Rows X [n, d] through o = (silu(X W1) * (X W3)) W2 with output gradient
    dO [n, d] -> (dX [n, d], dW1 [d, I], dW3 [d, I], dW2 [I, d], O [n, d]).

    silu(g) = g sigmoid(g), so silu'(g) = sigmoid(g) (1 + g (1 - sigmoid(g)))."""
    G = X @ W1
    U = X @ W3
    sg = _sigmoid(G)
    A = G * sg
    H = A * U
    O = H @ W2
    dW2 = H.T @ dO
    dH = dO @ W2.T
    dG = dH * U * (sg * (1.0 + G * (1.0 - sg)))
    dU = dH * A
    dW1 = X.T @ dG
    dW3 = X.T @ dU
    dX = dG @ W1.T + dU @ W3.T
    return dX, dW1, dW3, dW2, O


def combine_backward(dy: np.ndarray, Yp: np.ndarray, row_of: np.ndarray, w: np.ndarray):
    """Adjoint of y[t] = sum_j w[t,j] Yp[row_of[t,j]] (+ shared): for every
    (t, j) with r = row_of[t*k + j] >= 0, dO[r] = w[t,j] dy[t] and
    dw[t,j] = dy[t] . Yp[r]; dw is 0 where r < 0.  -> (dO [T*k, d], dw [T, k])."""
    dy = np.asarray(dy, dtype=np.float64)
    Yp = np.asarray(Yp, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    T, k = w.shape
    r = np.asarray(row_of).reshape(T, k)
    dO = np.zeros_like(Yp)
    dw = np.zeros((T, k))
    ok = r >= 0
    tt, jj = np.nonzero(ok)
    dO[r[tt, jj]] = w[tt, jj][:, None] * dy[tt]
    dw[tt, jj] = np.einsum("nd,nd->n", dy[tt], Yp[r[tt, jj]])
    return dO, dw


def routing_backward(lg_sel: np.ndarray, w: np.ndarray, dw: np.ndarray, route: int, route_scale: float) -> np.ndarray:
    """Gradient of the k selected logits of one token from the gradient dw of
    its routing weights.

    page-1 (w = softmax(l_sel)): dl = w * (dw - sum_i w_i dw_i).
    group (w_j = rs s_j / Z, Z = sum_i s_i, s = sigmoid(l_sel)):
      ds_m = rs (dw_m / Z - sum_j dw_j s_j / Z^2),  dl = ds * s (1 - s)."""
    if route == 0:
        return w * (dw - np.dot(w, dw))
    s = _sigmoid(lg_sel)
    Z = s.sum()
    ds = route_scale * (dw / Z - np.dot(dw, s) / (Z * Z))
    return ds * s * (1.0 - s)


def moe_backward(x, Wg, W1, W3, W2, W1s=None, W3s=None, W2s=None, *, dy, k: int, route: int = 0, bias=None,
                 n_group: int = 1, topk_group: int = 1, group_topn: int = 2, route_scale: float = 2.5,
                 force_idx=None):
    """Gradient of sum(dy * y) for the layer y = moe_forward(...) (fp64).

    Shapes as the forward oracle: x [T, d], Wg [E, d], W1/W3 [E, d, I],
    W2 [E, I, d], shared W1s/W3s [d, Is], W2s [Is, d] (or None).
    Returns a dict with dx, dWg, dW1, dW3, dW2 (and dW1s, dW3s, dW2s when the
    shared expert is present); the intermediate gradients dO_perm (of the
    routed expert outputs, permuted order), dw (of the routing weights) and dl
    (of the logits); and the selection idx, weights w, logits lg, permuted
    expert outputs Y_perm, row_of and the forward output y it was computed at.
    force_idx [T, k]: use this selection (weights from the same rule) instead
    of selecting, as the forward oracle's force_idx does."""
    x, Wg, W1, W3, W2, dy = (np.asarray(a, dtype=np.float64) for a in (x, Wg, W1, W3, W2, dy))
    T, d = x.shape
    E = W1.shape[0]
    lg = _logits(x, Wg)
    if force_idx is not None:
        idx = np.ascontiguousarray(force_idx, dtype=np.int32)
        w = _weights_for(lg, idx, route, route_scale)
    elif route == 0:
        idx, w, _ = _route_topk(lg, k)
    else:
        idx, w, _, _ = _route_group(lg, bias, k, n_group, topk_group, group_topn, route_scale)

    # forward: every routed expert output in the permuted row order (experts
    # ascending, then tokens), then y
    _, offsets, perm, row_of = _dispatch(idx, E)
    Yp = np.zeros((T * k, d))
    for e in range(E):
        rows = slice(offsets[e], offsets[e + 1])
        if offsets[e + 1] > offsets[e]:
            Yp[rows] = _swiglu_rows(x[perm[rows]], W1[e], W3[e], W2[e])
    r = row_of.reshape(T, k)
    y = np.einsum("tj,tjd->td", w, Yp[r])
    # backward through the combine, then through each expert's SwiGLU
    dO, dw = combine_backward(dy, Yp, row_of, w)
    dx = np.zeros((T, d))
    dW1 = np.zeros_like(W1)
    dW3 = np.zeros_like(W3)
    dW2 = np.zeros_like(W2)
    for e in range(E):
        if offsets[e + 1] == offsets[e]:
            continue
        rows = slice(offsets[e], offsets[e + 1])
        toks = perm[rows]
        dX, g1, g3, g2, _ = swiglu_backward(x[toks], W1[e], W3[e], W2[e], dO[rows])
        np.add.at(dx, toks, dX)
        dW1[e] += g1
        dW3[e] += g3
        dW2[e] += g2
    # routing weights -> logits -> x and Wg
    dl = np.zeros((T, E))
    for t in range(T):
        dl[t, idx[t]] = routing_backward(lg[t, idx[t]], w[t], dw[t], route, route_scale)
    dx += dl @ Wg
    dWg = dl.T @ x
    out = dict(dx=dx, dWg=dWg, dW1=dW1, dW3=dW3, dW2=dW2, idx=idx, w=w, lg=lg, dw=dw, dl=dl, dO_perm=dO,
               Y_perm=Yp, row_of=row_of)
    if W1s is not None:
        W1s, W3s, W2s = (np.asarray(a, dtype=np.float64) for a in (W1s, W3s, W2s))
        dXs, out["dW1s"], out["dW3s"], out["dW2s"], Os = swiglu_backward(x, W1s, W3s, W2s, dy)
        y += Os
        out["dx"] = dx + dXs
    out["y"] = y
    return out
