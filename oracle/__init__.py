"""fp64 CPU oracle of the DeepSeek-V3-style MoE feed-forward layer.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library in
``mixture_experts_ffn_17_b200`` never imports it and shares no code with it;
this package never imports that library either.

The arithmetic lives in ``moe_oracle.c`` (plain C, fp64, OpenMP over
independent tokens).  This module is a ctypes shim plus small composition
helpers written in the order of the pages' definitions:

* gate linear, top-k then softmax over the k (n4n.ai page, "The architecture
  in one diagram", simplified block pseudocode);
* bincount + per-expert token lists in token order, y += w * expert(x),
  y += shared(x) (atlas page "DeepSeek-V3.2-Exp / Mixture of experts / Shared
  expert", "Code" section, MoE forward block);
* SwiGLU g=xW1, u=xW3, a=g*sigmoid(g), h=a*u, y=hW2 (same atlas page, "All 5
  steps");
* sigmoid group-limited routing with selection bias (the FP8 group-routing
  workload's statement; the Baidu page's "Hierarchical Dynamic Routing" and the
  freedom251 page's "How V3 balances expert traffic" only hint at it).

``backward.py`` (numpy, fp64) holds the layer's gradient: the derivative of
the forward definition above, with the expert selection held fixed.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into libmoe_oracle.so (gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-fno-fast-math",
               "-ffp-contract=off", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        # ORACLE_LIB: load another build of moe_oracle.c instead (the mutation
        # test points it at deliberately broken copies to show the pins fail)
        path = os.environ.get("ORACLE_LIB") or build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64, i32, f64 = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        sig = {
            "oracle_decode_bf16": [i64, P, P],
            "oracle_decode_f32": [i64, P, P],
            "oracle_decode_e4m3_blocks": [i64, i64, i64, P, P, P],
            "oracle_logits": [i64, i64, i64, P, P, P],
            "oracle_route_topk_softmax": [i64, i32, i32, P, P, P, P],
            "oracle_route_sigmoid_group": [i64, i32, i32, i32, i32, i32, f64, P, P, P, P, P, P],
            "oracle_weights_topk_softmax": [i64, i32, i32, P, P, P],
            "oracle_weights_sigmoid": [i64, i32, i32, f64, P, P, P],
            "oracle_dispatch": [i64, i32, i32, P, P, P, P, P],
            "oracle_swiglu_rows": [i64, i64, i64, P, P, P, P, P],
            "oracle_combine": [i64, i32, i64, P, P, P, P, P],
            "oracle_route_topk_softmax_limited": [i64, i32, i32, P, P, P, P, P],
            "oracle_expert_utilisation": [i32, P, P, P],
            "oracle_moe_forward": [i64, i64, i32, i32, i64, i64, i32, i32, i32, i32, f64,
                                   P, P, P, P, P, P, P, P, P, P, P, P, P, P],
            "oracle_moe_forward_ep_rank": [i64, i64, i32, i32, i64, i64, i32, i32, i32, i32, f64,
                                           P, P, P, i32, i32, P, P, P, P, P, P, P],
        }
        for name, args in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int if name in ("oracle_dispatch", "oracle_moe_forward",
                                                  "oracle_moe_forward_ep_rank") else None
        L.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_value.restype = ctypes.c_double
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- decoding
def decode(a) -> np.ndarray:
    """Widen a stored array (numpy float32/float64, numpy uint16 holding bf16
    bits, or a CPU torch tensor of float32/bfloat16) to fp64, exactly."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().contiguous().cpu()
            if a.dtype == torch.bfloat16:
                a = a.view(torch.int16).numpy().view(np.uint16)
            elif a.dtype == torch.float32:
                a = a.numpy()
            elif a.dtype == torch.float64:
                return a.numpy().copy()
            else:
                raise TypeError(f"decode: unsupported torch dtype {a.dtype}")
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(a)
    out = np.empty(a.shape, dtype=np.float64)
    if a.dtype == np.uint16:
        lib().oracle_decode_bf16(a.size, _p(a), _p(out))
    elif a.dtype == np.float32:
        lib().oracle_decode_f32(a.size, _p(a), _p(out))
    elif a.dtype == np.float64:
        out[...] = a
    else:
        raise TypeError(f"decode: unsupported dtype {a.dtype}")
    return out


def decode_e4m3_blocks(q: np.ndarray, scale: np.ndarray, blk: int = 128) -> np.ndarray:
    """Dequantise a block-scaled FP8 e4m3 matrix [rows, cols] to fp64 (code * scale)."""
    q = _c(q, np.uint8)
    scale = _c(scale, np.float32)
    rows, cols = q.shape
    out = np.empty((rows, cols), dtype=np.float64)
    lib().oracle_decode_e4m3_blocks(rows, cols, blk, _p(q), _p(scale), _p(out))
    return out


def e4m3_value(code: int) -> float:
    return lib().oracle_e4m3_value(int(code))


# ---------------------------------------------------------------- router
def logits(x: np.ndarray, Wg: np.ndarray) -> np.ndarray:
    x = _c(x, np.float64)
    Wg = _c(Wg, np.float64)
    T, d = x.shape
    E = Wg.shape[0]
    out = np.empty((T, E), dtype=np.float64)
    lib().oracle_logits(T, d, E, _p(x), _p(Wg), _p(out))
    return out


def route_topk_softmax(lg: np.ndarray, k: int):
    """-> idx [T,k] int32 (descending), w [T,k] fp64, gaps [T,k] fp64."""
    lg = _c(lg, np.float64)
    T, E = lg.shape
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    gaps = np.empty((T, k), dtype=np.float64)
    lib().oracle_route_topk_softmax(T, E, k, _p(lg), _p(idx), _p(w), _p(gaps))
    return idx, w, gaps


def route_topk_softmax_limited(lg: np.ndarray, allowed: np.ndarray, k: int):
    """Device-limited page-1 routing: experts with allowed[e] == 0 are masked
    to -inf before the top-k.  -> idx, w, gaps as route_topk_softmax."""
    lg = _c(lg, np.float64)
    al = _c(allowed, np.uint8)
    T, E = lg.shape
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    gaps = np.empty((T, k), dtype=np.float64)
    lib().oracle_route_topk_softmax_limited(T, E, k, _p(lg), _p(al), _p(idx), _p(w), _p(gaps))
    return idx, w, gaps


def expert_utilisation(counts: np.ndarray):
    """-> utilisation [E] fp64 (counts / total), flags [E] int32 (+1 > 2x mean, -1 < 0.1x mean)."""
    c = _c(counts, np.int32)
    E = c.shape[0]
    util = np.empty(E, dtype=np.float64)
    flag = np.empty(E, dtype=np.int32)
    lib().oracle_expert_utilisation(E, _p(c), _p(util), _p(flag))
    return util, flag


def route_sigmoid_group(lg: np.ndarray, bias, k: int, n_group: int, topk_group: int,
                        group_topn: int = 2, route_scale: float = 2.5):
    """-> idx [T,k], w [T,k], gaps [T,k], group-boundary gap [T]."""
    lg = _c(lg, np.float64)
    T, E = lg.shape
    b = None if bias is None else _c(bias, np.float64)
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    gaps = np.empty((T, k), dtype=np.float64)
    ggap = np.empty((T,), dtype=np.float64)
    lib().oracle_route_sigmoid_group(T, E, k, n_group, topk_group, group_topn, route_scale,
                                     _p(lg), _p(b), _p(idx), _p(w), _p(gaps), _p(ggap))
    return idx, w, gaps, ggap


def weights_for(lg: np.ndarray, idx: np.ndarray, route: int = 0, route_scale: float = 2.5) -> np.ndarray:
    """Routing weights the rule assigns to a given index set (same slot order)."""
    lg = _c(lg, np.float64)
    idx = _c(idx, np.int32)
    T, E = lg.shape
    k = idx.shape[1]
    w = np.empty((T, k), dtype=np.float64)
    if route == 0:
        lib().oracle_weights_topk_softmax(T, E, k, _p(lg), _p(idx), _p(w))
    else:
        lib().oracle_weights_sigmoid(T, E, k, route_scale, _p(lg), _p(idx), _p(w))
    return w


# ---------------------------------------------------------------- dispatch
def dispatch(idx: np.ndarray, E: int):
    """-> counts [E], offsets [E+1], perm_token [T*k], row_of [T*k] (all int32)."""
    idx = _c(idx, np.int32)
    T, k = idx.shape
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    perm = np.empty(T * k, dtype=np.int32)
    row_of = np.empty(T * k, dtype=np.int32)
    rc = lib().oracle_dispatch(T, k, E, _p(idx), _p(counts), _p(offsets), _p(perm), _p(row_of))
    if rc != 0:
        raise ValueError("oracle.dispatch: expert index out of range")
    return counts, offsets, perm, row_of


# ---------------------------------------------------------------- experts
def swiglu_rows(x: np.ndarray, W1: np.ndarray, W3: np.ndarray, W2: np.ndarray) -> np.ndarray:
    """o = (silu(x W1) * (x W3)) W2 for every row of x, fp64."""
    x = _c(np.atleast_2d(x), np.float64)
    W1, W3, W2 = (_c(a, np.float64) for a in (W1, W3, W2))
    n, d = x.shape
    I = W1.shape[1]
    out = np.empty((n, d), dtype=np.float64)
    lib().oracle_swiglu_rows(n, d, I, _p(x), _p(W1), _p(W3), _p(W2), _p(out))
    return out


def combine(Yp: np.ndarray, Ys, row_of: np.ndarray, w: np.ndarray) -> np.ndarray:
    """y[t] = sum_j w[t,j] Yp[row_of[t,j]] + Ys[t] in fp64 (Ys may be None)."""
    Yp = _c(Yp, np.float64)
    Ys = None if Ys is None else _c(Ys, np.float64)
    row_of = _c(row_of, np.int32)
    w = _c(w, np.float64)
    T, k = w.shape
    d = Yp.shape[1]
    y = np.empty((T, d), dtype=np.float64)
    lib().oracle_combine(T, k, d, _p(Yp), _p(Ys), _p(row_of), _p(w), _p(y))
    return y


def moe_forward(x, Wg, W1, W3, W2, W1s=None, W3s=None, W2s=None, *, k: int, route: int = 0,
                bias=None, n_group: int = 1, topk_group: int = 1, group_topn: int = 2,
                route_scale: float = 2.5, force_idx=None):
    """Whole layer in fp64 for sizes that fit in host memory.

    Returns (y [T,d], idx [T,k], w [T,k], logits [T,E])."""
    x, Wg, W1, W3, W2 = (_c(a, np.float64) for a in (x, Wg, W1, W3, W2))
    T, d = x.shape
    E, _, I = W1.shape
    if W1s is None:
        Is = 0
        W1s = W3s = W2s = np.zeros(1)
    else:
        Is = W1s.shape[1]
    W1s, W3s, W2s = (_c(a, np.float64) for a in (W1s, W3s, W2s))
    b = None if bias is None else _c(bias, np.float64)
    fi = None if force_idx is None else _c(force_idx, np.int32)
    y = np.empty((T, d), dtype=np.float64)
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    lg = np.empty((T, E), dtype=np.float64)
    rc = lib().oracle_moe_forward(T, d, E, k, I, Is, route, n_group, topk_group, group_topn, route_scale,
                                  _p(x), _p(Wg), _p(b), _p(W1), _p(W3), _p(W2), _p(W1s), _p(W3s), _p(W2s),
                                  _p(fi), _p(y), _p(idx), _p(w), _p(lg))
    if rc != 0:
        raise MemoryError("oracle_moe_forward: allocation failed")
    return y, idx, w, lg


# ------------------------------------------------------- expert parallelism
def ep_partition(E: int, Is: int, rank: int, size: int):
    """Rank `rank` of `size` holds experts [e_lo, e_hi) and the shared expert's
    hidden features [i_lo, i_hi) (atlas page, "Code" section, MoE constructor
    block: n_local_experts = E // world_size, experts_start_idx = rank *
    n_local_experts; the shared MLP's W1/W3 are column-parallel and its W2
    row-parallel, so each rank holds an even slice of its hidden features)."""
    el, il = E // size, Is // size
    return rank * el, (rank + 1) * el, rank * il, (rank + 1) * il


def moe_forward_ep_rank(x, Wg, W1l, W3l, W2l, W1sl=None, W3sl=None, W2sl=None, *, e_lo: int, k: int,
                        route: int = 0, bias=None, n_group: int = 1, topk_group: int = 1, group_topn: int = 2,
                        route_scale: float = 2.5) -> np.ndarray:
    """One rank's partial y of the expert-parallel layer: its experts' weighted
    outputs (W1l/W3l/W2l hold experts e_lo, e_lo+1, ...) plus its slice of the
    shared expert (W1sl [d, Isl], W3sl [d, Isl], W2sl [Isl, d]); the all-reduce
    of these over the ranks is the layer (atlas page, "Code" section, MoE
    forward block)."""
    x, Wg, W1l, W3l, W2l = (_c(a, np.float64) for a in (x, Wg, W1l, W3l, W2l))
    T, d = x.shape
    E = Wg.shape[0]
    El, _, I = W1l.shape
    if W1sl is None or W1sl.shape[1] == 0:
        Isl = 0
        W1sl = W3sl = W2sl = np.zeros(1)
    else:
        Isl = W1sl.shape[1]
    W1sl, W3sl, W2sl = (_c(a, np.float64) for a in (W1sl, W3sl, W2sl))
    b = None if bias is None else _c(bias, np.float64)
    y = np.empty((T, d), dtype=np.float64)
    rc = lib().oracle_moe_forward_ep_rank(T, d, E, k, I, Isl, route, n_group, topk_group, group_topn, route_scale,
                                          _p(x), _p(Wg), _p(b), e_lo, El, _p(W1l), _p(W3l), _p(W2l), _p(W1sl),
                                          _p(W3sl), _p(W2sl), _p(y))
    if rc != 0:
        raise MemoryError("oracle_moe_forward_ep_rank: allocation failed")
    return y
