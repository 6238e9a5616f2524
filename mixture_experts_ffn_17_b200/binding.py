"""ctypes binding of libmoe (include/moe.h): argument marshalling only.

Every function takes torch CUDA tensors, passes their data pointers and the
current CUDA stream to the C entry point of the same name, and raises
MoeError on a non-OK status.  All computation happens in the library's
kernels; nothing here computes on the host.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, \
    MOE_ERR_DEVICE_TIMEOUT, MOE_ERR_DEVICE_BOUNDS = range(7)
MOE_BF16, MOE_E4M3, MOE_F32 = 0, 1, 2
MOE_ROUTE_TOPK_SOFTMAX, MOE_ROUTE_SIGMOID_GROUP = 0, 1

EXPORTED = ("moe_workspace_size", "moe_router_topk", "moe_permute", "moe_grouped_swiglu", "moe_combine",
            "moe_forward", "moe_forward_profiled", "moe_check_device_status", "moe_status_string", "moe_version",
            "moe_permute_noalloc", "moe_router_topk_limited", "moe_expert_utilisation", "moe_forward_ep",
            "moe_forward_launches", "moe_combine_backward", "moe_router_backward", "moe_backward_workspace_size",
            "moe_backward", "moe_shared_expert", "moe_ep_regroup_layout", "moe_gather_rows", "moe_forward_train",
            "moe_backward_saved")
NUM_STAGE_EVENTS = 6
STAGES = ("router", "dispatch", "experts_up", "experts_down", "combine")


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} (status {status})")
        self.status = status


class MoeShape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int32), ("E", ctypes.c_int32), ("k", ctypes.c_int32),
                ("inter", ctypes.c_int32), ("shared_inter", ctypes.c_int32), ("route", ctypes.c_int32),
                ("n_group", ctypes.c_int32), ("topk_group", ctypes.c_int32), ("group_topn", ctypes.c_int32),
                ("route_scale", ctypes.c_float), ("w_dtype", ctypes.c_int32), ("y_dtype", ctypes.c_int32)]


def make_shape(T, d, E, k, inter, shared_inter, route=0, n_group=1, topk_group=1, group_topn=2,
               route_scale=1.0, w_dtype=MOE_BF16, y_dtype=MOE_F32) -> MoeShape:
    return MoeShape(int(T), int(d), int(E), int(k), int(inter), int(shared_inter), int(route), int(n_group),
                    int(topk_group), int(group_topn), float(route_scale), int(w_dtype), int(y_dtype))


def shape_of(cfg, y_dtype=MOE_F32) -> MoeShape:
    """MoeShape of a workloads.Config."""
    return make_shape(cfg.T, cfg.d, cfg.E, cfg.k, cfg.inter, cfg.shared_inter, cfg.route, cfg.n_group,
                      cfg.topk_group, cfg.group_topn, cfg.route_scale, MOE_E4M3 if cfg.fp8 else MOE_BF16, y_dtype)


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmoe.so; raises when it is missing (there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libmoe.so not built ({LIB_PATH}); run `python -m mixture_experts_ffn_17_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, S, sz = ctypes.c_void_p, ctypes.POINTER(MoeShape), ctypes.c_size_t
        L.moe_workspace_size.argtypes = [S]
        L.moe_workspace_size.restype = sz
        L.moe_router_topk.argtypes = [S, P, P, P, P, P, P, P, sz, P]
        L.moe_permute.argtypes = [S, P, P, P, P, P, P, P, P, sz, P]
        L.moe_permute_noalloc.argtypes = [S, P, P, P, P, P, P, P, P]
        L.moe_router_topk_limited.argtypes = [S, P, P, P, P, P, P, P, sz, P]
        L.moe_router_topk_limited.restype = ctypes.c_int
        L.moe_expert_utilisation.argtypes = [S, P, P, P, P]
        L.moe_expert_utilisation.restype = ctypes.c_int
        L.moe_permute_noalloc.restype = ctypes.c_int
        L.moe_grouped_swiglu.argtypes = [S, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, sz, P]
        L.moe_combine.argtypes = [S, P, P, P, P, P, P]
        L.moe_combine_backward.argtypes = [S, P, P, P, P, P, P, P]
        L.moe_router_backward.argtypes = [S, P, P, P, P, P, P]
        L.moe_forward.argtypes = [S, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, sz, P]
        L.moe_forward_profiled.argtypes = [S, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, sz, P, P]
        I = ctypes.c_int
        L.moe_forward_ep.argtypes = [S, I, I, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, sz, P]
        L.moe_forward_launches.argtypes = [S]
        L.moe_forward_launches.restype = ctypes.c_int
        L.moe_shared_expert.argtypes = [S, P, P, P, P, P, P, sz, P]
        L.moe_ep_regroup_layout.argtypes = [ctypes.c_int, ctypes.c_int, P, P, P, P, P]
        L.moe_gather_rows.argtypes = [P, P, ctypes.c_int64, ctypes.c_int, P, P]
        L.moe_backward_workspace_size.argtypes = [S]
        L.moe_backward_workspace_size.restype = sz
        L.moe_backward.argtypes = [S] + [P] * 18 + [P, sz, P]
        L.moe_forward_train.argtypes = [S] + [P] * 10 + [P, sz, P]
        L.moe_backward_saved.argtypes = [S] + [P] * 17 + [P, sz, P]
        L.moe_check_device_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint32)]
        for fn in ("moe_router_topk", "moe_permute", "moe_grouped_swiglu", "moe_combine", "moe_combine_backward",
                   "moe_router_backward", "moe_forward",
                   "moe_forward_profiled", "moe_forward_ep", "moe_backward", "moe_shared_expert", "moe_ep_regroup_layout", "moe_gather_rows",
                   "moe_forward_train", "moe_backward_saved", "moe_check_device_status"):
            getattr(L, fn).restype = ctypes.c_int
        L.moe_status_string.argtypes = [ctypes.c_int]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_version.argtypes = []
        L.moe_version.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libmoe must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(rc: int, where: str):
    if rc != MOE_OK:
        raise MoeError(rc, where)


def workspace_size(shape: MoeShape) -> int:
    return int(lib().moe_workspace_size(ctypes.byref(shape)))


def alloc_workspace(shape: MoeShape, device="cuda") -> torch.Tensor:
    n = workspace_size(shape)
    if n == 0:
        raise MoeError(MOE_ERR_UNSUPPORTED, "moe_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def router_topk(shape, x, Wg, bias, topk_idx, topk_w, logits, ws, stream=None):
    _check(lib().moe_router_topk(ctypes.byref(shape), _ptr(x), _ptr(Wg), _ptr(bias), _ptr(topk_idx), _ptr(topk_w),
                                 _ptr(logits), _ptr(ws), ws.numel() if ws is not None else 0, _stream(stream)),
           "moe_router_topk")


def router_topk_limited(shape, x, Wg, allowed, topk_idx, topk_w, logits, ws, stream=None):
    _check(lib().moe_router_topk_limited(ctypes.byref(shape), _ptr(x), _ptr(Wg), _ptr(allowed), _ptr(topk_idx),
                                         _ptr(topk_w), _ptr(logits), _ptr(ws), ws.numel() if ws is not None else 0,
                                         _stream(stream)), "moe_router_topk_limited")


def expert_utilisation(shape, counts, utilisation, flags, stream=None):
    _check(lib().moe_expert_utilisation(ctypes.byref(shape), _ptr(counts), _ptr(utilisation), _ptr(flags),
                                        _stream(stream)), "moe_expert_utilisation")


def permute(shape, topk_idx, counts, offsets, perm_token, row_of, x, x_perm, ws, stream=None):
    _check(lib().moe_permute(ctypes.byref(shape), _ptr(topk_idx), _ptr(counts), _ptr(offsets), _ptr(perm_token),
                             _ptr(row_of), _ptr(x), _ptr(x_perm), _ptr(ws), ws.numel() if ws is not None else 0,
                             _stream(stream)), "moe_permute")


def grouped_swiglu(shape, x, x_perm, offsets, W1, W3, W2, s1, s3, s2, W1s, W3s, W2s, Y_perm, Y_shared, ws,
                   stream=None):
    _check(lib().moe_grouped_swiglu(ctypes.byref(shape), _ptr(x), _ptr(x_perm), _ptr(offsets), _ptr(W1), _ptr(W3),
                                    _ptr(W2), _ptr(s1), _ptr(s3), _ptr(s2), _ptr(W1s), _ptr(W3s), _ptr(W2s),
                                    _ptr(Y_perm), _ptr(Y_shared), _ptr(ws), ws.numel() if ws is not None else 0,
                                    _stream(stream)), "moe_grouped_swiglu")


def combine(shape, Y_perm, Y_shared, row_of, topk_w, y, stream=None):
    _check(lib().moe_combine(ctypes.byref(shape), _ptr(Y_perm), _ptr(Y_shared), _ptr(row_of), _ptr(topk_w), _ptr(y),
                             _stream(stream)), "moe_combine")


def combine_backward(shape, dy, Y_perm, row_of, topk_w, dO_perm, dw, stream=None):
    """Backward of the combine (moe_combine_backward): dO_perm rows and dw."""
    _check(lib().moe_combine_backward(ctypes.byref(shape), _ptr(dy), _ptr(Y_perm), _ptr(row_of), _ptr(topk_w),
                                      _ptr(dO_perm), _ptr(dw), _stream(stream)), "moe_combine_backward")


def router_backward(shape, logits, topk_idx, topk_w, dw, dlogits, stream=None):
    """Backward of the routing weights (moe_router_backward): dlogits [T, E]."""
    _check(lib().moe_router_backward(ctypes.byref(shape), _ptr(logits), _ptr(topk_idx), _ptr(topk_w), _ptr(dw),
                                     _ptr(dlogits), _stream(stream)), "moe_router_backward")


def forward(shape, x, Wg, bias, W1, W3, W2, s1, s3, s2, W1s, W3s, W2s, y, ws, topk_idx=None, topk_w=None,
            counts=None, stream=None):
    _check(lib().moe_forward(ctypes.byref(shape), _ptr(x), _ptr(Wg), _ptr(bias), _ptr(W1), _ptr(W3), _ptr(W2),
                             _ptr(s1), _ptr(s3), _ptr(s2), _ptr(W1s), _ptr(W3s), _ptr(W2s), _ptr(y), _ptr(topk_idx),
                             _ptr(topk_w), _ptr(counts), _ptr(ws), ws.numel() if ws is not None else 0,
                             _stream(stream)), "moe_forward")


def forward_launches(shape) -> int:
    """Kernel launches one moe_forward call issues for this shape on the current device."""
    n = int(lib().moe_forward_launches(ctypes.byref(shape)))
    if n < 0:
        raise MoeError(MOE_ERR_UNSUPPORTED, "moe_forward_launches")
    return n


def forward_ep(shape, ep_rank, ep_size, x, Wg, bias, W1, W3, W2, s1, s3, s2, W1s, W3s, W2s, y, ws, topk_idx=None,
               topk_w=None, counts=None, stream=None):
    """This rank's share of the expert-parallel layer (moe_forward_ep): W1/W3/W2
    (and scales) hold the rank's E/ep_size experts, W1s/W3s/W2s its slice of
    the shared expert's hidden features; y receives the partial sum that
    all_reduce_partial (or any sum over ranks) completes."""
    _check(lib().moe_forward_ep(ctypes.byref(shape), int(ep_rank), int(ep_size), _ptr(x), _ptr(Wg), _ptr(bias),
                                _ptr(W1), _ptr(W3), _ptr(W2), _ptr(s1), _ptr(s3), _ptr(s2), _ptr(W1s), _ptr(W3s),
                                _ptr(W2s), _ptr(y), _ptr(topk_idx), _ptr(topk_w), _ptr(counts), _ptr(ws),
                                ws.numel() if ws is not None else 0, _stream(stream)), "moe_forward_ep")


def forward_profiled(shape, x, Wg, bias, W1, W3, W2, s1, s3, s2, W1s, W3s, W2s, y, ws, events, topk_idx=None,
                     topk_w=None, counts=None, stream=None):
    """forward() that also records `events` (NUM_STAGE_EVENTS torch.cuda.Event
    objects with timing enabled) at the stage boundaries."""
    if len(events) != NUM_STAGE_EVENTS:
        raise ValueError(f"need {NUM_STAGE_EVENTS} events")
    for ev in events:
        if not ev.cuda_event:  # torch creates the CUDA event on its first record
            ev.record()
    handles = (ctypes.c_void_p * NUM_STAGE_EVENTS)(*[ev.cuda_event for ev in events])
    _check(lib().moe_forward_profiled(ctypes.byref(shape), _ptr(x), _ptr(Wg), _ptr(bias), _ptr(W1), _ptr(W3),
                                      _ptr(W2), _ptr(s1), _ptr(s3), _ptr(s2), _ptr(W1s), _ptr(W3s), _ptr(W2s),
                                      _ptr(y), _ptr(topk_idx), _ptr(topk_w), _ptr(counts), _ptr(ws),
                                      ws.numel() if ws is not None else 0, _stream(stream), handles),
           "moe_forward_profiled")


def shared_expert(shape, x, W1s, W3s, W2s, Y_shared, ws, stream=None):
    """The shared expert alone (moe_shared_expert): Y_shared [T, d] fp32."""
    _check(lib().moe_shared_expert(ctypes.byref(shape), _ptr(x), _ptr(W1s), _ptr(W3s), _ptr(W2s), _ptr(Y_shared),
                                   _ptr(ws), ws.numel() if ws is not None else 0, _stream(stream)), "moe_shared_expert")


def ep_regroup_layout(n_src, E_local, recv_counts, offsets_local, to_expert_major, to_source_major, stream=None):
    """Expert-major order of rows received from n_src ranks (moe_ep_regroup_layout)."""
    _check(lib().moe_ep_regroup_layout(int(n_src), int(E_local), _ptr(recv_counts), _ptr(offsets_local),
                                       _ptr(to_expert_major), _ptr(to_source_major), _stream(stream)),
           "moe_ep_regroup_layout")


def gather_rows(src, index, dst, stream=None):
    """dst[r] = src[index[r]] for every row of dst (moe_gather_rows, bf16 rows)."""
    rows = int(dst.shape[0])
    if rows == 0:
        return
    _check(lib().moe_gather_rows(_ptr(src), _ptr(index), rows, int(dst.shape[1]), _ptr(dst), _stream(stream)),
           "moe_gather_rows")


def backward_workspace_size(shape: MoeShape) -> int:
    return int(lib().moe_backward_workspace_size(ctypes.byref(shape)))


def alloc_backward_workspace(shape: MoeShape, device="cuda") -> torch.Tensor:
    n = backward_workspace_size(shape)
    if n == 0:
        raise MoeError(MOE_ERR_UNSUPPORTED, "moe_backward_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def backward(shape, x, Wg, bias, W1, W3, W2, W1s, W3s, W2s, dy, dx, dWg, dW1, dW3, dW2, dW1s, dW3s, dW2s, ws,
             stream=None):
    """Gradient of sum(dy * y) of the layer (moe_backward): dx, dWg, dW1, dW3,
    dW2 and the shared expert's dW1s, dW3s, dW2s, in shape.y_dtype."""
    _check(lib().moe_backward(ctypes.byref(shape), _ptr(x), _ptr(Wg), _ptr(bias), _ptr(W1), _ptr(W3), _ptr(W2),
                              _ptr(W1s), _ptr(W3s), _ptr(W2s), _ptr(dy), _ptr(dx), _ptr(dWg), _ptr(dW1), _ptr(dW3),
                              _ptr(dW2), _ptr(dW1s), _ptr(dW3s), _ptr(dW2s), _ptr(ws),
                              ws.numel() if ws is not None else 0, _stream(stream)), "moe_backward")


def forward_train(shape, x, Wg, bias, W1, W3, W2, W1s, W3s, W2s, y, ws, stream=None):
    """moe_forward_train: the layer's y, keeping the forward's state in the
    backward workspace `ws` for backward_saved."""
    _check(lib().moe_forward_train(ctypes.byref(shape), _ptr(x), _ptr(Wg), _ptr(bias), _ptr(W1), _ptr(W3), _ptr(W2),
                                   _ptr(W1s), _ptr(W3s), _ptr(W2s), _ptr(y), _ptr(ws),
                                   ws.numel() if ws is not None else 0, _stream(stream)), "moe_forward_train")


def backward_saved(shape, x, Wg, W1, W3, W2, W1s, W3s, W2s, dy, dx, dWg, dW1, dW3, dW2, dW1s, dW3s, dW2s, ws,
                   stream=None):
    """moe_backward_saved: every gradient from the state forward_train left in `ws`."""
    _check(lib().moe_backward_saved(ctypes.byref(shape), _ptr(x), _ptr(Wg), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(W1s),
                                    _ptr(W3s), _ptr(W2s), _ptr(dy), _ptr(dx), _ptr(dWg), _ptr(dW1), _ptr(dW3),
                                    _ptr(dW2), _ptr(dW1s), _ptr(dW3s), _ptr(dW2s), _ptr(ws),
                                    ws.numel() if ws is not None else 0, _stream(stream)), "moe_backward_saved")


def check_device_status(ws, stream=None) -> tuple[int, int]:
    raw = ctypes.c_uint32(0)
    rc = lib().moe_check_device_status(_ptr(ws), _stream(stream), ctypes.byref(raw))
    return rc, raw.value


def version() -> str:
    return lib().moe_version().decode()
