"""The C ABI without a GPU: the library loads, exports every symbol the header
declares, the header is plain C with the layout the binding assumes, and the
host-side validation rejects bad calls before touching CUDA."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from mixture_experts_ffn_17_b200 import binding as B
from mixture_experts_ffn_17_b200 import build as libbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    libbuild.build()


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert set(names) == set(B.EXPORTED)
    lib = ctypes.CDLL(B.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (moe_\w+)", out))
    assert set(names) <= exported


def test_header_is_plain_c_and_struct_layout_matches_binding(tmp_path):
    prog = tmp_path / "layout.c"
    prog.write_text(
        '#include <stdio.h>\n#include <stddef.h>\n#include "moe.h"\n'
        "int main(void){printf(\"%zu\", sizeof(moe_shape));\n"
        + "".join(f'printf(" %zu", offsetof(moe_shape, {f}));\n' for f, _ in B.MoeShape._fields_)
        + "return 0;}\n")
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), str(prog), "-o", str(exe)],
                   check=True)
    vals = [int(v) for v in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()]
    assert vals[0] == ctypes.sizeof(B.MoeShape)
    assert vals[1:] == [getattr(B.MoeShape, f).offset for f, _ in B.MoeShape._fields_]


def test_status_strings_and_version():
    for s in range(7):
        assert len(B.status_string(s)) > 0
    assert B.status_string(99) == "unknown status"
    assert "sm_100a" in B.version()


V3 = dict(T=4096, d=7168, E=256, k=8, inter=2048, shared_inter=2048)


def test_workspace_size_valid_shapes():
    s = B.make_shape(**V3)
    n = B.workspace_size(s)
    Tk = 4096 * 8
    # gathered rows + H + Y_perm + shared fp32 rows dominate
    big = Tk * 7168 * 2 + (Tk + 4096) * 2048 * 2 + Tk * 7168 * 2 + 4096 * 7168 * 4
    assert big <= n <= big + 64 * 1024 * 1024
    assert B.workspace_size(B.make_shape(T=0, d=512, E=32, k=4, inter=256, shared_inter=0)) > 0


@pytest.mark.parametrize("bad", [
    dict(T=-1), dict(d=0), dict(k=0), dict(k=300), dict(inter=0), dict(shared_inter=-128),
    dict(d=7000), dict(inter=2000), dict(E=48), dict(E=2048), dict(k=33, E=64),
    dict(route=2), dict(w_dtype=7), dict(y_dtype=1),
    dict(route=1, n_group=3), dict(route=1, n_group=8, topk_group=0),
    dict(route=1, n_group=8, topk_group=9), dict(route=1, n_group=256, topk_group=1, group_topn=1, k=1),
    dict(route=1, n_group=8, topk_group=1, group_topn=2, k=40),
])
def test_workspace_size_rejects_bad_shapes(bad):
    args = dict(V3)
    args.update(bad)
    assert B.workspace_size(B.make_shape(**args)) == 0


def _fake(n=1 << 20, align=256):
    # a host buffer only used as an aligned, non-null address: the calls below
    # must reject the arguments before any launch
    buf = ctypes.create_string_buffer(n + align)
    addr = ctypes.addressof(buf)
    return buf, ctypes.c_void_p(addr + (-addr) % align)


def test_forward_validation_without_gpu():
    L = B.lib()
    s = B.make_shape(T=128, d=512, E=32, k=4, inter=256, shared_inter=256)
    keep, p = _fake()
    n = B.workspace_size(s)
    nul = None
    args = [p, p, nul, p, p, p, nul, nul, nul, p, p, p, p, nul, nul, nul, p, n, nul]
    # missing x
    a = list(args); a[0] = nul
    assert L.moe_forward(ctypes.byref(s), *a) == B.MOE_ERR_INVALID_ARG
    # missing shared weights while shared_inter > 0
    a = list(args); a[9] = nul
    assert L.moe_forward(ctypes.byref(s), *a) == B.MOE_ERR_INVALID_ARG
    # misaligned y
    a = list(args); a[12] = ctypes.c_void_p(p.value + 8)
    assert L.moe_forward(ctypes.byref(s), *a) == B.MOE_ERR_INVALID_ARG
    # workspace too small / misaligned
    a = list(args); a[17] = n - 1
    assert L.moe_forward(ctypes.byref(s), *a) == B.MOE_ERR_WORKSPACE
    a = list(args); a[16] = ctypes.c_void_p(p.value + 16)
    assert L.moe_forward(ctypes.byref(s), *a) == B.MOE_ERR_WORKSPACE
    # E4M3 weights without scales
    s8 = B.make_shape(T=128, d=512, E=32, k=4, inter=256, shared_inter=256, w_dtype=B.MOE_E4M3)
    assert L.moe_forward(ctypes.byref(s8), *args) == B.MOE_ERR_INVALID_ARG
    # bad shape
    sb = B.make_shape(T=128, d=500, E=32, k=4, inter=256, shared_inter=256)
    assert L.moe_forward(ctypes.byref(sb), *args) == B.MOE_ERR_UNSUPPORTED
    assert L.moe_forward(None, *args) == B.MOE_ERR_INVALID_ARG


def test_stage_entry_points_validation_without_gpu():
    L = B.lib()
    s = B.make_shape(T=64, d=256, E=32, k=2, inter=128, shared_inter=0)
    keep, p = _fake()
    n = B.workspace_size(s)
    nul = None
    assert L.moe_router_topk(ctypes.byref(s), nul, p, nul, p, p, nul, p, n, nul) == B.MOE_ERR_INVALID_ARG
    assert L.moe_router_topk(ctypes.byref(s), p, p, nul, p, p, nul, p, 16, nul) == B.MOE_ERR_WORKSPACE
    # x given without x_perm
    assert L.moe_permute(ctypes.byref(s), p, p, p, p, p, p, nul, p, n, nul) == B.MOE_ERR_INVALID_ARG
    assert L.moe_grouped_swiglu(ctypes.byref(s), p, p, p, p, p, nul, nul, nul, nul, nul, nul, nul, p, nul, p, n,
                                nul) == B.MOE_ERR_INVALID_ARG
    assert L.moe_combine(ctypes.byref(s), p, nul, nul, p, p, nul) == B.MOE_ERR_INVALID_ARG
    assert L.moe_check_device_status(nul, nul, None) == B.MOE_ERR_INVALID_ARG
    # backward steps: a null or misaligned pointer is refused before any launch
    odd = ctypes.c_void_p(p.value + 4)
    assert L.moe_combine_backward(ctypes.byref(s), p, p, nul, p, p, p, nul) == B.MOE_ERR_INVALID_ARG
    assert L.moe_combine_backward(ctypes.byref(s), odd, p, p, p, p, p, nul) == B.MOE_ERR_INVALID_ARG
    assert L.moe_router_backward(ctypes.byref(s), p, p, p, nul, p, nul) == B.MOE_ERR_INVALID_ARG
    assert L.moe_router_backward(ctypes.byref(s), p, p, p, p, odd, nul) == B.MOE_ERR_INVALID_ARG


def test_empty_batch_is_a_no_op_without_gpu():
    # T = 0 passes validation and returns before any CUDA call
    L = B.lib()
    s = B.make_shape(T=0, d=256, E=32, k=2, inter=128, shared_inter=128)
    keep, p = _fake()
    n = B.workspace_size(s)
    assert L.moe_forward(ctypes.byref(s), p, p, None, p, p, p, None, None, None, p, p, p, p, None, None, None, p, n,
                         None) == B.MOE_OK
    assert L.moe_combine(ctypes.byref(s), p, p, p, p, p, None) == B.MOE_OK
    assert L.moe_combine_backward(ctypes.byref(s), p, p, p, p, p, p, None) == B.MOE_OK
    assert L.moe_router_backward(ctypes.byref(s), p, p, p, p, p, None) == B.MOE_OK


def test_binding_refuses_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(B, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(B, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        B.lib()


def test_forward_ep_validation_without_gpu():
    L = B.lib()
    s = B.make_shape(T=128, d=512, E=32, k=4, inter=256, shared_inter=256)
    keep, p = _fake()
    n = B.workspace_size(s)
    nul = None
    args = [p, p, nul, p, p, p, nul, nul, nul, p, p, p, p, nul, nul, nul, p, n, nul]
    assert L.moe_forward_ep(ctypes.byref(s), 0, 0, *args) == B.MOE_ERR_INVALID_ARG     # no ranks
    assert L.moe_forward_ep(ctypes.byref(s), 2, 2, *args) == B.MOE_ERR_INVALID_ARG     # rank out of range
    assert L.moe_forward_ep(ctypes.byref(s), -1, 2, *args) == B.MOE_ERR_INVALID_ARG
    assert L.moe_forward_ep(ctypes.byref(s), 0, 3, *args) == B.MOE_ERR_UNSUPPORTED     # 32 experts over 3 ranks
    assert L.moe_forward_ep(ctypes.byref(s), 0, 4, *args) == B.MOE_ERR_UNSUPPORTED     # shared slice of 64 features
    s0 = B.make_shape(T=0, d=512, E=32, k=4, inter=256, shared_inter=256)
    assert L.moe_forward_ep(ctypes.byref(s0), 1, 2, *args) == B.MOE_OK                 # empty batch


def test_forward_launch_count():
    # ten kernels; one more when the gate GEMM splits K (small batches), two
    # more with FP8 experts (the shared expert's bf16 launches) or with long
    # segments (the full 256-row tiles' CTA-pair launches)
    from mixture_experts_ffn_17_b200 import workloads
    counts = {n: B.forward_launches(B.shape_of(workloads.CONFIGS[n])) for n in ("decode", "prefill", "skewed", "fp8")}
    assert counts == {"decode": 11, "prefill": 10, "skewed": 12, "fp8": 12}  # skewed: + the CTA-pair launches
    assert B.forward_launches(B.make_shape(T=0, d=512, E=32, k=4, inter=256, shared_inter=256)) == 0
    with pytest.raises(B.MoeError):
        B.forward_launches(B.make_shape(T=16, d=500, E=32, k=4, inter=256, shared_inter=256))


def test_forward_launch_count_with_cta_pairs_forced(monkeypatch):
    # pairs add a launch per grouped GEMM (pair + one-CTA), and with FP8
    # experts the bf16 shared expert gets its own pair launch too
    from mixture_experts_ffn_17_b200 import workloads
    monkeypatch.setenv("MOE_PAIR_TILES", "1")
    assert B.forward_launches(B.shape_of(workloads.CONFIGS["prefill"])) == 12
    assert B.forward_launches(B.shape_of(workloads.CONFIGS["fp8"])) == 16
    monkeypatch.setenv("MOE_PAIR_TILES", "0")
    assert B.forward_launches(B.shape_of(workloads.CONFIGS["skewed"])) == 10


def test_backward_validation_without_gpu():
    L = B.lib()
    s = B.make_shape(T=128, d=512, E=32, k=4, inter=256, shared_inter=256)
    n = B.backward_workspace_size(s)
    assert n > B.workspace_size(s)           # the forward's buffers and the backward's after them
    keep, p = _fake()
    nul = None
    # x Wg bias W1 W3 W2 W1s W3s W2s dy | dx dWg dW1 dW3 dW2 dW1s dW3s dW2s | ws n stream
    args = [p, p, nul, p, p, p, p, p, p, p, p, p, p, p, p, p, p, p, p, n, nul]
    for i in (0, 1, 3, 9, 10, 11, 12, 13, 14, 15):
        a = list(args); a[i] = nul
        assert L.moe_backward(ctypes.byref(s), *a) == B.MOE_ERR_INVALID_ARG, i
    a = list(args); a[19] = n - 1
    assert L.moe_backward(ctypes.byref(s), *a) == B.MOE_ERR_WORKSPACE
    a = list(args); a[10] = ctypes.c_void_p(p.value + 4)
    assert L.moe_backward(ctypes.byref(s), *a) == B.MOE_ERR_INVALID_ARG
    # the backward pass takes bf16 experts only
    s8 = B.make_shape(T=128, d=512, E=32, k=4, inter=256, shared_inter=256, w_dtype=B.MOE_E4M3)
    assert B.backward_workspace_size(s8) == 0
    assert L.moe_backward(ctypes.byref(s8), *args) == B.MOE_ERR_UNSUPPORTED
    # without a shared expert its weights and gradients may be NULL
    s0 = B.make_shape(T=128, d=512, E=32, k=4, inter=256, shared_inter=0)
    assert B.backward_workspace_size(s0) > 0


def test_training_calls_validation_without_gpu():
    L = B.lib()
    s = B.make_shape(T=128, d=512, E=32, k=4, inter=256, shared_inter=256)
    n = B.backward_workspace_size(s)
    keep, p = _fake()
    nul = None
    # moe_forward_train: x Wg bias W1 W3 W2 W1s W3s W2s y | ws n stream
    fa = [p, p, nul, p, p, p, p, p, p, p, p, n, nul]
    for i in (0, 1, 3, 6, 9):
        a = list(fa); a[i] = nul
        assert L.moe_forward_train(ctypes.byref(s), *a) == B.MOE_ERR_INVALID_ARG, i
    a = list(fa); a[11] = B.workspace_size(s)          # the forward's workspace is too small
    assert L.moe_forward_train(ctypes.byref(s), *a) == B.MOE_ERR_WORKSPACE
    # moe_backward_saved: x Wg W1 W3 W2 W1s W3s W2s dy | dx dWg dW1 dW3 dW2 dW1s dW3s dW2s | ws n stream
    ba = [p] * 17 + [p, n, nul]
    for i in (0, 8, 9, 13, 16):
        a = list(ba); a[i] = nul
        assert L.moe_backward_saved(ctypes.byref(s), *a) == B.MOE_ERR_INVALID_ARG, i
    s8 = B.make_shape(T=128, d=512, E=32, k=4, inter=256, shared_inter=256, w_dtype=B.MOE_E4M3)
    assert L.moe_forward_train(ctypes.byref(s8), *fa) == B.MOE_ERR_UNSUPPORTED
    assert L.moe_backward_saved(ctypes.byref(s8), *ba) == B.MOE_ERR_UNSUPPORTED
