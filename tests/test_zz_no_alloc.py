"""The allocation-free dispatch entry point, moe_permute_noalloc.

Callers that cannot allocate device memory (for example a plugin that is
handed only its input and output buffers by the runtime hosting it) call this
variant of moe_permute; its scratch lives in a static array inside the
library.  This test calls it through the C ABI and checks that two calls in a
row each give exactly what moe_permute gives for the same input (the outputs
are integers and row copies, so equal means bit-identical).  It runs last so a
failure here leaves every other test already run, and it passes both alone in
a fresh process and after the rest of the suite."""
import ctypes

import numpy as np
import pytest
import torch

from mixture_experts_ffn_17_b200 import binding as B
from mixture_experts_ffn_17_b200 import build as libbuild

pytestmark = pytest.mark.gpu


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _outputs(T, k, E, d):
    dev = "cuda"
    return (torch.empty(E, dtype=torch.int32, device=dev), torch.empty(E + 1, dtype=torch.int32, device=dev),
            torch.empty(T * k, dtype=torch.int32, device=dev), torch.empty(T * k, dtype=torch.int32, device=dev),
            torch.empty(T * k, d, dtype=torch.bfloat16, device=dev))


def _routing(T, E, k, seed):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    if seed % 2:  # a skewed second input: one expert takes slot 0 of every token
        idx[:, 0] = 3
        for t in range(T):
            while 3 in idx[t, 1:]:
                idx[t, 1:] = rng.permutation(E)[:k - 1]
    return torch.as_tensor(idx, device="cuda")


def test_noalloc_permute_matches_workspace_permute_twice():
    libbuild.build()
    lib = B.lib()
    T, E, k, d = 4096, 256, 8, 512
    shape = B.make_shape(T=T, d=d, E=E, k=k, inter=128, shared_inter=0)
    ws = B.alloc_workspace(shape)
    g = torch.Generator(device="cuda").manual_seed(1)
    x = torch.randn(T, d, generator=g, device="cuda").to(torch.bfloat16)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, seed in enumerate((20, 21)):
        idx = _routing(T, E, k, seed)
        ref = _outputs(T, k, E, d)
        B.permute(shape, idx, *ref[:4], x, ref[4], ws)
        got = _outputs(T, k, E, d)
        for t in got:
            t.fill_(-7) if t.dtype == torch.int32 else t.zero_()
        rc = lib.moe_permute_noalloc(ctypes.byref(shape), _ptr(idx), *[_ptr(t) for t in got[:4]], _ptr(x),
                                     _ptr(got[4]), stream)
        assert rc == B.MOE_OK, B.status_string(rc)
        torch.cuda.synchronize()
        for name, a, b in zip(("counts", "offsets", "perm_token", "row_of", "x_perm"), ref, got):
            assert torch.equal(a, b), f"call {call}: {name} differs"


def test_noalloc_permute_rejects_shapes_beyond_its_scratch():
    lib = B.lib()
    shape = B.make_shape(T=65536, d=512, E=256, k=8, inter=128, shared_inter=0)
    dummy = torch.empty(16, dtype=torch.int32, device="cuda")
    p = _ptr(dummy)
    rc = lib.moe_permute_noalloc(ctypes.byref(shape), p, p, p, p, p, None, None, None)
    assert rc == B.MOE_ERR_UNSUPPORTED
