"""The allocation-free dispatch entry point, moe_permute_noalloc.

Callers that cannot allocate device memory (for example a plugin that is
handed only its input and output buffers by the runtime hosting it) call this
variant of moe_permute; its scratch lives in a static array inside the
library.  This test calls it through the C ABI and checks that two calls in a
row each give exactly what moe_permute gives for the same input (the outputs
are integers and row copies, so equal means bit-identical); also an empty
batch, out-of-range expert indices (skipped by both), and the largest shape
the array accepts, where the histograms and bases fill it exactly.  It runs
last so a failure here leaves every other test already run, and it passes
both alone in a fresh process and after the rest of the suite."""
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


def _compare(T, E, k, d, idx, n_rows=None):
    """moe_permute_noalloc vs moe_permute on the same input; the first n_rows
    permuted rows (all written rows) of perm_token and x_perm are compared."""
    lib = B.lib()
    shape = B.make_shape(T=T, d=d, E=E, k=k, inter=128, shared_inter=0)
    ws = B.alloc_workspace(shape)
    g = torch.Generator(device="cuda").manual_seed(2)
    x = torch.randn(max(T, 1), d, generator=g, device="cuda").to(torch.bfloat16)[:T]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ref = _outputs(T, k, E, d)
    B.permute(shape, idx, *ref[:4], x, ref[4], ws)
    got = _outputs(T, k, E, d)
    for t in got:
        t.fill_(-7) if t.dtype == torch.int32 else t.zero_()
    rc = lib.moe_permute_noalloc(ctypes.byref(shape), _ptr(idx), *[_ptr(t) for t in got[:4]], _ptr(x), _ptr(got[4]),
                                 stream)
    assert rc == B.MOE_OK, B.status_string(rc)
    torch.cuda.synchronize()
    n = T * k if n_rows is None else n_rows
    assert torch.equal(ref[0], got[0]) and torch.equal(ref[1], got[1]) and torch.equal(ref[3], got[3])
    assert torch.equal(ref[2][:n], got[2][:n]) and torch.equal(ref[4][:n], got[4][:n])
    return ref


def test_noalloc_permute_empty_batch():
    # empty tensors pass NULL pointers: an empty batch writes counts and
    # offsets only
    ref = _compare(0, 64, 4, 256, torch.empty(0, 4, dtype=torch.int32, device="cuda"))
    assert int(ref[1][-1]) == 0 and int(ref[0].sum()) == 0


def test_noalloc_permute_skips_out_of_range_indices_like_the_workspace_call():
    T, E, k = 500, 64, 4
    idx = _routing(T, E, k, 40).clone()
    idx[3, 1] = E + 1
    idx[77, 0] = -2
    idx[499, 3] = 1000
    ref = _compare(T, E, k, 256, idx, n_rows=T * k - 3)
    row_of = ref[3].view(T, k)
    assert int(row_of[3, 1]) == -1 and int(row_of[77, 0]) == -1 and int(row_of[499, 3]) == -1
    assert int(ref[1][-1]) == T * k - 3


def test_noalloc_permute_largest_accepted_shape():
    # ceil(65280 / 256) * 256 = 65280 histogram entries (and as many bases):
    # with the status word they fill the 512 KiB array to its last 64 ints
    _compare(65280, 256, 8, 128, _routing(65280, 256, 8, 42))


def test_noalloc_permute_rejects_shapes_beyond_its_scratch():
    lib = B.lib()
    shape = B.make_shape(T=65536, d=512, E=256, k=8, inter=128, shared_inter=0)
    dummy = torch.empty(16, dtype=torch.int32, device="cuda")
    p = _ptr(dummy)
    rc = lib.moe_permute_noalloc(ctypes.byref(shape), p, p, p, p, p, None, None, None)
    assert rc == B.MOE_ERR_UNSUPPORTED
