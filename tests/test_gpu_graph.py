"""moe_forward inside a CUDA graph: the call makes no host synchronisation and
allocates nothing, so it can be captured once and replayed on new inputs
written into the captured buffers.  Replays must equal eager calls bit for bit
(the path is deterministic) and stay correct across shapes that take the
router's K split, the CTA-pair tiles and the FP8 converters."""
import pytest
import torch

from mixture_experts_ffn_17_b200 import binding as B
from mixture_experts_ffn_17_b200 import build as libbuild
from mixture_experts_ffn_17_b200 import workloads

from gpu_util import to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    libbuild.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


CASES = {
    # several row tiles per expert, ragged tails, K-split router
    "bf16": dict(name="prefill", T=1000, d=1024, E=64, k=6, inter=512, shared_inter=384),
    # long segments: the CTA-pair kernels run (about 512 rows per expert)
    "bf16_pairs": dict(name="skewed", T=2048, d=512, E=32, k=8, inter=256, shared_inter=256),
    # e4m3 experts with group routing
    "fp8": dict(name="fp8", T=512, d=1024, E=32, k=8, inter=512, shared_inter=256),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_forward_replays_in_a_cuda_graph(case):
    kw = dict(CASES[case])
    name = kw.pop("name")
    w = to_device(workloads.make_small(name, **kw))
    cfg = w.cfg
    shape = B.shape_of(cfg, B.MOE_F32)
    ws = B.alloc_workspace(shape)
    dev = "cuda"
    y = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device=dev)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=dev)
    tw = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=dev)
    counts = torch.empty(cfg.E, dtype=torch.int32, device=dev)
    x_static = w.x.clone()

    def call(x, out):
        B.forward(shape, x, w.Wg, w.bias, w.W1, w.W3, w.W2, w.s1, w.s3, w.s2, w.W1s, w.W3s, w.W2s, out, ws, idx, tw,
                  counts)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        call(x_static, y)  # eager warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call(x_static, y)

    gen = torch.Generator(device="cpu").manual_seed(4242)
    for rep in range(3):
        # new tokens in the captured input buffer (scaled and shuffled rows of
        # the workload's own x, so routing and magnitudes stay typical)
        perm = torch.randperm(cfg.T, generator=gen).to(dev)
        scale = (0.5 + torch.rand(cfg.T, 1, generator=gen)).to(dev)
        x_new = (w.x[perm].float() * scale).to(w.x.dtype)
        x_static.copy_(x_new)
        g.replay()
        torch.cuda.synchronize()
        y_graph, idx_graph, tw_graph, counts_graph = y.clone(), idx.clone(), tw.clone(), counts.clone()

        y_eager = torch.empty_like(y)
        call(x_new, y_eager)
        torch.cuda.synchronize()
        rc, raw = B.check_device_status(ws)
        assert rc == B.MOE_OK, (rc, raw)
        assert torch.equal(idx_graph, idx), rep
        assert torch.equal(tw_graph, tw), rep
        assert torch.equal(counts_graph, counts), rep
        assert int(counts_graph.sum()) == cfg.T * cfg.k
        assert torch.equal(y_graph, y_eager), (rep, (y_graph - y_eager).abs().max().item())
        assert torch.isfinite(y_graph).all()
    del g


def test_backward_replays_in_a_cuda_graph():
    # moe_backward makes no host synchronisation either: a captured call
    # replayed on new output gradients equals eager calls bit for bit
    w = to_device(workloads.make_small("prefill", T=600, d=1024, E=64, k=6, inter=512, shared_inter=384))
    cfg = w.cfg
    shape = B.shape_of(cfg, B.MOE_BF16)
    ws = B.alloc_backward_workspace(shape)
    e = lambda *sz: torch.empty(sz, dtype=torch.bfloat16, device="cuda")
    grads = [e(cfg.T, cfg.d), e(cfg.E, cfg.d), e(cfg.E, cfg.d, cfg.inter), e(cfg.E, cfg.d, cfg.inter),
             e(cfg.E, cfg.inter, cfg.d), e(cfg.d, cfg.shared_inter), e(cfg.d, cfg.shared_inter),
             e(cfg.shared_inter, cfg.d)]
    dy_static = torch.zeros(cfg.T, cfg.d, dtype=torch.float32, device="cuda")

    def call(dy, out):
        B.backward(shape, w.x, w.Wg, w.bias, w.W1, w.W3, w.W2, w.W1s, w.W3s, w.W2s, dy, *out, ws)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        call(dy_static, grads)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call(dy_static, grads)
    gen = torch.Generator(device="cuda").manual_seed(77)
    for rep in range(2):
        dy = torch.randn(cfg.T, cfg.d, generator=gen, device="cuda")
        dy_static.copy_(dy)
        g.replay()
        torch.cuda.synchronize()
        got = [t.clone() for t in grads]
        eager = [torch.empty_like(t) for t in grads]
        call(dy, eager)
        torch.cuda.synchronize()
        rc, raw = B.check_device_status(ws)
        assert rc == B.MOE_OK, (rc, raw)
        for a, b in zip(got, eager):
            assert torch.equal(a, b), rep
        assert all(torch.isfinite(t.float()).all() for t in got)
    del g
