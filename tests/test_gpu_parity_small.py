"""CUDA path vs the fp64 oracle at sizes the oracle finishes in seconds: every
entry point of the C ABI, several tiles and ragged tails, and the degenerate
cases of the layer (empty experts, one oversize expert, T=1, k=1, k=E, no
shared expert, zero weights)."""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_ffn_17_b200 import binding as B
from mixture_experts_ffn_17_b200 import build as libbuild
from mixture_experts_ffn_17_b200 import workloads

from gpu_util import expert_weights_f64, oracle_full, route_with_exemptions, run_forward, to_device
from parity import TOL_BF16, TOL_FP8, bf16_stored_ok, dec, max_rel_err, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    libbuild.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _tiny():
    return to_device(workloads.make("tiny"))


def _medium(**kw):
    # several tiles per expert, ragged tails, inter != shared_inter
    shape = dict(T=1000, d=1024, E=64, k=6, inter=512, shared_inter=384)
    shape.update(kw)
    return to_device(workloads.make_small("prefill", **shape))


def _wide():
    # 32 token tiles x 4 expert blocks: enough CTAs that the gate GEMM runs
    # without a K split (tiny and medium split K into 8 and 16 parts)
    return to_device(workloads.make_small("prefill", T=4096, d=512, E=256, k=8, inter=128, shared_inter=0))


# --------------------------------------------------------------- router
@pytest.mark.parametrize("make", [_tiny, _medium, _wide])
def test_router_matches_oracle(make):
    w = make()
    cfg = w.cfg
    shape = B.shape_of(cfg)
    ws = B.alloc_workspace(shape)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device="cuda")
    tw = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device="cuda")
    lg_dev = torch.empty(cfg.T, cfg.E, dtype=torch.float32, device="cuda")
    B.router_topk(shape, w.x, w.Wg, w.bias, idx, tw, lg_dev, ws)
    torch.cuda.synchronize()
    lg = oracle.logits(dec(w.x), dec(w.Wg))
    err = np.abs(to_np(lg_dev).astype(np.float64) - lg)
    assert err.max() <= 1e-6 * (1 + np.abs(lg).max()), err.max()
    idx_o, w_o, merged, report, n_near = route_with_exemptions(w, lg, to_np(idx))
    assert len(report) <= n_near, report      # exemptions only where the oracle itself has a near-tie
    ok = np.all(to_np(idx) == merged, axis=1)
    assert np.allclose(to_np(tw)[ok], w_o[ok], rtol=0, atol=2e-6)


def test_router_group_mode_matches_oracle():
    w = to_device(workloads.make_small("fp8", T=700, d=512, E=64, k=6, inter=256, shared_inter=256, n_group=8,
                                       topk_group=3, fp8=False))
    cfg = w.cfg
    shape = B.shape_of(cfg)
    ws = B.alloc_workspace(shape)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device="cuda")
    tw = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device="cuda")
    B.router_topk(shape, w.x, w.Wg, w.bias, idx, tw, None, ws)
    torch.cuda.synchronize()
    lg = oracle.logits(dec(w.x), dec(w.Wg))
    idx_o, w_o, merged, report, n_near = route_with_exemptions(w, lg, to_np(idx))
    assert len(report) <= n_near, report
    ok = np.all(to_np(idx) == merged, axis=1)
    assert np.allclose(to_np(tw)[ok], w_o[ok], rtol=0, atol=1e-5)
    assert np.allclose(to_np(tw).sum(1), 2.5, atol=1e-5)


# --------------------------------------------------------------- permute
def _permute_case(idx_np, E, d=256, x=None):
    T, k = idx_np.shape
    shape = B.make_shape(T=T, d=d, E=E, k=k, inter=128, shared_inter=0)
    ws = B.alloc_workspace(shape)
    dev = lambda a: torch.as_tensor(a, device="cuda")
    idx = dev(np.ascontiguousarray(idx_np, dtype=np.int32))
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    row_of = torch.empty(T * k, dtype=torch.int32, device="cuda")
    if x is None:
        g = torch.Generator(device="cuda").manual_seed(5)
        x = torch.randn(T, d, generator=g, device="cuda").to(torch.bfloat16)
    x_perm = torch.empty(T * k, d, dtype=torch.bfloat16, device="cuda")
    B.permute(shape, idx, counts, offsets, perm, row_of, x, x_perm, ws)
    rc, raw = B.check_device_status(ws)
    c, o, p, r = oracle.dispatch(idx_np, E)
    assert np.array_equal(to_np(counts), c)
    assert np.array_equal(to_np(offsets), o)
    assert np.array_equal(to_np(perm), p)
    assert np.array_equal(to_np(row_of), r)
    assert torch.equal(x_perm, x[torch.as_tensor(p, device="cuda").long()])
    assert rc == B.MOE_OK, raw


@pytest.mark.parametrize("T,E,k", [(1, 32, 1), (255, 32, 4), (257, 64, 8), (1000, 256, 8), (16384, 256, 8)])
def test_permute_random_routing(T, E, k):
    rng = np.random.default_rng(T + E + k)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    _permute_case(idx, E)


def test_permute_one_expert_takes_everything():
    T, E, k = 700, 64, 2
    idx = np.zeros((T, k), dtype=np.int32)
    idx[:, 0] = 13
    idx[:, 1] = 40 + (np.arange(T) % 3)      # three busy experts, 60 empty ones
    _permute_case(idx, E)


def test_permute_duplicate_slots():
    # caller-supplied indices may repeat an expert within a token; each entry
    # still gets its own row, in (token, slot) order
    rng = np.random.default_rng(9)
    idx = rng.integers(0, 32, size=(300, 4)).astype(np.int32)
    idx[:, 1] = idx[:, 0]
    _permute_case(idx, 32)


def test_permute_reports_out_of_range_index():
    T, E, k = 64, 32, 2
    shape = B.make_shape(T=T, d=256, E=E, k=k, inter=128, shared_inter=0)
    ws = B.alloc_workspace(shape)
    idx = torch.randint(0, E, (T, k), dtype=torch.int32, device="cuda")
    idx[5, 1] = E + 3
    idx[9, 0] = -1
    out = [torch.empty(n, dtype=torch.int32, device="cuda") for n in (E, E + 1, T * k, T * k)]
    B.permute(shape, idx, *out, None, None, ws)
    rc, raw = B.check_device_status(ws)
    assert rc == B.MOE_ERR_DEVICE_BOUNDS and raw & 2
    row_of = to_np(out[3]).reshape(T, k)
    assert row_of[5, 1] == -1 and row_of[9, 0] == -1
    assert to_np(out[0]).sum() == T * k - 2


def test_permute_out_of_range_index_gathers_only_the_written_rows():
    # the skipped entries take no permuted position: the row gather copies the
    # offsets[E] = T*k - 2 rows the scatter wrote and leaves the tail alone
    T, E, k, d = 300, 64, 4, 256
    shape = B.make_shape(T=T, d=d, E=E, k=k, inter=128, shared_inter=0)
    ws = B.alloc_workspace(shape)
    rng = np.random.default_rng(31)
    idx_np = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    idx_np[17, 2] = E
    idx_np[250, 0] = -5
    idx = torch.as_tensor(idx_np, device="cuda")
    counts, offsets = (torch.empty(n, dtype=torch.int32, device="cuda") for n in (E, E + 1))
    perm = torch.zeros(T * k, dtype=torch.int32, device="cuda")
    row_of = torch.empty(T * k, dtype=torch.int32, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(6)
    x = torch.randn(T, d, generator=g, device="cuda").to(torch.bfloat16)
    x_perm = torch.full((T * k, d), 7.0, dtype=torch.bfloat16, device="cuda")
    B.permute(shape, idx, counts, offsets, perm, row_of, x, x_perm, ws)
    rc, raw = B.check_device_status(ws)
    assert rc == B.MOE_ERR_DEVICE_BOUNDS
    valid = np.where((idx_np >= 0) & (idx_np < E), idx_np, -1)
    n = T * k - 2
    assert int(to_np(offsets)[E]) == n and int(to_np(counts).sum()) == n
    assert np.array_equal(to_np(counts), np.bincount(valid[valid >= 0], minlength=E))
    # expert-major, then (token, slot) order over the valid entries
    tok, slot = np.nonzero(valid >= 0)
    order = np.lexsort((slot, tok, valid[tok, slot]))
    pv = to_np(perm)[:n]
    assert np.array_equal(pv, tok[order])
    assert torch.equal(x_perm[:n], x[torch.as_tensor(pv, device="cuda").long()])
    assert bool((x_perm[n:] == 7.0).all())


# --------------------------------------------------------------- experts
def _experts_case(w, idx_np):
    cfg = w.cfg
    T, k = idx_np.shape
    shape = B.shape_of(cfg)
    ws = B.alloc_workspace(shape)
    c, o, p, r = oracle.dispatch(idx_np, cfg.E)
    x_perm = w.x[torch.as_tensor(p, device="cuda").long()].contiguous()
    offsets = torch.as_tensor(o, device="cuda")
    Y_perm = torch.empty(T * k, cfg.d, dtype=torch.bfloat16, device="cuda")
    Y_sh = torch.empty(T, cfg.d, dtype=torch.float32, device="cuda") if cfg.shared_inter else None
    B.grouped_swiglu(shape, w.x, x_perm, offsets, w.W1, w.W3, w.W2, w.s1, w.s3, w.s2, w.W1s, w.W3s, w.W2s, Y_perm,
                     Y_sh, ws)
    rc, raw = B.check_device_status(ws)
    assert rc == B.MOE_OK, raw
    x = dec(w.x)
    ref = np.zeros((T * k, cfg.d))
    for e in range(cfg.E):
        if c[e]:
            W1, W3, W2 = expert_weights_f64(w, e)
            ref[o[e]:o[e + 1]] = oracle.swiglu_rows(x[p[o[e]:o[e + 1]]], W1, W3, W2)
    assert bf16_stored_ok(dec(Y_perm), ref, tol=(3e-2 if cfg.fp8 else 1e-2)), max_rel_err(dec(Y_perm), ref)
    if cfg.shared_inter:
        ref_s = oracle.swiglu_rows(x, dec(w.W1s), dec(w.W3s), dec(w.W2s))
        assert max_rel_err(to_np(Y_sh).astype(np.float64), ref_s) <= TOL_BF16


def test_grouped_swiglu_tiny_routing():
    w = _tiny()
    lg = oracle.logits(dec(w.x), dec(w.Wg))
    idx, _, _ = oracle.route_topk_softmax(lg, w.cfg.k)
    _experts_case(w, idx)


def test_grouped_swiglu_oversize_and_empty_segments():
    w = _medium(T=600, k=2)
    idx = np.zeros((600, 2), dtype=np.int32)
    idx[:, 0] = 7                                  # 600 rows: 5 tiles, ragged last
    idx[:, 1] = 20 + (np.arange(600) % 2)          # two 300-row segments
    _experts_case(w, idx)


# segment sizes around the tile-half boundaries: <= 64 rows runs as an M=64
# MMA, 65-128 as one M=128 half, 129-192 as a full half plus an M=64 half,
# 193-256 as two full halves, more as several tiles; 0 = empty expert
HALF_BOUNDARY_COUNTS = [1, 63, 64, 65, 127, 128, 129, 191, 192, 193, 255, 256, 257, 320, 385, 0, 2]


def _boundary_idx(E):
    counts = HALF_BOUNDARY_COUNTS + [0] * (E - len(HALF_BOUNDARY_COUNTS))
    idx = np.repeat(np.arange(E, dtype=np.int32), counts)
    np.random.default_rng(5).shuffle(idx)  # tokens of one expert are not contiguous
    return idx[:, None]


@pytest.mark.parametrize("fp8", [False, True])
def test_grouped_swiglu_tile_half_boundaries(fp8):
    T = sum(HALF_BOUNDARY_COUNTS)
    if fp8:
        w = to_device(workloads.make_small("fp8", T=T, d=256, E=32, k=1, inter=128, shared_inter=128, n_group=4,
                                           topk_group=2))
    else:
        w = to_device(workloads.make_small("prefill", T=T, d=256, E=32, k=1, inter=128, shared_inter=128))
    _experts_case(w, _boundary_idx(32))


def test_grouped_swiglu_cta_pairs_on_full_tiles(monkeypatch):
    # full 256-row tiles on 2-CTA clusters (tcgen05.mma.cta_group::2), the
    # partial tiles on the one-CTA kernel, shared expert included
    monkeypatch.setenv("MOE_PAIR_TILES", "1")
    w = to_device(workloads.make_small("prefill", T=sum(HALF_BOUNDARY_COUNTS), d=256, E=32, k=1, inter=128,
                                       shared_inter=128))
    _experts_case(w, _boundary_idx(32))


def test_forward_cta_pairs_match_one_cta_path(monkeypatch):
    w = _medium(T=1536, E=32, k=8, shared_inter=512)  # ~384 rows per expert, 6 full shared tiles
    monkeypatch.setenv("MOE_PAIR_TILES", "0")
    y1, *_ = run_forward(w)
    monkeypatch.setenv("MOE_PAIR_TILES", "1")
    y2, err = _check_forward(w)
    rms = float(y1.double().pow(2).mean().sqrt())
    assert float((y1 - y2).abs().max()) <= 1e-5 * rms


def test_grouped_swiglu_fp8_cta_pairs(monkeypatch):
    # FP8 experts on CTA pairs: each CTA converts its half of the weight
    # columns; the shared expert (bf16) runs on the bf16 pair kernel
    monkeypatch.setenv("MOE_PAIR_TILES", "1")
    w = to_device(workloads.make_small("fp8", T=sum(HALF_BOUNDARY_COUNTS), d=256, E=32, k=1, inter=128,
                                       shared_inter=128, n_group=4, topk_group=2))
    _experts_case(w, _boundary_idx(32))


def test_forward_fp8_cta_pairs(monkeypatch):
    monkeypatch.setenv("MOE_PAIR_TILES", "1")
    _check_forward(_fp8(T=2048, k=8, E=64), tol=TOL_FP8)


def test_grouped_swiglu_no_shared_expert():
    w = _medium(T=300, shared_inter=0)
    lg = oracle.logits(dec(w.x), dec(w.Wg))
    idx, _, _ = oracle.route_topk_softmax(lg, w.cfg.k)
    _experts_case(w, idx)


# --------------------------------------------------------------- combine
@pytest.mark.parametrize("shared", [True, False])
def test_combine_matches_oracle(shared):
    T, k, d, E = 333, 5, 768, 32
    rng = np.random.default_rng(11)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    _, _, _, row_of = oracle.dispatch(idx, E)
    g = torch.Generator().manual_seed(3)
    Yp = torch.randn(T * k, d, generator=g).to(torch.bfloat16)
    Ys = torch.randn(T, d, generator=g) if shared else None
    wts = torch.rand(T, k, generator=g)
    shape = B.make_shape(T=T, d=d, E=E, k=k, inter=128, shared_inter=128 if shared else 0)
    y = torch.empty(T, d, dtype=torch.float32, device="cuda")
    cu = lambda t: None if t is None else t.cuda()
    B.combine(shape, cu(Yp), cu(Ys), cu(torch.as_tensor(row_of)), cu(wts), y)
    torch.cuda.synchronize()
    ref = oracle.combine(dec(Yp), None if Ys is None else dec(Ys), row_of.reshape(T, k), dec(wts))
    assert max_rel_err(to_np(y).astype(np.float64), ref) <= 1e-5


# --------------------------------------------------------------- whole layer
def _check_forward(w, tol=TOL_BF16):
    y, idx, tw, counts, ws = run_forward(w)
    y_o, idx_o, w_o, lg = oracle_full(w)
    _, _, merged, report, n_near = route_with_exemptions(w, lg, to_np(idx))
    assert len(report) <= n_near, report
    if report:
        y_o, *_ = oracle_full(w, force_idx=merged)
    c, _, _, _ = oracle.dispatch(merged, w.cfg.E)
    assert np.array_equal(to_np(counts), c)
    err = max_rel_err(to_np(y).astype(np.float64), y_o)
    assert err <= tol, err
    return y, err


def test_forward_tiny():
    _check_forward(_tiny())


def test_forward_medium_ragged():
    _check_forward(_medium())


@pytest.mark.parametrize("kw", [dict(T=1), dict(T=129, k=1), dict(T=64, E=32, k=32), dict(T=200, shared_inter=0)])
def test_forward_edge_shapes(kw):
    shape = dict(T=100, d=512, E=32, k=4, inter=256, shared_inter=256)
    shape.update(kw)
    _check_forward(to_device(workloads.make_small("prefill", **shape)))


def test_forward_zero_down_projection_is_shared_only():
    w = _tiny()
    w.W2.zero_()
    y, _, _, _, _ = run_forward(w)
    ref = oracle.swiglu_rows(dec(w.x), dec(w.W1s), dec(w.W3s), dec(w.W2s))
    assert max_rel_err(to_np(y).astype(np.float64), ref) <= TOL_BF16


def test_forward_zero_input_gives_zero():
    w = _tiny()
    w.x.zero_()
    y, _, _, _, _ = run_forward(w)
    assert torch.count_nonzero(y) == 0


def test_forward_bf16_output_is_rounded_fp32_output():
    w = _tiny()
    y32, *_ = run_forward(w, B.MOE_F32)
    y16, *_ = run_forward(w, B.MOE_BF16)
    assert torch.equal(y16, y32.to(torch.bfloat16))


def test_forward_is_deterministic():
    w = _medium()
    a, ia, *_ = run_forward(w)
    b, ib, *_ = run_forward(w)
    assert torch.equal(a, b) and torch.equal(ia, ib)


# --------------------------------------------------------------- FP8 experts
def _fp8(**kw):
    shape = dict(T=700, d=512, E=64, k=6, inter=256, shared_inter=256, n_group=8, topk_group=3)
    shape.update(kw)
    return to_device(workloads.make_small("fp8", **shape))


def test_grouped_swiglu_fp8_weights():
    w = _fp8()
    lg = oracle.logits(dec(w.x), dec(w.Wg))
    idx, _, _, _ = oracle.route_sigmoid_group(lg, dec(w.bias), w.cfg.k, w.cfg.n_group, w.cfg.topk_group, 2, 2.5)
    _experts_case(w, idx)


def test_grouped_swiglu_fp8_oversize_segments():
    w = _fp8(T=600, k=2, E=32, n_group=4, topk_group=2, d=768, inter=384)
    idx = np.zeros((600, 2), dtype=np.int32)
    idx[:, 0] = 5
    idx[:, 1] = 30 + (np.arange(600) % 2)
    _experts_case(w, idx)


def test_forward_fp8_group_routing():
    _check_forward(_fp8(), tol=TOL_FP8)


def test_forward_fp8_no_shared_expert():
    _check_forward(_fp8(T=300, shared_inter=0), tol=TOL_FP8)


def test_forward_fp8_small_batch():
    # T <= 128: no expert segment can pass one 128-row half, so the FP8
    # kernels run with one-A-half stages and a deeper ring
    _check_forward(_fp8(T=100), tol=TOL_FP8)
    _check_forward(_fp8(T=1, shared_inter=0), tol=TOL_FP8)


def test_grouped_swiglu_fp8_short_segments():
    # T*k <= 128 rows through moe_grouped_swiglu (one-half stages): segments
    # of 65 (past the 64-row narrow half), 1, 16, 17, 0 and 21 rows
    w = _fp8(T=120, k=1, E=32, n_group=4, topk_group=2, d=512, inter=256)
    counts = [65, 1, 16, 17, 0, 21]
    idx = np.repeat(np.arange(len(counts), dtype=np.int32), counts)
    np.random.default_rng(7).shuffle(idx)
    _experts_case(w, idx[:, None])
    # T*k <= 64 rows (64-row A boxes when that layout is on): segments of 64
    # rows down to 1
    for counts in ([64], [40, 1, 16, 0, 7]):
        w = _fp8(T=64, k=1, E=32, n_group=4, topk_group=2, d=512, inter=256)
        idx = np.repeat(np.arange(len(counts), dtype=np.int32), counts)
        np.random.default_rng(8).shuffle(idx)
        _experts_case(w, idx[:, None])


# --------------------------------------------------- device-limited routing
def test_router_limited_matches_oracle():
    w = _medium()
    cfg = w.cfg
    rng = np.random.default_rng(21)
    allowed = (rng.random(cfg.E) < 0.4).astype(np.uint8)
    allowed[:cfg.k] = 1
    shape = B.shape_of(cfg)
    ws = B.alloc_workspace(shape)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device="cuda")
    tw = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device="cuda")
    B.router_topk_limited(shape, w.x, w.Wg, torch.as_tensor(allowed, device="cuda"), idx, tw, None, ws)
    torch.cuda.synchronize()
    lg = oracle.logits(dec(w.x), dec(w.Wg))
    idx_o, w_o, gaps = oracle.route_topk_softmax_limited(lg, allowed, cfg.k)
    masked = np.where(allowed[None, :] > 0, lg, -np.inf)
    from parity import compare_indices
    n_ex, report = compare_indices(to_np(idx), idx_o, masked, gaps, None, cfg.E)
    assert n_ex <= int(np.sum(np.any(gaps < 1e-6, axis=1))), report
    assert all(allowed[e] for e in to_np(idx).ravel())
    ok = np.all(to_np(idx) == idx_o, axis=1)
    assert np.allclose(to_np(tw)[ok], w_o[ok], rtol=0, atol=2e-6)


def test_router_limited_fewer_allowed_than_k():
    w = _tiny()
    cfg = w.cfg
    allowed = np.zeros(cfg.E, dtype=np.uint8)
    allowed[[3, 17]] = 1                     # 2 allowed experts, k = 4
    shape = B.shape_of(cfg)
    ws = B.alloc_workspace(shape)
    idx = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device="cuda")
    tw = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device="cuda")
    B.router_topk_limited(shape, w.x, w.Wg, torch.as_tensor(allowed, device="cuda"), idx, tw, None, ws)
    torch.cuda.synchronize()
    lg = oracle.logits(dec(w.x), dec(w.Wg))
    idx_o, w_o, _ = oracle.route_topk_softmax_limited(lg, allowed, cfg.k)
    assert np.array_equal(to_np(idx), idx_o)
    assert np.allclose(to_np(tw), w_o, rtol=0, atol=2e-6)
    assert np.all(to_np(tw)[:, 2:] == 0)


# ------------------------------------------------------ utilisation monitor
@pytest.mark.parametrize("kind", ["random", "crafted", "zero", "skewed"])
def test_expert_utilisation_matches_oracle(kind):
    E = 256
    rng = np.random.default_rng(22)
    if kind == "random":
        counts = rng.integers(0, 300, size=E)
    elif kind == "crafted":   # exactly on the thresholds: mean 10 -> hot above 20, cold below 1
        counts = np.full(E, 10); counts[:4] = [20, 21, 1, 0]; counts[4] = 10 + (20 - 21 - 1 - 0 + 10 * 4 - 40)
    elif kind == "zero":
        counts = np.zeros(E)
    else:
        counts = (1e5 / np.arange(1, E + 1) ** 1.1).astype(np.int64)
    counts = counts.astype(np.int32)
    cfg = workloads.CONFIGS["prefill"]
    shape = B.shape_of(cfg)
    c = torch.as_tensor(counts, device="cuda")
    util = torch.empty(E, dtype=torch.float32, device="cuda")
    flags = torch.empty(E, dtype=torch.int32, device="cuda")
    B.expert_utilisation(shape, c, util, flags)
    torch.cuda.synchronize()
    u_o, f_o = oracle.expert_utilisation(counts)
    assert np.array_equal(to_np(flags), f_o)
    assert np.allclose(to_np(util).astype(np.float64), u_o, rtol=1e-6, atol=1e-9)


def test_expert_utilisation_of_a_forward_pass():
    w = _medium()
    y, idx, tw, counts, ws = run_forward(w)
    shape = B.shape_of(w.cfg)
    util = torch.empty(w.cfg.E, dtype=torch.float32, device="cuda")
    B.expert_utilisation(shape, counts, util, None)
    torch.cuda.synchronize()
    c, _, _, _ = oracle.dispatch(to_np(idx), w.cfg.E)
    u_o, _ = oracle.expert_utilisation(c)
    assert np.allclose(to_np(util), u_o, rtol=1e-6) and abs(float(util.sum()) - 1.0) < 1e-5


# ------------------------------------------------- expert parallelism (next row)
@pytest.mark.parametrize("fp8,world,T", [(False, 2, None), (False, 4, None), (True, 2, None), (True, 2, 48)])
def test_forward_expert_parallel_shares_sum_to_the_layer(fp8, world, T):
    # every rank's share on this one GPU in turn (the all-reduce is the sum):
    # the sum matches the whole-layer launch up to fp32 summation order and
    # the oracle within the layer's tolerance (T=48: the FP8 small-batch
    # stage layout on each rank's slice of the experts)
    from mixture_experts_ffn_17_b200 import expert_parallel as ep
    w = (_fp8(T=T) if T else _fp8()) if fp8 else _medium(shared_inter=512)
    cfg = w.cfg
    y_full, idx, tw, counts, ws = run_forward(w)
    shape = B.shape_of(cfg)
    acc = torch.zeros_like(y_full)
    for r in range(world):
        wr = ep.shard_weights(w.W1, w.W3, w.W2, w.s1, w.s3, w.s2, w.W1s, w.W3s, w.W2s, r, world)
        y_r = torch.empty_like(y_full)
        idx_r = torch.empty_like(idx)
        B.forward_ep(shape, r, world, w.x, w.Wg, w.bias, wr.W1, wr.W3, wr.W2, wr.s1, wr.s3, wr.s2, wr.W1s, wr.W3s,
                     wr.W2s, y_r, ws, topk_idx=idx_r)
        rc, raw = B.check_device_status(ws)
        assert rc == B.MOE_OK, raw
        assert torch.equal(idx_r, idx)  # every rank routes every token the same way
        acc += y_r
    rms = float(y_full.double().pow(2).mean().sqrt())
    assert float((acc - y_full).abs().max()) <= 1e-4 * rms
    y_o, _, _, lg = oracle_full(w)
    _, _, merged, report, n_near = route_with_exemptions(w, lg, to_np(idx))
    assert len(report) <= n_near, report
    if report:
        y_o, *_ = oracle_full(w, force_idx=merged)
    assert max_rel_err(to_np(acc).astype(np.float64), y_o) <= (TOL_FP8 if fp8 else TOL_BF16)


def test_forward_expert_parallel_one_rank_is_the_layer():
    w = _tiny()
    y_full, idx, tw, counts, ws = run_forward(w)
    y1 = torch.empty_like(y_full)
    B.forward_ep(B.shape_of(w.cfg), 0, 1, w.x, w.Wg, w.bias, w.W1, w.W3, w.W2, w.s1, w.s3, w.s2, w.W1s, w.W3s,
                 w.W2s, y1, ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y_full)
