"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each test ties one oracle function to something it does not compute itself:
values the pages print, hand-worked cases, brute-force enumeration on tiny
inputs, invariants, or special cases that reduce to a library routine.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from mixture_experts_ffn_17_b200 import workloads

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------- shapes
def test_parameter_accounting_matches_page_table():
    g = _load("param_counts.json")
    for name in ("decode", "prefill", "skewed", "fp8"):
        c = workloads.CONFIGS[name]
        assert c.d * c.inter == g["gate_projection"] == g["up_projection"] == g["down_projection"]
        assert 3 * c.d * c.inter == g["per_instance_total"]
        assert 3 * c.d * c.shared_inter == g["per_instance_total"]   # shared = 1 x moe_inter
        assert g["per_instance_total"] * g["moe_blocks"] == g["across_moe_blocks"]
        assert (c.E, c.k) == (g["routed_experts"], g["top_k"])


def test_flops_per_token_v3():
    c = workloads.CONFIGS["prefill"]
    # router 2*d*E + (k routed + 1 shared) * 6*d*I
    assert c.flops_per_token() == 3_670_016 + 704_643_072 + 88_080_384 == 796_393_472


# ----------------------------------------------------------------- decoding
def test_e4m3_codes_from_format_definition():
    g = _load("e4m3_codes.json")
    for code, val in g["codes"].items():
        v = oracle.e4m3_value(int(code, 16))
        assert v == val and math.copysign(1, v) == math.copysign(1, val), code
    for code in g["nan_codes"]:
        assert math.isnan(oracle.e4m3_value(int(code, 16)))


def test_e4m3_all_codes_match_torch_float8():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([oracle.e4m3_value(i) for i in range(256)])
    both_nan = np.isnan(ref) & np.isnan(mine)
    assert np.array_equal(ref[~both_nan], mine[~both_nan])
    assert np.array_equal(np.isnan(ref), np.isnan(mine))


def test_e4m3_block_scale_indexing():
    # every code = 1.0, a different scale per block: each element must equal
    # its own block's scale (catches a transposed or mis-strided scale index)
    rows, cols, blk = 256, 384, 128
    q = np.full((rows, cols), 0x38, dtype=np.uint8)
    sc = (np.arange(2 * 3, dtype=np.float32).reshape(2, 3) + 1) * 0.5
    out = oracle.decode_e4m3_blocks(q, sc, blk)
    for r in (0, 127, 128, 255):
        for c in (0, 127, 128, 255, 256, 383):
            assert out[r, c] == sc[r // blk, c // blk]


def test_bf16_decode_is_exact_widening():
    t = torch.randn(1000, dtype=torch.float32).to(torch.bfloat16)
    assert np.array_equal(oracle.decode(t), t.to(torch.float64).numpy())


# ----------------------------------------------------------------- router
def test_logits_special_cases():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 7))
    E = 4
    Wg = np.zeros((E, 7))
    Wg[1, 3] = 1.0      # picks feature 3
    Wg[2] = 1.0         # row sums
    Wg[3, 0], Wg[3, 6] = 2.0, -1.0
    lg = oracle.logits(x, Wg)
    assert np.all(lg[:, 0] == 0.0)
    assert np.array_equal(lg[:, 1], x[:, 3])
    assert np.allclose(lg[:, 2], x.sum(1), rtol=0, atol=1e-14)
    assert np.array_equal(lg[:, 3], 2 * x[:, 0] - x[:, 6])


def test_logits_equal_library_matmul():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((33, 200))
    Wg = rng.standard_normal((17, 200))
    assert np.allclose(oracle.logits(x, Wg), x @ Wg.T, rtol=1e-13, atol=1e-12)


def test_routing_hand_cases():
    for case in _load("routing_hand_cases.json")["cases"]:
        lg = np.array([case["logits"]])
        idx, w, _ = oracle.route_topk_softmax(lg, case["k"])
        assert idx[0].tolist() == case["idx"]
        assert np.allclose(w[0], case["w"], rtol=0, atol=1e-15)


def _brute_topk(l, k):
    """Largest-sum k-subset; among equal sums the lexicographically smallest
    sorted index tuple; slots ordered by (score desc, index asc)."""
    best, best_key = None, None
    for comb in itertools.combinations(range(len(l)), k):
        s = sum(l[i] for i in comb)
        key = (-s, comb)
        if best_key is None or key < best_key:
            best, best_key = comb, key
    return sorted(best, key=lambda i: (-l[i], i))


@pytest.mark.parametrize("E,k", [(6, 2), (9, 3), (12, 4), (5, 5), (7, 1)])
def test_topk_brute_force_random(E, k):
    rng = np.random.default_rng(E * 10 + k)
    lg = rng.standard_normal((40, E))
    idx, w, gaps = oracle.route_topk_softmax(lg, k)
    for t in range(40):
        assert idx[t].tolist() == _brute_topk(lg[t].tolist(), k)
        # the margin that decides slot j is the j-th minus the (j+1)-th score
        # of all E experts in (score desc, index asc) order; +inf for the last
        # slot when k == E (no expert was dropped)
        ranked = sorted(range(E), key=lambda i: (-lg[t, i], i))
        ref = [lg[t, ranked[j]] - lg[t, ranked[j + 1]] if j + 1 < E else math.inf for j in range(k)]
        assert gaps[t].tolist() == ref


@pytest.mark.parametrize("E,k", [(8, 3), (12, 4), (10, 2)])
def test_topk_brute_force_with_exact_ties(E, k):
    # integer-valued logits: many exact ties, sums are exact
    rng = np.random.default_rng(E + k)
    lg = rng.integers(-2, 3, size=(60, E)).astype(np.float64)
    idx, _, _ = oracle.route_topk_softmax(lg, k)
    for t in range(60):
        assert idx[t].tolist() == _brute_topk(lg[t].tolist(), k)


def test_duplicated_gate_rows_lowest_index_wins():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((20, 16))
    Wg = rng.standard_normal((8, 16))
    Wg[5] = Wg[2]          # experts 2 and 5 always tie exactly
    lg = oracle.logits(x, Wg)
    idx, _, _ = oracle.route_topk_softmax(lg, 8)   # k = E: all present
    for t in range(20):
        row = idx[t].tolist()
        assert row.index(2) < row.index(5)


def test_softmax_weight_invariants():
    rng = np.random.default_rng(4)
    lg = rng.standard_normal((50, 32)) * 3
    idx, w, _ = oracle.route_topk_softmax(lg, 4)
    assert np.allclose(w.sum(1), 1.0, rtol=0, atol=1e-12)
    assert np.all(np.diff(w, axis=1) <= 0)            # descending slots
    # ratio of two weights is exp of the logit difference
    for t in range(50):
        r = w[t, 0] / w[t, 1]
        assert math.isclose(r, math.exp(lg[t, idx[t, 0]] - lg[t, idx[t, 1]]), rel_tol=1e-12)


def test_k_equals_E_is_dense_softmax():
    rng = np.random.default_rng(5)
    lg = rng.standard_normal((30, 10))
    idx, w, _ = oracle.route_topk_softmax(lg, 10)
    dense = scipy.special.softmax(lg, axis=1)
    for t in range(30):
        assert np.allclose(w[t], dense[t, idx[t]], rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------- group routing
def _brute_group(l, b, k, n_group, topk_group, topn, scale):
    E = len(l)
    gs = E // n_group
    s = [1 / (1 + math.exp(-v)) for v in l]
    sel = [s[i] + b[i] for i in range(E)]
    gscore = []
    for g in range(n_group):
        members = list(range(g * gs, (g + 1) * gs))
        gscore.append(max(sum(sel[i] for i in c) for c in itertools.combinations(members, topn)))
    keep = _brute_topk(gscore, topk_group)
    cand = sorted(i for g in keep for i in range(g * gs, (g + 1) * gs))
    best, best_key = None, None
    for comb in itertools.combinations(cand, k):
        key = (-sum(sel[i] for i in comb), comb)
        if best_key is None or key < best_key:
            best, best_key = comb, key
    chosen = sorted(best, key=lambda i: (-sel[i], i))
    den = sum(s[i] for i in chosen)
    # the margins: each slot against the next candidate in (sel desc, index
    # asc) order, and the last kept group's score against the best dropped one
    ranked = sorted(cand, key=lambda i: (-sel[i], i))
    gaps = [sel[ranked[j]] - sel[ranked[j + 1]] if j + 1 < len(ranked) else math.inf for j in range(k)]
    granked = sorted(range(n_group), key=lambda g: (-gscore[g], g))
    ggap = gscore[granked[topk_group - 1]] - gscore[granked[topk_group]] if topk_group < n_group else math.inf
    return chosen, [scale * s[i] / den for i in chosen], set(keep), gaps, ggap


@pytest.mark.parametrize("E,n_group,topk_group,k", [(16, 4, 2, 3), (12, 3, 2, 4), (16, 8, 4, 3)])
def test_group_routing_brute_force(E, n_group, topk_group, k):
    rng = np.random.default_rng(E * 7 + k)
    lg = rng.standard_normal((40, E)) * 2
    b = rng.standard_normal(E) * 0.05
    idx, w, gaps, ggap = oracle.route_sigmoid_group(lg, b, k, n_group, topk_group, 2, 2.5)
    gs = E // n_group
    for t in range(40):
        chosen, wref, keep, gref, ggref = _brute_group(lg[t].tolist(), b.tolist(), k, n_group, topk_group, 2, 2.5)
        assert idx[t].tolist() == chosen
        assert np.allclose(w[t], wref, rtol=1e-13, atol=0)
        assert all(i // gs in keep for i in idx[t])
        assert math.isclose(w[t].sum(), 2.5, rel_tol=1e-13)
        assert np.allclose(gaps[t], gref, rtol=0, atol=1e-15)
        assert math.isclose(ggap[t], ggref, rel_tol=0, abs_tol=1e-15)
    # the weight rule alone, on the brute-force selection: unbiased sigmoid
    # scores normalised to sum 1, times the scale
    brute_idx = np.array([_brute_group(lg[t].tolist(), b.tolist(), k, n_group, topk_group, 2, 2.5)[0]
                          for t in range(40)], dtype=np.int32)
    brute_w = np.array([_brute_group(lg[t].tolist(), b.tolist(), k, n_group, topk_group, 2, 2.5)[1]
                        for t in range(40)])
    assert np.allclose(oracle.weights_for(lg, brute_idx, route=1, route_scale=2.5), brute_w, rtol=1e-13, atol=0)


def test_group_routing_one_group_no_bias_reduces_to_topk_of_logits():
    # sigmoid is monotone: with one group and no bias the selection is the
    # page-1 top-k of the logits; weights are the sigmoids normalised x scale
    rng = np.random.default_rng(6)
    lg = rng.standard_normal((64, 32))
    i1, w1, _, _ = oracle.route_sigmoid_group(lg, np.zeros(32), 4, 1, 1, 2, 2.5)
    i0, _, _ = oracle.route_topk_softmax(lg, 4)
    assert np.array_equal(i0, i1)
    s = scipy.special.expit(np.take_along_axis(lg, i1.astype(np.int64), 1))
    assert np.allclose(w1, 2.5 * s / s.sum(1, keepdims=True), rtol=1e-13)


# ----------------------------------------------------------------- dispatch
def test_dispatch_matches_bincount_and_where():
    rng = np.random.default_rng(7)
    T, E, k = 300, 16, 4
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    counts, offsets, perm, row_of = oracle.dispatch(idx, E)
    assert np.array_equal(counts, np.bincount(idx.ravel(), minlength=E))
    assert offsets[0] == 0 and offsets[-1] == T * k
    assert np.array_equal(np.diff(offsets), counts)
    for e in range(E):
        tok, slot = np.nonzero(idx == e)          # the page's torch.where order
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.array_equal(seg, tok)
        assert np.array_equal(row_of[tok * k + slot], np.arange(offsets[e], offsets[e + 1]))
    assert np.array_equal(np.sort(row_of), np.arange(T * k))          # a permutation
    assert np.array_equal(perm[row_of], np.repeat(np.arange(T), k))   # inverse


def test_dispatch_empty_and_single_expert():
    T, E, k = 50, 8, 1
    idx = np.full((T, k), 6, dtype=np.int32)
    counts, offsets, perm, row_of = oracle.dispatch(idx, E)
    assert counts.tolist() == [0] * 6 + [T, 0]
    assert offsets.tolist() == [0] * 7 + [T, T]
    assert np.array_equal(perm, np.arange(T))
    with pytest.raises(ValueError):
        oracle.dispatch(np.array([[8]], dtype=np.int32), E)


# ----------------------------------------------------------------- SwiGLU
def test_swiglu_hand_cases():
    for case in _load("swiglu_hand_cases.json")["cases"]:
        o = oracle.swiglu_rows(np.array(case["x"]), np.array(case["W1"]), np.array(case["W3"]),
                               np.array(case["W2"]))
        assert np.allclose(o, case["o"], rtol=1e-15, atol=1e-15), case["name"]


def test_swiglu_zero_and_linearity():
    rng = np.random.default_rng(8)
    d, I = 24, 16
    x = rng.standard_normal((5, d))
    W1, W3, W2a, W2b = (rng.standard_normal(s) * 0.3 for s in ((d, I), (d, I), (I, d), (I, d)))
    assert np.all(oracle.swiglu_rows(np.zeros((2, d)), W1, W3, W2a) == 0)
    assert np.all(oracle.swiglu_rows(x, W1, W3, np.zeros((I, d))) == 0)
    assert np.all(oracle.swiglu_rows(x, W1, np.zeros((d, I)), W2a) == 0)
    lhs = oracle.swiglu_rows(x, W1, W3, W2a + W2b)
    rhs = oracle.swiglu_rows(x, W1, W3, W2a) + oracle.swiglu_rows(x, W1, W3, W2b)
    assert np.allclose(lhs, rhs, rtol=1e-12, atol=1e-13)


def test_swiglu_silu_odd_part_identity():
    # silu(g) - silu(-g) = g, so o(W1, W3) + o(-W1, -W3) = ((xW1) * (xW3)) W2
    rng = np.random.default_rng(9)
    d, I = 20, 12
    x = rng.standard_normal((4, d))
    W1, W3, W2 = rng.standard_normal((d, I)), rng.standard_normal((d, I)), rng.standard_normal((I, d))
    lhs = oracle.swiglu_rows(x, W1, W3, W2) + oracle.swiglu_rows(x, -W1, -W3, W2)
    rhs = ((x @ W1) * (x @ W3)) @ W2
    assert np.allclose(lhs, rhs, rtol=1e-11, atol=1e-11)


# ------------------------------------------------------------ whole layer
def _tiny(seed=11, T=24, d=32, E=8, I=16, Is=16, scale=0.3):
    rng = np.random.default_rng(seed)
    return dict(
        x=rng.standard_normal((T, d)), Wg=rng.standard_normal((E, d)) / math.sqrt(d),
        W1=rng.standard_normal((E, d, I)) * scale, W3=rng.standard_normal((E, d, I)) * scale,
        W2=rng.standard_normal((E, I, d)) * scale,
        W1s=rng.standard_normal((d, Is)) * scale, W3s=rng.standard_normal((d, Is)) * scale,
        W2s=rng.standard_normal((Is, d)) * scale)


def _shared(p):
    return oracle.swiglu_rows(p["x"], p["W1s"], p["W3s"], p["W2s"])


def test_forward_dense_masked_reference():
    # run every expert on every token, weight by a mask that is zero off the
    # selected set, add the shared expert
    p = _tiny()
    y, idx, w, lg = oracle.moe_forward(**p, k=3)
    T, E = lg.shape
    dense_w = np.zeros((T, E))
    for t in range(T):
        dense_w[t, idx[t]] = w[t]
    ref = _shared(p).copy()
    for e in range(E):
        ref += dense_w[:, e:e + 1] * oracle.swiglu_rows(p["x"], p["W1"][e], p["W3"][e], p["W2"][e])
    rms = np.sqrt(np.mean(ref ** 2))
    assert np.max(np.abs(y - ref)) <= 1e-12 * rms


def test_forward_k_equals_E_dense_softmax_moe():
    p = _tiny(seed=12)
    E = p["Wg"].shape[0]
    y, _, _, lg = oracle.moe_forward(**p, k=E)
    prob = scipy.special.softmax(lg, axis=1)
    ref = _shared(p).copy()
    for e in range(E):
        ref += prob[:, e:e + 1] * oracle.swiglu_rows(p["x"], p["W1"][e], p["W3"][e], p["W2"][e])
    assert np.allclose(y, ref, rtol=1e-11, atol=1e-12)


def test_forward_k1_is_argmax_expert_plus_shared():
    p = _tiny(seed=13)
    y, idx, w, lg = oracle.moe_forward(**p, k=1)
    assert np.all(w == 1.0)
    am = np.argmax(lg, axis=1)
    assert np.array_equal(idx[:, 0], am)
    ref = _shared(p)
    for t in range(len(am)):
        e = am[t]
        ref[t] += oracle.swiglu_rows(p["x"][t:t + 1], p["W1"][e], p["W3"][e], p["W2"][e])[0]
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-13)


def test_forward_special_cases():
    p = _tiny(seed=14)
    # W2 = 0: only the shared expert remains
    q = dict(p, W2=np.zeros_like(p["W2"]))
    y, *_ = oracle.moe_forward(**q, k=3)
    assert np.array_equal(y, _shared(p))
    # shared weights 0 == no shared expert
    q = dict(p, W2s=np.zeros_like(p["W2s"]))
    y0, *_ = oracle.moe_forward(**q, k=3)
    y1, *_ = oracle.moe_forward(**{k_: v for k_, v in p.items() if k_ not in ("W1s", "W3s", "W2s")}, k=3)
    assert np.array_equal(y0, y1)
    # x = 0: silu(0) = 0 everywhere
    q = dict(p, x=np.zeros_like(p["x"]))
    y, *_ = oracle.moe_forward(**q, k=3)
    assert np.all(y == 0)


def test_forward_identical_experts():
    p = _tiny(seed=15)
    E = p["Wg"].shape[0]
    for key in ("W1", "W3", "W2"):
        p[key] = np.repeat(p[key][:1], E, axis=0)
    one = oracle.swiglu_rows(p["x"], p["W1"][0], p["W3"][0], p["W2"][0])
    y, *_ = oracle.moe_forward(**p, k=3)
    assert np.allclose(y, one + _shared(p), rtol=1e-12, atol=1e-13)
    # group mode: the weights sum to route_scale
    y, *_ = oracle.moe_forward(**p, k=3, route=1, bias=np.zeros(E), n_group=4, topk_group=2, route_scale=2.5)
    assert np.allclose(y, 2.5 * one + _shared(p), rtol=1e-12, atol=1e-13)


def test_forward_token_permutation_equivariance():
    p = _tiny(seed=16)
    y, idx, w, _ = oracle.moe_forward(**p, k=2)
    perm = np.random.default_rng(0).permutation(p["x"].shape[0])
    q = dict(p, x=p["x"][perm])
    y2, idx2, w2, _ = oracle.moe_forward(**q, k=2)
    assert np.array_equal(y2, y[perm]) and np.array_equal(idx2, idx[perm])


def test_forward_force_idx_roundtrip():
    p = _tiny(seed=17)
    y, idx, w, lg = oracle.moe_forward(**p, k=3)
    y2, idx2, w2, _ = oracle.moe_forward(**p, k=3, force_idx=idx)
    assert np.array_equal(idx, idx2) and np.array_equal(y, y2)
    assert np.allclose(oracle.weights_for(lg, idx), w, rtol=1e-14)


def test_combine_special_cases():
    rng = np.random.default_rng(18)
    T, k, d = 6, 3, 5
    Yp = rng.standard_normal((T * k, d))
    Ys = rng.standard_normal((T, d))
    # identity placement, unit weight on slot 0 only: y = Yp[t*k] + Ys
    row_of = np.arange(T * k, dtype=np.int32).reshape(T, k)
    w = np.zeros((T, k)); w[:, 0] = 1.0
    assert np.array_equal(oracle.combine(Yp, Ys, row_of, w), Yp[::k] + Ys)
    # equal rows with weights summing to 1 reproduce the row; no shared part
    Yp2 = np.repeat(rng.standard_normal((1, d)), T * k, axis=0)
    w2 = np.full((T, k), 1.0 / 4); w2[:, 0] = 0.5
    assert np.allclose(oracle.combine(Yp2, None, row_of, w2), Yp2[:T], rtol=1e-15, atol=1e-15)
    # skipped rows (row_of < 0) contribute nothing
    row_of3 = row_of.copy(); row_of3[:, 1:] = -1
    assert np.array_equal(oracle.combine(Yp, None, row_of3, np.ones((T, k))), Yp[::k])


# ------------------------------------------------- device-limited routing
def test_device_limited_routing_brute_force_and_special_cases():
    rng = np.random.default_rng(19)
    E, k = 10, 3
    lg = rng.standard_normal((30, E))
    allowed = np.zeros(E, dtype=np.uint8)
    allowed[[1, 2, 5, 7, 8]] = 1
    idx, w, _ = oracle.route_topk_softmax_limited(lg, allowed, k)
    for t in range(30):
        cand = [e for e in range(E) if allowed[e]]
        sub = _brute_topk([lg[t, e] for e in cand], k)
        assert idx[t].tolist() == [cand[i] for i in sub]
        assert all(allowed[e] for e in idx[t])
    assert np.allclose(w.sum(1), 1.0, atol=1e-12)
    # everything allowed == page-1 routing
    i1, w1, _ = oracle.route_topk_softmax_limited(lg, np.ones(E, dtype=np.uint8), k)
    i0, w0, _ = oracle.route_topk_softmax(lg, k)
    assert np.array_equal(i0, i1) and np.array_equal(w0, w1)
    # exactly k allowed: those k, in descending logit order
    al = np.zeros(E, dtype=np.uint8); al[[0, 4, 9]] = 1
    idx, _, _ = oracle.route_topk_softmax_limited(lg, al, 3)
    for t in range(30):
        assert sorted(idx[t].tolist()) == [0, 4, 9]
        assert list(np.diff(lg[t, idx[t]]) <= 0) == [True, True]


# ------------------------------------------------- utilisation monitor
def test_expert_utilisation_definition_cases():
    counts = np.array([0, 1, 10, 10, 10, 10, 39, 0], dtype=np.int32)   # total 80, mean 10
    util, flag = oracle.expert_utilisation(counts)
    assert np.allclose(util, counts / 80.0, rtol=0, atol=0)
    # > 2x mean (20): expert 6; < 0.1x mean (1): experts 0 and 7 (1 is not below 1)
    assert flag.tolist() == [-1, 0, 0, 0, 0, 0, 1, -1]
    u0, f0 = oracle.expert_utilisation(np.zeros(4, dtype=np.int32))
    assert np.all(u0 == 0) and np.all(f0 == 0)
    # uniform load: nothing flagged, utilisation 1/E
    u, f = oracle.expert_utilisation(np.full(16, 7, dtype=np.int32))
    assert np.allclose(u, 1 / 16) and np.all(f == 0)


# ------------------------------------------------------- expert parallelism
def _ep_problem(seed, T=24, d=16, E=8, k=3, I=12, Is=8):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d))
    Wg = rng.standard_normal((E, d))
    W1, W3 = rng.standard_normal((E, d, I)) * 0.3, rng.standard_normal((E, d, I)) * 0.3
    W2 = rng.standard_normal((E, I, d)) * 0.3
    W1s, W3s, W2s = rng.standard_normal((d, Is)) * 0.3, rng.standard_normal((d, Is)) * 0.3, \
        rng.standard_normal((Is, d)) * 0.3
    return x, Wg, W1, W3, W2, W1s, W3s, W2s


def _ep_sum(x, Wg, W1, W3, W2, W1s, W3s, W2s, size, **kw):
    E, Is = W1.shape[0], W1s.shape[1]
    acc = np.zeros_like(x)
    for r in range(size):
        a, b, i0, i1 = oracle.ep_partition(E, Is, r, size)
        acc += oracle.moe_forward_ep_rank(x, Wg, W1[a:b], W3[a:b], W2[a:b], W1s[:, i0:i1], W3s[:, i0:i1],
                                          W2s[i0:i1], e_lo=a, **kw)
    return acc


@pytest.mark.parametrize("route", [0, 1])
def test_expert_parallel_ranks_sum_to_the_layer(route):
    # the all-reduce of the ranks' partial outputs is the layer: every routed
    # slot is owned by exactly one rank and the shared expert's hidden
    # features are split without overlap (SwiGLU is a sum over them)
    p = _ep_problem(3)
    kw = dict(k=3, route=route)
    if route == 1:
        kw.update(bias=np.random.default_rng(4).standard_normal(8) * 0.1, n_group=4, topk_group=2, group_topn=2,
                  route_scale=2.5)
    y_full, *_ = oracle.moe_forward(*p, **kw)
    rms = np.sqrt(np.mean(y_full ** 2))
    for size in (2, 4, 8):
        assert np.abs(_ep_sum(*p, size, **kw) - y_full).max() <= 1e-12 * rms
    # one rank is the layer itself, bit for bit
    assert np.array_equal(_ep_sum(*p, 1, **kw), y_full)


def test_expert_parallel_partition_covers_each_expert_once():
    for E, Is, size in ((256, 2048, 8), (8, 8, 4), (32, 0, 2)):
        seen_e, seen_i = [], []
        for r in range(size):
            a, b, i0, i1 = oracle.ep_partition(E, Is, r, size)
            seen_e += list(range(a, b))
            seen_i += list(range(i0, i1))
        assert seen_e == list(range(E)) and seen_i == list(range(Is))


def test_expert_parallel_rank_without_routed_tokens_is_its_shared_slice():
    # experts 4..7 (rank 1 of 2) get logit -500 on every token, so no slot is
    # theirs and rank 1's partial is exactly its slice of the shared expert
    x, Wg, W1, W3, W2, W1s, W3s, W2s = _ep_problem(5)
    x[:, 0] = 5.0
    Wg[4:] = 0.0
    Wg[4:, 0] = -100.0
    idx, _, _ = oracle.route_topk_softmax(oracle.logits(x, Wg), 3)
    assert (idx < 4).all()
    a, b, i0, i1 = oracle.ep_partition(8, 8, 1, 2)
    y1 = oracle.moe_forward_ep_rank(x, Wg, W1[a:b], W3[a:b], W2[a:b], W1s[:, i0:i1], W3s[:, i0:i1], W2s[i0:i1],
                                    e_lo=a, k=3)
    assert np.array_equal(y1, oracle.swiglu_rows(x, W1s[:, i0:i1], W3s[:, i0:i1], W2s[i0:i1]))
