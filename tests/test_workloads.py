"""Synthetic workload recipes (CPU): shapes, distributions, FP8 input
quantisation and the skewed-load statistics."""
import json
import os

import numpy as np
import torch

import oracle
from mixture_experts_ffn_17_b200 import workloads

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_tiny_workload_shapes_and_rms():
    w = workloads.make("tiny")
    c = w.cfg
    assert w.x.shape == (c.T, c.d) and w.x.dtype == torch.bfloat16
    assert w.W1.shape == (c.E, c.d, c.inter) and w.W2.shape == (c.E, c.inter, c.d)
    assert w.W1s.shape == (c.d, c.shared_inter) and w.W2s.shape == (c.shared_inter, c.d)
    rms = torch.sqrt(torch.mean(w.masters["x"] ** 2, dim=1))
    assert torch.allclose(rms, torch.ones_like(rms), atol=1e-5)
    assert abs(w.masters["W1"].std().item() - 0.02) < 1e-3
    assert abs(w.masters["Wg"].std().item() * np.sqrt(c.d) - 1.0) < 0.05
    # bf16 device copies are the fp32 masters rounded once
    assert torch.equal(w.W1, w.masters["W1"].to(torch.bfloat16))


def test_workload_is_deterministic():
    a = workloads.make_small("prefill", T=16, d=256, E=8, k=2, inter=128, shared_inter=128)
    b = workloads.make_small("prefill", T=16, d=256, E=8, k=2, inter=128, shared_inter=128)
    for n in ("x", "Wg", "W1", "W3", "W2", "W1s"):
        assert torch.equal(getattr(a, n), getattr(b, n))


def test_fp8_block_quantisation_error_bound():
    g = torch.Generator().manual_seed(0)
    w = torch.randn(256, 384, generator=g) * 0.006
    q, sc = workloads.quantise_e4m3_blocks(w)
    deq = oracle.decode_e4m3_blocks(q.numpy(), sc.numpy(), 128)
    err = np.abs(deq - w.double().numpy())
    # e4m3 keeps 3 mantissa bits: relative rounding <= 2^-4 for normals; the
    # block maximum maps to 448 exactly, small values fall into subnormals
    # whose absolute step is 2^-9 * scale
    scale_el = np.kron(sc.double().numpy(), np.ones((128, 128)))
    bound = np.maximum(np.abs(w.double().numpy()) * 2.0 ** -4, 2.0 ** -10 * scale_el) * (1 + 1e-6)
    assert np.all(err <= bound)
    amax = w.reshape(2, 128, 3, 128).abs().amax(dim=(1, 3))
    assert torch.allclose(sc, amax / 448.0)


def test_fp8_workload_small():
    w = workloads.make_small("fp8", T=32, d=256, E=16, k=4, inter=256, shared_inter=128,
                             n_group=4, topk_group=2)
    assert w.W1.dtype == torch.uint8 and w.s1.shape == (16, 2, 2) and w.s2.shape == (16, 2, 2)
    assert w.bias.shape == (16,) and w.W1s.dtype == torch.bfloat16


def test_zipf_share_at_calibrated_beta():
    # the logit distribution of the recipe does not depend on d (RMS-normalised
    # x has |x|^2 = d exactly), so a narrow copy re-checks the calibration
    with open(os.path.join(GOLD, "zipf_beta.json")) as f:
        cal = json.load(f)
    assert cal["beta"] == workloads.ZIPF_BETA
    w = workloads.make_small("skewed", d=512, inter=128, shared_inter=128)
    lg = oracle.logits(oracle.decode(w.x), oracle.decode(w.Wg))
    idx, _, _ = oracle.route_topk_softmax(lg, w.cfg.k)
    counts, _, _, _ = oracle.dispatch(idx, w.cfg.E)
    c = np.sort(counts)[::-1]
    share = c[:26].sum() / c.sum()
    assert 0.46 <= share <= 0.54, share
    assert c[0] > 20 * (c.sum() / len(c)) / 2      # an oversize segment: > 10x the mean
