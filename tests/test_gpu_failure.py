"""Failure detection on the GPU without a fault: the grouped-GEMM producers
are told to withhold their loads (MOE_DEBUG_WITHHOLD_LOADS=1), so the MMA
issuers' bounded waits run out (about 2 s); the launch must end by itself,
report MOE_ERR_DEVICE_TIMEOUT through the workspace status word, and leave the
CUDA context usable: the next call (switch off) is correct."""
import numpy as np
import pytest
import torch

from mixture_experts_ffn_17_b200 import binding as B
from mixture_experts_ffn_17_b200 import build as libbuild
from mixture_experts_ffn_17_b200 import workloads

from gpu_util import oracle_full, run_forward, to_device
from parity import TOL_BF16, max_rel_err, to_np

pytestmark = pytest.mark.gpu


def test_bounded_wait_timeout_is_reported_and_context_survives(monkeypatch):
    libbuild.build()
    w = to_device(workloads.make("tiny"))
    cfg = w.cfg
    shape = B.shape_of(cfg)
    ws = B.alloc_workspace(shape)
    y = torch.zeros(cfg.T, cfg.d, dtype=torch.float32, device="cuda")
    monkeypatch.setenv("MOE_DEBUG_WITHHOLD_LOADS", "1")
    B.forward(shape, w.x, w.Wg, None, w.W1, w.W3, w.W2, None, None, None, w.W1s, w.W3s, w.W2s, y, ws)
    rc, raw = B.check_device_status(ws)
    assert rc == B.MOE_ERR_DEVICE_TIMEOUT and (raw & 1), (rc, raw)
    monkeypatch.delenv("MOE_DEBUG_WITHHOLD_LOADS")
    y2, idx, _, _, _ = run_forward(w)          # asserts MOE_OK itself
    y_o, idx_o, _, _ = oracle_full(w)
    same = np.all(to_np(idx) == idx_o, axis=1)
    assert max_rel_err(to_np(y2).astype(np.float64)[same], y_o[same]) <= TOL_BF16


@pytest.mark.parametrize("fp8", [False, True])
def test_bounded_wait_timeout_on_cta_pairs(monkeypatch, fp8):
    # the same failure on the 2-CTA-cluster kernels: both CTAs of every pair
    # end their waits, meet at the final cluster barrier and free TMEM
    libbuild.build()
    kw = dict(T=1024, d=256, E=32, k=8, inter=128, shared_inter=128)  # ~256 rows per expert
    w = to_device(workloads.make_small("fp8", n_group=4, topk_group=2, **kw) if fp8
                  else workloads.make_small("prefill", **kw))
    cfg = w.cfg
    shape = B.shape_of(cfg)
    ws = B.alloc_workspace(shape)
    y = torch.zeros(cfg.T, cfg.d, dtype=torch.float32, device="cuda")
    monkeypatch.setenv("MOE_PAIR_TILES", "1")
    monkeypatch.setenv("MOE_DEBUG_WITHHOLD_LOADS", "1")
    B.forward(shape, w.x, w.Wg, w.bias, w.W1, w.W3, w.W2, w.s1, w.s3, w.s2, w.W1s, w.W3s, w.W2s, y, ws)
    rc, raw = B.check_device_status(ws)
    assert rc == B.MOE_ERR_DEVICE_TIMEOUT and (raw & 1), (rc, raw)
    monkeypatch.delenv("MOE_DEBUG_WITHHOLD_LOADS")
    y2, idx, _, _, _ = run_forward(w)
    y_o, idx_o, _, _ = oracle_full(w)
    same = np.all(to_np(idx) == idx_o, axis=1)
    assert max_rel_err(to_np(y2).astype(np.float64)[same], y_o[same]) <= (6e-2 if fp8 else TOL_BF16)
