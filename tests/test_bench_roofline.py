"""The benchmark's roofline arithmetic on the V3 layer shapes (CPU only)."""
import math
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
from mixture_experts_ffn_17_b200 import workloads  # noqa: E402

PEAKS = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0,
         "fp8_tflops": 3200.0, "fp8_tflops_sustained": 2800.0}


def test_prefill_layer_roofline_is_the_weight_stream():
    cfg = workloads.CONFIGS["prefill"]
    counts = np.full(cfg.E, cfg.T * cfg.k // cfg.E)
    r = bench.layer_roofline(cfg, counts, 5.0, PEAKS, "test")
    assert r["flops"] == cfg.T * 796_393_472
    # 256 experts x 3 x d x I bf16 + shared 3 x d x Is + Wg + x (bf16) + y (fp32)
    weights = 257 * 3 * 7168 * 2048 * 2
    assert r["bytes"] == weights + 256 * 7168 * 2 + 4096 * 7168 * (2 + 4)
    assert r["bound"] == "hbm"
    assert math.isclose(r["hbm_ms"], r["bytes"] / 6500e9 * 1e3)
    assert math.isclose(r["frac"], r["roofline_ms"] / 5.0)
    assert math.isclose(r["frac_datasheet"], r["bytes"] / 8000e9 * 1e3 / 5.0)
    assert "frac_bf16_rate" not in r


def test_fp8_layer_prices_routed_flops_at_the_fp8_peak():
    cfg = workloads.CONFIGS["fp8"]
    counts = np.full(cfg.E, cfg.T * cfg.k // cfg.E)
    r = bench.layer_roofline(cfg, counts, 9.0, PEAKS, "test")
    routed = cfg.T * cfg.k * 6 * cfg.d * cfg.inter
    rest = r["flops"] - routed
    assert math.isclose(r["tensor_ms"], (rest / 1400e12 + routed / 2800e12) * 1e3)
    t16 = r["flops"] / 1400e12 * 1e3
    assert math.isclose(r["frac_bf16_rate"], max(t16, r["hbm_ms"]) / 9.0)
    assert r["frac_bf16_rate"] > r["frac"]
    # e4m3 codes plus one fp32 scale per 128 x 128 block for the routed experts
    assert bench.touched_weight_bytes(cfg, counts) == 256 * (3 * 7168 * 2048 + 3 * 56 * 16 * 4) + 3 * 7168 * 2048 * 2


def test_decode_touched_weights_count_only_touched_experts():
    cfg = workloads.CONFIGS["decode"]
    counts = np.zeros(cfg.E, dtype=np.int64)
    counts[:200] = 2
    counts[200] = 112
    assert bench.touched_weight_bytes(cfg, counts) == 202 * 3 * 7168 * 2048 * 2


def test_backward_work_counts_two_weight_reads_and_every_gradient_write():
    cfg = workloads.CONFIGS["prefill"]
    counts = np.full(cfg.E, cfg.T * cfg.k // cfg.E)
    flops, nbytes, reads, writes = bench.backward_work(cfg, counts, 2)
    # the forward's FLOPs and twice them again (input and weight gradients)
    assert flops == cfg.T * cfg.flops_per_token() * 3
    weights = 257 * 3 * 7168 * 2048 * 2
    assert reads == 2 * weights + 2 * 256 * 7168 * 2 + 4096 * 7168 * (2 + 4)
    assert writes == weights + 256 * 7168 * 2 + 4096 * 7168 * 2     # dW*, dWg and dx in bf16
    assert nbytes == reads + writes
