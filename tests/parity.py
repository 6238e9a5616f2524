"""Comparison rules between the CUDA path and the fp64 oracle (test helpers).

Rules (the layer's stated parity bar):
  * expert indices, per-expert counts and the permutation are bit-exact, except
    that a token's indices may differ where the oracle's ordered scores have a
    near-tie: two scores that decide a slot (slot j's score vs slot j+1's, the
    k-th vs the (k+1)-th; in group mode also the last kept vs first dropped
    group score) closer than 1e-6.  Every such token is reported.  The device's
    choice must still be valid: distinct indices in range whose oracle scores
    are within 1e-6 of the oracle's k-th score or above it.
  * counts and permutation are compared against the oracle's dispatch of the
    device's indices once the exemptions above are accepted.
  * outputs: max |y - y_oracle| <= 2e-2 * rms(y_oracle) (bf16 weights) or
    6e-2 * rms (FP8 weights), fp32 accumulation on the device.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

NEAR_TIE = 1e-6
TOL_BF16 = 2e-2
TOL_FP8 = 6e-2


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def dec(t: torch.Tensor) -> np.ndarray:
    """Stored tensor (any device) -> fp64 numpy, exactly."""
    return oracle.decode(t.detach().cpu())


def oracle_route(cfg, lg: np.ndarray, bias=None):
    """(idx, w, scores_for_gap, gaps [T,k], group_gap [T] or None)."""
    if cfg.route == 0:
        idx, w, gaps = oracle.route_topk_softmax(lg, cfg.k)
        return idx, w, lg, gaps, None
    b = np.zeros(cfg.E) if bias is None else bias
    idx, w, gaps, ggap = oracle.route_sigmoid_group(lg, b, cfg.k, cfg.n_group, cfg.topk_group, cfg.group_topn,
                                                    cfg.route_scale)
    sel = 1.0 / (1.0 + np.exp(-lg)) + b[None, :]
    return idx, w, sel, gaps, ggap


def compare_indices(idx_dev: np.ndarray, idx_ora: np.ndarray, scores: np.ndarray, gaps: np.ndarray,
                    ggap=None, E=None):
    """Returns (n_exempt, report list).  Raises AssertionError on a violation."""
    T, k = idx_ora.shape
    assert idx_dev.shape == idx_ora.shape
    E = E if E is not None else scores.shape[1]
    diff = np.nonzero((idx_dev != idx_ora).any(axis=1))[0]
    report = []
    for t in diff:
        g = gaps[t].copy()
        near = bool(np.min(g) < NEAR_TIE) or (ggap is not None and ggap[t] < NEAR_TIE)
        row = idx_dev[t]
        valid = (len(set(row.tolist())) == k and row.min() >= 0 and row.max() < E)
        kth = scores[t, idx_ora[t, -1]]
        valid = valid and bool(np.all(scores[t, row] >= kth - NEAR_TIE))
        if not (near and valid):
            raise AssertionError(f"token {t}: device idx {row.tolist()} vs oracle {idx_ora[t].tolist()}, "
                                 f"gaps {g.tolist()} group gap {None if ggap is None else ggap[t]}")
        report.append((int(t), float(np.min(g))))
    return len(report), report


def max_rel_err(y_dev: np.ndarray, y_ora: np.ndarray) -> float:
    rms = float(np.sqrt(np.mean(y_ora ** 2)))
    return float(np.max(np.abs(y_dev - y_ora))) / rms


def bf16_stored_ok(y_dev: np.ndarray, y_ora: np.ndarray, tol: float = 1e-2) -> bool:
    """Check for an intermediate the device stores in bf16: per element,
    |y_dev - y_ora| <= 2^-8 |y_ora| (the rounding of the store itself, half an
    ulp of an 8-significant-bit format) + tol * rms(y_ora) (everything else)."""
    rms = float(np.sqrt(np.mean(y_ora ** 2)))
    bound = 2.0 ** -8 * np.abs(y_ora) + tol * rms
    return bool(np.all(np.abs(y_dev - y_ora) <= bound))
