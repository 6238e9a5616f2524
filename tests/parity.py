"""Comparison rules between the CUDA path and the fp64 oracle (test helpers).

Rules (the layer's stated parity bar):
  * expert indices, per-expert counts and the permutation are bit-exact.  The
    one allowed difference is a near-tie: the oracle's ordered scores of two
    neighbouring slots (slot j vs slot j+1, the k-th vs the (k+1)-th) closer
    than 1e-6.  The rule is applied slot by slot: a slot may differ from the
    oracle only where such a near-tie touches it, and the expert the device put
    there must score inside the tied run of the oracle's scores; every other
    slot must match the oracle index for index, slot order included.  In group
    mode, where the oracle's last kept and first dropped group scores are
    closer than 1e-6, the device may instead follow the selection the swapped
    group set gives (slot by slot again).  Every exempted token is reported
    with its slots and gaps.
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


def near_tie_tokens(gaps: np.ndarray, ggap=None) -> np.ndarray:
    """Tokens whose oracle routing has any near-tie (a slot gap, or in group
    mode the group-boundary gap, below NEAR_TIE)."""
    near = np.any(gaps < NEAR_TIE, axis=1)
    if ggap is not None:
        near |= ggap < NEAR_TIE
    return np.nonzero(near)[0]


def _slot_mismatches(dev_row, ora_row, score_row, gap_row):
    """Slot-by-slot check of one token.  Returns [(slot, gap), ...] for the
    slots that differ, or None when a differing slot is not covered by a
    near-tie or holds an expert outside the tied run of scores."""
    k = len(ora_row)
    out = []
    for j in range(k):
        if dev_row[j] == ora_row[j]:
            continue
        # the run of slots linked to j by gaps below NEAR_TIE; b == k means
        # the run reaches the first expert the oracle dropped
        a = j
        while a > 0 and gap_row[a - 1] < NEAR_TIE:
            a -= 1
        b = j
        while b < k and gap_row[b] < NEAR_TIE:
            b += 1
        if a == b:
            return None
        top = score_row[ora_row[a]]
        low = score_row[ora_row[b]] if b < k else score_row[ora_row[k - 1]] - gap_row[k - 1]
        s = score_row[dev_row[j]]
        if not (low - 1e-12 <= s <= top + 1e-12):
            return None
        out.append((j, float(min(gap_row[j], gap_row[j - 1] if j > 0 else np.inf))))
    return out


def _swapped_group_selection(sel_row, k, n_group, topk_group, group_topn):
    """Selection the group rule gives when the last kept group and the first
    dropped group trade places: (idx [k], gaps [k])."""
    E = len(sel_row)
    gsz = E // n_group
    gscore = np.array([np.sort(sel_row[g * gsz:(g + 1) * gsz])[::-1][:group_topn].sum() for g in range(n_group)])
    order = np.lexsort((np.arange(n_group), -gscore))
    keep = list(order[:topk_group - 1]) + [order[topk_group]]
    cand = np.array(sorted(e for g in keep for e in range(g * gsz, (g + 1) * gsz)))
    cs = sel_row[cand]
    o = cand[np.lexsort((cand, -cs))]
    sc = sel_row[o]
    gaps = np.array([sc[j] - sc[j + 1] if j + 1 < len(o) else np.inf for j in range(k)])
    return o[:k], gaps


def compare_indices(idx_dev: np.ndarray, idx_ora: np.ndarray, scores: np.ndarray, gaps: np.ndarray,
                    ggap=None, E=None, group=None):
    """Per-slot comparison of the device's routing with the oracle's.

    group: (n_group, topk_group, group_topn) in group mode, else None.
    Returns (n_exempt, report) where report lists (token, [(slot, gap), ...],
    group gap or None) for every exempted token.  Raises AssertionError on a
    violation."""
    T, k = idx_ora.shape
    assert idx_dev.shape == idx_ora.shape
    E = E if E is not None else scores.shape[1]
    diff = np.nonzero((idx_dev != idx_ora).any(axis=1))[0]
    report = []
    for t in diff:
        row = idx_dev[t]
        if not (len(set(row.tolist())) == k and row.min() >= 0 and row.max() < E):
            raise AssertionError(f"token {t}: device idx {row.tolist()} is not k distinct experts in range")
        slots = _slot_mismatches(row, idx_ora[t], scores[t], gaps[t])
        gg = None
        if slots is None and ggap is not None and group is not None and ggap[t] < NEAR_TIE:
            alt_idx, alt_gaps = _swapped_group_selection(scores[t], k, *group)
            slots = _slot_mismatches(row, alt_idx, scores[t], alt_gaps)
            gg = float(ggap[t])
            if slots is not None:   # report the slots that differ from the oracle's own selection
                slots = [(int(j), gg) for j in np.nonzero(row != idx_ora[t])[0]]
        if slots is None:
            raise AssertionError(f"token {t}: device idx {row.tolist()} vs oracle {idx_ora[t].tolist()}, "
                                 f"gaps {gaps[t].tolist()} group gap {None if ggap is None else ggap[t]}")
        report.append((int(t), slots, gg))
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
