"""The index-comparison rule of the parity tests, checked on hand-made routings
(CPU only): a slot may differ from the oracle only where an oracle near-tie
touches it, and every other slot must match index for index."""
import numpy as np
import pytest

import oracle

from parity import NEAR_TIE, compare_indices, near_tie_tokens


def _one_token(scores, k):
    lg = np.array([scores], dtype=np.float64)
    idx, _, gaps = oracle.route_topk_softmax(lg, k)
    return lg, idx, gaps


def test_identical_routing_has_no_exemption():
    lg, idx, gaps = _one_token([3.0, 1.0, 2.0, 0.5, -1.0, 0.0], 3)
    assert compare_indices(idx.copy(), idx, lg, gaps) == (0, [])


def test_swap_without_tie_fails():
    lg, idx, gaps = _one_token([3.0, 1.0, 2.0, 0.5, -1.0, 0.0], 3)
    dev = idx.copy()
    dev[0, [1, 2]] = dev[0, [2, 1]]
    with pytest.raises(AssertionError):
        compare_indices(dev, idx, lg, gaps)


def test_swap_at_a_near_tie_is_exempt_and_reported():
    lg, idx, gaps = _one_token([3.0, 2.0 + 0.4 * NEAR_TIE, 2.0, 0.5, -1.0, 0.0], 4)
    dev = idx.copy()
    dev[0, [1, 2]] = dev[0, [2, 1]]
    n, rep = compare_indices(dev, idx, lg, gaps)
    assert n == 1 and rep[0][0] == 0 and [j for j, _ in rep[0][1]] == [1, 2]
    assert len(near_tie_tokens(gaps)) == 1


def test_kth_against_first_dropped_at_a_near_tie():
    lg, idx, gaps = _one_token([3.0, 2.5, 1.0, 1.0 - 0.5 * NEAR_TIE, -1.0, 0.0], 3)
    dev = idx.copy()
    dev[0, 2] = 3                             # the (k+1)-th expert instead of the k-th
    n, rep = compare_indices(dev, idx, lg, gaps)
    assert n == 1 and rep[0][1][0][0] == 2
    dev[0, 2] = 5                             # an expert well below the k-th score
    with pytest.raises(AssertionError):
        compare_indices(dev, idx, lg, gaps)


def test_tie_at_one_slot_does_not_cover_another():
    # slot 1/2 near-tie, but the device also swapped slots 3 and 4 (no tie there)
    lg, idx, gaps = _one_token([9.0, 7.0 + 0.3 * NEAR_TIE, 7.0, 5.0, 4.0, 1.0, 0.0, -1.0], 6)
    dev = idx.copy()
    dev[0, [1, 2]] = dev[0, [2, 1]]
    dev[0, [3, 4]] = dev[0, [4, 3]]
    with pytest.raises(AssertionError):
        compare_indices(dev, idx, lg, gaps)
    # the last slot replaced by an expert outside the top-k, tie elsewhere
    dev = idx.copy()
    dev[0, [1, 2]] = dev[0, [2, 1]]
    dev[0, 5] = 7
    with pytest.raises(AssertionError):
        compare_indices(dev, idx, lg, gaps)


def test_invalid_rows_fail():
    lg, idx, gaps = _one_token([3.0, 2.0 + 0.4 * NEAR_TIE, 2.0, 0.5], 3)
    dev = idx.copy()
    dev[0, 2] = dev[0, 0]                     # duplicate expert
    with pytest.raises(AssertionError):
        compare_indices(dev, idx, lg, gaps)
    dev = idx.copy()
    dev[0, 1] = 4                             # out of range
    with pytest.raises(AssertionError):
        compare_indices(dev, idx, lg, gaps, E=4)


def _group_token(gap):
    # 4 groups of 4 experts; groups 1 and 2 tie up to `gap` at the boundary
    # (top-2 sum), keep 2 groups, pick 3 experts
    E, n_group, topk_group, k = 16, 4, 2, 3
    sel = np.full(E, 0.1)
    sel[0:4] = [0.9, 0.8, 0.2, 0.1]           # group 0: 1.7
    sel[4:8] = [0.55, 0.45, 0.1, 0.1]         # group 1: 1.0 + gap
    sel[8:12] = [0.7, 0.3, 0.1, 0.1]          # group 2: 1.0
    sel[4] += gap
    lg = np.log(sel / (1 - sel))[None, :]     # sigmoid(lg) = sel, bias 0
    idx, w, gaps, ggap = oracle.route_sigmoid_group(lg, np.zeros(E), k, n_group, topk_group, 2, 2.5)
    return lg, 1 / (1 + np.exp(-lg)), idx, gaps, ggap, (n_group, topk_group, 2)


def test_group_boundary_swap_only_at_a_near_tie():
    lg, sel, idx, gaps, ggap, group = _group_token(0.4 * NEAR_TIE)
    assert idx[0].tolist() == [0, 1, 4] and ggap[0] < NEAR_TIE
    dev = np.array([[0, 1, 8]], dtype=np.int32)   # group 2 kept instead of group 1
    n, rep = compare_indices(dev, idx, sel, gaps, ggap, 16, group=group)
    assert n == 1 and rep[0][2] == ggap[0]
    lg, sel, idx, gaps, ggap, group = _group_token(0.05)
    with pytest.raises(AssertionError):
        compare_indices(dev, idx, sel, gaps, ggap, 16, group=group)
