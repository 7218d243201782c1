"""Pins of the oracle's top-k router (reading R15) against facts that do not
depend on its own code: the full-softmax definition of the weights, the
k = 1 and all-equal special cases, the ordering property of a top-k set and
equivariance under a relabelling of the experts."""
import itertools

import numpy as np
from scipy.special import softmax

from oracle import moe


def _logits(T, E, seed):
    return np.random.default_rng(seed).standard_normal((T, E)).astype(np.float32)


def test_k1_is_argmax_with_weight_one():
    lg = _logits(50, 16, 1)
    idx, w = moe.route_topk(lg, 1)
    assert np.array_equal(idx[:, 0], np.argmax(lg, axis=1))
    assert np.all(w == 1.0)


def test_equal_logits_pick_the_lowest_ids_with_equal_weights():
    idx, w = moe.route_topk(np.zeros((3, 10), np.float32), 4)
    assert np.array_equal(idx, np.tile(np.arange(4), (3, 1)))
    assert np.allclose(w, 0.25, rtol=0, atol=1e-15)


def test_ties_inside_and_at_the_cut():
    lg = np.array([[0.5, 2.0, 2.0, -1.0, 0.5, 0.5]], np.float32)
    idx, _ = moe.route_topk(lg, 4)
    # 2.0 at ids 1, 2; then 0.5 at ids 0, 4, 5 -> the cut keeps the lowest id 0
    assert idx.tolist() == [[1, 2, 0, 4]]


def test_weights_equal_the_full_softmax_renormalised_over_the_chosen():
    lg = _logits(40, 128, 2)
    idx, w = moe.route_topk(lg, 8)
    p = softmax(lg.astype(np.float64), axis=1)
    sel = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    assert np.allclose(w, sel / sel.sum(axis=1, keepdims=True), rtol=1e-12, atol=0)
    assert np.allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert np.all(np.diff(w, axis=1) <= 0)   # slots in descending weight


def test_chosen_set_dominates_the_rest_brute_force():
    lg = np.random.default_rng(3).integers(-2, 3, size=(60, 7)).astype(np.float32)  # many ties
    for k in (1, 3, 7):
        idx, _ = moe.route_topk(lg, k)
        for t in range(lg.shape[0]):
            chosen = list(idx[t])
            # the unique k-subset whose members all precede every non-member in
            # the order (larger logit first, then lower id), listed in that order
            best = None
            for sub in itertools.combinations(range(7), k):
                rest = [e for e in range(7) if e not in sub]
                if all((lg[t, a], -a) > (lg[t, b], -b) for a in sub for b in rest):
                    best = sorted(sub, key=lambda e: (-lg[t, e], e))
            assert chosen == best


def test_relabelling_the_experts_relabels_the_choice():
    lg = _logits(30, 32, 4)                       # continuous values: no ties
    perm = np.random.default_rng(5).permutation(32)
    idx, w = moe.route_topk(lg, 6)
    idx_p, w_p = moe.route_topk(lg[:, perm], 6)   # column j of the new matrix is expert perm[j]
    assert np.array_equal(perm[idx_p], idx)
    assert np.array_equal(w_p, w)
