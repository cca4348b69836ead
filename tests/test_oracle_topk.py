"""Pins for the oracle's router step (top-k selection and gate weights).

Source: "Expert Coupling in MoE Pretraining" (PicX summary), Background (each
token goes to its top-k of E experts) and Method 1 (routing probabilities ride
with the rows).  Ties go to the lower expert index and the gates are a softmax
(top-k, then softmax); both are readings the pages leave open.
"""
import numpy as np
import pytest
import scipy.special

import oracle


def _rng(seed):
    return np.random.default_rng(seed)


def test_full_sort_is_numpys_stable_argsort():
    # k = E turns top-k into a full descending sort; numpy's stable argsort of
    # the negated logits gives the same order with ties by lower index.
    lg = _rng(1).standard_normal((50, 37)).astype(np.float32)
    idx, _ = oracle.route_topk(lg, 37)
    assert np.array_equal(idx, np.argsort(-lg, axis=1, kind="stable"))


@pytest.mark.parametrize("k", [1, 3, 16])
def test_ties_go_to_lower_index(k):
    # logits quantised to {-2..2} force many ties
    lg = _rng(2).integers(-2, 3, size=(200, 16)).astype(np.float32)
    idx, _ = oracle.route_topk(lg, k)
    E = lg.shape[1]
    for t in range(lg.shape[0]):
        order = np.lexsort((np.arange(E), -lg[t]))  # primary: -logit, then index
        assert list(idx[t]) == list(order[:k])


def test_signed_zero_and_infinity():
    row = np.array([[-0.0, 0.0, -np.inf, 1.0, 0.0]], np.float32)
    idx, w = oracle.route_topk(row, 5, 0)
    # -0.0 == +0.0 under IEEE comparison, so the three zeros keep index order
    assert list(idx[0]) == [3, 0, 1, 4, 2]
    assert w[0, 4] == 0.0  # exp(-inf) contributes nothing


def test_k1_gate_is_exactly_one():
    lg = _rng(3).standard_normal((64, 32)).astype(np.float32) * 5
    _, w = oracle.route_topk(lg, 1, 0)
    assert np.all(w == 1.0)


@pytest.mark.parametrize("mode", [0, 1])
def test_gates_match_scipy_softmax(mode):
    lg = (_rng(4).standard_normal((300, 64)) * 3).astype(np.float32)
    k = 6
    idx, w = oracle.route_topk(lg, k, mode)
    sel = np.take_along_axis(lg.astype(np.float64), idx.astype(np.int64), axis=1)
    if mode == 0:
        ref = scipy.special.softmax(sel, axis=1)
    else:
        full = scipy.special.softmax(lg.astype(np.float64), axis=1)
        ref = np.take_along_axis(full, idx.astype(np.int64), axis=1)
    # the oracle rounds a double result to float once: within 1 float ulp
    assert np.all(np.abs(w - ref) <= 2.0 ** -23 * ref + 1e-45)
    if mode == 0:
        assert np.allclose(w.astype(np.float64).sum(1), 1.0, atol=1e-6)
    else:
        assert np.all(w.astype(np.float64).sum(1) <= 1.0 + 1e-6)


def test_worked_example():
    # Worked by hand: token 0 has a tie between experts 1 and 2 at 3.0, so the
    # top-2 is [1, 2] with equal gates 1/2.  Token 1 is all zeros: top-2 is
    # [0, 1]; top-k gates are 1/2 each, full-softmax gates 1/4 each.
    lg = np.array([[1.0, 3.0, 3.0, 0.0], [0.0, 0.0, 0.0, 0.0]], np.float32)
    idx, w = oracle.route_topk(lg, 2, 0)
    assert idx.tolist() == [[1, 2], [0, 1]]
    assert w.tolist() == [[0.5, 0.5], [0.5, 0.5]]
    _, w1 = oracle.route_topk(lg, 2, 1)
    assert w1[1].tolist() == [0.25, 0.25]
    # token 0, full softmax: 1 / (2 + e^-2 + e^-3)
    assert abs(w1[0, 0] - 1.0 / (2.0 + np.exp(-2.0) + np.exp(-3.0))) < 1e-7


def test_rejects_bad_arguments():
    with pytest.raises(ValueError):
        oracle.route_topk(np.zeros((2, 4), np.float32), 5)
