"""Pins for the oracle's rounds-based capacity assignment.

Each round, every unassigned token proposes to its first preferred rank that
was not full when the round began; each rank accepts its highest-priority
proposers up to its remaining capacity.  Priorities and preference lists are
those of the sequential form ("Expert Coupling in MoE Pretraining", Method 2:
decreasing confidence, most preferred rank with capacity left)."""
import numpy as np
import pytest

import oracle
from combine_warp_top_router_b200 import synth


def test_hand_example_where_rounds_and_the_sequential_visit_differ():
    # R = 3 ranks of 2 tokens; experts 0..3 on ranks [0, 1, 2, 2].
    #   expert 0: confidence 1.0, prefers 0, 1, 2   (tokens 0, 1)
    #   expert 1: confidence 0.6, prefers 0, 1, 2   (token 2)
    #   expert 2: confidence 0.5, prefers 1, 2, 0   (tokens 3, 4)
    #   expert 3: confidence 3/7, prefers 2, 0, 1   (token 5)
    # Sequentially token 2 finds rank 0 full and takes rank 1 before tokens
    # 3 and 4 arrive.  In rounds, tokens 3 and 4 fill rank 1 in round 1 while
    # token 2 is turned away by rank 0, so token 2 ends on rank 2 in round 2.
    C = np.array([[10, 0, 0, 0], [6, 3, 1, 0], [1, 5, 4, 0], [2, 2, 0, 3]], np.uint32)
    p = np.array([0, 1, 2, 2], np.int32)
    idx = np.array([[0], [0], [1], [2], [2], [3]], np.int32)
    seq = oracle.token_shuffle(idx, C, p, 3)
    assert seq[0].tolist() == [0, 0, 1, 1, 2, 2]
    pred, perm, inv, rounds = oracle.token_shuffle_rounds(idx, C, p, 3)
    assert pred.tolist() == [0, 0, 2, 1, 1, 2] and rounds == 2
    assert perm.tolist() == [0, 1, 4, 2, 3, 5] and np.array_equal(inv[perm], np.arange(6))


def test_no_capacity_pressure_gives_the_first_choices_in_one_round():
    # every rank is the first choice of exactly T/R tokens
    E, R, T = 8, 4, 64
    p = (np.arange(E) // 2).astype(np.int32)
    C = np.eye(E, dtype=np.uint32) * 5 + 1
    idx = np.repeat(np.arange(E, dtype=np.int32), T // E)[:, None]
    idx = np.ascontiguousarray(np.random.default_rng(1).permutation(idx))
    pred, _, _, rounds = oracle.token_shuffle_rounds(idx, C, p, R)
    assert rounds == 1
    assert np.array_equal(pred, p[idx[:, 0]])
    assert np.array_equal(pred, oracle.token_shuffle(idx, C, p, R)[0])


@pytest.mark.parametrize("E,k,R,T", [(64, 2, 16, 16 * 60), (16, 3, 4, 4 * 300), (32, 1, 8, 8 * 50)])
def test_balanced_and_bounded(E, k, R, T):
    rng = np.random.default_rng(E + R)
    C = rng.integers(0, 3, size=(E, E)).astype(np.uint32)
    C[:, rng.choice(E, size=max(1, E // 8), replace=False)] += 40   # capacity pressure
    C[rng.choice(E, size=max(1, E // 10), replace=False), :] = 0       # empty rows
    idx = oracle.route_topk(synth.normal_f32(T, E, 4, 7).numpy(), k)[0]
    p = np.random.default_rng(2).permutation(np.arange(E) // (E // R)).astype(np.int32)
    pred, perm, inv, rounds = oracle.token_shuffle_rounds(idx, C, p, R)
    assert np.array_equal(np.bincount(pred, minlength=R), np.full(R, T // R))
    assert 1 <= rounds <= R + 1
    assert np.array_equal(np.sort(perm), np.arange(T)) and np.array_equal(inv[perm], np.arange(T))
    # positions: rank d's tokens take d*T/R .. in ascending t
    for d in range(R):
        toks = np.flatnonzero(pred == d)
        assert np.array_equal(perm[toks], d * (T // R) + np.arange(T // R))
