"""Pins for the oracle's Kernighan-Lin passes and two-level placement.

Source: "Expert Coupling in MoE Pretraining" (PicX summary), Correlated
Placement: a Kernighan-Lin-style local search swaps experts between GPUs to
maximise the co-located sum of W, every GPU keeping E/EP experts; multi-node
groups are partitioned across nodes first, then across each node's GPUs.
A KL pass (Kernighan and Lin's bisection heuristic) may take swaps with a
negative gain and keeps the best prefix, so it can leave a placement where no
single swap gains.
"""
import itertools

import numpy as np
import pytest

import oracle
from combine_warp_top_router_b200 import synth


def _objective(W, p):
    return oracle.placement_objective(W, p)


def _best_single_swap_gain(W, p):
    E = len(p)
    base, best = _objective(W, p), 0
    for a in range(E):
        for b in range(a + 1, E):
            if p[a] != p[b]:
                q = p.copy()
                q[a], q[b] = q[b], q[a]
                best = max(best, _objective(W, q) - base)
    return best


def _brute_force_optimum(W, R):
    E = W.shape[0]
    cap = E // R
    best = -1
    for rest in itertools.combinations(range(1, E), cap - 1):   # R = 2: rank of expert 0 fixed
        p = np.ones(E, np.int32)
        p[[0, *rest]] = 0
        best = max(best, _objective(W, p))
    return best


# co-selection counts (symmetric, zero diagonal) on 8 experts and 2 ranks:
# contiguous placement scores 22 and no single swap improves it, but the
# optimum (brute force over all 35 balanced bisections) scores 24
W_STUCK = np.array([[0, 1, 3, 3, 0, 2, 1, 2],
                    [1, 0, 3, 3, 1, 0, 2, 2],
                    [3, 3, 0, 1, 2, 1, 3, 1],
                    [3, 3, 1, 0, 0, 0, 2, 0],
                    [0, 1, 2, 0, 0, 0, 3, 1],
                    [2, 0, 1, 0, 0, 0, 0, 3],
                    [1, 2, 3, 2, 3, 0, 0, 1],
                    [2, 2, 1, 0, 1, 3, 1, 0]], np.uint32)


def test_kl_escapes_a_single_swap_local_optimum():
    contiguous = (np.arange(8) // 4).astype(np.int32)
    assert _objective(W_STUCK, contiguous) == 22
    assert _best_single_swap_gain(W_STUCK, contiguous) == 0
    assert _brute_force_optimum(W_STUCK, 2) == 24
    swaps = oracle.place_two_level(W_STUCK, 2, refine_mode=oracle.REFINE_SWAPS)
    assert np.array_equal(swaps, contiguous)
    kl = oracle.place_two_level(W_STUCK, 2, refine_mode=oracle.REFINE_KL)
    assert _objective(W_STUCK, kl) == 24


@pytest.mark.parametrize("E,R,seed_mode", [(16, 4, 0), (16, 2, 1), (32, 8, 0), (24, 3, 1)])
def test_kl_result_is_balanced_not_worse_and_swap_stable(E, R, seed_mode):
    lg = synth.group_boost_logits(512, E, 2, 3.0, E + R, 1, 5, 6).numpy()
    W, _ = oracle.coselect(oracle.route_topk(lg, 4)[0], None, E)
    seed = oracle.place_two_level(W, R, seed_mode=seed_mode, refine_mode=oracle.REFINE_NONE)
    kl = oracle.place_two_level(W, R, seed_mode=seed_mode, refine_mode=oracle.REFINE_KL)
    assert np.array_equal(np.bincount(kl, minlength=R), np.full(R, E // R))
    assert _objective(W, kl) >= _objective(W, seed)
    # a pass starts with the best single swap, so passes only stop where none gains
    assert _best_single_swap_gain(W, kl) == 0


def test_one_level_modes_match_the_single_level_oracle():
    lg = synth.group_boost_logits(400, 32, 2, 3.0, 3, 1, 5, 6).numpy()
    W, _ = oracle.coselect(oracle.route_topk(lg, 4)[0], None, 32)
    for seed_mode in (0, 1):
        assert np.array_equal(oracle.place_two_level(W, 8, 1, seed_mode, oracle.REFINE_SWAPS),
                              oracle.place_correlated(W, 8, seed_mode, True))
        assert np.array_equal(oracle.place_two_level(W, 8, 1, seed_mode, oracle.REFINE_NONE),
                              oracle.place_correlated(W, 8, seed_mode, False))


@pytest.mark.parametrize("refine_mode", [oracle.REFINE_SWAPS, oracle.REFINE_KL])
def test_two_level_structure(refine_mode):
    E, R, nodes = 32, 8, 2
    lg = synth.group_boost_logits(800, E, 2, 3.0, 5, 1, 5, 6).numpy()
    W, _ = oracle.coselect(oracle.route_topk(lg, 4)[0], None, E)
    p = oracle.place_two_level(W, R, nodes, 0, refine_mode)
    assert np.array_equal(np.bincount(p, minlength=R), np.full(R, E // R))
    node = p // (R // nodes)
    # level 1 alone: the same search with nodes as ranks
    assert np.array_equal(node, oracle.place_two_level(W, nodes, 1, 0, refine_mode))
    # level 2: each node's experts, in ascending id, on its R/nodes ranks
    for n in range(nodes):
        mem = np.flatnonzero(node == n)
        sub = np.ascontiguousarray(W[np.ix_(mem, mem)])
        want = oracle.place_two_level(sub, R // nodes, 1, 0, refine_mode)
        assert np.array_equal(p[mem] - n * (R // nodes), want)


def test_one_rank_per_node_is_one_level():
    lg = synth.group_boost_logits(300, 16, 2, 3.0, 9, 1, 5, 6).numpy()
    W, _ = oracle.coselect(oracle.route_topk(lg, 2)[0], None, 16)
    for mode in (oracle.REFINE_SWAPS, oracle.REFINE_KL):
        assert np.array_equal(oracle.place_two_level(W, 4, 4, 0, mode), oracle.place_two_level(W, 4, 1, 0, mode))
