"""Pins for the oracle's pair counts and pair-based shuffle prediction.

Source: "Expert Coupling in MoE Pretraining" (PicX summary), Method 2 (Token
Shuffling), Mechanism: the owner rank at layer l+1 is predicted from the
experts a token selected at the two preceding layers (a pair-based lookup),
falling back to the single-expert prediction where the pair was seen too
rarely.  Readings: the pair is (top-1 at l-1, top-1 at l); the pair counts
take every (a, b, e') triple of a token, as C takes every (b, e') pair; a pair
row is used when its total reaches min_obs.
"""
import numpy as np
import pytest

import oracle
from combine_warp_top_router_b200 import synth


def _routes(T, E, k, seed, tag):
    lg = synth.group_boost_logits(T, E, 2, 3.0, seed, tag, 5, 6).numpy()
    return oracle.route_topk(lg, k)[0]


def test_pair_counts_brute_force():
    T, E, k = 40, 6, 2
    a, b, c = (_routes(T, E, k, s, 1) for s in (1, 2, 3))
    got = oracle.coselect_pair(a, b, c, E, T_fit=30)
    want = np.zeros((E, E, E), np.int64)
    for t in range(30):
        for x in a[t]:
            for y in b[t]:
                for z in c[t]:
                    want[x, y, z] += 1
    assert np.array_equal(got, want)


@pytest.mark.parametrize("k", [1, 3, 6])
def test_pair_counts_sum_to_k_times_single_counts(k):
    # every token selects k distinct experts at l-1, so summing C2 over the
    # first expert gives k copies of the single cross-layer counts C
    T, E = 300, 16
    a, b, c = (_routes(T, E, k, s, 2) for s in (4, 5, 6))
    C2 = oracle.coselect_pair(a, b, c, E)
    _, C = oracle.coselect(b, c, E)
    assert np.array_equal(C2.sum(axis=0, dtype=np.int64), k * C.astype(np.int64))


def test_rare_pairs_fall_back_to_single_prediction():
    # min_obs above every pair total: the single-expert form exactly
    T, E, k, R = 256, 16, 3, 4
    a, b, c = (_routes(T, E, k, s, 3) for s in (7, 8, 9))
    C2 = oracle.coselect_pair(a, b, c, E)
    _, C = oracle.coselect(b, c, E)
    p = np.random.default_rng(1).permutation(np.arange(E) // (E // R)).astype(np.int32)
    pred, perm, inv, use = oracle.token_shuffle_pair(a, b, C, C2, p, R, int(C2.sum()) + 1)
    assert not use.any()
    want = oracle.token_shuffle(b, C, p, R)
    assert np.array_equal(pred, want[0]) and np.array_equal(perm, want[1])
    assert np.array_equal(inv, want[2])


def test_constant_first_layer_makes_pair_rows_single_rows():
    # every token selects the same experts at l-1, top-1 first: each pair row
    # (a0, b) is exactly the single row C[b], so the results agree and every
    # token with a non-empty row uses its pair row
    T, E, k, R = 192, 16, 2, 4
    b, c = (_routes(T, E, k, s, 4) for s in (10, 11))
    a = np.tile(np.array([[5, 9]], np.int32), (T, 1))
    C2 = oracle.coselect_pair(a, b, c, E)
    _, C = oracle.coselect(b, c, E)
    assert np.array_equal(C2[5], C)
    p = (np.arange(E) // (E // R)).astype(np.int32)
    pred, perm, inv, use = oracle.token_shuffle_pair(a, b, C, C2, p, R, 1)
    want = oracle.token_shuffle(b, C, p, R)
    assert np.array_equal(pred, want[0]) and np.array_equal(perm, want[1])
    assert np.array_equal(use, (C[b[:, 0]].sum(axis=1) > 0).astype(np.int32))


def test_planted_pair_successor_is_recovered():
    # k = 1; the next expert is a fixed function of the (l-1, l) pair that a
    # single layer cannot tell, and not symmetric in it: f(a, b) = (2a + b)
    # mod E.  The pair rows are
    # one-hot (confidence 1), so without capacity pressure every token goes
    # to p_next[f(a, b)].  Pairs are drawn so that each rank gets T/R tokens.
    E, R = 8, 4
    rng = np.random.default_rng(3)
    p = (np.arange(E) // (E // R)).astype(np.int32)
    rows = []
    for d in range(R):
        for _ in range(16):
            a = int(rng.integers(E))
            e_next = int(rng.choice(np.flatnonzero(p == d)))
            rows.append((a, (e_next - 2 * a) % E, e_next))
    rng.shuffle(rows)
    arr = np.array(rows, np.int32)
    a, b, c = arr[:, :1], arr[:, 1:2], arr[:, 2:3]
    C2 = oracle.coselect_pair(a, b, c, E)
    _, C = oracle.coselect(b, c, E)
    pred, _, _, use = oracle.token_shuffle_pair(a, b, C, C2, p, R, 1)
    assert use.all()
    assert np.array_equal(pred, p[(2 * a[:, 0] + b[:, 0]) % E])


def test_min_obs_boundary():
    # one pair row with total 3: used at min_obs 3, not at 4
    E, R = 4, 2
    a = np.array([[0], [0], [0], [1]], np.int32)
    b = np.array([[2], [2], [2], [3]], np.int32)
    c = np.array([[1], [1], [3], [0]], np.int32)
    C2 = oracle.coselect_pair(a, b, c, E)
    _, C = oracle.coselect(b, c, E)
    assert C2[0, 2].sum() == 3
    p = np.array([0, 0, 1, 1], np.int32)
    _, _, _, use3 = oracle.token_shuffle_pair(a, b, C, C2, p, R, 3)
    _, _, _, use4 = oracle.token_shuffle_pair(a, b, C, C2, p, R, 4)
    assert use3.tolist() == [1, 1, 1, 0] and use4.tolist() == [0, 0, 0, 0]
