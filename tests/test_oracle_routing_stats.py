"""Pins for the oracle's routing statistics.

Source: "Expert Coupling in MoE Pretraining" (PicX summary):
  Offline Placement and Prediction Statistics, Table I -- "Same GPU" (tokens
  whose experts all sit on one rank), "GPUs" (distinct ranks per token),
  "Dedup" (rows removed by deduplication);
  Cross-layer correlation -- the share of a layer-l expert's tokens that go
  to one layer-l+1 expert (112 of 128 experts at >= 30 %, median 48 %);
  Correlation Formation and Stability -- Pearson correlation between fitted
  and held-out co-selection tables.
"""
import json
import os

import numpy as np
import pytest

import oracle
from combine_warp_top_router_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _routes(T, E, k, seed, tag=1):
    lg = synth.group_boost_logits(T, E, 2, 3.0, seed, tag, 5, 6).numpy()
    return oracle.route_topk(lg, k)[0]


@pytest.mark.parametrize("E,k,R", [(32, 4, 8), (64, 6, 16), (16, 8, 2), (8, 1, 4)])
def test_rank_stats_agree_with_the_dedup_layout(E, k, R):
    # the dedup layout has one row per distinct (token, rank): its row count
    # is sum_D D * hist[D], and tokens with a single row are the "Same GPU" ones
    T = 640
    idx = _routes(T, E, k, E + k)
    p = np.random.default_rng(R).permutation(np.arange(E) // (E // R)).astype(np.int32)
    hist = oracle.rank_stats(idx, E, R, p)
    L = oracle.dispatch_layout(idx, E, R, p, 1)
    assert hist.sum() == T and hist[0] == 0
    assert int((np.arange(k + 1) * hist).sum()) == L["n_rows"]
    rows_per_token = np.bincount(L["row_token"], minlength=T)
    assert hist[1] == int((rows_per_token == 1).sum())
    assert np.array_equal(hist, np.bincount(rows_per_token, minlength=k + 1))


def test_rank_stats_reproduce_table1_contiguous_rows():
    # uniformly random top-2 routing over 128 experts, contiguous placement:
    # the printed contiguous rows of Table I (integers / two decimals)
    g = json.load(open(os.path.join(GOLDEN, "table1_contiguous.json")))
    E, T = g["E"], 200_000
    rng = np.random.default_rng(5)
    idx = np.argsort(rng.random((T, E)), axis=1)[:, :2].astype(np.int32)
    for row in g["top2"]:
        R = row["ep"]
        hist = oracle.rank_stats(idx, E, R, (np.arange(E) // (E // R)).astype(np.int32))
        same = 100 * hist[1] / T
        gpus = (np.arange(3) * hist).sum() / T
        dedup = 100 * (1 - gpus / 2)
        assert abs(same - row["same_gpu_pct"]) < 0.6
        assert abs(gpus - row["gpus_per_token"]) < 0.006
        assert abs(dedup - row["dedup_pct"]) < 0.6


def test_successor_share_of_a_planted_successor():
    # k = 1 at both layers and the next expert is a fixed successor of the
    # current one: every expert sends all of its tokens to one expert
    T, E = 500, 16
    cur = np.random.default_rng(1).integers(0, E, (T, 1)).astype(np.int32)
    succ = np.random.default_rng(2).permutation(E).astype(np.int32)
    nxt = succ[cur]
    W, C = oracle.coselect(cur, nxt, E)
    num, den = oracle.successor_share(C, W)
    assert np.array_equal(num, den)
    assert np.array_equal(den, np.bincount(cur[:, 0], minlength=E))


def test_successor_share_is_at_most_one_and_matches_counts():
    T, E, k = 800, 32, 4
    a, b = _routes(T, E, k, 3), _routes(T, E, k, 4, tag=2)
    W, C = oracle.coselect(a, b, E)
    num, den = oracle.successor_share(C, W)
    assert np.all(num <= den)
    # den = tokens selecting e; num = the most tokens that select e, then one e'
    loads = np.bincount(a.ravel(), minlength=E)
    assert np.array_equal(den, loads)
    both = np.zeros((E, E), np.int64)
    for t in range(T):
        for e in a[t]:
            for e2 in b[t]:
                both[e, e2] += 1
    assert np.array_equal(num, both.max(axis=1))


def test_pearson_against_numpy():
    rng = np.random.default_rng(7)
    x = rng.integers(0, 5000, (64, 64)).astype(np.uint32)
    y = (x + rng.integers(0, 3000, (64, 64))).astype(np.uint32)
    r = oracle.pearson(x, y)
    assert r == pytest.approx(np.corrcoef(x.ravel().astype(np.float64), y.ravel())[0, 1], rel=1e-12)
    assert oracle.pearson(x, x) == pytest.approx(1.0, rel=1e-15)
    sx, sy, sxx, syy, sxy = oracle.count_sums(x, y)
    xi, yi = x.ravel().astype(object), y.ravel().astype(object)
    assert (sx, sy, sxx, syy, sxy) == (sum(xi), sum(yi), sum(xi * xi), sum(yi * yi), sum(xi * yi))


def test_count_sums_are_exact_beyond_64_bits():
    x = np.full(1000, 2 ** 32 - 1, np.uint32)
    sx, _, sxx, _, sxy = oracle.count_sums(x, x)
    assert sx == 1000 * (2 ** 32 - 1) and sxx == sxy == 1000 * (2 ** 32 - 1) ** 2
