"""md_table1_row and md_pearson_from_sums: the library's host helpers that
finish the routing statistics ("Expert Coupling in MoE Pretraining", Offline
Placement and Prediction Statistics, Table I; Correlation Formation and
Stability).  Host-only calls: no GPU needed.

The histograms and sums they take come from the oracle here (the same values
md_rank_stats and md_count_sums return on the GPU, which the -m gpu tests
check bit for bit), and the results are checked against numpy and against
hand-worked values."""
import json
import os

import numpy as np
import pytest

import oracle
from combine_warp_top_router_b200 import binding, synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_table1_row_hand_example():
    # 100 tokens, k = 3: 10 on one rank, 30 on two, 60 on three
    same, gpus, dedup = binding.table1_row(np.array([0, 10, 30, 60], np.int64))
    assert same == 10.0
    assert gpus == 2.5
    assert dedup == pytest.approx(100.0 * (1 - 2.5 / 3), abs=1e-12)


def test_table1_row_rejects_empty_and_negative():
    with pytest.raises(binding.MoeDispatchError):
        binding.table1_row(np.zeros(3, np.int64))
    with pytest.raises(binding.MoeDispatchError):
        binding.table1_row(np.array([0, 5, -1], np.int64))


@pytest.mark.parametrize("R", [8, 16, 32])
def test_table1_row_contiguous_uniform_routing(R):
    # iid N(0,1) logits (a uniform random 2-subset of 128 experts) under
    # contiguous placement: the Table I contiguous rows of the golden file,
    # which hold the page's printed values and the closed form
    E, k, T = 128, 2, 1 << 16
    idx = oracle.route_topk(synth.normal_f32(T, E, 5, 1).numpy(), k)[0]
    hist = oracle.rank_stats(idx, E, R, synth.contiguous_placement(E, R).numpy())
    same, gpus, dedup = binding.table1_row(hist)
    # definitions
    assert same == pytest.approx(100.0 * hist[1] / T, rel=1e-15)
    assert gpus == pytest.approx(float((np.arange(k + 1) * hist).sum()) / T, rel=1e-15)
    assert dedup == pytest.approx(100.0 * (1.0 - gpus / k), rel=1e-12)
    # the page's printed contiguous rows: GPUs to two decimals, Dedup in
    # whole percent
    g = json.load(open(os.path.join(GOLDEN, "table1_contiguous.json")))
    row = next(r for r in g["top2"] if r["ep"] == R)
    assert abs(gpus - row["gpus_per_token"]) <= 0.01
    assert abs(dedup - row["dedup_pct"]) <= 0.6


@pytest.mark.parametrize("n,hi,seed", [(16, 5, 0), (4096, 1 << 16, 1), (65536, 1 << 31, 2)])
def test_pearson_matches_numpy(n, hi, seed):
    rng = np.random.default_rng(seed)
    x = rng.integers(0, hi, n, dtype=np.int64).astype(np.uint32)
    y = (x.astype(np.int64) // 2 + rng.integers(0, hi // 2 + 1, n)).astype(np.uint32)
    r = binding.pearson_from_sums(n, oracle.count_sums(x, y))
    want = np.corrcoef(x.astype(np.float64), y.astype(np.float64))[0, 1]
    assert r == pytest.approx(want, rel=1e-12, abs=1e-14)
    assert r == pytest.approx(oracle.pearson(x, y), rel=1e-15, abs=1e-15)


def test_pearson_special_cases():
    x = np.array([3, 1, 4, 1, 5, 9, 2, 6], np.uint32)
    assert binding.pearson_from_sums(8, oracle.count_sums(x, x)) == pytest.approx(1.0, abs=1e-15)
    y = (20 - x.astype(np.int64)).astype(np.uint32)  # y = 20 - x
    assert binding.pearson_from_sums(8, oracle.count_sums(x, y)) == pytest.approx(-1.0, abs=1e-15)
    big = np.full(1000, 2**32 - 1, np.uint32)        # zero variance: undefined
    assert np.isnan(binding.pearson_from_sums(1000, oracle.count_sums(big, x.repeat(125))))


def test_pearson_beyond_64_bits():
    # counts near 2^32 over 2^20 entries: the sums of products need more than
    # 64 bits; r^2 and the sign of r match exact rational arithmetic
    from fractions import Fraction
    rng = np.random.default_rng(9)
    n = 1 << 20
    x = (2**32 - 1 - rng.integers(0, 1000, n)).astype(np.uint32)
    y = (2**32 - 1 - rng.integers(0, 1000, n) - (x.astype(np.int64) % 7)).astype(np.uint32)
    sums = oracle.count_sums(x, y)
    assert sums[2] >= 2**64
    sx, sy, sxx, syy, sxy = sums
    cov = n * sxy - sx * sy
    r2 = Fraction(cov * cov, (n * sxx - sx * sx) * (n * syy - sy * sy))
    r = binding.pearson_from_sums(n, sums)
    assert r * r == pytest.approx(float(r2), rel=1e-12)
    assert (r > 0) == (cov > 0)
