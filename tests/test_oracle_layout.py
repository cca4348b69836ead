"""Pins for the oracle's dispatch layout (send matrix, row positions, dedup rows).

Sources:
  "DODOCO: MoE AlltoAll Traffic Matrices on Real Text" -- Setup (ranks route
  contiguous token blocks; contiguous expert placement), send_matrices.csv
  (combine is the transposed matrix), Reading the counts (rows sum to tokens
  per rank x top-k; each rank's expert block matches its receive total;
  summing contiguous rank blocks gives the matrix at a smaller EP width).
  "Expert Coupling in MoE Pretraining" -- Method 1 (one row per distinct
  (token, destination rank) pair) and Table I (contiguous-placement rows).
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from combine_warp_top_router_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _routes(T, E, k, seed=0, gen="iid"):
    if gen == "iid":
        lg = synth.normal_f32(T, E, seed, 1).numpy()
    else:
        lg = synth.group_boost_logits(T, E, 2, 3.0, seed, 1, 5, 6).numpy()
    idx, _ = oracle.route_topk(lg, k)
    return idx


def _contig(E, R):
    return synth.contiguous_placement(E, R).numpy()


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("gen", ["iid", "groups"])
def test_row_sums_and_transposed_combine(mode, gen):
    T, E, k, R = 2048, 64, 6, 16
    idx = _routes(T, E, k, gen=gen)
    p = _contig(E, R)
    L = oracle.dispatch_layout(idx, E, R, p, mode)
    S = L["send_counts"]
    Tr = T // R
    if mode == 0:
        # each row sums to (tokens per rank) x top-k
        assert np.all(S.sum(1) == Tr * k)
    else:
        # one row per distinct (token, destination) pair, counted by brute force
        for s in range(R):
            distinct = {(t, int(p[e])) for t in range(s * Tr, (s + 1) * Tr) for e in idx[t]}
            assert S[s].sum() == len(distinct)
            assert Tr <= S[s].sum() <= Tr * min(k, R)
    # combine returns the same volumes in reverse: count rows of rank d's block
    # by the source rank of their token and compare with the transpose
    ro = L["rank_offsets"]
    back = np.zeros((R, R), np.int64)
    for d in range(R):
        for r in range(ro[d], ro[d + 1]):
            back[d, L["row_token"][r] // Tr] += 1
    assert np.array_equal(back, S.T)


def test_receive_totals_match_expert_blocks():
    T, E, k, R = 2048, 64, 6, 16
    idx = _routes(T, E, k, gen="groups")
    p = _contig(E, R)
    L = oracle.dispatch_layout(idx, E, R, p, 0)
    ec = L["expert_counts"]
    assert np.array_equal(ec, np.bincount(idx.ravel(), minlength=E))
    for d in range(R):
        assert L["send_counts"][:, d].sum() == ec[p == d].sum()


def test_coarsening_contiguous_blocks():
    # EP16 matrix summed over 2x2 contiguous blocks equals the EP8 matrix
    T, E, k = 4096, 128, 8
    idx = _routes(T, E, k, gen="groups")
    S16 = oracle.dispatch_layout(idx, E, 16, _contig(E, 16), 0)["send_counts"]
    S8 = oracle.dispatch_layout(idx, E, 8, _contig(E, 8), 0)["send_counts"]
    assert np.array_equal(S16.reshape(8, 2, 8, 2).sum(axis=(1, 3)), S8)
    S4 = oracle.dispatch_layout(idx, E, 4, _contig(E, 4), 0)["send_counts"]
    assert np.array_equal(S16.reshape(4, 4, 4, 4).sum(axis=(1, 3)), S4)


@pytest.mark.parametrize("placement", ["contiguous", "shuffled"])
def test_positions_are_a_lexsort(placement):
    T, E, k, R = 512, 32, 4, 8
    idx = _routes(T, E, k, seed=3)
    p = _contig(E, R)
    if placement == "shuffled":
        p = np.random.default_rng(5).permutation(p).astype(np.int32)
    L = oracle.dispatch_layout(idx, E, R, p, 1)
    t_of = np.repeat(np.arange(T), k)
    e_of = idx.ravel()
    order = np.lexsort((t_of, e_of, p[e_of]))  # keys: rank, expert, token
    conv = np.empty(T * k, np.int64)
    conv[order] = np.arange(T * k)
    assert np.array_equal(L["assign_row"].ravel(), conv)
    # dedup rows: distinct (t, d) pairs ordered by (d, t)
    pairs = sorted({(int(p[e]), t) for t in range(T) for e in idx[t]})
    assert L["n_rows"] == len(pairs)
    assert [(int(np.searchsorted(L["rank_offsets"], r, "right") - 1), int(L["row_token"][r]))
            for r in range(L["n_rows"])] == pairs
    # every slot points at the row of its (t, p[e]) pair, whose mask has its bit
    where = {pr: i for i, pr in enumerate(pairs)}
    for t in range(T):
        for j in range(k):
            r = L["row_of_slot"][t, j]
            assert r == where[(int(p[idx[t, j]]), t)]
            assert (L["row_mask"][r] >> j) & 1
    for r, (d, t) in enumerate(pairs):
        want = sum(1 << j for j in range(k) if p[idx[t, j]] == d)
        assert L["row_mask"][r] == want


def test_conventional_offsets_and_masks():
    T, E, k, R = 256, 16, 3, 4
    idx = _routes(T, E, k, seed=7)
    p = np.random.default_rng(9).permutation(_contig(E, R)).astype(np.int32)
    L = oracle.dispatch_layout(idx, E, R, p, 0)
    assert L["n_rows"] == T * k
    assert np.array_equal(L["row_of_slot"], L["assign_row"])
    # row r carries exactly one slot; its expert, read back through the mask
    rows_expert = np.array([idx[L["row_token"][r], int(L["row_mask"][r]).bit_length() - 1]
                            for r in range(T * k)])
    assert all(bin(int(m)).count("1") == 1 for m in L["row_mask"])
    for e in range(E):
        got = np.nonzero(rows_expert == e)[0]
        if len(got):
            assert L["expert_offsets"][e] == got[0]
            assert len(got) == L["expert_counts"][e]
    assert L["expert_offsets"][E] == T * k
    # row destinations follow rank_offsets
    for d in range(R):
        assert np.all(p[rows_expert[L["rank_offsets"][d]:L["rank_offsets"][d + 1]]] == d)


def _expected_distinct(E, R, k):
    n = E // R
    q1 = math.comb(E - n, k) / math.comb(E, k)
    q2 = math.comb(E - 2 * n, k) / math.comb(E, k) if E - 2 * n >= 0 else 0.0
    mean = R * (1 - q1)
    second = R * (1 - q1) + R * (R - 1) * (1 - 2 * q1 + q2)
    return mean, second - mean * mean


def test_table1_contiguous_rows_closed_form():
    # Uniformly random routing under contiguous placement reproduces the
    # contiguous rows of Table I; this pins what "Same GPU", "GPUs" and
    # "Dedup" mean.  The page's router is trained, so allow half a printed unit
    # plus a little.
    g = json.load(open(os.path.join(GOLDEN, "table1_contiguous.json")))
    E = g["E"]
    for row in g["top2"]:
        R = row["ep"]
        mean, _ = _expected_distinct(E, R, 2)
        same = 100.0 * (E // R - 1) / (E - 1)
        dedup = 100.0 * (1 - mean / 2)
        assert abs(same - row["same_gpu_pct"]) <= 0.6
        assert abs(mean - row["gpus_per_token"]) <= 0.011
        assert abs(dedup - row["dedup_pct"]) <= 0.6
        assert abs(mean - (2 - same / 100.0)) < 1e-12
    for row in g["top6"]:
        mean, _ = _expected_distinct(E, row["ep"], 6)
        assert abs(100.0 * (1 - mean / 6) - row["dedup_pct"]) <= 0.6


@pytest.mark.parametrize("E,k,R", [(128, 2, 8), (128, 2, 16), (128, 2, 32), (128, 6, 8),
                                   (64, 6, 16), (128, 8, 16)])
def test_dedup_rows_match_closed_form(E, k, R):
    # the oracle's dedup row count on iid logits agrees with
    # E[D] = R (1 - C(E - E/R, k) / C(E, k)) within 5 sigma
    T = 16384
    idx = _routes(T, E, k, seed=11)
    L = oracle.dispatch_layout(idx, E, R, _contig(E, R), 1)
    mean, var = _expected_distinct(E, R, k)
    got = L["n_rows"] / T
    assert abs(got - mean) <= 5 * math.sqrt(var / T)


def test_dodoco_row_sum_rule():
    g = json.load(open(os.path.join(GOLDEN, "dodoco_models.json")))
    R, Tr = g["ranks"], g["tokens_per_rank"]
    for m in g["models"][:3]:
        E, k = m["experts"], m["top_k"]
        idx = _routes(R * Tr, E, k, seed=13, gen="groups")
        S = oracle.dispatch_layout(idx, E, R, _contig(E, R), 0)["send_counts"]
        assert np.all(S.sum(1) == Tr * k)


def test_empty_and_degenerate():
    E, k = 8, 2
    L = oracle.dispatch_layout(np.zeros((0, k), np.int32), E, 2, _contig(E, 2), 1)
    assert L["n_rows"] == 0 and L["send_counts"].sum() == 0
    # one rank: dedup leaves one row per token
    idx = _routes(64, E, k, seed=1)
    L = oracle.dispatch_layout(idx, E, 1, np.zeros(E, np.int32), 1)
    assert L["n_rows"] == 64 and np.all(L["row_mask"] == 3)
    # one expert per rank: dedup removes nothing
    L1 = oracle.dispatch_layout(idx, E, E, np.arange(E, dtype=np.int32), 1)
    L0 = oracle.dispatch_layout(idx, E, E, np.arange(E, dtype=np.int32), 0)
    assert L1["n_rows"] == L0["n_rows"] == 64 * k
    assert np.array_equal(L1["send_counts"], L0["send_counts"])
