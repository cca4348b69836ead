"""md_coselect_stats, md_place_correlated and md_token_shuffle on the GPU
against the oracle: all integer outputs bit-exact."""
import numpy as np
import pytest
import torch

import combine_warp_top_router_b200 as md
import oracle
from combine_warp_top_router_b200 import synth

from _util import DEV, i32, shuffled_placement, u32

pytestmark = pytest.mark.gpu


def _two_layer(name, T, seed=0):
    w = synth.make_workload(name, seed=seed, T=T, with_rows=False)
    k = w.k
    a = oracle.route_topk(w.logits.numpy(), k)[0]
    nxt = w.logits_next if w.logits_next is not None else synth.normal_f32(T, w.E, seed, 99)
    b = oracle.route_topk(nxt.numpy(), k)[0]
    return w, a, b


@pytest.mark.parametrize("name,T,T_fit", [("two_layer_e128_k6", 8192, 4096),
                                          ("boost_pairs_e128_k2", 8192, 4096),
                                          ("full_e256_k8", 16384, 16384),
                                          ("iid_e64_k6", 4096, 1000)])
def test_coselect_matches_oracle(name, T, T_fit):
    w, a, b = _two_layer(name, T)
    W, C = md.md_coselect_stats(i32(a), i32(b), w.E, T_fit=T_fit)
    torch.cuda.synchronize()
    oW, oC = oracle.coselect(a, b, w.E, T_fit=T_fit)
    assert np.array_equal(u32(W), oW)
    assert np.array_equal(u32(C), oC)


def test_coselect_accumulate_and_single_table():
    w, a, b = _two_layer("iid_e64_k6", 2048)
    W, C = md.md_coselect_stats(i32(a[:1000]), i32(b[:1000]), 64)
    md.md_coselect_stats(i32(a[1000:]), i32(b[1000:]), 64, W=W, C=C, accumulate=True)
    W2, _ = md.md_coselect_stats(i32(a), None, 64)
    torch.cuda.synchronize()
    oW, oC = oracle.coselect(a, b, 64)
    assert np.array_equal(u32(W), oW) and np.array_equal(u32(C), oC)
    assert np.array_equal(u32(W2), oW)


def test_coselect_full_size():
    # full-pipeline workload: W and C over all T=262144 tokens, E=256, k=8
    w = synth.make_workload("full_e256_k8", device=DEV, with_rows=False)
    a, _ = md.md_route_topk(w.logits, 8)
    b, _ = md.md_route_topk(w.logits_next, 8)
    W, C = md.md_coselect_stats(a, b, 256)
    torch.cuda.synchronize()
    oa = oracle.route_topk(w.logits.cpu().numpy(), 8)[0]
    ob = oracle.route_topk(w.logits_next.cpu().numpy(), 8)[0]
    assert np.array_equal(a.cpu().numpy(), oa) and np.array_equal(b.cpu().numpy(), ob)
    oW, oC = oracle.coselect(oa, ob, 256)
    assert np.array_equal(u32(W), oW)
    assert np.array_equal(u32(C), oC)


@pytest.mark.parametrize("name,T,R", [("boost_pairs_e128_k2", 4096, 8), ("boost_pairs_e128_k2", 4096, 32),
                                      ("full_e256_k8", 16384, 64), ("iid_e64_k6", 2048, 16),
                                      ("two_layer_e128_k6", 4096, 16)])
@pytest.mark.parametrize("seed_mode", [0, 1])
def test_placement_matches_oracle(name, T, R, seed_mode):
    w, a, _ = _two_layer(name, T)
    oW, _ = oracle.coselect(a, None, w.E)
    p = md.md_place_correlated(torch.from_numpy(oW.view(np.int32)).to(DEV), R, seed_mode)
    torch.cuda.synchronize()
    want = oracle.place_correlated(oW, R, seed_mode)
    assert np.array_equal(p.cpu().numpy(), want)


def test_placement_small_and_unrefined():
    W = np.zeros((6, 6), np.uint32)
    for (x, y, v) in [(0, 5, 9), (1, 4, 7), (0, 1, 5), (2, 3, 1)]:
        W[x, y] = W[y, x] = v
    Wd = torch.from_numpy(W.view(np.int32)).to(DEV)
    for seed_mode in (0, 1):
        for refine in (False, True):
            p = md.md_place_correlated(Wd, 3, seed_mode, refine)
            torch.cuda.synchronize()
            assert np.array_equal(p.cpu().numpy(), oracle.place_correlated(W, 3, seed_mode, refine))


def _random_w(E, seed, hi):
    rng = np.random.default_rng(seed)
    W = np.triu(rng.integers(0, hi, size=(E, E)), 1).astype(np.uint32)
    W = W + W.T
    W[np.arange(E), np.arange(E)] = rng.integers(0, 4 * hi, size=E).astype(np.uint32)
    return W


# small value ranges force many equal weights and gains (tie rules); E=1024
# covers the largest tables, R=16 keeps A (E x R) in shared memory and R=64
# puts it in the workspace; E/R=1 and R=1 leave nothing to swap
@pytest.mark.parametrize("E,R,hi", [(8, 2, 3), (16, 4, 2), (64, 64, 5), (64, 8, 1000),
                                    (256, 2, 7), (256, 64, 4), (1024, 16, 9), (1024, 64, 50),
                                    (128, 1, 5)])
@pytest.mark.parametrize("seed_mode", [0, 1])
def test_placement_random_weights(E, R, hi, seed_mode):
    W = _random_w(E, E * 7 + R, hi)
    p = md.md_place_correlated(torch.from_numpy(W.view(np.int32)).to(DEV), R, seed_mode)
    torch.cuda.synchronize()
    want = oracle.place_correlated(W, R, seed_mode)
    assert np.array_equal(p.cpu().numpy(), want)


def _shuffle_both(a, C, p, R):
    pred, perm, inv = md.md_token_shuffle(i32(a), torch.from_numpy(C.view(np.int32)).to(DEV), i32(p), R)
    torch.cuda.synchronize()
    want = oracle.token_shuffle(a, C, p, R)
    return (pred.cpu().numpy(), perm.cpu().numpy(), inv.cpu().numpy()), want


@pytest.mark.parametrize("name,T,R", [("two_layer_e128_k6", 8192, 16), ("two_layer_e128_k6", 4096, 4),
                                      ("full_e256_k8", 8192, 64), ("iid_e64_k6", 16 * 37, 16)])
def test_shuffle_matches_oracle(name, T, R):
    w, a, b = _two_layer(name, T)
    _, C = oracle.coselect(a, b, w.E, T_fit=min(T, 4096))
    C[5, :] = 0  # an empty row
    p = shuffled_placement(w.E, R, 4)
    got, want = _shuffle_both(a, C, p, R)
    for g, o in zip(got, want):
        assert np.array_equal(g, o)


# counts skewed toward a few ranks, so that ranks fill one after another in
# the middle of chunks and most tokens fall back down their preference lists
@pytest.mark.parametrize("E,k,R,T", [(64, 2, 64, 64 * 40), (128, 6, 16, 16 * 700), (1024, 8, 64, 64 * 80),
                                     (32, 1, 4, 4 * 1000), (16, 3, 2, 2 * 2500)])
def test_shuffle_skewed_counts(E, k, R, T):
    rng = np.random.default_rng(E + R)
    C = rng.integers(0, 3, size=(E, E)).astype(np.uint32)
    hot = rng.choice(E, size=max(1, E // 16), replace=False)
    C[:, hot] += 40
    C[rng.choice(E, size=max(1, E // 10), replace=False), :] = 0  # empty rows
    a = oracle.route_topk(synth.normal_f32(T, E, 3, 7).numpy(), k)[0]
    p = shuffled_placement(E, R, 9)
    got, want = _shuffle_both(a, C, p, R)
    for g, o in zip(got, want):
        assert np.array_equal(g, o)


def test_shuffle_hand_cases():
    C = np.array([[0, 0, 3, 1], [2, 0, 0, 0], [0, 0, 0, 0], [0, 1, 0, 1]], np.uint32)
    p = np.array([0, 0, 1, 1], np.int32)
    a = np.array([[0, 1], [3, 0], [0, 2], [2, 3]], np.int32)
    got, want = _shuffle_both(a, C, p, 2)
    assert got[0].tolist() == [1, 0, 1, 0] and got[1].tolist() == [2, 0, 3, 1]
    C2 = np.zeros((4, 4), np.uint32)
    C2[0, 2] = 5
    a2 = np.array([[0, 3]] * 2 + [[1, 3]] * 6, np.int32)
    got, _ = _shuffle_both(a2, C2, p, 2)
    assert got[0].tolist() == [1, 1, 0, 0, 1, 1, 0, 0]
    # no counts at all: nobody moves
    got, _ = _shuffle_both(a2, np.zeros((4, 4), np.uint32), p, 2)
    assert got[1].tolist() == list(range(8))


def test_shuffle_full_size_and_gather_round_trip():
    # two-layer workload at full size: T=65536, E=128, k=6, R=16, C fitted on
    # the first 4096 tokens; then the shuffled rows go back with perm
    w = synth.make_workload("two_layer_e128_k6", device=DEV)
    a, _ = md.md_route_topk(w.logits, 6)
    b, _ = md.md_route_topk(w.logits_next, 6)
    _, C = md.md_coselect_stats(a, b, 128, T_fit=4096, want_W=False)
    pred, perm, inv = md.md_token_shuffle(a, C, w.expert_to_rank, 16)
    xs = md.md_gather_rows(w.x, inv)
    back = md.md_gather_rows(xs, perm)
    torch.cuda.synchronize()
    # the oracle runs its own chain from the same logits
    oa = oracle.route_topk(w.logits.cpu().numpy(), 6)[0]
    ob = oracle.route_topk(w.logits_next.cpu().numpy(), 6)[0]
    _, oC = oracle.coselect(oa, ob, 128, T_fit=4096)
    assert np.array_equal(u32(C), oC)
    want = oracle.token_shuffle(oa, oC, w.expert_to_rank.cpu().numpy(), 16)
    assert np.array_equal(pred.cpu().numpy(), want[0])
    assert np.array_equal(perm.cpu().numpy(), want[1])
    assert np.array_equal(inv.cpu().numpy(), want[2])
    assert torch.equal(back, w.x)  # shuffle then restore is the identity


# ------------------------------------------------- KL passes and two levels
@pytest.mark.parametrize("E,R,nodes,hi", [(8, 2, 1, 4), (64, 8, 1, 1000), (128, 16, 1, 5),
                                          (256, 64, 1, 4), (128, 16, 4, 9), (256, 64, 8, 50),
                                          (64, 8, 8, 7), (1024, 64, 8, 9)])
@pytest.mark.parametrize("refine_mode", [0, 1, 2])
@pytest.mark.parametrize("seed_mode", [0, 1])
def test_place_two_level_matches_oracle(E, R, nodes, hi, refine_mode, seed_mode):
    if E == 1024 and refine_mode == 2 and seed_mode == 1:
        pytest.skip("covered by the contiguous seed at this size (oracle minutes)")
    W = _random_w(E, E * 3 + R + nodes, hi)
    p = md.md_place_two_level(torch.from_numpy(W.view(np.int32)).to(DEV), R, nodes, seed_mode,
                              refine_mode)
    torch.cuda.synchronize()
    want = oracle.place_two_level(W, R, nodes, seed_mode, refine_mode)
    assert np.array_equal(p.cpu().numpy(), want)


def test_kl_escapes_where_swaps_stop():
    # the 8-expert instance from the oracle pins: KL reaches the optimum 24
    from test_oracle_placement_kl import W_STUCK
    Wd = torch.from_numpy(W_STUCK.view(np.int32)).to(DEV)
    sw = md.md_place_two_level(Wd, 2, 1, 0, md.MD_REFINE_SWAPS)
    kl = md.md_place_two_level(Wd, 2, 1, 0, md.MD_REFINE_KL)
    torch.cuda.synchronize()
    assert oracle.placement_objective(W_STUCK, sw.cpu().numpy()) == 22
    assert oracle.placement_objective(W_STUCK, kl.cpu().numpy()) == 24


@pytest.mark.parametrize("nodes", [1, 8])
@pytest.mark.parametrize("refine_mode", [1, 2])
def test_place_two_level_full_workload(nodes, refine_mode):
    # full-pipeline workload: W over all T=262144 tokens, E=256, R=64
    w = synth.make_workload("full_e256_k8", device=DEV, with_rows=False)
    a, _ = md.md_route_topk(w.logits, 8)
    W, _ = md.md_coselect_stats(a, None, 256)
    p = md.md_place_two_level(W, 64, nodes, 0, refine_mode)
    torch.cuda.synchronize()
    want = oracle.place_two_level(u32(W), 64, nodes, 0, refine_mode)
    assert np.array_equal(p.cpu().numpy(), want)


# The search keeps W and A in shared memory (uint16 / int32) when W is
# symmetric with entries below 2^16; otherwise it reads W from global memory.
# Both paths must give the oracle's placements.
@pytest.mark.parametrize("kind", ["large_values", "asymmetric", "large_diagonal"])
@pytest.mark.parametrize("refine_mode", [1, 2])
@pytest.mark.parametrize("seed_mode", [0, 1])
def test_placement_outside_the_compact_path(kind, refine_mode, seed_mode):
    E, R = 64, 8
    rng = np.random.default_rng(17)
    if kind == "large_values":
        W = _random_w(E, 5, 200_000)
    elif kind == "asymmetric":
        W = rng.integers(0, 50, (E, E)).astype(np.uint32)
    else:
        W = _random_w(E, 6, 30)
        W[np.arange(E), np.arange(E)] = 70_000   # only the diagonal is too large
    p = md.md_place_two_level(torch.from_numpy(W.view(np.int32)).to(DEV), R, 1, seed_mode,
                              refine_mode)
    torch.cuda.synchronize()
    assert np.array_equal(p.cpu().numpy(), oracle.place_two_level(W, R, 1, seed_mode, refine_mode))


# ------------------------------------------------ rounds-based assignment
def _rounds_both(a, C, p, R):
    pred, perm, inv, rounds = md.md_token_shuffle_rounds(
        i32(a), torch.from_numpy(C.view(np.int32)).to(DEV), i32(p), R)
    torch.cuda.synchronize()
    return ((pred.cpu().numpy(), perm.cpu().numpy(), inv.cpu().numpy(), int(rounds.item())),
            oracle.token_shuffle_rounds(a, C, p, R))


@pytest.mark.parametrize("name,T,R", [("two_layer_e128_k6", 8192, 16), ("two_layer_e128_k6", 4096, 4),
                                      ("full_e256_k8", 8192, 64), ("iid_e64_k6", 16 * 37, 16),
                                      ("two_layer_e128_k6", 65536, 16)])
def test_rounds_match_oracle(name, T, R):
    w, a, b = _two_layer(name, T)
    _, C = oracle.coselect(a, b, w.E, T_fit=min(T, 4096))
    C[5, :] = 0
    p = shuffled_placement(w.E, R, 4)
    got, want = _rounds_both(a, C, p, R)
    for g, o in zip(got, want):
        assert np.array_equal(g, o)


@pytest.mark.parametrize("E,k,R,T", [(64, 2, 64, 64 * 40), (128, 6, 16, 16 * 700), (1024, 8, 64, 64 * 80),
                                     (32, 1, 4, 4 * 1000), (16, 3, 2, 2 * 2500)])
def test_rounds_skewed_counts(E, k, R, T):
    rng = np.random.default_rng(E + R)
    C = rng.integers(0, 3, size=(E, E)).astype(np.uint32)
    hot = rng.choice(E, size=max(1, E // 16), replace=False)
    C[:, hot] += 40
    C[rng.choice(E, size=max(1, E // 10), replace=False), :] = 0
    a = oracle.route_topk(synth.normal_f32(T, E, 3, 7).numpy(), k)[0]
    p = shuffled_placement(E, R, 9)
    got, want = _rounds_both(a, C, p, R)
    for g, o in zip(got, want):
        assert np.array_equal(g, o)


def test_rounds_hand_example():
    C = np.array([[10, 0, 0, 0], [6, 3, 1, 0], [1, 5, 4, 0], [2, 2, 0, 3]], np.uint32)
    p = np.array([0, 1, 2, 2], np.int32)
    a = np.array([[0], [0], [1], [2], [2], [3]], np.int32)
    got, want = _rounds_both(a, C, p, 3)
    assert got[0].tolist() == [0, 0, 2, 1, 1, 2] and got[3] == 2
