"""md_coselect_pair_stats and md_token_shuffle_pair on the GPU against the
oracle: all integer outputs bit-exact."""
import numpy as np
import pytest
import torch

import combine_warp_top_router_b200 as md
import oracle
from combine_warp_top_router_b200 import synth

from _util import DEV, i32, shuffled_placement, u32

pytestmark = pytest.mark.gpu


def _three_layer(T, seed=0):
    w = synth.make_workload("three_layer_e128_k6", seed=seed, T=T, with_rows=False)
    k = w.k
    a, b, c = (oracle.route_topk(l.numpy(), k)[0] for l in (w.logits_prev, w.logits, w.logits_next))
    return w, a, b, c


def _gpu_shuffle(a, b, C, C2, p, R, min_obs):
    t32 = lambda m: torch.from_numpy(np.ascontiguousarray(m).view(np.int32)).to(DEV)
    st = md.new_status(DEV)
    out = md.md_token_shuffle_pair(i32(a), i32(b), t32(C), t32(C2), i32(p), R, min_obs,
                                   dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == md.MD_OK
    return [o.cpu().numpy() for o in out]


@pytest.mark.parametrize("T,T_fit", [(8192, 4096), (16 * 37, 16 * 37)])
def test_pair_counts_match_oracle(T, T_fit):
    w, a, b, c = _three_layer(T)
    C2 = md.md_coselect_pair_stats(i32(a), i32(b), i32(c), w.E, T_fit=T_fit)
    torch.cuda.synchronize()
    assert np.array_equal(u32(C2), oracle.coselect_pair(a, b, c, w.E, T_fit=T_fit))


def test_pair_counts_accumulate():
    w, a, b, c = _three_layer(2048)
    C2 = md.md_coselect_pair_stats(i32(a[:700]), i32(b[:700]), i32(c[:700]), w.E)
    md.md_coselect_pair_stats(i32(a[700:]), i32(b[700:]), i32(c[700:]), w.E, C2=C2, accumulate=True)
    torch.cuda.synchronize()
    assert np.array_equal(u32(C2), oracle.coselect_pair(a, b, c, w.E))


@pytest.mark.parametrize("T,R,min_obs", [(8192, 16, 48), (8192, 16, 1), (8192, 4, 200),
                                         (16 * 37, 16, 24), (4096, 16, 10 ** 9)])
def test_pair_shuffle_matches_oracle(T, R, min_obs):
    w, a, b, c = _three_layer(T)
    C2 = oracle.coselect_pair(a, b, c, w.E, T_fit=min(T, 4096))
    _, C = oracle.coselect(b, c, w.E, T_fit=min(T, 4096))
    C[7, :] = 0                       # an empty single row
    p = shuffled_placement(w.E, R, 4)
    got = _gpu_shuffle(a, b, C, C2, p, R, min_obs)
    want = oracle.token_shuffle_pair(a, b, C, C2, p, R, min_obs)
    for g, o in zip(got, want):
        assert np.array_equal(g, o)


# counts skewed toward a few ranks so that ranks fill in the middle of chunks;
# E = 256 is the largest pair table
@pytest.mark.parametrize("E,k,R,T,min_obs", [(64, 2, 64, 64 * 40, 3), (256, 4, 64, 64 * 64, 8),
                                             (32, 1, 4, 4 * 1000, 2)])
def test_pair_shuffle_skewed(E, k, R, T, min_obs):
    rng = np.random.default_rng(E + R)
    a, b, c = (oracle.route_topk(synth.normal_f32(T, E, s, 7).numpy(), k)[0] for s in (1, 2, 3))
    C2 = oracle.coselect_pair(a, b, c, E)
    hot = rng.choice(E, size=max(1, E // 16), replace=False)
    C2[:, :, hot] += 5                # pull many pair rows toward the same ranks
    C = rng.integers(0, 3, size=(E, E)).astype(np.uint32)
    C[:, hot] += 40
    C[rng.choice(E, size=max(1, E // 10), replace=False), :] = 0
    p = shuffled_placement(E, R, 9)
    got = _gpu_shuffle(a, b, C, C2, p, R, min_obs)
    want = oracle.token_shuffle_pair(a, b, C, C2, p, R, min_obs)
    for g, o in zip(got, want):
        assert np.array_equal(g, o)


def test_pair_shuffle_reports_bad_experts():
    w, a, b, c = _three_layer(512)
    C2 = oracle.coselect_pair(a, b, c, w.E)
    _, C = oracle.coselect(b, c, w.E)
    bad = a.copy()
    bad[3, 0] = w.E + 1
    t32 = lambda m: torch.from_numpy(np.ascontiguousarray(m).view(np.int32)).to(DEV)
    st = md.new_status(DEV)
    md.md_token_shuffle_pair(i32(bad), i32(b), t32(C), t32(C2), w.expert_to_rank.to(DEV), w.R, 8,
                             dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == md.MD_ERR_DATA


def test_pair_shuffle_full_size():
    # three-layer workload at full size: T=65536, E=128, k=6, R=16, counts
    # fitted on the first 4096 tokens; the oracle runs its own chain
    w = synth.make_workload("three_layer_e128_k6", device=DEV, with_rows=False)
    g = [md.md_route_topk(l, w.k)[0] for l in (w.logits_prev, w.logits, w.logits_next)]
    C2 = md.md_coselect_pair_stats(g[0], g[1], g[2], w.E, T_fit=4096)
    _, C = md.md_coselect_stats(g[1], g[2], w.E, T_fit=4096, want_W=False)
    pred, perm, inv, use = md.md_token_shuffle_pair(g[0], g[1], C, C2, w.expert_to_rank, w.R, 8 * w.k)
    torch.cuda.synchronize()
    o = [oracle.route_topk(l.cpu().numpy(), w.k)[0] for l in (w.logits_prev, w.logits, w.logits_next)]
    for gi, oi in zip(g, o):
        assert np.array_equal(gi.cpu().numpy(), oi)
    oC2 = oracle.coselect_pair(o[0], o[1], o[2], w.E, T_fit=4096)
    _, oC = oracle.coselect(o[1], o[2], w.E, T_fit=4096)
    assert np.array_equal(u32(C2), oC2) and np.array_equal(u32(C), oC)
    want = oracle.token_shuffle_pair(o[0], o[1], oC, oC2, w.expert_to_rank.cpu().numpy(), w.R, 8 * w.k)
    for gv, ov in zip((pred, perm, inv, use), want):
        assert np.array_equal(gv.cpu().numpy(), ov)


# Row totals up to 2^b: the visit order's sort keys then need 2b+2 bits, so the
# cases run one (all rows empty) to six radix passes; every
# confidence is distinct at high precision, so a dropped pass or a wrong shift
# changes the order.
@pytest.mark.parametrize("bits", [0, 8, 15, 18, 22, 30])
def test_pair_shuffle_wide_keys(bits):
    E, k, R, T, min_obs = 64, 2, 16, 16 * 160, 1
    rng = np.random.default_rng(100 + bits)
    a, b, _ = (oracle.route_topk(synth.normal_f32(T, E, s, 11).numpy(), k)[0] for s in (4, 5, 6))
    if bits == 0:
        C2 = np.zeros((E, E, E), dtype=np.uint32)
        C = np.zeros((E, E), dtype=np.uint32)
    else:
        top = 1 << max(0, bits - 6)  # 64 entries per row: totals below 2^bits
        C2 = rng.integers(0, top, size=(E, E, E), dtype=np.uint64).astype(np.uint32)
        C = rng.integers(0, top, size=(E, E), dtype=np.uint64).astype(np.uint32)
        C2[:, :, 0] = top - 1         # no empty pair rows at the top of the range
        C2[rng.choice(E, size=8, replace=False), :, :] = 0  # some tokens fall back to C
    p = shuffled_placement(E, R, 5)
    got = _gpu_shuffle(a, b, C, C2, p, R, min_obs)
    want = oracle.token_shuffle_pair(a, b, C, C2, p, R, min_obs)
    for g, o in zip(got, want):
        assert np.array_equal(g, o)
