"""md_rank_stats, md_successor_share and md_count_sums on the GPU against the
oracle: counts bit-exact, derived ratios equal."""
import numpy as np
import pytest
import torch

import combine_warp_top_router_b200 as md
import oracle
from combine_warp_top_router_b200 import synth

from _util import DEV, i32, shuffled_placement, u32

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,R", [("zipf_pairs_e128_k8", 16), ("boost_pairs_e128_k2", 32),
                                    ("iid_e64_k6", 64), ("full_e256_k8", 64)])
@pytest.mark.parametrize("pl", ["contiguous", "shuffled"])
def test_rank_stats_match_oracle(name, R, pl):
    w = synth.make_workload(name, T=8192 if name != "iid_e64_k6" else 4096, R=R, with_rows=False)
    idx = oracle.route_topk(w.logits.numpy(), w.k)[0]
    p = synth.contiguous_placement(w.E, R).numpy() if pl == "contiguous" else shuffled_placement(w.E, R, 2)
    hist = md.md_rank_stats(i32(idx), w.E, R, i32(p))
    torch.cuda.synchronize()
    want = oracle.rank_stats(idx, w.E, R, p)
    assert np.array_equal(hist.cpu().numpy(), want)


def test_rank_stats_report_bad_experts_and_empty():
    idx = np.zeros((10, 2), np.int32)
    idx[:, 1] = 1
    idx[4, 1] = 99
    st = md.new_status(DEV)
    md.md_rank_stats(i32(idx), 8, 2, i32(np.array([0, 0, 0, 0, 1, 1, 1, 1], np.int32)), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == md.MD_ERR_DATA
    h = md.md_rank_stats(i32(np.zeros((0, 3), np.int32)), 8, 2, i32(np.zeros(8, np.int32)))
    torch.cuda.synchronize()
    assert h.cpu().tolist() == [0, 0, 0, 0]


@pytest.mark.parametrize("name", ["two_layer_e128_k6", "full_e256_k8"])
def test_successor_share_matches_oracle(name):
    w = synth.make_workload(name, T=8192, with_rows=False)
    a = oracle.route_topk(w.logits.numpy(), w.k)[0]
    b = oracle.route_topk(w.logits_next.numpy(), w.k)[0]
    W, C = oracle.coselect(a, b, w.E)
    t32 = lambda m: torch.from_numpy(np.ascontiguousarray(m).view(np.int32)).to(DEV)
    num, den = md.md_successor_share(t32(C), t32(W))
    torch.cuda.synchronize()
    onum, oden = oracle.successor_share(C, W)
    assert np.array_equal(u32(num), onum) and np.array_equal(u32(den), oden)


@pytest.mark.parametrize("n,hi", [(128 * 128, 5000), (256 * 256, 2 ** 32 - 1), (1, 7), (1000, 1)])
def test_count_sums_match_oracle(n, hi):
    rng = np.random.default_rng(n)
    x = rng.integers(0, hi, n, dtype=np.uint64).astype(np.uint32)
    y = rng.integers(0, hi, n, dtype=np.uint64).astype(np.uint32)
    t32 = lambda m: torch.from_numpy(m.view(np.int32)).to(DEV)
    got = md.md_count_sums(t32(x), t32(y))
    want = oracle.count_sums(x, y)
    assert got == want
    if n > 1 and hi > 1:
        assert md.pearson_from_sums(n, got) == pytest.approx(oracle.pearson(x, y), rel=1e-15)


def test_fitted_vs_held_out_correlation_full_size():
    # the pages' stability statistic on the full-pipeline workload: W fitted
    # on the first 4096 tokens against W on the next 4096
    w = synth.make_workload("full_e256_k8", device=DEV, with_rows=False)
    idx, _ = md.md_route_topk(w.logits, 8)
    W1, _ = md.md_coselect_stats(idx[:4096], None, 256)
    W2, _ = md.md_coselect_stats(idx[4096:8192], None, 256)
    got = md.md_count_sums(W1, W2)
    torch.cuda.synchronize()
    oi = oracle.route_topk(w.logits[:8192].cpu().numpy(), 8)[0]
    assert np.array_equal(idx[:8192].cpu().numpy(), oi)
    oW1, _ = oracle.coselect(oi[:4096], None, 256)
    oW2, _ = oracle.coselect(oi[4096:], None, 256)
    assert got == oracle.count_sums(oW1, oW2)
