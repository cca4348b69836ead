"""md_route_topk on the GPU against the oracle.

Expert indices must match bit for bit; gate weights within 1e-6 relative."""
import numpy as np
import pytest
import torch

import combine_warp_top_router_b200 as md
import oracle
from combine_warp_top_router_b200 import synth

from _util import DEV

pytestmark = pytest.mark.gpu


def _run(lg_np, k, mode):
    lg = torch.from_numpy(np.ascontiguousarray(lg_np, np.float32)).to(DEV)
    idx, w = md.md_route_topk(lg, k, mode)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), w.cpu().numpy()


def _compare(lg_np, k, mode):
    gi, gw = _run(lg_np, k, mode)
    oi, ow = oracle.route_topk(lg_np, k, mode)
    assert np.array_equal(gi, oi)
    rel = np.abs(gw.astype(np.float64) - ow) / np.maximum(np.abs(ow.astype(np.float64)), 1e-300)
    assert rel.max() <= 1e-6, rel.max()
    return gi, gw


@pytest.mark.parametrize("E,k,T", [(64, 6, 4096), (128, 8, 1000), (128, 2, 777), (256, 8, 3000),
                                   (40, 5, 300), (384, 8, 257), (1024, 32, 64), (8, 8, 50),
                                   (1, 1, 33), (96, 3, 129)])
@pytest.mark.parametrize("mode", [0, 1])
def test_iid_shapes(E, k, T, mode):
    lg = synth.normal_f32(T, E, 7, 1).numpy() * 2.0
    _compare(lg, k, mode)


@pytest.mark.parametrize("name", ["iid_e64_k6", "zipf_pairs_e128_k8", "boost_pairs_e128_k2",
                                  "full_e256_k8"])
def test_workload_logits(name):
    w = synth.make_workload(name, T=4096 if name != "full_e256_k8" else 8192, with_rows=False)
    _compare(w.logits.numpy(), synth.SPECS[name]["k"], 0)


@pytest.mark.parametrize("E", [16, 128, 256])
def test_ties_and_signed_zero(E):
    rng = np.random.default_rng(E)
    lg = rng.integers(-2, 3, size=(512, E)).astype(np.float32)
    lg[rng.random(lg.shape) < 0.2] = -0.0
    lg[rng.random(lg.shape) < 0.05] = -np.inf
    lg[0] = 0.0
    lg[0, ::2] = -0.0
    for k in (1, 4, min(E, 32)):
        _compare(lg, k, 0)


@pytest.mark.parametrize("E", [64, 128, 256])
@pytest.mark.parametrize("k", [1, 2, 4, 6, 8])
def test_per_token_kernel_ties_and_many_candidates(E, k):
    # E in {64, 128, 256} with k <= 8 takes the one-thread-per-token kernel.
    # Integer logits tie heavily, so many tokens have far more than 16
    # candidates at or above the threshold (several batches of 8); rows of
    # equal logits leave every element a candidate.  T = 32*13 + 7 leaves a
    # ragged last warp.
    rng = np.random.default_rng(100 * E + k)
    T = 32 * 13 + 7
    lg = rng.integers(-3, 2, size=(T, E)).astype(np.float32)
    lg[rng.random(lg.shape) < 0.1] = -0.0
    lg[1] = 1.0
    lg[2] = -np.inf
    lg[2, E - 1] = 0.0
    lg[3] = rng.standard_normal(E).astype(np.float32)
    for mode in (0, 1):
        _compare(lg, k, mode)


@pytest.mark.parametrize("E,k", [(128, 8), (64, 6), (256, 4)])
def test_per_token_kernel_unaligned_outputs(E, k):
    T = 100
    lg_np = synth.normal_f32(T, E, 5, 1).numpy()
    lg = torch.from_numpy(lg_np).to(DEV)
    raw_i = torch.full((T * k + 1,), -9, dtype=torch.int32, device=DEV)
    raw_w = torch.full((T * k + 1,), -9.0, dtype=torch.float32, device=DEV)
    idx, w = md.md_route_topk(lg, k, 0, topk_idx=raw_i[1:].view(T, k),
                            topk_w=raw_w[1:].view(T, k))
    torch.cuda.synchronize()
    oi, ow = oracle.route_topk(lg_np, k, 0)
    assert np.array_equal(idx.cpu().numpy(), oi)
    assert np.allclose(w.cpu().numpy(), ow, rtol=1e-6, atol=0)
    assert int(raw_i[0].item()) == -9 and float(raw_w[0].item()) == -9.0


def test_k1_gate_is_one_and_empty_batch():
    lg = synth.normal_f32(100, 64, 3, 1).numpy()
    _, w = _compare(lg, 1, 0)
    assert np.all(w == 1.0)
    idx, w = md.md_route_topk(torch.empty(0, 64, device=DEV), 4)
    assert idx.shape == (0, 4)


def test_full_size_sampled():
    # the benchmark's router shape: T=65536, E=128, k=8; every row checked
    w = synth.make_workload("zipf_pairs_e128_k8", device=DEV, with_rows=False)
    idx, gw = md.md_route_topk(w.logits, 8)
    torch.cuda.synchronize()
    rows = np.random.default_rng(0).choice(w.T, 4096, replace=False)
    lg = w.logits.cpu().numpy()
    oi, ow = oracle.route_topk(lg[rows], 8)
    assert np.array_equal(idx.cpu().numpy()[rows], oi)
    assert np.allclose(gw.cpu().numpy()[rows], ow, rtol=1e-6, atol=0)


@pytest.mark.parametrize("E,k", [(128, 8), (64, 6), (256, 2), (40, 5)])
def test_nan_rows_give_valid_distinct_experts(E, k):
    # NaN logits are outside the contract; the router must still return k
    # distinct experts in [0, E) for every token, and the same ones each time
    rng = np.random.default_rng(E + k)
    T = 96
    lg = rng.standard_normal((T, E)).astype(np.float32)
    lg[0] = np.nan                                  # all NaN
    lg[1, : E - k + 1] = np.nan                     # fewer than k numbers
    lg[2, ::3] = np.nan                             # scattered NaN
    lg[3] = -np.nan
    gi, _ = _run(lg, k, 0)
    gi2, _ = _run(lg, k, 0)
    assert np.array_equal(gi, gi2)
    assert gi.min() >= 0 and gi.max() < E
    assert all(len(set(r)) == k for r in gi.tolist())
    # rows without NaN are unaffected
    oi, _ = oracle.route_topk(lg[4:], k, 0)
    assert np.array_equal(gi[4:], oi)


@pytest.mark.parametrize("E,k", [(64, 6), (128, 8), (256, 8), (256, 2)])
def test_bounded_tile_wait_fallback_is_exact(E, k):
    # The per-token kernel stages each 32-row tile with one bulk copy and a
    # bounded wait; when the bound runs out it copies the same bytes with
    # plain loads.  A poll limit of 1 makes that path likely; either way the
    # result must be the oracle's.
    lg = synth.normal_f32(4096 + 17, E, E + k, 1).numpy()
    md.md_set_test_hooks(poll_limit=1)
    try:
        _compare(lg, k, 0)
    finally:
        md.md_set_test_hooks()
    _compare(lg, k, 1)
