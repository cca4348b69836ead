"""Full-size parity of the workloads the benchmark times, in the launch
configuration it times them.

* the top-2, H=4096 workload (T=65536) at EP 8 and 32 with the placement
  fitted on tokens [0, 4096): placement, every layout output, the dispatch
  rows, the combine;
* the E=256 workload (T=262144, H=2048, R=64) with the correlated placement
  fitted on all tokens: the same, with rows of 4 KiB (the bulk-copy permute);
* the E=128, top-8 workload (T=65536, H=2048, R=16, contiguous placement) in
  both dispatch modes, with the two-stage ("wire") combine and the dedup
  expand the benchmark also times;
* the token shuffle followed by the dedup layout of the next layer in the
  shuffled order (single-expert and pair-based prediction).

Integer outputs (placements, layouts, shuffles) are compared whole with the
oracle's.  Dispatch rows are checked whole by the inverse identity
out[row_of_slot[t][j]] == x[t] (which holds at any size) and on sampled rows
against the oracle's permute; combine outputs on sampled tokens the oracle
computes one by one.  Inputs come from the seeded generator; the oracle
routes the same logits itself."""
import numpy as np
import pytest
import torch

import combine_warp_top_router_b200 as md
import oracle
from combine_warp_top_router_b200 import synth

from _util import DEV, bits, i32

pytestmark = pytest.mark.gpu


def _inverse_identity(buf, x, row_of_slot, chunk=8192):
    """Every slot's dispatch row holds its token's x row, bit for bit."""
    T, k = row_of_slot.shape
    H = x.shape[1]
    for t0 in range(0, T, chunk):
        t1 = min(T, t0 + chunk)
        got = buf[row_of_slot[t0:t1].reshape(-1).long()].view(t1 - t0, k, H)
        if not torch.equal(got.view(torch.int16),
                           x[t0:t1].unsqueeze(1).expand(t1 - t0, k, H).view(torch.int16)):
            return False
    return True


def _check_layout(L, OL):
    assert int(L.n_rows.item()) == OL["n_rows"]
    n = OL["n_rows"]
    for name in ("row_of_slot", "assign_row", "send_counts", "expert_counts", "expert_offsets",
                 "rank_offsets"):
        assert np.array_equal(getattr(L, name).cpu().numpy(), OL[name]), name
    assert np.array_equal(L.row_token[:n].cpu().numpy(), OL["row_token"])
    assert np.array_equal(L.row_mask[:n].cpu().numpy().view(np.uint32), OL["row_mask"])


def _check_rows_and_combine(w, idx, gates, L, OL, oi, ow, buf, out, n_rows_sample, n_tok_sample):
    assert _inverse_identity(buf, w.x, L.row_of_slot)
    rng = np.random.default_rng(1)
    n = OL["n_rows"]
    rows = np.sort(rng.choice(n, n_rows_sample, replace=False))
    xb = bits(w.x)
    want = oracle.dispatch_permute(xb, OL["row_token"][rows])
    assert np.array_equal(bits(buf[torch.from_numpy(rows).long().to(DEV)]), want)
    toks = np.sort(rng.choice(w.T, n_tok_sample, replace=False))
    ar = OL["assign_row"][toks]
    ysub = bits(w.y[torch.from_numpy(ar.ravel()).long().to(DEV)])
    want = oracle.combine(ysub, np.arange(ar.size, dtype=np.int32).reshape(ar.shape), oi[toks],
                          ow[toks])
    assert np.array_equal(bits(out[torch.from_numpy(toks).long().to(DEV)]), want)


@pytest.mark.parametrize("R", [8, 32])
def test_boost_pairs_top2_h4096_full_size(R):
    # T=65536, H=4096 (8 KiB rows: two bulk-copy pieces each), E=128, top-2;
    # placement from W on tokens [0, 4096), greedy pair seed then swaps
    w = synth.make_workload("boost_pairs_e128_k2", device=DEV, R=R)
    E, k = w.E, w.k
    idx, gates = md.md_route_topk(w.logits, k)
    W, _ = md.md_coselect_stats(idx, None, E, T_fit=w.fit_tokens)
    p = md.md_place_correlated(W, R, seed_mode=md.MD_SEED_GREEDY_PAIRS)
    L = md.md_dispatch_layout(idx, E, R, p, md.MD_DEDUP)
    buf = md.md_dispatch_permute(w.x, L.row_of_slot, out_rows=L.row_capacity)
    out = md.md_combine(w.y, L.assign_row, idx, gates)
    torch.cuda.synchronize()
    oi, ow = oracle.route_topk(w.logits.cpu().numpy(), k)
    assert np.array_equal(idx.cpu().numpy(), oi)
    assert np.allclose(gates.cpu().numpy(), ow, rtol=1e-6, atol=0)
    oW, _ = oracle.coselect(oi, None, E, T_fit=w.fit_tokens)
    assert np.array_equal(W.cpu().numpy().view(np.uint32), oW)
    op = oracle.place_correlated(oW, R, seed_mode=1)
    assert np.array_equal(p.cpu().numpy(), op)
    OL = oracle.dispatch_layout(oi, E, R, op, oracle.DEDUP)
    _check_layout(L, OL)
    _check_rows_and_combine(w, idx, gates, L, OL, oi, ow, buf, out, 4096, 2048)


def test_full_e256_k8_full_size():
    # T=262144, H=2048, E=256, k=8, R=64; placement from W over all tokens
    w = synth.make_workload("full_e256_k8", device=DEV)
    w.logits_next = None
    E, k, R = w.E, w.k, w.R
    idx, gates = md.md_route_topk(w.logits, k)
    W, _ = md.md_coselect_stats(idx, None, E, T_fit=w.fit_tokens)
    p = md.md_place_correlated(W, R)
    L = md.md_dispatch_layout(idx, E, R, p, md.MD_DEDUP)
    buf = md.md_dispatch_permute(w.x, L.row_of_slot, out_rows=L.row_capacity)
    out = md.md_combine(w.y, L.assign_row, idx, gates)
    torch.cuda.synchronize()
    oi, ow = oracle.route_topk(w.logits.cpu().numpy(), k)
    assert np.array_equal(idx.cpu().numpy(), oi)
    assert np.allclose(gates.cpu().numpy(), ow, rtol=1e-6, atol=0)
    oW, _ = oracle.coselect(oi, None, E)
    assert np.array_equal(W.cpu().numpy().view(np.uint32), oW)
    op = oracle.place_correlated(oW, R)
    assert np.array_equal(p.cpu().numpy(), op)
    OL = oracle.dispatch_layout(oi, E, R, op, oracle.DEDUP)
    _check_layout(L, OL)
    _check_rows_and_combine(w, idx, gates, L, OL, oi, ow, buf, out, 8192, 1024)


@pytest.mark.parametrize("mode", [0, 1])
def test_zipf_pairs_e128_k8_full_size(mode):
    # T=65536, H=2048, E=128, k=8, R=16, contiguous placement
    w = synth.make_workload("zipf_pairs_e128_k8", device=DEV)
    E, k, R = w.E, w.k, w.R
    idx, gates = md.md_route_topk(w.logits, k)
    L = md.md_dispatch_layout(idx, E, R, w.expert_to_rank, mode)
    buf = md.md_dispatch_permute(w.x, L.row_of_slot, out_rows=L.row_capacity)
    out = md.md_combine(w.y, L.assign_row, idx, gates)
    torch.cuda.synchronize()
    oi, ow = oracle.route_topk(w.logits.cpu().numpy(), k)
    assert np.array_equal(idx.cpu().numpy(), oi)
    p = w.expert_to_rank.cpu().numpy()
    OL = oracle.dispatch_layout(oi, E, R, p, mode)
    _check_layout(L, OL)
    _check_rows_and_combine(w, idx, gates, L, OL, oi, ow, buf, out, 8192, 1024)
    if mode != md.MD_DEDUP:
        return
    # the expand: every (token, expert) row holds the token's x row
    xe = md.md_dedup_expand(buf, L.row_of_slot, L.assign_row)
    torch.cuda.synchronize()
    assert _inverse_identity(xe, w.x, L.assign_row)
    del xe
    # the two-stage combine on sampled tokens: a token's stage-1 rows are its
    # own, so the oracle runs on the sample with its rows renumbered
    n = OL["n_rows"]
    z = torch.empty(n, w.H, dtype=torch.bfloat16, device=DEV)
    wire = md.md_combine(w.y, L.assign_row, idx, gates, md.MD_COMBINE_WIRE,
                         row_of_slot=L.row_of_slot, z=z)
    torch.cuda.synchronize()
    rng = np.random.default_rng(2)
    toks = np.sort(rng.choice(w.T, 1024, replace=False))
    ar = OL["assign_row"][toks]
    rs = OL["row_of_slot"][toks]
    uniq, local = np.unique(rs, return_inverse=True)
    ysub = bits(w.y[torch.from_numpy(ar.ravel()).long().to(DEV)])
    want_out, want_z = oracle.combine(ysub, np.arange(ar.size, dtype=np.int32).reshape(ar.shape),
                                      oi[toks], ow[toks], oracle.COMBINE_WIRE, p,
                                      local.reshape(rs.shape).astype(np.int32), len(uniq))
    assert np.array_equal(bits(wire[torch.from_numpy(toks).long().to(DEV)]), want_out)
    assert np.array_equal(bits(z[torch.from_numpy(uniq).long().to(DEV)]), want_z)


def _chain_gpu(idx_next, inv, E, R, p):
    ordered = md.md_gather_rows(idx_next, inv)
    return ordered, md.md_dispatch_layout(ordered, E, R, p, md.MD_DEDUP)


def test_dedup_layout_after_single_shuffle_full_size():
    # two_layer_e128_k6 (T=65536, E=128, top-6, R=16): C fitted on [0, 4096);
    # shuffle by single-expert prediction; the layer-(l+1) top-k in the
    # shuffled order; dedup layout with src = the token's new block
    w = synth.make_workload("two_layer_e128_k6", device=DEV, with_rows=False)
    E, k, R = w.E, w.k, w.R
    a, _ = md.md_route_topk(w.logits, k)
    b, _ = md.md_route_topk(w.logits_next, k)
    _, C = md.md_coselect_stats(a, b, E, T_fit=w.fit_tokens, want_W=False)
    pred, perm, inv = md.md_token_shuffle(a, C, w.expert_to_rank, R)
    ordered, L = _chain_gpu(b, inv, E, R, w.expert_to_rank)
    torch.cuda.synchronize()
    oa = oracle.route_topk(w.logits.cpu().numpy(), k)[0]
    ob = oracle.route_topk(w.logits_next.cpu().numpy(), k)[0]
    _, oC = oracle.coselect(oa, ob, E, T_fit=w.fit_tokens)
    p0 = w.expert_to_rank.cpu().numpy()
    opred, operm, oinv = oracle.token_shuffle(oa, oC, p0, R)
    for got, want in zip((pred, perm, inv), (opred, operm, oinv)):
        assert np.array_equal(got.cpu().numpy(), want)
    ob_shuf = ob[oinv]  # X'[perm[t]] = X[t]: row t' of the shuffled order is token inv[t']
    assert np.array_equal(ordered.cpu().numpy(), ob_shuf)
    OL = oracle.dispatch_layout(ob_shuf, E, R, p0, oracle.DEDUP)
    _check_layout(L, OL)
    # the shuffle keeps more rows on their source rank than the original order
    base = oracle.dispatch_layout(ob, E, R, p0, oracle.DEDUP)["send_counts"]
    off = lambda m: int(m.sum() - np.trace(m))
    assert off(OL["send_counts"]) < off(base)


def test_dedup_layout_after_pair_shuffle_full_size():
    w = synth.make_workload("three_layer_e128_k6", device=DEV, with_rows=False)
    E, k, R = w.E, w.k, w.R
    g = [md.md_route_topk(lg, k)[0] for lg in (w.logits_prev, w.logits, w.logits_next)]
    C2 = md.md_coselect_pair_stats(g[0], g[1], g[2], E, T_fit=w.fit_tokens)
    _, C = md.md_coselect_stats(g[1], g[2], E, T_fit=w.fit_tokens, want_W=False)
    pred, perm, inv, use = md.md_token_shuffle_pair(g[0], g[1], C, C2, w.expert_to_rank, R, 8 * k)
    ordered, L = _chain_gpu(g[2], inv, E, R, w.expert_to_rank)
    torch.cuda.synchronize()
    og = [oracle.route_topk(lg.cpu().numpy(), k)[0]
          for lg in (w.logits_prev, w.logits, w.logits_next)]
    oC2 = oracle.coselect_pair(og[0], og[1], og[2], E, T_fit=w.fit_tokens)
    _, oC = oracle.coselect(og[1], og[2], E, T_fit=w.fit_tokens)
    p0 = w.expert_to_rank.cpu().numpy()
    want = oracle.token_shuffle_pair(og[0], og[1], oC, oC2, p0, R, 8 * k)
    for got, exp in zip((pred, perm, inv, use), want):
        assert np.array_equal(got.cpu().numpy(), exp)
    ob_shuf = og[2][want[2]]
    assert np.array_equal(ordered.cpu().numpy(), ob_shuf)
    _check_layout(L, oracle.dispatch_layout(ob_shuf, E, R, p0, oracle.DEDUP))
