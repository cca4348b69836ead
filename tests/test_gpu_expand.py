"""md_dedup_expand on the GPU against the oracle: bit-exact.

The receiver-side expand copies each slot's deduplicated row to its
expert-grouped (conventional) position, so the result must also equal the
conventional dispatch buffer."""
import numpy as np
import pytest
import torch

import combine_warp_top_router_b200 as md
import oracle
from combine_warp_top_router_b200 import synth

from _util import DEV, bits, from_bits, i32, shuffled_placement

pytestmark = pytest.mark.gpu

POISON_BITS = 0x7FA1


def _layouts(idx, E, R, seed):
    p = shuffled_placement(E, R, seed)
    return oracle.dispatch_layout(idx, E, R, p, 1), oracle.dispatch_layout(idx, E, R, p, 0)


def _check_expand(x_bits, idx, E, R, seed=3):
    T, k = idx.shape
    H = x_bits.shape[1]
    Ld, Lc = _layouts(idx, E, R, seed)
    wire = oracle.dispatch_permute(x_bits, Ld["row_token"])
    out = from_bits(np.full((T * k + 2, H), POISON_BITS, np.uint16))
    st = md.new_status(DEV)
    md.md_dedup_expand(from_bits(wire), i32(Ld["row_of_slot"]), i32(Ld["assign_row"]), out=out,
                       dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == md.MD_OK
    got = bits(out)
    want = oracle.dedup_expand(wire, Ld["row_of_slot"], Ld["assign_row"])
    assert np.array_equal(got[:T * k], want)
    assert np.array_equal(got[:T * k], oracle.dispatch_permute(x_bits, Lc["row_token"]))
    assert np.all(got[T * k:] == POISON_BITS)


@pytest.mark.parametrize("name,T,R,H", [("zipf_pairs_e128_k8", 4096, None, None),
                                        ("boost_pairs_e128_k2", 2048, 8, None),
                                        ("two_layer_e128_k6", 16 * 41, None, 264),
                                        ("iid_e64_k6", 1024, None, 2056),
                                        ("full_e256_k8", 2048, None, 8)])
def test_expand_matches_oracle(name, T, R, H):
    w = synth.make_workload(name, T=T, R=R, H=H, with_rows=True)
    idx = oracle.route_topk(w.logits.numpy(), w.k)[0]
    _check_expand(bits(w.x), idx, w.E, w.R)


# rows just under / at the bulk-copy size, a 16-byte last piece, three
# pieces; k without a specialised kernel and the largest k
@pytest.mark.parametrize("H", [504, 512, 2056, 4104])
@pytest.mark.parametrize("k", [1, 5, 32])
def test_expand_row_pieces(H, k):
    T, E, R = 300, 64, 4
    idx = oracle.route_topk(synth.normal_f32(T, E, H + k, 1).numpy(), k)[0]
    _check_expand(bits(synth.normal_bf16(T, H, k, 3)), idx, E, R, seed=H)


@pytest.mark.parametrize("H", [16, 1024])
def test_expand_reports_bad_rows(H):
    T, k = 64, 2
    wire = synth.normal_bf16(T, H, 0, 3).to(DEV)
    rs = torch.arange(T * k, dtype=torch.int32, device=DEV).view(T, k) // 2
    ar = torch.arange(T * k, dtype=torch.int32, device=DEV).view(T, k)
    rs[3, 1] = 10_000          # source out of range
    ar[5, 0] = -1              # destination out of range
    st = md.new_status(DEV)
    out = torch.zeros(T * k, H, dtype=torch.bfloat16, device=DEV)
    md.md_dedup_expand(wire, rs, ar, out=out, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == md.MD_ERR_DATA
    assert torch.equal(out[6], wire[3]) and torch.equal(out[11], wire[5])  # valid slots landed
    assert not out[7].any()


def test_expand_empty():
    out = md.md_dedup_expand(torch.zeros(0, 64, dtype=torch.bfloat16, device=DEV),
                             torch.zeros(0, 4, dtype=torch.int32, device=DEV),
                             torch.zeros(0, 4, dtype=torch.int32, device=DEV))
    torch.cuda.synchronize()
    assert out.shape == (0, 64)


def test_expand_full_size_sampled():
    # the benchmark workload at full size, after the GPU dedup dispatch: the
    # expanded buffer must hold x[token] at every conventional row; the oracle
    # runs its own router and conventional layout and names the tokens
    w = synth.make_workload("zipf_pairs_e128_k8", device=DEV)
    idx, _ = md.md_route_topk(w.logits, 8)
    L = md.md_dispatch_layout(idx, w.E, w.R, w.expert_to_rank, md.MD_DEDUP)
    wire = md.md_dispatch_permute(w.x, L.row_of_slot, out_rows=L.row_capacity)
    out = md.md_dedup_expand(wire, L.row_of_slot, L.assign_row)
    torch.cuda.synchronize()
    oi = oracle.route_topk(w.logits.cpu().numpy(), 8)[0]
    assert np.array_equal(idx.cpu().numpy(), oi)
    Lc = oracle.dispatch_layout(oi, w.E, w.R, w.expert_to_rank.cpu().numpy(), 0)
    rows = np.random.default_rng(1).choice(w.T * 8, 4096, replace=False)
    got = bits(out[torch.from_numpy(rows).to(DEV)])
    want = bits(w.x[torch.from_numpy(Lc["row_token"][rows]).long().to(DEV)])
    assert np.array_equal(got, want)
