"""md_dispatch_permute and md_combine on the GPU against the oracle.

Permute: bit-exact.  Combine: bit-exact (fp32 FMA in ascending expert order on
both sides), which is inside the stated 1e-2 absolute / 1 bf16 ulp bound."""
import numpy as np
import pytest
import torch

import combine_warp_top_router_b200 as md
import oracle
from combine_warp_top_router_b200 import synth

from _util import DEV, bits, f32, from_bits, i32, shuffled_placement

pytestmark = pytest.mark.gpu

POISON_BITS = 0x7FA1  # a NaN pattern no kernel writes


@pytest.fixture(params=[md.MD_PERMUTE_BULK, md.MD_PERMUTE_VECTOR, md.MD_PERMUTE_AUTO],
                ids=["bulk", "vector", "auto"])
def permute_path(request):
    """Run a permute test with each of md_dispatch_permute's kernels (the
    bulk-copy ring only takes rows of 1 KiB and more)."""
    md.md_set_permute_path(request.param)
    yield request.param
    md.md_set_permute_path(md.MD_PERMUTE_AUTO)


def _case(name, T, R=None, H=None, mode=None, seed=0, placement="contiguous"):
    w = synth.make_workload(name, seed=seed, T=T, R=R, H=H, mode=mode)
    k, E = w.k, w.E
    idx, gates = oracle.route_topk(w.logits.numpy(), k)
    p = w.expert_to_rank.numpy() if placement == "contiguous" else shuffled_placement(E, w.R, 9)
    L = oracle.dispatch_layout(idx, E, w.R, p, w.mode)
    return w, idx, gates, p, L


def _within_tolerance(a_bits, b_bits):
    a = torch.from_numpy(a_bits.view(np.int16)).view(torch.bfloat16).float()
    b = torch.from_numpy(b_bits.view(np.int16)).view(torch.bfloat16).float()
    ulp = torch.abs(b) * 2.0 ** -7
    return bool(torch.all((a - b).abs() <= torch.maximum(torch.full_like(b, 1e-2), ulp)))


CASES = [("iid_e64_k6", 4096, None, None, 0), ("zipf_pairs_e128_k8", 4096, None, None, 1),
         ("zipf_pairs_e128_k8", 4096, None, None, 0), ("boost_pairs_e128_k2", 2048, 32, None, 1),
         ("two_layer_e128_k6", 16 * 41, None, 264, 1), ("full_e256_k8", 4096, None, 8, 1)]


@pytest.mark.parametrize("name,T,R,H,mode", CASES)
def test_permute_matches_oracle(name, T, R, H, mode, permute_path):
    w, idx, gates, p, L = _case(name, T, R, H, mode, placement="shuffled")
    n = L["n_rows"]
    cap = n + 5
    out = from_bits(np.full((cap, w.H), POISON_BITS, np.uint16))
    st = md.new_status(DEV)
    md.md_dispatch_permute(w.x.to(DEV), i32(L["row_of_slot"]), out=out, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == md.MD_OK
    got = bits(out)
    want = oracle.dispatch_permute(bits(w.x), L["row_token"])
    assert np.array_equal(got[:n], want)
    assert np.all(got[n:] == POISON_BITS)


@pytest.mark.parametrize("name,T,R,H,mode", CASES)
def test_combine_fused_matches_oracle(name, T, R, H, mode):
    w, idx, gates, p, L = _case(name, T, R, H, mode)
    out = md.md_combine(w.y.to(DEV), i32(L["assign_row"]), i32(idx), f32(gates))
    torch.cuda.synchronize()
    want = oracle.combine(bits(w.y), L["assign_row"], idx, gates)
    got = bits(out)
    assert _within_tolerance(got, want)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("name,T,R,H", [("zipf_pairs_e128_k8", 4096, None, None),
                                        ("boost_pairs_e128_k2", 2048, 8, 64),
                                        ("full_e256_k8", 2048, None, 16),
                                        ("iid_e64_k6", 64 * 5, 64, 24)])
def test_combine_wire_matches_oracle(name, T, R, H):
    w, idx, gates, p, L = _case(name, T, R, H, 1, placement="shuffled")
    n = L["n_rows"]
    z = from_bits(np.full((n + 3, w.H), POISON_BITS, np.uint16))
    out = md.md_combine(w.y.to(DEV), i32(L["assign_row"]), i32(idx), f32(gates),
                        md.MD_COMBINE_WIRE, row_of_slot=i32(L["row_of_slot"]), z=z)
    torch.cuda.synchronize()
    want_out, want_z = oracle.combine(bits(w.y), L["assign_row"], idx, gates, oracle.COMBINE_WIRE,
                                      p, L["row_of_slot"], n)
    assert np.array_equal(bits(out), want_out)
    gz = bits(z)
    assert np.array_equal(gz[:n], want_z)
    assert np.all(gz[n:] == POISON_BITS)


@pytest.mark.parametrize("k", [1, 3, 5, 12, 32])
def test_generic_k(k, permute_path):
    # k values without a specialised kernel (and k = 1)
    T, E, R, H = 256, 64, 4, 40
    lg = synth.normal_f32(T, E, k, 1).numpy()
    idx, gates = oracle.route_topk(lg, k)
    p = shuffled_placement(E, R, 2)
    L = oracle.dispatch_layout(idx, E, R, p, 1)
    x = synth.normal_bf16(T, H, 1, 3)
    y = synth.normal_bf16(T * k, H, 1, 4)
    out = md.md_dispatch_permute(x.to(DEV), i32(L["row_of_slot"]), out_rows=L["n_rows"])
    fused = md.md_combine(y.to(DEV), i32(L["assign_row"]), i32(idx), f32(gates))
    z = torch.empty(L["n_rows"], H, dtype=torch.bfloat16, device=DEV)
    wire = md.md_combine(y.to(DEV), i32(L["assign_row"]), i32(idx), f32(gates), md.MD_COMBINE_WIRE,
                         row_of_slot=i32(L["row_of_slot"]), z=z)
    torch.cuda.synchronize()
    assert np.array_equal(bits(out), oracle.dispatch_permute(bits(x), L["row_token"]))
    assert np.array_equal(bits(fused), oracle.combine(bits(y), L["assign_row"], idx, gates))
    wo, wz = oracle.combine(bits(y), L["assign_row"], idx, gates, oracle.COMBINE_WIRE, p,
                            L["row_of_slot"], L["n_rows"])
    assert np.array_equal(bits(wire), wo)
    assert np.array_equal(bits(z), wz)


# rows of 1 KiB and more move by bulk copies in pieces of at most 4 KiB:
# just under and at that size, a 16-byte last piece, three pieces; several k
# (5 has no specialised kernel)
@pytest.mark.parametrize("H", [504, 512, 2056, 4104])
@pytest.mark.parametrize("k", [2, 5, 8, 32])
def test_permute_row_pieces(H, k, permute_path):
    T, E, R = 300, 64, 4
    idx = oracle.route_topk(synth.normal_f32(T, E, H + k, 1).numpy(), k)[0]
    L = oracle.dispatch_layout(idx, E, R, shuffled_placement(E, R, 6), 1)
    x = synth.normal_bf16(T, H, k, 3)
    n = L["n_rows"]
    out = from_bits(np.full((n + 3, H), POISON_BITS, np.uint16))
    st = md.new_status(DEV)
    md.md_dispatch_permute(x.to(DEV), i32(L["row_of_slot"]), out=out, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == md.MD_OK
    got = bits(out)
    assert np.array_equal(got[:n], oracle.dispatch_permute(bits(x), L["row_token"]))
    assert np.all(got[n:] == POISON_BITS)


@pytest.mark.parametrize("H", [16, 1024])
def test_bad_rows_are_skipped_and_reported(H, permute_path):
    T, k = 64, 2
    x = synth.normal_bf16(T, H, 0, 3).to(DEV)
    rows = torch.arange(T * k, dtype=torch.int32, device=DEV).view(T, k)
    rows[3, 1] = 10_000
    st = md.new_status(DEV)
    out = md.md_dispatch_permute(x, rows, out_rows=T * k, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == md.MD_ERR_DATA
    assert torch.equal(out[6], x[3])  # the valid slot of token 3 still landed
    st2 = md.new_status(DEV)
    y = synth.normal_bf16(T * k, H, 0, 4).to(DEV)
    w = torch.full((T, k), 0.5, device=DEV)
    idx = torch.zeros(T, k, dtype=torch.int32, device=DEV)
    idx[:, 1] = 1
    md.md_combine(y, rows, idx, w, dev_status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == md.MD_ERR_DATA


def test_gather_rows():
    T, H = 1000, 48
    x = synth.normal_bf16(T, H, 2, 3).to(DEV)
    perm = torch.randperm(T, generator=torch.Generator().manual_seed(1)).to(torch.int32).to(DEV)
    got = md.md_gather_rows(x, perm)
    assert torch.equal(got, x[perm.long()])
    ids = torch.randint(0, 50, (T, 6), dtype=torch.int32, device=DEV)  # 24-byte rows
    got2 = md.md_gather_rows(ids, perm)
    assert torch.equal(got2, ids[perm.long()])


def test_permute_path_selector_rejects_unknown_values():
    with pytest.raises(md.MoeDispatchError):
        md.md_set_permute_path(7)
    md.md_set_permute_path(md.MD_PERMUTE_AUTO)


def test_full_size_sampled():
    # the benchmark workload at full size (T=65536, H=2048, E=128, k=8, R=16,
    # dedup), in the launch configuration the benchmark times.  The oracle
    # runs its own router and layout on the same logits; permute rows and
    # combine outputs are checked on samples it computes one by one.
    w = synth.make_workload("zipf_pairs_e128_k8", device=DEV)
    idx, gates = md.md_route_topk(w.logits, 8)
    L = md.md_dispatch_layout(idx, w.E, w.R, w.expert_to_rank, md.MD_DEDUP)
    buf = md.md_dispatch_permute(w.x, L.row_of_slot, out_rows=L.row_capacity)
    out = md.md_combine(w.y, L.assign_row, idx, gates)
    torch.cuda.synchronize()
    oi, ow = oracle.route_topk(w.logits.cpu().numpy(), 8)
    OL = oracle.dispatch_layout(oi, w.E, w.R, w.expert_to_rank.cpu().numpy(), 1)
    n = OL["n_rows"]
    assert np.array_equal(idx.cpu().numpy(), oi)
    assert np.allclose(gates.cpu().numpy(), ow, rtol=1e-6, atol=0)
    assert int(L.n_rows.item()) == n
    assert np.array_equal(L.row_of_slot.cpu().numpy(), OL["row_of_slot"])
    assert np.array_equal(L.assign_row.cpu().numpy(), OL["assign_row"])
    rng = np.random.default_rng(0)
    rows = rng.choice(n, 2048, replace=False)
    assert np.array_equal(bits(buf[torch.from_numpy(rows).to(DEV)]),
                          bits(w.x[torch.from_numpy(OL["row_token"][rows]).long().to(DEV)]))
    toks = np.sort(rng.choice(w.T, 512, replace=False))
    ar = OL["assign_row"][toks]
    ysub = bits(w.y[torch.from_numpy(ar.ravel()).long().to(DEV)])
    want = oracle.combine(ysub, np.arange(ar.size, dtype=np.int32).reshape(ar.shape), oi[toks],
                          ow[toks])
    assert np.array_equal(bits(out[torch.from_numpy(toks).long().to(DEV)]), want)
