"""md_dispatch_layout on the GPU against the oracle: every output bit-exact.

Inputs (top-k lists, placements) come from the seeded generator and the
oracle; the GPU and the oracle see the same arrays."""
import numpy as np
import pytest
import torch

import combine_warp_top_router_b200 as md
import oracle
from combine_warp_top_router_b200 import synth

from _util import DEV, i32, shuffled_placement

pytestmark = pytest.mark.gpu

POISON = -7


@pytest.fixture(params=[md.MD_LAYOUT_COOPERATIVE, md.MD_LAYOUT_SPLIT], ids=["coop", "split"])
def layout_path(request):
    """Run a layout test with each launch form: one cooperative launch with
    the arrival wait, and the split form (counts, then ranks)."""
    md.md_set_layout_path(request.param)
    yield request.param
    md.md_set_layout_path(md.MD_LAYOUT_AUTO)


def gpu_layout(idx_np, E, R, p_np, mode):
    idx = i32(idx_np)
    T, k = idx_np.shape
    L = md.alloc_layout(T, E, k, R, mode, DEV)
    L.row_token.fill_(POISON)
    L.row_mask.fill_(POISON)
    st = md.new_status(DEV)
    md.md_dispatch_layout(idx, E, R, i32(p_np), mode, out=L, dev_status=st)
    torch.cuda.synchronize()
    return L, int(st.item())


def assert_layout_equal(L, O, T, k):
    n = O["n_rows"]
    assert int(L.n_rows.item()) == n
    assert np.array_equal(L.assign_row.cpu().numpy(), O["assign_row"])
    assert np.array_equal(L.row_of_slot.cpu().numpy(), O["row_of_slot"])
    rt = L.row_token.cpu().numpy()
    rm = L.row_mask.cpu().numpy().view(np.uint32)
    assert np.array_equal(rt[:n], O["row_token"])
    assert np.array_equal(rm[:n], O["row_mask"])
    assert np.all(rt[n:] == POISON)  # rows past n_rows are never written
    assert np.array_equal(L.send_counts.cpu().numpy(), O["send_counts"])
    assert np.array_equal(L.expert_counts.cpu().numpy(), O["expert_counts"])
    assert np.array_equal(L.expert_offsets.cpu().numpy(), O["expert_offsets"])
    assert np.array_equal(L.rank_offsets.cpu().numpy(), O["rank_offsets"])


def _routes(name, T, seed=0):
    w = synth.make_workload(name, seed=seed, T=T, with_rows=False)
    return oracle.route_topk(w.logits.numpy(), synth.SPECS[name]["k"])[0]


CASES = [
    # (workload, T, R, placement)
    ("iid_e64_k6", 4096, 16, "contiguous"),
    ("zipf_pairs_e128_k8", 8192, 16, "contiguous"),
    ("boost_pairs_e128_k2", 8192, 8, "shuffled"),
    ("boost_pairs_e128_k2", 8192, 32, "shuffled"),
    ("two_layer_e128_k6", 8192, 16, "shuffled"),
    ("full_e256_k8", 8192, 64, "contiguous"),
    ("zipf_pairs_e128_k8", 16 * 37, 16, "contiguous"),   # ragged last tile
    ("iid_e64_k6", 64 * 3, 64, "shuffled"),              # 3 tokens per rank
]


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("name,T,R,pl", CASES)
def test_layout_matches_oracle(name, T, R, pl, mode, layout_path):
    idx = _routes(name, T)
    E = synth.SPECS[name]["E"]
    p = synth.contiguous_placement(E, R).numpy() if pl == "contiguous" else shuffled_placement(E, R, 3)
    L, st = gpu_layout(idx, E, R, p, mode)
    assert st == md.MD_OK
    assert_layout_equal(L, oracle.dispatch_layout(idx, E, R, p, mode), *idx.shape)


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("E,k,R,T", [(8, 1, 2, 100), (8, 8, 8, 64), (16, 3, 1, 48), (12, 5, 3, 99),
                                     (1024, 32, 64, 128), (256, 16, 4, 256), (64, 6, 64, 4096)])
def test_layout_edge_shapes(E, k, R, T, mode, layout_path):
    lg = synth.normal_f32(T, E, 11, 1).numpy()
    idx = oracle.route_topk(lg, k)[0]
    p = shuffled_placement(E, R, 5)
    L, st = gpu_layout(idx, E, R, p, mode)
    assert st == md.MD_OK
    assert_layout_equal(L, oracle.dispatch_layout(idx, E, R, p, mode), T, k)


def test_layout_empty(layout_path):
    E, k, R = 16, 2, 4
    L, st = gpu_layout(np.zeros((0, k), np.int32), E, R, synth.contiguous_placement(E, R).numpy(), 1)
    assert st == md.MD_OK and int(L.n_rows.item()) == 0
    assert int(L.send_counts.sum().item()) == 0
    assert L.rank_offsets.cpu().tolist() == [0] * (R + 1)


def test_layout_reports_bad_data(layout_path):
    E, k, R, T = 16, 3, 4, 64
    idx = oracle.route_topk(synth.normal_f32(T, E, 1, 1).numpy(), k)[0]
    p = synth.contiguous_placement(E, R).numpy()
    bad = idx.copy()
    bad[5, 1] = E + 3                 # out of range
    _, st = gpu_layout(bad, E, R, p, 1)
    assert st == md.MD_ERR_DATA
    dup = idx.copy()
    dup[7, 2] = dup[7, 0]             # same expert twice
    _, st = gpu_layout(dup, E, R, p, 0)
    assert st == md.MD_ERR_DATA
    q = p.copy()
    q[0] = 1                          # rank 0 has E/R - 1 experts
    _, st = gpu_layout(idx, E, R, q, 0)
    assert st == md.MD_ERR_DATA
    _, st = gpu_layout(idx, E, R, p, 1)  # and a clean call resets the status
    assert st == md.MD_OK


def test_layout_rejects_bad_arguments():
    idx = torch.zeros(10, 2, dtype=torch.int32, device=DEV)
    p = torch.zeros(8, dtype=torch.int32, device=DEV)
    with pytest.raises(md.MoeDispatchError):
        md.md_dispatch_layout(idx, 8, 4, p, 0)           # T % R != 0
    with pytest.raises(md.MoeDispatchError):
        md.md_dispatch_layout(idx, 8, 2, p, 0, workspace=torch.empty(256, dtype=torch.uint8,
                                                                    device=DEV))


@pytest.mark.parametrize("mode", [0, 1])
def test_layout_full_size(mode, layout_path):
    # the full-pipeline workload at full size: T=262144, E=256, k=8, R=64
    w = synth.make_workload("full_e256_k8", device=DEV, with_rows=False)
    idx_g, _ = md.md_route_topk(w.logits, 8)
    idx = idx_g.cpu().numpy()
    # the layout's input is the oracle's own top-k of the same logits
    oi = oracle.route_topk(w.logits.cpu().numpy(), 8)[0]
    assert np.array_equal(idx, oi)
    p = synth.contiguous_placement(256, 64).numpy()
    L, st = gpu_layout(oi, 256, 64, p, mode)
    assert st == md.MD_OK
    assert_layout_equal(L, oracle.dispatch_layout(oi, 256, 64, p, mode), *oi.shape)


@pytest.mark.parametrize("mode", [0, 1])
def test_layout_unaligned_outputs(mode):
    # outputs that are not 16-byte aligned take the scalar-store kernel
    name, T, R = "zipf_pairs_e128_k8", 2048, 16
    idx = _routes(name, T)
    E, k = 128, 8
    p = synth.contiguous_placement(E, R).numpy()
    L = md.alloc_layout(T, E, k, R, mode, DEV)
    raw_a = torch.full((T * k + 1,), -5, dtype=torch.int32, device=DEV)
    raw_r = torch.full((T * k + 1,), -5, dtype=torch.int32, device=DEV)
    L.assign_row = raw_a[1:].view(T, k)
    L.row_of_slot = raw_r[1:].view(T, k)
    L.row_token.fill_(POISON)
    md.md_dispatch_layout(i32(idx), E, R, i32(p), mode, out=L)
    torch.cuda.synchronize()
    assert_layout_equal(L, oracle.dispatch_layout(idx, E, R, p, mode), T, k)


def test_layout_replays_in_cuda_graph(layout_path):
    # A captured layout replays with new inputs: the capture also records the
    # clear of the arrival words, so every replay waits for its own counts.
    from combine_warp_top_router_b200 import binding
    name, T, R, E, k = "zipf_pairs_e128_k8", 4096, 16, 128, 8
    p = synth.contiguous_placement(E, R).numpy()
    runs = [_routes(name, T, seed=s) for s in (0, 1, 2)]
    static_idx = i32(runs[0])
    pg = i32(p)
    L = md.alloc_layout(T, E, k, R, 1, DEV)
    ws = binding.alloc_workspace(binding.dispatch_layout_workspace_size(T, E, k, R, 1), DEV)
    st = md.new_status(DEV)
    md.md_dispatch_layout(static_idx, E, R, pg, 1, out=L, workspace=ws, dev_status=st)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        md.md_dispatch_layout(static_idx, E, R, pg, 1, out=L, workspace=ws, dev_status=st)
    for idx in (runs[1], runs[2], runs[0], runs[1]):
        static_idx.copy_(torch.from_numpy(idx))
        L.row_token.fill_(POISON)
        g.replay()
        torch.cuda.synchronize()
        assert int(st.item()) == md.MD_OK
        assert_layout_equal(L, oracle.dispatch_layout(idx, E, R, p, 1), T, k)
    del g


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("T", [512 * 148 * 3 + 64, 512 * 300, 512 * 148, 512 * 149])
def test_layout_several_tiles_per_cta(T, mode, layout_path):
    # more tiles than resident CTAs: each CTA walks a run of tiles and carries
    # its bucket starts from one tile to the next (T = 512*148*3 + 64 leaves a
    # short last tile).  512*148 tiles launch one CTA per SM, so the arrival
    # wait reads more than 128 stamps; 512*149 gives two tiles per CTA.  R = 8
    # divides every size.
    E, k, R = 64, 6, 8
    lg = synth.normal_f32(T, E, 21, 1).numpy()
    idx = oracle.route_topk(lg, k)[0]
    p = shuffled_placement(E, R, 9)
    L, st = gpu_layout(idx, E, R, p, mode)
    assert st == md.MD_OK
    assert_layout_equal(L, oracle.dispatch_layout(idx, E, R, p, mode), T, k)


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("fill", ["stamp", "ones_bits", "random"])
def test_layout_ignores_stale_workspace(fill, mode, layout_path):
    # Whatever the workspace holds on entry -- every 32-bit word equal to the
    # value a CTA stamps on arrival (1), all bits set, or random words such as
    # a recycled allocation holds -- the layout is the oracle's: the call
    # clears its arrival words on the stream before the kernel, so no CTA can
    # pass the arrival wait before every other CTA has published its counts.
    E, k, R = 128, 8, 16
    T = 512 * 148 * 2  # two tiles per CTA
    lg = synth.make_workload("zipf_pairs_e128_k8", seed=4, T=T, with_rows=False).logits.numpy()
    idx = oracle.route_topk(lg, k)[0]
    p = shuffled_placement(E, R, 2)
    O = oracle.dispatch_layout(idx, E, R, p, mode)
    from combine_warp_top_router_b200 import binding
    ws = binding.alloc_workspace(binding.dispatch_layout_workspace_size(T, E, k, R, mode), DEV)
    words = ws.view(torch.int32)
    gen = torch.Generator(device=DEV)
    gen.manual_seed(17)
    for rep in range(3):
        if fill == "stamp":
            words.fill_(1)
        elif fill == "ones_bits":
            words.fill_(-1)
        else:
            words.copy_(torch.randint(-2**31, 2**31 - 1, words.shape, generator=gen, device=DEV,
                                      dtype=torch.int64).to(torch.int32))
        L = md.alloc_layout(T, E, k, R, mode, DEV)
        L.row_token.fill_(POISON)
        st = torch.full((1,), 99, dtype=torch.int32, device=DEV)  # cleared by the call
        md.md_dispatch_layout(i32(idx), E, R, i32(p), mode, out=L, workspace=ws, dev_status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == md.MD_OK
        assert_layout_equal(L, O, T, k)


def test_layout_path_selector_rejects_unknown_values():
    with pytest.raises(md.MoeDispatchError):
        md.md_set_layout_path(5)
    md.md_set_layout_path(md.MD_LAYOUT_AUTO)
