"""md_dispatch_layout_noalloc: the layout for callers that cannot allocate
device memory (for example a plug-in whose host framework owns all GPU memory
through its own pool).  It must give exactly what md_dispatch_layout gives with
a caller-allocated workspace, call after call, although every call reuses the
same fixed scratch array inside the library (and, for the smaller shapes,
exactly the oracle's layout).

Called through the C ABI with ctypes.  This file is collected last on purpose;
it also passes when run alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

import combine_warp_top_router_b200 as md
from combine_warp_top_router_b200 import binding, synth

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _outputs(T, E, k, R, mode):
    L = md.alloc_layout(T, E, k, R, mode, DEV)
    for t in (L.row_of_slot, L.assign_row, L.row_token, L.row_mask, L.send_counts,
              L.expert_counts, L.expert_offsets, L.rank_offsets, L.n_rows):
        t.fill_(-3)
    return L


def _noalloc(idx, E, R, p, mode, status, stream):
    T, k = idx.shape
    L = _outputs(T, E, k, R, mode)
    rc = binding.lib().md_dispatch_layout_noalloc(
        _p(idx), T, E, k, R, _p(p), mode, _p(L.row_of_slot), _p(L.assign_row), _p(L.row_token),
        _p(L.row_mask), _p(L.send_counts), _p(L.expert_counts), _p(L.expert_offsets),
        _p(L.rank_offsets), _p(L.n_rows), _p(status), ctypes.c_void_p(stream.cuda_stream))
    assert rc == md.MD_OK, binding.status_string(rc)
    return L


def _with_workspace(idx, E, R, p, mode, stream):
    T, k = idx.shape
    L = _outputs(T, E, k, R, mode)
    ws = md.alloc_workspace(md.dispatch_layout_workspace_size(T, E, k, R, mode), DEV)
    lib = binding.lib()
    rc = lib.md_dispatch_layout(
        _p(idx), T, E, k, R, _p(p), mode, _p(L.row_of_slot), _p(L.assign_row), _p(L.row_token),
        _p(L.row_mask), _p(L.send_counts), _p(L.expert_counts), _p(L.expert_offsets),
        _p(L.rank_offsets), _p(L.n_rows), _p(ws), ws.numel(), None,
        ctypes.c_void_p(stream.cuda_stream))
    assert rc == md.MD_OK
    return L


def _same(a, b):
    n = int(b.n_rows.item())
    assert int(a.n_rows.item()) == n
    for name in ("row_of_slot", "assign_row", "send_counts", "expert_counts", "expert_offsets",
                 "rank_offsets"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    assert torch.equal(a.row_token[:n], b.row_token[:n])
    assert torch.equal(a.row_mask[:n], b.row_mask[:n])


@pytest.mark.parametrize("name,T,mode", [("zipf_pairs_e128_k8", 65536, md.MD_DEDUP),
                                         ("full_e256_k8", 262144, md.MD_DEDUP),
                                         ("iid_e64_k6", 4096, md.MD_CONV)])
def test_noalloc_matches_workspace_entry_point_twice(name, T, mode):
    spec = synth.SPECS[name]
    E, k, R = spec["E"], spec["k"], spec["R"]
    assert binding.lib().md_dispatch_layout_workspace_size(T, E, k, R, mode) <= \
        binding.lib().md_dispatch_layout_noalloc_max_scratch()
    stream = torch.cuda.current_stream()
    p = synth.contiguous_placement(E, R, DEV)
    status = torch.full((1,), 77, dtype=torch.int32, device=DEV)
    # two calls in a row on different routings: the second starts from the
    # first call's leftovers in the shared scratch array
    for seed in (0, 1):
        w = synth.make_workload(name, seed=seed, device=DEV, T=T, with_rows=False)
        idx, _ = md.md_route_topk(w.logits, k)
        got = _noalloc(idx, E, R, p, mode, status, stream)
        want = _with_workspace(idx, E, R, p, mode, stream)
        torch.cuda.synchronize()
        assert int(status.item()) == md.MD_OK
        _same(got, want)
        if T <= 65536:  # and the oracle's layout of the same top-k lists
            import oracle
            O = oracle.dispatch_layout(idx.cpu().numpy(), E, R, p.cpu().numpy(), mode)
            n = O["n_rows"]
            assert int(got.n_rows.item()) == n
            for name_ in ("row_of_slot", "assign_row", "send_counts", "rank_offsets"):
                assert np.array_equal(getattr(got, name_).cpu().numpy(), O[name_]), name_
            assert np.array_equal(got.row_token[:n].cpu().numpy(), O["row_token"])


def test_noalloc_takes_sizes_whose_old_scratch_need_was_larger():
    # the workspace does not grow with T: a million tokens (E=256, k=8, R=64,
    # about 5 MB of per-tile scratch in a per-tile lookback design) fits
    T, E, k, R = 1 << 20, 256, 8, 64
    lib = binding.lib()
    assert lib.md_dispatch_layout_workspace_size(T, E, k, R, md.MD_DEDUP) <= \
        lib.md_dispatch_layout_noalloc_max_scratch()
    stream = torch.cuda.current_stream()
    p = synth.contiguous_placement(E, R, DEV)
    status = torch.full((1,), 77, dtype=torch.int32, device=DEV)
    idx, _ = md.md_route_topk(synth.normal_f32(T, E, 5, 1, DEV), k)
    got = _noalloc(idx, E, R, p, md.MD_DEDUP, status, stream)
    want = _with_workspace(idx, E, R, p, md.MD_DEDUP, stream)
    torch.cuda.synchronize()
    assert int(status.item()) == md.MD_OK
    _same(got, want)
