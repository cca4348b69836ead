"""Failure detection without a GPU fault: every device-side wait is bounded.

md_set_test_hooks shortens the poll limit and leaves one CTA's arrival stamp
(the dispatch layout) or one bulk-copy load (the dedup expand) out, so that a
wait runs out.  The call must end with MD_ERR_TIMEOUT in its status word -- no
trap, no hang -- and the next call, with the hooks cleared, must be exact."""
import numpy as np
import pytest
import torch

import combine_warp_top_router_b200 as md
import oracle
from combine_warp_top_router_b200 import synth

from _util import DEV, bits, from_bits, i32

pytestmark = pytest.mark.gpu


@pytest.fixture
def hooks():
    yield md.md_set_test_hooks
    md.md_set_test_hooks()  # defaults, whatever happened


def _routes(T):
    w = synth.make_workload("zipf_pairs_e128_k8", T=T, with_rows=False)
    return w, oracle.route_topk(w.logits.numpy(), 8)[0]


@pytest.mark.parametrize("mode", [0, 1])
def test_layout_arrival_wait_runs_out(hooks, mode):
    w, idx = _routes(8192)                    # 16 tiles of 512 tokens, one per CTA
    p = w.expert_to_rank.numpy()
    hooks(poll_limit=4096, layout_skip_tile=0)
    st = md.new_status(DEV)
    md.md_dispatch_layout(i32(idx), w.E, w.R, i32(p), mode, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == md.MD_ERR_TIMEOUT
    md.md_set_test_hooks()
    st = md.new_status(DEV)
    L = md.md_dispatch_layout(i32(idx), w.E, w.R, i32(p), mode, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == md.MD_OK
    O = oracle.dispatch_layout(idx, w.E, w.R, p, mode)
    assert np.array_equal(L.row_of_slot.cpu().numpy(), O["row_of_slot"])
    assert np.array_equal(L.assign_row.cpu().numpy(), O["assign_row"])


def test_bulk_copy_wait_runs_out(hooks):
    T, E, k, R, H = 512, 64, 4, 8, 1024     # 2 KiB rows: the bulk-copy path
    idx = oracle.route_topk(synth.normal_f32(T, E, 3, 1).numpy(), k)[0]
    p = (np.arange(E) // (E // R)).astype(np.int32)
    Ld = oracle.dispatch_layout(idx, E, R, p, 1)
    Lc = oracle.dispatch_layout(idx, E, R, p, 0)
    x = bits(synth.normal_bf16(T, H, 3, 3))
    wire = from_bits(oracle.dispatch_permute(x, Ld["row_token"]))
    hooks(poll_limit=1000, expand_skip_unit=0)
    st = md.new_status(DEV)
    md.md_dedup_expand(wire, i32(Ld["row_of_slot"]), i32(Ld["assign_row"]), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == md.MD_ERR_TIMEOUT
    md.md_set_test_hooks()
    st = md.new_status(DEV)
    out = md.md_dedup_expand(wire, i32(Ld["row_of_slot"]), i32(Ld["assign_row"]), dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == md.MD_OK
    assert np.array_equal(bits(out), oracle.dispatch_permute(x, Lc["row_token"]))
