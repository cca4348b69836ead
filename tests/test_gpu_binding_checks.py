"""The Python binding refuses buffers that are too small for what a kernel
would write, before anything is enqueued."""
import pytest
import torch

import combine_warp_top_router_b200 as md

from _util import DEV

pytestmark = pytest.mark.gpu


def test_small_outputs_are_refused():
    T, E, k, R, H = 64, 16, 2, 4, 64
    logits = torch.randn(T, E, device=DEV)
    with pytest.raises(ValueError):
        md.md_route_topk(logits, k, topk_idx=torch.empty(T * k - 1, dtype=torch.int32, device=DEV))
    idx, gates = md.md_route_topk(logits, k)
    p = (torch.arange(E, device=DEV) // (E // R)).to(torch.int32)
    L = md.alloc_layout(T, E, k, R, md.MD_DEDUP, DEV)
    L.row_token = L.row_token[:-1]
    with pytest.raises(ValueError):
        md.md_dispatch_layout(idx, E, R, p, md.MD_DEDUP, out=L)
    L = md.md_dispatch_layout(idx, E, R, p, md.MD_DEDUP)
    y = torch.zeros(T * k, H, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ValueError):
        md.md_combine(y, L.assign_row, idx, gates,
                      out=torch.empty(T - 1, H, dtype=torch.bfloat16, device=DEV))
    x = torch.zeros(T, H, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ValueError):
        md.md_dispatch_permute(x, L.row_of_slot, out=torch.empty(8, H // 2, dtype=torch.bfloat16,
                                                                 device=DEV))
    W, C = md.md_coselect_stats(idx, idx, E)
    with pytest.raises(ValueError):
        md.md_coselect_stats(idx, idx, E, W=torch.empty(E * E - 1, dtype=torch.int32, device=DEV))
    with pytest.raises(ValueError):
        md.md_token_shuffle(idx, C, p, R, pred_rank=torch.empty(T - 1, dtype=torch.int32, device=DEV))
    with pytest.raises(ValueError):
        md.md_place_correlated(W, R, out=torch.empty(E - 1, dtype=torch.int32, device=DEV))
    with pytest.raises(ValueError):
        md.md_rank_stats(idx, E, R, p, hist=torch.empty(k, dtype=torch.int64, device=DEV))
    torch.cuda.synchronize()
