"""Guard bands: every output buffer sits inside a larger allocation whose
margins (4 KiB before and after) are poison-filled; after the call the margins
must be intact, so no kernel writes outside the buffer it was given."""
import numpy as np
import pytest
import torch

import combine_warp_top_router_b200 as md
import oracle
from combine_warp_top_router_b200 import synth

from _util import DEV, bits, from_bits, i32

pytestmark = pytest.mark.gpu

MARGIN = 4096          # bytes on each side
POISON = 0x5A


class Guarded:
    """A tensor of `shape`/`dtype` inside a byte buffer with poisoned margins."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape)) * torch.empty(0, dtype=dtype).element_size()
        self.raw = torch.full((MARGIN + n + MARGIN,), POISON, dtype=torch.uint8, device=DEV)
        self.t = self.raw[MARGIN:MARGIN + n].view(dtype).view(*shape)
        self.n = n

    def intact(self):
        r = self.raw.cpu().numpy()
        return bool(np.all(r[:MARGIN] == POISON) and np.all(r[MARGIN + self.n:] == POISON))


@pytest.mark.parametrize("H", [256, 2048])
def test_path_writes_stay_inside_their_buffers(H):
    w = synth.make_workload("zipf_pairs_e128_k8", T=2048, H=H)
    T, E, k, R = w.T, w.E, w.k, w.R
    logits = w.logits.to(DEV)
    idx = Guarded((T, k), torch.int32)
    gates = Guarded((T, k), torch.float32)
    md.md_route_topk(logits, k, topk_idx=idx.t, topk_w=gates.t)
    L = md.alloc_layout(T, E, k, R, md.MD_DEDUP, DEV)
    g = {n: Guarded(tuple(getattr(L, n).shape), getattr(L, n).dtype)
         for n in ("row_of_slot", "assign_row", "row_token", "row_mask", "send_counts",
                   "expert_counts", "expert_offsets", "rank_offsets", "n_rows")}
    for n, gg in g.items():
        setattr(L, n, gg.t)
    md.md_dispatch_layout(idx.t, E, R, w.expert_to_rank.to(DEV), md.MD_DEDUP, out=L)
    buf = Guarded((L.row_capacity, H), torch.bfloat16)
    md.md_dispatch_permute(w.x.to(DEV), L.row_of_slot, out=buf.t)
    out = Guarded((T, H), torch.bfloat16)
    md.md_combine(w.y.to(DEV), L.assign_row, idx.t, gates.t, out=out.t)
    z = Guarded((L.row_capacity, H), torch.bfloat16)
    wire = Guarded((T, H), torch.bfloat16)
    md.md_combine(w.y.to(DEV), L.assign_row, idx.t, gates.t, md.MD_COMBINE_WIRE,
                  row_of_slot=L.row_of_slot, z=z.t, out=wire.t)
    xc = Guarded((T * k, H), torch.bfloat16)
    md.md_dedup_expand(buf.t, L.row_of_slot, L.assign_row, out=xc.t)
    torch.cuda.synchronize()
    for name, gg in [("idx", idx), ("gates", gates), ("permute", buf), ("combine", out),
                     ("wire z", z), ("wire out", wire), ("expand", xc)] + list(g.items()):
        assert gg.intact(), name
    # and the results are the oracle's
    oi, ow = oracle.route_topk(w.logits.numpy(), k)
    OL = oracle.dispatch_layout(oi, E, R, w.expert_to_rank.numpy(), 1)
    assert np.array_equal(idx.t.cpu().numpy(), oi)
    assert np.array_equal(bits(buf.t)[:OL["n_rows"]], oracle.dispatch_permute(bits(w.x), OL["row_token"]))
    assert np.array_equal(bits(out.t), oracle.combine(bits(w.y), OL["assign_row"], oi, ow))


def test_planner_writes_stay_inside_their_buffers():
    w = synth.make_workload("three_layer_e128_k6", T=4096, with_rows=False)
    E, k, R = w.E, w.k, w.R
    a, b, c = (md.md_route_topk(lg.to(DEV), k)[0] for lg in (w.logits_prev, w.logits, w.logits_next))
    W = Guarded((E, E), torch.int32)
    C = Guarded((E, E), torch.int32)
    md.md_coselect_stats(b, c, E, W=W.t, C=C.t)
    C2 = Guarded((E, E, E), torch.int32)
    md.md_coselect_pair_stats(a, b, c, E, C2=C2.t)
    p = Guarded((E,), torch.int32)
    md.md_place_correlated(W.t, R, out=p.t)
    q = Guarded((E,), torch.int32)
    md.md_place_two_level(W.t, R, 4, 0, md.MD_REFINE_KL, out=q.t)
    outs = [Guarded((w.T,), torch.int32) for _ in range(3)]
    md.md_token_shuffle(b, C.t, w.expert_to_rank.to(DEV), R, *[o.t for o in outs])
    pouts = [Guarded((w.T,), torch.int32) for _ in range(4)]
    md.md_token_shuffle_pair(a, b, C.t, C2.t, w.expert_to_rank.to(DEV), R, 48, *[o.t for o in pouts])
    hist = Guarded((k + 1,), torch.int64)
    md.md_rank_stats(b, E, R, p.t, hist=hist.t)
    torch.cuda.synchronize()
    for name, gg in [("W", W), ("C", C), ("C2", C2), ("placement", p), ("placement kl", q),
                     ("hist", hist)] + [(f"shuffle {i}", o) for i, o in enumerate(outs)] + \
            [(f"pair shuffle {i}", o) for i, o in enumerate(pouts)]:
        assert gg.intact(), name
