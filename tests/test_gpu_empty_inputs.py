"""Empty inputs through the entry points that the other files exercise only with
tokens: T = 0 (or no rows) returns MD_OK, leaves the status word clear, and
writes nothing outside what the call defines (tables it zeroes come back zero,
canary-filled outputs keep their canaries)."""
import pytest
import torch

import combine_warp_top_router_b200 as md

from _util import DEV

pytestmark = pytest.mark.gpu

E, k, R, H = 64, 4, 8, 256
CANARY = -7


def _i32(*shape, fill=CANARY):
    return torch.full(shape, fill, dtype=torch.int32, device=DEV)


def _ok(st):
    torch.cuda.synchronize()
    assert int(st.item()) == md.MD_OK


def test_movement_with_no_tokens():
    st = md.new_status(DEV)
    x = torch.empty(0, H, dtype=torch.bfloat16, device=DEV)
    none = torch.empty(0, k, dtype=torch.int32, device=DEV)
    w = torch.empty(0, k, dtype=torch.float32, device=DEV)
    buf = torch.full((4, H), 3.0, dtype=torch.bfloat16, device=DEV)
    md.md_dispatch_permute(x, none, out=buf, dev_status=st)
    _ok(st)
    assert bool((buf == 3.0).all())
    y = torch.ones(4, H, dtype=torch.bfloat16, device=DEV)
    out = md.md_combine(y, none, none, w, dev_status=st)
    _ok(st)
    assert out.shape == (0, H)
    z = torch.full((4, H), 5.0, dtype=torch.bfloat16, device=DEV)
    md.md_combine(y, none, none, w, md.MD_COMBINE_WIRE, row_of_slot=none, z=z, dev_status=st)
    _ok(st)
    assert bool((z == 5.0).all())
    # no rows gathered from a non-empty source
    src = torch.ones(16, H, dtype=torch.bfloat16, device=DEV)
    g = md.md_gather_rows(src, torch.empty(0, dtype=torch.int32, device=DEV), dev_status=st)
    _ok(st)
    assert g.shape == (0, H)


def test_tables_with_no_tokens_are_zero():
    st = md.new_status(DEV)
    none = torch.empty(0, k, dtype=torch.int32, device=DEV)
    W = torch.full((E, E), 9, dtype=torch.int32, device=DEV)
    C = torch.full((E, E), 9, dtype=torch.int32, device=DEV)
    md.md_coselect_stats(none, none, E, W=W, C=C, dev_status=st)
    _ok(st)
    assert int(W.abs().sum()) == 0 and int(C.abs().sum()) == 0
    C2 = torch.full((E, E, E), 9, dtype=torch.int32, device=DEV)
    md.md_coselect_pair_stats(none, none, none, E, C2=C2, dev_status=st)
    _ok(st)
    assert int(C2.abs().sum()) == 0


def test_shuffles_with_no_tokens():
    st = md.new_status(DEV)
    none = torch.empty(0, k, dtype=torch.int32, device=DEV)
    p = torch.arange(E, dtype=torch.int32, device=DEV) // (E // R)
    C = torch.ones(E, E, dtype=torch.int32, device=DEV)
    C2 = torch.ones(E, E, E, dtype=torch.int32, device=DEV)
    for out in (md.md_token_shuffle(none, C, p, R, dev_status=st),
                md.md_token_shuffle_rounds(none, C, p, R, dev_status=st),
                md.md_token_shuffle_pair(none, none, C, C2, p, R, 8, dev_status=st)):
        _ok(st)
        assert all(o.numel() == 0 for o in out[:3])


def test_exchange_with_no_tokens():
    st = md.new_status(DEV)
    Rx = 2
    none = torch.empty(0, k, dtype=torch.int32, device=DEV)
    x = torch.empty(0, H, dtype=torch.bfloat16, device=DEV)
    p = torch.arange(E, dtype=torch.int32, device=DEV) // (E // Rx)
    ro = torch.zeros(Rx + 1, dtype=torch.int32, device=DEV)
    cap = 4
    bufs = [dict(rows=torch.full((cap, H), 2.0, dtype=torch.bfloat16, device=DEV),
                 token=_i32(cap), slot_idx=_i32(cap, k),
                 slot_w=torch.zeros(cap, k, dtype=torch.float32, device=DEV)) for _ in range(Rx)]
    peers = [md.PeerRows(rows=b["rows"], row_base=0, rows_cap=cap, token=b["token"],
                         slot_idx=b["slot_idx"], slot_w=b["slot_w"]) for b in bufs]
    md.md_dispatch_exchange(x, none, torch.empty(0, k, dtype=torch.float32, device=DEV), p, E,
                            none, ro, 0, peers, dev_status=st)
    _ok(st)
    for b in bufs:
        assert bool((b["rows"] == 2.0).all()) and bool((b["token"] == CANARY).all())
    z = md.md_combine_partials(torch.ones(4, H, dtype=torch.bfloat16, device=DEV), none, none,
                               torch.empty(0, k, dtype=torch.float32, device=DEV), dev_status=st)
    _ok(st)
    assert z.shape == (0, H)
    ret = [md.PeerRows(rows=b["rows"], row_base=0, rows_cap=cap) for b in bufs]
    out = md.md_combine_exchange(ret, none, p, E, none, ro, H, dev_status=st)
    _ok(st)
    assert out.shape == (0, H)
