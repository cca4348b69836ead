"""ep.py's per-rank orchestration on real hardware, as a one-rank NCCL group.

The exchange kernels are checked with many ranks played on one GPU in
test_gpu_exchange.py.  Here the plumbing around them runs as it would on
every rank of a multi-GPU job: a NCCL process group, receive buffers from
torch symmetric memory (rendezvous, peer pointers), the all-gather of the
layout offsets, the plan, the dispatch, the receiver's partial sums and the
combine.  With one rank every row stays on this GPU; the outputs must be the
oracle's (dedup layout rows for the dispatch, the fused combine -- with one
rank the wire form rounds one partial per token, which changes nothing)."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch

import combine_warp_top_router_b200 as md
import oracle
from combine_warp_top_router_b200 import ep, synth

from _util import DEV, bits, f32, i32

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.fixture
def one_rank_group():
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        yield dist.group.WORLD
    finally:
        torch.cuda.synchronize()
        dist.destroy_process_group()


@pytest.mark.parametrize("symmetric", [True, False])
def test_ep_dispatch_and_combine_one_rank(one_rank_group, symmetric):
    T, H = 2048, 512
    w = synth.make_workload("zipf_pairs_e128_k8", seed=3, T=T, H=H, R=1)
    E, k = w.E, w.k
    oi, ow = oracle.route_topk(w.logits.numpy(), k)
    p = np.zeros(E, np.int32)  # one rank holds every expert
    idx, gates, pg = i32(oi), f32(ow), i32(p)
    bufs = ep.ExchangeBuffers(T, H, k, DEV, group=one_rank_group, symmetric=symmetric)
    st = md.new_status(DEV)
    L, n = ep.dispatch(w.x.to(DEV), idx, gates, pg, E, bufs, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == md.MD_OK
    O = oracle.dispatch_layout(oi, E, 1, p, oracle.DEDUP)
    assert n == O["n_rows"] == T
    assert np.array_equal(bits(bufs.local["rows"][:n]), oracle.dispatch_permute(bits(w.x), O["row_token"]))
    assert np.array_equal(bufs.local["token"][:n].cpu().numpy(), O["row_token"])
    assert np.array_equal(bufs.local["slot_idx"][:n].cpu().numpy(), oi[O["row_token"]])
    assert np.array_equal(bufs.local["slot_w"][:n].cpu().numpy(), ow[O["row_token"]])
    # the receiver's experts: identity stand-ins whose outputs are y's
    # conventional rows; every received row carries all k slots here
    y_row = i32(O["assign_row"][O["row_token"]])
    md.md_combine_partials(w.y.to(DEV), y_row, bufs.local["slot_idx"][:n], bufs.local["slot_w"][:n],
                           out=bufs.local["ret"][:n], dev_status=st)
    out = ep.combine(L, idx, pg, E, bufs, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == md.MD_OK
    want = oracle.combine(bits(w.y), O["assign_row"], oi, ow)
    assert np.array_equal(bits(out), want)
