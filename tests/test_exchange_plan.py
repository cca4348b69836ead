"""md_exchange_plan and the count exchange of the EP path, on the CPU.

Every source rank lays out its own block of tokens; after the all-gather of
those layouts' rank offsets, the plan must place every row exactly where the
single-GPU layout of all tokens puts it: for token t of source s and its
row on rank d,
    global row = rank_offsets[d] + dst_row_base_s[d] + (local row - local rank_offsets_s[d]).
The layouts here are the oracle's (the library's own layout is checked
against it on the GPU).  The multi-process test runs the all-gather on gloo
with two ranks, as a two-GPU job would on NCCL."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from combine_warp_top_router_b200 import binding as md
from combine_warp_top_router_b200 import ep, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _routes(name, T, R, seed=0):
    w = synth.make_workload(name, seed=seed, T=T, R=R, with_rows=False)
    return oracle.route_topk(w.logits.numpy(), w.k)[0], w.E


def _check_source(s, R, Tr, idx, E, p, G, base, local_ro, local_ros):
    """Every row of source s lands at its row of the global layout."""
    k = idx.shape[1]
    for tl in range(Tr):
        t = s * Tr + tl
        for j in range(k):
            d = p[idx[t, j]]
            lr = local_ros[tl, j]
            assert G["rank_offsets"][d] + base[d] + (lr - local_ro[d]) == G["row_of_slot"][t, j]


@pytest.mark.parametrize("name,T,R,mode", [("zipf_pairs_e128_k8", 1024, 4, 1),
                                           ("iid_e64_k6", 4096, 16, 1),
                                           ("full_e256_k8", 4096, 64, 1),
                                           ("iid_e64_k6", 1024, 8, 0)])
def test_plan_places_rows_like_the_single_gpu_layout(name, T, R, mode):
    idx, E = _routes(name, T, R)
    p = synth.contiguous_placement(E, R).numpy()
    p = np.random.default_rng(3).permutation(p).astype(np.int32)
    G = oracle.dispatch_layout(idx, E, R, p, mode)
    Tr = T // R
    locs = [oracle.dispatch_layout(idx[s * Tr:(s + 1) * Tr], E, R, p, mode) for s in range(R)]
    gathered = np.stack([L["rank_offsets"] for L in locs]).astype(np.int64)
    plans = [md.md_exchange_plan(gathered, s) for s in range(R)]
    for s in range(R):
        base, recv = plans[s]
        if mode == 1:
            # dedup: the same (d, t) order as the single-GPU layout
            _check_source(s, R, Tr, idx, E, p, G, base, locs[s]["rank_offsets"],
                          locs[s]["row_of_slot"])
        # the receive buffer of rank s holds its whole block of the global layout
        assert recv[R] == G["rank_offsets"][s + 1] - G["rank_offsets"][s]
        assert recv == [0] + list(np.cumsum(G["send_counts"][:, s]))
    # on every destination the sources' blocks tile its receive buffer in
    # source order (conventional rows arrive by (source, expert, token))
    for d in range(R):
        run = 0
        for s in range(R):
            assert plans[s][0][d] == run
            run += gathered[s, d + 1] - gathered[s, d]
        assert run == plans[d][1][R]
    # the gathered counts are the global send matrix (sources are contiguous blocks)
    assert np.array_equal(np.diff(gathered, axis=1), G["send_counts"])


def test_plan_rejects_bad_offsets():
    good = [[0, 2, 5], [0, 1, 1]]
    assert md.md_exchange_plan(good, 1) == ([2, 3], [0, 3, 3])
    with pytest.raises(md.MoeDispatchError):
        md.md_exchange_plan([[0, 2, 1], [0, 1, 1]], 0)     # decreasing
    with pytest.raises(md.MoeDispatchError):
        md.md_exchange_plan([[1, 2, 3], [0, 1, 1]], 0)     # does not start at 0
    with pytest.raises(md.MoeDispatchError):
        md.md_exchange_plan(good, 2)                       # no such rank


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime

    import torch.distributed as dist

    import oracle as orc
    from combine_warp_top_router_b200 import binding as mdb
    from combine_warp_top_router_b200 import ep as epm
    from combine_warp_top_router_b200 import synth as sy
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        R, T = world, 512 * world
        w = sy.make_workload("zipf_pairs_e128_k8", seed=2, T=T, R=R, with_rows=False)
        idx = orc.route_topk(w.logits.numpy(), w.k)[0]
        p = w.expert_to_rank.numpy()
        Tr = T // R
        L = orc.dispatch_layout(idx[rank * Tr:(rank + 1) * Tr], w.E, R, p, 1)
        gathered = epm.gather_rank_offsets(torch.from_numpy(L["rank_offsets"]))
        base, recv = epm.plan(gathered, rank)
        q.put((rank, gathered.numpy().tolist(), base, recv))
    finally:
        dist.destroy_process_group()


def test_count_exchange_on_two_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    out = sorted(q.get(timeout=240) for _ in range(world))
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    # the same computation in one process
    R, T = world, 512 * world
    w = synth.make_workload("zipf_pairs_e128_k8", seed=2, T=T, R=R, with_rows=False)
    idx = oracle.route_topk(w.logits.numpy(), w.k)[0]
    p = w.expert_to_rank.numpy()
    G = oracle.dispatch_layout(idx, w.E, R, p, 1)
    Tr = T // R
    locs = [oracle.dispatch_layout(idx[s * Tr:(s + 1) * Tr], w.E, R, p, 1) for s in range(R)]
    for rank, gathered, base, recv in out:
        assert gathered == [list(L["rank_offsets"]) for L in locs]   # every rank sees every row
        _check_source(rank, R, Tr, idx, w.E, p, G, base, locs[rank]["rank_offsets"],
                      locs[rank]["row_of_slot"])
        assert recv[R] == G["rank_offsets"][rank + 1] - G["rank_offsets"][rank]
