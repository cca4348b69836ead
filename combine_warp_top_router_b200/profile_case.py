"""Run selected steps of the path a few times on a synthetic workload, for
profiling a single kernel under ncu on a small case.

    python -m combine_warp_top_router_b200.profile_case --steps layout,permute \
        --workload zipf_pairs_e128_k8 --T 16384 --reps 3

Steps: topk, layout, permute, combine, wire, expand, coselect, place, shuffle, shuffle_rounds,
shuffle_pair (three_layer_e128_k6 only), gather, exchange (the EP exchange with every rank on
this GPU: R dispatch-exchange calls, R partials calls, R combine-exchange calls).
Every listed step runs once as warm-up and then `reps` times.
"""
from __future__ import annotations

import argparse

import torch

from . import binding as md
from . import synth


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--steps", default="topk,layout,permute,combine")
    ap.add_argument("--workload", default="zipf_pairs_e128_k8")
    ap.add_argument("--T", type=int, default=None)
    ap.add_argument("--H", type=int, default=None)
    ap.add_argument("--R", type=int, default=None)
    ap.add_argument("--mode", choices=["dedup", "conv"], default="dedup")
    ap.add_argument("--reps", type=int, default=3)
    a = ap.parse_args()
    steps = a.steps.split(",")
    dev = torch.device("cuda", 0)
    rows = any(s in steps for s in ("permute", "combine", "wire", "expand", "gather", "exchange"))
    w = synth.make_workload(a.workload, device=dev, T=a.T, H=a.H, R=a.R, with_rows=rows)
    mode = md.MD_DEDUP if a.mode == "dedup" else md.MD_CONV
    T, E, k, R = w.T, w.E, w.k, w.R
    idx, gates = md.md_route_topk(w.logits, k)
    L = md.md_dispatch_layout(idx, E, R, w.expert_to_rank, mode)
    ws = md.alloc_workspace(md.dispatch_layout_workspace_size(T, E, k, R, mode), dev)
    nxt = w.logits_next if w.logits_next is not None else w.logits
    idx2, _ = md.md_route_topk(nxt, k)
    W, C = md.md_coselect_stats(idx, idx2, E, T_fit=w.fit_tokens or T)
    buf = torch.empty(L.row_capacity, w.H, dtype=torch.bfloat16, device=dev) if rows else None
    out = torch.empty(T, w.H, dtype=torch.bfloat16, device=dev) if rows else None
    z = torch.empty(L.row_capacity, w.H, dtype=torch.bfloat16, device=dev) if "wire" in steps else None
    xc = torch.empty(T * k, w.H, dtype=torch.bfloat16, device=dev) if "expand" in steps else None
    if "shuffle_pair" in steps:
        if w.logits_prev is None:
            raise SystemExit("shuffle_pair needs a three-layer workload")
        idx0, _ = md.md_route_topk(w.logits_prev, k)
        C2 = md.md_coselect_pair_stats(idx0, idx, idx2, E, T_fit=w.fit_tokens or T)
    ex = _exchange_setup(w, idx, gates, dev) if "exchange" in steps else None
    torch.cuda.synchronize()

    def once():
        for s in steps:
            if s == "topk":
                md.md_route_topk(w.logits, k, topk_idx=idx, topk_w=gates)
            elif s == "layout":
                md.md_dispatch_layout(idx, E, R, w.expert_to_rank, mode, out=L, workspace=ws)
            elif s == "permute":
                md.md_dispatch_permute(w.x, L.row_of_slot, out=buf)
            elif s == "combine":
                md.md_combine(w.y, L.assign_row, idx, gates, out=out)
            elif s == "wire":
                md.md_combine(w.y, L.assign_row, idx, gates, md.MD_COMBINE_WIRE,
                              row_of_slot=L.row_of_slot, z=z, out=out)
            elif s == "expand":
                md.md_dedup_expand(buf, L.row_of_slot, L.assign_row, out=xc)
            elif s == "shuffle_pair":
                md.md_token_shuffle_pair(idx0, idx, C, C2, w.expert_to_rank, R, 8 * k)
            elif s == "coselect":
                md.md_coselect_stats(idx, idx2, E, T_fit=w.fit_tokens or T, W=W, C=C)
            elif s == "place":
                md.md_place_correlated(W, R)
            elif s == "shuffle":
                md.md_token_shuffle(idx, C, w.expert_to_rank, R)
            elif s == "shuffle_rounds":
                md.md_token_shuffle_rounds(idx, C, w.expert_to_rank, R)
            elif s == "gather":
                md.md_gather_rows(w.x, torch.arange(T, dtype=torch.int32, device=dev).flip(0))
            elif s == "exchange":
                _exchange_run(w, idx, gates, ex)
            else:
                raise SystemExit(f"unknown step {s}")

    for _ in range(1 + a.reps):
        once()
    torch.cuda.synchronize()
    print("ok", a.workload, "T", T, "steps", steps, "reps", a.reps)


def _exchange_setup(w, idx, gates, dev):
    """Every source rank's own layout, the plan, and R sets of receive and
    return buffers (all on this GPU); each destination's expert rows are the
    conventional rows of y (identity experts)."""
    T, H, E, k, R = w.T, w.H, w.E, w.k, w.R
    Tr = T // R
    p = w.expert_to_rank
    local = [md.md_dispatch_layout(idx[s * Tr:(s + 1) * Tr], E, R, p, md.MD_DEDUP) for s in range(R)]
    gathered = torch.stack([L.rank_offsets for L in local]).cpu().to(torch.int64)
    plans = [md.md_exchange_plan(gathered, s) for s in range(R)]
    caps = [plans[d][1][R] for d in range(R)]
    G = md.md_dispatch_layout(idx, E, R, p, md.MD_DEDUP)
    ro = G.rank_offsets.cpu().tolist()
    carried = (G.row_mask[:ro[R]].view(-1, 1) >> torch.arange(k, device=dev).view(1, -1)) & 1
    yr = torch.where(carried.bool(), G.assign_row[G.row_token[:ro[R]].long()], -1).to(torch.int32)
    buf = lambda *shape, dt=torch.bfloat16: [torch.empty(max(c, 1), *shape, dtype=dt, device=dev)
                                             for c in caps]
    ex = dict(Tr=Tr, local=local, plans=plans, caps=caps, recv=buf(H), tok=buf(dt=torch.int32),
              sidx=buf(k, dt=torch.int32), sw=buf(k, dt=torch.float32), ret=buf(H),
              y_row=[yr[ro[d]:ro[d + 1]].contiguous() for d in range(R)],
              out=torch.empty(T, H, dtype=torch.bfloat16, device=dev))
    return ex


def _exchange_run(w, idx, gates, ex):
    E, R, H = w.E, w.R, w.H
    Tr, plans, caps = ex["Tr"], ex["plans"], ex["caps"]
    for s in range(R):
        sl = slice(s * Tr, (s + 1) * Tr)
        peers = [md.PeerRows(rows=ex["recv"][d], token=ex["tok"][d], slot_idx=ex["sidx"][d],
                             slot_w=ex["sw"][d], row_base=plans[s][0][d], rows_cap=caps[d])
                 for d in range(R)]
        md.md_dispatch_exchange(w.x[sl], idx[sl], gates[sl], w.expert_to_rank, E,
                                ex["local"][s].row_of_slot, ex["local"][s].rank_offsets, s * Tr, peers)
    for d in range(R):
        md.md_combine_partials(w.y, ex["y_row"][d], ex["sidx"][d][:caps[d]], ex["sw"][d][:caps[d]],
                               out=ex["ret"][d][:caps[d]])
    for s in range(R):
        sl = slice(s * Tr, (s + 1) * Tr)
        peers = [md.PeerRows(rows=ex["ret"][d], row_base=plans[s][0][d], rows_cap=caps[d])
                 for d in range(R)]
        md.md_combine_exchange(peers, idx[sl], w.expert_to_rank, E, ex["local"][s].row_of_slot,
                               ex["local"][s].rank_offsets, H, out=ex["out"][sl])


if __name__ == "__main__":
    main()
