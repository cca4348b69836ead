"""Run selected steps of the path a few times on a synthetic workload, for
profiling a single kernel under ncu on a small case.

    python -m combine_warp_top_router_b200.profile_case --steps layout,permute \
        --workload zipf_pairs_e128_k8 --T 16384 --reps 3

Steps: topk, layout, permute, combine, wire, expand, coselect, place, shuffle, shuffle_rounds,
shuffle_pair (three_layer_e128_k6 only), gather.
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
    rows = any(s in steps for s in ("permute", "combine", "wire", "expand", "gather"))
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
            else:
                raise SystemExit(f"unknown step {s}")

    for _ in range(1 + a.reps):
        once()
    torch.cuda.synchronize()
    print("ok", a.workload, "T", T, "steps", steps, "reps", a.reps)


if __name__ == "__main__":
    main()
