"""Benchmark: MoE dispatch + combine throughput on B200.

One step = one pass of the per-layer hot path over one batch:
    md_route_topk -> md_dispatch_layout (dedup) -> md_dispatch_permute -> md_combine
on the workload "zipf_pairs_e128_k8" (T=65536 tokens, hidden 2048 bf16, E=128,
top-8, 16 virtual EP ranks, correlated Zipf(1.1) pair logits, contiguous
placement).  Inputs are synthetic, seeded, resident in HBM, and larger than L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

Under torchrun each rank runs an independent replica on its own GPU (the
virtual EP ranks live inside one GPU; nothing is sharded), times K steps with
CUDA events, and rank 0 prints one JSON line with the max over ranks.
--impl reference times the CPU oracle on the host instead (bounded samples).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "dispatch+combine Mtokens/s at 1 B200; achieved HBM GB/s vs ~8 TB/s peak"
UNIT = "Mtokens/s"
WORKLOAD = "zipf_pairs_e128_k8"
NOMINAL_HBM_GBS = 8000.0    # B200 HBM3e, nominal (context only; the roofline uses the measured peak)
FALLBACK_HBM_GBS = 6650.0
CPU_TOKENS_PER_S_GUESS = 16000.0  # oracle, one core, this workload's shape


# ------------------------------------------------------------- environment

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(ws, backend):
    if ws <= 1:
        return None
    import datetime
    import torch.distributed as dist
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(dist, value: float, device) -> float:
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist, device):
    if dist is not None:
        dist.barrier(device_ids=[device.index] if device.type == "cuda" else None)


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 50):
        self.gpu_index = gpu_index
        self.period_ms = period_ms
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu_index), "-lms", str(self.period_ms)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        if not self.lines:
            return None
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------ bytes model

def algorithmic_bytes(T, H, k, E, n_rows):
    """Bytes each kernel must move (inputs read once, outputs written once)."""
    return {
        "route_topk": T * (4 * E + 8 * k),
        "dispatch_layout": T * k * (4 + 8) + n_rows * 8,
        "dispatch_permute": T * (2 * H + 4 * k) + n_rows * 2 * H,
        "combine": T * (2 * H * (k + 1) + 12 * k),
    }


def kernel_traffic(name, launches_units, units_per_launch):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current source of the kernel; else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(name)
    except Exception:
        return None
    if not rec:
        return None
    src = os.path.join(ROOT, "combine_warp_top_router_b200", "csrc", rec["source"])
    try:
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    except Exception:
        return None
    if digest != rec.get("source_sha256_16"):
        return None
    return rec["dram_bytes_per_unit"] * units_per_launch


# -------------------------------------------------------------- native arm

def run_native(args):
    import combine_warp_top_router_b200 as md
    from combine_warp_top_router_b200 import synth

    ws, rank, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist = init_dist(ws, "nccl")
    md.lib()  # fail loudly if the library is missing

    w = synth.make_workload(WORKLOAD, seed=args.seed, device=device)
    T, H, E, k, R = w.T, w.H, w.E, w.k, w.R
    mode = md.MD_DEDUP if args.dispatch == "dedup" else md.MD_CONV
    stream = torch.cuda.Stream(device)
    cap = T * k if mode == md.MD_CONV else T * min(k, R)
    idx = torch.empty(T, k, dtype=torch.int32, device=device)
    gates = torch.empty(T, k, dtype=torch.float32, device=device)
    L = md.alloc_layout(T, E, k, R, mode, device)
    wsp = md.alloc_workspace(md.dispatch_layout_workspace_size(T, E, k, R, mode), device)
    buf = torch.empty(cap, H, dtype=torch.bfloat16, device=device)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=device)
    status = md.new_status(device)
    torch.cuda.synchronize()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        md.md_route_topk(w.logits, k, md.MD_GATE_TOPK_SOFTMAX, idx, gates, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        md.md_dispatch_layout(idx, E, R, w.expert_to_rank, mode, out=L, workspace=wsp,
                              dev_status=status, stream=stream)
        if ev is not None:
            ev[2].record(stream)
        md.md_dispatch_permute(w.x, L.row_of_slot, out=buf, stream=stream)
        if ev is not None:
            ev[3].record(stream)
        md.md_combine(w.y, L.assign_row, idx, gates, out=out, stream=stream)
        if ev is not None:
            ev[4].record(stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    stream.synchronize()
    md.check_status(status, "layout status after warm-up")

    events = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    barrier(dist, device)
    torch.cuda.synchronize()
    launches0 = md.launch_count()
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        with torch.cuda.stream(stream):
            for i in range(args.steps):
                step(events[i])
        stream.synchronize()
    launches = md.launch_count() - launches0
    torch.cuda.synchronize()
    barrier(dist, device)

    total_ms = events[0][0].elapsed_time(events[-1][4])
    per = {n: 0.0 for n in ("route_topk", "dispatch_layout", "dispatch_permute", "combine")}
    for ev in events:
        for j, n in enumerate(per):
            per[n] += ev[j].elapsed_time(ev[j + 1])
    per = {n: v / args.steps for n, v in per.items()}  # ms per launch
    total_ms_max = max_over_ranks(dist, total_ms, device)
    n_rows = int(L.n_rows.item())
    md.check_status(status, "layout status")

    # end to end through host buffers: inputs copied in, the result copied out
    e2e = run_e2e(args, md, w, mode, device, stream, idx, gates, L, wsp, buf, status, dist)

    if rank != 0:
        return None
    peaks = measured_peaks()
    peak = float(peaks["hbm_gbs"]) if peaks and "hbm_gbs" in peaks else FALLBACK_HBM_GBS
    peak_src = "of measured" if peaks and "hbm_gbs" in peaks else "of fallback"
    ab = algorithmic_bytes(T, H, k, E, n_rows)
    kernels = {n: {"us": round(per[n] * 1e3, 2), "bytes": ab[n],
                   "GBps": round(ab[n] / (per[n] * 1e-3) / 1e9, 1),
                   "frac": round(ab[n] / (per[n] * 1e-3) / 1e9 / peak, 3),
                   "frac_of_nominal_8TBps": round(ab[n] / (per[n] * 1e-3) / 1e9 / NOMINAL_HBM_GBS, 3)}
               for n in per}
    dom = max(("dispatch_permute", "combine"), key=lambda n: per[n])
    achieved = ab[dom] / (per[dom] * 1e-3) / 1e9
    traffic = kernel_traffic(dom, args.steps, T)
    value = T * args.steps * ws / (total_ms_max * 1e-3) / 1e6
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_ms_max / args.steps, 4), "higher_is_better": True,
        "dispatch_combine_excl_router": round(
            T * ws / ((per["dispatch_layout"] + per["dispatch_permute"] + per["combine"]) * 1e-3) / 1e6, 3),
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "T": T, "H": H, "E": E, "top_k": k, "ep_ranks": R,
                   "dispatch": args.dispatch, "combine": "fused", "gates": "topk_softmax",
                   "placement": "contiguous", "parallelism": f"replicas x{ws}",
                   "l2": "not flushed: every step moves >2.6 GB through HBM, 20x the 126 MB L2",
                   "dedup_rows_per_token": round(n_rows / T, 4)},
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1),
                     "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "peak_source": peak_src,
                     "traffic": None if traffic is None else int(traffic),
                     "algorithmic_bytes_per_launch": ab[dom]},
        "kernels": kernels,
        "gpu_launches": int(launches),
        "e2e": e2e,
        "clocks": clk.summary(),
    }
    if args.rows:
        del w, buf, out
        torch.cuda.empty_cache()
        line["rows"] = run_rows(args, md, device, stream, peak)
    line["cpu_baseline"] = cpu_baseline(args)
    return line


def _time(fn, stream, reps):
    """Average device time (ms) of fn() over reps launches on `stream`, after a warm-up.
    Inputs are produced on the default stream, which the (non-blocking) timing
    stream does not wait for: synchronise the device first."""
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        fn()
    stream.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
    stream.synchronize()
    return e0.elapsed_time(e1) / reps


def run_rows(args, md, device, stream, peak):
    """Every step of the path on the workload it belongs to (one GPU)."""
    from combine_warp_top_router_b200 import synth
    rows = {}
    reps = args.row_reps

    def gbps(nbytes, ms):
        return {"GBps": round(nbytes / (ms * 1e-3) / 1e9, 1), "frac": round(nbytes / (ms * 1e-3) / 1e9 / peak, 3)}

    # conventional dispatch and the two-stage (wire) combine, same workload as the headline
    w = synth.make_workload(WORKLOAD, seed=args.seed, device=device)
    T, H, E, k, R = w.T, w.H, w.E, w.k, w.R
    idx, gates = md.md_route_topk(w.logits, k)
    for name, mode in (("conv", md.MD_CONV), ("dedup", md.MD_DEDUP)):
        L = md.alloc_layout(T, E, k, R, mode, device)
        wsp = md.alloc_workspace(md.dispatch_layout_workspace_size(T, E, k, R, mode), device)
        buf = torch.empty(L.row_capacity, H, dtype=torch.bfloat16, device=device)
        out = torch.empty(T, H, dtype=torch.bfloat16, device=device)
        t_lay = _time(lambda: md.md_dispatch_layout(idx, E, R, w.expert_to_rank, mode, out=L,
                                                      workspace=wsp, stream=stream), stream, reps)
        n = int(L.n_rows.item())
        t_perm = _time(lambda: md.md_dispatch_permute(w.x, L.row_of_slot, out=buf, stream=stream),
                       stream, reps)
        t_comb = _time(lambda: md.md_combine(w.y, L.assign_row, idx, gates, out=out, stream=stream),
                       stream, reps)
        pb = T * (2 * H + 4 * k) + n * 2 * H
        cb = T * (2 * H * (k + 1) + 12 * k)
        r = {"rows_per_token": round(n / T, 4), "layout_us": round(t_lay * 1e3, 2),
             "permute_us": round(t_perm * 1e3, 2), "permute": gbps(pb, t_perm),
             "combine_us": round(t_comb * 1e3, 2), "combine": gbps(cb, t_comb),
             "dispatch_combine_Mtokens_per_s": round(T / ((t_lay + t_perm + t_comb) * 1e-3) / 1e6, 2)}
        if mode == md.MD_DEDUP:
            z = torch.empty(L.row_capacity, H, dtype=torch.bfloat16, device=device)
            t_wire = _time(lambda: md.md_combine(w.y, L.assign_row, idx, gates, md.MD_COMBINE_WIRE,
                                                 row_of_slot=L.row_of_slot, z=z, out=out,
                                                 stream=stream), stream, reps)
            wb = T * (2 * H * k + 2 * H + 16 * k) + n * 2 * H
            r["combine_wire_us"] = round(t_wire * 1e3, 2)
            r["combine_wire"] = gbps(wb, t_wire)
            del z
            # receiver side: dedup rows -> one row per (token, expert), expert-grouped
            xc = torch.empty(T * k, H, dtype=torch.bfloat16, device=device)
            t_exp = _time(lambda: md.md_dedup_expand(buf, L.row_of_slot, L.assign_row, out=xc,
                                                     stream=stream), stream, reps)
            eb = n * 2 * H + T * k * (2 * H + 8)
            r["dedup_expand_us"] = round(t_exp * 1e3, 2)
            r["dedup_expand"] = gbps(eb, t_exp)
            del xc
        rows[f"zipf_pairs_e128_k8_{name}"] = r
        del L, wsp, buf, out
    t_topk = _time(lambda: md.md_route_topk(w.logits, k, topk_idx=idx, topk_w=gates, stream=stream),
                   stream, reps)
    rows["route_topk_e128_k8"] = {"us": round(t_topk * 1e3, 2), **gbps(T * (4 * E + 8 * k), t_topk)}
    del w, idx, gates
    torch.cuda.empty_cache()

    # token shuffle on the two-layer workload (C fitted on the first 4096 tokens)
    w = synth.make_workload("two_layer_e128_k6", seed=args.seed, device=device)
    a, _ = md.md_route_topk(w.logits, w.k)
    b, _ = md.md_route_topk(w.logits_next, w.k)
    _, C = md.md_coselect_stats(a, b, w.E, T_fit=w.fit_tokens, want_W=False)
    sws = md.alloc_workspace(int(md.lib().md_token_shuffle_workspace_size(w.T, w.E, w.R)), device)
    pred = torch.empty(w.T, dtype=torch.int32, device=device)
    perm = torch.empty_like(pred)
    inv = torch.empty_like(pred)
    t_sh = _time(lambda: md.md_token_shuffle(a, C, w.expert_to_rank, w.R, pred, perm, inv,
                                             workspace=sws, stream=stream), stream, reps)
    xs = torch.empty_like(w.x)
    t_g = _time(lambda: md.md_gather_rows(w.x, inv, out=xs, stream=stream), stream, reps)
    loc_before = float((torch.arange(w.T, device=device) // (w.T // w.R)).eq(
        w.expert_to_rank[b.long()].T).float().mean())
    bs = b[inv.long()]
    loc_after = float((torch.arange(w.T, device=device) // (w.T // w.R)).eq(
        w.expert_to_rank[bs.long()].T).float().mean())
    # the rounds-based parallel assignment on the same inputs
    rws = md.alloc_workspace(int(md.lib().md_token_shuffle_rounds_workspace_size(w.T, w.E, w.R)),
                             device)
    rp, rperm, rinv = torch.empty_like(pred), torch.empty_like(pred), torch.empty_like(pred)
    holder = {}
    t_rd = _time(lambda: holder.__setitem__("r", md.md_token_shuffle_rounds(
        a, C, w.expert_to_rank, w.R, rp, rperm, rinv, workspace=rws, stream=stream)[3]), stream, reps)
    n_rounds = int(holder["r"].item())
    loc_rounds = float((torch.arange(w.T, device=device) // (w.T // w.R)).eq(
        w.expert_to_rank[b[rinv.long()].long()].T).float().mean())
    rows["token_shuffle_e128_k6"] = {
        "T": w.T, "shuffle_us": round(t_sh * 1e3, 2), "gather_x_us": round(t_g * 1e3, 2),
        "gather": gbps(2 * w.T * 2 * w.H + 4 * w.T, t_g),
        "locality_before": round(loc_before, 4), "locality_after": round(loc_after, 4),
        "rounds_variant": {"us": round(t_rd * 1e3, 2), "rounds": n_rounds,
                           "locality_after": round(loc_rounds, 4)}}
    del w, a, b, C, sws, xs
    torch.cuda.empty_cache()

    # pair-based shuffle prediction on the three-layer workload (counts fitted
    # on the first 4096 tokens; a pair row is used when its total reaches 8k)
    w = synth.make_workload("three_layer_e128_k6", seed=args.seed, device=device, with_rows=False)
    g = [md.md_route_topk(lg, w.k)[0] for lg in (w.logits_prev, w.logits, w.logits_next)]
    C2 = torch.empty(w.E, w.E, w.E, dtype=torch.int32, device=device)
    t_c2 = _time(lambda: md.md_coselect_pair_stats(g[0], g[1], g[2], w.E, T_fit=w.fit_tokens, C2=C2,
                                                   stream=stream), stream, reps)
    _, C = md.md_coselect_stats(g[1], g[2], w.E, T_fit=w.fit_tokens, want_W=False)
    pws = md.alloc_workspace(int(md.lib().md_token_shuffle_pair_workspace_size(w.T, w.E, w.R)), device)
    pred = torch.empty(w.T, dtype=torch.int32, device=device)
    perm, inv, use = torch.empty_like(pred), torch.empty_like(pred), torch.empty_like(pred)
    min_obs = 8 * w.k
    t_sp = _time(lambda: md.md_token_shuffle_pair(g[0], g[1], C, C2, w.expert_to_rank, w.R, min_obs,
                                                  pred, perm, inv, use, workspace=pws,
                                                  stream=stream), stream, reps)
    nxt_rank = w.expert_to_rank[g[2].long()]
    loc_pair = float(pred[:, None].eq(nxt_rank).float().mean())
    use_share = float(use.float().mean())
    sp = md.md_token_shuffle(g[1], C, w.expert_to_rank, w.R)[0]
    loc_single = float(sp[:, None].eq(nxt_rank).float().mean())
    loc_none = float((torch.arange(w.T, device=device) // (w.T // w.R))[:, None].eq(nxt_rank)
                     .float().mean())
    rows["token_shuffle_pair_e128_k6"] = {
        "T": w.T, "min_obs": min_obs, "pair_counts_us": round(t_c2 * 1e3, 2),
        "shuffle_pair_us": round(t_sp * 1e3, 2), "tokens_on_pair_rows": round(use_share, 4),
        "locality_no_shuffle": round(loc_none, 4), "locality_single": round(loc_single, 4),
        "locality_pair": round(loc_pair, 4)}
    del w, g, C2, C, pws
    torch.cuda.empty_cache()

    # the full pipeline at full size: T=262144, E=256, k=8, R=64
    w = synth.make_workload("full_e256_k8", seed=args.seed, device=device)
    T, H, E, k, R = w.T, w.H, w.E, w.k, w.R
    a = torch.empty(T, k, dtype=torch.int32, device=device)
    g = torch.empty(T, k, dtype=torch.float32, device=device)
    b = torch.empty_like(a)
    gb = torch.empty_like(g)
    W = torch.empty(E, E, dtype=torch.int32, device=device)
    C = torch.empty_like(W)
    p = torch.empty(E, dtype=torch.int32, device=device)
    pws = md.alloc_workspace(int(md.lib().md_place_correlated_workspace_size(E, R)), device)
    L = md.alloc_layout(T, E, k, R, md.MD_DEDUP, device)
    lws = md.alloc_workspace(md.dispatch_layout_workspace_size(T, E, k, R, md.MD_DEDUP), device)
    buf = torch.empty(L.row_capacity, H, dtype=torch.bfloat16, device=device)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=device)
    parts = {}

    def pipeline(ev=None):
        steps = [
            ("route_topk_x2", lambda: (md.md_route_topk(w.logits, k, topk_idx=a, topk_w=g, stream=stream),
                                       md.md_route_topk(w.logits_next, k, topk_idx=b, topk_w=gb,
                                                        stream=stream))),
            ("coselect_W_C", lambda: md.md_coselect_stats(a, b, E, W=W, C=C, stream=stream)),
            ("place_correlated", lambda: md.md_place_correlated(W, R, out=p, workspace=pws,
                                                                stream=stream)),
            ("dispatch_layout", lambda: md.md_dispatch_layout(a, E, R, p, md.MD_DEDUP, out=L,
                                                              workspace=lws, stream=stream)),
            ("dispatch_permute", lambda: md.md_dispatch_permute(w.x, L.row_of_slot, out=buf,
                                                                stream=stream)),
            ("combine", lambda: md.md_combine(w.y, L.assign_row, a, g, out=out, stream=stream)),
        ]
        for name, fn in steps:
            if ev is None:
                fn()
                continue
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            ev.append((name, e0, e1))

    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        pipeline()
    stream.synchronize()
    evs = []
    with torch.cuda.stream(stream):
        for _ in range(max(1, reps // 5)):
            pipeline(evs)
    stream.synchronize()
    for name, e0, e1 in evs:
        parts[name] = parts.get(name, 0.0) + e0.elapsed_time(e1) / max(1, reps // 5)
    total = sum(parts.values())
    n = int(L.n_rows.item())
    contiguous = synth.contiguous_placement(E, R, device)
    torch.cuda.synchronize()
    Lc = md.md_dispatch_layout(a, E, R, contiguous, md.MD_DEDUP)
    # placement refinements on this workload: best single swaps vs
    # Kernighan-Lin passes, one level vs 8 nodes of 8 GPUs
    modes = {}
    for label, nodes, refine in (("swaps", 1, md.MD_REFINE_SWAPS), ("kl", 1, md.MD_REFINE_KL),
                                 ("kl_8_nodes", 8, md.MD_REFINE_KL)):
        q = torch.empty(E, dtype=torch.int32, device=device)
        qws = md.alloc_workspace(int(md.lib().md_place_two_level_workspace_size(E, R, nodes)), device)
        t_q = _time(lambda: md.md_place_two_level(W, R, nodes, md.MD_SEED_CONTIGUOUS, refine, out=q,
                                                  workspace=qws, stream=stream), stream, 3)
        torch.cuda.synchronize()
        Lq = md.md_dispatch_layout(a, E, R, q, md.MD_DEDUP)
        modes[label] = {"us": round(t_q * 1e3, 1),
                        "rows_per_token": round(int(Lq.n_rows.item()) / T, 4)}
    rows["placement_modes_e256_k8"] = modes

    # the pages' routing statistics on this workload: Table I columns for both
    # placements, the cross-layer successor share, fitted vs held-out W
    s_corr = md.table1_row(md.md_rank_stats(a, E, R, p))
    s_cont = md.table1_row(md.md_rank_stats(a, E, R, contiguous))
    Wf, Cf = md.md_coselect_stats(a[:4096], b[:4096], E)
    Wh, _ = md.md_coselect_stats(a[4096:8192], None, E)
    num, den = md.md_successor_share(Cf, Wf)
    share = (num.double() / den.double().clamp(min=1)).cpu()
    rows["routing_stats_e256_k8"] = {
        "same_rank_pct": {"contiguous": round(s_cont[0], 2), "correlated": round(s_corr[0], 2)},
        "ranks_per_token": {"contiguous": round(s_cont[1], 3), "correlated": round(s_corr[1], 3)},
        "dedup_pct": {"contiguous": round(s_cont[2], 2), "correlated": round(s_corr[2], 2)},
        "experts_with_successor_share_ge_30pct": int((share >= 0.30).sum()),
        "median_successor_share": round(float(share.median()), 4),
        "pearson_W_fit4096_vs_next4096": round(md.pearson_from_sums(E * E, md.md_count_sums(Wf, Wh)), 4)}
    rows["full_e256_k8_pipeline"] = {
        "T": T, "ms": round(total, 3), "Mtokens_per_s": round(T / (total * 1e-3) / 1e6, 2),
        "parts_us": {kk: round(v * 1e3, 1) for kk, v in parts.items()},
        "rows_per_token_correlated": round(n / T, 4),
        "rows_per_token_contiguous": round(int(Lc.n_rows.item()) / T, 4),
        "permute": gbps(T * (2 * H + 4 * k) + n * 2 * H, parts["dispatch_permute"]),
        "combine": gbps(T * (2 * H * (k + 1) + 12 * k), parts["combine"])}
    del w, buf, out
    torch.cuda.empty_cache()
    return rows


def run_e2e(args, md, w, mode, device, stream, idx, gates, L, wsp, buf, status, dist):
    """Same step through host buffers: pinned inputs -> HBM, path, result -> host.

    Steps are pipelined over two device buffer sets, as a serving loop would
    run them: the inputs of step i+1 copy in (one copy stream) while step i
    computes and step i-1's result copies out (another copy stream).  Every
    step still moves all of its own inputs in and its result out."""
    T, H, E, k, R = w.T, w.H, w.E, w.k, w.R
    h_logits = w.logits.cpu().pin_memory()
    h_x = w.x.cpu().pin_memory()
    h_y = w.y.cpu().pin_memory()
    h_out = [torch.empty(T, H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    d_in = [(w.logits, w.x, w.y)] + [(torch.empty_like(w.logits), torch.empty_like(w.x),
                                      torch.empty_like(w.y))]
    d_out = [torch.empty(T, H, dtype=torch.bfloat16, device=device) for _ in range(2)]
    s_in = torch.cuda.Stream(device)
    s_out = torch.cuda.Stream(device)
    steps = max(1, min(args.steps, args.e2e_steps))
    ev = lambda: torch.cuda.Event()
    in_done = [ev(), ev()]      # inputs of set b are in HBM
    used = [ev(), ev()]         # the step on set b no longer reads its inputs
    out_done = [ev(), ev()]     # the result of set b is on the host

    def step(i):
        b = i % 2
        d_logits, d_x, d_y = d_in[b]
        s_in.wait_event(used[b])
        with torch.cuda.stream(s_in):
            d_logits.copy_(h_logits, non_blocking=True)
            d_x.copy_(h_x, non_blocking=True)
            d_y.copy_(h_y, non_blocking=True)
        in_done[b].record(s_in)
        stream.wait_event(in_done[b])
        stream.wait_event(out_done[b])
        md.md_route_topk(d_logits, k, md.MD_GATE_TOPK_SOFTMAX, idx, gates, stream=stream)
        md.md_dispatch_layout(idx, E, R, w.expert_to_rank, mode, out=L, workspace=wsp,
                              dev_status=status, stream=stream)
        md.md_dispatch_permute(d_x, L.row_of_slot, out=buf, stream=stream)
        md.md_combine(d_y, L.assign_row, idx, gates, out=d_out[b], stream=stream)
        used[b].record(stream)
        s_out.wait_event(used[b])
        with torch.cuda.stream(s_out):
            h_out[b].copy_(d_out[b], non_blocking=True)
        out_done[b].record(s_out)

    for e in used + out_done:
        e.record(stream)
    for i in range(2):
        step(i)
    torch.cuda.synchronize()
    barrier(dist, device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(steps):
        step(i)
    s_in.wait_stream(s_out)
    s_in.wait_stream(stream)
    e1.record(s_in)
    torch.cuda.synchronize()
    ms = max_over_ranks(dist, e0.elapsed_time(e1), device)
    # the last step's result is the step's own output
    assert torch.equal(h_out[(steps - 1) % 2], d_out[(steps - 1) % 2].cpu())
    ws = dist.get_world_size() if dist is not None else 1
    h2d = (h_logits.numel() * 4 + h_x.numel() * 2 + h_y.numel() * 2)
    return {"value": round(T * steps * ws / (ms * 1e-3) / 1e6, 4), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(h_out[0].numel() * 2),
            "steps": steps,
            "note": "pinned host buffers; two device buffer sets, inputs of the next step "
                    "copy in while the result of the previous one copies out"}


# -------------------------------------------------------- oracle (CPU) arm

def oracle_sample(T_s, seed):
    """Inputs for a T_s-token sample of the workload (same recipe, E, k, R, H)."""
    from combine_warp_top_router_b200 import synth
    w = synth.make_workload(WORKLOAD, seed=seed, device="cpu", T=T_s)
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    return (w.logits.numpy(), bits(w.x), bits(w.y), w.expert_to_rank.numpy(), w.E, w.k, w.R)


def oracle_step(oracle, inp, dedup=True):
    lg, x, y, p, E, k, R = inp
    idx, g = oracle.route_topk(lg, k)
    L = oracle.dispatch_layout(idx, E, R, p, 1 if dedup else 0)
    oracle.dispatch_permute(x, L["row_token"])
    oracle.combine(y, L["assign_row"], idx, g)


def cpu_baseline(args):
    import oracle
    oracle.build()
    T_s = args.cpu_sample_tokens
    inp = oracle_sample(T_s, args.seed)
    oracle_step(oracle, oracle_sample(256, args.seed + 1))  # load the library
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle_step(oracle, inp, args.dispatch == "dedup")
        reps += 1
        if time.perf_counter() - t0 >= args.cpu_seconds:
            break
    dt = time.perf_counter() - t0
    out = {"value": round(T_s * reps / dt / 1e6, 5), "unit": UNIT, "cores": 1, "kind": "oracle",
           "sample": f"{reps} x {T_s}-token sample of the same workload recipe "
                     f"(E=128, top-8, 16 ranks, H=2048), single-threaded C oracle, "
                     f"{dt:.1f} s", "host_cores": os.cpu_count()}
    if args.rows:
        out["rows"] = cpu_rows(oracle, args.seed)
    return out


def cpu_rows(oracle, seed):
    """The oracle timed on the planner rows' workloads (single core, one run
    each), beside the GPU times of the `rows` object."""
    from combine_warp_top_router_b200 import synth

    def timed(fn):
        t0 = time.perf_counter()
        r = fn()
        return r, round((time.perf_counter() - t0) * 1e3, 1)

    res = {}
    w = synth.make_workload("two_layer_e128_k6", seed=seed, with_rows=False)
    a = oracle.route_topk(w.logits.numpy(), w.k)[0]
    b = oracle.route_topk(w.logits_next.numpy(), w.k)[0]
    _, C = oracle.coselect(a, b, w.E, T_fit=w.fit_tokens)
    _, res["token_shuffle_e128_k6_ms"] = timed(
        lambda: oracle.token_shuffle(a, C, w.expert_to_rank.numpy(), w.R))
    w = synth.make_workload("three_layer_e128_k6", seed=seed, with_rows=False)
    g = [oracle.route_topk(lg.numpy(), w.k)[0] for lg in (w.logits_prev, w.logits, w.logits_next)]
    C2, res["pair_counts_ms"] = timed(lambda: oracle.coselect_pair(g[0], g[1], g[2], w.E,
                                                                   T_fit=w.fit_tokens))
    _, C = oracle.coselect(g[1], g[2], w.E, T_fit=w.fit_tokens)
    _, res["token_shuffle_pair_e128_k6_ms"] = timed(
        lambda: oracle.token_shuffle_pair(g[0], g[1], C, C2, w.expert_to_rank.numpy(), w.R, 8 * w.k))
    w = synth.make_workload("full_e256_k8", seed=seed, with_rows=False)
    a, res["route_topk_e256_k8_T262144_ms"] = timed(lambda: oracle.route_topk(w.logits.numpy(), 8)[0])
    (W, _), res["coselect_W_e256_ms"] = timed(lambda: oracle.coselect(a, None, 256))
    for label, refine in (("swaps", oracle.REFINE_SWAPS), ("kl", oracle.REFINE_KL)):
        _, res[f"place_{label}_e256_r64_ms"] = timed(
            lambda: oracle.place_two_level(W, 64, 1, 0, refine))
    _, res["place_kl_8_nodes_e256_r64_ms"] = timed(
        lambda: oracle.place_two_level(W, 64, 8, 0, oracle.REFINE_KL))
    _, res["layout_dedup_e256_T262144_ms"] = timed(
        lambda: oracle.dispatch_layout(a, 256, 64, w.expert_to_rank.numpy(), 1))
    return res


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return None
    import oracle
    oracle.build()
    R = 16
    # bound the run to about a minute of CPU for K + W steps
    per_step = 60.0 / max(1, args.steps + args.warmup)
    T_s = int(per_step * CPU_TOKENS_PER_S_GUESS) // R * R
    T_s = max(R, min(16384, T_s))
    inp = oracle_sample(T_s, args.seed)
    for _ in range(args.warmup):
        oracle_step(oracle, inp, args.dispatch == "dedup")
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(oracle, inp, args.dispatch == "dedup")
    dt = time.perf_counter() - t0
    value = T_s * args.steps / dt / 1e6
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": UNIT,
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "T": T_s, "H": 2048, "E": 128, "top_k": 8, "ep_ranks": R,
                   "dispatch": args.dispatch, "combine": "fused",
                   "note": "each step is a bounded sample of the workload"},
        "cpu_baseline": {"value": round(value, 5), "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"{T_s}-token sample per step"},
        "e2e": {"value": round(value, 5), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--dispatch", choices=["dedup", "conv"], default="dedup")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-sample-tokens", type=int, default=32768)
    ap.add_argument("--cpu-seconds", type=float, default=8.0)
    ap.add_argument("--rows", action=argparse.BooleanOptionalAction, default=True,
                    help="also time every step of the path on its own workload")
    ap.add_argument("--row-reps", type=int, default=20)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    line = run_reference(args) if args.impl == "reference" else run_native(args)
    if line is not None:
        print(json.dumps(line), flush=True)
    ws, _, _ = dist_env()
    if ws > 1 and args.impl == "native":
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
