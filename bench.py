"""Benchmark: MoE dispatch + combine throughput on B200.

One step = one pass of the per-layer hot path over one batch:
    md_route_topk -> md_dispatch_layout (dedup) -> md_dispatch_permute -> md_combine
on the workload "full_e256_k8": T=262144 tokens, hidden 2048 bf16, E=256,
top-8 (softmax over the selected logits), 64 virtual EP ranks, correlated
Zipf(1.1) group logits with a x4 expert-load skew.  The expert placement is
the correlated one, fitted once before the timed steps (co-selection counts W
over all tokens, then best single swaps from contiguous placement), as the
pages refit it only every ~1000 steps.  Inputs are synthetic, seeded, resident
in HBM, and each step moves ~17 GB, far more than the 126 MB L2.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

Under torchrun each rank runs an independent replica on its own GPU (the
virtual EP ranks live inside one GPU; nothing is sharded), times K steps with
CUDA events, and rank 0 prints one JSON line with the max over ranks.  The
`rows` object times every other workload of the path on its own (the E=128
top-8 workload in conventional and dedup dispatch, the L2-flushed T=4096 E=64
workload, the top-2 H=4096 workload at EP 8 and 32, the token shuffle and the
dedup dispatch after it, placement modes, routing statistics, the full E=256
pipeline, the EP exchange on one GPU).
--impl reference times the CPU oracle on the host instead (bounded samples).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import platform
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
WORKLOAD = "full_e256_k8"
NOMINAL_HBM_GBS = 8000.0    # B200 HBM3e, nominal (context only; the roofline uses the measured peak)
FALLBACK_HBM_GBS = 6650.0
CPU_TOKENS_PER_S_GUESS = 12000.0  # oracle, one core, this workload's shape


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


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


def kernel_traffic(name, workload, units_per_launch):
    """DRAM bytes per launch from the committed ncu record of this kernel on
    this workload's shape, if it was taken on the current source of the kernel;
    else None.  The record holds bytes per token of a smaller capture of the
    same (E, k, H, R) workload; every token moves the same rows."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(f"{name}@{workload}")
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


def hbm_peak():
    peaks = measured_peaks()
    if peaks and "hbm_gbs" in peaks:
        return float(peaks["hbm_gbs"]), "of measured"
    return FALLBACK_HBM_GBS, "of fallback"


def gbps(nbytes, ms, peak):
    a = nbytes / (ms * 1e-3) / 1e9
    return {"GBps": round(a, 1), "frac": round(a / peak, 3),
            "frac_of_nominal_8TBps": round(a / NOMINAL_HBM_GBS, 3)}


def fit_placement(md, idx, E, R, T_fit, seed_mode, stream=None):
    """Correlated placement from the co-selection counts of tokens [0, T_fit)."""
    W, _ = md.md_coselect_stats(idx, None, E, T_fit=T_fit, stream=stream)
    return md.md_place_correlated(W, R, seed_mode=seed_mode, stream=stream), W


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
    w.logits_next = None  # the headline step routes one layer
    torch.cuda.empty_cache()
    T, H, E, k, R = w.T, w.H, w.E, w.k, w.R
    mode = md.MD_DEDUP if args.dispatch == "dedup" else md.MD_CONV
    stream = torch.cuda.Stream(device)
    # the placement: fitted once, before the timed steps
    with torch.cuda.stream(stream):
        idx0, _ = md.md_route_topk(w.logits, k, stream=stream)
        p, _ = fit_placement(md, idx0, E, R, w.fit_tokens, md.MD_SEED_CONTIGUOUS, stream)
    stream.synchronize()
    del idx0
    idx = torch.empty(T, k, dtype=torch.int32, device=device)
    gates = torch.empty(T, k, dtype=torch.float32, device=device)
    L = md.alloc_layout(T, E, k, R, mode, device)
    wsp = md.alloc_workspace(md.dispatch_layout_workspace_size(T, E, k, R, mode), device)
    buf = torch.empty(L.row_capacity, H, dtype=torch.bfloat16, device=device)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=device)
    status = md.new_status(device)
    torch.cuda.synchronize()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        md.md_route_topk(w.logits, k, md.MD_GATE_TOPK_SOFTMAX, idx, gates, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        md.md_dispatch_layout(idx, E, R, p, mode, out=L, workspace=wsp, dev_status=status,
                              stream=stream)
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
    launches0, memsets0 = md.launch_count(), md.memset_count()
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        with torch.cuda.stream(stream):
            for i in range(args.steps):
                step(events[i])
        stream.synchronize()
    launches = md.launch_count() - launches0
    memsets = md.memset_count() - memsets0
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
    contiguous = synth.contiguous_placement(E, R, device)
    n_rows_contiguous = int(md.md_dispatch_layout(idx, E, R, contiguous, mode).n_rows.item())

    # end to end through host buffers: inputs copied in, the result copied out
    e2e = run_e2e(args, md, w, p, mode, device, stream, idx, gates, L, wsp, buf, status, dist)
    torch.cuda.synchronize()

    if rank != 0:
        return None
    peak, peak_src = hbm_peak()
    ab = algorithmic_bytes(T, H, k, E, n_rows)
    kernels = {n: {"us": round(per[n] * 1e3, 2), "bytes": ab[n], **gbps(ab[n], per[n], peak)}
               for n in per}
    dom = max(("dispatch_permute", "combine"), key=lambda n: per[n])
    achieved = ab[dom] / (per[dom] * 1e-3) / 1e9
    traffic = kernel_traffic(dom, WORKLOAD, T)
    value = T * args.steps * ws / (total_ms_max * 1e-3) / 1e6
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_ms_max / args.steps, 4), "higher_is_better": True,
        "dispatch_combine_excl_router": round(
            T * ws / ((per["dispatch_layout"] + per["dispatch_permute"] + per["combine"]) * 1e-3) / 1e6, 3),
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; shapes of the pages' E=256 top-8 model)",
        "config": {"workload": WORKLOAD, "T": T, "H": H, "E": E, "top_k": k, "ep_ranks": R,
                   "dispatch": args.dispatch, "combine": "fused", "gates": "topk_softmax",
                   "placement": "correlated: W over all tokens, best single swaps from "
                                "contiguous, fitted once before the timed steps",
                   "parallelism": f"replicas x{ws}",
                   "l2": "not flushed: every step moves ~17 GB through HBM, >100x the 126 MB L2",
                   "dedup_rows_per_token": round(n_rows / T, 4),
                   "dedup_rows_per_token_contiguous": round(n_rows_contiguous / T, 4)},
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1),
                     "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "peak_source": peak_src,
                     "frac_of_nominal_8TBps": round(achieved / NOMINAL_HBM_GBS, 4),
                     "traffic": None if traffic is None else int(traffic),
                     "algorithmic_bytes_per_launch": ab[dom]},
        "step_roofline": {"bytes_per_step": sum(ab.values()),
                          "achieved_GBps": round(sum(ab.values()) / (total_ms_max / args.steps * 1e-3) / 1e9, 1),
                          "frac": round(sum(ab.values()) / (total_ms_max / args.steps * 1e-3) / 1e9 / peak, 4)},
        "kernels": kernels,
        "gpu_launches": int(launches),
        "device_memsets": int(memsets),
        "e2e": e2e,
        "clocks": clk.summary(),
    }
    del buf, out, L, wsp
    w.y = None
    w.x = None
    torch.cuda.empty_cache()
    if args.rows:
        line["rows"] = run_rows(args, md, device, stream, peak)
    line["cpu_baseline"] = cpu_baseline(args)
    return line


def _time(fn, stream, reps, graph=True):
    """Average device time (ms) of fn() over reps calls on `stream`, after a warm-up.
    With graph=True the reps calls are captured in one CUDA graph and replayed, so
    the host's marshalling of each call does not leave the GPU idle between them
    (a short kernel would otherwise measure the Python call, not the kernel);
    graph=False times an eager loop, for calls that cannot be captured.  Inputs
    are produced on the default stream, which the (non-blocking) timing stream
    does not wait for: synchronise the device first."""
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        fn()
    stream.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(reps):
                fn()
        with torch.cuda.stream(stream):
            g.replay()  # warm replay, on the timing stream like the timed one
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            e0.record(stream)
            g.replay()
            e1.record(stream)
        stream.synchronize()
        del g
        return e0.elapsed_time(e1) / reps
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
    stream.synchronize()
    return e0.elapsed_time(e1) / reps


def _remote_rows(send_counts):
    """Rows that leave their source rank: the off-diagonal sum of the send matrix."""
    sc = send_counts.to(torch.int64)
    return int(sc.sum().item() - sc.diagonal().sum().item())


def run_rows(args, md, device, stream, peak):
    """Every other workload of the path, each on its own (one GPU)."""
    rows = {}
    rows.update(rows_e128_k8(args, md, device, stream, peak))
    rows.update(rows_e64_k6_l2_flushed(args, md, device, stream, peak))
    rows.update(rows_e128_k2_fitted(args, md, device, stream, peak))
    rows.update(rows_token_shuffle(args, md, device, stream, peak))
    rows.update(rows_e256_k8_planning(args, md, device, stream, peak))
    rows.update(rows_ep_exchange(args, md, device, stream, peak))
    return rows


def rows_ep_exchange(args, md, device, stream, peak):
    """The EP exchange kernels on one GPU: the E=128 top-8 workload split into its
    16 source ranks of 4096 tokens, each laid out on its own; the dispatch
    exchange writes every source's rows into 16 separate destination buffers,
    every destination forms its return rows, and the combine exchange reads
    them back.  Across GPUs the same kernels store to and load from the peers'
    memory over NVLink; here every buffer is local, so this times the
    kernels' HBM side."""
    from combine_warp_top_router_b200 import synth
    reps = max(3, args.row_reps // 4)
    w = synth.make_workload("zipf_pairs_e128_k8", seed=args.seed, device=device)
    T, H, E, k, R = w.T, w.H, w.E, w.k, w.R
    Tr = T // R
    idx, gates = md.md_route_topk(w.logits, k)
    p = w.expert_to_rank
    local = [md.md_dispatch_layout(idx[s * Tr:(s + 1) * Tr], E, R, p, md.MD_DEDUP) for s in range(R)]
    gathered = torch.stack([L.rank_offsets for L in local]).cpu().to(torch.int64)
    plans = [md.md_exchange_plan(gathered, s) for s in range(R)]
    caps = [plans[d][1][R] for d in range(R)]
    recv = [torch.empty(max(c, 1), H, dtype=torch.bfloat16, device=device) for c in caps]
    tok = [torch.empty(max(c, 1), dtype=torch.int32, device=device) for c in caps]
    sidx = [torch.empty(max(c, 1), k, dtype=torch.int32, device=device) for c in caps]
    sw = [torch.empty(max(c, 1), k, dtype=torch.float32, device=device) for c in caps]
    G = md.md_dispatch_layout(idx, E, R, p, md.MD_DEDUP)   # the receivers' expert rows
    ro = G.rank_offsets.cpu().tolist()
    y_row = [torch.empty(max(c, 1), k, dtype=torch.int32, device=device) for c in caps]
    # receiver d's expert-output row of each carried slot (identity mapping
    # onto y's conventional rows; built once, outside the timing)
    carried = (G.row_mask[:ro[R]].view(-1, 1) >> torch.arange(k, device=device).view(1, -1)) & 1
    yr_all = torch.where(carried.bool(), G.assign_row[G.row_token[:ro[R]].long()], -1).to(torch.int32)
    for d in range(R):
        y_row[d][:caps[d]].copy_(yr_all[ro[d]:ro[d + 1]])
    ret = [torch.empty(max(c, 1), H, dtype=torch.bfloat16, device=device) for c in caps]
    out = torch.empty(T, H, dtype=torch.bfloat16, device=device)
    dpeers = [[md.PeerRows(rows=recv[d], token=tok[d], slot_idx=sidx[d], slot_w=sw[d],
                           row_base=plans[s][0][d], rows_cap=caps[d]) for d in range(R)]
              for s in range(R)]
    cpeers = [[md.PeerRows(rows=ret[d], row_base=plans[s][0][d], rows_cap=caps[d]) for d in range(R)]
              for s in range(R)]

    # the calls enqueue on the current stream; each phase's 16 calls are
    # captured in a CUDA graph and replayed, so host marshalling stays out of
    # the timed region (16 small launches per phase would otherwise leave the
    # GPU waiting on the host)
    def dispatch():
        for s_ in range(R):
            sl = slice(s_ * Tr, (s_ + 1) * Tr)
            md.md_dispatch_exchange(w.x[sl], idx[sl], gates[sl], p, E, local[s_].row_of_slot,
                                    local[s_].rank_offsets, s_ * Tr, dpeers[s_])

    def partials():
        for d in range(R):
            md.md_combine_partials(w.y, y_row[d][:caps[d]], sidx[d][:caps[d]], sw[d][:caps[d]],
                                   out=ret[d][:caps[d]])

    def combine():
        for s_ in range(R):
            sl = slice(s_ * Tr, (s_ + 1) * Tr)
            md.md_combine_exchange(cpeers[s_], idx[sl], p, E, local[s_].row_of_slot,
                                   local[s_].rank_offsets, H, out=out[sl])

    def graphed(fn):
        torch.cuda.synchronize()
        fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        return g

    graphs = [graphed(f) for f in (dispatch, partials, combine)]
    t_d, t_p, t_c = (_time(g.replay, stream, reps, graph=False) for g in graphs)
    del graphs
    n = sum(caps)
    # dispatch: x once, each row written once with its metadata (4 + 8k B)
    db = T * (2 * H + 12 * k) + n * (2 * H + 4 + 8 * k)
    # partials: the carried slots' expert rows and metadata in, one row out
    pb = T * k * 2 * H + n * (12 * k + 2 * H)
    # combine: each return row read once, one row out per token
    cb = n * 2 * H + T * (2 * H + 8 * k)
    r = {"T": T, "ranks": R, "tokens_per_rank": Tr, "rows_per_token": round(n / T, 4),
         "dispatch_exchange_us": round(t_d * 1e3, 1), "dispatch_exchange": gbps(db, t_d, peak),
         "combine_partials_us": round(t_p * 1e3, 1), "combine_partials": gbps(pb, t_p, peak),
         "combine_exchange_us": round(t_c * 1e3, 1), "combine_exchange": gbps(cb, t_c, peak),
         "note": "16 calls of each kernel (one per source or destination rank), replayed from a "
                 "CUDA graph; all buffers on this GPU"}
    del w, recv, tok, sidx, sw, ret, out, y_row, local, G
    torch.cuda.empty_cache()
    return {"ep_exchange_zipf_pairs_e128_k8": r}


def rows_e128_k8(args, md, device, stream, peak):
    """zipf_pairs_e128_k8: conventional and dedup dispatch, wire combine, expand."""
    from combine_warp_top_router_b200 import synth
    rows = {}
    reps = args.row_reps
    w = synth.make_workload("zipf_pairs_e128_k8", seed=args.seed, device=device)
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
        r = {"T": T, "rows_per_token": round(n / T, 4), "layout_us": round(t_lay * 1e3, 2),
             "permute_us": round(t_perm * 1e3, 2), "permute": gbps(pb, t_perm, peak),
             "combine_us": round(t_comb * 1e3, 2), "combine": gbps(cb, t_comb, peak),
             "dispatch_combine_Mtokens_per_s": round(T / ((t_lay + t_perm + t_comb) * 1e-3) / 1e6, 2)}
        if mode == md.MD_DEDUP:
            z = torch.empty(L.row_capacity, H, dtype=torch.bfloat16, device=device)
            t_wire = _time(lambda: md.md_combine(w.y, L.assign_row, idx, gates, md.MD_COMBINE_WIRE,
                                                 row_of_slot=L.row_of_slot, z=z, out=out,
                                                 stream=stream), stream, reps)
            wb = T * (2 * H * k + 2 * H + 16 * k) + n * 2 * H
            r["combine_wire_us"] = round(t_wire * 1e3, 2)
            r["combine_wire"] = gbps(wb, t_wire, peak)
            del z
            # receiver side: dedup rows -> one row per (token, expert), expert-grouped
            xc = torch.empty(T * k, H, dtype=torch.bfloat16, device=device)
            t_exp = _time(lambda: md.md_dedup_expand(buf, L.row_of_slot, L.assign_row, out=xc,
                                                     stream=stream), stream, reps)
            eb = n * 2 * H + T * k * (2 * H + 8)
            r["dedup_expand_us"] = round(t_exp * 1e3, 2)
            r["dedup_expand"] = gbps(eb, t_exp, peak)
            del xc
        rows[f"zipf_pairs_e128_k8_{name}"] = r
        del L, wsp, buf, out
    t_topk = _time(lambda: md.md_route_topk(w.logits, k, topk_idx=idx, topk_w=gates, stream=stream),
                   stream, reps)
    rows["route_topk_e128_k8"] = {"us": round(t_topk * 1e3, 2), **gbps(T * (4 * E + 8 * k), t_topk, peak)}
    del w, idx, gates
    torch.cuda.empty_cache()
    return rows


def rows_e64_k6_l2_flushed(args, md, device, stream, peak):
    """iid_e64_k6 (T=4096, 117 MB per kernel, about the size of L2): L2 is
    flushed (a write of twice its size) before every timed launch, and medians
    are reported.  Each kernel, and the whole step, is captured in a CUDA graph
    and replayed right after the flush, so the host's marshalling of the four
    calls does not leave the GPU idle inside the timed region."""
    from combine_warp_top_router_b200 import synth
    w = synth.make_workload("iid_e64_k6", seed=args.seed, device=device)
    T, H, E, k, R = w.T, w.H, w.E, w.k, w.R
    mode = md.MD_CONV
    idx = torch.empty(T, k, dtype=torch.int32, device=device)
    gates = torch.empty(T, k, dtype=torch.float32, device=device)
    L = md.alloc_layout(T, E, k, R, mode, device)
    wsp = md.alloc_workspace(md.dispatch_layout_workspace_size(T, E, k, R, mode), device)
    buf = torch.empty(L.row_capacity, H, dtype=torch.bfloat16, device=device)
    out = torch.empty(T, H, dtype=torch.bfloat16, device=device)
    l2 = int(getattr(torch.cuda.get_device_properties(device), "L2_cache_size", 126 << 20))
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=device)
    parts = ("route_topk", "dispatch_layout", "dispatch_permute", "combine")
    calls = (
        lambda: md.md_route_topk(w.logits, k, md.MD_GATE_TOPK_SOFTMAX, idx, gates),
        lambda: md.md_dispatch_layout(idx, E, R, w.expert_to_rank, mode, out=L, workspace=wsp),
        lambda: md.md_dispatch_permute(w.x, L.row_of_slot, out=buf),
        lambda: md.md_combine(w.y, L.assign_row, idx, gates, out=out),
    )

    def graphed(fns):
        torch.cuda.synchronize()
        for f in fns:
            f()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for f in fns:
                f()
        return g

    graphs = {n: graphed([c]) for n, c in zip(parts, calls)}
    graphs["step"] = graphed(calls)
    n_steps = max(20, args.row_reps)
    times = {n: [] for n in graphs}
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(3 + n_steps):
            for name, g in graphs.items():
                flush.fill_(i & 0xff)
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                g.replay()
                e1.record(stream)
                stream.synchronize()
                if i >= 3:
                    times[name].append(e0.elapsed_time(e1))
    med = {n: statistics.median(v) for n, v in times.items()}
    n = int(L.n_rows.item())
    ab = algorithmic_bytes(T, H, k, E, n)
    r = {"T": T, "H": H, "E": E, "top_k": k, "ep_ranks": R, "dispatch": "conv",
         "placement": "contiguous", "l2": f"flushed before every timed launch ({2 * l2 >> 20} MiB write)",
         "timing": "CUDA graph replay per kernel and per step; medians",
         "steps": n_steps, "median_step_us": round(med["step"] * 1e3, 2),
         "Mtokens_per_s": round(T / (med["step"] * 1e-3) / 1e6, 2),
         "dispatch_combine_excl_router": round(
             T / ((med["dispatch_layout"] + med["dispatch_permute"] + med["combine"]) * 1e-3) / 1e6, 2)}
    for nme in parts:
        r[nme] = {"us": round(med[nme] * 1e3, 2), **gbps(ab[nme], med[nme], peak)}
    del graphs, w, idx, gates, L, wsp, buf, out, flush
    torch.cuda.empty_cache()
    return {"iid_e64_k6_l2_flushed": r}


def rows_e128_k2_fitted(args, md, device, stream, peak):
    """boost_pairs_e128_k2 (T=65536, H=4096, top-2) at EP 8 and 32: placement
    fitted on tokens [0, 4096) (greedy pair seed, then best single swaps),
    dedup dispatch and fused combine; rows per token against contiguous."""
    from combine_warp_top_router_b200 import synth
    rows = {}
    reps = args.row_reps
    w = synth.make_workload("boost_pairs_e128_k2", seed=args.seed, device=device)
    T, H, E, k = w.T, w.H, w.E, w.k
    idx, gates = md.md_route_topk(w.logits, k)
    for R in (8, 32):
        p, _ = fit_placement(md, idx, E, R, w.fit_tokens, md.MD_SEED_GREEDY_PAIRS)
        mode = md.MD_DEDUP
        L = md.alloc_layout(T, E, k, R, mode, device)
        wsp = md.alloc_workspace(md.dispatch_layout_workspace_size(T, E, k, R, mode), device)
        buf = torch.empty(L.row_capacity, H, dtype=torch.bfloat16, device=device)
        out = torch.empty(T, H, dtype=torch.bfloat16, device=device)
        t_lay = _time(lambda: md.md_dispatch_layout(idx, E, R, p, mode, out=L, workspace=wsp,
                                                      stream=stream), stream, reps)
        n = int(L.n_rows.item())
        t_perm = _time(lambda: md.md_dispatch_permute(w.x, L.row_of_slot, out=buf, stream=stream),
                       stream, reps)
        t_comb = _time(lambda: md.md_combine(w.y, L.assign_row, idx, gates, out=out, stream=stream),
                       stream, reps)
        Lc = md.md_dispatch_layout(idx, E, R, synth.contiguous_placement(E, R, device), mode)
        ab = algorithmic_bytes(T, H, k, E, n)
        rows[f"boost_pairs_e128_k2_ep{R}"] = {
            "T": T, "H": H, "rows_per_token": round(n / T, 4),
            "rows_per_token_contiguous": round(int(Lc.n_rows.item()) / T, 4),
            "remote_rows_per_token": round(_remote_rows(L.send_counts) / T, 4),
            "remote_rows_per_token_contiguous": round(_remote_rows(Lc.send_counts) / T, 4),
            "layout_us": round(t_lay * 1e3, 2),
            "permute_us": round(t_perm * 1e3, 2), "permute": gbps(ab["dispatch_permute"], t_perm, peak),
            "combine_us": round(t_comb * 1e3, 2), "combine": gbps(ab["combine"], t_comb, peak),
            "dispatch_combine_Mtokens_per_s": round(T / ((t_lay + t_perm + t_comb) * 1e-3) / 1e6, 2)}
        del L, wsp, buf, out, Lc
    del w, idx, gates
    torch.cuda.empty_cache()
    return rows


def rows_token_shuffle(args, md, device, stream, peak):
    """The token shuffle and the dedup dispatch after it.  Single form on
    two_layer_e128_k6, pair form on three_layer_e128_k6; counts fitted on
    tokens [0, 4096); contiguous placement at layer l+1.  After the shuffle the
    layer-(l+1) top-k rows are gathered into the shuffled order and the dedup
    layout runs with src = the token's new block."""
    from combine_warp_top_router_b200 import synth
    rows = {}
    reps = args.row_reps

    def after_shuffle(nxt, inv, E, R, p_next):
        """dedup rows and remote rows per token at l+1 in the given token order"""
        T = nxt.shape[0]
        ordered = nxt if inv is None else md.md_gather_rows(nxt, inv)
        L = md.md_dispatch_layout(ordered, E, R, p_next, md.MD_DEDUP)
        return {"rows_per_token": round(int(L.n_rows.item()) / T, 4),
                "remote_rows_per_token": round(_remote_rows(L.send_counts) / T, 4)}

    # single-expert prediction
    w = synth.make_workload("two_layer_e128_k6", seed=args.seed, device=device)
    T, E, R = w.T, w.E, w.R
    a, _ = md.md_route_topk(w.logits, w.k)
    b, _ = md.md_route_topk(w.logits_next, w.k)
    _, C = md.md_coselect_stats(a, b, E, T_fit=w.fit_tokens, want_W=False)
    sws = md.alloc_workspace(int(md.lib().md_token_shuffle_workspace_size(T, E, R)), device)
    pred = torch.empty(T, dtype=torch.int32, device=device)
    perm = torch.empty_like(pred)
    inv = torch.empty_like(pred)
    t_sh = _time(lambda: md.md_token_shuffle(a, C, w.expert_to_rank, R, pred, perm, inv,
                                             workspace=sws, stream=stream), stream, reps)
    xs = torch.empty_like(w.x)
    t_g = _time(lambda: md.md_gather_rows(w.x, inv, out=xs, stream=stream), stream, reps)
    bs = torch.empty_like(b)
    t_gi = _time(lambda: md.md_gather_rows(b, inv, out=bs, stream=stream), stream, reps)
    Ls = md.alloc_layout(T, E, w.k, R, md.MD_DEDUP, device)
    lws = md.alloc_workspace(md.dispatch_layout_workspace_size(T, E, w.k, R, md.MD_DEDUP), device)
    t_lay = _time(lambda: md.md_dispatch_layout(bs, E, R, w.expert_to_rank, md.MD_DEDUP, out=Ls,
                                                  workspace=lws, stream=stream), stream, reps)
    none = after_shuffle(b, None, E, R, w.expert_to_rank)
    single = after_shuffle(b, inv, E, R, w.expert_to_rank)
    # the rounds-based parallel assignment on the same inputs
    rws = md.alloc_workspace(int(md.lib().md_token_shuffle_rounds_workspace_size(T, E, R)), device)
    rp, rperm, rinv = torch.empty_like(pred), torch.empty_like(pred), torch.empty_like(pred)
    holder = {}
    t_rd = _time(lambda: holder.__setitem__("r", md.md_token_shuffle_rounds(
        a, C, w.expert_to_rank, R, rp, rperm, rinv, workspace=rws, stream=stream)[3]), stream, reps)
    n_rounds = int(holder["r"].item())
    rounds = after_shuffle(b, rinv, E, R, w.expert_to_rank)
    loc = lambda order: float((torch.arange(T, device=device) // (T // R)).eq(
        w.expert_to_rank[order.long()].T).float().mean())
    rows["token_shuffle_e128_k6"] = {
        "T": T, "shuffle_us": round(t_sh * 1e3, 2), "gather_x_us": round(t_g * 1e3, 2),
        "gather": gbps(2 * T * 2 * w.H + 4 * T, t_g, peak),
        "gather_topk_us": round(t_gi * 1e3, 2), "layout_after_shuffle_us": round(t_lay * 1e3, 2),
        "locality_before": round(loc(b), 4), "locality_after": round(loc(b[inv.long()]), 4),
        "dedup_dispatch_at_next_layer": {"no_shuffle": none, "single": single,
                                         "rounds": rounds},
        "rounds_variant": {"us": round(t_rd * 1e3, 2), "rounds": n_rounds,
                           "locality_after": round(loc(b[rinv.long()]), 4)}}
    del w, a, b, C, sws, xs, bs, Ls, lws
    torch.cuda.empty_cache()

    # pair-based prediction on the three-layer workload (a pair row is used
    # when its total reaches 8k)
    w = synth.make_workload("three_layer_e128_k6", seed=args.seed, device=device, with_rows=False)
    T, E, R = w.T, w.E, w.R
    g = [md.md_route_topk(lg, w.k)[0] for lg in (w.logits_prev, w.logits, w.logits_next)]
    C2 = torch.empty(E, E, E, dtype=torch.int32, device=device)
    t_c2 = _time(lambda: md.md_coselect_pair_stats(g[0], g[1], g[2], E, T_fit=w.fit_tokens, C2=C2,
                                                   stream=stream), stream, reps)
    _, C = md.md_coselect_stats(g[1], g[2], E, T_fit=w.fit_tokens, want_W=False)
    pws = md.alloc_workspace(int(md.lib().md_token_shuffle_pair_workspace_size(T, E, R)), device)
    pred = torch.empty(T, dtype=torch.int32, device=device)
    perm, inv, use = torch.empty_like(pred), torch.empty_like(pred), torch.empty_like(pred)
    min_obs = 8 * w.k
    t_sp = _time(lambda: md.md_token_shuffle_pair(g[0], g[1], C, C2, w.expert_to_rank, R, min_obs,
                                                  pred, perm, inv, use, workspace=pws,
                                                  stream=stream), stream, reps)
    nxt_rank = w.expert_to_rank[g[2].long()]
    sp, _, sinv = md.md_token_shuffle(g[1], C, w.expert_to_rank, R)
    rows["token_shuffle_pair_e128_k6"] = {
        "T": T, "min_obs": min_obs, "pair_counts_us": round(t_c2 * 1e3, 2),
        "shuffle_pair_us": round(t_sp * 1e3, 2), "tokens_on_pair_rows": round(float(use.float().mean()), 4),
        "locality_no_shuffle": round(float((torch.arange(T, device=device) // (T // R))[:, None]
                                           .eq(nxt_rank).float().mean()), 4),
        "locality_single": round(float(sp[:, None].eq(nxt_rank).float().mean()), 4),
        "locality_pair": round(float(pred[:, None].eq(nxt_rank).float().mean()), 4),
        "dedup_dispatch_at_next_layer": {"no_shuffle": after_shuffle(g[2], None, E, R, w.expert_to_rank),
                                         "single": after_shuffle(g[2], sinv, E, R, w.expert_to_rank),
                                         "pair": after_shuffle(g[2], inv, E, R, w.expert_to_rank)}}
    del w, g, C2, C, pws
    torch.cuda.empty_cache()
    return rows


def rows_e256_k8_planning(args, md, device, stream, peak):
    """The E=256 workload's planning steps: the full pipeline with co-selection
    counts and placement inside every step, placement modes, routing statistics."""
    from combine_warp_top_router_b200 import synth
    rows = {}
    reps = args.row_reps
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
    n_runs = max(1, reps // 5)
    with torch.cuda.stream(stream):
        for _ in range(n_runs):
            pipeline(evs)
    stream.synchronize()
    for name, e0, e1 in evs:
        parts[name] = parts.get(name, 0.0) + e0.elapsed_time(e1) / n_runs
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
                                                  workspace=qws, stream=stream), stream, 3, graph=False)
        torch.cuda.synchronize()
        Lq = md.md_dispatch_layout(a, E, R, q, md.MD_DEDUP)
        modes[label] = {"us": round(t_q * 1e3, 1),
                        "rows_per_token": round(int(Lq.n_rows.item()) / T, 4)}
    rows["placement_modes_e256_k8"] = modes

    # the pages' routing statistics on this workload: Table I columns for both
    # placements, the cross-layer successor share, fitted vs held-out W
    s_corr = md.table1_row(md.md_rank_stats(a, E, R, p).cpu())
    s_cont = md.table1_row(md.md_rank_stats(a, E, R, contiguous).cpu())
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
        "permute": gbps(T * (2 * H + 4 * k) + n * 2 * H, parts["dispatch_permute"], peak),
        "combine": gbps(T * (2 * H * (k + 1) + 12 * k), parts["combine"], peak)}
    del w, buf, out
    torch.cuda.empty_cache()
    return rows


def _pinned_copy(t):
    h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
    h.copy_(t)
    return h


def run_e2e(args, md, w, p, mode, device, stream, idx, gates, L, wsp, buf, status, dist):
    """The same step through host buffers: pinned inputs -> HBM, the path, the
    result -> host.  Two forms:

    * main: every input of the timed step (logits, x and the expert outputs y)
      is copied in each step, and the combined rows are copied out;
    * y_on_device: only logits and x are copied in; the expert outputs are made
      on the device by identity experts (the receiver-side expand of the dedup
      rows, md_dedup_expand, gives each (token, expert) its row), so the step
      is router -> layout -> permute -> expand -> combine.

    Steps are pipelined over two device buffer sets, as a serving loop would
    run them: the inputs of step i+1 copy in (one copy stream) while step i
    computes and step i-1's result copies out (another copy stream).  Every
    step still moves all of its own inputs in and its result out."""
    T, H, E, k, R = w.T, w.H, w.E, w.k, w.R
    h_logits = _pinned_copy(w.logits)
    h_x = _pinned_copy(w.x)
    h_out = [torch.empty(T, H, dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    d_out = [torch.empty(T, H, dtype=torch.bfloat16, device=device) for _ in range(2)]
    s_in = torch.cuda.Stream(device)
    s_out = torch.cuda.Stream(device)
    steps = max(1, min(args.steps, args.e2e_steps))
    ws = dist.get_world_size() if dist is not None else 1

    def measure(y_from_host):
        h_y = _pinned_copy(w.y) if y_from_host else None
        d_in = [(w.logits, w.x, w.y)] + [(torch.empty_like(w.logits), torch.empty_like(w.x),
                                          torch.empty_like(w.y))]
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
                if y_from_host:
                    d_y.copy_(h_y, non_blocking=True)
            in_done[b].record(s_in)
            stream.wait_event(in_done[b])
            stream.wait_event(out_done[b])
            md.md_route_topk(d_logits, k, md.MD_GATE_TOPK_SOFTMAX, idx, gates, stream=stream)
            md.md_dispatch_layout(idx, E, R, p, mode, out=L, workspace=wsp, dev_status=status,
                                  stream=stream)
            md.md_dispatch_permute(d_x, L.row_of_slot, out=buf, stream=stream)
            if not y_from_host:
                md.md_dedup_expand(buf, L.row_of_slot, L.assign_row, out=d_y, stream=stream)
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
        h2d = h_logits.numel() * 4 + h_x.numel() * 2 + (w.y.numel() * 2 if y_from_host else 0)
        del d_in, h_y
        torch.cuda.empty_cache()
        return ms, h2d

    if mode != md.MD_DEDUP:
        raise SystemExit("the end-to-end leg expects the dedup dispatch")
    ms, h2d = measure(True)       # first: it copies the synthetic y to the host
    ms_y, h2d_y = measure(False)  # then the expand overwrites the device y
    d2h = int(h_out[0].numel() * 2)
    return {"value": round(T * steps * ws / (ms * 1e-3) / 1e6, 4), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": d2h, "steps": steps,
            "note": "pinned host buffers; logits, x and the expert outputs y copied in every "
                    "step, the combined rows copied out; two device buffer sets, inputs of the "
                    "next step copy in while the result of the previous one copies out",
            "y_on_device": {
                "value": round(T * steps * ws / (ms_y * 1e-3) / 1e6, 4), "unit": UNIT,
                "h2d_bytes_per_step": int(h2d_y), "d2h_bytes_per_step": d2h,
                "note": "logits and x copied in; identity experts on the device (md_dedup_expand "
                        "of the dedup rows) make y; router -> layout -> permute -> expand -> "
                        "combine; result copied out"}}


# -------------------------------------------------------- oracle (CPU) arm

def oracle_sample(T_s, seed):
    """Inputs for a T_s-token sample of the headline workload (same recipe, E, k,
    R, H), with the oracle's own correlated placement fitted on the sample
    (untimed, as the GPU arm fits its placement before timing)."""
    import oracle
    from combine_warp_top_router_b200 import synth
    w = synth.make_workload(WORKLOAD, seed=seed, device="cpu", T=T_s)
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    lg = w.logits.numpy()
    idx = oracle.route_topk(lg, w.k)[0]
    W, _ = oracle.coselect(idx, None, w.E)
    p = oracle.place_correlated(W, w.R)
    return (lg, bits(w.x), bits(w.y), p, w.E, w.k, w.R)


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
                     f"(E=256, top-8, 64 ranks, H=2048, correlated placement fitted on the "
                     f"sample), single-threaded C oracle, {dt:.1f} s",
           "host_cores": os.cpu_count(), "cpu_model": cpu_model()}
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
    from combine_warp_top_router_b200 import synth
    oracle.build()
    spec = synth.SPECS[WORKLOAD]
    R = spec["R"]
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
        "config": {"workload": WORKLOAD, "T": T_s, "H": spec["H"], "E": spec["E"],
                   "top_k": spec["k"], "ep_ranks": R, "dispatch": args.dispatch, "combine": "fused",
                   "placement": "correlated, fitted on the sample before timing",
                   "note": "each step is a bounded sample of the workload"},
        "cpu_baseline": {"value": round(value, 5), "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"{T_s}-token sample per step", "cpu_model": cpu_model()},
        "e2e": {"value": round(value, 5), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--dispatch", choices=["dedup", "conv"], default="dedup")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-sample-tokens", type=int, default=16384)
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
