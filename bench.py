#!/usr/bin/env python
"""Benchmark of the balanced expert-parallel hot path on B200.

One step is one MoE layer's forward pass through the library's C ABI at the
training shape (R=8 emulated EP ranks, S=4096 tokens per rank, K=8, E=256,
B=32, H=7168, token_padding=128): plan -> dispatch -> combine, with the
dispatch buffer itself as the expert output.  Steps cycle through routings at
maxvio 0, 0.5, 1, 2 and 4.  The headline value is dispatch+combine algorithmic
HBM bytes / wall time of the whole step (planner included).

Also measured in the same run (unless switched off):
  * per-kernel CUDA-event times (planner us/layer, dispatch and combine GB/s,
    per-maxvio spread) and the roofline of the dominant kernel;
  * legs: prefetch_weight at the inference shape (B=4, H'=2048, 3
    projections) and reduce_grad at the backward shape (B=32, H'=2048 fp32);
  * e2e: the same step from pinned host buffers, host<->device copies
    included;
  * cpu_baseline: the CPU oracle on a bounded sample, one host core.

`--impl reference` times the CPU oracle itself on the same workload (see the
reference-arm section below).

Multi-GPU (`torchrun ... --gpus N`, N > 1): the workload's EP group of R=8
ranks is sharded over the N processes, R/N ranks per process and GPU (one EP
rank per process at N = 8).  Each process owns its ranks' dispatch buffers
and maps its peers' with CUDA IPC; per step it all-gathers the router counts,
plans its ranks' shares, dispatches their rows into the owners' buffers over
NVLink, and after a barrier combines its tokens from them (strong scaling:
the layer is fixed, N GPUs share it).  Time is the max over processes.
`--replicas` runs the old mode instead: an independent emulated group per GPU.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from load_balancing_planner_b200 import synth  # noqa: E402

METRIC = "dispatch+combine HBM GB/s (% of peak) vs maxvio; planner µs/layer; 1 B200"
NOMINAL_HBM_GBS = 8000.0

WORKLOADS = {
    "train": dict(R=8, S=4096, K=8, E=256, B=32, H=7168, tp=128, mode=0, profile="hot8",
                  maxvio=(0.0, 0.5, 1.0, 2.0, 4.0)),
    "zipf": dict(R=8, S=1024, K=8, E=64, B=8, H=2048, tp=128, mode=0, profile="zipf",
                 maxvio=(0.0, 0.5, 1.0, 2.0)),
    # training rows (H=7168) with fewer tokens: ~1.5 GB on the device, for
    # profiler captures that must stay small
    "train_s512": dict(R=8, S=512, K=8, E=256, B=32, H=7168, tp=128, mode=0, profile="hot8",
                       maxvio=(0.0, 2.0)),
    # training rows with 64 experts and 1024 tokens per rank: the group GEMM's
    # profiler case (about 3 GB on the device at H' = 1024)
    "gemm_small": dict(R=8, S=1024, K=8, E=64, B=8, H=7168, tp=128, mode=0, profile="hot8",
                       maxvio=(2.0,)),
}


def describe(w):
    return (f"R={w['R']} S={w['S']} K={w['K']} E={w['E']} B={w['B']} H={w['H']} "
            f"token_padding={w['tp']} {'training' if w['mode'] == 0 else 'inference'}, "
            f"routing {w['profile']} at maxvio " + "/".join(f"{m:g}" for m in w["maxvio"]))


def dc_bytes(R, S, K, H):
    """Algorithmic bytes of dispatch + combine for one layer (all R ranks):
    dispatch reads each row once and writes it K times, plus dst, w and w_nvs;
    combine reads K rows per token and writes one, plus dst, the slot weights
    and the gathered weights it writes back in token order."""
    disp = R * (S * H * 2 + S * K * H * 2 + 3 * S * K * 4)
    comb = R * (S * K * H * 2 + S * H * 2 + 3 * S * K * 4)
    return disp, comb


# kernels one step launches: plan_kernel, one dispatch kernel, combine_kernel
KERNELS_PER_STEP = 3
# the pages' own benchmark also reports maxvio 10 and 20 (outside the sweep
# that `value` covers); timed after the run on the training shape
PAGES_POINTS = (10.0, 20.0)


def copy_source_hash():
    """Hash of the sources of the copy kernels (copy.cu and the bulk-copy helpers)."""
    import hashlib
    h = hashlib.sha256()
    for name in ("copy.cu", "bulk.cuh"):
        with open(os.path.join(ROOT, "load_balancing_planner_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel):
    """DRAM bytes per launch of `kernel` at the training shape, from the ncu
    record in profiles/dram_traffic_train.txt -- only if that record was taken
    on the current source of the copy kernels (hash match), else None."""
    import re
    try:
        sha = copy_source_hash()
        with open(os.path.join(ROOT, "profiles", "dram_traffic_train.txt")) as f:
            for line in f:
                m = re.search(r"traffic: kernel=(\w+) bytes_per_launch=(\d+) copy_src_sha256=(\w+)", line)
                if m and m.group(1) == kernel and m.group(3) == sha:
                    return int(m.group(2))
    except OSError:
        pass
    return None


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def tensor_peaks():
    """Dense bf16 TFLOP/s: (burst, sustained, kind)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------- clocks
class Clocks:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        self.t0 = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- helpers
def setup_dist(args):
    """(world, rank, device index).  One GPU per process over NCCL; with
    --share-gpu every process uses GPU 0 over gloo (a correctness run of the
    sharded path on one GPU: the processes time-share it)."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = 0 if args.share_gpu else int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        if args.share_gpu:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
        else:
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()


def max_over_ranks(x, world):
    """Largest value over the ranks (a timing, never data of the path)."""
    import torch
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(seed, rank):
    """Every rank draws its own EP group's inputs: independent problems."""
    return seed + rank


def aggregate_gbs(bytes_per_rank_step, steps, world, max_ms):
    """Whole-job throughput: the bytes all ranks moved over the slowest rank's time."""
    return world * bytes_per_rank_step * steps / (max_ms * 1e-3) / 1e9


def make_inputs(w, seed, dev):
    import torch
    R, S, K, E, H = w["R"], w["S"], w["K"], w["E"], w["H"]
    hidden = synth.hidden_bf16(R, S, H, seed).to(dev)
    weights = torch.from_numpy(synth.route_weights(R, S, K, seed)).to(dev)
    routes = []
    for mv in w["maxvio"]:
        tk, real, _ = synth.routing(R, S, K, E, mv, w["profile"], seed=seed)
        routes.append(dict(target=mv, realised=real,
                           topk=torch.from_numpy(tk).to(dev),
                           tpe=torch.from_numpy(synth.local_counts(tk, E)).to(dev),
                           topk_np=tk))
    return hidden, weights, routes


# ---------------------------------------------------------------- our arm
def run_ours(args, world, rank, local):
    import torch
    from load_balancing_planner_b200 import moonep

    w = WORKLOADS[args.config]
    R, S, K, E, B, H, tp = w["R"], w["S"], w["K"], w["E"], w["B"], w["H"], w["tp"]
    dev = torch.device("cuda", local if world > 1 else 0)
    seed = rank_seed(args.seed, rank)
    hidden, weights, routes = make_inputs(w, seed, dev)
    h = moonep.moonep_create(S, H, K, E, R, B, tp, mode=w["mode"])
    nvs = h.nvs
    plan = moonep.Plan(h, dev)
    buf = torch.empty((R, nvs, H), dtype=torch.bfloat16, device=dev)
    wn = torch.empty((R, nvs), dtype=torch.float32, device=dev)
    out = torch.empty((R, S, H), dtype=torch.bfloat16, device=dev)
    gw = torch.empty((R, S, K), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    npts = len(routes)

    def step(i, ev=None):
        r = routes[i % npts]
        if ev:
            ev[0].record(stream)
        moonep.moonep_plan(h, r["topk"], r["tpe"], plan)
        if ev:
            ev[1].record(stream)
        moonep.moonep_dispatch(h, plan, hidden, weights, buf, wn)
        if ev:
            ev[2].record(stream)
        moonep.moonep_combine(h, plan, buf, wn, out, gw)
        if ev:
            ev[3].record(stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    st = moonep.moonep_read_status(plan)
    if st != 0:
        raise RuntimeError(f"plan status {st}")

    clocks = Clocks(local if world > 1 else 0)
    clocks.start()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    barrier(world)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(i, evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    total_ms = t_start.elapsed_time(t_end)
    total_ms_max = max_over_ranks(total_ms, world)

    # the planner alone, launched back to back (outside the timed region)
    b0 = torch.cuda.Event(enable_timing=True)
    b1 = torch.cuda.Event(enable_timing=True)
    nb = 200
    b0.record(stream)
    for i in range(nb):
        r = routes[i % npts]
        moonep.moonep_plan(h, r["topk"], r["tpe"], plan)
    b1.record(stream)
    torch.cuda.synchronize()
    plan_b2b_us = b0.elapsed_time(b1) * 1e3 / nb

    # The same steps without planning, each routing's plan computed ahead:
    # the planner's cost per layer is the difference in step time.  Both
    # loops record the same four events per step.
    saved = []
    for r in routes:
        saved.append(moonep.moonep_plan(h, r["topk"], r["tpe"], moonep.Plan(h, dev)))

    def step_saved(i, ev=None):
        p = saved[i % npts]
        if ev:
            ev[0].record(stream)
            ev[1].record(stream)
        moonep.moonep_dispatch(h, p, hidden, weights, buf, wn)
        if ev:
            ev[2].record(stream)
        moonep.moonep_combine(h, p, buf, wn, out, gw)
        if ev:
            ev[3].record(stream)

    for i in range(args.warmup):
        step_saved(i)
    # The planner's cost inside the step: the same steps with and without
    # planning (the plans computed ahead), events only at the step
    # boundaries, the two arms alternating, n_rep steps per routing and arm.
    # The difference of the medians is what planning adds to a layer.
    n_rep = 24
    arms = {j: ([], []) for j in range(npts)}
    for rep in range(n_rep + 1):
        for j, r in enumerate(routes):
            for arm in (0, 1):
                a0 = torch.cuda.Event(enable_timing=True)
                a1 = torch.cuda.Event(enable_timing=True)
                a0.record(stream)
                if arm == 0:
                    moonep.moonep_plan(h, r["topk"], r["tpe"], plan)
                p = plan if arm == 0 else saved[j]
                moonep.moonep_dispatch(h, p, hidden, weights, buf, wn)
                moonep.moonep_combine(h, p, buf, wn, out, gw)
                a1.record(stream)
                if rep:
                    arms[j][arm].append((a0, a1))
    torch.cuda.synchronize()
    with_ms = {j: [a.elapsed_time(b) for a, b in v[0]] for j, v in arms.items()}
    without_ms = {j: [a.elapsed_time(b) for a, b in v[1]] for j, v in arms.items()}

    # The launch floor of the planner in the same place of the step: a
    # two-block plan (R=2, S=64, K=2, E=8) right after a full combine,
    # between the same two events.  It is what an almost empty cooperative
    # launch costs there; the planner's in-step time sits on top of it.
    tk_t, _, _ = synth.routing(2, 64, 2, 8, 1.0, "boost0", seed=0)
    h_t = moonep.moonep_create(64, 8, 2, 8, 2, 4, 8)
    t_tk = torch.from_numpy(tk_t).to(dev)
    p_t = moonep.Plan(h_t, dev)
    floor = []
    for i in range(max(8, min(args.steps, 20)) + 3):
        moonep.moonep_combine(h, saved[i % npts], buf, wn, out, gw)
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        moonep.moonep_plan(h_t, t_tk, None, p_t)
        a1.record(stream)
        floor.append((a0, a1))
    torch.cuda.synchronize()
    plan_floor_us = statistics.median(a.elapsed_time(b) for a, b in floor[3:]) * 1e3
    h_t.close()

    plan_ms = [e[0].elapsed_time(e[1]) for e in evs]
    disp_ms = [e[1].elapsed_time(e[2]) for e in evs]
    comb_ms = [e[2].elapsed_time(e[3]) for e in evs]
    db, cb = dc_bytes(R, S, K, H)
    peak, peak_kind = peaks()
    value = aggregate_gbs(db + cb, args.steps, world, total_ms_max)

    sweep = {}
    for j, r in enumerate(routes):
        idx = [i for i in range(args.steps) if i % npts == j]
        if not idx:
            continue
        dc = statistics.median([disp_ms[i] + comb_ms[i] for i in idx])
        gbs = (db + cb) / (dc * 1e-3) / 1e9
        sweep[f"{r['target']:g}"] = dict(
            realised_maxvio=round(r["realised"], 4),
            planner_us=round((statistics.median(with_ms[j]) - statistics.median(without_ms[j])) * 1e3, 2),
            planner_us_event_bracketed=round(statistics.median([plan_ms[i] for i in idx]) * 1e3, 2),
            dispatch_us=round(statistics.median([disp_ms[i] for i in idx]) * 1e3, 1),
            combine_us=round(statistics.median([comb_ms[i] for i in idx]) * 1e3, 1),
            dc_gbs=round(gbs, 1), dc_frac_measured=round(gbs / peak, 4), dc_frac_8tbs=round(gbs / NOMINAL_HBM_GBS, 4))
    dcs = [v["dispatch_us"] + v["combine_us"] for v in sweep.values()]
    spread = (max(dcs) - min(dcs)) / min(dcs) if dcs else None

    d_avg = statistics.mean(disp_ms)
    c_avg = statistics.mean(comb_ms)
    dom = ("dispatch", d_avg, db) if d_avg >= c_avg else ("combine", c_avg, cb)
    achieved = dom[2] / (dom[1] * 1e-3) / 1e9
    roofline = dict(bound="hbm", kernel=dom[0], achieved=round(achieved, 1), peak=peak, unit="GB/s",
                    frac=round(achieved / peak, 4), peak_kind=peak_kind,
                    frac_of_nominal_8tbs=round(achieved / NOMINAL_HBM_GBS, 4),
                    traffic=args.traffic if args.traffic is not None else recorded_traffic(dom[0] + "_kernel"),
                    bytes_per_launch=dom[2])

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms_max / args.steps, 4),
        "higher_is_better": True, "scaling": "weak" if args.replicas else "strong", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{args.config}: " + describe(w), "maxvio": list(w["maxvio"]),
                   "parallelism": (f"EP={R} emulated on each GPU; independent EP groups per GPU" if args.replicas
                                   else f"EP={R} emulated on one GPU (--gpus N shards the same group over N GPUs)"),
                   "l2": "inputs larger than L2 (hidden rows 470 MB, dispatch buffer 4.7 GB per layer)"
                   if args.config == "train" else "inputs larger than L2",
                   "step": "plan + dispatch + combine of one layer; combine reads the dispatch buffer"},
        # planner per layer: median step time with planning minus median
        # step time with saved plans (24 steps per routing and arm, events at
        # the step boundaries only), per routing, averaged over the sweep;
        # also the median planner time between two CUDA events in each step
        # (those come in ~2 us steps and carry the gap an event pair opens
        # between two kernels), launched back to back alone, and the in-step
        # event time of a two-block planner launch (the launch floor)
        "planner_us": round(statistics.mean(v["planner_us"] for v in sweep.values()), 2),
        "planner_us_event_bracketed": round(statistics.median(plan_ms) * 1e3, 2),
        "planner_us_back_to_back": round(plan_b2b_us, 2),
        "planner_launch_floor_us": round(plan_floor_us, 2),
        "dispatch_gbs": round(db / (statistics.median(disp_ms) * 1e-3) / 1e9, 1),
        "combine_gbs": round(cb / (statistics.median(comb_ms) * 1e-3) / 1e9, 1),
        "dc_frac_measured_min": round(min(v["dc_frac_measured"] for v in sweep.values()), 4),
        "dc_frac_8tbs_min": round(min(v["dc_frac_8tbs"] for v in sweep.values()), 4),
        "spread_vs_maxvio": round(spread, 4) if spread is not None else None,
        "sweep": sweep,
        "roofline": roofline,
        "gpu_launches": KERNELS_PER_STEP * args.steps,
        "clocks": clk,
    }

    if not args.no_legs:
        result["legs"] = run_legs(args, dev, world)
        if args.config == "train":
            result["legs"]["pages_maxvio_points"] = run_pages_points(w, seed, dev, h, plan, hidden, weights,
                                                                     buf, wn, out, gw, stream)
            result["legs"]["group_gemm"] = run_group_gemm_leg(dev, seed)
            result["legs"]["fewest_copies"] = run_copies_leg(w, seed, dev)
            result["legs"]["rank_local"] = run_rank_local_leg(w, seed, dev, hidden, weights, routes, stream)
    if not args.no_e2e:
        result["e2e"] = run_e2e(args, h, plan, w, routes, dev, stream, world)
    h.close()
    return result, routes


def run_pages_points(w, seed, dev, h, plan, hidden, weights, buf, wn, out, gw, stream, reps=20):
    """plan + dispatch + combine at the maxvio 10 and 20 points of the pages'
    benchmark, on the training shape and buffers (CUDA events, medians)."""
    import torch
    from load_balancing_planner_b200 import moonep
    R, S, K, E, H = w["R"], w["S"], w["K"], w["E"], w["H"]
    db, cb = dc_bytes(R, S, K, H)
    pts = {}
    for mv in PAGES_POINTS:
        tk, real, _ = synth.routing(R, S, K, E, mv, w["profile"], seed=seed)
        topk = torch.from_numpy(tk).to(dev)
        tpe = torch.from_numpy(synth.local_counts(tk, E)).to(dev)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(reps + 3)]
        for e in evs:
            e[0].record(stream)
            moonep.moonep_plan(h, topk, tpe, plan)
            e[1].record(stream)
            moonep.moonep_dispatch(h, plan, hidden, weights, buf, wn)
            e[2].record(stream)
            moonep.moonep_combine(h, plan, buf, wn, out, gw)
            e[3].record(stream)
        torch.cuda.synchronize()
        if moonep.moonep_read_status(plan) != 0:
            raise RuntimeError(f"plan status at maxvio {mv}")
        evs = evs[3:]
        dc = statistics.median([e[1].elapsed_time(e[3]) for e in evs])
        pts[f"{mv:g}"] = dict(realised_maxvio=round(real, 4),
                              planner_us_event_bracketed=round(
                                  statistics.median([e[0].elapsed_time(e[1]) for e in evs]) * 1e3, 2),
                              dispatch_us=round(statistics.median([e[1].elapsed_time(e[2]) for e in evs]) * 1e3, 1),
                              combine_us=round(statistics.median([e[2].elapsed_time(e[3]) for e in evs]) * 1e3, 1),
                              dc_gbs=round((db + cb) / (dc * 1e-3) / 1e9, 1),
                              used_slots=int((plan.slots() >= 0).sum().item()))
    return pts


def run_rank_local_leg(w, seed, dev, hidden, weights, routes, stream, reps=10):
    """The layer in its per-rank form, as each GPU of a real EP group runs
    it: moonep_plan_rank from the rank's own picks and the gathered counts,
    then moonep_dispatch_rank / moonep_combine_rank through a table of the R
    ranks' buffers (R separate allocations here).  All R ranks' launches run
    back to back on this GPU; bytes and routing are the headline step's.
    Each phase (R plans, R dispatches, R combines) is captured once in a CUDA
    graph and replayed between CUDA events, so the 3R launches carry no host
    gaps; the eager loop is timed as well."""
    import torch
    from load_balancing_planner_b200 import moonep
    R, S, K, E, B, H, tp = w["R"], w["S"], w["K"], w["E"], w["B"], w["H"], w["tp"]
    h = moonep.moonep_create(S, H, K, E, R, B, tp, mode=w["mode"])
    nvs = h.nvs
    bufs = [torch.empty((nvs, H), dtype=torch.bfloat16, device=dev) for _ in range(R)]
    wbufs = [torch.empty((nvs,), dtype=torch.float32, device=dev) for _ in range(R)]
    out = torch.empty((R, S, H), dtype=torch.bfloat16, device=dev)
    gw = torch.empty((R, S, K), dtype=torch.float32, device=dev)
    plans = [moonep.Plan(h, dev, rank=r) for r in range(R)]
    db, cb = dc_bytes(R, S, K, H)
    res = {}
    for rt in routes:
        if rt["target"] not in (0.0, 2.0):
            continue
        topk = [rt["topk"][r].contiguous() for r in range(R)]
        tpe = rt["tpe"]

        def plan_all():
            for r in range(R):
                moonep.moonep_plan_rank(h, r, topk[r], tpe, plans[r])

        def dispatch_all():
            for r in range(R):
                moonep.moonep_dispatch_rank(h, plans[r], hidden[r], weights[r], bufs, wbufs)

        def combine_all():
            for r in range(R):
                moonep.moonep_combine_rank(h, plans[r], bufs, wbufs, out[r], gw[r])

        phases = (plan_all, dispatch_all, combine_all)

        def timed(run):
            evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(reps + 3)]
            for e in evs:
                for j, f in enumerate(run):
                    e[j].record(stream)
                    f()
                e[3].record(stream)
            torch.cuda.synchronize()
            evs = evs[3:]
            return [statistics.median([e[j].elapsed_time(e[j + 1]) for e in evs]) for j in range(3)]

        for f in phases:
            f()
        torch.cuda.synchronize()
        if any(moonep.moonep_read_status(p) != 0 for p in plans):
            raise RuntimeError("rank plan status")
        eager = timed(phases)
        point = dict(eager=dict(planner_us_per_rank=round(eager[0] * 1e3 / R, 2),
                                dispatch_us=round(eager[1] * 1e3, 1), combine_us=round(eager[2] * 1e3, 1),
                                dc_gbs=round((db + cb) / ((eager[1] + eager[2]) * 1e-3) / 1e9, 1)))
        try:
            graphs = []
            for f in phases:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    f()
                graphs.append(g)
            torch.cuda.synchronize()
            pt, dt, ct = timed([g.replay for g in graphs])
            if any(moonep.moonep_read_status(p) != 0 for p in plans):
                raise RuntimeError("rank plan status after graph replays")
            point.update(planner_us_per_rank=round(pt * 1e3 / R, 2),
                         dispatch_us=round(dt * 1e3, 1), combine_us=round(ct * 1e3, 1),
                         dc_gbs=round((db + cb) / ((dt + ct) * 1e-3) / 1e9, 1))
            del graphs
        except RuntimeError as ex:  # capture refused: the eager numbers stand alone
            point["graph_error"] = str(ex)[:200]
        res[f"{rt['target']:g}"] = point
    h.close()
    return dict(workload=describe(w) + "; per-rank calls of all R ranks, buffers as R allocations",
                planner="R rank plans back to back per layer, reported per rank (each GPU of a real group "
                        "plans only its own share, concurrently)",
                timing="each phase's R launches as one CUDA graph, replayed between CUDA events; "
                       "'eager' = the same calls from Python",
                points=res)


def run_copies_leg(w, seed, dev, Hp=2048, n_proj=3, reps=50):
    """Copies per layer of the two training planners on the same routings
    (the sweep plus the pages' maxvio 10 and 20 points): used slots, i.e.
    distinct (expert, recipient) pairs, and the weight bytes the prefetch of
    those slots moves per layer (n_proj projections of [H, H'] bf16: each
    distinct copied expert read once, each slot written once).  Mode 0 gives
    a donor's experts away in id order, mode 3 largest first.  Also the
    back-to-back planner time of each mode."""
    import torch
    from load_balancing_planner_b200 import moonep
    R, S, K, E, B, H, tp = w["R"], w["S"], w["K"], w["E"], w["B"], w["H"], w["tp"]
    hs = {m: moonep.moonep_create(S, H, K, E, R, B, tp, mode=m) for m in (0, 3)}
    out = {"mv": [], "copies_mode0": [], "copies_mode3": [], "prefetch_gb_mode0": [], "prefetch_gb_mode3": []}
    b2b = {}
    routes = []
    for mv in tuple(w["maxvio"]) + PAGES_POINTS:
        tk, real, _ = synth.routing(R, S, K, E, mv, w["profile"], seed=seed)
        routes.append((torch.from_numpy(tk).to(dev), torch.from_numpy(synth.local_counts(tk, E)).to(dev)))
        out["mv"].append(mv)
        for m, h in hs.items():
            p = moonep.moonep_plan(h, *routes[-1])
            torch.cuda.synchronize()
            if moonep.moonep_read_status(p) != 0:
                raise RuntimeError(f"mode {m} plan status")
            se = p.slots().cpu().numpy()
            U = int((se >= 0).sum())
            D = int(np.unique(se[se >= 0]).size)
            out[f"copies_mode{m}"].append(U)
            out[f"prefetch_gb_mode{m}"].append(round(n_proj * (D + U) * H * Hp * 2 / 1e9, 2))
    # Each mode's planner back to back on the GPU: the plans of every routing,
    # three times over, as one CUDA graph replayed between CUDA events (an
    # eager loop here would time the host's launches as much as the GPU).
    stream = torch.cuda.Stream(dev)
    for m, h in hs.items():
        p = moonep.Plan(h, dev)
        stream.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(stream):
            for i in range(len(routes)):
                moonep.moonep_plan(h, *routes[i], p)
        torch.cuda.current_stream(dev).wait_stream(stream)
        torch.cuda.synchronize()
        n = 3 * len(routes)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(n):
                moonep.moonep_plan(h, *routes[i % len(routes)], p)
        g.replay()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps // 10):
            g.replay()
        b.record()
        torch.cuda.synchronize()
        if moonep.moonep_read_status(p) != 0:
            raise RuntimeError(f"mode {m} plan status after graph replays")
        b2b[f"mode{m}"] = round(a.elapsed_time(b) * 1e3 / (n * (reps // 10)), 2)
        del g
        h.close()
    out["planner_us_graph_back_to_back"] = b2b
    out["workload"] = f"{describe(w)}; prefetch of {n_proj} projections [H, H'={Hp}] bf16 per copy"
    return out


def run_group_gemm_leg(dev, seed, mv=2.0, Hp=2048, reps=10, config="train"):
    """The VM group GEMM that consumes a dispatched training layer: one
    [H, H'] projection per plan row (home experts from W, slot rows from the
    prefetched pool), H' = 2048, bf16 in, fp32 accumulation, bf16 out.
    FLOPs count the real slots only (2 * R*S*K * H * H'); the kernel also
    multiplies each row's padding up to a multiple of 128."""
    import torch
    from load_balancing_planner_b200 import moonep
    w = WORKLOADS[config]
    R, S, K, E, B, H, tp = w["R"], w["S"], w["K"], w["E"], w["B"], w["H"], w["tp"]
    tk, real, _ = synth.routing(R, S, K, E, mv, w["profile"], seed=seed)
    h = moonep.moonep_create(S, H, K, E, R, B, tp)
    plan = moonep.moonep_plan(h, torch.from_numpy(tk).to(dev), torch.from_numpy(synth.local_counts(tk, E)).to(dev))
    x, _ = moonep.moonep_dispatch(h, plan, synth.hidden_bf16(R, S, H, seed).to(dev))
    g = torch.Generator(device=dev).manual_seed(seed)
    W = (torch.randn((E, H, Hp), generator=g, device=dev) * H ** -0.5).to(torch.bfloat16)
    pool = torch.empty((R, B, H, Hp), dtype=torch.bfloat16, device=dev)
    moonep.moonep_prefetch_weight(h, plan, [W], [pool])
    y = torch.empty((R, h.nvs, Hp), dtype=torch.bfloat16, device=dev)
    for _ in range(3):
        moonep.moonep_group_gemm(h, plan, x, W, pool, y)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in evs:
        a.record()
        moonep.moonep_group_gemm(h, plan, x, W, pool, y)
        b.record()
    torch.cuda.synchronize()
    if moonep.moonep_read_status(plan) != 0:
        raise RuntimeError("group GEMM: plan status")
    us = statistics.median(a.elapsed_time(b) for a, b in evs) * 1e3
    rows_computed = int(plan.cu_seqlens[:, -1].sum().item())
    flops = 2.0 * R * S * K * H * Hp
    burst, sustained, kind = tensor_peaks()
    tf = flops / (us * 1e-6) / 1e12
    h.close()
    return {"workload": f"{config}: {describe(w)}; plan at maxvio {mv:g}, H'={Hp}, bf16 -> fp32 accumulate -> bf16",
            "realised_maxvio": round(real, 4), "flops": flops, "us": round(us, 1), "tflops": round(tf, 1),
            "frac_of_bf16_burst": round(tf / burst, 4), "frac_of_bf16_sustained": round(tf / sustained, 4),
            "peak_kind": kind, "rows_real": R * S * K, "rows_computed": rows_computed}


def run_legs(args, dev, world, Hp=2048, reps=5):
    """prefetch_weight at the inference shape and reduce_grad at the backward
    shape, timed with CUDA events (median of reps).  A smaller H' gives the
    same kernels on less memory, for profiler captures."""
    import torch
    from load_balancing_planner_b200 import moonep
    legs = {}
    peak, _ = peaks()
    R, S, K, E, H, tp = 8, 4096, 8, 256, 7168, 128
    gen = torch.Generator(device=dev).manual_seed(args.seed)

    def timed(fn):
        # All launches are enqueued back to back, so each start event is
        # reached while the launch before it runs and the launch itself is
        # already queued: the events time the kernel, not the host's launch
        # latency.  The first pair starts on an idle stream and is dropped.
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps + 1)]
        for a, b in evs:
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in evs[1:])

    # prefetch_weight: inference, B = 4, three projections
    h = moonep.moonep_create(S, H, K, E, R, 4, tp, mode=1)
    Ws = [torch.randn((E, H, Hp), generator=gen, device=dev, dtype=torch.bfloat16) for _ in range(3)]
    pools = [torch.empty((R, 4, H, Hp), dtype=torch.bfloat16, device=dev) for _ in range(3)]
    out = {}
    for mv in (1.0, 4.0):
        tk, real, _ = synth.routing(R, S, K, E, mv, "hot8", seed=args.seed)
        p = moonep.moonep_plan(h, torch.from_numpy(tk).to(dev), torch.from_numpy(synth.local_counts(tk, E)).to(dev))
        torch.cuda.synchronize()
        se = p.slots().cpu().numpy()
        U = int((se >= 0).sum())
        D = int(np.unique(se[se >= 0]).size)
        ms = timed(lambda: moonep.moonep_prefetch_weight(h, p, Ws, pools))
        by = 3 * (D + U) * H * Hp * 2
        # picks left on overflow rows (weights read from the home rank), with
        # the slots given by id (mode 1, timed here) and by picks (mode 2)
        ovf = {}
        for mode in (1, 2):
            hm = moonep.moonep_create(S, H, K, E, R, 4, tp, mode=mode)
            pm = moonep.moonep_plan(hm, torch.from_numpy(tk).to(dev),
                                    torch.from_numpy(synth.local_counts(tk, E)).to(dev))
            rc = pm.row_counts.cpu().numpy()
            ovf[mode] = int(sum(rc[r, e] for r in range(R) for e in range(E) if e // (E // R) != r))
            hm.close()
        out[f"{mv:g}"] = dict(realised_maxvio=round(real, 4), used_slots=U, distinct_experts=D,
                              us=round(ms * 1e3, 1), gbs=round(by / (ms * 1e-3) / 1e9, 1),
                              frac_measured=round(by / (ms * 1e-3) / 1e9 / peak, 4),
                              overflow_picks_slots_by_id=ovf[1], overflow_picks_slots_by_count=ovf[2])
    legs["prefetch_weight"] = dict(workload=f"inference R=8 S=4096 K=8 E=256 B=4 H=7168 H'={Hp}, 3 projections",
                                   bytes="3*(D+U)*H*H'*2", points=out)
    del Ws, pools
    h.close()

    # reduce_grad: training plan at maxvio 2, one fp32 projection
    h = moonep.moonep_create(S, H, K, E, R, 32, tp, mode=0)
    tk, real, _ = synth.routing(R, S, K, E, 2.0, "hot8", seed=args.seed)
    p = moonep.moonep_plan(h, torch.from_numpy(tk).to(dev), torch.from_numpy(synth.local_counts(tk, E)).to(dev))
    G = torch.randn((E, H, Hp), generator=gen, device=dev).mul_(1e-3)
    RB = torch.randn((R, 32, H, Hp), generator=gen, device=dev).mul_(1e-3)
    torch.cuda.synchronize()
    se = p.slots().cpu().numpy()
    U = int((se >= 0).sum())
    D = int(np.unique(se[se >= 0]).size)
    ms = timed(lambda: moonep.moonep_reduce_grad(h, p, [G], [RB]))
    by = (2 * D + 2 * U) * H * Hp * 4
    legs["reduce_grad"] = dict(workload=f"backward E=256 R=8 B=32 H=7168 H'={Hp} fp32, plan at maxvio 2",
                               bytes="(2D+2U)*H*H'*4", realised_maxvio=round(real, 4), used_slots=U,
                               distinct_experts=D, us=round(ms * 1e3, 1),
                               gbs=round(by / (ms * 1e-3) / 1e9, 1),
                               frac_measured=round(by / (ms * 1e-3) / 1e9 / peak, 4))
    del G, RB
    h.close()
    torch.cuda.empty_cache()
    return legs


def run_e2e(args, h, plan, w, routes, dev, stream, world):
    """The same step through the C ABI from pinned host buffers: H2D of the
    step's inputs, plan, dispatch, combine, D2H of the combined output.

    Steps are pipelined over three streams with two buffer sets, the way a
    data loader feeds a GPU: step i+1's inputs go up and step i-1's output
    comes down (PCIe is full duplex) while step i computes.  Every step's
    copies are inside the timed region, which runs from the first upload to
    the last download."""
    import torch
    from load_balancing_planner_b200 import moonep
    R, S, K, E, H = w["R"], w["S"], w["K"], w["E"], w["H"]
    nvs = h.nvs
    hid_h = synth.hidden_bf16(R, S, H, args.seed).pin_memory()
    wts_h = torch.from_numpy(synth.route_weights(R, S, K, args.seed)).pin_memory()
    tks_h = [r["topk"].cpu().pin_memory() for r in routes]
    tpe_h = [r["tpe"].cpu().pin_memory() for r in routes]
    out_h = [torch.empty((R, S, H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    hid_d = [torch.empty((R, S, H), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    wts_d = [torch.empty((R, S, K), dtype=torch.float32, device=dev) for _ in range(2)]
    tk_d = [torch.empty((R, S, K), dtype=torch.int32, device=dev) for _ in range(2)]
    tpe_d = [torch.empty((R, E), dtype=torch.int32, device=dev) for _ in range(2)]
    out = [torch.empty((R, S, H), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    buf = torch.empty((R, nvs, H), dtype=torch.bfloat16, device=dev)
    wn = torch.empty((R, nvs), dtype=torch.float32, device=dev)
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("up", "done", "down")}
    used = {k: [False, False] for k in ev}

    def step(i):
        j, sl = i % len(routes), i % 2
        with torch.cuda.stream(up):
            if used["done"][sl]:
                up.wait_event(ev["done"][sl])  # step i-2 no longer reads these inputs
            hid_d[sl].copy_(hid_h, non_blocking=True)
            wts_d[sl].copy_(wts_h, non_blocking=True)
            tk_d[sl].copy_(tks_h[j], non_blocking=True)
            tpe_d[sl].copy_(tpe_h[j], non_blocking=True)
            ev["up"][sl].record(up)
        stream.wait_event(ev["up"][sl])
        if used["down"][sl]:
            stream.wait_event(ev["down"][sl])  # step i-2's output has left the device
        moonep.moonep_plan(h, tk_d[sl], tpe_d[sl], plan, stream=stream)
        moonep.moonep_dispatch(h, plan, hid_d[sl], wts_d[sl], buf, wn, stream=stream)
        moonep.moonep_combine(h, plan, buf, wn, out[sl], None, gather=False, stream=stream)
        ev["done"][sl].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(ev["done"][sl])
            out_h[sl].copy_(out[sl], non_blocking=True)
            ev["down"][sl].record(down)
        for k in ev:
            used[k][sl] = True

    # enough steps that the pipeline's fill (first upload) and drain (last
    # download) weigh little against the steady state
    n = max(6, min(args.steps, 6 * len(routes)))
    for i in range(2):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    up.wait_stream(stream)  # the first upload starts after the start mark
    for i in range(n):
        step(i)
    stream.wait_stream(down)  # the end mark follows the last download
    b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(a.elapsed_time(b), world)
    db, cb = dc_bytes(R, S, K, H)
    cb -= R * S * K * 4  # this combine does not gather the weights back
    h2d = hid_h.numel() * 2 + wts_h.numel() * 4 + tks_h[0].numel() * 4 + tpe_h[0].numel() * 4
    return {"value": round(aggregate_gbs(db + cb, n, world, ms), 1), "unit": "GB/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(out_h[0].numel() * 2),
            "ms_per_step": round(ms / n, 3), "steps": n,
            "pipelined": "uploads, compute and downloads of consecutive steps overlap on 3 streams"}


# ---------------------------------------------------------------- EP over processes
def ep_layout(R, world, rank):
    """The EP ranks process `rank` of `world` owns: R/world consecutive ranks."""
    if R % world:
        raise ValueError(f"{R} EP ranks do not split over {world} processes")
    per = R // world
    return list(range(rank * per, (rank + 1) * per))


def ep_bytes(R, S, K, H):
    """Algorithmic bytes of one sharded layer: the same rows move as in the
    emulated group (dispatch + combine of all R ranks' tokens)."""
    return sum(dc_bytes(R, S, K, H))


def run_ep(args, world, rank, local):
    """One EP group of R ranks sharded over `world` processes (see the module
    docstring).  Host barriers order the phases of every step: all plans
    before any dispatch writes, all dispatches before any combine reads, all
    combines before the next step's dispatch."""
    import datetime

    import torch
    import torch.distributed as dist
    from load_balancing_planner_b200 import ep, moonep

    w = WORKLOADS[args.config]
    R, S, K, E, B, H, tp = w["R"], w["S"], w["K"], w["E"], w["B"], w["H"], w["tp"]
    mine = ep_layout(R, world, rank)
    dev = torch.device("cuda", local)
    nccl = dist.get_backend() == "nccl"
    host = dist.new_group(backend="gloo", timeout=datetime.timedelta(seconds=120)) if nccl else None

    # the whole group's routing from the shared seed; this process keeps its ranks' share
    hid_all = synth.hidden_bf16(R, S, H, args.seed)
    w_all = synth.route_weights(R, S, K, args.seed)
    hidden = [hid_all[r].contiguous().to(dev) for r in mine]
    weights = [torch.from_numpy(w_all[r].copy()).to(dev) for r in mine]
    del hid_all
    routes = []
    for mv in w["maxvio"]:
        tk, real, _ = synth.routing(R, S, K, E, mv, w["profile"], seed=args.seed)
        tpe = synth.local_counts(tk, E)
        routes.append(dict(target=mv, realised=real,
                           topk=[torch.from_numpy(np.ascontiguousarray(tk[r])).to(dev) for r in mine],
                           tpe=torch.from_numpy(tpe[mine].copy()).to(dev if nccl else "cpu")))
    h = moonep.moonep_create(S, H, K, E, R, B, tp, mode=w["mode"])
    nvs = h.nvs
    bufs = [torch.empty((nvs, H), dtype=torch.bfloat16, device=dev) for _ in mine]
    wbufs = [torch.empty((nvs,), dtype=torch.float32, device=dev) for _ in mine]
    peers = ep.IpcPeers(bufs + wbufs, group=host)
    per = len(mine)
    # rank q's buffer: tensor (q % per) of process q // per
    buf_tab = moonep.PeerTable([peers.rows[q // per][q % per] for q in range(R)], (nvs, H), torch.bfloat16)
    w_tab = moonep.PeerTable([peers.rows[q // per][per + q % per] for q in range(R)], (nvs,), torch.float32)
    plans = [moonep.Plan(h, dev, rank=r) for r in mine]
    outs = [torch.empty((S, H), dtype=torch.bfloat16, device=dev) for _ in mine]
    gws = [torch.empty((S, K), dtype=torch.float32, device=dev) for _ in mine]
    stream = torch.cuda.current_stream(dev)
    npts = len(routes)

    def sync():
        torch.cuda.synchronize(dev)
        dist.barrier(group=host)

    def gather(r):
        # every rank's router counts, [R, E], in rank order
        parts = [torch.empty_like(r["tpe"]) for _ in range(world)]
        dist.all_gather(parts, r["tpe"])
        return torch.cat(parts).to(dev)

    def step(i, ev=None):
        r = routes[i % npts]
        if ev:
            ev[0].record(stream)
        counts = gather(r)
        for j, q in enumerate(mine):
            moonep.moonep_plan_rank(h, q, r["topk"][j], counts, plans[j])
        sync()
        if ev:
            ev[1].record(stream)
        for j in range(per):
            moonep.moonep_dispatch_rank(h, plans[j], hidden[j], weights[j], buf_tab, w_tab)
        sync()
        if ev:
            ev[2].record(stream)
        for j in range(per):
            moonep.moonep_combine_rank(h, plans[j], buf_tab, w_tab, outs[j], gws[j])
        sync()
        if ev:
            ev[3].record(stream)

    for i in range(args.warmup):
        step(i)
    sync()
    st = max(moonep.moonep_read_status(p) for p in plans)
    if st != 0:
        raise RuntimeError(f"plan status {st}")
    # the sharded step equals the emulated group's: each rank's plan against
    # the group planner on the same routing, and the combined rows of the last
    # step (weighted combine of the dispatched rows = the token itself)
    check = moonep.moonep_plan(h, torch.from_numpy(synth.routing(R, S, K, E, w["maxvio"][(args.warmup - 1) % npts],
                                                                 w["profile"], seed=args.seed)[0]).to(dev))
    torch.cuda.synchronize(dev)
    for j, q in enumerate(mine):
        if not torch.equal(plans[j].dst, check.dst[q]):
            raise RuntimeError(f"rank {q}: plan differs from the group plan")
        if not torch.equal(outs[j].float(), hidden[j].float()):
            raise RuntimeError(f"rank {q}: combine(dispatch(x)) is not x")
    clocks = Clocks(local)
    clocks.start()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    sync()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        step(i, evs[i])
    t1.record(stream)
    sync()
    clk = clocks.stop()
    total_ms = max_over_ranks(t0.elapsed_time(t1), world)
    phase = [max_over_ranks(statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs), world) for j in range(3)]
    total_b = ep_bytes(R, S, K, H)
    value = total_b * args.steps / (total_ms * 1e-3) / 1e9
    remote = sum(int((p.dst // nvs != q).sum().item()) for p, q in zip(plans, mine))
    remote_rows = max_over_ranks(remote, world)

    # e2e: every step also brings this process's ranks' inputs up from pinned
    # host memory and takes their combined rows back down
    hid_h = [x.cpu().pin_memory() for x in hidden]
    w_h = [x.cpu().pin_memory() for x in weights]
    tk_h = [[t.cpu().pin_memory() for t in r["topk"]] for r in routes]
    out_h = [torch.empty((S, H), dtype=torch.bfloat16).pin_memory() for _ in mine]

    def e2e_step(i):
        r = routes[i % npts]
        for j in range(per):
            hidden[j].copy_(hid_h[j], non_blocking=True)
            weights[j].copy_(w_h[j], non_blocking=True)
            r["topk"][j].copy_(tk_h[i % npts][j], non_blocking=True)
        step(i)
        for j in range(per):
            out_h[j].copy_(outs[j], non_blocking=True)
        torch.cuda.synchronize(dev)

    n_e2e = max(3, min(args.steps, 2 * npts))
    e2e_step(0)
    sync()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(n_e2e):
        e2e_step(i)
    b.record(stream)
    sync()
    e2e_ms = max_over_ranks(a.elapsed_time(b), world)
    h2d = per * (S * H * 2 + S * K * 4 + S * K * 4)  # this process's hidden rows, route weights and picks
    peers_n = world
    peers.close()
    h.close()
    return {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4),
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"{args.config}: " + describe(w), "maxvio": list(w["maxvio"]),
                   "parallelism": f"EP={R} sharded over {peers_n} processes, {per} ranks each; buffers mapped "
                                  f"with CUDA IPC; phases ordered by host barriers",
                   "l2": "inputs larger than L2",
                   "step": "counts all-gather + plan_rank, dispatch_rank, combine_rank of every rank"},
        "phase_ms_max_over_ranks": {"plan+gather": round(phase[0], 4), "dispatch": round(phase[1], 4),
                                    "combine": round(phase[2], 4)},
        "remote_picks_per_process_max": remote_rows,
        "gpu_launches": 3 * per * args.steps,
        "clocks": clk,
        "e2e": {"value": round(total_b * n_e2e / (e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                "h2d_bytes_per_step": int(h2d * world), "d2h_bytes_per_step": int(R * S * H * 2),
                "ms_per_step": round(e2e_ms / n_e2e, 3), "steps": n_e2e},
    }


# ---------------------------------------------------------------- the oracle
def oracle_sample(w, routes_np, ranks_sampled, seed):
    """Time the CPU oracle as it stands on one host core: the full plan of
    every routing, then dispatch and combine of every token of the first
    `ranks_sampled` source ranks (their slots remapped to a compact buffer).
    Returns (dispatch+combine bytes, seconds)."""
    import torch

    import oracle
    R, S, K, E, B, H, tp = w["R"], w["S"], w["K"], w["E"], w["B"], w["H"], w["tp"]
    n = ranks_sampled
    x = synth.bf16_bits(torch.from_numpy(synth.normal_f32((n, S, H), seed)).to(torch.bfloat16))
    wts = synth.route_weights(n, S, K, seed)
    total_b, total_s = 0, 0.0
    for tk in routes_np:
        t0 = time.perf_counter()
        p = oracle.plan(tk, E, B, tp, w["mode"], synth.local_counts(tk, E))
        d = p["dst"][:n]
        # compact slot numbering of the sampled picks, in the plan's own slot order
        order = np.argsort(d.reshape(-1), kind="stable")
        comp = np.empty(d.size, np.int32)
        comp[order] = np.arange(d.size, dtype=np.int32)
        comp = comp.reshape(d.shape)
        buf, wn = oracle.dispatch(comp, x, wts, d.size // n)
        oracle.combine(comp, buf, wn)
        total_s += time.perf_counter() - t0
        db, cb = dc_bytes(n, S, K, H)
        total_b += db + cb
    return total_b, total_s


def oracle_weight_legs(seed, H=7168, Hp=2048, experts=2):
    """The oracle's prefetch and reduce_grad on one host core, on a sample of
    the inference / backward legs: `experts` expert matrices [H, H'], each
    copied to two slots (prefetch) or summed from two slots (reduce_grad).
    Returns {leg: GB/s} over the legs' algorithmic bytes."""
    import oracle
    hhp = H * Hp
    g = np.random.default_rng(seed)
    se = np.full((2, experts), -1, np.int32)
    se[0, :] = np.arange(experts)
    se[1, :] = np.arange(experts)  # two holders per expert
    W = g.integers(0, 1 << 16, size=(experts, hhp), dtype=np.uint16)
    pool = np.zeros((2 * experts, hhp), np.uint16)
    t0 = time.perf_counter()
    oracle.prefetch(se, W, pool)
    t_pf = time.perf_counter() - t0
    G = g.standard_normal((experts, hhp), dtype=np.float32)
    RB = g.standard_normal((2 * experts, hhp), dtype=np.float32)
    t0 = time.perf_counter()
    oracle.reduce_grad(se, G, RB)
    t_rg = time.perf_counter() - t0
    d, u = experts, 2 * experts
    return {"prefetch_weight_gbs": round((d + u) * hhp * 2 / t_pf / 1e9, 3),
            "reduce_grad_gbs": round((2 * d + 2 * u) * hhp * 4 / t_rg / 1e9, 3),
            "sample": f"{experts} expert matrices [{H}, {Hp}], two slots each"}


def cpu_baseline(w, routes, seed):
    ranks = 4
    b, s = oracle_sample(w, [r["topk_np"] for r in routes], ranks, seed)
    return {"value": round(b / s / 1e9, 3), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"plan of {len(routes)} routings + D/C of {ranks} of {w['R']} source ranks, 1 thread, {s:.1f} s",
            "host_cores_available": os.cpu_count(),
            "legs": oracle_weight_legs(seed)}


# ---------------------------------------------------------------- reference arm
def run_reference(args, world, rank):
    """The base contract's reference arm is the CPU oracle here: each step is a
    bounded sample of the same workload (full plan + dispatch/combine of one
    source rank's tokens) timed on the host."""
    if rank != 0:
        return None
    w = WORKLOADS[args.config]
    routes = []
    for mv in w["maxvio"]:
        tk, real, _ = synth.routing(w["R"], w["S"], w["K"], w["E"], mv, w["profile"], seed=args.seed)
        routes.append(tk)
    for i in range(args.warmup):
        oracle_sample(w, [routes[i % len(routes)]], 1, args.seed)
    tb, ts = 0, 0.0
    for i in range(args.steps):
        b, s = oracle_sample(w, [routes[i % len(routes)]], 1, args.seed)
        tb += b
        ts += s
    v = round(tb / ts / 1e9, 3)
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ts / args.steps * 1e3, 1),
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"{args.config}: " + describe(w), "maxvio": list(w["maxvio"])},
        "cpu_baseline": {"value": v, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": "per step: full plan of one routing (all ranks) + dispatch and combine of "
                                   "every token of 1 source rank, single-threaded C"},
        "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_planner_only(args):
    """The planner alone on the workload's routings, back to back: a small
    program (the routing and plan arrays only) for profiler captures."""
    import torch
    from load_balancing_planner_b200 import moonep
    w = WORKLOADS[args.config]
    R, S, K, E, B, H, tp = w["R"], w["S"], w["K"], w["E"], w["B"], w["H"], w["tp"]
    dev = torch.device("cuda", 0)
    routes = []
    for mv in w["maxvio"]:
        tk, _, _ = synth.routing(R, S, K, E, mv, w["profile"], seed=args.seed)
        routes.append((torch.from_numpy(tk).to(dev), torch.from_numpy(synth.local_counts(tk, E)).to(dev)))
    h = moonep.moonep_create(S, H, K, E, R, B, tp, mode=w["mode"])
    plan = moonep.Plan(h, dev)
    for i in range(args.warmup):
        moonep.moonep_plan(h, *routes[i % len(routes)], plan)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(args.steps):
        moonep.moonep_plan(h, *routes[i % len(routes)], plan)
    b.record()
    torch.cuda.synchronize()
    st = moonep.moonep_read_status(plan)
    h.close()
    return {"planner_only": args.config, "launches": args.warmup + args.steps, "status": st,
            "back_to_back_us": round(a.elapsed_time(b) * 1e3 / args.steps, 2)}


def split_result(result):
    """(detail, line): the bulky parts of a run (legs, the full per-maxvio
    sweep, the CPU legs) and the contract line, which keeps every headline
    figure -- planner us per layer, dispatch+combine GB/s and fraction at each
    maxvio, the spread -- in a compact form."""
    line = dict(result)
    detail = {}
    if "legs" in line:
        detail["legs"] = line.pop("legs")
    sweep = line.pop("sweep", {})
    detail["sweep"] = sweep
    line["sweep"] = {mv: {"dc_gbs": v["dc_gbs"], "frac": v["dc_frac_measured"], "plan_us": v["planner_us"],
                          "plan_ev_us": v["planner_us_event_bracketed"]} for mv, v in sweep.items()}
    pts = detail.get("legs", {}).get("pages_maxvio_points")
    if pts:
        line["pages_points"] = {mv: {"dc_gbs": v["dc_gbs"], "plan_ev_us": v["planner_us_event_bracketed"]}
                                for mv, v in pts.items()}
        evs = [v["plan_ev_us"] for v in line["sweep"].values()] + [v["plan_ev_us"] for v in line["pages_points"].values()]
        line["planner_us_event_bracketed_max"] = max(evs)
    fc = detail.get("legs", {}).get("fewest_copies")
    if fc:
        line["copies_by_maxvio"] = {"mv": fc["mv"], "mode0": fc["copies_mode0"], "mode3": fc["copies_mode3"]}
    for k in ("prefetch_weight", "reduce_grad", "group_gemm"):
        leg = detail.get("legs", {}).get(k)
        if leg is None:
            continue
        if k == "prefetch_weight":
            line["prefetch_frac"] = {mv: v["frac_measured"] for mv, v in leg["points"].items()}
        elif k == "reduce_grad":
            line["reduce_grad_frac"] = leg["frac_measured"]
        else:
            line["group_gemm_tflops"] = leg["tflops"]
    if "cpu_baseline" in line:
        cb = dict(line["cpu_baseline"])
        if "legs" in cb:
            detail["cpu_legs"] = cb.pop("legs")
        line["cpu_baseline"] = cb
    if "e2e" in line:
        e = dict(line["e2e"])
        detail["e2e_pipelining"] = e.pop("pipelined", None)
        line["e2e"] = e
    return detail, line


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--config", choices=tuple(WORKLOADS), default="train")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-legs", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu DRAM bytes per launch of the dominant kernel, if measured for this build")
    ap.add_argument("--gemm-only", action="store_true",
                    help="time only the group GEMM on the workload (first maxvio of its sweep), for profiler "
                         "captures; prints the leg's JSON, not a bench line")
    ap.add_argument("--hp", type=int, default=2048, help="H' of the group GEMM and of the weight legs")
    ap.add_argument("--weights-only", action="store_true",
                    help="run only the prefetch_weight and reduce_grad legs at H' = --hp, --steps timed launches "
                         "per point, for profiler captures; prints the legs' JSON, not a bench line")
    ap.add_argument("--share-gpu", action="store_true",
                    help="under torchrun: every process on GPU 0 over gloo (checks the sharded path on one GPU; "
                         "its timings are not a measurement)")
    ap.add_argument("--replicas", action="store_true",
                    help="with --gpus N > 1: an independent emulated EP group per GPU instead of one group "
                         "sharded over the GPUs")
    ap.add_argument("--planner-only", action="store_true",
                    help="launch only the planner (every routing of the workload), for profiler captures; "
                         "prints its back-to-back time, not a bench line")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.planner_only:
        print(json.dumps(run_planner_only(args)), flush=True)
        return
    if args.weights_only:
        import torch
        print(json.dumps(run_legs(args, torch.device("cuda", 0), 1, Hp=args.hp, reps=args.steps)), flush=True)
        return
    if args.gemm_only:
        import torch
        w = WORKLOADS[args.config]
        print(json.dumps(run_group_gemm_leg(torch.device("cuda", 0), args.seed, mv=w["maxvio"][0], Hp=args.hp,
                                            reps=args.steps, config=args.config)), flush=True)
        return

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        res = run_reference(args, world, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    world, rank, local = setup_dist(args)
    if world > 1 and not args.replicas:
        result = run_ep(args, world, rank, local)
        if rank == 0:
            print(json.dumps(result), flush=True)
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
        return
    result, routes = run_ours(args, world, rank, local)
    if rank == 0 and world == 1 and not args.no_cpu:
        result["cpu_baseline"] = cpu_baseline(WORKLOADS[args.config], routes, args.seed)
    if rank == 0:
        detail, line = split_result(result)
        # the detail first, on its own line; the contract line stays short and last
        print(json.dumps({"detail": detail}), flush=True)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
