"""The N-GPU path of bench.py on CPU with gloo, world size 2: every rank runs
its own independent EP group (different seeds, no data-path collective), the
timing is the max over ranks, and the value aggregates all ranks' bytes."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from load_balancing_planner_b200 import synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    try:
        # each rank plans its own routing with the oracle (host stand-in for
        # the device planner): independent problems, nothing exchanged
        seed = bench.rank_seed(0, rank)
        tk, mv, _ = synth.routing(4, 64, 4, 16, 1.5, "hot8", seed=seed)
        p = oracle.plan(tk, 16, 4, 8)
        t_ms = 10.0 * (rank + 1)
        tmax = bench.max_over_ranks(t_ms, world)
        q.put((rank, int(p["status"]), int(p["dst"].sum()), tmax))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_rank_bench_logic_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for pr in procs:
        pr.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    (r0, st0, s0, m0), (r1, st1, s1, m1) = res
    assert st0 == st1 == 0
    assert s0 != s1, "ranks must draw different problems"
    assert m0 == m1 == 20.0, "timing is the max over ranks"


def test_aggregate_value_counts_all_ranks():
    import bench
    assert bench.aggregate_gbs(1e9, 10, 4, 1000.0) == pytest.approx(40.0)
    assert bench.rank_seed(3, 2) == 5


def _gather_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    import torch
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from load_balancing_planner_b200.ep import gather_counts
    try:
        # one EP group of `world` ranks: the same seeded routing everywhere,
        # each rank keeping only its own picks and their local counts
        tk, _, _ = synth.routing(world, 64, 4, 16, 1.5, "hot8", seed=7)
        mine = torch.from_numpy(synth.local_counts(tk[rank:rank + 1], 16)[0].copy())
        table = gather_counts(mine).numpy()
        # what the rank planner needs: the group's counts in rank order, which
        # the oracle accepts as the router counts of the group's picks
        ok = np.array_equal(table, synth.local_counts(tk, 16))
        st = oracle.plan(tk, 16, 8, 8, 0, table)["status"]
        # this rank's share from its own picks and the gathered table equals
        # its slice of the plan of the whole group
        mine = oracle.plan_rank(tk[rank], table, rank, 16, 8, 8, 0)
        group = oracle.plan(tk, 16, 8, 8, 0)
        ok = ok and mine["status"] == 0 and np.array_equal(mine["dst"], group["dst"][rank]) and \
            np.array_equal(mine["cu_seqlens"], group["cu_seqlens"])
        q.put((rank, bool(ok), int(st), table.tobytes()))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_rank_count_gather_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_worker, args=(r, 2, port, q)) for r in range(2)]
    for pr in procs:
        pr.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    (_, ok0, st0, t0), (_, ok1, st1, t1) = res
    assert ok0 and ok1
    assert st0 == st1 == 0
    assert t0 == t1, "every rank holds the same table"


def test_reference_arm_prints_one_contract_line():
    # `bench.py --impl reference` (the CPU oracle, the base contract's
    # reference arm) prints one JSON line with the keys the driver reads
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "zipf", "--steps", "1",
                          "--warmup", "3"], cwd=root, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-500:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1 and d["warmup"] == 3
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_bench_contract_line_is_short_and_keeps_the_headline_figures():
    # the driver keeps only the tail of stdout: the bulky legs go on an
    # earlier line, and the last line keeps the planner us, the per-maxvio
    # fractions and the spread
    import json

    import bench
    sweep = {f"{m:g}": dict(realised_maxvio=m, planner_us=18.5, planner_us_event_bracketed=19.9, dispatch_us=740.0,
                            combine_us=672.0, dc_gbs=5990.1, dc_frac_measured=0.9144, dc_frac_8tbs=0.7488)
             for m in (0.0, 0.5, 1.0, 2.0, 4.0)}
    legs = {"pages_maxvio_points": {"10": dict(planner_us_event_bracketed=19.8, dc_gbs=5950.0),
                                    "20": dict(planner_us_event_bracketed=19.7, dc_gbs=5960.0)},
            "prefetch_weight": {"points": {"1": dict(frac_measured=0.88), "4": dict(frac_measured=0.92)}},
            "reduce_grad": dict(frac_measured=0.905), "group_gemm": dict(tflops=1370.2),
            "rank_local": {"workload": "x" * 3000}}
    result = {"metric": bench.METRIC, "value": 5900.0, "unit": "GB/s", "n_gpus": 1, "steps": 20, "warmup": 5,
              "ms_per_step": 1.43, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
              "dtype": "bf16", "data": "synthetic",
              "config": {"workload": "train: " + bench.describe(bench.WORKLOADS["train"]), "maxvio": [0, 0.5, 1, 2, 4],
                         "parallelism": "EP=8 emulated on each GPU; independent EP groups per GPU",
                         "l2": "inputs larger than L2 (hidden rows 470 MB, dispatch buffer 4.7 GB per layer)",
                         "step": "plan + dispatch + combine of one layer; combine reads the dispatch buffer"},
              "planner_us": 18.5, "planner_us_event_bracketed": 19.9, "planner_us_back_to_back": 17.0,
              "dispatch_gbs": 5700.0, "combine_gbs": 6300.0, "dc_frac_measured_min": 0.91, "dc_frac_8tbs_min": 0.74,
              "spread_vs_maxvio": 0.004, "sweep": sweep, "legs": legs,
              "roofline": dict(bound="hbm", kernel="dispatch", achieved=5700.1, peak=6551.0, unit="GB/s", frac=0.87,
                               peak_kind="measured", frac_of_nominal_8tbs=0.71, traffic=4175256576,
                               bytes_per_launch=4231004160),
              "gpu_launches": 60, "clocks": {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 3},
              "e2e": {"value": 835.6, "unit": "GB/s", "h2d_bytes_per_step": 471867392,
                      "d2h_bytes_per_step": 469762048, "ms_per_step": 10.1, "steps": 20, "pipelined": "y" * 200},
              "cpu_baseline": {"value": 1.766, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": "s" * 80,
                               "host_cores_available": 16, "legs": {"x": 1}}}
    detail, line = bench.split_result(result)
    text = json.dumps(line)
    assert len(text) < 2600, len(text)
    assert "legs" not in line and "legs" in detail and "legs" not in line["cpu_baseline"]
    for k in ("planner_us", "planner_us_event_bracketed", "planner_us_event_bracketed_max", "spread_vs_maxvio",
              "roofline", "cpu_baseline", "e2e", "clocks", "gpu_launches", "pages_points", "prefetch_frac"):
        assert k in line, k
    assert set(line["sweep"]) == set(sweep) and line["sweep"]["4"]["frac"] == 0.9144
    assert line["planner_us_event_bracketed_max"] == 19.9


def test_ep_layout_splits_the_group_over_processes():
    import bench
    assert bench.ep_layout(8, 1, 0) == list(range(8))
    assert bench.ep_layout(8, 2, 1) == [4, 5, 6, 7]
    assert bench.ep_layout(8, 8, 3) == [3]
    owned = sorted(q for p in range(4) for q in bench.ep_layout(8, 4, p))
    assert owned == list(range(8))
    with pytest.raises(ValueError):
        bench.ep_layout(8, 3, 0)
    assert bench.ep_bytes(8, 4096, 8, 7168) == sum(bench.dc_bytes(8, 4096, 8, 7168))
