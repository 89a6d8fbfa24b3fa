"""One EP rank per process: R processes share the GPU, each owns its rank's
dispatch buffer, route-weight slots, home expert weights, prefetch pool, grad
rows and grad slots, and maps the other ranks' into itself with the library's
CUDA IPC calls (the exports are all-gathered over a gloo group).  Counts go
through the gloo all-gather, every rank plans its share, dispatches into its
peers' buffers, then (after a host barrier) combines from them, prefetches
its slots from the home ranks' weights and reduces its home experts' grads
from every rank's slots.  Every rank checks its own results against the
oracle's group computation: plan, dispatch buffer (padding included) and
prefetch bit for bit, combine within the bf16 tolerance (and >= 99.9 % bit
equal) with exact gathered weights, reduce_grad within fp32 1e-5 and the
consumed slots +0.0.  No kernel waits on another process: the ranks' phases
are ordered by host barriers."""
import os
import socket
import traceback

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

SENT = 0xFFFF

# (name, R, S, K, E, B, H, token_padding, mode, profile, maxvio, H')
CASES = [
    ("tiny", 2, 64, 2, 8, 4, 128, 8, 0, "boost0", 1.0, 16),
    ("bulk_rows", 4, 512, 4, 32, 8, 1024, 16, 0, "hot8", 2.0, 64),
    ("infer_overflow", 3, 300, 3, 24, 2, 264, 16, 1, "hot8", 3.0, 24),
    ("fewest_copies", 4, 512, 4, 32, 8, 1024, 16, 3, "hot8", 2.0, 64),
]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, case, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        q.put((rank, _run(rank, world, case)))
    except Exception:
        q.put((rank, {"error": traceback.format_exc()[-3000:]}))
    finally:
        try:
            dist.barrier()
            dist.destroy_process_group()
        except Exception:
            pass


def _run(rank, world, case):
    import torch.distributed as dist

    import oracle
    from load_balancing_planner_b200 import ep, moonep, synth
    from tests.conftest import bf16_to_f64, rel_close
    name, R, S, K, E, B, H, tp, mode, profile, mv, Hp = case
    assert R == world
    G = E // R
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    res = {}
    # every rank draws the whole group's inputs from the shared seed and keeps its own
    tk, _, _ = synth.routing(R, S, K, E, mv, profile, seed=31)
    tpe = synth.local_counts(tk, E)
    xall = synth.hidden_bf16(R, S, H, seed=31)
    wall = synth.route_weights(R, S, K, seed=31)
    Wall = [synth.hidden_bf16(1, E, H * Hp, seed=40 + p).view(E, H, Hp) for p in range(2)]
    Gall = [synth.normal_f32((E, H, Hp), 50 + p, scale=1e-3) for p in range(2)]
    RBall = [synth.normal_f32((R, B, H, Hp), 60 + p, scale=1e-3) for p in range(2)]

    nvs = ep.RankBuffer.nvs_of(S, K, E, R, tp)
    buf = torch.empty((nvs, H), dtype=torch.int16, device=dev).fill_(-1).view(torch.bfloat16)
    wbuf = torch.full((nvs,), float("nan"), dtype=torch.float32, device=dev)
    Wmine = [Wall[p][rank * G:(rank + 1) * G].contiguous().to(dev) for p in range(2)]
    pools = [torch.zeros((B, H, Hp), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    Gmine = [torch.from_numpy(Gall[p][rank * G:(rank + 1) * G].copy()).to(dev) for p in range(2)]
    RBmine = [torch.from_numpy(RBall[p][rank].copy()).to(dev) for p in range(2)]
    peers = ep.IpcPeers([buf, wbuf, *Wmine, *RBmine], group=None)

    counts = ep.gather_counts(torch.from_numpy(tpe[rank].copy()))   # over gloo, [R, E]
    res["gathered"] = bool(np.array_equal(counts.numpy(), tpe))
    rb = ep.RankBuffer(S, H, K, E, R, rank, hidden_nvs=peers.table(0), route_weights_nvs=peers.table(1),
                       token_padding=tp, B=B, mode=mode)
    plan = rb.plan(torch.from_numpy(np.ascontiguousarray(tk[rank])).to(dev), counts_all=counts.to(dev))
    torch.cuda.synchronize()
    o = oracle.plan(tk, E, B, tp, mode, tpe)
    assert o["status"] == 0
    res["plan_status"] = moonep.moonep_read_status(plan)
    ok = np.array_equal(plan.dst.cpu().numpy(), o["dst"][rank])
    for k in ("cu_seqlens", "row_counts", "counts", "assign"):
        ok = ok and np.array_equal(getattr(plan, k).cpu().numpy(), o[k])
    ok = ok and np.array_equal(plan.slots().cpu().numpy(), o["slot_expert"])
    res["plan"] = bool(ok)

    dist.barrier()                      # every buffer is sentinel-filled before anyone writes
    rb.dispatch(plan, xall[rank].contiguous().to(dev), torch.from_numpy(wall[rank].copy()).to(dev))
    torch.cuda.synchronize()
    dist.barrier()                      # every rank's rows have landed
    obuf, own = oracle.dispatch(o["dst"], synth.bf16_bits(xall), wall, o["nvs"], sentinel=SENT)
    mine = slice(rank * nvs, (rank + 1) * nvs)
    res["dispatch"] = bool(np.array_equal(buf.cpu().view(torch.int16).numpy().view(np.uint16), obuf[mine]))
    res["dispatch_w"] = bool(np.array_equal(wbuf.cpu().numpy().view(np.uint32), own[mine].view(np.uint32)))

    out, gw = rb.combine(plan)          # weighted, reading every rank's buffer
    torch.cuda.synchronize()
    oout, ogw = oracle.combine(o["dst"], obuf, own)
    g = out.cpu().view(torch.int16).numpy().view(np.uint16)
    res["combine_close"] = bool(rel_close(bf16_to_f64(g), bf16_to_f64(oout[rank]), 1e-2).all())
    res["combine_bits"] = float(np.mean(g == oout[rank]))
    res["combine_w"] = bool(np.array_equal(gw.cpu().numpy(), ogw[rank]))

    rb.prefetch_weight(plan, [peers.table(2), peers.table(3)], pools)
    torch.cuda.synchronize()
    ok = True
    for p in range(2):
        opool = np.zeros((R * B, H * Hp), np.uint16)
        oracle.prefetch(o["slot_expert"], synth.bf16_bits(Wall[p]).reshape(E, -1), opool)
        ok = ok and np.array_equal(pools[p].cpu().view(torch.int16).numpy().view(np.uint16).reshape(B, -1),
                                   opool[rank * B:(rank + 1) * B])
    res["prefetch"] = bool(ok)

    dist.barrier()                      # nobody reduces before every rank's slots are final
    rb.reduce_grad(plan, Gmine, [peers.table(4), peers.table(5)])
    torch.cuda.synchronize()
    dist.barrier()                      # every home rank has consumed its slots everywhere
    ok_g, ok_rb = True, True
    for p in range(2):
        oG, oRB = Gall[p].reshape(E, -1).copy(), RBall[p].reshape(R * B, -1).copy()
        oracle.reduce_grad(o["slot_expert"], oG, oRB)
        ok_g = ok_g and bool(rel_close(Gmine[p].cpu().numpy().reshape(G, -1), oG[rank * G:(rank + 1) * G], 1e-5).all())
        ok_rb = ok_rb and np.array_equal(RBmine[p].cpu().numpy().reshape(B, -1).view(np.uint32),
                                         oRB[rank * B:(rank + 1) * B].view(np.uint32))
    res["reduce_grad"] = ok_g
    res["reduce_slots"] = ok_rb
    res["used_slots"] = int((o["slot_expert"] >= 0).sum())
    res["remote_picks"] = int(sum(1 for d in o["dst"][rank].reshape(-1) if d // o["nvs"] != rank))
    dist.barrier()                      # no rank unmaps while another still reads
    peers.close()
    rb.destroy()
    return res


@pytest.mark.parametrize("case", [pytest.param(c, id=c[0]) for c in CASES])
def test_one_rank_per_process_matches_the_oracle(cuda, case):
    R = case[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, R, port, case, q)) for r in range(R)]
    for p in procs:
        p.start()
    try:
        got = dict(q.get(timeout=600) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=120)
            if p.is_alive():
                p.kill()
    for r in range(R):
        res = got[r]
        assert "error" not in res, f"rank {r}: {res.get('error')}"
        assert res["gathered"] and res["plan_status"] == 0 and res["plan"], (r, res)
        assert res["dispatch"] and res["dispatch_w"], (r, res)
        assert res["combine_close"] and res["combine_bits"] > 0.999 and res["combine_w"], (r, res)
        assert res["prefetch"], (r, res)
        assert res["reduce_grad"] and res["reduce_slots"], (r, res)
    assert any(got[r]["remote_picks"] for r in range(R)), "the case must send rows to other ranks"
    assert got[0]["used_slots"] > 0, "the case must use prefetch slots"
    for p in procs:
        assert p.exitcode == 0


@pytest.mark.parametrize("nproc", [2, 4])
def test_bench_sharded_ep_mode_on_one_gpu(cuda, nproc):
    # `bench.py --gpus N` in its sharded mode, with every process on this GPU
    # (--share-gpu, gloo): each process owns 8/N of the 8 EP ranks, maps the
    # others' buffers with CUDA IPC, and checks its plans against the group
    # planner and combine(dispatch(x)) = x before timing; one contract line
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", str(nproc),
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--gpus", str(nproc),
           "--share-gpu", "--config", "zipf", "--steps", "3", "--warmup", "3"]
    out = subprocess.run(cmd, cwd=root, capture_output=True, text=True, timeout=900)
    assert out.returncode == 0, (out.stdout[-2000:], out.stderr[-3000:])
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    d = json.loads(lines[0])
    assert d["n_gpus"] == nproc and d["scaling"] == "strong" and d["value"] > 0
    assert f"EP=8 sharded over {nproc} processes, {8 // nproc} ranks each" in d["config"]["parallelism"]
    assert d["remote_picks_per_process_max"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] > 0
