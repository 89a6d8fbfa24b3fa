"""The hot path captured in a CUDA graph and replayed on new routings: the
group step (plan -> dispatch -> combine) and the per-rank step of all ranks.
Replays must give exactly what eager calls give on the same inputs (the
planner's grid barrier and parity slots carry over from launch to launch)."""
import numpy as np
import pytest
import torch

from load_balancing_planner_b200 import synth
from tests.gpu_util import problem

pytestmark = pytest.mark.gpu

R, S, K, E, B, H, TP = 8, 1024, 8, 64, 8, 2048, 128


def _routings():
    return [problem(R, S, K, E, mv, "hot8", seed=31 + i)[:2] for i, mv in enumerate((0.0, 2.0, 4.0, 1.0))]


def test_group_step_graph_replays_match_eager(cuda):
    from load_balancing_planner_b200 import moonep
    h = moonep.moonep_create(S, H, K, E, R, B, TP)
    dev = torch.device("cuda:0")
    hidden = synth.hidden_bf16(R, S, H, seed=31).to(dev)
    w = torch.from_numpy(synth.route_weights(R, S, K, seed=31)).to(dev)
    topk = torch.empty((R, S, K), dtype=torch.int32, device=dev)
    tpe = torch.empty((R, E), dtype=torch.int32, device=dev)
    plan = moonep.Plan(h, dev)
    buf = torch.empty((R, h.nvs, H), dtype=torch.bfloat16, device=dev)
    wn = torch.empty((R, h.nvs), dtype=torch.float32, device=dev)
    out = torch.empty((R, S, H), dtype=torch.bfloat16, device=dev)
    gw = torch.empty((R, S, K), dtype=torch.float32, device=dev)
    routes = _routings()

    def step():
        moonep.moonep_plan(h, topk, tpe, plan)
        moonep.moonep_dispatch(h, plan, hidden, w, buf, wn)
        moonep.moonep_combine(h, plan, buf, wn, out, gw)

    topk.copy_(torch.from_numpy(routes[0][0]))
    tpe.copy_(torch.from_numpy(routes[0][1]))
    step()  # eager warm-up
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for tk, c in routes:
        topk.copy_(torch.from_numpy(tk))
        tpe.copy_(torch.from_numpy(c))
        g.replay()
        torch.cuda.synchronize()
        assert moonep.moonep_read_status(plan) == 0
        got = (plan.dst.clone(), plan.cu_seqlens.clone(), out.clone(), gw.clone())
        p2 = moonep.moonep_plan(h, torch.from_numpy(tk).to(dev), torch.from_numpy(c).to(dev))
        b2, w2 = moonep.moonep_dispatch(h, p2, hidden, w)
        o2, g2 = moonep.moonep_combine(h, p2, b2, w2)
        torch.cuda.synchronize()
        for x, y in zip(got, (p2.dst, p2.cu_seqlens, o2, g2)):
            assert torch.equal(x, y)
    del g
    h.close()


def test_rank_step_graph_replays_match_eager(cuda):
    from load_balancing_planner_b200 import moonep
    h = moonep.moonep_create(S, H, K, E, R, B, TP)
    dev = torch.device("cuda:0")
    hidden = synth.hidden_bf16(R, S, H, seed=32).to(dev)
    w = torch.from_numpy(synth.route_weights(R, S, K, seed=32)).to(dev)
    topk = [torch.empty((S, K), dtype=torch.int32, device=dev) for _ in range(R)]
    counts = torch.empty((R, E), dtype=torch.int32, device=dev)
    plans = [moonep.Plan(h, dev, rank=r) for r in range(R)]
    bufs = [torch.empty((h.nvs, H), dtype=torch.bfloat16, device=dev) for _ in range(R)]
    wbufs = [torch.empty((h.nvs,), dtype=torch.float32, device=dev) for _ in range(R)]
    out = torch.empty((R, S, H), dtype=torch.bfloat16, device=dev)
    gw = torch.empty((R, S, K), dtype=torch.float32, device=dev)
    routes = _routings()

    def load(tk, c):
        for r in range(R):
            topk[r].copy_(torch.from_numpy(np.ascontiguousarray(tk[r])))
        counts.copy_(torch.from_numpy(c))

    def step():
        for r in range(R):
            moonep.moonep_plan_rank(h, r, topk[r], counts, plans[r])
        for r in range(R):
            moonep.moonep_dispatch_rank(h, plans[r], hidden[r], w[r], bufs, wbufs)
        for r in range(R):
            moonep.moonep_combine_rank(h, plans[r], bufs, wbufs, out[r], gw[r])

    load(*routes[0])
    step()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for tk, c in routes:
        load(tk, c)
        g.replay()
        torch.cuda.synchronize()
        assert all(moonep.moonep_read_status(p) == 0 for p in plans)
        got = ([p.dst.clone() for p in plans], out.clone(), gw.clone())
        step()  # eager, same inputs
        torch.cuda.synchronize()
        assert all(torch.equal(a, p.dst) for a, p in zip(got[0], plans))
        assert torch.equal(got[1], out) and torch.equal(got[2], gw)
    del g
    h.close()
