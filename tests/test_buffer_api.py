"""The Buffer API (MoonEP README, "API guide" and "zero_copy"): defaults,
zero_copy views, async_finish events on the communication stream, the
status check, and that it gives the same results as the C-ABI calls."""
import numpy as np
import pytest
import torch

from load_balancing_planner_b200 import synth
from tests.gpu_util import problem

pytestmark = pytest.mark.gpu

R, S, K, E, H, TP = 8, 1024, 8, 64, 256, 128


def _inputs(mv=1.0, seed=31):
    dev = torch.device("cuda:0")
    tk, tpe, _ = problem(R, S, K, E, mv, "zipf", seed=seed)
    x = synth.hidden_bf16(R, S, H, seed=seed).to(dev)
    w = torch.from_numpy(synth.route_weights(R, S, K, seed=seed)).to(dev)
    return torch.from_numpy(tk).to(dev), torch.from_numpy(tpe).to(dev), x, w


def test_defaults_and_same_results_as_the_c_abi(cuda):
    from load_balancing_planner_b200 import moonep
    from load_balancing_planner_b200.buffer import Buffer
    topk, tpe, x, w = _inputs()
    buf = Buffer(S=S, H=H, K=K, E=E, num_ep_ranks=R, token_padding=TP)
    assert buf.B == E // R and buf.nvs == moonep.moonep_nvs(buf.handle)
    hn, wn, cu, plan = buf.dispatch(x, w, topk, tpe)
    out, gw, _ = buf.combine(plan, hn, wn)

    h = moonep.moonep_create(S, H, K, E, R, E // R, TP)
    p2 = moonep.moonep_plan(h, topk, tpe)
    hn2, wn2 = moonep.moonep_dispatch(h, p2, x, w)
    out2, gw2 = moonep.moonep_combine(h, p2, hn2, wn2)
    torch.cuda.synchronize()
    assert torch.equal(cu, p2.cu_seqlens) and torch.equal(plan.dst, p2.dst)
    real = plan.dst.view(-1).long()
    assert torch.equal(hn.view(-1, H)[real], hn2.view(-1, H)[real])
    assert torch.equal(wn.view(-1)[real], wn2.view(-1)[real])
    assert torch.equal(out, out2) and torch.equal(gw, gw2) and torch.equal(gw, w)
    h.close()
    buf.destroy()
    with pytest.raises(RuntimeError):
        buf.dispatch(x, w, topk, tpe)


def test_zero_copy_returns_views_of_one_static_buffer(cuda):
    from load_balancing_planner_b200.buffer import Buffer
    topk, tpe, x, w = _inputs()
    buf = Buffer(S, H, K, E, R, token_padding=TP)
    hn, wn, _, plan = buf.dispatch(x, w, topk, tpe, zero_copy=True)
    hn_b, wn_b, _, _ = buf.dispatch(x, w, plan=plan, zero_copy=True)
    assert hn.data_ptr() == hn_b.data_ptr() and wn.data_ptr() == wn_b.data_ptr()
    hn_c, _, _, _ = buf.dispatch(x, w, plan=plan)  # a fresh tensor
    assert hn_c.data_ptr() != hn.data_ptr()
    out, gw, _ = buf.combine(plan, hn, wn, zero_copy=True)
    out_c, _, _ = buf.combine(plan, hn_c, wn)
    torch.cuda.synchronize()
    assert torch.equal(out, out_c)
    with pytest.raises(ValueError):
        buf.combine(plan, hn_c, wn, zero_copy=True)
    buf.destroy()


def test_async_finish_runs_on_the_comm_stream_and_returns_an_event(cuda):
    from load_balancing_planner_b200.buffer import Buffer
    topk, tpe, x, w = _inputs(mv=2.0, seed=32)
    buf = Buffer(S, H, K, E, R, token_padding=TP)
    hn, wn, cu, plan, ev = buf.dispatch(x, w, topk, tpe, async_finish=True)
    assert isinstance(ev, torch.cuda.Event)
    torch.cuda.current_stream().wait_event(ev)
    out, gw, _, ev2 = buf.combine(plan, hn, wn, async_finish=True)
    torch.cuda.current_stream().wait_event(ev2)
    hn_s, wn_s, _, plan_s = buf.dispatch(x, w, topk, tpe)
    out_s, _, _ = buf.combine(plan_s, hn_s, wn_s)
    Wt = torch.randn(E, H, 32, device="cuda").to(torch.bfloat16)
    pool = torch.zeros(R, buf.B, H, 32, dtype=torch.bfloat16, device="cuda")
    ev3 = buf.prefetch_weight(plan, [Wt], [pool], async_finish=True)
    torch.cuda.current_stream().wait_event(ev3)
    G = torch.zeros(E, H, 32, device="cuda")
    RB = torch.ones(R, buf.B, H, 32, device="cuda")
    ev4 = buf.reduce_grad(plan, [G], [RB], async_finish=True)
    torch.cuda.current_stream().wait_event(ev4)
    torch.cuda.synchronize()
    assert torch.equal(out, out_s) and torch.equal(plan.dst, plan_s.dst)
    se = plan.slots().cpu().numpy()
    for r in range(R):
        for b in range(buf.B):
            if se[r, b] >= 0:
                assert torch.equal(pool[r, b], Wt[se[r, b]])
    copies = np.bincount(se[se >= 0], minlength=E)
    assert torch.equal(G[:, 0, 0].cpu(), torch.from_numpy(copies.astype(np.float32)))
    buf.destroy()


def test_check_raises_on_bad_routing(cuda):
    from load_balancing_planner_b200 import moonep
    from load_balancing_planner_b200.buffer import Buffer, PlanStatusError
    topk, tpe, x, w = _inputs()
    buf = Buffer(S, H, K, E, R, token_padding=TP)
    bad = topk.clone()
    bad[3, 5, 0] = E  # an expert id outside [0, E)
    _, _, _, plan = buf.dispatch(x, w, bad)
    with pytest.raises(PlanStatusError) as e:
        buf.check(plan)
    assert e.value.status & moonep.STATUS_BAD_EXPERT
    _, _, _, plan = buf.dispatch(x, w, topk, tpe + 1)  # counts that disagree with top-k
    with pytest.raises(PlanStatusError) as e:
        buf.check(plan)
    assert e.value.status == moonep.STATUS_COUNT_MISMATCH
    buf.destroy()
