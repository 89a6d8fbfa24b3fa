"""Device-side errors become status bits, later calls on that plan do
nothing, and the handle keeps working.  Every failure is made on the host
(corrupted inputs or plan arrays); every index the kernels read from a plan is
bounds-checked, so none of these cases can fault the GPU."""
import numpy as np
import pytest
import torch

import oracle
from load_balancing_planner_b200 import synth
from tests.gpu_util import assert_plans_equal, gpu_plan, plan_to_numpy, problem

pytestmark = pytest.mark.gpu

R, S, K, E, B, H, TP = 4, 256, 4, 32, 8, 64, 8


def _setup():
    from load_balancing_planner_b200 import moonep
    tk, tpe, _ = problem(R, S, K, E, 2.0, "hot8", seed=1)
    return moonep, moonep.moonep_create(S, H, K, E, R, B, TP), tk, tpe


@pytest.mark.parametrize("kind,bit", [("bad_id", 1), ("neg_id", 1), ("dup", 2), ("count", 4)])
def test_bad_router_output_sets_status_and_blocks_later_calls(cuda, kind, bit):
    moonep, h, tk, tpe = _setup()
    bad, btpe = tk.copy(), tpe.copy()
    if kind == "bad_id":
        bad[2, 17, 1] = E
    elif kind == "neg_id":
        bad[0, 3, 0] = -1
    elif kind == "dup":
        bad[1, 5, 2] = bad[1, 5, 0]
    else:
        btpe[3, 7] += 1
    # without local counts each fault shows alone; with them a changed pick
    # also breaks the count check, and both sides report the same bits
    p = gpu_plan(h, bad, btpe if kind == "count" else None)
    st = moonep.moonep_read_status(p)
    assert st == bit
    p2 = gpu_plan(h, bad, btpe)
    st2 = moonep.moonep_read_status(p2)
    assert st2 == oracle.plan(bad, E, B, TP, 0, btpe)["status"]
    assert st2 & bit
    # dispatch / combine / prefetch / reduce_grad do nothing on a failed plan
    x = synth.hidden_bf16(R, S, H, seed=1).cuda()
    buf = torch.empty((R, h.nvs, H), dtype=torch.int16, device="cuda").fill_(-1).view(torch.bfloat16)
    moonep.moonep_dispatch(h, p, x, None, buf)
    out = torch.empty((R, S, H), dtype=torch.int16, device="cuda").fill_(7).view(torch.bfloat16)
    moonep.moonep_combine(h, p, buf, None, out)
    W = torch.ones((E, H, 8), dtype=torch.bfloat16, device="cuda")
    pool = torch.zeros((R, B, H, 8), dtype=torch.bfloat16, device="cuda")
    moonep.moonep_prefetch_weight(h, p, [W], [pool])
    G = torch.ones((E, H, 8), device="cuda")
    RBf = torch.ones((R, B, H, 8), device="cuda")
    moonep.moonep_reduce_grad(h, p, [G], [RBf])
    torch.cuda.synchronize()
    assert bool((buf.view(torch.int16) == -1).all())
    assert bool((out.view(torch.int16) == 7).all())
    assert bool((pool == 0).all()) and bool((G == 1).all()) and bool((RBf == 1).all())
    # the handle recovers: the next valid plan is exact
    good = plan_to_numpy(gpu_plan(h, tk, tpe))
    assert_plans_equal(good, oracle.plan(tk, E, B, TP, 0, tpe))
    h.close()


def test_out_of_range_slot_in_plan_is_skipped(cuda):
    moonep, h, tk, tpe = _setup()
    p = gpu_plan(h, tk, tpe)
    p.dst[1, 2, 3] = R * h.nvs + 5      # past the buffer
    p.dst[0, 0, 0] = -3
    x = synth.hidden_bf16(R, S, H, seed=1).cuda()
    buf = torch.zeros((R, h.nvs, H), dtype=torch.bfloat16, device="cuda")
    moonep.moonep_dispatch(h, p, x, None, buf)
    torch.cuda.synchronize()
    assert moonep.moonep_read_status(p) == moonep.STATUS_BAD_PLAN
    h.close()


def test_out_of_range_dst_in_combine_is_skipped(cuda):
    moonep, h, tk, tpe = _setup()
    p = gpu_plan(h, tk, tpe)
    p.dst[3, 1, 1] = 1 << 30
    y = torch.zeros((R, h.nvs, H), dtype=torch.bfloat16, device="cuda")
    moonep.moonep_combine(h, p, y, None)
    torch.cuda.synchronize()
    assert moonep.moonep_read_status(p) == moonep.STATUS_BAD_PLAN
    h.close()


@pytest.mark.parametrize("corrupt", ["past_E", "unsorted"])
def test_malformed_slot_table_is_rejected(cuda, corrupt):
    moonep, h, tk, tpe = _setup()
    p = gpu_plan(h, tk, tpe)
    se = p.slot_expert
    if corrupt == "past_E":
        se[2, 0] = E + 3
    else:
        se[1, 0], se[1, 1] = 5, 3
    W = torch.ones((E, H, 8), dtype=torch.bfloat16, device="cuda")
    pool = torch.zeros((R, B, H, 8), dtype=torch.bfloat16, device="cuda")
    moonep.moonep_prefetch_weight(h, p, [W], [pool])
    torch.cuda.synchronize()
    assert moonep.moonep_read_status(p) == moonep.STATUS_BAD_PLAN
    assert bool((pool == 0).all())
    h.close()


def test_host_side_errors(cuda):
    moonep, h, tk, tpe = _setup()
    p = gpu_plan(h, tk, tpe)
    x = synth.hidden_bf16(R, S, H, seed=1).cuda()
    raw = torch.empty(R * h.nvs * H + 8, dtype=torch.bfloat16, device="cuda")
    mis = raw[1:1 + R * h.nvs * H].view(R, h.nvs, H)       # 2-byte offset: not 16-byte aligned
    with pytest.raises(moonep.MoonepError) as e:
        moonep.moonep_dispatch(h, p, x, None, mis)
    assert e.value.code == moonep.ERR_ALIGN
    W = torch.ones((E, H, 8), dtype=torch.bfloat16, device="cuda")
    pool = torch.zeros((R, B, H, 8), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moonep.MoonepError) as e:
        moonep.moonep_prefetch_weight(h, p, [W] * 9, [pool] * 9)
    assert e.value.code == moonep.ERR_SIZE
    h.close()


def test_planner_barrier_timeout_is_reported_and_the_handle_recovers(cuda):
    # A bounded wait made to run out from the host: the hook makes the
    # planner's grid barrier wait for one block arrival that never comes and
    # give up after a few thousand polls.  Every block returns with
    # MOONEP_STATUS_TIMEOUT within milliseconds, and the tables the next call
    # uses are left clean, so the same handle plans bit-exactly afterwards
    # (the timed-out call is not the handle's first, so its count tables were
    # in use).  A fresh handle plans bit-exactly too.
    import time

    from load_balancing_planner_b200 import moonep
    Rz, Sz, Kz, Ez, Bz, tp = 8, 1024, 8, 64, 8, 128
    tk, tpe, _ = problem(Rz, Sz, Kz, Ez, 2.0, "zipf", seed=3)
    tk2, tpe2, _ = problem(Rz, Sz, Kz, Ez, 0.5, "zipf", seed=4)
    h = moonep.moonep_create(Sz, 8, Kz, Ez, Rz, Bz, tp)
    warm = plan_to_numpy(gpu_plan(h, tk2, tpe2))
    assert_plans_equal(warm, oracle.plan(tk2, Ez, Bz, tp, 0, tpe2))

    moonep.moonep_set_plan_barrier(h, 4096, 1)
    p = moonep.Plan(h)
    p.dst.fill_(-7)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    moonep.moonep_plan(h, torch.from_numpy(tk).cuda(), torch.from_numpy(tpe).cuda(), p)
    st = moonep.moonep_read_status(p)
    dt = time.perf_counter() - t0
    assert st == moonep.STATUS_TIMEOUT
    assert dt < 1.0, dt
    assert bool((p.dst == -7).all())  # nothing past the barrier was written
    assert moonep.moonep_plan_status(p) == moonep.STATUS_TIMEOUT
    # later calls on the timed-out plan do nothing
    x = synth.hidden_bf16(Rz, Sz, 8, seed=1).cuda()
    buf = torch.empty((Rz, h.nvs, 8), dtype=torch.int16, device="cuda").fill_(-1).view(torch.bfloat16)
    moonep.moonep_dispatch(h, p, x, None, buf)
    torch.cuda.synchronize()
    assert bool((buf.view(torch.int16) == -1).all())

    moonep.moonep_set_plan_barrier(h, 0, 0)
    want = oracle.plan(tk, Ez, Bz, tp, 0, tpe)
    for _ in range(2):  # both parities of the handle's tables
        assert_plans_equal(plan_to_numpy(gpu_plan(h, tk, tpe)), want)

    # the one-rank planner of the same handle: its own barrier, same hook
    c = torch.from_numpy(tpe).cuda()
    moonep.moonep_set_plan_barrier(h, 4096, 2)
    pr = moonep.moonep_plan_rank(h, 3, torch.from_numpy(np.ascontiguousarray(tk[3])).cuda(), c)
    assert moonep.moonep_read_status(pr) == moonep.STATUS_TIMEOUT
    moonep.moonep_set_plan_barrier(h, 0, 0)
    wr = oracle.plan_rank(tk[3], tpe, 3, Ez, Bz, tp, 0)
    for _ in range(2):
        pr = moonep.moonep_plan_rank(h, 3, torch.from_numpy(np.ascontiguousarray(tk[3])).cuda(), c)
        assert moonep.moonep_read_status(pr) == 0
        assert np.array_equal(pr.dst.cpu().numpy(), wr["dst"])
        assert np.array_equal(pr.cu_seqlens.cpu().numpy(), wr["cu_seqlens"])
    h.close()

    fresh = moonep.moonep_create(Sz, 8, Kz, Ez, Rz, Bz, tp)
    assert_plans_equal(plan_to_numpy(gpu_plan(fresh, tk, tpe)), want)
    with pytest.raises(moonep.MoonepError) as e:
        moonep.moonep_set_plan_barrier(fresh, 0, -1)
    assert e.value.code == moonep.ERR_SIZE
    fresh.close()
