"""moonep_plan_noalloc: the planner for callers that cannot call cudaMalloc in
the layer path (their device memory belongs to a caching allocator or to a
reservation made at start-up).  It must give exactly the plan of the handle
path, call after call, while the shared scratch array keeps the previous
call's contents.  Collected last on purpose (its own file)."""
import numpy as np
import pytest
import torch

from tests.gpu_util import PLAN_KEYS, problem

pytestmark = pytest.mark.gpu


def _plan_arrays(p):
    out = {k: getattr(p, k).cpu().numpy() for k in PLAN_KEYS}
    out["slot_expert"] = out["slot_expert"][:, : p.B]
    out["maxvio"] = float(p.maxvio.cpu().numpy()[0])
    out["status"] = int(p.status.cpu().numpy()[0])
    return out


def _same(a, b):
    assert a["status"] == b["status"] == 0
    for k in PLAN_KEYS:
        assert np.array_equal(a[k], b[k]), k
    assert a["maxvio"] == b["maxvio"]


def test_noalloc_plan_equals_handle_plan_twice_in_a_row(cuda):
    from load_balancing_planner_b200 import moonep
    dev = torch.device("cuda:0")
    # two different shapes back to back: the training shape at maxvio 4, then
    # R=8, S=1024, K=8, E=64 at maxvio 2 (another grid size, so the shared
    # array's leftovers from the first call must not matter)
    cases = [(8, 4096, 8, 256, 32, 128, "hot8", 4.0), (8, 1024, 8, 64, 8, 128, "zipf", 2.0)]
    inputs, cfgs, plans = [], [], []
    for (R, S, K, E, B, tp, prof, mv) in cases:
        tk, tpe, _ = problem(R, S, K, E, mv, prof, seed=7)
        inputs.append((torch.from_numpy(tk).to(dev), torch.from_numpy(tpe).to(dev)))
        cfg = moonep.Config(S, 8, K, E, R, B, tp, 0, 0)
        cfgs.append(cfg)
        plans.append(moonep.Plan(cfg, dev))
    torch.cuda.synchronize()
    free_before = None
    for i, ((t, c), cfg, p) in enumerate(zip(inputs, cfgs, plans)):
        if i == 1:
            torch.cuda.synchronize()
            free_before = torch.cuda.mem_get_info(dev)[0]
        moonep.moonep_plan_noalloc(cfg, t, c, p)
        torch.cuda.synchronize()
        if i == 1:
            assert torch.cuda.mem_get_info(dev)[0] == free_before, "the call allocated device memory"
    for (t, c), cfg, p in zip(inputs, cfgs, plans):
        h = moonep.moonep_create(cfg.S, cfg.H, cfg.K, cfg.E, cfg.R, cfg.B, cfg.token_padding)
        ref = moonep.moonep_plan(h, t, c)
        torch.cuda.synchronize()
        _same(_plan_arrays(p), _plan_arrays(ref))
        h.close()


def test_noalloc_rejects_a_workspace_past_its_array(cuda):
    from load_balancing_planner_b200 import moonep
    # R=16, S=2048, E=4096: chunk histograms + count tables exceed 1 MiB
    cfg = moonep.Config(2048, 8, 8, 4096, 16, 256, 128, 0, 0)
    p = moonep.Plan(cfg, torch.device("cuda:0"))
    tk = torch.zeros((16, 2048, 8), dtype=torch.int32, device="cuda")
    with pytest.raises(moonep.MoonepError) as e:
        moonep.moonep_plan_noalloc(cfg, tk, None, p)
    assert e.value.code == moonep.ERR_SIZE
