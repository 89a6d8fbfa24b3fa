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


@pytest.mark.parametrize("mode", [1, 2])
def test_noalloc_inference_modes_without_router_counts(cuda, mode):
    # the inference shape (R=8, S=4096, K=8, E=256, B=4) at maxvio 4, where
    # copies past the B slots overflow to their home rows, with no
    # tokens_per_expert given: the same plan as the handle path, twice
    from load_balancing_planner_b200 import moonep
    dev = torch.device("cuda:0")
    R, S, K, E, B, tp = 8, 4096, 8, 256, 4, 128
    tk, _, _ = problem(R, S, K, E, 4.0, "hot8", seed=11)
    t = torch.from_numpy(tk).to(dev)
    cfg = moonep.Config(S, 8, K, E, R, B, tp, 0, mode)
    h = moonep.moonep_create(S, 8, K, E, R, B, tp, mode=mode)
    ref = _plan_arrays(moonep.moonep_plan(h, t, None))
    home = np.arange(E) // (E // R)
    assert any(ref["row_counts"][r, e] > 0 for r in range(R) for e in range(E) if home[e] != r)
    for _ in range(2):
        p = moonep.moonep_plan_noalloc(cfg, t, None, moonep.Plan(cfg, dev))
        torch.cuda.synchronize()
        _same(_plan_arrays(p), ref)
    h.close()


def test_noalloc_error_then_clean_call(cuda):
    # a call that fails on the device (an expert id past E) leaves its counts
    # in the shared array; the next clean call must not see them
    from load_balancing_planner_b200 import moonep
    dev = torch.device("cuda:0")
    R, S, K, E, B, tp = 8, 1024, 8, 64, 8, 128
    tk, tpe, _ = problem(R, S, K, E, 2.0, "zipf", seed=13)
    bad = tk.copy()
    bad[5, 100, 3] = E + 1
    cfg = moonep.Config(S, 8, K, E, R, B, tp, 0, 0)
    pb = moonep.moonep_plan_noalloc(cfg, torch.from_numpy(bad).to(dev), torch.from_numpy(tpe).to(dev),
                                    moonep.Plan(cfg, dev))
    assert moonep.moonep_read_status(pb) & moonep.STATUS_BAD_EXPERT
    t, c = torch.from_numpy(tk).to(dev), torch.from_numpy(tpe).to(dev)
    p = moonep.moonep_plan_noalloc(cfg, t, c, moonep.Plan(cfg, dev))
    torch.cuda.synchronize()
    h = moonep.moonep_create(S, 8, K, E, R, B, tp)
    _same(_plan_arrays(p), _plan_arrays(moonep.moonep_plan(h, t, c)))
    h.close()
