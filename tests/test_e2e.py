"""One MoE layer end to end through the C ABI -- plan, dispatch, an expert,
combine -- against the same pipeline on the oracle, at R=8, S=1024, K=8,
E=64, H=2048 for every maxvio of the sweep.  The expert is diagonal: row r of
the buffer is scaled by a_e of the expert whose weights serve that row (a
signed power of two, so its bf16 output is exact on both sides)."""
import numpy as np
import pytest
import torch

import oracle
from load_balancing_planner_b200 import synth
from tests.conftest import bf16_to_f64, rel_close
from tests.gpu_util import bits, gpu_plan, plan_to_numpy, problem, assert_plans_equal

pytestmark = pytest.mark.gpu


def _row_expert(cu, rc, se, E, B, R, nvs):
    """Expert served by each buffer row (-1 = padding), from a plan."""
    ex = np.full(R * nvs, -1, np.int64)
    for r in range(R):
        prev = 0
        for i in range(E + B):
            n = rc[r, i]
            if n:
                ex[r * nvs + prev: r * nvs + prev + n] = i if i < E else se[r, i - E]
            prev = cu[r, i]
    return ex


@pytest.mark.parametrize("mv", [0.0, 0.5, 1.0, 2.0])
def test_layer_round_trip_matches_oracle(cuda, mv):
    from load_balancing_planner_b200 import moonep
    R, S, K, E, B, H, tp = 8, 1024, 8, 64, 8, 2048, 128
    tk, tpe, real = problem(R, S, K, E, mv, "zipf", seed=13)
    x = synth.hidden_bf16(R, S, H, seed=13)
    w = synth.route_weights(R, S, K, seed=13)
    a = np.random.default_rng(13).choice([0.5, -0.5, 1.0, -1.0, 2.0, -2.0, 4.0], size=E)

    # CUDA path
    h = moonep.moonep_create(S, H, K, E, R, B, tp)
    p = gpu_plan(h, tk, tpe)
    buf, wn = moonep.moonep_dispatch(h, p, x.cuda(), torch.from_numpy(w).cuda())
    got_plan = plan_to_numpy(p)
    rows_e = torch.from_numpy(_row_expert(got_plan["cu_seqlens"], got_plan["row_counts"],
                                          got_plan["slot_expert"], E, B, R, h.nvs)).cuda()
    scale = torch.where(rows_e >= 0, torch.from_numpy(a).cuda()[rows_e.clamp(min=0)], torch.zeros_like(rows_e, dtype=torch.float64))
    y = (buf.view(R * h.nvs, H).double() * scale[:, None]).to(torch.bfloat16).view(R, h.nvs, H)
    out, gw = moonep.moonep_combine(h, p, y, wn)
    torch.cuda.synchronize()
    assert moonep.moonep_read_status(p) == 0

    # oracle pipeline
    o = oracle.plan(tk, E, B, tp, 0, tpe)
    assert_plans_equal(got_plan, o)
    obuf, own = oracle.dispatch(o["dst"], synth.bf16_bits(x), w, o["nvs"], sentinel=0)
    oe = _row_expert(o["cu_seqlens"], o["row_counts"], o["slot_expert"], E, B, R, o["nvs"])
    oy = bf16_to_f64(obuf) * np.where(oe >= 0, a[np.clip(oe, 0, None)], 0.0)[:, None]
    oybits = synth.bf16_bits(torch.from_numpy(oy.astype(np.float32)).to(torch.bfloat16))
    oout, ogw = oracle.combine(o["dst"], oybits, own)

    assert rel_close(bf16_to_f64(bits(out)), bf16_to_f64(oout), 1e-2).all()
    assert np.array_equal(gw.cpu().numpy(), ogw)
    h.close()
