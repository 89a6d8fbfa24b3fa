"""GPU reduce_grad against the oracle: grads within fp32 rel 1e-5 (as
|a-b| <= 1e-5 (|b| + rms b)), consumed slots exactly +0.0, unused slots
untouched; the full backward shape (E=256, R=8, B=32, H=7168, H'=2048) checked
on sampled experts and element ranges."""
import numpy as np
import pytest
import torch

import oracle
from load_balancing_planner_b200 import synth
from tests.conftest import rel_close
from tests.gpu_util import gpu_plan, problem

pytestmark = pytest.mark.gpu
RTOL_F32 = 1e-5


@pytest.mark.parametrize("R,S,K,E,B,tp,mode,mv,H,Hp,n_proj", [
    (4, 96, 4, 16, 4, 8, 0, 3.0, 16, 48, 2),
    (8, 1024, 8, 64, 8, 128, 0, 2.0, 64, 64, 1),
    (8, 1024, 8, 64, 3, 128, 1, 2.0, 8, 36, 3),
    (3, 1000, 3, 24, 8, 16, 0, 1.5, 24, 20, 1),
    # 16 KB pieces through the bulk path, the last one short
    (8, 1024, 8, 64, 8, 128, 0, 2.0, 72, 100, 2),
    (8, 1024, 8, 64, 3, 128, 1, 4.0, 128, 64, 3),
])
def test_reduce_grad_matches_oracle(cuda, R, S, K, E, B, tp, mode, mv, H, Hp, n_proj):
    from load_balancing_planner_b200 import moonep
    tk, tpe, _ = problem(R, S, K, E, mv, "hot8", seed=8)
    h = moonep.moonep_create(S, H, K, E, R, B, tp, mode=mode)
    p = gpu_plan(h, tk, tpe)
    o = oracle.plan(tk, E, B, tp, mode, tpe)
    Gs = [synth.normal_f32((E, H, Hp), 30 + i, scale=1e-3) for i in range(n_proj)]
    RBs = [synth.normal_f32((R, B, H, Hp), 40 + i, scale=1e-3) for i in range(n_proj)]
    gG = [torch.from_numpy(g).cuda() for g in Gs]
    gRB = [torch.from_numpy(r).cuda() for r in RBs]
    moonep.moonep_reduce_grad(h, p, gG, gRB)
    torch.cuda.synchronize()
    assert moonep.moonep_read_status(p) == 0
    se = o["slot_expert"].reshape(-1)
    for G, RB, g, rb in zip(Gs, RBs, gG, gRB):
        oG, oRB = G.reshape(E, -1).copy(), RB.reshape(R * B, -1).copy()
        oracle.reduce_grad(o["slot_expert"], oG, oRB)
        got = g.cpu().numpy().reshape(E, -1)
        assert rel_close(got, oG, RTOL_F32).all()
        touched = np.unique(se[se >= 0])
        untouched = np.setdiff1d(np.arange(E), touched)
        assert np.array_equal(got[untouched].view(np.uint32), G.reshape(E, -1)[untouched].view(np.uint32))
        grb = rb.cpu().numpy().reshape(R * B, -1)
        for s in range(R * B):
            if se[s] >= 0:
                assert np.all(grb[s].view(np.uint32) == 0), "consumed slots are +0.0"
            else:
                assert np.array_equal(grb[s].view(np.uint32), RB.reshape(R * B, -1)[s].view(np.uint32))
    h.close()


def test_reduce_grad_backward_shape_sampled(cuda):
    from load_balancing_planner_b200 import moonep
    R, S, K, E, B, H, Hp, tp = 8, 4096, 8, 256, 32, 7168, 2048, 128
    tk, tpe, _ = problem(R, S, K, E, 2.0, "hot8", seed=0)
    h = moonep.moonep_create(S, H, K, E, R, B, tp)
    p = gpu_plan(h, tk, tpe)
    o = oracle.plan(tk, E, B, tp, 0, tpe)
    se = o["slot_expert"].reshape(-1)
    assert np.array_equal(p.slots().cpu().numpy().reshape(-1), se)
    gen = torch.Generator(device="cuda").manual_seed(1)
    G = torch.randn((E, H * Hp), generator=gen, device="cuda") * 1e-3
    RB = torch.randn((R * B, H * Hp), generator=gen, device="cuda") * 1e-3
    # samples: a few element ranges of every expert and every slot, taken before
    n = H * Hp
    starts = [0, n // 3 + 5, n - 4096]
    G0 = [G[:, s:s + 4096].cpu().numpy() for s in starts]
    RB0 = [RB[:, s:s + 4096].cpu().numpy() for s in starts]
    unused = [s for s in range(R * B) if se[s] < 0]
    assert unused
    # unused slots: sampled ranges bitwise, and the sum of every slot's 32-bit
    # patterns (as integers) over the whole slot
    bitsum_before = RB[unused].view(torch.int32).long().sum(dim=1).cpu()
    moonep.moonep_reduce_grad(h, p, [G.view(E, H, Hp)], [RB.view(R, B, H, Hp)])
    torch.cuda.synchronize()
    assert moonep.moonep_read_status(p) == 0
    touched = np.unique(se[se >= 0])
    untouched_e = np.setdiff1d(np.arange(E), touched)
    for s0, g0, rb0 in zip(starts, G0, RB0):
        og, orb = g0.copy(), rb0.copy()
        oracle.reduce_grad(o["slot_expert"], og, orb)
        got = G[:, s0:s0 + 4096].cpu().numpy()
        assert rel_close(got, og, RTOL_F32).all()
        assert np.array_equal(got[untouched_e].view(np.uint32), g0[untouched_e].view(np.uint32))
        # the oracle's slots after its reduction: consumed +0.0, unused as before
        grb = RB[:, s0:s0 + 4096].cpu().numpy()
        assert np.array_equal(grb.view(np.uint32), orb.view(np.uint32))
    used = [s for s in range(R * B) if se[s] >= 0]
    assert used
    assert bool((RB[used].view(torch.int32) == 0).all())
    assert torch.equal(RB[unused].view(torch.int32).long().sum(dim=1).cpu(), bitsum_before)
    h.close()
