"""GPU weight prefetch == oracle (bit copy into every used slot, unused slots
untouched), for several projections at once; the inference shape with its
overflow rows at full size."""
import numpy as np
import pytest
import torch

import oracle
from load_balancing_planner_b200 import synth
from tests.gpu_util import bits, gpu_plan, problem

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("R,S,K,E,B,tp,mode,mv,Hp,n_proj", [
    (4, 96, 4, 16, 4, 8, 0, 3.0, 48, 3),
    (8, 1024, 8, 64, 8, 128, 0, 2.0, 64, 1),
    (8, 1024, 8, 64, 2, 128, 1, 2.0, 40, 2),
    (4, 333, 3, 24, 6, 16, 0, 1.5, 8, 8),
])
def test_prefetch_matches_oracle(cuda, R, S, K, E, B, tp, mode, mv, Hp, n_proj):
    from load_balancing_planner_b200 import moonep
    H = 16
    tk, tpe, _ = problem(R, S, K, E, mv, "hot8", seed=2)
    h = moonep.moonep_create(S, H, K, E, R, B, tp, mode=mode)
    p = gpu_plan(h, tk, tpe)
    Ws = [synth.hidden_bf16(1, E, H * Hp, seed=20 + i).view(E, H, Hp) for i in range(n_proj)]
    pools = [torch.empty((R, B, H, Hp), dtype=torch.int16, device="cuda").fill_(0x7F7F).view(torch.bfloat16)
             for _ in range(n_proj)]
    moonep.moonep_prefetch_weight(h, p, [W.cuda() for W in Ws], pools)
    torch.cuda.synchronize()
    assert moonep.moonep_read_status(p) == 0
    o = oracle.plan(tk, E, B, tp, mode, tpe)
    assert (o["slot_expert"] >= 0).any()
    for W, pool in zip(Ws, pools):
        opool = np.full((R * B, H * Hp), 0x7F7F, np.uint16)
        oracle.prefetch(o["slot_expert"], synth.bf16_bits(W).reshape(E, H * Hp), opool)
        assert np.array_equal(bits(pool).reshape(R * B, H * Hp), opool)
    h.close()


def test_prefetch_inference_shape_full(cuda):
    # R=8, S=4096, K=8, E=256, B=4, H=7168, H'=2048, three projections, maxvio 4
    from load_balancing_planner_b200 import moonep
    R, S, K, E, B, H, Hp, tp = 8, 4096, 8, 256, 4, 7168, 2048, 128
    tk, tpe, _ = problem(R, S, K, E, 4.0, "hot8", seed=0)
    h = moonep.moonep_create(S, H, K, E, R, B, tp, mode=1)
    p = gpu_plan(h, tk, tpe)
    o = oracle.plan(tk, E, B, tp, 1, tpe)
    assert np.array_equal(p.slots().cpu().numpy(), o["slot_expert"])
    gen = torch.Generator(device="cuda").manual_seed(0)
    Ws = [torch.randn((E, H, Hp), generator=gen, device="cuda", dtype=torch.bfloat16) for _ in range(3)]
    pools = [torch.empty((R, B, H, Hp), dtype=torch.int16, device="cuda").fill_(0x7F7F).view(torch.bfloat16)
             for _ in range(3)]
    moonep.moonep_prefetch_weight(h, p, Ws, pools)
    torch.cuda.synchronize()
    se = o["slot_expert"]
    for W, pool in zip(Ws, pools):
        for r in range(R):
            for b in range(B):
                if se[r, b] >= 0:
                    assert torch.equal(pool[r, b].view(torch.int16), W[se[r, b]].view(torch.int16))
                else:
                    assert bool((pool[r, b].view(torch.int16) == 0x7F7F).all())
    # overflow experts are served from their home rows: at least one exists here
    rc = o["row_counts"]
    assert any(rc[r, e] > 0 for r in range(R) for e in range(E) if e // 32 != r)
    h.close()


@pytest.mark.parametrize("H,Hp", [(136, 200), (256, 128)])
def test_prefetch_bulk_path_with_a_ragged_last_piece(cuda, H, Hp):
    # expert matrices of 54,400 and 65,536 bytes: moved in 32 KB bulk pieces,
    # the first with a shorter last piece
    from load_balancing_planner_b200 import moonep
    R, S, K, E, B, tp = 8, 1024, 8, 64, 8, 128
    tk, tpe, _ = problem(R, S, K, E, 2.0, "hot8", seed=5)
    h = moonep.moonep_create(S, H, K, E, R, B, tp)
    p = gpu_plan(h, tk, tpe)
    Ws = [synth.hidden_bf16(1, E, H * Hp, seed=30 + i).view(E, H, Hp) for i in range(2)]
    pools = [torch.empty((R, B, H, Hp), dtype=torch.int16, device="cuda").fill_(0x7F7F).view(torch.bfloat16)
             for _ in range(2)]
    moonep.moonep_prefetch_weight(h, p, [W.cuda() for W in Ws], pools)
    torch.cuda.synchronize()
    assert moonep.moonep_read_status(p) == 0
    o = oracle.plan(tk, E, B, tp, 0, tpe)
    for W, pool in zip(Ws, pools):
        opool = np.full((R * B, H * Hp), 0x7F7F, np.uint16)
        oracle.prefetch(o["slot_expert"], synth.bf16_bits(W).reshape(E, H * Hp), opool)
        assert np.array_equal(bits(pool).reshape(R * B, H * Hp), opool)
    h.close()
