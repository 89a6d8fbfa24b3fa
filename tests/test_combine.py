"""GPU combine against the oracle (bf16 output within rel 1e-2 of the fp64
oracle, as |a-b| <= 1e-2 (|b| + rms b); gathered weights exact), and the
exact round trips: unweighted combine(dispatch(x)) = K x, softmax-weighted
combine(dispatch(x)) = x."""
import numpy as np
import pytest
import torch

import oracle
from load_balancing_planner_b200 import synth
from tests.conftest import bf16_to_f64, rel_close
from tests.gpu_util import bits, gpu_plan, problem

pytestmark = pytest.mark.gpu
RTOL_BF16 = 1e-2


def _expert_output(R, nvs, H, seed):
    # arbitrary expert output over the whole buffer, padding included
    return synth.hidden_bf16(R, nvs, H, seed=seed + 100)


@pytest.mark.parametrize("R,S,K,E,B,H,tp,mode,profile,mv", [
    (2, 64, 2, 8, 4, 128, 8, 0, "boost0", 1.0),
    (8, 1024, 8, 64, 8, 2048, 128, 0, "zipf", 0.5),
    (8, 1024, 8, 64, 8, 2048, 128, 0, "zipf", 2.0),
    (3, 1000, 3, 24, 8, 264, 16, 0, "hot8", 1.5),
    (4, 333, 3, 24, 0, 72, 16, 1, "hot8", 1.5),
    (2, 100, 32, 64, 32, 8, 4, 0, "zipf", 0.5),
    (4, 200, 6, 48, 12, 136, 8, 0, "hot8", 2.0),
    (4, 200, 5, 40, 10, 40, 8, 0, "hot8", 2.0),
])
@pytest.mark.parametrize("weighted", [True, False])
def test_combine_matches_oracle(cuda, R, S, K, E, B, H, tp, mode, profile, mv, weighted):
    from load_balancing_planner_b200 import moonep
    tk, tpe, _ = problem(R, S, K, E, mv, profile, seed=9)
    h = moonep.moonep_create(S, H, K, E, R, B, tp, mode=mode)
    p = gpu_plan(h, tk, tpe)
    y = _expert_output(R, h.nvs, H, 9)
    wn = torch.from_numpy(synth.normal_f32((R, h.nvs), 9, stream=3)).cuda() if weighted else None
    out, gw = moonep.moonep_combine(h, p, y.cuda(), wn)
    torch.cuda.synchronize()
    assert moonep.moonep_read_status(p) == 0
    o = oracle.plan(tk, E, B, tp, mode, tpe)
    oout, ogw = oracle.combine(o["dst"], synth.bf16_bits(y).reshape(-1, H),
                               None if wn is None else wn.cpu().numpy().reshape(-1))
    g = bf16_to_f64(bits(out))
    want = bf16_to_f64(oout)
    ok = rel_close(g, want, RTOL_BF16)
    assert ok.all(), f"{(~ok).sum()} of {ok.size} outside tolerance"
    # the fp32 sum rounds to the same bf16 as the fp64 sum almost everywhere
    assert np.mean(bits(out) == oout) > 0.999
    if weighted:
        assert np.array_equal(gw.cpu().numpy(), ogw)
    h.close()


@pytest.mark.parametrize("K,E", [(2, 16), (8, 256)])
def test_roundtrip_exact(cuda, K, E):
    from load_balancing_planner_b200 import moonep
    R, S, B, H, tp = 8, 4096, E // 8, 7168, 128
    tk, tpe, _ = problem(R, S, K, E, min(4.0, E / K - 1.5), "hot8", seed=3)
    x = synth.hidden_bf16(R, S, H, seed=3).cuda()
    w = torch.from_numpy(synth.route_weights(R, S, K, seed=3)).cuda()
    h = moonep.moonep_create(S, H, K, E, R, B, tp)
    p = gpu_plan(h, tk, tpe)
    buf, wn = moonep.moonep_dispatch(h, p, x, w)
    out, gw = moonep.moonep_combine(h, p, buf, None)
    # K copies of one bf16 value sum exactly in fp32; K*x is a bf16 value
    # (K = 2^n).  The sum starts from +0, so x = -0 gives +0: adding 0.0 to
    # the expected value makes the same choice.
    want = (x.float() * K + 0.0).to(torch.bfloat16)
    assert torch.equal(out.view(torch.int16), want.view(torch.int16))
    out, gw = moonep.moonep_combine(h, p, buf, wn)
    # softmax weights sum to 1 within fp32 rounding, far inside bf16's half-ulp
    assert torch.equal(out.view(torch.int16), (x.float() + 0.0).to(torch.bfloat16).view(torch.int16))
    assert torch.equal(gw, w)
    h.close()


def test_combine_training_shape_sampled(cuda):
    # full training shape; 512 tokens checked against the oracle one by one
    from load_balancing_planner_b200 import moonep
    R, S, K, E, B, H, tp = 8, 4096, 8, 256, 32, 7168, 128
    tk, tpe, _ = problem(R, S, K, E, 4.0, "hot8", seed=6)
    h = moonep.moonep_create(S, H, K, E, R, B, tp)
    p = gpu_plan(h, tk, tpe)
    gen = torch.Generator(device="cuda").manual_seed(6)
    y = torch.randn((R, h.nvs, H), generator=gen, device="cuda").to(torch.bfloat16)
    wn = torch.randn((R, h.nvs), generator=gen, device="cuda")
    out, gw = moonep.moonep_combine(h, p, y, wn)
    torch.cuda.synchronize()
    o = oracle.plan(tk, E, B, tp, 0, tpe)
    assert np.array_equal(p.dst.cpu().numpy(), o["dst"])
    rng = np.random.default_rng(6)
    toks = rng.choice(R * S, size=512, replace=False)
    d = o["dst"].reshape(R * S, K)[toks]                       # [n, K]
    rows = y.view(-1, H)[torch.from_numpy(d.reshape(-1)).cuda().long()]
    ysmall = bits(rows)                                         # [n*K, H]
    wsmall = wn.view(-1)[torch.from_numpy(d.reshape(-1)).cuda().long()].cpu().numpy()
    dsmall = np.arange(len(toks) * K, dtype=np.int32).reshape(1, len(toks), K)
    oout, ogw = oracle.combine(dsmall, ysmall, wsmall)
    g = bf16_to_f64(bits(out.view(R * S, H)[torch.from_numpy(toks).cuda()]))
    ok = rel_close(g, bf16_to_f64(oout[0]), RTOL_BF16)
    assert ok.all()
    assert np.array_equal(gw.view(R * S, K)[torch.from_numpy(toks).cuda()].cpu().numpy(), ogw[0])
    h.close()


def test_dispatch_combine_inference_shape_sampled(cuda):
    # the inference shape (R=8, S=4096, K=8, E=256, B=4, H=7168, maxvio 4):
    # copies past the B slots are read from their home rows.  Dispatch then a
    # weighted combine of the dispatched buffer; 512 tokens against the
    # oracle's dispatch and combine of those tokens' picks, one by one
    from load_balancing_planner_b200 import moonep
    R, S, K, E, B, H, tp = 8, 4096, 8, 256, 4, 7168, 128
    tk, tpe, _ = problem(R, S, K, E, 4.0, "hot8", seed=12)
    xh = synth.hidden_bf16(R, S, H, seed=12)
    wh = synth.route_weights(R, S, K, seed=12)
    h = moonep.moonep_create(S, H, K, E, R, B, tp, mode=1)
    p = gpu_plan(h, tk, tpe)
    o = oracle.plan(tk, E, B, tp, 1, tpe)
    assert np.array_equal(p.dst.cpu().numpy(), o["dst"])
    home = np.arange(E) // (E // R)
    assert any(o["row_counts"][r, e] > 0 for r in range(R) for e in range(E) if home[e] != r), "no overflow rows"
    buf, wn = moonep.moonep_dispatch(h, p, xh.cuda(), torch.from_numpy(wh).cuda())
    out, gw = moonep.moonep_combine(h, p, buf, wn)
    torch.cuda.synchronize()
    assert moonep.moonep_read_status(p) == 0
    rng = np.random.default_rng(12)
    toks = rng.choice(R * S, size=512, replace=False)
    d = o["dst"].reshape(R * S, K)[toks]                        # [n, K] slots of the sampled picks
    dsmall = np.arange(len(toks) * K, dtype=np.int32).reshape(1, len(toks), K)
    xb = synth.bf16_bits(xh).reshape(R * S, H)[toks].reshape(1, len(toks), H)
    wsm = wh.reshape(R * S, K)[toks].reshape(1, len(toks), K)
    obuf, own = oracle.dispatch(dsmall, xb, wsm, len(toks) * K)  # the oracle's slots, renumbered
    sl = torch.from_numpy(d.reshape(-1)).cuda().long()
    assert np.array_equal(bits(buf.view(-1, H)[sl]), obuf)
    assert np.array_equal(wn.view(-1)[sl].cpu().numpy().view(np.uint32), own.view(np.uint32))
    oout, ogw = oracle.combine(dsmall, obuf, own)
    g = bf16_to_f64(bits(out.view(R * S, H)[torch.from_numpy(toks).cuda()]))
    ok = rel_close(g, bf16_to_f64(oout[0]), RTOL_BF16)
    assert ok.all(), f"{(~ok).sum()} of {ok.size} outside tolerance"
    assert np.array_equal(gw.view(R * S, K)[torch.from_numpy(toks).cuda()].cpu().numpy(), ogw[0])
    h.close()
