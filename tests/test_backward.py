"""The backward pair (MoonEP README, "dispatch bwd" and "combine bwd") through
the Buffer API, and one whole training step of a MoE layer -- dispatch,
prefetch_weight, an expert, combine, then backward through the same calls and
reduce_grad -- against plain PyTorch fp32 autograd of the same layer.

combine backward  = dispatch(grad_output, plan=saved): no planning, no weights.
dispatch backward = combine(plan, grad_hidden_nvs) unweighted, plus
                    reduce_grad of the redundant experts' weight gradients.
The route-weight gradient is gathered back to [R,S,K] by combine's
gathered-weights output.  The expert (one [H,H] projection per expert) and
the per-slot elementwise products are the consumer's work and are plain
PyTorch here."""
import numpy as np
import pytest
import torch

import oracle
from load_balancing_planner_b200 import synth
from tests.conftest import bf16_to_f64, rel_close
from tests.gpu_util import bits, problem

pytestmark = pytest.mark.gpu

R, S, K, E, B, H, TP = 4, 256, 4, 16, 4, 64, 16


def _layer(mv, seed):
    from load_balancing_planner_b200.buffer import Buffer
    tk, tpe, _ = problem(R, S, K, E, mv, "zipf", seed=seed)
    dev = torch.device("cuda:0")
    x = synth.hidden_bf16(R, S, H, seed=seed).to(dev)
    w = torch.from_numpy(synth.route_weights(R, S, K, seed=seed)).to(dev)
    buf = Buffer(S, H, K, E, R, token_padding=TP, device=dev)
    return buf, tk, tpe, x, w


def _rows(plan):
    """(rank, start, n, row) of every non-empty row of a plan."""
    cu, rc = plan.cu_seqlens.cpu().numpy(), plan.row_counts.cpu().numpy()
    out = []
    for r in range(cu.shape[0]):
        prev = 0
        for i in range(cu.shape[1]):
            if rc[r, i]:
                out.append((r, prev, int(rc[r, i]), i))
            prev = int(cu[r, i])
    return out


@pytest.mark.parametrize("mv", [0.0, 2.0])
def test_combine_backward_is_dispatch_with_the_saved_plan(cuda, mv):
    buf, tk, tpe, x, w = _layer(mv, seed=21)
    dev = x.device
    _, _, _, plan = buf.dispatch(x, w, torch.from_numpy(tk).to(dev), torch.from_numpy(tpe).to(dev))
    saved = {k: getattr(plan, k).clone() for k in ("dst", "cu_seqlens", "row_counts", "slot_expert")}
    g_cpu = synth.hidden_bf16(R, S, H, seed=99)
    gn, gwn, cu, p2 = buf.dispatch(g_cpu.to(dev), plan=plan)
    torch.cuda.synchronize()
    assert p2 is plan and gwn is None and cu is plan.cu_seqlens
    for k, v in saved.items():  # no planning happened
        assert torch.equal(getattr(plan, k), v), k
    o = oracle.plan(tk, E, B, TP, 0, tpe)
    obuf, _ = oracle.dispatch(o["dst"], synth.bf16_bits(g_cpu), None, o["nvs"], sentinel=0)
    real = np.zeros(R * o["nvs"], bool)
    real[o["dst"].ravel()] = True
    assert np.array_equal(bits(gn).reshape(R * o["nvs"], H)[real], obuf.reshape(R * o["nvs"], H)[real])
    buf.destroy()


@pytest.mark.parametrize("mv", [0.0, 2.0])
def test_dispatch_backward_is_unweighted_combine(cuda, mv):
    buf, tk, tpe, x, w = _layer(mv, seed=22)
    dev = x.device
    _, _, _, plan = buf.dispatch(x, w, torch.from_numpy(tk).to(dev), torch.from_numpy(tpe).to(dev))
    gy_cpu = synth.hidden_bf16(R, buf.nvs, H, seed=98)
    gx, gw, none = buf.combine(plan, gy_cpu.to(dev))
    torch.cuda.synchronize()
    assert gw is None and none is None
    o = oracle.plan(tk, E, B, TP, 0, tpe)
    want, _ = oracle.combine(o["dst"], synth.bf16_bits(gy_cpu), None)
    assert rel_close(bf16_to_f64(bits(gx)), bf16_to_f64(want), 1e-2).all()
    buf.destroy()


@pytest.mark.parametrize("mv", [0.5, 2.0])
def test_training_step_matches_torch_autograd(cuda, mv):
    buf, tk, tpe, x, w = _layer(mv, seed=23)
    dev = x.device
    g = torch.Generator(device="cpu").manual_seed(5)
    W = (torch.randn(E, H, H, generator=g) / H ** 0.5).to(torch.bfloat16).to(dev)
    dout = torch.randn(R, S, H, generator=g).to(torch.bfloat16).to(dev)
    topk = torch.from_numpy(tk).to(dev)

    # ---- forward through the library ----
    hn, wn, _, plan = buf.dispatch(x, w, topk, torch.from_numpy(tpe).to(dev))
    pool = torch.zeros(R, B, H, H, dtype=torch.bfloat16, device=dev)
    buf.prefetch_weight(plan, [W], [pool])
    buf.check(plan)
    slot_e = plan.slots().cpu().numpy()
    rows = _rows(plan)
    assert any(i >= E for _, _, _, i in rows) == (mv > 0)  # copies exist iff skewed

    def weight_of(r, i):
        return W[i] if i < E else pool[r, i - E]

    y = torch.zeros(R, buf.nvs, H, dtype=torch.bfloat16, device=dev)
    for r, st, n, i in rows:
        if i < E:
            assert i // (E // R) == r  # training: rows below E are home rows
        else:
            assert torch.equal(pool[r, i - E], W[slot_e[r, i - E]])
        y[r, st:st + n] = (hn[r, st:st + n].float() @ weight_of(r, i).float()).to(torch.bfloat16)
    out, gathered, _ = buf.combine(plan, y, wn)

    # ---- backward through the library ----
    dd, _, _, _ = buf.dispatch(dout, plan=plan)                  # combine bwd
    dwn = torch.zeros(R, buf.nvs, dtype=torch.float32, device=dev)
    dxn = torch.zeros(R, buf.nvs, H, dtype=torch.bfloat16, device=dev)
    Gsum = torch.zeros(E, H, H, dtype=torch.float32, device=dev)
    RB = torch.zeros(R, B, H, H, dtype=torch.float32, device=dev)
    for r, st, n, i in rows:
        d = dd[r, st:st + n].float()
        dwn[r, st:st + n] = (d * y[r, st:st + n].float()).sum(-1)
        dy = d * wn[r, st:st + n, None]
        dxn[r, st:st + n] = (dy @ weight_of(r, i).float().T).to(torch.bfloat16)
        gW = hn[r, st:st + n].float().T @ dy
        if i < E:
            Gsum[i] += gW
        else:
            RB[r, i - E] = gW
    _, dw, _ = buf.combine(plan, dd, dwn)                        # gather dL/dw to [R,S,K]
    dx, _, _ = buf.combine(plan, dxn)                            # dispatch bwd
    buf.reduce_grad(plan, [Gsum], [RB])
    torch.cuda.synchronize()
    assert torch.count_nonzero(RB[torch.from_numpy(slot_e >= 0).to(dev)]) == 0  # consumed slots zeroed

    # ---- plain PyTorch fp32 autograd of the same layer ----
    xf = x.float().requires_grad_()
    wf = w.clone().requires_grad_()
    Wf = W.float().requires_grad_()
    y_ref = torch.einsum("rsh,rskhj->rskj", xf, Wf[topk.long()])
    out_ref = torch.einsum("rsk,rskj->rsj", wf, y_ref)
    out_ref.backward(dout.float())

    def close(a, b, tol):
        return rel_close(a.detach().double().cpu().numpy(), b.detach().double().cpu().numpy(), tol).all()

    assert torch.equal(gathered, w)
    assert close(out.float(), out_ref, 1e-2)
    assert close(dx.float(), xf.grad, 1e-2)
    assert close(dw, wf.grad, 1e-2)
    assert close(Gsum, Wf.grad, 1e-3)
    buf.destroy()
