"""One rank of a real EP group, run on one GPU: every rank plans from its own
picks and the gathered counts (moonep_plan_rank), and dispatch/combine reach
the R ranks' buffers through a pointer table (R separate allocations here,
peer mappings on R GPUs).  Plans and dispatched buffers are checked bit for
bit against the oracle's group plan and dispatch on the same routing; combine
bit for bit against the group combine, and against the oracle's fp64 sum within
the bf16 tolerance."""
import numpy as np
import pytest
import torch

import oracle
from load_balancing_planner_b200 import synth
from tests.conftest import bf16_to_f64, rel_close
from tests.gpu_util import bits, gpu_plan, plan_to_numpy, problem

pytestmark = pytest.mark.gpu

SENT = 0xFFFF
RTOL_BF16 = 1e-2  # bf16 output tolerance against the oracle's fp64 sum
PLAN_WHOLE = ("cu_seqlens", "row_counts", "slot_expert", "counts", "assign")


def _rank_plans(h, tk, counts_all):
    from load_balancing_planner_b200 import moonep
    c = torch.from_numpy(np.ascontiguousarray(counts_all)).cuda()
    out = []
    for r in range(h.R):
        t = torch.from_numpy(np.ascontiguousarray(tk[r])).cuda()
        out.append(moonep.moonep_plan_rank(h, r, t, c))
    torch.cuda.synchronize()
    return out


# (name, R, S, K, E, B, token_padding, mode, routing profile, maxvio)
CASES = [
    ("tiny", 2, 64, 2, 8, 4, 8, 0, "boost0", 1.0),
    ("zipf", 8, 1024, 8, 64, 8, 128, 0, "zipf", 2.0),
    ("train", 8, 4096, 8, 256, 32, 128, 0, "hot8", 0.0),
    ("train_mv2", 8, 4096, 8, 256, 32, 128, 0, "hot8", 2.0),
    ("train_mv20", 8, 4096, 8, 256, 32, 128, 0, "hot8", 20.0),
    ("infer", 8, 4096, 8, 256, 4, 128, 1, "hot8", 4.0),
    ("infer_count", 8, 4096, 8, 256, 4, 128, 2, "hot8", 4.0),
    ("ragged", 3, 1000, 3, 24, 8, 16, 0, "hot8", 1.5),
    ("k32", 2, 100, 32, 64, 32, 4, 0, "zipf", 0.5),
    ("many_ranks", 64, 40, 4, 256, 4, 8, 0, "hot8", 3.0),
    ("long_seq", 8, 16384, 8, 256, 32, 128, 0, "hot8", 2.0),
    ("fewest_train", 8, 4096, 8, 256, 32, 128, 3, "hot8", 2.0),
    ("fewest_ragged", 3, 1000, 3, 24, 8, 16, 3, "hot8", 1.5),
]


@pytest.mark.parametrize("case", [pytest.param(c, id=c[0]) for c in CASES])
def test_rank_plans_match_the_group_plan_of_the_oracle(cuda, case):
    from load_balancing_planner_b200 import moonep
    name, R, S, K, E, B, tp, mode, profile, mv = case
    tk, tpe, _ = problem(R, S, K, E, mv, profile, seed=21)
    want = oracle.plan(tk, E, B, tp, mode, tpe)
    assert want["status"] == 0
    h = moonep.moonep_create(S, 8, K, E, R, B, tp, mode=mode)
    for r, p in enumerate(_rank_plans(h, tk, tpe)):
        assert moonep.moonep_read_status(p) == 0, r
        assert p.dst.shape == (S, K)
        assert np.array_equal(p.dst.cpu().numpy(), want["dst"][r]), f"dst of rank {r}"
        mine = oracle.plan_rank(tk[r], tpe, r, E, B, tp, mode)  # the rank's share, placed in closed form
        assert mine["status"] == 0 and np.array_equal(mine["dst"], want["dst"][r])
        for k in PLAN_WHOLE:
            g = getattr(p, k).cpu().numpy()
            if k == "slot_expert":
                g = g[:, :B]
            assert np.array_equal(g, np.asarray(want[k])), f"{k} on rank {r}"
        assert np.float32(p.maxvio.item()) == np.float32(want["maxvio"])
    h.close()


def test_rank_plans_alternate_with_group_plans(cuda):
    # the two planners keep separate workspaces on one handle
    from load_balancing_planner_b200 import moonep
    R, S, K, E, B, tp = 8, 1024, 8, 64, 8, 128
    h = moonep.moonep_create(S, 8, K, E, R, B, tp)
    for seed in (1, 2, 3):
        tk, tpe, _ = problem(R, S, K, E, 1.0 + seed, "zipf", seed=seed)
        want = oracle.plan(tk, E, B, tp, 0, tpe)
        g = plan_to_numpy(gpu_plan(h, tk, tpe))
        assert np.array_equal(g["dst"], want["dst"])
        ps = _rank_plans(h, tk, tpe)
        for r, p in enumerate(ps):
            assert np.array_equal(p.dst.cpu().numpy(), want["dst"][r])
    h.close()


# (R, S, K, E, B, H, token_padding, mode, profile, maxvio): bulk-copy rows
# (H*2 >= 2 KB), 16-byte-vector rows, a K without a compiled case
@pytest.mark.parametrize("R,S,K,E,B,H,tp,mode,profile,mv", [
    (8, 1024, 8, 64, 8, 2048, 128, 0, "zipf", 2.0),
    (3, 1000, 3, 24, 8, 264, 16, 0, "hot8", 1.5),
    (4, 333, 3, 24, 0, 72, 16, 1, "hot8", 1.5),
])
def test_rank_dispatch_and_combine_match_the_oracle(cuda, R, S, K, E, B, H, tp, mode, profile, mv):
    from load_balancing_planner_b200 import moonep
    tk, tpe, _ = problem(R, S, K, E, mv, profile, seed=22)
    x = synth.hidden_bf16(R, S, H, seed=22)
    w = synth.route_weights(R, S, K, seed=22)
    h = moonep.moonep_create(S, H, K, E, R, B, tp, mode=mode)
    nvs = h.nvs
    plans = _rank_plans(h, tk, tpe)
    # R separate buffers, prefilled so that untouched padding shows
    bufs = [torch.full((nvs, H), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16) for _ in range(R)]
    wbufs = [torch.full((nvs,), float("nan"), dtype=torch.float32, device="cuda") for _ in range(R)]
    xd, wd = x.cuda(), torch.from_numpy(w).cuda()
    for r in range(R):
        moonep.moonep_dispatch_rank(h, plans[r], xd[r].contiguous(), wd[r].contiguous(), bufs, wbufs)
    torch.cuda.synchronize()

    o = oracle.plan(tk, E, B, tp, mode, tpe)
    obuf, own = oracle.dispatch(o["dst"], synth.bf16_bits(x), w, o["nvs"], sentinel=SENT)
    got = np.concatenate([bits(b) for b in bufs])
    assert np.array_equal(got, obuf)
    gw = np.concatenate([b.cpu().numpy() for b in wbufs])
    assert np.array_equal(gw.view(np.uint32), own.view(np.uint32))

    # combine of expert outputs that live on R separate buffers: bit for bit
    # the group combine (same kernel, same k order in fp32), and within the
    # bf16 tolerance of the oracle's fp64 sum
    y = synth.hidden_bf16(1, R * nvs, H, seed=23)[0]
    ys = [y[q * nvs:(q + 1) * nvs].cuda().contiguous() for q in range(R)]
    w_all = np.nan_to_num(own)
    wn = [torch.from_numpy(w_all[q * nvs:(q + 1) * nvs]).cuda() for q in range(R)]
    gp = gpu_plan(h, tk, tpe)
    y_dev = y.reshape(R, nvs, H).cuda()
    w_dev = torch.from_numpy(w_all.reshape(R, nvs)).cuda()
    group_w, group_gw = moonep.moonep_combine(h, gp, y_dev, w_dev)
    group_u, _ = moonep.moonep_combine(h, gp, y_dev, None)
    want, want_gw = oracle.combine(o["dst"], synth.bf16_bits(y), w_all)
    want_u, _ = oracle.combine(o["dst"], synth.bf16_bits(y), None)
    for r in range(R):
        out, g = moonep.moonep_combine_rank(h, plans[r], ys, wn)
        out_u, g_u = moonep.moonep_combine_rank(h, plans[r], ys, None)
        torch.cuda.synchronize()
        assert moonep.moonep_read_status(plans[r]) == 0
        assert torch.equal(out, group_w[r]) and torch.equal(out_u, group_u[r]), r
        assert np.array_equal(g.cpu().numpy().view(np.uint32), want_gw[r].view(np.uint32)), r
        assert torch.equal(g, group_gw[r])
        assert g_u is None
        for got, ref in ((out, want[r]), (out_u, want_u[r])):
            assert rel_close(bf16_to_f64(bits(got)), bf16_to_f64(ref), RTOL_BF16).all(), r
            assert np.mean(bits(got) == ref) > 0.999
    h.close()


def test_rank_path_roundtrip_through_rank_buffer(cuda):
    # RankBuffer (the per-rank user API) on R local buffers: unweighted
    # combine of an untouched dispatch gives K * x exactly (K = 8, bf16)
    from load_balancing_planner_b200.ep import RankBuffer
    R, S, K, E, H = 8, 512, 8, 64, 1024
    tk, tpe, _ = problem(R, S, K, E, 2.0, "hot8", seed=24)
    nvs = RankBuffer.nvs_of(S, K, E, R)
    bufs = [torch.zeros((nvs, H), dtype=torch.bfloat16, device="cuda") for _ in range(R)]
    wbufs = [torch.zeros((nvs,), dtype=torch.float32, device="cuda") for _ in range(R)]
    ranks = [RankBuffer(S, H, K, E, R, r, bufs, wbufs) for r in range(R)]
    assert ranks[0].nvs == nvs
    x = synth.hidden_bf16(R, S, H, seed=24).cuda()
    w = torch.from_numpy(synth.route_weights(R, S, K, seed=24)).cuda()
    c = torch.from_numpy(tpe).cuda()
    plans = []
    for r, rb in enumerate(ranks):
        p = rb.plan(torch.from_numpy(np.ascontiguousarray(tk[r])).cuda(), counts_all=c)
        rb.dispatch(p, x[r].contiguous(), w[r].contiguous())
        plans.append(p)
    from load_balancing_planner_b200 import moonep
    table = moonep.PeerTable(bufs, (nvs, H), torch.bfloat16)
    for r, rb in enumerate(ranks):
        out, gw = rb.combine(plans[r], bufs, weighted=False)
        assert gw is None
        assert torch.equal(out, (x[r].float() * K).to(torch.bfloat16))
        # the same through a table checked once, and through the rank's own tables
        assert torch.equal(rb.combine(plans[r], table, weighted=False)[0], out)
        assert torch.equal(rb.combine(plans[r], weighted=False)[0], out)
        _, gw = rb.combine(plans[r], bufs)
        assert torch.equal(gw, w[r])  # each slot's weight travelled with its row
    with pytest.raises(ValueError):  # a table of the wrong tensors
        ranks[0].combine(plans[0], moonep.PeerTable(wbufs, (nvs,), torch.float32))
    for rb in ranks:
        rb.destroy()


def test_rank_plan_errors(cuda):
    from load_balancing_planner_b200 import moonep
    R, S, K, E, B, H, tp = 4, 256, 4, 16, 4, 64, 16
    tk, tpe, _ = problem(R, S, K, E, 1.0, "hot8", seed=25)
    h = moonep.moonep_create(S, H, K, E, R, B, tp)

    def plan(r, topk, counts):
        p = moonep.moonep_plan_rank(h, r, torch.from_numpy(np.ascontiguousarray(topk)).cuda(),
                                    torch.from_numpy(np.ascontiguousarray(counts)).cuda())
        return p, moonep.moonep_read_status(p)

    # rank 1's row moved by one pick between two experts: rank 1 sees the
    # mismatch; rank 0 checks only its own row (and the row sums, still S*K)
    bad = tpe.copy()
    e0, e1 = int(np.argmax(bad[1])), int(np.argmin(bad[1]))
    bad[1, e0] -= 1
    bad[1, e1] += 1
    assert plan(1, tk[1], bad)[1] == moonep.STATUS_COUNT_MISMATCH
    assert plan(0, tk[0], bad)[1] == 0
    # a negative count, or a row that does not sum to S*K: every rank refuses
    for r2 in (0, 3):
        neg = tpe.copy()
        neg[2, 0] = -1
        neg[2, 1] += 1
        assert plan(r2, tk[r2], neg)[1] == moonep.STATUS_COUNT_MISMATCH
        short = tpe.copy()
        short[2, int(np.argmax(short[2]))] -= 1
        assert plan(r2, tk[r2], short)[1] == moonep.STATUS_COUNT_MISMATCH
    # an expert id outside [0, E) in the rank's own picks
    t2 = tk[2].copy()
    t2[5, 0] = E
    p, st = plan(2, t2, tpe)
    assert st & moonep.STATUS_BAD_EXPERT
    # a failed plan moves nothing
    bufs = [torch.full((h.nvs, H), 3.0, dtype=torch.bfloat16, device="cuda") for _ in range(R)]
    moonep.moonep_dispatch_rank(h, p, torch.zeros((S, H), dtype=torch.bfloat16, device="cuda"), None, bufs)
    torch.cuda.synchronize()
    assert all(bool((b == 3.0).all()) for b in bufs)
    # host checks
    c = torch.from_numpy(tpe).cuda()
    with pytest.raises(moonep.MoonepError) as e:
        moonep.moonep_plan_rank(h, R, torch.from_numpy(np.ascontiguousarray(tk[0])).cuda(), c)
    assert e.value.code == moonep.ERR_SIZE
    with pytest.raises(ValueError):
        moonep.moonep_dispatch(h, p, torch.zeros((R, S, H), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(ValueError):
        moonep.moonep_dispatch_rank(h, p, torch.zeros((S, H), dtype=torch.bfloat16, device="cuda"), None,
                                    bufs[:R - 1])
    odd = [b for b in bufs]
    odd[1] = torch.zeros((h.nvs * H + 1,), dtype=torch.bfloat16, device="cuda")[1:].view(h.nvs, H)
    with pytest.raises(moonep.MoonepError) as e:
        moonep.moonep_dispatch_rank(h, p, torch.zeros((S, H), dtype=torch.bfloat16, device="cuda"), None, odd)
    assert e.value.code == moonep.ERR_ALIGN
    h.close()


# (R, S, K, E, B, token_padding, mode, maxvio, H, Hp): bulk-copy matrices,
# plain-vector matrices, inference with overflow (mode 1) and slots by count
@pytest.mark.parametrize("R,S,K,E,B,tp,mode,mv,H,Hp", [
    (8, 512, 8, 64, 8, 128, 0, 2.0, 256, 64),
    (4, 200, 4, 32, 8, 16, 0, 1.5, 64, 32),
    (8, 512, 8, 64, 2, 128, 1, 4.0, 256, 72),
    (8, 512, 8, 64, 2, 128, 2, 4.0, 64, 40),
])
def test_rank_prefetch_and_reduce_grad_match_the_oracle(cuda, R, S, K, E, B, tp, mode, mv, H, Hp):
    from load_balancing_planner_b200 import moonep
    G, P = E // R, 2
    tk, tpe, _ = problem(R, S, K, E, mv, "hot8", seed=26)
    h = moonep.moonep_create(S, H, K, E, R, B, tp, mode=mode)
    plans = _rank_plans(h, tk, tpe)
    se = plans[0].slots().cpu().numpy()
    assert (se >= 0).any()
    gen = torch.Generator().manual_seed(26)
    W = [torch.randn((E, H, Hp), generator=gen).to(torch.bfloat16) for _ in range(P)]
    # every rank's home experts and slots as separate allocations
    home = [[W[p][q * G:(q + 1) * G].cuda().contiguous() for q in range(R)] for p in range(P)]
    pools = [[torch.full((B, H, Hp), -1, dtype=torch.int16, device="cuda").view(torch.bfloat16)
              for _ in range(P)] for _ in range(R)]
    for r in range(R):
        moonep.moonep_prefetch_weight_rank(h, plans[r], r, home, pools[r])
    torch.cuda.synchronize()
    for p in range(P):
        want = np.full((R * B, H * Hp), 0xFFFF, np.uint16)
        oracle.prefetch(se, bits(W[p]).reshape(E, H * Hp), want)
        got = np.concatenate([bits(pools[r][p]).reshape(B, H * Hp) for r in range(R)])
        assert np.array_equal(got, want), p

    Gr = [torch.randn((E, H, Hp), generator=gen) * 1e-3 for _ in range(P)]
    RB = [torch.randn((R, B, H, Hp), generator=gen) * 1e-3 for _ in range(P)]
    grads = [[Gr[p][q * G:(q + 1) * G].cuda().contiguous() for p in range(P)] for q in range(R)]
    rbs = [[RB[p][q].cuda().contiguous() for q in range(R)] for p in range(P)]
    for q in range(R):
        moonep.moonep_reduce_grad_rank(h, plans[q], q, grads[q], rbs)
    # the group call on the same data: same kernel, same (rank, slot) order
    gG, gRB = [g.cuda() for g in Gr], [rb.cuda() for rb in RB]
    moonep.moonep_reduce_grad(h, plans[0], gG, gRB)
    torch.cuda.synchronize()
    for p in range(P):
        wg = Gr[p].numpy().reshape(E, H * Hp).copy()
        wrb = RB[p].numpy().reshape(R * B, H * Hp).copy()
        oracle.reduce_grad(se, wg, wrb)
        got_g = np.concatenate([grads[q][p].cpu().numpy().reshape(G, H * Hp) for q in range(R)])
        got_rb = np.concatenate([rbs[p][q].cpu().numpy().reshape(B, H * Hp) for q in range(R)])
        assert np.array_equal(got_g.view(np.uint32), gG[p].cpu().numpy().reshape(E, -1).view(np.uint32)), p
        assert rel_close(got_g, wg, 1e-5).all(), p
        # consumed slots exactly +0.0, the others untouched
        assert np.array_equal(got_rb.view(np.uint32), wrb.view(np.uint32)), p
    # host checks: rank range, one table row per rank
    with pytest.raises(moonep.MoonepError) as e:
        moonep.moonep_prefetch_weight_rank(h, plans[0], R, home, pools[0])
    assert e.value.code == moonep.ERR_SIZE
    with pytest.raises(ValueError):
        moonep.moonep_reduce_grad_rank(h, plans[0], 0, grads[0], [row[:R - 1] for row in rbs])
    h.close()
