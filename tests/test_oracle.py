"""Pins of the CPU oracle to things other than itself: hand-worked examples,
closed forms, invariants the pages state, library routines in the special
cases that reduce to them, and brute force on tiny inputs.  Host only."""
import itertools
import json
import os

import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
from load_balancing_planner_b200 import synth
from tests.conftest import bf16_to_f64
from tests.plan_checks import check_plan, copies_of

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------- golden plans
@pytest.mark.parametrize("name", sorted(f for f in os.listdir(GOLDEN) if f.startswith("plan_")))
def test_golden_plan(name):
    g = json.load(open(os.path.join(GOLDEN, name)))
    c = g["config"]
    p = oracle.plan(np.array(g["topk"], np.int32), c["E"], c["B"], c["tp"], c["mode"])
    for key, want in g["expect"].items():
        got = p[key]
        if isinstance(want, float):
            assert got == pytest.approx(want, abs=1e-6), key
        else:
            assert np.array_equal(np.asarray(got), np.asarray(want)), (key, np.asarray(got).tolist())
    check_plan(np.array(g["topk"]), p, c["E"], c["B"], c["tp"], c["mode"])


# ------------------------------------------------------------ bf16 rounding
def test_bf16_rounding_matches_torch():
    g = np.random.default_rng(0)
    x = np.concatenate([
        g.standard_normal(4000).astype(np.float32),
        (g.standard_normal(1000) * 1e-39).astype(np.float32),  # bf16 subnormals
        (g.standard_normal(1000) * 1e30).astype(np.float32),
        np.array([0.0, -0.0, 1.0, 3.0e38, -3.4e38, 1e-45], np.float32),
    ])
    # exact ties between two bf16 values: bit 15 set, bits 0..14 clear
    ties = (g.integers(0, 1 << 15, 500).astype(np.uint32) << 16) | 0x8000
    x = np.concatenate([x, ties.view(np.float32)])
    x = x[np.isfinite(x)]
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.double_to_bf16(x.astype(np.float64))
    assert np.array_equal(got, want)


def test_bf16_rounding_from_fp64_is_single_rounding():
    # 1 + 2^-8 + 2^-30 lies just above the tie between 1 and 1+2^-7: a single
    # rounding from fp64 goes up; rounding first to fp32 would give the tie
    # (1 + 2^-8) and then round down to even.
    x = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert oracle.double_to_bf16(np.array([x]))[0] == 0x3F81
    assert oracle.double_to_bf16(np.array([1.0 + 2.0 ** -8]))[0] == 0x3F80


# -------------------------------------------------------------- maxvio
def test_maxvio_balanced_is_zero():
    tk, mv, _ = synth.routing(8, 1024, 8, 64, 0.0)
    p = oracle.plan(tk, 64, 8, 128)
    assert p["status"] == 0 and p["maxvio"] == 0.0


def test_maxvio_all_tokens_same_experts():
    # every token picks experts 0..K-1: T_0 = R*S, T_bar = R*S*K/E -> maxvio = E/K - 1
    R, S, K, E = 4, 16, 4, 32
    tk = np.broadcast_to(np.arange(K, dtype=np.int32), (R, S, K)).copy()
    p = oracle.plan(tk, E, E // R, 4)
    assert p["status"] == 0
    assert p["maxvio"] == pytest.approx(E / K - 1, abs=1e-6)


# ---------------------------------------------------------- invariants
CASES = [
    dict(R=2, S=64, K=2, E=8, B=4, tp=8, mode=0, mv=1.0, profile="boost0"),
    dict(R=8, S=1024, K=8, E=64, B=8, tp=128, mode=0, mv=2.0, profile="zipf"),
    dict(R=8, S=1024, K=8, E=64, B=8, tp=128, mode=0, mv=0.5, profile="zipf"),
    dict(R=8, S=1024, K=8, E=64, B=2, tp=128, mode=1, mv=2.0, profile="zipf"),
    dict(R=4, S=333, K=3, E=24, B=6, tp=16, mode=0, mv=1.5, profile="hot8"),
    dict(R=4, S=333, K=3, E=24, B=0, tp=16, mode=1, mv=1.5, profile="hot8"),
    dict(R=1, S=100, K=4, E=16, B=16, tp=8, mode=0, mv=1.0, profile="zipf"),
    dict(R=8, S=64, K=1, E=8, B=1, tp=1, mode=0, mv=3.0, profile="boost0"),
    dict(R=8, S=1024, K=8, E=64, B=8, tp=128, mode=3, mv=2.0, profile="zipf"),
    dict(R=4, S=333, K=3, E=24, B=6, tp=16, mode=3, mv=1.5, profile="hot8"),
    dict(R=8, S=4096, K=8, E=256, B=32, tp=128, mode=3, mv=0.5, profile="hot8"),
]


@pytest.mark.parametrize("c", CASES, ids=lambda c: f"R{c['R']}S{c['S']}K{c['K']}E{c['E']}B{c['B']}m{c['mode']}")
def test_plan_invariants(c):
    tk, mv, _ = synth.routing(c["R"], c["S"], c["K"], c["E"], c["mv"], c["profile"], seed=3)
    tpe = synth.local_counts(tk, c["E"])
    p = oracle.plan(tk, c["E"], c["B"], c["tp"], c["mode"], tpe)
    assert p["status"] == 0
    assert p["nvs"] == -(-(c["S"] * c["K"] + 2 * (c["E"] // c["R"]) * (c["tp"] - 1)) // c["tp"]) * c["tp"]
    check_plan(tk, p, c["E"], c["B"], c["tp"], c["mode"])
    if c["R"] == 1:
        assert copies_of(p, c["E"], c["B"], 1) == 0


def test_inference_overflow_occurs():
    # the inference shape at maxvio 4 needs more distinct remote experts than B=4
    tk, mv, _ = synth.routing(8, 4096, 8, 256, 4.0, "hot8", 0)
    p = oracle.plan(tk, 256, 4, 128, 1)
    assert p["status"] == 0
    rc = p["row_counts"]
    overflow = sum(int(rc[r, e] > 0) for r in range(8) for e in range(256) if e // 32 != r)
    assert overflow >= 1
    check_plan(tk, p, 256, 4, 128, 1)


@st.composite
def small_problem(draw):
    R = draw(st.integers(1, 4))
    G = draw(st.integers(1, 4))
    E = R * G
    K = draw(st.integers(1, min(E, 4)))
    S = draw(st.integers(1, 12))
    tp = draw(st.integers(1, 4))
    mode = draw(st.integers(0, 3))
    B = draw(st.integers(G, G + 1)) if mode in (0, 3) else draw(st.integers(0, G))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    hot = draw(st.floats(0.0, 4.0))
    g = np.random.default_rng(seed)
    w = np.ones(E)
    w[g.integers(0, E)] += hot * E
    tk = np.stack([g.choice(E, size=K, replace=False, p=w / w.sum()) for _ in range(R * S)])
    return tk.reshape(R, S, K).astype(np.int32), E, B, tp, mode


@settings(max_examples=400, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(small_problem())
def test_plan_invariants_random(prob):
    tk, E, B, tp, mode = prob
    p = oracle.plan(tk, E, B, tp, mode)
    assert p["status"] == 0
    check_plan(tk, p, E, B, tp, mode)
    if mode in (1, 2):
        _check_slot_choice(p, E, B, tk.shape[0], by_count=mode == 2)
    if mode == 3:
        _check_largest_experts_donated(tk, p, E)


def _check_largest_experts_donated(tk, p, E):
    """Mode 3: a donor keeps its smallest experts.  Ordering a group's experts
    by (count, id), every expert the donor keeps whole comes before every
    expert it gives away whole, and at most one expert is split."""
    R = tk.shape[0]
    G = E // R
    T = np.bincount(tk.reshape(-1), minlength=E)
    rc = p["row_counts"]
    for h in range(R):
        if not any(p["assign"][s, 1] == h for s in range(R)):
            continue
        kept = {e: int(rc[h, e]) for e in range(h * G, (h + 1) * G)}
        whole_kept = [(T[e], e) for e, n in kept.items() if T[e] and n == T[e]]
        whole_given = [(T[e], e) for e, n in kept.items() if T[e] and n == 0]
        split = [e for e, n in kept.items() if 0 < n < T[e]]
        assert len(split) <= 1
        if whole_kept and whole_given:
            assert max(whole_kept) < min(whole_given), (h, whole_kept, whole_given)


def _check_slot_choice(p, E, B, R, by_count):
    """Inference slots: in ascending id; by id (mode 1) they hold the lowest
    ids among the received experts, by count (mode 2) no overflow expert has
    more picks on the rank than a slot expert, and on a tie the slot expert
    has the lower id."""
    G = E // R
    rc, se = p["row_counts"], p["slot_expert"]
    for r in range(R):
        slots = [int(e) for e in se[r] if e >= 0]
        assert slots == sorted(slots)
        got = {e: int(rc[r, E + b]) for b, e in enumerate(slots)}
        ovf = {e: int(rc[r, e]) for e in range(E) if e // G != r and rc[r, e] > 0}
        for e, n in got.items():
            for f, m in ovf.items():
                if by_count:
                    assert n > m or (n == m and e < f), (r, e, n, f, m)
                else:
                    assert e < f


def test_inference_slots_by_count_and_by_id():
    # training-shape inference at maxvio 4: ranks receive more distinct
    # experts than B = 4, so the two rules must pick differently somewhere
    tk, mv, _ = synth.routing(8, 4096, 8, 256, 4.0, "hot8", 0)
    p1 = oracle.plan(tk, 256, 4, 128, 1)
    p2 = oracle.plan(tk, 256, 4, 128, 2)
    for p, by_count in ((p1, False), (p2, True)):
        assert p["status"] == 0
        check_plan(tk, p, 256, 4, 128, 1)
        _check_slot_choice(p, 256, 4, 8, by_count)
    assert not np.array_equal(p1["slot_expert"], p2["slot_expert"])
    # the per-expert totals and the alias chain do not depend on the rule
    assert np.array_equal(p1["assign"], p2["assign"]) and np.array_equal(p1["counts"], p2["counts"])
    # with enough slots for every received expert the two rules coincide
    q1 = oracle.plan(tk, 256, 32, 128, 1)
    q2 = oracle.plan(tk, 256, 32, 128, 2)
    for k in ("dst", "cu_seqlens", "row_counts", "slot_expert"):
        assert np.array_equal(q1[k], q2[k]), k


@pytest.mark.parametrize("rank1,slot1,slot2", [
    # e2 and e3 each give 2 picks: both rules take e2 (a tie goes to the lower id)
    ([2, 2, 3, 3, 4, 5, 6, 7], 2, 2),
    # e2 gives 1 pick, e3 gives 3: by id e2, by count e3
    ([2, 3, 3, 3, 4, 5, 6, 7], 2, 3),
])
def test_inference_slot_choice_worked_example(rank1, slot1, slot2):
    # Worked by hand.  R=2, E=8 (G=4), S=8, K=1, B=1, token_padding=1.
    # Rank 0 picks e0 x4, e1 x4; rank 1 picks rank1.  Group 0's sequence is
    # e0[0,4) e1[4,8) then e2, e3: L_0 = 12, L_1 = 4, C = 8, so rank 1 takes
    # the last 4 picks of group 0, i.e. all of e2's and e3's.  With one slot,
    # the expert not taken stays on rank 1's overflow home row.
    tk = np.array([[0] * 4 + [1] * 4, rank1], np.int32).reshape(2, 8, 1)
    n2, n3 = rank1.count(2), rank1.count(3)
    for mode, slot in ((1, slot1), (2, slot2)):
        p = oracle.plan(tk, 8, 1, 1, mode)
        assert p["status"] == 0
        assert p["assign"].tolist() == [[8, -1, 0, 0], [4, 0, 8, 4]]
        assert p["slot_expert"].tolist() == [[-1], [slot]]
        ovf = 5 - slot  # the other of e2, e3
        want = [0] * 9
        want[ovf] = n2 if ovf == 2 else n3
        want[4:8] = [1, 1, 1, 1]
        want[8] = n2 if slot == 2 else n3
        assert p["row_counts"][1].tolist() == want
        assert p["row_counts"][0].tolist() == [4, 4, 0, 0, 0, 0, 0, 0, 0]


# ------------------------------------------------ special cases: stable sort
def _sorted_layout(tk, E, B, tp, h, G):
    """Where rank h's picks go when no copies are made: a stable argsort by
    expert id over the picks of group h taken in (source rank, token, k) order,
    each row padded to tp, rows in expert order."""
    R = tk.shape[0]
    flat_idx = np.arange(tk.size).reshape(tk.shape)
    mine = (tk // G) == h
    ids = flat_idx[mine]  # (r, t, k) order
    ex = tk[mine]
    order = np.argsort(ex, kind="stable")
    want = {}
    counts = np.bincount(ex, minlength=E)
    padded = np.where(counts > 0, -(-counts // tp) * tp, 0)
    starts = np.concatenate([[0], np.cumsum(padded)[:-1]])
    seen = np.zeros(E, np.int64)
    for j in order:
        e = ex[j]
        want[int(ids[j])] = int(starts[e] + seen[e])
        seen[e] += 1
    return want


@pytest.mark.parametrize("mode", [0, 3])
@pytest.mark.parametrize("R,S,K,E,tp", [(8, 1024, 8, 64, 128), (4, 96, 4, 16, 8), (2, 64, 2, 8, 1)])
def test_balanced_plan_is_stable_argsort(R, S, K, E, tp, mode):
    tk, mv, _ = synth.routing(R, S, K, E, 0.0, seed=5)
    G = E // R
    p = oracle.plan(tk, E, G, tp, mode)
    assert p["status"] == 0 and copies_of(p, E, G, R) == 0
    assert np.all(p["assign"][:, 1] == -1)
    flat = p["dst"].reshape(-1)
    for h in range(R):
        for i, pos in _sorted_layout(tk, E, G, tp, h, G).items():
            assert flat[i] == h * p["nvs"] + pos


def test_single_rank_plan_is_stable_argsort():
    tk, mv, _ = synth.routing(1, 500, 4, 16, 2.0, "zipf", seed=2)
    p = oracle.plan(tk, 16, 16, 4)
    assert p["status"] == 0
    flat = p["dst"].reshape(-1)
    for i, pos in _sorted_layout(tk, 16, 16, 4, 0, 16).items():
        assert flat[i] == pos


# ------------------------------------------------------- dispatch / combine
def _problem(R=4, S=96, K=4, E=16, B=4, H=64, tp=8, mode=0, mv=1.5, seed=1):
    tk, _, _ = synth.routing(R, S, K, E, mv, "hot8", seed=seed)
    p = oracle.plan(tk, E, B, tp, mode)
    assert p["status"] == 0
    x = synth.hidden_bf16(R, S, H, seed)
    w = synth.route_weights(R, S, K, seed)
    return tk, p, x, w


def test_dispatch_places_rows_and_leaves_padding():
    tk, p, x, w = _problem()
    xb = synth.bf16_bits(x)
    buf, w_nvs = oracle.dispatch(p["dst"], xb, w, p["nvs"])
    R, S, K = tk.shape
    hit = np.zeros(buf.shape[0], bool)
    for r in range(R):
        for t in range(S):
            for k in range(K):
                d = p["dst"][r, t, k]
                assert np.array_equal(buf[d], xb[r, t])
                assert w_nvs[d] == w[r, t, k]
                hit[d] = True
    assert np.all(buf[~hit] == 0xFFFF) and np.all(np.isnan(w_nvs[~hit]))
    assert hit.sum() == R * S * K


def test_roundtrip_unweighted_is_K_times_x():
    # the K copies of x summed in any precision >= fp32 are exactly K*x, and
    # K*x is a bf16 value for K a power of two
    for K in (2, 4, 8):
        tk, p, x, w = _problem(K=K, E=32, B=8, mv=1.0)
        xb = synth.bf16_bits(x)
        buf, _ = oracle.dispatch(p["dst"], xb, None, p["nvs"])
        out, _ = oracle.combine(p["dst"], buf, None)
        # the sum starts from +0, so x = -0 gives +0 (adding 0.0 does the same)
        want = (x.to(torch.float32) * K + 0.0).to(torch.bfloat16)
        assert np.array_equal(out, synth.bf16_bits(want))


def test_roundtrip_softmax_weights_is_identity():
    # sum_k w_k = 1 within a few fp32 ulps, far inside bf16's half-ulp
    tk, p, x, w = _problem(K=8, E=32, B=8)
    xb = synth.bf16_bits(x)
    buf, w_nvs = oracle.dispatch(p["dst"], xb, w, p["nvs"])
    out, gw = oracle.combine(p["dst"], buf, w_nvs)
    assert np.array_equal(out, synth.bf16_bits((x.to(torch.float32) + 0.0).to(torch.bfloat16)))
    assert np.array_equal(gw, w)


def _row_expert(p, E, B, R):
    """Expert whose weights serve each buffer row (-1 for padding)."""
    nvs = p["nvs"]
    ex = np.full(R * nvs, -1, np.int64)
    for r in range(R):
        prev = 0
        for i in range(E + B):
            n = p["row_counts"][r, i]
            if n:
                e = i if i < E else p["slot_expert"][r, i - E]
                ex[r * nvs + prev: r * nvs + prev + n] = e
            prev = p["cu_seqlens"][r, i]
    return ex


def test_combine_pairs_weights_with_their_experts():
    # a diagonal "expert" scales its rows by a_e (a signed power of two,
    # so its bf16 output is exact): by linearity combine gives
    # (sum_k w_k * a_{e_k}) * x, exact in fp32 when the weights are short
    # dyadic numbers, so fp32 -> bf16 (torch) is the one rounding.
    R, S, K, E, B, H, tp = 4, 96, 4, 16, 4, 64, 8
    tk, p, x, _ = _problem(R, S, K, E, B, H, tp)
    g = np.random.default_rng(7)
    w = (g.integers(1, 16, (R, S, K)) / 8.0).astype(np.float32)
    a = g.choice([0.5, -0.5, 1.0, -1.0, 2.0, -2.0, 4.0], size=E)
    xb = synth.bf16_bits(x)
    buf, w_nvs = oracle.dispatch(p["dst"], xb, w, p["nvs"])
    rows_e = _row_expert(p, E, B, R)
    y = bf16_to_f64(buf)
    live = rows_e >= 0
    y[live] *= a[rows_e[live]][:, None]
    y[~live] = 0.0
    ybits = synth.bf16_bits(torch.from_numpy(y.astype(np.float32)).to(torch.bfloat16))
    out, gw = oracle.combine(p["dst"], ybits, w_nvs)
    scale = (w.astype(np.float64) * a[tk]).sum(-1)
    want = torch.from_numpy((x.double().numpy() * scale[..., None]).astype(np.float32)).to(torch.bfloat16)
    # compared as values: a sum that cancels to zero is +0, x * 0 may be -0
    assert np.array_equal(bf16_to_f64(out), want.double().numpy())
    assert np.array_equal(gw, w)


# ------------------------------------------------------- prefetch / grads
def test_prefetch_copies_slots_only():
    tk, p, _, _ = _problem(E=16, B=4, mv=3.0)
    E, R, B = 16, 4, 4
    HHp = 48
    W = synth.bf16_bits(torch.from_numpy(synth.normal_f32((E, HHp), 3)).to(torch.bfloat16)).copy()
    pool = np.full((R * B, HHp), 0x7F7F, np.uint16)
    oracle.prefetch(p["slot_expert"], W, pool)
    se = p["slot_expert"].reshape(-1)
    assert (se >= 0).any()
    for s, e in enumerate(se):
        if e >= 0:
            assert np.array_equal(pool[s], W[e])
        else:
            assert np.all(pool[s] == 0x7F7F)


def test_reduce_grad_powers_of_two_identify_slots():
    # G = 0 and slot s holding 2^s: the fp32 result names exactly the slots
    # that were added into each expert (all sums are exact).
    tk, p, _, _ = _problem(R=4, E=16, B=4, mv=3.0)
    R, B, E = 4, 4, 16
    se = p["slot_expert"]
    nslot = R * B
    G = np.zeros((E, 3), np.float32)
    RB = np.array([[2.0 ** s] * 3 for s in range(nslot)], np.float32)
    oracle.reduce_grad(se, G, RB)
    flat = se.reshape(-1)
    for e in range(E):
        want = sum(2.0 ** s for s in range(nslot) if flat[s] == e)
        assert np.all(G[e] == want)
    for s in range(nslot):
        assert np.all(RB[s] == (0.0 if flat[s] >= 0 else 2.0 ** s))
        if flat[s] >= 0:
            assert not np.signbit(RB[s]).any()


def test_reduce_grad_constant_slots():
    tk, p, _, _ = _problem(R=4, E=16, B=4, mv=3.0)
    R, B, E = 4, 4, 16
    G = np.full((E, 5), 1.5, np.float32)
    RB = np.full((R * B, 5), 0.25, np.float32)
    oracle.reduce_grad(p["slot_expert"], G, RB)
    copies = np.bincount(p["slot_expert"][p["slot_expert"] >= 0], minlength=E)
    assert np.array_equal(G[:, 0], 1.5 + 0.25 * copies)


# ------------------------------------------------------------- errors
def test_errors_set_status_bits():
    tk, _, _ = synth.routing(2, 16, 2, 8, 0.0)
    bad = tk.copy(); bad[1, 3, 1] = 8
    assert oracle.plan(bad, 8, 4, 4)["status"] == oracle.STATUS_BAD_EXPERT
    bad = tk.copy(); bad[0, 0, 0] = -1
    assert oracle.plan(bad, 8, 4, 4)["status"] == oracle.STATUS_BAD_EXPERT
    bad = tk.copy(); bad[0, 5, 1] = bad[0, 5, 0]
    assert oracle.plan(bad, 8, 4, 4)["status"] == oracle.STATUS_DUP_EXPERT
    tpe = synth.local_counts(tk, 8); tpe[1, 2] += 1
    assert oracle.plan(tk, 8, 4, 4, 0, tpe)["status"] == oracle.STATUS_COUNT_MISMATCH
    assert oracle.plan(tk, 8, 3, 4, 0)["status"] == oracle.STATUS_BAD_ARGS  # training needs B >= E/R
    assert oracle.plan(tk, 8, 3, 4, 1)["status"] == 0


# ------------------------------------------------------------ brute force
def _feasible_transfers(L, C):
    """All group-level plans: X[h][s] picks of group h served by rank s, with
    every rank serving exactly C and each rank taking from at most one remote
    group.  Exhaustive over the donor choice of each rank."""
    R = len(L)
    out = []
    for donors in itertools.product(range(-1, R), repeat=R):
        if any(d == s for s, d in enumerate(donors)):
            continue
        # rank s keeps k_s of its own group and takes C - k_s from donors[s]
        # (0 if none); group h's picks are kept plus given away.
        # Solve: k_s + take_s = C, take_s = 0 if donor -1;
        #        k_h + sum_{s: donors[s]=h} take_s = L_h
        # unknowns take_s for ranks with a donor; k_s = C - take_s.
        ok = True
        take = [0] * R
        # iterate: k_h = L_h - given_h, and take_h = C - k_h
        # => take_h = C - L_h + sum_{s: donors[s] = h} take_s (a tree recursion)
        def solve(h, seen):
            if h in seen:
                raise ValueError
            seen = seen | {h}
            return C - L[h] + sum(solve(s, seen) for s in range(R) if donors[s] == h)
        try:
            for s in range(R):
                take[s] = solve(s, frozenset())
        except (ValueError, RecursionError):
            continue
        for s in range(R):
            if donors[s] == -1 and take[s] != 0:
                ok = False
            if donors[s] != -1 and take[s] <= 0:
                ok = False
            if C - take[s] < 0 or C - take[s] > L[s]:
                ok = False
        if ok:
            out.append((donors, take))
    return out


@pytest.mark.parametrize("R,C", [(2, 3), (3, 2), (3, 4), (4, 2)])
def test_bruteforce_group_plans_always_exist_and_rule_is_one(R, C):
    # every load vector with sum R*C admits a plan with <= 1 donor per rank
    # (the alias construction's guarantee); the oracle's plan is one of them
    # and never uses more donations than R-1.
    G, K = 1, 1
    E = R * G
    S = C
    total = R * C
    for L in itertools.product(range(total + 1), repeat=R):
        if sum(L) != total or max(L) > R * S:
            continue
        plans = _feasible_transfers(list(L), C)
        assert plans, f"no plan for loads {L}"
        # routing realising the loads: expert h picked L_h times, spread over ranks
        picks = np.repeat(np.arange(E, dtype=np.int32), L)
        tk = picks.reshape(R, S, K)
        p = oracle.plan(tk, E, G, 1)
        assert p["status"] == 0
        check_plan(tk, p, E, G, 1, 0)
        donors = tuple(int(d) for d in p["assign"][:, 1])
        take = [int(p["assign"][s, 3]) for s in range(R)]
        assert (donors, take) in [(tuple(d), t) for d, t in plans]
        assert sum(d >= 0 for d in donors) <= R - 1
        assert sum(d >= 0 for d in donors) >= min(sum(x >= 0 for x in d) for d, _ in plans)


def _min_copies_bruteforce(tk, E, R):
    """Fewest (expert, remote rank) copies over every assignment of picks to
    ranks that gives each rank S*K picks with at most one remote group."""
    G = E // R
    picks = tk.reshape(-1)
    C = tk.shape[1] * tk.shape[2]
    best = None
    for assign in itertools.product(range(R), repeat=picks.size):
        a = np.array(assign)
        if np.any(np.bincount(a, minlength=R) != C):
            continue
        ok = True
        copies = 0
        for s in range(R):
            remote = {int(e) for e in picks[a == s] if e // G != s}
            if len({e // G for e in remote}) > 1:
                ok = False
                break
            copies += len(remote)
        if ok and (best is None or copies < best):
            best = copies
    return best


def test_bruteforce_min_copies_tiny():
    # R=2, E=4, S=3, K=1: every routing.  The rule always finds a plan; the
    # gap to the fewest possible copies is measured, not bounded by the pages.
    R, E, S, K = 2, 4, 3, 1
    gaps = []
    for picks in itertools.product(range(E), repeat=R * S * K):
        tk = np.array(picks, np.int32).reshape(R, S, K)
        p = oracle.plan(tk, E, E // R, 1)
        assert p["status"] == 0
        best = _min_copies_bruteforce(tk, E, R)
        assert best is not None
        mine = copies_of(p, E, E // R, R)
        assert mine >= best
        gaps.append(mine - best)
    gaps = np.array(gaps)
    assert gaps.max() <= 1  # observed on this tiny space; reported, not a page claim


def test_fewest_copies_mode_reaches_the_bruteforce_minimum_tiny():
    # R=2, E=4, S=3, K=1, every routing: with one donor and one recipient,
    # giving away the largest experts first covers the deficit with the
    # fewest experts, so mode 3's copy count is the brute-force minimum
    R, E, S, K = 2, 4, 3, 1
    for picks in itertools.product(range(E), repeat=R * S * K):
        tk = np.array(picks, np.int32).reshape(R, S, K)
        p = oracle.plan(tk, E, E // R, 1, 3)
        assert p["status"] == 0
        check_plan(tk, p, E, E // R, 1, 3)
        assert copies_of(p, E, E // R, R) == _min_copies_bruteforce(tk, E, R), picks


def test_fewest_copies_mode_with_equal_counts_is_the_id_order():
    # within each group all experts have one count: the count order is the id
    # order (ties by id), so mode 3 plans exactly as mode 0
    R, S, K, E = 2, 8, 1, 4
    # T = [3, 3, 5, 5]: group 0 under-loaded (6), group 1 over-loaded (10)
    picks = [0, 0, 0, 1, 1, 1, 2, 2, 2, 2, 2, 3, 3, 3, 3, 3]
    tk = np.array(picks, np.int32).reshape(R, S, K)
    a, b = oracle.plan(tk, E, 2, 2, 0), oracle.plan(tk, E, 2, 2, 3)
    assert a["status"] == b["status"] == 0
    assert np.any(a["assign"][:, 1] >= 0), "the case must donate"
    for k in ("dst", "cu_seqlens", "row_counts", "slot_expert", "assign"):
        assert np.array_equal(a[k], b[k]), k


def test_fewest_copies_mode_never_copies_more_with_one_donor_per_recipient_pair():
    # where the alias chain makes a single donation (R=2), mode 3 never makes
    # more copies than mode 0; across larger groups its count is reported
    for seed in range(40):
        tk, _, _ = synth.routing(2, 64, 4, 16, 0.5 + 0.5 * (seed % 5), "hot8", seed=seed)
        a, b = oracle.plan(tk, 16, 8, 4, 0), oracle.plan(tk, 16, 8, 4, 3)
        assert copies_of(b, 16, 8, 2) <= copies_of(a, 16, 8, 2)


# ------------------------------------------------ one rank's share of the plan
@pytest.mark.parametrize("R,S,K,E,B,tp,mode,mv,profile", [
    (8, 1024, 8, 64, 8, 128, 0, 2.0, "zipf"),
    (8, 1024, 8, 64, 8, 128, 0, 0.0, "hot8"),
    (3, 1000, 3, 24, 8, 16, 0, 1.5, "hot8"),
    (4, 333, 3, 24, 0, 16, 1, 1.5, "hot8"),
    (8, 512, 8, 64, 2, 128, 1, 4.0, "hot8"),
    (8, 512, 8, 64, 2, 128, 2, 4.0, "hot8"),
    (2, 100, 32, 64, 32, 4, 0, 0.5, "zipf"),
    (16, 64, 4, 64, 4, 8, 0, 6.0, "hot8"),
    (8, 1024, 8, 64, 8, 128, 3, 2.0, "zipf"),
    (3, 1000, 3, 24, 8, 16, 3, 1.5, "hot8"),
])
def test_rank_share_is_the_slice_of_the_group_plan(R, S, K, E, B, tp, mode, mv, profile):
    # The group plan walks every group sequence with all ranks' picks; a
    # rank's share places its own picks from the counts in closed form.  The
    # two must agree on every rank, which is what lets each rank of a real
    # group plan for itself after one all-gather of the counts.
    tk, _, _ = synth.routing(R, S, K, E, mv, profile, seed=17)
    cnt = synth.local_counts(tk, E)
    want = oracle.plan(tk, E, B, tp, mode, cnt)
    assert want["status"] == 0
    for r in range(R):
        got = oracle.plan_rank(tk[r], cnt, r, E, B, tp, mode)
        assert got["status"] == 0
        assert np.array_equal(got["dst"], want["dst"][r]), r
        for k in ("cu_seqlens", "row_counts", "slot_expert", "assign"):
            assert np.array_equal(got[k], want[k]), (r, k)
        assert np.float32(got["maxvio"]) == np.float32(want["maxvio"])


def test_rank_share_refuses_inconsistent_counts():
    R, S, K, E, B, tp = 4, 64, 4, 16, 4, 8
    tk, _, _ = synth.routing(R, S, K, E, 1.0, "hot8", seed=18)
    cnt = synth.local_counts(tk, E)
    moved = cnt.copy()
    e0, e1 = int(np.argmax(moved[1])), int(np.argmin(moved[1]))
    moved[1, e0] -= 1
    moved[1, e1] += 1
    assert oracle.plan_rank(tk[1], moved, 1, E, B, tp)["status"] == oracle.STATUS_COUNT_MISMATCH
    assert oracle.plan_rank(tk[0], moved, 0, E, B, tp)["status"] == 0  # rank 0 sees only its own row
    short = cnt.copy()
    short[2, int(np.argmax(short[2]))] -= 1
    assert oracle.plan_rank(tk[0], short, 0, E, B, tp)["status"] == oracle.STATUS_COUNT_MISMATCH
    bad = tk[3].copy()
    bad[0, 0] = E
    assert oracle.plan_rank(bad, cnt, 3, E, B, tp)["status"] & oracle.STATUS_BAD_EXPERT
    assert oracle.plan_rank(tk[0], cnt, R, E, B, tp)["status"] == oracle.STATUS_BAD_ARGS
