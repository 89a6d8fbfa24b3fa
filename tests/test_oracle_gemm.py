"""Pins of the group-GEMM oracle (MoonEP README, "Integration", "Weight
buffer") against what the plan and the routing fix independently of it:
every pick's slot lies in a segment that uses the pick's own expert, the
segments cover exactly S*K slots per rank, diagonal experts scale rows by
their expert's factor, and slot rows read the rank's pool, not the home
weights."""
import numpy as np

import oracle
from load_balancing_planner_b200 import synth


def _plan(R=4, S=96, K=4, E=16, B=4, tp=16, mode=0, mv=1.5, seed=3, profile="zipf"):
    tk, _, _ = synth.routing(R, S, K, E, mv, profile, seed=seed)
    return tk, oracle.plan(tk, E, B, tp, mode)


def _expert_of_slot(p, tk, R, nvs):
    ex = np.full(R * nvs, -1)
    ex[p["dst"].ravel()] = tk.ravel()
    return ex


def test_segments_hold_each_pick_under_its_own_expert():
    for mode, B, mv in ((0, 4, 1.5), (1, 1, 3.0), (0, 4, 0.0)):
        R, S, K, E, tp = 4, 96, 4, 16, 16
        tk, p = _plan(R, S, K, E, B, tp, mode, mv)
        assert p["status"] == 0
        nvs = p["nvs"]
        segs = oracle.segments(p["cu_seqlens"], p["row_counts"], E, tp)
        ex = _expert_of_slot(p, tk, R, nvs)
        covered = np.zeros(R * nvs, int)
        per_rank = np.zeros(R, int)
        for r, s0, n, i in segs:
            assert s0 % tp == 0 and 0 <= s0 and s0 + n <= nvs
            e = i if i < E else p["slot_expert"][r, i - E]
            assert (ex[r * nvs + s0: r * nvs + s0 + n] == e).all()
            covered[r * nvs + s0: r * nvs + s0 + n] += 1
            per_rank[r] += n
        assert (per_rank == S * K).all()
        assert covered.max() == 1 and covered.sum() == R * S * K
        assert (covered[p["dst"].ravel()] == 1).all()


def _bits(a):
    import torch
    return synth.bf16_bits(torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16))


def test_diagonal_experts_scale_rows_and_slots_read_the_pool():
    R, S, K, E, B, tp, H = 4, 96, 4, 16, 4, 16, 8
    tk, p = _plan(R, S, K, E, B, tp)
    nvs = p["nvs"]
    assert (p["slot_expert"] >= 0).any()
    g = np.random.default_rng(0)
    a = g.choice([0.5, -1.0, 2.0, 4.0, -0.25], size=E)
    W = np.stack([a[e] * np.eye(H) for e in range(E)])
    x = g.standard_normal((R * nvs, H))
    xb = _bits(x)
    x64 = (xb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ex = _expert_of_slot(p, tk, R, nvs)
    is_slot_row = np.zeros(R * nvs, bool)
    for r, s0, n, i in oracle.segments(p["cu_seqlens"], p["row_counts"], E, tp):
        is_slot_row[r * nvs + s0: r * nvs + s0 + n] = i >= E
    # the pool holds twice its expert's weights: slot rows must show it
    pool = np.zeros((R * B, H, H))
    for r in range(R):
        for b in range(B):
            e = p["slot_expert"][r, b]
            if e >= 0:
                pool[r * B + b] = 2 * W[e]
    y, mask = oracle.group_gemm(p["cu_seqlens"], p["row_counts"], xb, _bits(W), _bits(pool), E, tp, nvs)
    real = ex >= 0
    assert (mask == real).all()
    scale = np.where(is_slot_row, 2.0, 1.0) * a[np.clip(ex, 0, None)]
    assert np.array_equal(y[real], x64[real] * scale[real, None])
    assert np.isnan(y[~real]).all()


def test_random_weights_match_per_pick_products():
    R, S, K, E, B, tp, H, Hp = 2, 64, 2, 8, 4, 8, 16, 12
    tk, p = _plan(R, S, K, E, B, tp, mv=1.0, seed=5)
    nvs = p["nvs"]
    g = np.random.default_rng(1)
    Wb = _bits(g.standard_normal((E, H, Hp)))
    pool = np.zeros((R * B, H * Hp), np.uint16)
    oracle.prefetch(p["slot_expert"], np.ascontiguousarray(Wb.reshape(E, H * Hp)), pool)
    xb = _bits(g.standard_normal((R * nvs, H)))
    y, mask = oracle.group_gemm(p["cu_seqlens"], p["row_counts"], xb, Wb, pool.reshape(R * B, H, Hp), E, tp, nvs)
    f = lambda b: (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for (r, t, k), d in np.ndenumerate(p["dst"]):
        e = tk[r, t, k]
        want = sum(f(xb[d, j]) * f(Wb[e, j]) for j in range(H))
        assert np.allclose(y[d], want, rtol=1e-12, atol=1e-12)
