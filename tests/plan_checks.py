"""Checks of a plan against what the MoonEP pages fix, written independently
of both the oracle and the CUDA planner.

What is checked (sources are the MoonEP README and the MarkTechPost article):
  * every rank holds exactly S*K real slots ("Perfect balance");
  * every (token, k) pick is placed exactly once, in a real slot of a row
    whose weights are that pick's expert (rows [0,E) are the experts
    themselves, rows [E,E+B) the prefetch slots: "Weight buffer");
  * the rows of an expert on all ranks add up to its global count T_e;
  * a rank's copied experts come from at most one remote home group, and in
    training fit its B slots ("How to set B");
  * rows are padded to token_padding, cu_seqlens is the inclusive running sum
    of padded lengths and stays within NvS ("dispatch fwd", notation of NvS);
  * maxvio = max_e T_e / T_bar - 1 ("Performance").
"""
from __future__ import annotations

import numpy as np


def check_plan(topk, p, E, B, tp, mode, nvs=None):
    topk = np.asarray(topk)
    R, S, K = topk.shape
    G = E // R
    C = S * K
    NR = E + B
    dst = np.asarray(p["dst"]).reshape(R, S, K).astype(np.int64)
    cu = np.asarray(p["cu_seqlens"]).reshape(R, NR).astype(np.int64)
    rc = np.asarray(p["row_counts"]).reshape(R, NR).astype(np.int64)
    se = np.asarray(p["slot_expert"]).reshape(R, B).astype(np.int64)
    NvS = int(nvs if nvs is not None else p["nvs"])

    # counts and maxvio
    T = np.bincount(topk.reshape(-1), minlength=E)
    for r in range(R):
        assert np.array_equal(np.asarray(p["counts"])[r], np.bincount(topk[r].reshape(-1), minlength=E))
    tbar = R * S * K / E
    assert abs(float(p["maxvio"]) - (T.max() / tbar - 1.0)) <= 1e-6 * max(1.0, T.max() / tbar)

    # per-rank balance and padding
    assert np.all(rc >= 0)
    assert np.all(rc.sum(axis=1) == C), "every rank must hold exactly S*K real slots"
    padded = np.where(rc > 0, -(-rc // tp) * tp, 0)
    assert np.array_equal(cu, np.cumsum(padded, axis=1)), "cu_seqlens = inclusive padded ends"
    assert np.all(cu[:, -1] <= NvS)
    start = cu - padded

    # row -> expert of its weights, and which rows may be non-empty
    for r in range(R):
        used = se[r][se[r] >= 0]
        assert np.all(se[r][: used.size] >= 0) and np.all(se[r][used.size:] == -1), "slots fill from 0"
        assert len(set(used.tolist())) == used.size, "an expert takes one slot per rank"
        assert np.all((used // G) != r), "slots hold remote experts only"
        for b in range(B):
            if se[r, b] < 0:
                assert rc[r, E + b] == 0
            else:
                assert rc[r, E + b] > 0, "a used slot holds picks"
        remote_rows = [e for e in range(E) if e // G != r and rc[r, e] > 0]  # overflow rows
        if mode in (0, 3):
            assert not remote_rows, "training never reads a remote home row"
        remote_experts = set(used.tolist()) | set(remote_rows)
        groups = {e // G for e in remote_experts}
        assert len(groups) <= 1, "copies come from at most one remote home group"
        if remote_rows:
            assert used.size == B, "overflow only once all B slots are taken"
        assert len(remote_experts) <= G

    # every pick placed exactly once, inside a real slot of a row of its expert
    flat = dst.reshape(-1)
    assert np.all((flat >= 0) & (flat < R * NvS))
    assert np.unique(flat).size == flat.size, "dst must be injective"
    rank = flat // NvS
    pos = flat % NvS
    e_of = topk.reshape(-1)
    # locate the row of each slot
    row = np.empty_like(flat)
    for r in range(R):
        m = rank == r
        idx = np.searchsorted(cu[r], pos[m], side="right")
        assert np.all(idx < NR)
        row[m] = idx
        assert np.all(pos[m] - start[r, idx] < rc[r, idx]), "dst lands in a real slot, not padding"
    if B:
        w_expert = np.where(row < E, row, se[rank, np.clip(row - E, 0, B - 1)])
    else:
        w_expert = row
    assert np.array_equal(w_expert, e_of), "each pick lands in a row holding its expert's weights"
    # each expert's rows add up to T_e
    tot = np.zeros(E, np.int64)
    for r in range(R):
        for i in range(NR):
            if rc[r, i]:
                e = i if i < E else se[r, i - E]
                tot[e] += rc[r, i]
    assert np.array_equal(tot, T)
    return dict(copies=int(sum((se[r] >= 0).sum() for r in range(R))))


def copies_of(p, E, B, R):
    """Distinct (expert, remote rank) pairs: slot copies plus overflow rows."""
    rc = np.asarray(p["row_counts"]).reshape(R, E + B)
    se = np.asarray(p["slot_expert"]).reshape(R, B)
    G = E // R
    n = 0
    for r in range(R):
        n += int((se[r] >= 0).sum())
        n += sum(1 for e in range(E) if e // G != r and rc[r, e] > 0)
    return n
