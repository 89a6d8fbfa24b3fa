"""Helpers shared by the GPU tests: seeded problems, the CUDA path through the
binding, and the oracle on the same inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from load_balancing_planner_b200 import synth

PLAN_KEYS = ("dst", "cu_seqlens", "row_counts", "slot_expert", "counts", "assign")


def problem(R, S, K, E, mv, profile="hot8", seed=0):
    tk, real, _ = synth.routing(R, S, K, E, mv, profile, seed=seed)
    return tk, synth.local_counts(tk, E), real


def gpu_plan(h, topk, tpe=None):
    from load_balancing_planner_b200 import moonep
    dev = torch.device("cuda:0")
    t = torch.from_numpy(np.ascontiguousarray(topk)).to(dev)
    c = None if tpe is None else torch.from_numpy(np.ascontiguousarray(tpe)).to(dev)
    p = moonep.moonep_plan(h, t, c)
    torch.cuda.synchronize()
    return p


def plan_to_numpy(p):
    out = {k: getattr(p, k).cpu().numpy() for k in PLAN_KEYS}
    out["slot_expert"] = out["slot_expert"][:, : p.B]
    out["maxvio"] = float(p.maxvio.cpu().numpy()[0])
    out["status"] = int(p.status.cpu().numpy()[0])
    out["nvs"] = p.nvs
    return out


def assert_plans_equal(got, want):
    assert got["status"] == want["status"]
    if want["status"]:
        return
    for k in PLAN_KEYS:
        g, w = np.asarray(got[k]), np.asarray(want[k])
        assert g.shape == w.shape, (k, g.shape, w.shape)
        if not np.array_equal(g, w):
            bad = np.argwhere(g != w)
            raise AssertionError(f"{k}: {len(bad)} mismatches, first at {bad[0].tolist()}: "
                                 f"got {g[tuple(bad[0])]} want {w[tuple(bad[0])]}")
    assert np.float32(got["maxvio"]) == np.float32(want["maxvio"])
    assert got["nvs"] == want["nvs"]


def bf16_dev(bits_or_tensor):
    if isinstance(bits_or_tensor, np.ndarray):
        return torch.from_numpy(bits_or_tensor.view(np.int16)).view(torch.bfloat16).cuda()
    return bits_or_tensor.cuda()


def bits(t):
    """uint16 bit patterns of a bf16 tensor (any device)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
