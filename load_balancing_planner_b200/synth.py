"""Seeded synthetic inputs for the balanced expert-parallel hot path.

This module draws what a MoE router and the layer before it would hand to
``dispatch``: top-K expert picks per token at a controlled imbalance, the fp32
route weights of those picks, the local per-expert counts, and bf16 hidden rows.
It is shared by the tests, ``bench.py`` and the CPU oracle's callers, and it
holds none of the planner's, dispatch's or combine's arithmetic.  The one
quantity it measures is the realised imbalance of the routing it draws
(largest per-expert count over the count under perfect balance), which it
needs to hit a requested target; the definition of that imbalance ("maxvio")
is from the MoonEP README, section "Performance".

Recipe (every draw uses numpy's PCG64, seeded with ``[seed, stream]``):

* hidden rows: N(0, 1) in fp32, rounded to bf16 (round to nearest even).
* route weights: softmax, in fp64 then rounded to fp32, of N(0, 1) logits over
  each token's K picks.
* routing, maxvio = 0: consecutive blocks of E/K tokens (over all ranks) each
  take a fresh random permutation of the E experts, cut into K-sized picks, so
  every expert receives exactly R*S*K/E picks.
* routing, maxvio > 0: K experts drawn per token without replacement from a
  distribution p_e, by Gumbel-top-K over log p_e (equivalent to drawing one
  after the other without replacement).  p_e has one free parameter that is
  bisected on the realised imbalance (same Gumbel noise every time) until it
  is within ``tol`` of the target:

  - ``"boost0"``: uniform, expert 0 weighted by beta;
  - ``"zipf"``: p_e proportional to (e+1)^-s, expert 0 hottest;
  - ``"hot8"``: uniform, experts 0..7 weighted by beta.

  The hot experts sit in the first home group, the worst case for one rank.
"""
from __future__ import annotations

import functools

import numpy as np

# streams of the per-seed generator
_ROUTE, _HIDDEN, _WEIGHTS, _NOISE, _AUX = range(5)


def rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([int(seed), int(stream)]))


def realised_maxvio(topk: np.ndarray, E: int) -> float:
    """max_e(T_e / T_bar) - 1 of a routing, T_bar = picks / E."""
    counts = np.bincount(np.asarray(topk).reshape(-1), minlength=E)
    tbar = topk.size / E
    return float(counts.max() / tbar - 1.0)


def local_counts(topk: np.ndarray, E: int) -> np.ndarray:
    """Per-rank per-expert pick counts [R, E] int32 (the router's local count)."""
    R = topk.shape[0]
    out = np.zeros((R, E), dtype=np.int32)
    for r in range(R):
        out[r] = np.bincount(topk[r].reshape(-1), minlength=E)
    return out


def balanced_topk(R: int, S: int, K: int, E: int, seed: int) -> np.ndarray:
    """Routing with every expert picked exactly R*S*K/E times (maxvio = 0)."""
    if E % K or (R * S) % (E // K):
        raise ValueError("exact balance needs K | E and (E/K) | R*S")
    g = rng(seed, _ROUTE)
    nblk = R * S // (E // K)
    perms = np.argsort(g.random((nblk, E)), axis=1, kind="stable")
    return perms.reshape(R, S, K).astype(np.int32)


def _logp(profile: str, E: int, param: float) -> np.ndarray:
    lp = np.zeros(E, dtype=np.float64)
    if profile == "boost0":
        lp[0] = param  # param = log beta
    elif profile == "hot8":
        lp[: min(8, E)] = param
    elif profile == "zipf":
        lp = -param * np.log(np.arange(1, E + 1, dtype=np.float64))
    else:
        raise ValueError(f"unknown routing profile {profile!r}")
    return lp


def _gumbel_topk(lp: np.ndarray, noise: np.ndarray, K: int) -> np.ndarray:
    scores = noise + lp[None, :].astype(noise.dtype)
    idx = np.argpartition(-scores, K - 1, axis=1)[:, :K]
    s = np.take_along_axis(scores, idx, 1)
    order = np.argsort(-s, axis=1, kind="stable")  # descending score, like a router's top-k
    return np.take_along_axis(idx, order, 1)


@functools.lru_cache(maxsize=64)
def _skewed(R, S, K, E, target, profile, seed, tol):
    g = rng(seed, _NOISE)
    u = g.random((R * S, E), dtype=np.float32)
    noise = -np.log(-np.log(np.clip(u, 1e-30, 1.0 - 1e-7)))
    hi_cap = E / K - 1.0
    if target > hi_cap + 1e-9:
        raise ValueError(f"maxvio {target} unreachable: the largest is E/K-1 = {hi_cap}")

    def draw(param):
        tk = _gumbel_topk(_logp(profile, E, param), noise, K)
        return tk, realised_maxvio(tk, E)

    lo, hi = 0.0, 1.0
    tk, mv = draw(hi)
    while mv < target and hi < 64.0:
        lo, hi = hi, hi * 2.0
        tk, mv = draw(hi)
    best = (abs(mv - target), hi, tk, mv)
    for _ in range(48):
        mid = 0.5 * (lo + hi)
        tk, mv = draw(mid)
        if abs(mv - target) < best[0]:
            best = (abs(mv - target), mid, tk, mv)
        if abs(mv - target) <= tol:
            break
        if mv < target:
            lo = mid
        else:
            hi = mid
    _, param, tk, mv = best
    return tk.reshape(R, S, K).astype(np.int32), float(mv), float(param)


def routing(R: int, S: int, K: int, E: int, maxvio: float, profile: str = "hot8",
            seed: int = 0, tol: float = 0.05):
    """Top-K picks [R, S, K] int32 at a realised imbalance within ``tol`` of ``maxvio``.

    Returns ``(topk, realised_maxvio, param)``; ``param`` is the profile's
    parameter (log beta, or the Zipf exponent), NaN for exact balance.
    """
    if maxvio == 0.0:
        tk = balanced_topk(R, S, K, E, seed)
        return tk, realised_maxvio(tk, E), float("nan")
    tk, mv, p = _skewed(R, S, K, E, float(maxvio), profile, int(seed), float(tol))
    return tk.copy(), mv, p


def route_weights(R: int, S: int, K: int, seed: int = 0) -> np.ndarray:
    """fp32 softmax of N(0,1) logits over each token's K picks, [R, S, K]."""
    g = rng(seed, _WEIGHTS)
    lg = g.standard_normal((R, S, K))
    lg -= lg.max(axis=-1, keepdims=True)
    ex = np.exp(lg)
    return (ex / ex.sum(axis=-1, keepdims=True)).astype(np.float32)


def normal_f32(shape, seed: int = 0, stream: int = _HIDDEN, scale: float = 1.0) -> np.ndarray:
    g = rng(seed, stream)
    x = g.standard_normal(shape, dtype=np.float32)
    if scale != 1.0:
        x *= np.float32(scale)
    return x


def hidden_bf16(R: int, S: int, H: int, seed: int = 0):
    """bf16 hidden rows [R, S, H] ~ N(0, 1) as a CPU torch tensor."""
    import torch
    return torch.from_numpy(normal_f32((R, S, H), seed, _HIDDEN)).to(torch.bfloat16)


def bf16_bits(t) -> np.ndarray:
    """uint16 bit patterns of a CPU bf16 torch tensor (no copy)."""
    import torch
    assert t.dtype == torch.bfloat16 and t.device.type == "cpu"
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


CONFIGS = {
    # name: shapes; the routing sweep is given next to each
    "tiny": dict(R=2, S=64, K=2, E=8, B=4, H=128, tp=8, mode=0,
                 profile="boost0", maxvio=(1.0,)),
    "zipf": dict(R=8, S=1024, K=8, E=64, B=8, H=2048, tp=128, mode=0,
                 profile="zipf", maxvio=(0.0, 0.5, 1.0, 2.0)),
    "train": dict(R=8, S=4096, K=8, E=256, B=32, H=7168, tp=128, mode=0,
                  profile="hot8", maxvio=(0.0, 0.5, 1.0, 2.0, 4.0)),
    "infer": dict(R=8, S=4096, K=8, E=256, B=4, H=7168, tp=128, mode=1, Hp=2048,
                  profile="hot8", maxvio=(1.0, 4.0)),
    "grad": dict(R=8, S=4096, K=8, E=256, B=32, H=7168, tp=128, mode=0, Hp=2048,
                 profile="hot8", maxvio=(2.0,)),
}

