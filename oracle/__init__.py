"""ctypes handle on the CPU oracle in ``moonep_oracle.c``.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the library.  It shares no
code with the CUDA path.  Arrays cross as numpy buffers; bf16 data crosses as
its uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moonep_oracle.c")
LIB = os.path.join(HERE, "libmoonep_oracle.so")
CFLAGS = ["-O2", "-ffp-contract=off", "-std=c99", "-Wall", "-Wextra", "-fPIC", "-shared"]

STATUS_BAD_EXPERT = 1
STATUS_DUP_EXPERT = 2
STATUS_COUNT_MISMATCH = 4
STATUS_BAD_ARGS = 256

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (single-threaded, no FP contraction)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, SRC, "-lm"], check=True)
        os.replace(tmp, LIB)
    return LIB


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i, i64 = ctypes.c_int, ctypes.c_int64
        L.oracle_nvs.argtypes = [i, i, i, i, i]
        L.oracle_nvs.restype = i64
        L.oracle_double_to_bf16.argtypes = [ctypes.c_double]
        L.oracle_double_to_bf16.restype = ctypes.c_uint16
        L.oracle_plan.argtypes = [i, i, i, i, i, i, i, P, P, P, P, P, P, P, P, P]
        L.oracle_plan.restype = i
        L.oracle_plan_rank.argtypes = [i, i, i, i, i, i, i, i, P, P, P, P, P, P, P, P]
        L.oracle_plan_rank.restype = i
        L.oracle_dispatch.argtypes = [i, i, i, i, P, P, P, P, P]
        L.oracle_dispatch.restype = None
        L.oracle_combine.argtypes = [i, i, i, i, P, P, P, P, P]
        L.oracle_combine.restype = None
        L.oracle_prefetch.argtypes = [i, i, i64, P, P, P]
        L.oracle_prefetch.restype = None
        L.oracle_reduce_grad.argtypes = [i, i, i, i64, P, P, P]
        L.oracle_reduce_grad.restype = None
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def nvs(S: int, K: int, E: int, R: int, tp: int) -> int:
    return int(lib().oracle_nvs(S, K, E, R, tp))


def double_to_bf16(x) -> np.ndarray:
    """Round fp64 values to bf16 bit patterns (nearest, ties to even)."""
    f = lib().oracle_double_to_bf16
    x = np.asarray(x, dtype=np.float64)
    return np.array([f(float(v)) for v in x.reshape(-1)], dtype=np.uint16).reshape(x.shape)


def plan(topk, E: int, B: int, tp: int, mode: int = 0, tpe=None) -> dict:
    """Run the planning rule.  ``topk`` is [R, S, K] int32."""
    topk = _c(topk, np.int32)
    R, S, K = topk.shape
    NR = E + B
    out = dict(
        dst=np.full((R, S, K), -1, np.int32),
        cu_seqlens=np.zeros((R, NR), np.int32),
        row_counts=np.zeros((R, NR), np.int32),
        slot_expert=np.full((R, max(B, 0)), -1, np.int32),
        counts=np.zeros((R, E), np.int32),
        maxvio=np.zeros(1, np.float32),
        assign=np.zeros((R, 4), np.int32),
    )
    tpe_a = None if tpe is None else _c(tpe, np.int32)
    st = lib().oracle_plan(R, S, K, E, B, tp, mode, _p(topk), _p(tpe_a),
                           _p(out["dst"]), _p(out["cu_seqlens"]), _p(out["row_counts"]),
                           _p(out["slot_expert"]), _p(out["counts"]), _p(out["maxvio"]),
                           _p(out["assign"]))
    out["status"] = int(st)
    out["maxvio"] = float(out["maxvio"][0])
    out["nvs"] = nvs(S, K, E, R, tp) if st != STATUS_BAD_ARGS else 0
    return out


def plan_rank(topk, counts, rank: int, E: int, B: int, tp: int, mode: int = 0) -> dict:
    """One rank's share of the plan from its own picks ``topk`` [S, K] and
    every rank's counts ``counts`` [R, E]: dst [S, K] and the group layout."""
    topk = _c(topk, np.int32)
    counts = _c(counts, np.int32)
    S, K = topk.shape
    R = counts.shape[0]
    NR = E + B
    out = dict(
        dst=np.full((S, K), -1, np.int32),
        cu_seqlens=np.zeros((R, NR), np.int32),
        row_counts=np.zeros((R, NR), np.int32),
        slot_expert=np.full((R, max(B, 0)), -1, np.int32),
        maxvio=np.zeros(1, np.float32),
        assign=np.zeros((R, 4), np.int32),
    )
    st = lib().oracle_plan_rank(R, S, K, E, B, tp, mode, rank, _p(topk), _p(counts), _p(out["dst"]),
                                _p(out["cu_seqlens"]), _p(out["row_counts"]), _p(out["slot_expert"]),
                                _p(out["maxvio"]), _p(out["assign"]))
    out["status"] = int(st)
    out["maxvio"] = float(out["maxvio"][0])
    return out


def dispatch(dst, hidden_bits, w, nvs_: int, sentinel: int = 0xFFFF, w_sentinel=np.nan):
    """Scatter bf16 rows [R, S, H] (uint16 bits) into a fresh [R*NvS, H] buffer
    prefilled with ``sentinel``; returns (buf bits, w_nvs)."""
    dst = _c(dst, np.int32)
    hidden_bits = _c(hidden_bits, np.uint16)
    R, S, K = dst.shape
    H = hidden_bits.shape[-1]
    buf = np.full((R * nvs_, H), sentinel, np.uint16)
    w_nvs = None
    wa = None
    if w is not None:
        wa = _c(w, np.float32)
        w_nvs = np.full(R * nvs_, w_sentinel, np.float32)
    lib().oracle_dispatch(R, S, K, H, _p(dst), _p(hidden_bits), _p(wa), _p(buf), _p(w_nvs))
    return buf, w_nvs


def combine(dst, y_bits, w_nvs=None, gather: bool = True):
    """Gather K rows per token from ``y_bits`` [rows, H] and weight them;
    returns (out bits [R, S, H], gathered_w [R, S, K] or None)."""
    dst = _c(dst, np.int32)
    y_bits = _c(y_bits, np.uint16)
    R, S, K = dst.shape
    H = y_bits.shape[-1]
    out = np.zeros((R, S, H), np.uint16)
    wa = None if w_nvs is None else _c(w_nvs, np.float32)
    gw = np.zeros((R, S, K), np.float32) if (gather and wa is not None) else None
    lib().oracle_combine(R, S, K, H, _p(dst), _p(y_bits), _p(wa), _p(out), _p(gw))
    return out, gw


def prefetch(slot_expert, W_bits, pool_bits):
    """In place: pool[s] = W[slot_expert[s]] for used slots.  W [E, HHp],
    pool [R*B, HHp], both uint16 bf16 bits."""
    se = _c(slot_expert, np.int32)
    R, B = se.shape
    assert W_bits.flags.c_contiguous and pool_bits.flags.c_contiguous
    HHp = W_bits.shape[-1]
    lib().oracle_prefetch(R, B, HHp, _p(se), _p(W_bits), _p(pool_bits))


def reduce_grad(slot_expert, G, RB):
    """In place: G [E, HHp] += slot grads, consumed RB [R*B, HHp] slots zeroed."""
    se = _c(slot_expert, np.int32)
    R, B = se.shape
    assert G.dtype == np.float32 and RB.dtype == np.float32
    assert G.flags.c_contiguous and RB.flags.c_contiguous
    E, HHp = G.shape
    lib().oracle_reduce_grad(R, B, E, HHp, _p(se), _p(G), _p(RB))


from .group_gemm import group_gemm, segments  # noqa: E402,F401  (numpy, fp64)
