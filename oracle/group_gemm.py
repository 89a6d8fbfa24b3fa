"""The VM group GEMM on the CPU, in fp64 (numpy).

TEST INFRASTRUCTURE ONLY: imported by ``tests/`` and ``bench.py``'s CPU
baseline, never by the library; it shares no code with the CUDA path.

MoonEP README, "Integration": the consumer of a dispatched layer is a group
GEMM over one [E+B, H, H'] weight tensor per projection, and the planner's
cu_seqlens[E+B] selects which expert row each token segment of the buffer
uses.  "Weight buffer": rows [0, E) are the home experts (shared by every
rank), rows [E, E+B) the rank's own prefetch slots.  So for rank r and plan
row i with n = row_counts[r][i] > 0, the segment's real tokens are the n
slots starting at cu_seqlens[r][i] - pad(n) (cu_seqlens holds inclusive,
padded end offsets), and they are multiplied by W[i] if i < E, else by
pool[r][i - E].  Only real slots are defined; padding slots are not.
"""
from __future__ import annotations

import numpy as np


def _bf16_to_f64(bits):
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _pad(n, tp):
    return -(-n // tp) * tp if n else 0


def segments(cu_seqlens, row_counts, E, tp):
    """(rank, first slot, n, plan row) of every non-empty row, in row order."""
    cu = np.asarray(cu_seqlens)
    rc = np.asarray(row_counts)
    out = []
    for r in range(cu.shape[0]):
        for i in range(cu.shape[1]):
            n = int(rc[r, i])
            if n:
                out.append((r, int(cu[r, i]) - _pad(n, tp), n, i))
    return out


def group_gemm(cu_seqlens, row_counts, x_bits, W_bits, pool_bits, E, tp, nvs):
    """fp64 products of every real slot: returns (y [R*nvs, Hp] fp64 with NaN
    outside real slots, mask [R*nvs] of real slots).  x_bits [R*nvs, H],
    W_bits [E, H, Hp], pool_bits [R*B, H, Hp] or None, all bf16 bit patterns."""
    x_bits = np.asarray(x_bits)
    R = np.asarray(cu_seqlens).shape[0]
    Hp = W_bits.shape[-1]
    B = 0 if pool_bits is None else pool_bits.shape[0] // R
    y = np.full((R * nvs, Hp), np.nan)
    mask = np.zeros(R * nvs, bool)
    for r, s0, n, i in segments(cu_seqlens, row_counts, E, tp):
        w = W_bits[i] if i < E else pool_bits[r * B + (i - E)]
        rows = slice(r * nvs + s0, r * nvs + s0 + n)
        y[rows] = _bf16_to_f64(x_bits[rows]) @ _bf16_to_f64(w)
        mask[rows] = True
    return y, mask
