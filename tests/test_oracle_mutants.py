"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake (a dropped term, a wrong index or sign, a
swapped loop, a queue order) in a temporary copy of the oracle's C source,
on the CPU, and runs the oracle pin suite against that copy; the suite has to
fail.  The real oracle is never modified."""
import os
import shutil
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTANTS = {
    "kept prefix ignores donations": (
        "if (don_from[j] == h) keep[h] -= don_amt[j];", "if (don_from[j] == h) keep[h] -= 0;"),
    "donor taken from the back of the queue": (
        "int l = largeq[lh];", "int l = largeq[lt > lh + 1 ? lh + 1 : lh];"),
    "drained donor served last": (
        "if (cur[l] < C) { lh++; smallq[--sh] = l; }", "if (cur[l] < C) { lh++; smallq[st++] = l; }"),
    "expert start off by one term": (
        "            estart[e] = run;\n            run += T[e];",
        "            run += T[e];\n            estart[e] = run;"),
    "fewest-copies order descending": (
        "while (i >= 0 && (T[o[i]] > T[e] || (T[o[i]] == T[e] && o[i] > e))) {",
        "while (i >= 0 && (T[o[i]] < T[e] || (T[o[i]] == T[e] && o[i] > e))) {"),
    "fewest-copies ties to the higher id": (
        "while (i >= 0 && (T[o[i]] > T[e] || (T[o[i]] == T[e] && o[i] > e))) {",
        "while (i >= 0 && (T[o[i]] > T[e] || (T[o[i]] == T[e] && o[i] < e))) {"),
    "fewest-copies walk in id order": (
        "            const int e = y.order[(int64_t)h * G + jj];",
        "            const int e = h * G + jj;"),
    "cu_seqlens exclusive": (
        "cu_seqlens[(int64_t)s * NR + i] = (int32_t)run;\n",
        "cu_seqlens[(int64_t)s * NR + i] = (int32_t)(run - (n ? pad_up(n, tp) : 0));\n"),
    "empty rows padded": ("run += n ? pad_up(n, tp) : 0;", "run += n ? pad_up(n, tp) : tp;"),
    "combine drops the weight": (
        "double wk = w_nvs ? (double)w_nvs[d[k]] : 1.0;", "double wk = 1.0;"),
    "combine reads one row": (
        "for (int k = 0; k < K; k++) {\n                    double wk",
        "for (int k = 0; k < 1; k++) {\n                    double wk"),
    "maxvio sign": ("*maxvio = (float)((double)maxT / Tbar - 1.0);",
                    "*maxvio = (float)((double)maxT / Tbar + 1.0);"),
    "slots in descending order": (
        "slot_expert[(int64_t)s * B + q] = rx_e[j];", "slot_expert[(int64_t)s * B + (B - 1 - q)] = rx_e[j];"),
    "consumed slots not zeroed": (
        "for (int64_t i = 0; i < HHp; i++) RB[holders[j] * HHp + i] = 0.0f;", "(void)0;"),
    "reduction adds one slot": (
        "for (int64_t j = 0; j < nh; j++) acc += (double)RB[holders[j] * HHp + i];",
        "for (int64_t j = 0; j < 1; j++) acc += (double)RB[holders[j] * HHp + i];"),
    "bf16 truncates": ("double v = nearbyint(ax / q) * q;", "double v = floor(ax / q) * q;"),
    "NvS too small": ("return pad_up(C + 2 * G * (tp - 1), tp);", "return pad_up(C + G * (tp - 1), tp);"),
    "sequence ordered by token before rank": (
        "            for (int r = 0; r < R; r++)\n                for (int t = 0; t < S; t++)\n"
        "                    for (int k = 0; k < K; k++) {\n                        int64_t idx",
        "            for (int t = 0; t < S; t++)\n                for (int r = 0; r < R; r++)\n"
        "                    for (int k = 0; k < K; k++) {\n                        int64_t idx"),
    "duplicate check off": ("if (tok[k2] == e) status |= ORC_DUP_EXPERT;", "(void)0;"),
    "overflow goes to the last slot": (
        "n[rx_e[j]] += (int32_t)rx_n[j]; /* overflow: the expert's home row */",
        "n[E + B - 1] += (int32_t)rx_n[j];"),
    "slots by count take the fewest picks": (
        "if (rx_n[m] > rx_n[j] || (rx_n[m] == rx_n[j] && m < j)) better++;",
        "if (rx_n[m] < rx_n[j] || (rx_n[m] == rx_n[j] && m < j)) better++;"),
    "rank share counts its own rank in the prefix": (
        "for (int q = 0; q < rank; q++) pre += counts[(int64_t)q * E + e];",
        "for (int q = 0; q <= rank; q++) pre += counts[(int64_t)q * E + e];"),
    "rank share positions from the expert start only": (
        "first = y.estart[e] > y.don_start[j] ? y.estart[e] : y.don_start[j];", "first = y.estart[e];"),
    "slots by count break ties to the higher id": (
        "if (rx_n[m] > rx_n[j] || (rx_n[m] == rx_n[j] && m < j)) better++;",
        "if (rx_n[m] > rx_n[j] || (rx_n[m] == rx_n[j] && m > j)) better++;"),
}


def _run_mutant(name, a, b, base):
    src = open(os.path.join(ROOT, "oracle", "moonep_oracle.c")).read()
    assert src.count(a) >= 1, f"mutation site for {name!r} not found"
    d = os.path.join(base, name.replace(" ", "_"))
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(d, "oracle"),
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    shutil.copytree(os.path.join(ROOT, "tests"), os.path.join(d, "tests"),
                    ignore=shutil.ignore_patterns("__pycache__", "test_oracle_mutants.py"))
    pkg = os.path.join(d, "load_balancing_planner_b200")
    os.makedirs(pkg)
    for f in ("__init__.py", "synth.py"):
        shutil.copy(os.path.join(ROOT, "load_balancing_planner_b200", f), pkg)
    open(os.path.join(d, "oracle", "moonep_oracle.c"), "w").write(src.replace(a, b, 1))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        "tests/test_oracle.py"], cwd=d, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-300:]


def test_every_planted_mistake_fails_a_pin():
    base = tempfile.mkdtemp(prefix="oracle_mutants_")
    try:
        with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 2)) as ex:
            futs = {n: ex.submit(_run_mutant, n, a, b, base) for n, (a, b) in MUTANTS.items()}
            survivors = {n: f.result()[1] for n, f in futs.items() if f.result()[0] == 0}
    finally:
        shutil.rmtree(base, ignore_errors=True)
    assert not survivors, f"mutants not caught by any pin: {list(survivors)}"
