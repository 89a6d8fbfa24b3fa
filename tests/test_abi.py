"""The C ABI library loads and exports every symbol include/moonep.h declares;
host-side validation rejects bad configurations before touching the GPU."""
import ctypes
import os
import re

import pytest

from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "moonep.h")


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"MOONEP_API\s+[\w\s\*]*?\b(moonep_\w+)\s*\(", src)))


def test_header_declares_the_hot_path():
    names = declared_symbols()
    for n in ("moonep_plan", "moonep_dispatch", "moonep_combine", "moonep_prefetch_weight",
              "moonep_reduce_grad", "moonep_create", "moonep_destroy"):
        assert n in names


def test_library_exports_every_declared_symbol():
    from load_balancing_planner_b200 import build
    path = build.build()
    lib = ctypes.CDLL(path)
    for n in declared_symbols():
        assert hasattr(lib, n), f"{n} declared but not exported"


def test_binding_covers_every_declared_symbol():
    from load_balancing_planner_b200 import moonep
    assert set(declared_symbols()) == set(moonep.EXPORTS)


def test_error_strings():
    from load_balancing_planner_b200 import moonep
    assert moonep.error_string(moonep.ERR_CONFIG) == "configuration rejected"
    assert moonep.error_string(0) == "ok"


def test_every_error_code_is_bound_and_described():
    # each MOONEP_ERR_* the header defines has the same value in the binding
    # and a description of its own in the library
    from load_balancing_planner_b200 import moonep
    codes = dict(re.findall(r"#define MOONEP_(ERR_\w+)\s+\((-\d+)\)", open(HEADER).read()))
    assert "ERR_DEVICE" in codes and len(codes) >= 6
    texts = set()
    for name, value in codes.items():
        assert getattr(moonep, name) == int(value), name
        text = moonep.error_string(int(value))
        assert text != "unknown moonep error", name
        texts.add(text)
    assert len(texts) == len(codes)


@pytest.mark.parametrize("bad", [
    dict(E=10, R=4),             # E % R != 0
    dict(K=9, E=8),              # K > E
    dict(H=100),                 # H % 8 != 0
    dict(B=1, mode=0),           # training needs B >= E/R
    dict(R=65, E=65 * 4),        # R past the limit
    dict(E=8192, R=8),           # E past the limit
    dict(K=33, E=64),            # K past the limit
    dict(token_padding=0),
    dict(mode=4),
    dict(B=1, mode=3),           # the fewest-copies training mode needs B >= E/R too
    dict(S=0),
    dict(S=1 << 20, K=32, R=64, E=256),  # R*S*K >= 2^31
])
def test_create_rejects_bad_configs_without_a_gpu(bad):
    from load_balancing_planner_b200 import moonep
    cfg = dict(S=64, H=128, K=2, E=8, R=2, B=4, token_padding=8, num_sms=0, mode=0)
    cfg.update(bad)
    c = moonep.Config(*(cfg[k] for k in ("S", "H", "K", "E", "R", "B", "token_padding", "num_sms", "mode")))
    out = ctypes.c_void_p(123)
    rc = moonep.lib.moonep_create(ctypes.byref(c), ctypes.byref(out))
    assert rc == moonep.ERR_CONFIG
    assert out.value is None


def test_null_arguments_are_rejected():
    from load_balancing_planner_b200 import moonep
    P = ctypes.c_void_p
    assert moonep.lib.moonep_create(None, ctypes.byref(P())) == moonep.ERR_NULL
    assert moonep.lib.moonep_plan(None, None, None, None, None) == moonep.ERR_NULL
    assert moonep.lib.moonep_dispatch(None, None, None, None, None, None, None) == moonep.ERR_NULL
    assert moonep.lib.moonep_combine(None, None, None, None, None, None, None) == moonep.ERR_NULL
    assert moonep.lib.moonep_prefetch_weight(None, None, 1, None, None, 8, None) == moonep.ERR_NULL
    assert moonep.lib.moonep_reduce_grad(None, None, 1, None, None, 8, None) == moonep.ERR_NULL
    assert moonep.lib.moonep_plan_rank(None, 0, None, None, None, None) == moonep.ERR_NULL
    assert moonep.lib.moonep_dispatch_rank(None, None, None, None, None, None, None) == moonep.ERR_NULL
    assert moonep.lib.moonep_combine_rank(None, None, None, None, None, None, None) == moonep.ERR_NULL
    assert moonep.lib.moonep_destroy(None) == moonep.OK
    assert moonep.lib.moonep_nvs(None) < 0


def test_buffer_layer_imports_and_names_status_bits():
    from load_balancing_planner_b200 import moonep
    from load_balancing_planner_b200.buffer import Buffer, PlanStatusError
    e = PlanStatusError(moonep.STATUS_BAD_EXPERT | moonep.STATUS_COUNT_MISMATCH)
    assert e.status == 5 and "outside [0, E)" in str(e) and "tokens_per_expert" in str(e)
    for name in ("dispatch", "combine", "prefetch_weight", "reduce_grad", "destroy", "check"):
        assert callable(getattr(Buffer, name))


@pytest.mark.parametrize("S,K,E,R,tp", [(4096, 8, 256, 8, 128), (1024, 8, 64, 8, 128), (64, 2, 8, 2, 8),
                                        (333, 3, 24, 4, 16), (40, 4, 256, 64, 8), (100, 32, 64, 2, 4)])
def test_rank_buffer_slot_count_matches_the_oracle(S, K, E, R, tp):
    # RankBuffer sizes peer buffers before any handle exists; its NvS must be
    # the oracle's (both written from the same definition, separately)
    import oracle
    from load_balancing_planner_b200.ep import RankBuffer
    assert RankBuffer.nvs_of(S, K, E, R, tp) == oracle.nvs(S, K, E, R, tp)


def test_gather_counts_rejects_bad_tables_without_a_process_group():
    import torch
    from load_balancing_planner_b200.ep import gather_counts
    with pytest.raises(ValueError):
        gather_counts(torch.zeros((2, 8), dtype=torch.int32))
    with pytest.raises(ValueError):
        gather_counts(torch.zeros(8, dtype=torch.int64))


def test_rank_calls_check_their_tables_before_the_device():
    # host-side checks of the per-rank weight calls, with no handle: a NULL
    # handle is refused before any table is read
    from load_balancing_planner_b200 import moonep
    P = ctypes.c_void_p
    tab = (P * 2)()
    assert moonep.lib.moonep_prefetch_weight_rank(None, None, 0, 1, tab, tab, 8, None) == moonep.ERR_NULL
    assert moonep.lib.moonep_reduce_grad_rank(None, None, 0, 1, tab, tab, 8, None) == moonep.ERR_NULL


C_CALLER = r"""
#include <stdio.h>
#include <string.h>
#include "moonep.h"
int main(void) {
    moonep_config_t c = {64, 128, 2, 10, 4, 4, 8, 0, 0};  /* E % R != 0 */
    moonep_config_t ok = {64, 128, 2, 8, 2, 4, 8, 0, 0};
    moonep_handle_t h = (moonep_handle_t)0;
    moonep_plan_sizes_t sz;
    if (moonep_create(&c, &h) != MOONEP_ERR_CONFIG || h) return 1;
    if (strcmp(moonep_error_string(MOONEP_ERR_CONFIG), "configuration rejected") != 0) return 2;
    if (moonep_plan_rank(0, 0, 0, 0, 0, 0) != MOONEP_ERR_NULL) return 3;
    if (moonep_dispatch_rank(0, 0, 0, 0, 0, 0, 0) != MOONEP_ERR_NULL) return 4;
    if (moonep_destroy(0) != MOONEP_OK) return 5;
    if (moonep_plan_sizes(&c, 0, &sz) != MOONEP_ERR_CONFIG || sz.dst != 0) return 6;
    if (moonep_plan_sizes(&ok, 0, &sz) != MOONEP_OK || sz.dst != 2 * 64 * 2 || sz.nvs != 184) return 7;
    if (moonep_plan_status(0, 0) != MOONEP_ERR_NULL || moonep_set_plan_barrier(0, 0, 0) != MOONEP_ERR_NULL) return 8;
    puts("ok");
    return 0;
}
"""


def test_header_is_plain_c_and_the_library_links_from_c(tmp_path):
    # the boundary is a C ABI: a C99 program includes the header (pedantic,
    # warnings as errors), links the library and calls it, with no GPU needed
    import subprocess
    from load_balancing_planner_b200 import build
    lib = build.build()
    src = tmp_path / "caller.c"
    src.write_text(C_CALLER)
    exe = tmp_path / "caller"
    libdir = os.path.dirname(lib)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I",
                    os.path.join(ROOT, "include"), "-o", str(exe), str(src), "-L", libdir, "-lmoonep",
                    f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", (out.returncode, out.stdout, out.stderr)


@pytest.mark.parametrize("R,S,K,E,B,tp,mode", [(2, 64, 2, 8, 4, 8, 0), (8, 4096, 8, 256, 32, 128, 0),
                                               (8, 4096, 8, 256, 4, 128, 1), (4, 333, 3, 24, 0, 16, 1),
                                               (64, 40, 4, 256, 4, 8, 2)])
def test_plan_sizes_match_the_oracle_arrays(R, S, K, E, B, tp, mode):
    # moonep_plan_sizes (host only) against the shapes of the arrays the
    # oracle fills for the same configuration, group and one-rank forms
    import numpy as np

    import oracle
    from load_balancing_planner_b200 import moonep
    cfg = moonep.Config(S, 8, K, E, R, B, tp, 0, mode)
    sz = moonep.moonep_plan_sizes(cfg)
    rng = np.random.default_rng(0)
    tk = np.stack([np.stack([rng.permutation(E)[:K] for _ in range(S)]) for _ in range(R)]).astype(np.int32)
    o = oracle.plan(tk, E, B, tp, mode)
    assert o["status"] == 0
    for k in ("dst", "cu_seqlens", "row_counts", "slot_expert", "counts", "assign"):
        assert getattr(sz, k) == o[k].size, k
    assert sz.maxvio == 1 and sz.status == 1
    assert sz.nvs == o["nvs"] == oracle.nvs(S, K, E, R, tp)
    counts = np.stack([np.bincount(tk[r].reshape(-1), minlength=E) for r in range(R)]).astype(np.int32)
    orank = oracle.plan_rank(tk[R - 1], counts, R - 1, E, B, tp, mode)
    assert moonep.moonep_plan_sizes(cfg, True).dst == orank["dst"].size == S * K


C_GPU_CALLER = r"""
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include <cuda_runtime_api.h>
#include "moonep.h"

/* Plans and dispatches one layer through the C ABI, with every device array
   sized from moonep_plan_sizes alone.  argv: input file (topk int32 [R*S*K],
   tokens_per_expert int32 [R*E], hidden bf16 bits [R*S*H], route weights fp32
   [R*S*K]), output file (the plan arrays in moonep_plan_t order, then the
   dispatch buffer [R*NvS*H] and its weights [R*NvS]). */
static void *dev(int64_t bytes, unsigned char fill) {
    void *p = NULL;
    if (cudaMalloc(&p, (size_t)(bytes > 0 ? bytes : 4)) != cudaSuccess) exit(20);
    if (cudaMemset(p, fill, (size_t)(bytes > 0 ? bytes : 4)) != cudaSuccess) exit(21);
    return p;
}
static void *up(FILE *f, int64_t bytes) {
    void *h = malloc((size_t)bytes), *d = dev(bytes, 0);
    if (!h || fread(h, 1, (size_t)bytes, f) != (size_t)bytes) exit(22);
    if (cudaMemcpy(d, h, (size_t)bytes, cudaMemcpyHostToDevice) != cudaSuccess) exit(23);
    free(h);
    return d;
}
static void down(FILE *f, const void *d, int64_t bytes) {
    void *h = malloc((size_t)bytes);
    if (!h || cudaMemcpy(h, d, (size_t)bytes, cudaMemcpyDeviceToHost) != cudaSuccess) exit(24);
    if (fwrite(h, 1, (size_t)bytes, f) != (size_t)bytes) exit(25);
    free(h);
}
int main(int argc, char **argv) {
    moonep_config_t c = {64, 128, 2, 8, 2, 4, 8, 0, 0};
    moonep_plan_sizes_t n;
    moonep_plan_t p;
    moonep_handle_t h = NULL;
    int32_t st = -1;
    FILE *in, *out;
    void *topk, *tpe, *hidden, *w, *buf, *wbuf;
    const int64_t R = c.R, S = c.S, K = c.K, E = c.E, H = c.H;
    if (argc != 3 || !(in = fopen(argv[1], "rb")) || !(out = fopen(argv[2], "wb"))) return 10;
    if (moonep_plan_sizes(&c, 0, &n) != MOONEP_OK) return 11;
    p.dst = (int32_t *)dev(4 * n.dst, 0xFF);
    p.cu_seqlens = (int32_t *)dev(4 * n.cu_seqlens, 0xFF);
    p.row_counts = (int32_t *)dev(4 * n.row_counts, 0xFF);
    p.slot_expert = (int32_t *)dev(4 * n.slot_expert, 0xFF);
    p.counts = (int32_t *)dev(4 * n.counts, 0xFF);
    p.assign = (int32_t *)dev(4 * n.assign, 0xFF);
    p.maxvio = (float *)dev(4 * n.maxvio, 0xFF);
    p.status = (int32_t *)dev(4 * n.status, 0xFF);
    topk = up(in, 4 * R * S * K);
    tpe = up(in, 4 * R * E);
    hidden = up(in, 2 * R * S * H);
    w = up(in, 4 * R * S * K);
    buf = dev(2 * R * n.nvs * H, 0xFF);
    wbuf = dev(4 * R * n.nvs, 0xFF);
    if (moonep_create(&c, &h) != MOONEP_OK) return 12;
    if (moonep_nvs(h) != n.nvs) return 13;
    if (moonep_plan(h, (const int32_t *)topk, (const int32_t *)tpe, &p, NULL) != MOONEP_OK) return 14;
    if (moonep_dispatch(h, &p, hidden, (const float *)w, buf, (float *)wbuf, NULL) != MOONEP_OK) return 15;
    if (moonep_plan_status(&p, &st) != MOONEP_OK || st != 0) return 16;
    down(out, p.dst, 4 * n.dst);
    down(out, p.cu_seqlens, 4 * n.cu_seqlens);
    down(out, p.row_counts, 4 * n.row_counts);
    down(out, p.slot_expert, 4 * n.slot_expert);
    down(out, p.counts, 4 * n.counts);
    down(out, p.assign, 4 * n.assign);
    down(out, p.maxvio, 4 * n.maxvio);
    down(out, p.status, 4 * n.status);
    down(out, buf, 2 * R * n.nvs * H);
    down(out, wbuf, 4 * R * n.nvs);
    fclose(out);
    fclose(in);
    if (moonep_destroy(h) != MOONEP_OK) return 17;
    puts("ok");
    return 0;
}
"""


@pytest.mark.gpu
def test_c_caller_sizes_plans_and_dispatches_on_the_gpu(tmp_path, cuda):
    # a C99 program allocates a plan from moonep_plan_sizes alone, plans and
    # dispatches the tiny case on the GPU; its plan is bit-exact against the
    # oracle and so is the dispatch buffer, untouched padding included
    import subprocess

    import numpy as np

    import oracle
    from load_balancing_planner_b200 import build, synth
    R, S, K, E, B, H, tp = 2, 64, 2, 8, 4, 128, 8
    tk, _, _ = synth.routing(R, S, K, E, 1.0, "boost0", seed=0)
    tpe = synth.local_counts(tk, E)
    xb = synth.bf16_bits(synth.hidden_bf16(R, S, H, seed=0))
    w = synth.route_weights(R, S, K, seed=0)
    inp = tmp_path / "in.bin"
    with open(inp, "wb") as f:
        for a in (tk.astype(np.int32), tpe.astype(np.int32), xb.astype(np.uint16), w.astype(np.float32)):
            f.write(np.ascontiguousarray(a).tobytes())
    lib = build.build()
    src = tmp_path / "gpu_caller.c"
    src.write_text(C_GPU_CALLER)
    exe = tmp_path / "gpu_caller"
    libdir = os.path.dirname(lib)
    cuda_home = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(cuda_home, "include"), "-o", str(exe), str(src), "-L", libdir, "-lmoonep",
                    "-L", os.path.join(cuda_home, "lib64"), "-lcudart",
                    f"-Wl,-rpath,{libdir}", f"-Wl,-rpath,{os.path.join(cuda_home, 'lib64')}"], check=True)
    outp = tmp_path / "out.bin"
    r = subprocess.run([str(exe), str(inp), str(outp)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)

    o = oracle.plan(tk, E, B, tp, 0, tpe)
    nvs = o["nvs"]
    raw = open(outp, "rb").read()
    off = 0

    def take(dtype, n):
        nonlocal off
        a = np.frombuffer(raw, dtype=dtype, count=n, offset=off)
        off += a.nbytes
        return a

    got = {}
    for k in ("dst", "cu_seqlens", "row_counts", "slot_expert", "counts", "assign"):
        got[k] = take(np.int32, o[k].size).reshape(o[k].shape)
        assert np.array_equal(got[k], o[k]), k
    assert np.float32(take(np.float32, 1)[0]) == np.float32(o["maxvio"])
    assert take(np.int32, 1)[0] == 0
    gbuf = take(np.uint16, R * nvs * H).reshape(R * nvs, H)
    gw = take(np.uint32, R * nvs)
    assert off == len(raw)
    obuf, own = oracle.dispatch(o["dst"], xb, w, nvs)
    assert np.array_equal(gbuf, obuf)  # real slots and the untouched 0xFFFF padding
    live = o["dst"].reshape(-1)
    assert np.array_equal(gw[live], own[live].view(np.uint32))
    dead = np.setdiff1d(np.arange(R * nvs), live)
    assert np.all(gw[dead] == 0xFFFFFFFF)
