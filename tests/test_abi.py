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


@pytest.mark.parametrize("bad", [
    dict(E=10, R=4),             # E % R != 0
    dict(K=9, E=8),              # K > E
    dict(H=100),                 # H % 8 != 0
    dict(B=1, mode=0),           # training needs B >= E/R
    dict(R=65, E=65 * 4),        # R past the limit
    dict(E=8192, R=8),           # E past the limit
    dict(K=33, E=64),            # K past the limit
    dict(token_padding=0),
    dict(mode=3),
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
    moonep_handle_t h = (moonep_handle_t)0;
    if (moonep_create(&c, &h) != MOONEP_ERR_CONFIG || h) return 1;
    if (strcmp(moonep_error_string(MOONEP_ERR_CONFIG), "configuration rejected") != 0) return 2;
    if (moonep_plan_rank(0, 0, 0, 0, 0, 0) != MOONEP_ERR_NULL) return 3;
    if (moonep_dispatch_rank(0, 0, 0, 0, 0, 0, 0) != MOONEP_ERR_NULL) return 4;
    if (moonep_destroy(0) != MOONEP_OK) return 5;
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
