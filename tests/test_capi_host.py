"""Host-side checks of the C ABI: the library loads, exports every declared
symbol, and rejects bad arguments before touching a GPU (CPU only)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def capi():
    from long_convolution_sequence_hyena_b200 import build
    build.build()
    from long_convolution_sequence_hyena_b200 import capi as c
    return c


def _declared_symbols():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"HYENA_API\s+[\w\s\*]+?\b(hyena_\w+)\s*\(", src)
    return names


def test_every_declared_symbol_is_exported(capi):
    declared = _declared_symbols()
    assert set(capi.EXPORTED) <= set(declared) and len(declared) >= len(capi.EXPORTED)
    lib = ctypes.CDLL(capi.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name


def test_status_strings(capi):
    for code in range(7):
        assert capi.hyena_status_string(code) not in ("", "unknown status")
    assert capi.hyena_status_string(99) == "unknown status"


@pytest.mark.parametrize("args,expect", [
    ((1, [256], 0, 2, 1, 1), "HYENA_ERR_INVALID_ARG"),        # no channels
    ((1, [256], 4, 0, 1, 1), "HYENA_ERR_INVALID_ARG"),        # order 0
    ((1, [256], 4, 9, 1, 1), "HYENA_ERR_INVALID_ARG"),        # order above HYENA_MAX_ORDER
    ((1, [0], 4, 2, 1, 1), "HYENA_ERR_INVALID_ARG"),          # empty sequence
    ((1, [256], 4, 2, 7, 1), "HYENA_ERR_INVALID_ARG"),        # bad dtype
    ((4, [4, 4, 4, 4], 4, 1, 1, 0), "HYENA_ERR_INVALID_ARG"), # 4D
    ((3, [4, 4, 4], 4, 1, 1, 0), "HYENA_ERR_UNSUPPORTED"),    # 3D extents outside 16, 32, 64
    ((3, [16, 16, 16], 4, 1, 1, 1), "HYENA_ERR_UNSUPPORTED"), # causal 3D
    ((1, [256], 4, 2, 1, 0), "HYENA_ERR_UNSUPPORTED"),        # non-causal 1D
    ((2, [64, 64], 4, 1, 1, 1), "HYENA_ERR_UNSUPPORTED"),     # causal 2D
    ((1, [524289], 4, 1, 1, 1), "HYENA_ERR_UNSUPPORTED"),     # longer than the longest path (M = 2^20)
])
def test_plan_create_rejects(capi, args, expect):
    st, h = capi.hyena_plan_create(*args)
    assert capi.STATUS_NAMES[st] == expect and h is None


def test_null_plan_rejected(capi):
    assert capi.hyena_plan_destroy(None) == capi.HYENA_OK
    assert capi.hyena_plan_info(None)[0] == capi.HYENA_ERR_INVALID_ARG
    assert capi.hyena_workspace_bytes(None, 4) == 0
    assert capi.hyena_forward(None, 1, 16, [16], 16, None, 16) == capi.HYENA_ERR_INVALID_ARG
    assert capi.hyena_filter_spectrum(None, 16, None, 16) == capi.HYENA_ERR_INVALID_ARG
    assert capi.hyena_implicit_filter(None, None, 16) == capi.HYENA_ERR_INVALID_ARG
    assert capi.hyena_forward_host_workspace_bytes(None, 4) == 0
    assert capi.hyena_forward_host(None, 1, 16, [16], 16, None, 16, 16, 1 << 20) == capi.HYENA_ERR_INVALID_ARG


C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "hyena.h"

int main(void) {
    int bad = 0;
    for (int s = HYENA_OK; s <= HYENA_ERR_NOMEM; ++s) {
        const char *name = hyena_status_string((hyena_status_t)s);
        if (!name || !name[0]) bad = 1;
    }
    const void *gates[1] = {0};
    if (hyena_plan_destroy(NULL) != HYENA_OK) bad = 2;
    if (hyena_workspace_bytes(NULL, 4) != 0) bad = 3;
    if (hyena_forward_host_workspace_bytes(NULL, 4) != 0) bad = 4;
    if (hyena_forward(NULL, 1, 0, gates, 0, NULL, 0, NULL, 0, NULL) != HYENA_ERR_INVALID_ARG) bad = 5;
    if (hyena_forward_host(NULL, 1, 0, gates, 0, NULL, 0, NULL, 0, NULL) != HYENA_ERR_INVALID_ARG) bad = 6;
    if (hyena_forward_no_alloc(NULL, 1, 0, gates, 0, NULL, 0, NULL) != HYENA_ERR_INVALID_ARG) bad = 7;
    if (hyena_filter_spectrum(NULL, NULL, NULL, NULL, NULL) != HYENA_ERR_INVALID_ARG) bad = 8;
    int64_t launches = -1;
    if (hyena_launch_count(NULL) != HYENA_ERR_INVALID_ARG) bad = 9;
    if (hyena_launch_count(&launches) != HYENA_OK || launches != 0) bad = 10;
    if (hyena_filter_spectrum_ws(NULL, NULL, NULL, NULL, NULL, 0, NULL) != HYENA_ERR_INVALID_ARG) bad = 11;
    if (hyena_filter_spectrum_workspace_bytes(NULL) != 0) bad = 12;
    if (hyena_debug_fail_allocation(-1) != HYENA_ERR_INVALID_ARG) bad = 13;
    if (hyena_debug_fail_allocation(0) != HYENA_OK) bad = 14;
    if (hyena_debug_plan_resources(NULL) != HYENA_ERR_INVALID_ARG) bad = 15;
    if (hyena_plan_device_errors(NULL, NULL, 0) != HYENA_ERR_INVALID_ARG) bad = 16;
    if (hyena_plan_set_layout(NULL, HYENA_LAYOUT_BLD) != HYENA_ERR_INVALID_ARG) bad = 17;
    if (hyena_forward_gated(NULL, 1, NULL, NULL, gates, NULL, NULL, NULL, NULL, 0, NULL) != HYENA_ERR_INVALID_ARG)
        bad = 18;
    printf("%s\n", bad ? "FAIL" : "OK");
    return bad;
}
"""


def test_header_compiles_as_c_and_links(capi, tmp_path):
    """include/hyena.h is a plain C header: a C99 program includes it with warnings as
    errors, links libhyena.so and calls the entry points that need no GPU."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    src = tmp_path / "prog.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "prog"
    pkg = os.path.dirname(capi.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                           str(src), "-o", str(exe), "-L", pkg, "-lhyena", "-Wl,-rpath," + pkg])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0 and out.stdout.strip() == "OK", (out.returncode, out.stdout, out.stderr)


def test_plan_create_ex_rejects_unknown_flags(capi):
    st, h = capi.hyena_plan_create_ex(1, [3000], 4, 2, capi.HYENA_F32, 1, 0x10)
    assert st == capi.HYENA_ERR_INVALID_ARG and h is None


def test_launch_count_without_a_gpu(capi):
    """The launch counter reads without touching the device; calls rejected before
    any launch leave it unchanged."""
    n0 = capi.hyena_launch_count()
    assert n0 >= 0
    assert capi.hyena_forward(None, 1, 16, [16], 16, None, 16) == capi.HYENA_ERR_INVALID_ARG
    assert capi.hyena_launch_count() == n0
    assert capi.lib.hyena_launch_count(None) == capi.HYENA_ERR_INVALID_ARG


def test_debug_hooks_reject_bad_arguments(capi):
    """The plan-failure test hooks check their arguments without a GPU."""
    assert capi.lib.hyena_debug_fail_allocation(-1) == capi.HYENA_ERR_INVALID_ARG
    assert capi.lib.hyena_debug_fail_allocation(0) == capi.HYENA_OK
    assert capi.lib.hyena_debug_plan_resources(None) == capi.HYENA_ERR_INVALID_ARG
    assert capi.hyena_debug_plan_resources() >= 0
