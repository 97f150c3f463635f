"""Small and odd shapes through every forward family of the index-checking
debug build (run by test_gpu_check_bounds.py in a process of its own, with
HYENA_LIBRARY=checked): each result against the fp64 oracle, and the plan's
device error word must stay clear (no index check failed)."""
import dataclasses
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

from hyena_cases import (compare, compare_2d, compare_gated_2d, explicit_case, explicit_case_2d,  # noqa: E402
                         oracle_filters_1d, oracle_kernels_2d, to_gpu)
from long_convolution_sequence_hyena_b200 import api, capi  # noqa: E402
from long_convolution_sequence_hyena_b200.workloads import make_inputs  # noqa: E402

assert capi.LIB_PATH.endswith("libhyena_checked.so"), capi.LIB_PATH


def clean(plan, what):
    st, flags = capi.hyena_plan_device_errors(plan.handle, clear=True)
    assert st == capi.HYENA_OK and flags == 0, "%s: device error word %d" % (what, flags)


def run_1d(B, D, L, N, dtype, path, seed):
    w = explicit_case(B, D, L, N, dtype, seed=seed, alpha=(1e-4, 1e-2))
    inp = make_inputs(w)
    g = to_gpu(inp)
    plan = api.Plan((L,), D, N, torch.float32 if dtype == "f32" else torch.bfloat16)
    assert plan.path == path, (L, plan.path)
    H = plan.filter_spectrum(h=g["h"])
    y = plan.forward(g["v"], g["gates"], H, g["dskip"])
    torch.cuda.synchronize()
    what = "1d B%d D%d L%d N%d %s" % (B, D, L, N, dtype)
    clean(plan, what)
    compare(w, inp, oracle_filters_1d(w, inp), y, context=what)
    plan.close()


def run_2d(B, C, Hw, N, dtype, gated, seed):
    w = explicit_case_2d(B, C, Hw, N, dtype, seed=seed)
    if gated:
        w = dataclasses.replace(w, gated=True)
    inp = make_inputs(w)
    g = to_gpu(inp)
    plan = api.Plan((Hw, Hw), C, N, torch.float32 if dtype == "f32" else torch.bfloat16)
    H = plan.filter_spectrum(h=g["h"])
    if gated:
        y = plan.forward_gated(g["v"], inp["k"].cuda(), g["gates"], H, g["dskip"])
    else:
        y = plan.forward(g["v"], g["gates"], H, g["dskip"])
    torch.cuda.synchronize()
    what = "2d B%d C%d %d N%d %s%s" % (B, C, Hw, N, dtype, " gated" if gated else "")
    clean(plan, what)
    k64 = oracle_kernels_2d(w, inp)
    (compare_gated_2d if gated else compare_2d)(w, inp, k64, y, context=what)
    plan.close()


CTA, STAGED = capi.HYENA_PATH_CTA, capi.HYENA_PATH_STAGED
for i, (B, D, L, N, dt, path) in enumerate([
    (1, 3, 1, 1, "f32", CTA), (3, 2, 3, 2, "f32", CTA), (1, 5, 255, 3, "bf16", CTA),
    (3, 3, 1000, 2, "f32", CTA),        # one row per thread group
    (2, 3, 2047, 2, "bf16", CTA),       # two rows of a channel per thread group
    (4, 2, 4096, 1, "f32", CTA),
    (1, 3, 16385, 2, "f32", STAGED),    # M = 65536: three rows, one chunk, odd count
    (1, 5, 40001, 1, "bf16", STAGED),   # M = 131072
    (2, 1, 65536, 3, "bf16", STAGED),
]):
    run_1d(B, D, L, N, dt, path, seed=7000 + i)
for i, (B, C, Hw, N, dt, gated) in enumerate([
    (1, 3, 32, 1, "f32", False), (2, 1, 64, 2, "bf16", False),
    (1, 3, 256, 1, "f32", False),       # staged 2D: three planes, odd count
    (2, 1, 256, 1, "bf16", True),
]):
    run_2d(B, C, Hw, N, dt, gated, seed=7100 + i)
print("OK")
