"""Rows beyond M = 262144 (L up to 524288, M up to 2^20) on the staged
four-step path, and the HYENA_FORCE_PATH override.

A full O(L^2) oracle row at these lengths takes minutes, so the checks use
what the operator's causality fixes exactly ("Hyena — Long Convolutions
Math", "The Toeplitz picture": y_t depends on inputs up to t only):
  * prefix window: y[0:T) equals the oracle on the first T positions;
  * tail window: with v zero before s = L - T, every z^n is zero there, and
    y[s:L) equals the oracle on the inputs shifted by s (filters cut to T);
  * order 1: sampled outputs anywhere, each by its own direct sum.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from hyena_cases import compare, explicit_case, oracle_filters_1d, to_gpu
from long_convolution_sequence_hyena_b200.workloads import make_inputs

pytestmark = pytest.mark.gpu

T = 3000
TOL = {"f32": 1e-5, "bf16": 2e-2}


def _run(w, inp):
    from long_convolution_sequence_hyena_b200 import api
    g = to_gpu(inp)
    plan = api.Plan(w.shape, w.D, w.order, torch.float32 if w.dtype == "f32" else torch.bfloat16)
    H = plan.filter_spectrum(h=g["h"])
    y = plan.forward(g["v"], g["gates"], H, g["dskip"])
    torch.cuda.synchronize()
    return plan, y.double().cpu().reshape(w.B * w.D, -1).numpy()


def _rows(w, inp):
    R, L, N = w.B * w.D, w.shape[0], w.order
    v = inp["v"].double().reshape(R, L).numpy()
    g = inp["gates"].double().reshape(N, R, L).numpy()
    return v, g, inp["h"].double().numpy(), inp["dskip"].double().numpy()


def _rel(got, ref):
    return np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)


@pytest.mark.parametrize("L,B,D,N,dtype", [
    (131073, 1, 2, 2, "f32"),     # M = 524288, odd length
    (262144, 1, 3, 3, "bf16"),    # M = 524288
    (300001, 2, 1, 1, "f32"),     # M = 1048576, odd
    (524288, 1, 2, 2, "bf16"),    # M = 1048576, the longest
])
def test_long_row_prefix_and_tail_windows(L, B, D, N, dtype):
    w = explicit_case(B, D, L, N, dtype, seed=3000 + L % 1009, alpha=(1e-5, 1e-3))
    inp = make_inputs(w)
    R = B * D
    s = L - T
    v = inp["v"].clone()
    v_tail = v.clone()
    v_tail[..., :s] = 0                           # the tail case: nothing before s
    plan = None
    for which, vv in (("prefix", v), ("tail", v_tail)):
        inp2 = dict(inp, v=vv)
        plan, y = _run(w, inp2)
        assert plan.path == 3 and plan.fft_len == 1 << (2 * L - 1).bit_length()
        vr, gr, h, dsk = _rows(w, inp2)
        fidx = np.arange(R) % D
        if which == "prefix":
            ref = oracle.hyena_1d(vr[:, :T], gr[:, :, :T], h[:, :, :T], dsk, fidx=fidx)
            got = y[:, :T]
        else:
            ref = oracle.hyena_1d(vr[:, s:], gr[:, :, s:], h[:, :, :T], dsk, fidx=fidx)
            got = y[:, s:]
            # before s the exact result is zero; the transform leaves only rounding there
            assert np.abs(y[:, :s]).max() <= 1e-4 * np.abs(y[:, s:]).max()
        err = _rel(got, ref)
        assert err <= TOL[dtype], (which, err)
        plan.close()


def test_long_row_order1_sampled_outputs():
    """Order 1 at L = 400000 (M = 2^20): outputs across the whole row, each by its direct sum."""
    L = 400000
    w = explicit_case(1, 2, L, 1, "f32", seed=3100, alpha=(1e-5, 1e-4))
    inp = make_inputs(w)
    plan, y = _run(w, inp)
    vr, gr, h, dsk = _rows(w, inp)
    rng = np.random.default_rng(3)
    pos = np.concatenate([[0, 1, L // 2, L - 2, L - 1], rng.integers(0, L, 40)])
    for r in range(2):
        ref = oracle.hyena_1d_order1_at(vr[r], gr[0, r], h[0, r], dsk[0, r], pos)
        err = _rel(y[r, pos], ref)
        assert err <= 1e-5, (r, err)
    plan.close()


@pytest.fixture
def force_path():
    old = os.environ.get("HYENA_FORCE_PATH")

    def set_(value):
        os.environ["HYENA_FORCE_PATH"] = value
    yield set_
    if old is None:
        os.environ.pop("HYENA_FORCE_PATH", None)
    else:
        os.environ["HYENA_FORCE_PATH"] = old


def test_forced_cluster_path_matches_oracle(force_path):
    """M = 262144 through the thread-block-cluster kernel (whole row on chip), forced."""
    force_path("cluster")
    w = explicit_case(1, 2, 100000, 2, "f32", seed=3200, alpha=(1e-4, 1e-2))
    inp = make_inputs(w)
    from long_convolution_sequence_hyena_b200 import api
    g = to_gpu(inp)
    plan = api.Plan(w.shape, w.D, w.order, torch.float32)
    assert plan.path == 1
    H = plan.filter_spectrum(h=g["h"])
    y = plan.forward(g["v"], g["gates"], H, g["dskip"])
    torch.cuda.synchronize()
    compare(w, inp, oracle_filters_1d(w, inp), y, context="forced cluster")
    plan.close()


def test_forced_path_rejections(force_path):
    from long_convolution_sequence_hyena_b200 import capi
    for value, L, expect in (("cta", 20000, capi.HYENA_ERR_UNSUPPORTED),      # M = 65536: no single-CTA kernel
                             ("staged", 1000, capi.HYENA_ERR_UNSUPPORTED),
                             ("cluster", 300000, capi.HYENA_ERR_UNSUPPORTED),
                             ("bogus", 1000, capi.HYENA_ERR_INVALID_ARG)):
        force_path(value)
        st, h = capi.hyena_plan_create(1, [L], 2, 1, capi.HYENA_F32, 1)
        assert st == expect and h is None, value
    force_path("staged")
    st, h = capi.hyena_plan_create(1, [100000], 2, 1, capi.HYENA_F32, 1)
    assert st == capi.HYENA_OK
    assert capi.hyena_plan_info(h)[3] == capi.HYENA_PATH_STAGED
    capi.hyena_plan_destroy(h)
