"""GPU parity of the 1D path against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

from hyena_cases import compare, explicit_case, oracle_filters_1d, to_gpu
from long_convolution_sequence_hyena_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    from long_convolution_sequence_hyena_b200 import api as a
    return a


def _run(api, w, inp, g=None):
    g = g or to_gpu(inp)
    plan = api.Plan(w.shape, w.D, w.order, torch.float32 if w.dtype == "f32" else torch.bfloat16)
    if "h" in g:
        H = plan.filter_spectrum(h=g["h"])
    else:
        H = plan.filter_spectrum(implicit=g["implicit"])
    y = plan.forward(g["v"], g["gates"], H, g["dskip"])
    torch.cuda.synchronize()
    return plan, H, y


def test_spectrum_matches_dft():
    """Filter spectra equal the fp64 DFT of the zero-padded taps (fp32 rounding)."""
    from long_convolution_sequence_hyena_b200 import api
    for L in (1, 7, 256, 1000, 2048, 8192, 16384):
        w = explicit_case(1, 6, L, 2, "f32", seed=L)
        inp = make_inputs(w)
        plan = api.Plan((L,), 6, 2, torch.float32)
        H = plan.filter_spectrum(h=inp["h"].cuda())
        torch.cuda.synchronize()
        M = plan.fft_len
        ref = np.fft.rfft(inp["h"].double().numpy(), n=M, axis=-1)
        got = H.cpu().numpy().astype(np.complex128)
        assert got.shape == ref.shape
        err = np.abs(got - ref).max() / np.abs(inp["h"].double().numpy()).sum(axis=-1).max()
        assert err < 2e-6, (L, err)


@pytest.mark.parametrize("L", [1, 2, 3, 5, 16, 17, 31, 100, 255, 256, 257, 1000, 1023, 2048, 3001, 4096, 8192, 16384])
def test_lengths_fp32(api, L):
    w = explicit_case(2, 3, L, 2, "f32", seed=100 + L)
    inp = make_inputs(w)
    _, _, y = _run(api, w, inp)
    compare(w, inp, oracle_filters_1d(w, inp), y, context="L=%d" % L)


@pytest.mark.parametrize("N", [1, 2, 3, 4, 8])
def test_orders(api, N):
    w = explicit_case(2, 5, 600, N, "f32", seed=200 + N)
    inp = make_inputs(w)
    _, _, y = _run(api, w, inp)
    compare(w, inp, oracle_filters_1d(w, inp), y, context="N=%d" % N)


@pytest.mark.parametrize("L", [1, 3, 64, 255, 2048, 8191, 16384])
def test_lengths_bf16(api, L):
    w = explicit_case(3, 4, L, 3, "bf16", seed=300 + L)
    inp = make_inputs(w)
    _, _, y = _run(api, w, inp)
    assert y.dtype == torch.bfloat16
    compare(w, inp, oracle_filters_1d(w, inp), y, context="bf16 L=%d" % L)


def test_many_rows_small_length(api):
    """Rows packed several per CTA, with a ragged last CTA."""
    w = explicit_case(3, 37, 40, 2, "f32", seed=7)
    inp = make_inputs(w)
    _, _, y = _run(api, w, inp)
    compare(w, inp, oracle_filters_1d(w, inp), y, context="many rows")


def test_no_feedthrough_and_unit_gates(api):
    w = explicit_case(1, 4, 500, 2, "f32", seed=8)
    inp = make_inputs(w)
    inp["gates"] = torch.ones_like(inp["gates"])
    g = to_gpu(inp)
    plan = api.Plan(w.shape, w.D, w.order, torch.float32)
    H = plan.filter_spectrum(h=g["h"])
    y = plan.forward(g["v"], g["gates"], H, None)
    torch.cuda.synchronize()
    inp["dskip"] = torch.zeros_like(inp["dskip"])
    compare(w, inp, oracle_filters_1d(w, inp), y, context="no feedthrough")


def test_output_may_alias_input(api):
    w = explicit_case(2, 8, 1000, 2, "bf16", seed=9)
    inp = make_inputs(w)
    g = to_gpu(inp)
    plan = api.Plan(w.shape, w.D, w.order, torch.bfloat16)
    H = plan.filter_spectrum(h=g["h"])
    ref = plan.forward(g["v"], g["gates"], H, g["dskip"])
    plan.forward(g["v"], g["gates"], H, g["dskip"], out=g["v"])
    torch.cuda.synchronize()
    assert torch.equal(ref, g["v"])


def test_batch_zero_and_repeatability(api):
    w = explicit_case(4, 16, 2048, 2, "bf16", seed=10)
    inp = make_inputs(w)
    g = to_gpu(inp)
    plan = api.Plan(w.shape, w.D, w.order, torch.bfloat16)
    H = plan.filter_spectrum(h=g["h"])
    empty = torch.empty((0, 16, 2048), dtype=torch.bfloat16, device="cuda")
    plan.forward(empty, [empty, empty], H, g["dskip"])
    y1 = plan.forward(g["v"], g["gates"], H, g["dskip"])
    y2 = plan.forward(g["v"], g["gates"], H, g["dskip"])
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_implicit_filter_matches_oracle(api):
    w = WORKLOADS["order2_bf16_b4_d1024_l8192_implicit"].scaled(B=1, D=16, shape=(1000,))
    inp = make_inputs(w)
    g = to_gpu(inp)
    plan = api.Plan(w.shape, w.D, w.order, torch.bfloat16)
    h = plan.implicit_filter(g["implicit"])
    torch.cuda.synchronize()
    ref = oracle_filters_1d(w, inp)
    err = np.abs(h.cpu().double().numpy() - ref).max() / np.abs(ref).max()
    assert err < 1e-5, err
    # the in-place implicit spectrum equals the spectrum of the materialised taps
    H1 = plan.filter_spectrum(h=h)
    H2 = plan.filter_spectrum(implicit=g["implicit"])
    torch.cuda.synchronize()
    assert torch.equal(H1, H2)


@pytest.mark.parametrize("name", ["order2_f32_b1_d4_l256"])
def test_workload_full(api, name):
    w = WORKLOADS[name]
    inp = make_inputs(w)
    _, _, y = _run(api, w, inp)
    compare(w, inp, oracle_filters_1d(w, inp), y, context=name)


@pytest.mark.parametrize("name,B,D", [
    ("order2_bf16_b8_d768_l2048", 2, 40),
    ("order2_bf16_b4_d1024_l8192_implicit", 2, 12),
])
def test_workload_scaled(api, name, B, D):
    w = WORKLOADS[name].scaled(B=B, D=D)
    inp = make_inputs(w)
    _, _, y = _run(api, w, inp)
    compare(w, inp, oracle_filters_1d(w, inp), y, context=name + " scaled")


@pytest.mark.parametrize("name", ["order2_bf16_b8_d768_l2048", "order2_bf16_b4_d1024_l8192_implicit"])
def test_workload_full_size_sampled_rows(api, name):
    """Full-size launch (as the benchmark runs it); the oracle checks sampled rows."""
    w = WORKLOADS[name]
    inp = make_inputs(w)
    _, _, y = _run(api, w, inp)
    R = w.B * w.D
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, 1, w.D - 1, w.D, R - 2, R - 1], rng.choice(R, 58, replace=False)]))
    compare(w, inp, oracle_filters_1d(w, inp), y, rows=rows, context=name + " sampled")
