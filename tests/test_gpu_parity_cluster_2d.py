"""GPU parity of the long-row paths (1D rows with M > 32768: staged and cluster)
and of the 2D cluster path against the fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

from hyena_cases import (compare, compare_2d, explicit_case, explicit_case_2d, oracle_filters_1d, oracle_kernels_2d,
                         to_gpu)
from long_convolution_sequence_hyena_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    from long_convolution_sequence_hyena_b200 import api as a
    return a


def long_path(plan):
    """Path the library takes for a 1D plan with M > 32768: the staged four-step path (the
    cluster kernel only when forced)."""
    return 3


def _run(api, w, inp):
    g = to_gpu(inp)
    plan = api.Plan(w.shape, w.D, w.order, torch.float32 if w.dtype == "f32" else torch.bfloat16)
    H = plan.filter_spectrum(h=g["h"]) if "h" in g else plan.filter_spectrum(implicit=g["implicit"])
    y = plan.forward(g["v"], g["gates"], H, g["dskip"])
    torch.cuda.synchronize()
    return plan, H, y


# ------------------------------------------------------------- 1D cluster --

@pytest.mark.parametrize("L", [16385, 32768, 40001, 65536, 100000, 131072])
def test_cluster_spectrum_matches_dft(api, L):
    w = explicit_case(1, 3, L, 1, "f32", seed=L, alpha=(1e-4, 1e-2))
    inp = make_inputs(w)
    plan = api.Plan((L,), 3, 1, torch.float32)
    assert plan.path == long_path(plan)
    H = plan.filter_spectrum(h=inp["h"].cuda())
    torch.cuda.synchronize()
    ref = np.fft.rfft(inp["h"].double().numpy(), n=plan.fft_len, axis=-1)
    err = np.abs(H.cpu().numpy().astype(np.complex128) - ref).max() / np.abs(inp["h"].double().numpy()).sum(-1).max()
    assert err < 2e-6, (L, err)


@pytest.mark.parametrize("L,N,dtype", [(16385, 2, "f32"), (32768, 2, "f32"), (40001, 1, "bf16"),
                                       (65536, 1, "f32"), (100000, 1, "f32"), (131072, 1, "bf16")])
def test_cluster_lengths(api, L, N, dtype):
    w = explicit_case(1, 2, L, N, dtype, seed=500 + L, alpha=(1e-4, 1e-2))
    inp = make_inputs(w)
    plan, _, y = _run(api, w, inp)
    assert plan.path == long_path(plan)
    compare(w, inp, oracle_filters_1d(w, inp), y, context="long row L=%d N=%d" % (L, N))


@pytest.mark.parametrize("L,B,D,N,dtype", [(16385, 3, 1, 2, "f32"), (40001, 1, 3, 1, "bf16"), (32768, 2, 3, 1, "f32"),
                                         (65536, 2, 1, 1, "f32")])
def test_cluster_batches_and_channels(api, L, B, D, N, dtype):
    """Cluster rows over several batches and channels: odd row counts, B = 1, B odd and B even
    (rows are visited d-major, b-minor)."""
    w = explicit_case(B, D, L, N, dtype, seed=700 + L + B, alpha=(1e-4, 1e-2))
    inp = make_inputs(w)
    plan, _, y = _run(api, w, inp)
    assert plan.path == long_path(plan)
    compare(w, inp, oracle_filters_1d(w, inp), y, context="long row L=%d B=%d D=%d" % (L, B, D))


def test_staged_chunks(api):
    """More rows than one workspace chunk holds (M = 65536: 64 rows per 16 MB chunk, three
    chunks in flight on three streams); rows on both sides of the chunk boundaries are checked."""
    w = explicit_case(2, 150, 16385, 2, "bf16", seed=1234, alpha=(1e-4, 1e-2))
    inp = make_inputs(w)
    plan, _, y = _run(api, w, inp)
    assert plan.path == 3 and plan.workspace_bytes(2) == 3 * 64 * 32768 * 8
    # visit order is d-major, b-minor: visit index o -> flat row (o % B) * D + o // B
    visits = np.array([0, 1, 63, 64, 127, 128, 191, 192, 255, 256, 298, 299])
    rows = (visits % 2) * 150 + visits // 2
    compare(w, inp, oracle_filters_1d(w, inp), y, rows=rows, context="staged chunks")


def test_staged_workspace_checks(api):
    from long_convolution_sequence_hyena_b200 import capi
    plan = api.Plan((65536,), 2, 1, torch.bfloat16)
    need = plan.workspace_bytes(3)
    assert plan.path == 3 and need == 6 * 65536 * 8
    v = torch.zeros(3, 2, 65536, dtype=torch.bfloat16, device="cuda")
    H = torch.zeros(plan.spectrum_shape, dtype=torch.complex64, device="cuda")
    ws = torch.empty(need + 16, dtype=torch.uint8, device="cuda")
    args = (plan.handle, 3, v.data_ptr(), [v.data_ptr()], H.data_ptr(), None, v.data_ptr())
    assert capi.hyena_forward(*args, None, 0) == capi.HYENA_ERR_WORKSPACE
    assert capi.hyena_forward(*args, ws.data_ptr(), need - 8) == capi.HYENA_ERR_WORKSPACE
    assert capi.hyena_forward(*args, ws.data_ptr() + 8, need) == capi.HYENA_ERR_ALIGNMENT
    assert capi.hyena_forward(*args, ws.data_ptr(), need) == capi.HYENA_OK
    torch.cuda.synchronize()
    assert plan.workspace_bytes(0) == 0 and api.Plan((8192,), 2, 1).workspace_bytes(3) == 0


def test_cluster_implicit_in_place(api):
    w = WORKLOADS["order2_bf16_b4_d1024_l8192_implicit"].scaled(B=1, D=2, shape=(20000,))
    inp = make_inputs(w)
    g = to_gpu(inp)
    plan = api.Plan(w.shape, w.D, w.order, torch.bfloat16)
    h = plan.implicit_filter(g["implicit"])
    H1 = plan.filter_spectrum(h=h)
    H2 = plan.filter_spectrum(implicit=g["implicit"])
    torch.cuda.synchronize()
    assert torch.equal(H1, H2)
    y = plan.forward(g["v"], g["gates"], H2, g["dskip"])
    torch.cuda.synchronize()
    compare(w, inp, oracle_filters_1d(w, inp), y, context="cluster implicit")


def test_order3_long_workload_full_size_sampled_rows(api):
    """The order-3 bf16 B=1 D=768 L=65536 workload at full size; the oracle checks sampled rows."""
    w = WORKLOADS["order3_bf16_b1_d768_l65536"]
    inp = make_inputs(w)
    _, _, y = _run(api, w, inp)
    rows = np.array([0, 1, 383, 766, 767, 100, 500, 250])
    compare(w, inp, oracle_filters_1d(w, inp), y, rows=rows, context="order3 L=65536 sampled")


# --------------------------------------------------------------------- 2D --

@pytest.mark.parametrize("Hw", [32, 64, 128, 256])
def test_2d_spectrum_matches_dft(api, Hw):
    w = explicit_case_2d(1, 2, Hw, 1, "f32", seed=Hw)
    inp = make_inputs(w)
    plan = api.Plan((Hw, Hw), 2, 1, torch.float32)
    assert plan.path == 2
    K = plan.filter_spectrum(h=inp["h"].cuda())
    torch.cuda.synchronize()
    k64 = inp["h"].double().numpy()
    cyc = np.roll(k64, shift=(-Hw, -Hw), axis=(-2, -1))     # offset o at index o mod 2H, o mod 2W
    ref = np.fft.rfft2(cyc)                                   # [.., ky, kx]; the library stores [.., kx, ky]
    assert K.shape[-2:] == (Hw + 1, 2 * Hw)
    err = np.abs(K.transpose(-1, -2).cpu().numpy().astype(np.complex128) - ref).max() / np.abs(k64).sum(axis=(-2, -1)).max()
    assert err < 2e-6, (Hw, err)


@pytest.mark.parametrize("Hw,B,C,N,dtype", [(32, 2, 3, 1, "f32"), (32, 1, 2, 2, "f32"), (64, 2, 2, 1, "f32"),
                                            (64, 1, 3, 2, "bf16"), (128, 1, 2, 1, "f32"), (128, 1, 2, 2, "bf16"),
                                            (256, 1, 2, 1, "f32"), (256, 3, 1, 2, "bf16")])
def test_2d_parity(api, Hw, B, C, N, dtype):
    w = explicit_case_2d(B, C, Hw, N, dtype, seed=900 + Hw + N)
    inp = make_inputs(w)
    _, _, y = _run(api, w, inp)
    compare_2d(w, inp, oracle_kernels_2d(w, inp), y, context="2d %d N=%d %s" % (Hw, N, dtype))


def test_2d_implicit_kernel_matches_oracle(api):
    w = WORKLOADS["order1_bf16_2d_b2_c256_256x256"].scaled(B=1, D=4, shape=(64, 64))
    inp = make_inputs(w)
    g = to_gpu(inp)
    plan = api.Plan(w.shape, w.D, w.order, torch.bfloat16)
    k = plan.implicit_filter(g["implicit"])
    torch.cuda.synchronize()
    ref = oracle_kernels_2d(w, inp)
    err = np.abs(k.cpu().double().numpy() - ref).max() / np.abs(ref).max()
    assert err < 1e-5, err
    K1 = plan.filter_spectrum(h=k)
    K2 = plan.filter_spectrum(implicit=g["implicit"])
    torch.cuda.synchronize()
    assert torch.equal(K1, K2)
    y = plan.forward(g["v"], g["gates"], K2, g["dskip"])
    torch.cuda.synchronize()
    compare_2d(w, inp, ref, y, context="2d implicit 64")


def test_2d_workload_full_size_sampled_planes(api):
    """The 2D order-1 bf16 B=2 C=256 256x256 workload at full size; sampled planes."""
    w = WORKLOADS["order1_bf16_2d_b2_c256_256x256"]
    inp = make_inputs(w)
    _, _, y = _run(api, w, inp)
    planes = np.array([0, 1, 255, 256, 511, 77, 300, 420])
    compare_2d(w, inp, oracle_kernels_2d(w, inp), y, planes=planes, context="2d workload sampled")
