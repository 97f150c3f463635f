"""Channels-last activations ([B, L, D], the layout of u in "Hyena, Long
Convolution, and Linear Attention", "FFTConv"): a plan set to HYENA_LAYOUT_BLD
reads v and the gates and writes y in that layout directly. The oracle runs on
the same values transposed to [B, D, L]; every 1D kernel family is covered
(single-CTA rows, staged long rows, cluster rows), through hyena_forward, the
host-buffer forward and the no-alloc forward."""
import numpy as np
import pytest
import torch

from hyena_cases import compare, explicit_case, oracle_filters_1d, to_gpu
from long_convolution_sequence_hyena_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def _bld(x):
    """[..., B, D, L] -> [..., B, L, D] contiguous."""
    return x.transpose(-1, -2).contiguous()


def _bdl(x):
    return x.transpose(-1, -2).contiguous()


def _plan(w, layout="bld"):
    from long_convolution_sequence_hyena_b200 import api
    return api.Plan(w.shape, w.D, w.order, torch.float32 if w.dtype == "f32" else torch.bfloat16, layout=layout)


@pytest.mark.parametrize("L,B,D,N,dtype,path", [
    (2048, 2, 8, 2, "bf16", 0),
    (1000, 3, 5, 2, "f32", 0),       # odd channel count, ragged tail
    (7, 2, 3, 1, "f32", 0),
    (65536, 1, 6, 3, "bf16", 3),     # staged long rows: lanes are adjacent channels
    (40001, 2, 3, 2, "f32", 3),      # staged, odd length
    (100000, 1, 2, 1, "f32", 3),     # staged, M = 262144
])
def test_bld_forward_matches_oracle(L, B, D, N, dtype, path):
    w = explicit_case(B, D, L, N, dtype, seed=2000 + L % 97 + D, alpha=(1e-4, 1e-2) if L > 16384 else (1e-3, 1e-1))
    inp = make_inputs(w)
    g = to_gpu(inp)
    plan = _plan(w)
    assert plan.path == path
    H = plan.filter_spectrum(h=g["h"])
    v = _bld(g["v"])
    gates = [_bld(x) for x in g["gates"]]
    y = plan.forward(v, gates, H, g["dskip"])
    torch.cuda.synchronize()
    assert y.shape == (B, L, D)
    compare(w, inp, oracle_filters_1d(w, inp), _bdl(y), context="bld L=%d" % L)
    # the same call on a [B, D, L] plan gives the same values
    plan2 = _plan(w, "bdl")
    y2 = plan2.forward(g["v"], g["gates"], H, g["dskip"])
    torch.cuda.synchronize()
    a, b = _bdl(y).double().cpu(), y2.double().cpu()
    assert float(torch.linalg.vector_norm(a - b) / torch.linalg.vector_norm(b)) <= (1e-5 if dtype == "f32" else 2e-2)
    plan.close()
    plan2.close()


def test_bld_host_and_no_alloc_forwards():
    from long_convolution_sequence_hyena_b200 import capi
    w = explicit_case(2, 4, 32768, 2, "bf16", seed=2101, alpha=(1e-4, 1e-2))
    inp = make_inputs(w)
    g = to_gpu(inp)
    plan = _plan(w)
    H = plan.filter_spectrum(h=g["h"])
    v, gates = _bld(g["v"]), [_bld(x) for x in g["gates"]]
    ref = plan.forward(v, gates, H, g["dskip"])
    yh = plan.forward_host(v.cpu().pin_memory(), [x.cpu().pin_memory() for x in gates], H, g["dskip"])
    y0 = torch.empty_like(v)
    st = capi.hyena_forward_no_alloc(plan.handle, w.B, v.data_ptr(), [x.data_ptr() for x in gates], H.data_ptr(),
                                     g["dskip"].data_ptr(), y0.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == capi.HYENA_OK
    torch.cuda.synchronize()
    assert torch.equal(yh.cuda(), ref) and torch.equal(y0, ref)
    compare(w, inp, oracle_filters_1d(w, inp), _bdl(ref), rows=np.array([0, 3, 4, 7]), context="bld host/no-alloc")
    plan.close()


def test_bld_layout_rejected_on_2d_plans():
    from long_convolution_sequence_hyena_b200 import api, capi
    plan = api.Plan((32, 32), 2, 1, torch.float32)
    assert capi.hyena_plan_set_layout(plan.handle, capi.HYENA_LAYOUT_BLD) == capi.HYENA_ERR_UNSUPPORTED
    assert capi.hyena_plan_set_layout(plan.handle, 7) == capi.HYENA_ERR_INVALID_ARG
    plan.close()


@pytest.mark.parametrize("name,rows", [
    ("order2_bf16_b8_d768_l2048", [0, 767, 768, 3000, 6143]),
    ("order3_bf16_b1_d768_l65536", [0, 1, 383, 767]),
])
def test_bld_workloads_full_size_sampled_rows(name, rows):
    """The L = 2048 and L = 65536 workloads at full size in channels-last layout; sampled rows."""
    w = WORKLOADS[name]
    inp = make_inputs(w)
    g = to_gpu(inp)
    plan = _plan(w)
    H = plan.filter_spectrum(h=g["h"])
    y = plan.forward(_bld(g["v"]), [_bld(x) for x in g["gates"]], H, g["dskip"])
    torch.cuda.synchronize()
    compare(w, inp, oracle_filters_1d(w, inp), _bdl(y), rows=np.array(rows), context="bld " + name)
    plan.close()
