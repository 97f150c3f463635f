"""The implicit filter network with its head on the tensor cores (width 64:
3xTF32 tcgen05 MMAs, fp32 accumulation in tensor memory) against the fp64
network: ragged position tiles, several output slices and a ragged last
slice, 1D and 2D; a width that is not 64 takes the CUDA-core kernel and
must agree too. No bounded wait may have run out (the plan's device error
word stays 0)."""
import numpy as np
import pytest
import torch

import oracle
from hyena_cases import oracle_filters_1d, oracle_kernels_2d, to_gpu
from long_convolution_sequence_hyena_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def _max_rel(got, ref):
    return float(np.abs(got - ref).max() / np.abs(ref).max())


@pytest.mark.parametrize("L,D,N,width", [
    (1000, 300, 2, 64),     # 8 position tiles (the last ragged); 600 outputs: two CTA slices, ragged last MMA slice
    (8192, 1024, 2, 64),    # the implicit L = 8192 workload's network at full size
    (333, 5, 1, 32),        # width 32: the CUDA-core kernel
])
def test_implicit_1d(L, D, N, width):
    from long_convolution_sequence_hyena_b200 import api, capi
    base = WORKLOADS["order2_bf16_b4_d1024_l8192_implicit"]
    w = base.scaled(B=1, D=D, shape=(L,), order=N)
    import dataclasses
    w = dataclasses.replace(w, width=width)
    inp = make_inputs(w)
    g = to_gpu(inp)
    plan = api.Plan(w.shape, w.D, w.order, torch.bfloat16)
    h = plan.implicit_filter(g["implicit"])
    torch.cuda.synchronize()
    ref = oracle_filters_1d(w, inp)
    err = _max_rel(h.double().cpu().numpy(), ref)
    assert err < 1e-5, err
    st, flags = capi.hyena_plan_device_errors(plan.handle)
    assert st == capi.HYENA_OK and flags == 0
    plan.close()


@pytest.mark.parametrize("Hw,C", [(32, 3), (64, 130)])
def test_implicit_2d(Hw, C):
    from long_convolution_sequence_hyena_b200 import api, capi
    w = WORKLOADS["order1_bf16_2d_b2_c256_256x256"].scaled(B=1, D=C, shape=(Hw, Hw))
    inp = make_inputs(w)
    g = to_gpu(inp)
    plan = api.Plan(w.shape, w.D, w.order, torch.bfloat16)
    k = plan.implicit_filter(g["implicit"])
    torch.cuda.synchronize()
    ref = oracle_kernels_2d(w, inp)
    err = _max_rel(k.double().cpu().numpy(), ref)
    assert err < 1e-5, err
    st, flags = capi.hyena_plan_device_errors(plan.handle, clear=True)
    assert st == capi.HYENA_OK and flags == 0
    plan.close()
