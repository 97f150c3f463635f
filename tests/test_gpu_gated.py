"""GPU parity of the HyenaND gate sandwich (hyena_forward_gated) against the
fp64 oracle: z^0 = q ⊙ SiLU(k), z^n = SiLU(x^n) ⊙ (K^n ∗ z^{n-1} + Dskip^n z^{n-1})
("How HyenaND works", "Putting it together: the HyenaND operator"), on both 2D
kernel families (cluster, grids 32..128; staged, 256 x 256)."""
import dataclasses

import numpy as np
import pytest
import torch

from hyena_cases import compare_gated_2d, explicit_case_2d, oracle_kernels_2d, to_gpu
from long_convolution_sequence_hyena_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def _run_gated(w, inp):
    from long_convolution_sequence_hyena_b200 import api
    g = to_gpu(inp)
    plan = api.Plan(w.shape, w.D, w.order, torch.float32 if w.dtype == "f32" else torch.bfloat16)
    H = plan.filter_spectrum(h=g["h"]) if "h" in g else plan.filter_spectrum(implicit=g["implicit"])
    y = plan.forward_gated(g["v"], inp["k"].cuda(), g["gates"], H, g["dskip"])
    torch.cuda.synchronize()
    return plan, y


@pytest.mark.parametrize("Hw,B,C,N,dtype", [(32, 1, 3, 1, "f32"), (64, 2, 2, 2, "f32"), (64, 1, 3, 1, "bf16"),
                                            (128, 1, 2, 1, "f32"), (256, 1, 2, 1, "f32"), (256, 2, 35, 1, "bf16"),
                                            (256, 1, 2, 2, "f32")])
def test_gated_2d_parity(Hw, B, C, N, dtype):
    w = dataclasses.replace(explicit_case_2d(B, C, Hw, N, dtype, seed=1300 + Hw + N), gated=True)
    inp = make_inputs(w)
    plan, y = _run_gated(w, inp)
    compare_gated_2d(w, inp, oracle_kernels_2d(w, inp), y, context="gated 2d %d N=%d %s" % (Hw, N, dtype))
    plan.close()


def test_gated_without_feedthrough_is_the_page_sandwich():
    """Dskip = NULL, one order: O = (K ∗ (q ⊙ SiLU(k))) ⊙ SiLU(v), v the single gate."""
    from long_convolution_sequence_hyena_b200 import api
    w = dataclasses.replace(explicit_case_2d(1, 2, 64, 1, "f32", seed=1400), gated=True)
    inp = make_inputs(w)
    g = to_gpu(inp)
    plan = api.Plan(w.shape, w.D, 1, torch.float32)
    H = plan.filter_spectrum(h=g["h"])
    y = plan.forward_gated(g["v"], inp["k"].cuda(), g["gates"], H, None)
    torch.cuda.synchronize()
    inp = dict(inp, dskip=torch.zeros_like(inp["dskip"]))
    compare_gated_2d(w, inp, oracle_kernels_2d(w, inp), y, context="page sandwich")
    plan.close()


def test_gated_rejects_1d_plans_and_missing_key():
    from long_convolution_sequence_hyena_b200 import api, capi
    plan = api.Plan((1024,), 2, 1, torch.float32)
    x = torch.zeros(1, 2, 1024, device="cuda")
    H = torch.zeros(plan.spectrum_shape, dtype=torch.complex64, device="cuda")
    assert capi.hyena_forward_gated(plan.handle, 1, x.data_ptr(), x.data_ptr(), [x.data_ptr()], H.data_ptr(),
                                    None, x.data_ptr()) == capi.HYENA_ERR_UNSUPPORTED
    plan2 = api.Plan((32, 32), 2, 1, torch.float32)
    x2 = torch.zeros(1, 2, 32, 32, device="cuda")
    H2 = torch.zeros(plan2.spectrum_shape, dtype=torch.complex64, device="cuda")
    assert capi.hyena_forward_gated(plan2.handle, 1, x2.data_ptr(), None, [x2.data_ptr()], H2.data_ptr(),
                                    None, x2.data_ptr()) == capi.HYENA_ERR_INVALID_ARG
    plan.close()
    plan2.close()


def test_gated_workload_full_size_sampled_planes():
    """The gated B=2 C=256 256x256 bf16 workload (implicit kernels) at full size; sampled planes."""
    w = WORKLOADS["gated_order1_bf16_2d_b2_c256_256x256"]
    inp = make_inputs(w)
    plan, y = _run_gated(w, inp)
    planes = np.array([0, 1, 255, 256, 511, 130])
    compare_gated_2d(w, inp, oracle_kernels_2d(w, inp), y, planes=planes, context="gated workload sampled")
    plan.close()
