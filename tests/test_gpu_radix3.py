"""Plans with HYENA_PLAN_RADIX3 pad to M = 6 * 2^j when that is below the power
of two ("Hyena — Long Convolutions Math", "Linear vs circular": any transform
of at least 2L points keeps the product causal), and run a radix-3 step and
three power-of-two transforms. The result does not depend on M: parity with
the fp64 oracle as for every other length; the spectra against numpy's DFT of
the taps on M points."""
import numpy as np
import pytest
import torch

from hyena_cases import compare, explicit_case, oracle_filters_1d, to_gpu
from long_convolution_sequence_hyena_b200.workloads import make_inputs

pytestmark = pytest.mark.gpu

CASES = [   # L, expected M
    (40, 96), (1500, 3072), (3000, 6144), (3001, 6144), (5000, 12288), (12288, 24576),
]


def _plan(w, radix3=True):
    from long_convolution_sequence_hyena_b200 import api
    return api.Plan(w.shape, w.D, w.order, torch.float32 if w.dtype == "f32" else torch.bfloat16, radix3=radix3)


@pytest.mark.parametrize("L,M", CASES)
def test_radix3_length_choice_and_spectrum(L, M):
    w = explicit_case(1, 3, L, 2, "f32", seed=5000 + L)
    inp = make_inputs(w)
    plan = _plan(w)
    assert plan.fft_len == M and plan.path == 0 and plan.spectrum_elems == M // 2 + 1
    H = plan.filter_spectrum(h=inp["h"].cuda())
    torch.cuda.synchronize()
    ref = np.fft.rfft(inp["h"].double().numpy(), n=M, axis=-1)
    err = np.abs(H.cpu().numpy().astype(np.complex128) - ref).max() / np.abs(inp["h"].double().numpy()).sum(-1).max()
    assert err < 2e-6, err
    plan.close()


@pytest.mark.parametrize("L,B,D,N,dtype", [
    (40, 2, 3, 1, "f32"), (1500, 1, 4, 2, "f32"), (3000, 2, 3, 2, "bf16"), (3001, 3, 2, 3, "f32"),
    (5000, 1, 2, 2, "bf16"), (12288, 1, 2, 1, "f32"),
])
def test_radix3_forward_matches_oracle(L, B, D, N, dtype):
    w = explicit_case(B, D, L, N, dtype, seed=5100 + L + N)
    inp = make_inputs(w)
    g = to_gpu(inp)
    plan = _plan(w)
    assert plan.fft_len % 3 == 0
    H = plan.filter_spectrum(h=g["h"])
    y = plan.forward(g["v"], g["gates"], H, g["dskip"])
    torch.cuda.synchronize()
    compare(w, inp, oracle_filters_1d(w, inp), y, context="radix3 L=%d" % L)
    plan.close()


def test_radix3_channels_last_and_implicit():
    """The channels-last layout and the implicit filter path on a radix-3 plan."""
    from long_convolution_sequence_hyena_b200 import api
    from long_convolution_sequence_hyena_b200.workloads import WORKLOADS
    w = WORKLOADS["order2_bf16_b4_d1024_l8192_implicit"].scaled(B=2, D=4, shape=(3000,))
    inp = make_inputs(w)
    g = to_gpu(inp)
    plan = api.Plan(w.shape, w.D, w.order, torch.bfloat16, layout="bld", radix3=True)
    assert plan.fft_len == 6144
    H = plan.filter_spectrum(implicit=g["implicit"])
    y = plan.forward(g["v"].transpose(1, 2).contiguous(), [x.transpose(1, 2).contiguous() for x in g["gates"]], H,
                     g["dskip"])
    torch.cuda.synchronize()
    compare(w, inp, oracle_filters_1d(w, inp), y.transpose(1, 2).contiguous(), context="radix3 bld implicit")
    plan.close()
