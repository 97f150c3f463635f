"""GPU parity of the 3D grid path (HyenaND on a volume: "How HyenaND works",
"2. The convolution theorem (FFT)") against the fp64 direct-sum oracle: the
plain chain and the gate sandwich, fp32 and bf16, cubic and non-cubic grids,
chunks of volumes; the kernel spectra against numpy's 3D DFT; the implicit
network on 3D coordinates against its fp64 evaluation."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from hyena_cases import case_3d, compare_3d, inputs_3d

pytestmark = pytest.mark.gpu


def _plan(w):
    from long_convolution_sequence_hyena_b200 import api
    return api.Plan(w.shape, w.D, w.order, torch.float32 if w.dtype == "f32" else torch.bfloat16)


@pytest.mark.parametrize("shape", [(16, 16, 16), (32, 16, 64), (64, 32, 16)])
def test_3d_spectrum_matches_numpy_fftn(shape):
    w = case_3d(1, 2, shape, 1, "f32", seed=sum(shape))
    inp = inputs_3d(w)
    plan = _plan(w)
    assert plan.path == 4 and plan.spectrum_shape == (1, 2) + tuple(2 * e for e in shape)
    K = plan.filter_spectrum(h=inp["h"].cuda())
    torch.cuda.synchronize()
    k64 = inp["h"].double().numpy()
    cyc = np.roll(k64, shift=tuple(-e for e in shape), axis=(-3, -2, -1))   # offset o at index o mod 2 extent
    ref = np.fft.fftn(cyc, axes=(-3, -2, -1))
    err = np.abs(K.cpu().numpy().astype(np.complex128) - ref).max() / np.abs(k64).sum(axis=(-3, -2, -1)).max()
    assert err < 2e-6, err
    plan.close()


@pytest.mark.parametrize("shape,B,C,N,dtype", [
    ((16, 16, 16), 1, 3, 1, "f32"),
    ((16, 16, 16), 2, 2, 2, "f32"),
    ((32, 16, 64), 1, 2, 1, "bf16"),
    ((16, 32, 32), 2, 1, 2, "bf16"),
    ((32, 32, 32), 1, 2, 1, "f32"),
])
def test_3d_parity(shape, B, C, N, dtype):
    w = case_3d(B, C, shape, N, dtype, seed=4000 + sum(shape) + N)
    inp = inputs_3d(w)
    plan = _plan(w)
    H = plan.filter_spectrum(h=inp["h"].cuda())
    y = plan.forward(inp["v"].cuda(), [g.cuda() for g in inp["gates"]], H, inp["dskip"].cuda())
    torch.cuda.synchronize()
    compare_3d(w, inp, inp["h"].double().numpy(), y, context="3d %s N=%d %s" % (shape, N, dtype))
    plan.close()


def test_3d_gated_parity():
    w = case_3d(2, 2, (16, 32, 16), 1, "f32", seed=4100)
    inp = inputs_3d(w)
    plan = _plan(w)
    H = plan.filter_spectrum(h=inp["h"].cuda())
    y = plan.forward_gated(inp["v"].cuda(), inp["k"].cuda(), [g.cuda() for g in inp["gates"]], H,
                           inp["dskip"].cuda())
    torch.cuda.synchronize()
    compare_3d(w, inp, inp["h"].double().numpy(), y, gated=True, context="3d gated")
    plan.close()


def test_3d_chunks_and_large_grid_sampled_voxels():
    """64^3 volumes (8 MB of workspace each, four per chunk): 9 volumes span three chunks; order-1
    outputs at sampled voxels against their own direct sums."""
    w = case_3d(3, 3, (64, 64, 64), 1, "bf16", seed=4200)
    inp = inputs_3d(w)
    plan = _plan(w)
    assert plan.workspace_bytes(3) == 4 * 64 * 128 * 128 * 8
    H = plan.filter_spectrum(h=inp["h"].cuda())
    y = plan.forward(inp["v"].cuda(), [g.cuda() for g in inp["gates"]], H, inp["dskip"].cuda())
    torch.cuda.synchronize()
    rng = np.random.default_rng(9)
    vox = [(0, 0, 0), (63, 63, 63), (31, 5, 60)] + [tuple(rng.integers(0, 64, 3)) for _ in range(5)]
    P = 9
    v = inp["v"].double().reshape(P, 64, 64, 64).numpy()
    x = inp["gates"].double().reshape(1, P, 64, 64, 64).numpy()[0]
    got = y.double().cpu().reshape(P, 64, 64, 64).numpy()
    ref, val = [], []
    for p in (0, 4, 8):
        c = p % 3
        ref += list(oracle.hyena_3d_order1_at(v[p], x[p], inp["h"][0, c].double().numpy(),
                                              float(inp["dskip"][0, c]), vox))
        val += [got[p][i] for i in vox]
    ref, val = np.array(ref), np.array(val)
    err = np.linalg.norm(val - ref) / np.linalg.norm(ref)
    assert err <= 2e-2, err
    plan.close()


def test_3d_implicit_network_matches_oracle():
    from long_convolution_sequence_hyena_b200 import capi
    from long_convolution_sequence_hyena_b200.workloads import WORKLOADS, make_inputs
    base = WORKLOADS["order1_bf16_2d_b2_c256_256x256"].scaled(B=1, D=3, shape=(16, 16))
    p = make_inputs(base)["implicit"]
    g = torch.Generator().manual_seed(11)
    p = dict(p, W1=torch.randn(64, 3, generator=g) / 8.0)       # three input coordinates
    w = case_3d(1, 3, (16, 32, 16), 1, "f32", seed=1)
    plan = _plan(w)
    dev = {k: (x.cuda() if torch.is_tensor(x) else x) for k, x in p.items()}
    k = plan.implicit_filter(dev)
    torch.cuda.synchronize()
    names = ("W1", "b1", "W2", "b2", "W3", "b3")
    ref = oracle.implicit_filter_3d(16, 32, 16, 1, 3, *(p[n].double().numpy() for n in names),
                                    p["sigma"].double().numpy(), p["omega0"], p["omega_hidden"])
    assert k.shape == ref.shape
    err = float(np.abs(k.double().cpu().numpy() - ref).max() / np.abs(ref).max())
    assert err < 1e-5, err
    assert capi.hyena_plan_device_errors(plan.handle)[0] == capi.HYENA_OK
    plan.close()
