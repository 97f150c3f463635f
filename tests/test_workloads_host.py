"""The seeded input recipe (CPU): the named workloads have the stated sizes, and
the drawn inputs have the stated dtypes, distributions and parameter ranges,
reproducibly per seed."""
import math

import pytest
import torch

from long_convolution_sequence_hyena_b200.workloads import WORKLOADS, make_inputs

STATED = {   # name: (ndim, B, D, shape, order, dtype, filter kind)
    "order2_f32_b1_d4_l256": (1, 1, 4, (256,), 2, "f32", "explicit"),
    "order2_bf16_b8_d768_l2048": (1, 8, 768, (2048,), 2, "bf16", "explicit"),
    "order2_bf16_b4_d1024_l8192_implicit": (1, 4, 1024, (8192,), 2, "bf16", "implicit1d"),
    "order3_bf16_b1_d768_l65536": (1, 1, 768, (65536,), 3, "bf16", "explicit"),
    "order1_bf16_2d_b2_c256_256x256": (2, 2, 256, (256, 256), 1, "bf16", "implicit2d"),
    "gated_order1_bf16_2d_b2_c256_256x256": (2, 2, 256, (256, 256), 1, "bf16", "implicit2d"),
    "order3_bf16_b1_d768_l65536_bld": (1, 1, 768, (65536,), 3, "bf16", "explicit"),
}


def test_bld_workload_is_the_transposed_recipe():
    import dataclasses
    w = WORKLOADS["order3_bf16_b1_d768_l65536_bld"].scaled(B=2, D=3, shape=(64,))
    a, b = make_inputs(w), make_inputs(dataclasses.replace(w, layout="bdl"))
    assert a["v"].shape == (2, 64, 3) and a["gates"].shape == (3, 2, 64, 3)
    assert torch.equal(a["v"], b["v"].transpose(1, 2)) and torch.equal(a["gates"], b["gates"].transpose(2, 3))
    assert torch.equal(a["h"], b["h"])


def test_gated_workload_draws_k_last():
    """The gate sandwich's key k is drawn after every other tensor: the other tensors follow
    the plain recipe for the same seed, and k is N(0, 1) in the activation dtype."""
    import dataclasses
    w = WORKLOADS["gated_order1_bf16_2d_b2_c256_256x256"].scaled(B=1, D=4, shape=(16, 16))
    plain = dataclasses.replace(w, gated=False)
    a, b = make_inputs(w), make_inputs(plain)
    assert "k" in a and "k" not in b
    assert torch.equal(a["v"], b["v"]) and torch.equal(a["gates"], b["gates"])
    assert a["k"].dtype == torch.bfloat16 and a["k"].shape == a["v"].shape
    assert abs(a["k"].double().mean()) < 0.2 and 0.8 < a["k"].double().std() < 1.2


def test_named_workloads_have_the_stated_sizes():
    assert set(WORKLOADS) == set(STATED)
    for name, (ndim, B, D, shape, N, dt, filt) in STATED.items():
        w = WORKLOADS[name]
        assert (w.ndim, w.B, w.D, w.shape, w.order, w.dtype, w.filt) == (ndim, B, D, shape, N, dt, filt), name
    assert len({w.seed for w in WORKLOADS.values()}) == len(WORKLOADS)
    assert WORKLOADS["order2_bf16_b8_d768_l2048"].elements == 8 * 768 * 2048
    assert WORKLOADS["order1_bf16_2d_b2_c256_256x256"].elements == 2 * 256 * 256 * 256


@pytest.mark.parametrize("name", sorted(STATED))
def test_draws_are_reproducible_and_typed(name):
    w = WORKLOADS[name]
    small = w.scaled(B=1, D=8, shape=(64,) if w.ndim == 1 else (16, 16))
    a, b = make_inputs(small), make_inputs(small)
    c = make_inputs(small, seed=small.seed + 100)
    assert torch.equal(a["v"], b["v"]) and not torch.equal(a["v"], c["v"])
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    assert a["v"].dtype == dt and a["gates"].dtype == dt and a["dskip"].dtype == torch.float32
    expect = (w.order, 1, 8) + small.shape if w.layout == "bdl" else (w.order, 1) + small.shape + (8,)
    assert a["gates"].shape == expect


def test_activations_are_standard_normal():
    w = WORKLOADS["order2_bf16_b8_d768_l2048"].scaled(B=2, D=64, shape=(2048,))
    x = make_inputs(w)["v"].double()
    assert abs(x.mean().item()) < 0.01 and abs(x.std().item() - 1.0) < 0.01


def _fitted_rates(name, T, D=256):
    """Per-channel decay rate of h[d, t] = z * exp(-alpha_d t): minus the least-squares slope of
    log|h| over t < T (log|z| adds zero-slope noise)."""
    w = WORKLOADS[name].scaled(B=1, D=D, shape=(T,), order=1)
    h = make_inputs(w)["h"].double()[0]
    t = torch.arange(T, dtype=torch.float64)
    y = torch.log(h.abs().clamp_min(1e-300))
    tm = t.mean()
    return -(((t - tm) * (y - y.mean(dim=1, keepdim=True))).sum(dim=1) / ((t - tm) ** 2).sum())


def test_explicit_decay_rates_are_log_uniform_in_range():
    # long rows, slow rates: a window of 4096 taps fits each rate to a few per cent
    a = _fitted_rates("order3_bf16_b1_d768_l65536", 4096)
    assert (a > 1e-4 * 0.8).all() and (a < 1e-2 * 1.2).all()
    assert abs(torch.log(a).mean().item() - 0.5 * (math.log(1e-4) + math.log(1e-2))) < 0.2
    # fast rates (up to 0.1) underflow fp32 within a few hundred taps: fit over t < 200, where the
    # slope's noise is about 0.003, and check the range and the log-uniform median sqrt(lo hi)
    b = _fitted_rates("order2_bf16_b8_d768_l2048", 200)
    assert (b > 1e-3 - 0.01).all() and (b < 1e-1 + 0.01).all()
    assert abs(b.median().item() - math.sqrt(1e-3 * 1e-1)) < 0.004


def test_fixed_decay_of_the_small_fp32_workload():
    w = WORKLOADS["order2_f32_b1_d4_l256"]
    h = make_inputs(w)["h"].double()
    t = torch.arange(256, dtype=torch.float64)
    z = h * torch.exp(0.02 * t)          # undo the stated envelope: standard normal taps remain
    assert abs(z.std().item() - 1.0) < 0.1 and abs(z.mean().item()) < 0.15


def test_implicit_parameters():
    w1 = WORKLOADS["order2_bf16_b4_d1024_l8192_implicit"].scaled(D=512)
    p = make_inputs(w1)["implicit"]
    assert p["W1"].shape == (64, 33) and p["W2"].shape == (64, 64) and p["W3"].shape == (2 * 512, 64)
    assert abs(p["W3"].double().std().item() - 1 / 8) < 0.005          # N(0, 1/64)
    a = p["alpha"].double()
    assert a.shape == (2, 512) and (a >= 1e-3).all() and (a <= 1e-1).all()
    w2 = WORKLOADS["order1_bf16_2d_b2_c256_256x256"]
    p2 = make_inputs(w2.scaled(B=1, D=16, shape=(8, 8)))["implicit"]
    assert p2["W1"].shape == (64, 2) and torch.equal(p2["sigma"], torch.full((1, 16), 0.5))
    assert (p2["omega0"], p2["omega_hidden"], p2["num_freqs"]) == (10.0, 1.0, 0)
