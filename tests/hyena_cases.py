"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
and the fp64 oracle on the same seeded inputs, then compare with the stated
tolerances.

Tolerances (from the operator's accuracy target):
  fp32 I/O: relative L2 error <= 1e-5, and per element
            |y - y_ref| <= 1e-4 * S_row,
            S_row = |v_row|_inf * prod_n (|h^n_d|_1 + |Dskip^n_d|) * |x^n_row|_inf
            (the a-priori bound on |y| for that row);
  bf16 I/O: relative L2 error <= 2e-2 (fp32 accumulation, bf16 output rounding).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from long_convolution_sequence_hyena_b200.workloads import Workload, make_inputs

REL_L2 = {"f32": 1e-5, "bf16": 2e-2}
MAXABS_FACTOR = 1e-4


def explicit_case(B, D, L, N, dtype="f32", seed=0, alpha=(1e-3, 1e-1)):
    return Workload("case_b%d_d%d_l%d_n%d_%s" % (B, D, L, N, dtype), 1, B, D, (L,), N, dtype, "explicit",
                    alpha_lo=alpha[0], alpha_hi=alpha[1], seed=seed)


def to_gpu(inp):
    g = {"v": inp["v"].cuda(), "gates": [x.cuda() for x in inp["gates"]], "dskip": inp["dskip"].cuda()}
    if "h" in inp:
        g["h"] = inp["h"].cuda()
    if "implicit" in inp:
        g["implicit"] = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp["implicit"].items()}
    return g


def oracle_filters_1d(w: Workload, inp):
    """fp64 filters [N, D, L] the oracle uses: the given taps, or the implicit network in fp64."""
    if "h" in inp:
        return inp["h"].double().numpy()
    p = inp["implicit"]
    return oracle.implicit_filter_1d(w.shape[0], w.order, w.D, p["W1"].double().numpy(), p["b1"].double().numpy(),
                                     p["W2"].double().numpy(), p["b2"].double().numpy(), p["W3"].double().numpy(),
                                     p["b3"].double().numpy(), p["alpha"].double().numpy(), p["num_freqs"],
                                     p["omega0"], p["omega_hidden"])


def oracle_1d(w: Workload, inp, h64, rows=None):
    """Oracle output for the selected flat rows (b * D + d), fp64 [len(rows), L]."""
    N, B, D, L = w.order, w.B, w.D, w.shape[0]
    R = B * D
    rows = np.arange(R) if rows is None else np.asarray(rows)
    v = inp["v"].double().reshape(R, L).numpy()[rows]
    gates = inp["gates"].double().reshape(N, R, L).numpy()[:, rows]
    return oracle.hyena_1d(v, gates, h64, inp["dskip"].double().numpy(), fidx=rows % D)


def row_bound(w: Workload, inp, h64, rows):
    """S_row for each selected row (see module docstring)."""
    N, B, D, L = w.order, w.B, w.D, w.shape[0]
    R = B * D
    v = inp["v"].double().reshape(R, L).numpy()[rows]
    gates = inp["gates"].double().reshape(N, R, L).numpy()[:, rows]
    dsk = inp["dskip"].double().numpy()
    d = rows % D
    s = np.abs(v).max(axis=1)
    for n in range(N):
        s = s * (np.abs(h64[n, d]).sum(axis=1) + np.abs(dsk[n, d])) * np.abs(gates[n]).max(axis=1)
    return s


def compare(w: Workload, inp, h64, y_gpu, rows=None, context=""):
    """Check the GPU output (torch tensor [B, D, L]) on the given rows against the oracle."""
    N, B, D, L = w.order, w.B, w.D, w.shape[0]
    R = B * D
    rows = np.arange(R) if rows is None else np.asarray(rows)
    ref = oracle_1d(w, inp, h64, rows)
    got = y_gpu.detach().double().cpu().reshape(R, L).numpy()[rows]
    assert np.all(np.isfinite(got)), context + ": non-finite output"
    err = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    assert err <= REL_L2[w.dtype], "%s: relative L2 error %.3e > %.1e" % (context, err, REL_L2[w.dtype])
    if w.dtype == "f32":
        bound = MAXABS_FACTOR * row_bound(w, inp, h64, rows)
        worst = (np.abs(got - ref) / np.maximum(bound, 1e-300)[:, None]).max()
        assert worst <= 1.0, "%s: per-element error %.3f x the bound" % (context, worst)
    return err


# ------------------------------------------------------------------------ 2D --

def explicit_case_2d(B, C, Hw, N, dtype="f32", seed=0, sigma=0.5):
    return Workload("case2d_b%d_c%d_%d_n%d_%s" % (B, C, Hw, N, dtype), 2, B, C, (Hw, Hw), N, dtype, "explicit",
                    sigma=sigma, seed=seed)


def oracle_kernels_2d(w: Workload, inp):
    """fp64 kernels [N, C, 2H, 2W] on the offset grid."""
    if "h" in inp:
        return inp["h"].double().numpy()
    p = inp["implicit"]
    H, W = w.shape
    return oracle.implicit_filter_2d(H, W, w.order, w.D, p["W1"].double().numpy(), p["b1"].double().numpy(),
                                     p["W2"].double().numpy(), p["b2"].double().numpy(), p["W3"].double().numpy(),
                                     p["b3"].double().numpy(), p["sigma"].double().numpy(), p["omega0"],
                                     p["omega_hidden"])


def compare_2d(w: Workload, inp, k64, y_gpu, planes=None, context=""):
    N, B, C = w.order, w.B, w.D
    H, W = w.shape
    P = B * C
    planes = np.arange(P) if planes is None else np.asarray(planes)
    v = inp["v"].double().reshape(P, H, W).numpy()[planes]
    gates = inp["gates"].double().reshape(N, P, H, W).numpy()[:, planes]
    dsk = inp["dskip"].double().numpy()
    ref = oracle.hyena_2d(v, gates, k64, dsk, fidx=planes % C)
    got = y_gpu.detach().double().cpu().reshape(P, H, W).numpy()[planes]
    assert np.all(np.isfinite(got)), context + ": non-finite output"
    err = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    assert err <= REL_L2[w.dtype], "%s: relative L2 error %.3e > %.1e" % (context, err, REL_L2[w.dtype])
    if w.dtype == "f32":
        c = planes % C
        bound = np.abs(v).reshape(len(planes), -1).max(axis=1)
        for n in range(N):
            bound = bound * (np.abs(k64[n, c]).reshape(len(planes), -1).sum(axis=1) + np.abs(dsk[n, c])) \
                * np.abs(gates[n]).reshape(len(planes), -1).max(axis=1)
        worst = (np.abs(got - ref) / (MAXABS_FACTOR * np.maximum(bound, 1e-300))[:, None, None]).max()
        assert worst <= 1.0, "%s: per-element error %.3f x the bound" % (context, worst)
    return err


# ------------------------------------------------------------- gate sandwich --

def compare_gated_2d(w: Workload, inp, k64, y_gpu, planes=None, context=""):
    """The gate sandwich (q = inp["v"], key inp["k"], SiLU of every gate) against the fp64 oracle."""
    N, B, C = w.order, w.B, w.D
    H, W = w.shape
    P = B * C
    planes = np.arange(P) if planes is None else np.asarray(planes)
    q = inp["v"].double().reshape(P, H, W).numpy()[planes]
    kk = inp["k"].double().reshape(P, H, W).numpy()[planes]
    gates = inp["gates"].double().reshape(N, P, H, W).numpy()[:, planes]
    dsk = inp["dskip"].double().numpy()
    ref = oracle.hyena_gated(q, kk, gates, k64, dsk, fidx=planes % C)
    got = y_gpu.detach().double().cpu().reshape(P, H, W).numpy()[planes]
    assert np.all(np.isfinite(got)), context + ": non-finite output"
    err = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    assert err <= REL_L2[w.dtype], "%s: relative L2 error %.3e > %.1e" % (context, err, REL_L2[w.dtype])
    if w.dtype == "f32":
        c = planes % C
        z0 = q * oracle.silu(kk)
        bound = np.abs(z0).reshape(len(planes), -1).max(axis=1)
        for n in range(N):
            bound = bound * (np.abs(k64[n, c]).reshape(len(planes), -1).sum(axis=1) + np.abs(dsk[n, c])) \
                * np.abs(oracle.silu(gates[n])).reshape(len(planes), -1).max(axis=1)
        worst = (np.abs(got - ref) / (MAXABS_FACTOR * np.maximum(bound, 1e-300))[:, None, None]).max()
        assert worst <= 1.0, "%s: per-element error %.3f x the bound" % (context, worst)
    return err


# ------------------------------------------------------------------------ 3D --

def case_3d(B, C, shape, N, dtype="f32", seed=0, sigma=0.5):
    """A 3D workload (shape (Dz, H, W)) with explicit kernels: Gaussian taps on the offset grid
    under a Gaussian envelope of |p|^2, p = (oz / Dz, oy / H, ox / W)."""
    return Workload("case3d_b%d_c%d_%dx%dx%d_n%d_%s" % ((B, C) + tuple(shape) + (N, dtype)), 3, B, C, tuple(shape), N,
                    dtype, "explicit", sigma=sigma, seed=seed)


def inputs_3d(w: Workload):
    """Seeded inputs of a 3D case: v, gates ~ N(0, 1) in the io dtype, dskip ~ N(0, 1), kernels [N, C, 2Dz, 2H, 2W]."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    Dz, H, W = w.shape
    adt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    v = torch.randn((w.B, w.D, Dz, H, W), generator=g, dtype=torch.float64).to(adt)
    gates = torch.randn((w.order, w.B, w.D, Dz, H, W), generator=g, dtype=torch.float64).to(adt)
    dskip = torch.randn((w.order, w.D), generator=g, dtype=torch.float64).to(torch.float32)
    oz = torch.arange(-Dz, Dz, dtype=torch.float64) / Dz
    oy = torch.arange(-H, H, dtype=torch.float64) / H
    ox = torch.arange(-W, W, dtype=torch.float64) / W
    r2 = oz[:, None, None] ** 2 + oy[None, :, None] ** 2 + ox[None, None, :] ** 2
    h = (torch.randn((w.order, w.D, 2 * Dz, 2 * H, 2 * W), generator=g, dtype=torch.float64)
         * torch.exp(-r2 / (2 * w.sigma ** 2))).to(torch.float32)
    k = torch.randn((w.B, w.D, Dz, H, W), generator=g, dtype=torch.float64).to(adt)
    return {"v": v, "gates": gates, "dskip": dskip, "h": h, "k": k}


def compare_3d(w: Workload, inp, k64, y_gpu, vols=None, gated=False, context=""):
    N, B, C = w.order, w.B, w.D
    Dz, H, W = w.shape
    P = B * C
    vols = np.arange(P) if vols is None else np.asarray(vols)
    v = inp["v"].double().reshape(P, Dz, H, W).numpy()[vols]
    gates = inp["gates"].double().reshape(N, P, Dz, H, W).numpy()[:, vols]
    dsk = inp["dskip"].double().numpy()
    if gated:
        kk = inp["k"].double().reshape(P, Dz, H, W).numpy()[vols]
        ref = oracle.hyena_gated(v, kk, gates, k64, dsk, fidx=vols % C)
    else:
        ref = oracle.hyena_3d(v, gates, k64, dsk, fidx=vols % C)
    got = y_gpu.detach().double().cpu().reshape(P, Dz, H, W).numpy()[vols]
    assert np.all(np.isfinite(got)), context + ": non-finite output"
    err = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    assert err <= REL_L2[w.dtype], "%s: relative L2 error %.3e > %.1e" % (context, err, REL_L2[w.dtype])
    return err
