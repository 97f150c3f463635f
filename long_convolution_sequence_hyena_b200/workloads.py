"""Seeded synthetic inputs for the Hyena operator.

This module draws random numbers and nothing else: it holds none of the
operator's arithmetic (no convolution, transform, gate or filter network), so
both the CUDA path and the fp64 oracle can take their inputs from it.

Everything is drawn on the CPU from a seeded ``torch.Generator`` in fp64 and
then cast once to the storage dtype; the oracle must widen those stored values
back to fp64, never use the fp64 draws.

Named workloads (sizes as stated; activations v, x^n and Dskip ~ N(0, 1)):

* ``order2_f32_b1_d4_l256``            -- B=1, D=4, L=256, order 2, fp32 I/O,
  h[d, t] = N(0,1) * exp(-0.02 t).
* ``order2_bf16_b8_d768_l2048``        -- B=8, D=768, L=2048, order 2, bf16 I/O,
  h[d, t] = N(0,1) * exp(-alpha_d t), alpha_d log-uniform in [1e-3, 1e-1].
* ``order2_bf16_b4_d1024_l8192_implicit`` -- B=4, D=1024, L=8192, order 2, bf16
  I/O, filters from the implicit sine network (33 positional features, width 64,
  weights and biases ~ N(0, 1/64)) times exp(-alpha_d t), alpha_d log-uniform in
  [1e-3, 1e-1].
* ``order3_bf16_b1_d768_l65536``       -- B=1, D=768, L=65536, order 3, bf16,
  alpha_d log-uniform in [1e-4, 1e-2].
* ``order1_bf16_2d_b2_c256_256x256``   -- 2D, B=2, C=256, 256 x 256 grid, order 1,
  bf16, kernels from the 2D sine network on (y, x) in [-1, 1)^2 (first-layer
  frequency 10, hidden 1, width 64, weights ~ N(0, 1/64)) times a Gaussian
  window with sigma = 0.5.
* ``gated_order1_bf16_2d_b2_c256_256x256`` -- the same grid, channels and
  kernels through the HyenaND gate sandwich: q (drawn as v), k and the outer
  gate v (drawn as x^1) ~ N(0, 1).
* ``order3_bf16_b1_d768_l65536_bld`` -- the L=65536 order-3 recipe with
  channels-last activations [B, L, D] (drawn as [B, D, L], then transposed).
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    ndim: int                 # 1: sequence, 2: grid
    B: int
    D: int                    # channels (C in 2D)
    shape: tuple              # (L,) or (H, W)
    order: int
    dtype: str                # "f32" or "bf16" (activation storage)
    filt: str                 # "explicit" | "implicit1d" | "implicit2d"
    alpha_lo: float = 0.0     # decay-rate range (1D), log-uniform; lo == hi means fixed
    alpha_hi: float = 0.0
    width: int = 64           # implicit network width
    num_freqs: int = 16       # 1D positional frequencies (features = 1 + 2K)
    omega0: float = 1.0
    omega_hidden: float = 1.0
    sigma: float = 0.5        # 2D Gaussian window
    seed: int = 0
    gated: bool = False       # the gate sandwich: an inner-gate key k is drawn too
    layout: str = "bdl"       # 1D activations [B, D, L] ("bdl") or channels-last [B, L, D] ("bld")

    @property
    def L(self) -> int:
        return self.shape[0] if self.ndim == 1 else self.shape[0] * self.shape[1]

    @property
    def elements(self) -> int:
        """B * D * L (1D) or B * C * H * W (2D): the unit the throughput counts."""
        return self.B * self.D * self.L

    def scaled(self, B=None, D=None, shape=None, order=None, name=None):
        """Same recipe at other sizes (for parity cases the oracle finishes quickly)."""
        return dataclasses.replace(
            self, B=self.B if B is None else B, D=self.D if D is None else D,
            shape=self.shape if shape is None else tuple(shape),
            order=self.order if order is None else order,
            name=name or self.name + "_scaled")


WORKLOADS = {
    w.name: w for w in [
        Workload("order2_f32_b1_d4_l256", 1, 1, 4, (256,), 2, "f32", "explicit",
                 alpha_lo=0.02, alpha_hi=0.02, seed=1),
        Workload("order2_bf16_b8_d768_l2048", 1, 8, 768, (2048,), 2, "bf16", "explicit",
                 alpha_lo=1e-3, alpha_hi=1e-1, seed=2),
        Workload("order2_bf16_b4_d1024_l8192_implicit", 1, 4, 1024, (8192,), 2, "bf16", "implicit1d",
                 alpha_lo=1e-3, alpha_hi=1e-1, width=64, num_freqs=16, seed=3),
        Workload("order3_bf16_b1_d768_l65536", 1, 1, 768, (65536,), 3, "bf16", "explicit",
                 alpha_lo=1e-4, alpha_hi=1e-2, seed=4),
        Workload("order1_bf16_2d_b2_c256_256x256", 2, 2, 256, (256, 256), 1, "bf16", "implicit2d",
                 width=64, omega0=10.0, omega_hidden=1.0, sigma=0.5, seed=5),
        Workload("gated_order1_bf16_2d_b2_c256_256x256", 2, 2, 256, (256, 256), 1, "bf16", "implicit2d",
                 width=64, omega0=10.0, omega_hidden=1.0, sigma=0.5, seed=6, gated=True),
        Workload("order3_bf16_b1_d768_l65536_bld", 1, 1, 768, (65536,), 3, "bf16", "explicit",
                 alpha_lo=1e-4, alpha_hi=1e-2, seed=7, layout="bld"),
    ]
}

TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _alphas(w: Workload, n: int, g: torch.Generator) -> torch.Tensor:
    if w.alpha_lo == w.alpha_hi:
        return torch.full((n,), w.alpha_lo, dtype=torch.float64)
    u = torch.rand(n, generator=g, dtype=torch.float64)
    return torch.exp(math.log(w.alpha_lo) + u * (math.log(w.alpha_hi) - math.log(w.alpha_lo)))


def make_inputs(w: Workload, seed=None) -> dict:
    """Draw one batch of inputs for ``w`` on the CPU.

    Returns a dict of CPU tensors:
      v      [B, D, *shape]      activation dtype
      gates  [N, B, D, *shape]   activation dtype
      dskip  [N, D]              float32
      h      [N, D, L]           float32 (explicit filters only; 2D: [N, C, 2H, 2W] on
                                 the offset grid, N(0,1) under exp(-|p|^2 / (2 sigma^2)))
      implicit: dict of float32 weights W1 b1 W2 b2 W3 b3 and the window
               parameter (alpha [N, D] in 1D, sigma [N, D] in 2D), plus the
               scalars width, num_freqs, omega0, omega_hidden (implicit only)
      k      [B, D, *shape]      activation dtype (gate sandwich only; v is then q)
    With layout "bld" v and the gates are [B, L, D] and [N, B, L, D].
    """
    g = _gen(w.seed if seed is None else seed)
    N, B, D = w.order, w.B, w.D
    adt = TORCH_DTYPE[w.dtype]
    out = {}
    out["v"] = torch.randn((B, D) + w.shape, generator=g, dtype=torch.float64).to(adt)
    out["gates"] = torch.randn((N, B, D) + w.shape, generator=g, dtype=torch.float64).to(adt)
    out["dskip"] = torch.randn((N, D), generator=g, dtype=torch.float64).to(torch.float32)
    if w.filt == "explicit" and w.ndim == 2:
        H, W = w.shape
        oy = torch.arange(-H, H, dtype=torch.float64) / H
        ox = torch.arange(-W, W, dtype=torch.float64) / W
        r2 = oy[:, None] ** 2 + ox[None, :] ** 2
        # explicit 2D kernels on the offset grid: Gaussian taps under a Gaussian envelope
        out["h"] = (torch.randn((N, D, 2 * H, 2 * W), generator=g, dtype=torch.float64)
                    * torch.exp(-r2 / (2 * w.sigma ** 2))).to(torch.float32)
    elif w.filt == "explicit":
        L = w.shape[0]
        alpha = _alphas(w, N * D, g).reshape(N, D, 1)
        t = torch.arange(L, dtype=torch.float64)
        # The filter recipe of the explicit-filter workloads: Gaussian taps under
        # a per-channel exponential envelope (the decay window is part of the
        # synthetic data here, not computed by the operator).
        out["h"] = (torch.randn((N, D, L), generator=g, dtype=torch.float64) * torch.exp(-alpha * t)).to(torch.float32)
    else:
        fin = 1 + 2 * w.num_freqs if w.filt == "implicit1d" else 2
        std = 1.0 / math.sqrt(w.width)
        p = {
            "W1": torch.randn((w.width, fin), generator=g, dtype=torch.float64) * std,
            "b1": torch.randn((w.width,), generator=g, dtype=torch.float64) * std,
            "W2": torch.randn((w.width, w.width), generator=g, dtype=torch.float64) * std,
            "b2": torch.randn((w.width,), generator=g, dtype=torch.float64) * std,
            "W3": torch.randn((N * D, w.width), generator=g, dtype=torch.float64) * std,
            "b3": torch.randn((N * D,), generator=g, dtype=torch.float64) * std,
        }
        p = {k: val.to(torch.float32) for k, val in p.items()}
        if w.filt == "implicit1d":
            p["alpha"] = _alphas(w, N * D, g).reshape(N, D).to(torch.float32)
        else:
            p["sigma"] = torch.full((N, D), w.sigma, dtype=torch.float32)
        p.update(width=w.width, num_freqs=w.num_freqs if w.filt == "implicit1d" else 0,
                 omega0=w.omega0, omega_hidden=w.omega_hidden)
        out["implicit"] = p
    if w.gated:   # drawn last, so that the other tensors follow the plain recipe
        out["k"] = torch.randn((B, D) + w.shape, generator=g, dtype=torch.float64).to(adt)
    if w.layout == "bld":   # channels-last copies of the same values
        out["v"] = out["v"].transpose(-1, -2).contiguous()
        out["gates"] = out["gates"].transpose(-1, -2).contiguous()
    return out
