"""The HyenaND gate sandwich, fp64 numpy. TEST INFRASTRUCTURE.

"How HyenaND works", "How HyenaND stays data-dependent: gating" and "Putting
it together: the HyenaND operator": the inner gate Z = q ⊙ SiLU(k) is
convolved with the kernel, and the outer gate multiplies the result by
SiLU(v). Written as the order-N chain of the Hyena operator:

    z^0 = q ⊙ SiLU(k)
    z^n = SiLU(x^n) ⊙ (K^n ∗ z^{n-1} + Dskip^n ⊙ z^{n-1})     n = 1..N
    y   = z^N

With N = 1, Dskip = 0 and x^1 = v this is O = (K ∗ (q ⊙ SiLU(k))) ⊙ SiLU(v).
SiLU(x) = x · σ(x), σ the logistic function, evaluated as 1 / (1 + e^{-x})
for x >= 0 and e^{x} / (1 + e^{x}) for x < 0, so that neither branch
overflows or cancels.

The convolution chain itself is the direct sum of ``hyena_1d`` / ``hyena_2d``
(``hyena_oracle.c``); this file only forms the gated inputs in fp64.
"""
from __future__ import annotations

import numpy as np


def silu(x):
    x = np.asarray(x, dtype=np.float64)
    e = np.exp(-np.abs(x))                       # in (0, 1]
    sig = np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))
    return x * sig


def hyena_gated(q, k, gates, filters, dskip=None, fidx=None, threads: int = 0):
    """Gate sandwich over independent rows (1D: q, k [R, L]) or planes (2D: [P, H, W]).

    gates   [N, R, ...] raw outer gates (SiLU is applied here)
    filters [N, F, L] causal taps (1D) or [N, F, 2H, 2W] kernels on the offset grid (2D)
    Returns y fp64 shaped like q.
    """
    from . import hyena_1d, hyena_2d
    q = np.asarray(q, dtype=np.float64)
    z0 = q * silu(k)
    g = silu(gates)
    if q.ndim == 2:
        return hyena_1d(z0, g, filters, dskip, fidx=fidx, threads=threads)
    if q.ndim == 3:
        return hyena_2d(z0, g, filters, dskip, fidx=fidx, threads=threads)
    if q.ndim == 4:
        from . import hyena_3d
        return hyena_3d(z0, g, filters, dskip, fidx=fidx, threads=threads)
    raise ValueError("q must be [R, L], [P, H, W] or [P, Dz, H, W]")
