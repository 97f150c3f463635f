"""Implicit filters of the Hyena operator, fp64 numpy. TEST INFRASTRUCTURE.

Parity of these two functions is pinned by special cases in which the
network reduces to a closed form (see the CPU test suite): one feature through
one unit per layer, the window alone, a non-zero bias in each hidden layer
(which fixes the bias inside the sine's frequency), and an off-diagonal hidden
weight (which fixes W2's orientation). The network itself is a reading of the
pages, not something they print.

1D filter ("Hyena — Long Convolutions Math", "Implicit filters: an MLP over
positions" and "The decay window, and why it is not optional";
"Hyena, Long Convolution, and Linear Attention", "FFTConv", filter indexed by
t / L):

    gamma(t) = [t/L, cos(2 pi 1 t/L), sin(2 pi 1 t/L), ..., cos(2 pi K t/L), sin(2 pi K t/L)]
    a1 = sin(omega0       * (W1 gamma(t) + b1))
    a2 = sin(omega_hidden * (W2 a1 + b2))
    o  = W3 a2 + b3                                   (one value per (order, channel))
    h[n, d, t] = exp(-alpha[n, d] * t) * o[n * D + d]

2D filter ("How HyenaND works", "1. An implicit filter": a SIREN MLP on the
grid coordinates times a Gaussian window):

    p = (oy / H, ox / W) for offsets oy in [-H, H), ox in [-W, W)
    a1 = sin(omega0 * (W1 p + b1)); a2 = sin(omega_hidden * (W2 a1 + b2)); o = W3 a2 + b3
    K[n, c, oy + H, ox + W] = exp(-|p|^2 / (2 sigma[n, c]^2)) * o[n * C + c]

Weight shapes: W1 [width, in], b1 [width], W2 [width, width], b2 [width],
W3 [out, width], b3 [out]; out = N * D (1D) or N * C (2D).
"""
from __future__ import annotations

import numpy as np


def positional_features_1d(L: int, num_freqs: int) -> np.ndarray:
    """gamma(t) for t = 0..L-1 as a [L, 1 + 2 * num_freqs] fp64 array."""
    t = np.arange(L, dtype=np.float64)
    cols = [t / L]
    for k in range(1, num_freqs + 1):
        ang = 2.0 * np.pi * k * t / L
        cols.append(np.cos(ang))
        cols.append(np.sin(ang))
    return np.stack(cols, axis=1)


def _mlp(feat, W1, b1, W2, b2, W3, b3, omega0, omega_hidden):
    W1, b1, W2, b2, W3, b3 = (np.asarray(a, dtype=np.float64) for a in (W1, b1, W2, b2, W3, b3))
    a1 = np.sin(omega0 * (feat @ W1.T + b1))
    a2 = np.sin(omega_hidden * (a1 @ W2.T + b2))
    return a2 @ W3.T + b3                               # [positions, out]


def implicit_filter_1d(L, N, D, W1, b1, W2, b2, W3, b3, alpha, num_freqs, omega0=1.0, omega_hidden=1.0):
    """Returns h [N, D, L] fp64."""
    feat = positional_features_1d(L, num_freqs)
    o = _mlp(feat, W1, b1, W2, b2, W3, b3, omega0, omega_hidden)          # [L, N*D]
    alpha = np.asarray(alpha, dtype=np.float64).reshape(N * D)
    t = np.arange(L, dtype=np.float64)
    window = np.exp(-alpha[:, None] * t[None, :])                         # [N*D, L]
    return (window * o.T).reshape(N, D, L)


def implicit_filter_2d(H, W, N, C, W1, b1, W2, b2, W3, b3, sigma, omega0=10.0, omega_hidden=1.0):
    """Returns K [N, C, 2H, 2W] fp64 on the offset grid."""
    oy = np.arange(-H, H, dtype=np.float64) / H
    ox = np.arange(-W, W, dtype=np.float64) / W
    py, px = np.meshgrid(oy, ox, indexing="ij")
    feat = np.stack([py.ravel(), px.ravel()], axis=1)                     # [4HW, 2] as (y, x)
    o = _mlp(feat, W1, b1, W2, b2, W3, b3, omega0, omega_hidden)          # [4HW, N*C]
    sigma = np.asarray(sigma, dtype=np.float64).reshape(N * C)
    r2 = (py ** 2 + px ** 2).ravel()
    window = np.exp(-r2[None, :] / (2.0 * sigma[:, None] ** 2))           # [N*C, 4HW]
    return (window * o.T).reshape(N, C, 2 * H, 2 * W)


def implicit_filter_3d(Dz, H, W, N, C, W1, b1, W2, b2, W3, b3, sigma, omega0=10.0, omega_hidden=1.0):
    """Returns K [N, C, 2Dz, 2H, 2W] fp64 on the offset grid: the 2D network on the
    coordinates p = (oz / Dz, oy / H, ox / W) of a volume's offsets, with the Gaussian
    window of |p|^2 ("How HyenaND works", "1. An implicit filter": the kernel as a
    continuous function of the grid coordinates, here of a 3D grid)."""
    oz = np.arange(-Dz, Dz, dtype=np.float64) / Dz
    oy = np.arange(-H, H, dtype=np.float64) / H
    ox = np.arange(-W, W, dtype=np.float64) / W
    pz, py, px = np.meshgrid(oz, oy, ox, indexing="ij")
    feat = np.stack([pz.ravel(), py.ravel(), px.ravel()], axis=1)         # [8 Dz H W, 3] as (z, y, x)
    o = _mlp(feat, W1, b1, W2, b2, W3, b3, omega0, omega_hidden)          # [8 Dz H W, N*C]
    sigma = np.asarray(sigma, dtype=np.float64).reshape(N * C)
    r2 = (pz ** 2 + py ** 2 + px ** 2).ravel()
    window = np.exp(-r2[None, :] / (2.0 * sigma[:, None] ** 2))
    return (window * o.T).reshape(N, C, 2 * Dz, 2 * H, 2 * W)
