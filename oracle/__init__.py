"""Oracle for the order-N Hyena operator (fp64, CPU). TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. It shares no code with the CUDA library
and never calls it; the library never calls this package.

Contents
--------
* ``hyena_1d``  -- the order-N causal chain, direct O(L^2) sum, in C
  (``hyena_oracle.c``); see that file for the definition and its citations.
* ``hyena_3d``  -- the same chain on a 3D grid (volumes), direct sum, in C.
* ``hyena_1d_order1_at`` -- single order-1 outputs by their own direct sums,
  for rows too long for the full chain.
* ``hyena_2d``  -- the 2D gated global (non-causal, linear) convolution chain,
  direct O((HW)^2) sum, in C.
* ``implicit_filter_1d`` / ``implicit_filter_2d`` -- the implicit filters in
  numpy fp64 (``implicit.py``).
* ``hyena_gated`` / ``silu`` -- the HyenaND gate sandwich (inner gate
  q ⊙ SiLU(k), outer gates SiLU(x^n)) around the same chains (``gated.py``).

All arrays are float64 numpy arrays; callers pass the exact values the GPU path
receives (bf16 inputs are widened exactly before they get here).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from .gated import hyena_gated, silu  # noqa: F401
from .implicit import implicit_filter_1d, implicit_filter_2d, implicit_filter_3d, positional_features_1d  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hyena_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``hyena_oracle.c`` into ``liboracle.so`` with gcc (plain -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC, "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        p = ctypes.c_void_p
        i64 = ctypes.c_int64
        lib.hyena_oracle_1d.argtypes = [i64, i64, i64, i64, p, p, p, p, p, p, ctypes.c_int]
        lib.hyena_oracle_1d.restype = ctypes.c_int
        lib.hyena_oracle_2d.argtypes = [i64, i64, i64, i64, i64, p, p, p, p, p, p, ctypes.c_int]
        lib.hyena_oracle_2d.restype = ctypes.c_int
        lib.hyena_oracle_3d.argtypes = [i64, i64, i64, i64, i64, i64, p, p, p, p, p, p, ctypes.c_int]
        lib.hyena_oracle_3d.restype = ctypes.c_int
        lib.hyena_oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def num_threads() -> int:
    """Threads the oracle uses when ``threads <= 0`` (one per online CPU)."""
    return int(_load().hyena_oracle_num_threads())


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def hyena_1d(v, gates, h, dskip=None, fidx=None, threads: int = 0):
    """Order-N Hyena chain over R independent rows.

    v      [R, L]     input of the first convolution
    gates  [N, R, L]  gates x^1..x^N
    h      [N, F, L]  causal filters (filter taps 0..L-1)
    dskip  [N, F]     feedthrough per order and filter row, or None (zero)
    fidx   [R]        filter row of each data row (default: row r uses r % F)
    Returns y [R, L] float64.
    """
    v, gates, h = _f64(v), _f64(gates), _f64(h)
    R, L = v.shape
    N, F, Lh = h.shape
    if gates.shape != (N, R, L) or Lh != L:
        raise ValueError("shape mismatch: v %s gates %s h %s" % (v.shape, gates.shape, h.shape))
    dskip = None if dskip is None else _f64(dskip)
    if dskip is not None and dskip.shape != (N, F):
        raise ValueError("dskip must be [N, F]")
    fidx = np.arange(R, dtype=np.int64) % F if fidx is None else np.ascontiguousarray(fidx, dtype=np.int64)
    y = np.zeros((R, L), dtype=np.float64)
    rc = _load().hyena_oracle_1d(R, L, N, F, _ptr(v), _ptr(gates), _ptr(h), _ptr(dskip), _ptr(fidx), _ptr(y), threads)
    if rc != 0:
        raise RuntimeError("hyena_oracle_1d failed (%d)" % rc)
    return y


def hyena_1d_order1_at(v, x, h, dskip=None, positions=()):
    """Order-1 outputs at selected positions only, each by its own direct sum
    (the causal sum of "Hyena — Long Convolutions Math", "The primitive", with
    the feedthrough of "FFTConv"):  y[t] = x[t] (sum_{tau <= t} h[t - tau] v[tau] + dskip v[t]).

    v, x, h  [L] one row, its gate and its filter;  dskip  scalar or None.
    Returns fp64 [len(positions)]. O(t) per position, for rows too long for
    the full O(L^2) chain.
    """
    v, x, h = _f64(v), _f64(x), _f64(h)
    d = 0.0 if dskip is None else float(dskip)
    out = np.empty(len(positions), dtype=np.float64)
    for i, t in enumerate(positions):
        t = int(t)
        c = float(np.dot(h[t::-1], v[:t + 1]))        # h[t - tau] v[tau], tau = 0..t
        out[i] = x[t] * (c + d * v[t])
    return out


def hyena_2d(v, gates, k, dskip=None, fidx=None, threads: int = 0):
    """2D gated global-convolution chain over P independent planes.

    v      [P, H, W]
    gates  [N, P, H, W]
    k      [N, F, 2H, 2W]  kernels on the offset grid: element (oy, ox), with
                          oy in [-H, H) and ox in [-W, W), at [oy + H, ox + W]
    dskip  [N, F] or None
    fidx   [P] (default: plane p uses p % F)
    Returns y [P, H, W] float64.
    """
    v, gates, k = _f64(v), _f64(gates), _f64(k)
    P, H, W = v.shape
    N, F, H2, W2 = k.shape
    if gates.shape != (N, P, H, W) or H2 != 2 * H or W2 != 2 * W:
        raise ValueError("shape mismatch: v %s gates %s k %s" % (v.shape, gates.shape, k.shape))
    dskip = None if dskip is None else _f64(dskip)
    if dskip is not None and dskip.shape != (N, F):
        raise ValueError("dskip must be [N, F]")
    fidx = np.arange(P, dtype=np.int64) % F if fidx is None else np.ascontiguousarray(fidx, dtype=np.int64)
    y = np.zeros((P, H, W), dtype=np.float64)
    rc = _load().hyena_oracle_2d(P, H, W, N, F, _ptr(v), _ptr(gates), _ptr(k), _ptr(dskip), _ptr(fidx), _ptr(y), threads)
    if rc != 0:
        raise RuntimeError("hyena_oracle_2d failed (%d)" % rc)
    return y


def hyena_3d(v, gates, k, dskip=None, fidx=None, threads: int = 0):
    """3D gated global-convolution chain over P independent volumes.

    v      [P, Dz, H, W]
    gates  [N, P, Dz, H, W]
    k      [N, F, 2Dz, 2H, 2W]  kernels on the offset grid: element (oz, oy, ox),
                                oz in [-Dz, Dz) etc., at [oz + Dz, oy + H, ox + W]
    dskip  [N, F] or None
    fidx   [P] (default: volume p uses p % F)
    Returns y [P, Dz, H, W] float64.
    """
    v, gates, k = _f64(v), _f64(gates), _f64(k)
    P, Dz, H, W = v.shape
    N, F, D2, H2, W2 = k.shape
    if gates.shape != (N, P, Dz, H, W) or (D2, H2, W2) != (2 * Dz, 2 * H, 2 * W):
        raise ValueError("shape mismatch: v %s gates %s k %s" % (v.shape, gates.shape, k.shape))
    dskip = None if dskip is None else _f64(dskip)
    if dskip is not None and dskip.shape != (N, F):
        raise ValueError("dskip must be [N, F]")
    fidx = np.arange(P, dtype=np.int64) % F if fidx is None else np.ascontiguousarray(fidx, dtype=np.int64)
    y = np.zeros((P, Dz, H, W), dtype=np.float64)
    rc = _load().hyena_oracle_3d(P, Dz, H, W, N, F, _ptr(v), _ptr(gates), _ptr(k), _ptr(dskip), _ptr(fidx),
                                 _ptr(y), threads)
    if rc != 0:
        raise RuntimeError("hyena_oracle_3d failed (%d)" % rc)
    return y


def hyena_3d_order1_at(v, x, k, dskip=None, voxels=()):
    """Order-1 outputs of one volume at selected voxels only, each by its own direct sum:
    y[i] = x[i] (sum_s K[i - s] v[s] + dskip v[i]), the kernel on the offset grid
    [2Dz, 2H, 2W] (offset o at [o + extent]). O(Dz H W) per voxel.

    v, x  [Dz, H, W];  k  [2Dz, 2H, 2W];  voxels: iterable of (iz, iy, ix).
    """
    v, x, k = _f64(v), _f64(x), _f64(k)
    Dz, H, W = v.shape
    d = 0.0 if dskip is None else float(dskip)
    out = []
    for iz, iy, ix in voxels:
        # K[iz - sz + Dz, iy - sy + H, ix - sx + W] over sz < Dz, sy < H, sx < W: a reversed window
        win = k[iz + 1:iz + Dz + 1, iy + 1:iy + H + 1, ix + 1:ix + W + 1][::-1, ::-1, ::-1]
        c = float(np.sum(win * v))
        out.append(x[iz, iy, ix] * (c + d * v[iz, iy, ix]))
    return np.array(out)
