"""Pins of the fp64 oracle to what the pages and the mathematics fix (CPU only).

Each test checks the oracle against something other than its own formula: a
value printed on the pages, a library routine for a special case, a closed form,
or an invariant the pages state. A plausible slip in the oracle (a dropped
feedthrough, a wrong index direction, a transposed gate, a circular instead of
a linear convolution, a wrong kernel offset) fails at least one of them.
"""
import os

import numpy as np
import pytest
import scipy.linalg
import scipy.signal
import scipy.special

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *nums = line.split()
            vals[key] = np.array([float(x) for x in nums])
    return vals


def _ones(shape):
    return np.ones(shape, dtype=np.float64)


# ---------------------------------------------------------------- 1D chain --

def test_worked_example_printed_values():
    """'Linear vs circular': h=[1,.5,.25,.125], x=[1,2,0,0] -> y=[1,2.5,1.25,.625]."""
    g = _read_golden("worked_example_causal_conv.txt")
    y = oracle.hyena_1d(g["x"][None], _ones((1, 1, 4)), g["h"][None, None])
    np.testing.assert_array_equal(y[0], g["y_linear_causal"])
    # The page's negative control: an unpadded circular convolution puts 1.25 at
    # t = 0; the causal oracle must not.
    assert y[0, 0] != g["y_circular_unpadded_t0"][0]


@pytest.mark.parametrize("N", [1, 2, 3])
def test_toeplitz_matrix_form(N):
    """'The Toeplitz picture': the chain equals D_{x^N}(S_{h^N}+D^N I)...D_{x^1}(S_{h^1}+D^1 I) v."""
    rng = np.random.default_rng(10 + N)
    L = 37
    v = rng.standard_normal((1, L))
    gates = rng.standard_normal((N, 1, L))
    h = rng.standard_normal((N, 1, L))
    dskip = rng.standard_normal((N, 1))
    z = v[0]
    for n in range(N):
        S = scipy.linalg.toeplitz(h[n, 0], np.zeros(L))          # S[t, tau] = h[t - tau], t >= tau
        z = gates[n, 0] * ((S + dskip[n, 0] * np.eye(L)) @ z)
    y = oracle.hyena_1d(v, gates, h, dskip)
    np.testing.assert_allclose(y[0], z, rtol=1e-12, atol=1e-12)


def test_causality():
    """'The primitive': y_t never depends on inputs at tau > t."""
    rng = np.random.default_rng(1)
    L, N = 64, 3
    v = rng.standard_normal((2, L))
    gates = rng.standard_normal((N, 2, L))
    h = rng.standard_normal((N, 2, L))
    dskip = rng.standard_normal((N, 2))
    y0 = oracle.hyena_1d(v, gates, h, dskip)
    for tau in (0, 17, 40, 63):
        v1 = v.copy()
        v1[:, tau] += 3.0
        y1 = oracle.hyena_1d(v1, gates, h, dskip)
        np.testing.assert_array_equal(y1[:, :tau], y0[:, :tau])
        assert np.all(y1[:, tau] != y0[:, tau])
        g1 = gates.copy()
        g1[0, :, tau] += 2.0
        y2 = oracle.hyena_1d(v, g1, h, dskip)
        np.testing.assert_array_equal(y2[:, :tau], y0[:, :tau])


def test_impulse_returns_filter():
    """v = delta_0, unit gates, no feedthrough: order 1 returns h; order 2 returns h2 * h1."""
    rng = np.random.default_rng(2)
    L = 50
    h = rng.standard_normal((2, 1, L))
    v = np.zeros((1, L))
    v[0, 0] = 1.0
    y1 = oracle.hyena_1d(v, _ones((1, 1, L)), h[:1])
    np.testing.assert_array_equal(y1[0], h[0, 0])
    y2 = oracle.hyena_1d(v, _ones((2, 1, L)), h)
    np.testing.assert_allclose(y2[0], np.convolve(h[0, 0], h[1, 0])[:L], rtol=1e-12, atol=1e-12)


def test_shift_equivariance():
    """'The primitive': shifting v and the gates right by s shifts y by s."""
    rng = np.random.default_rng(3)
    L, N, s = 80, 2, 13
    v = rng.standard_normal((1, L))
    gates = rng.standard_normal((N, 1, L))
    h = rng.standard_normal((N, 1, L))
    dskip = rng.standard_normal((N, 1))
    y = oracle.hyena_1d(v, gates, h, dskip)
    vs = np.zeros_like(v)
    vs[:, s:] = v[:, :L - s]
    gs = rng.standard_normal(gates.shape)          # gates before s see a zero state
    gs[:, :, s:] = gates[:, :, :L - s]
    ys = oracle.hyena_1d(vs, gs, h, dskip)
    np.testing.assert_array_equal(ys[:, :s], 0.0)
    np.testing.assert_allclose(ys[:, s:], y[:, :L - s], rtol=1e-13, atol=1e-13)


def test_order_collapse():
    """'The Hyena operator': with x^2 = 1, h^2 = delta, D^2 = 0 the order-2 chain is the order-1 one."""
    rng = np.random.default_rng(4)
    L = 64
    v = rng.standard_normal((3, L))
    g1 = rng.standard_normal((1, 3, L))
    h1 = rng.standard_normal((1, 3, L))
    d1 = rng.standard_normal((1, 3))
    y1 = oracle.hyena_1d(v, g1, h1, d1)
    delta = np.zeros((1, 3, L))
    delta[..., 0] = 1.0
    y2 = oracle.hyena_1d(v, np.concatenate([g1, _ones((1, 3, L))]), np.concatenate([h1, delta]),
                         np.concatenate([d1, np.zeros((1, 3))]))
    np.testing.assert_allclose(y2, y1, rtol=1e-14, atol=1e-14)


@pytest.mark.parametrize("L", [1, 2, 5, 16, 31])
def test_convolution_theorem_naive_dft(L):
    """'The convolution theorem' + padding: a naive DFT product on inputs padded to
    M = next_pow2(2L) equals the direct causal convolution; without padding it does not."""
    rng = np.random.default_rng(5 + L)
    h = rng.standard_normal(L)
    v = rng.standard_normal(L)

    def naive_circular(a, b, M):
        t = np.arange(M)
        Fm = np.exp(-2j * np.pi * np.outer(t, t) / M)          # DFT matrix from its definition
        ap = np.zeros(M); ap[:len(a)] = a
        bp = np.zeros(M); bp[:len(b)] = b
        return (np.conj(Fm) @ ((Fm @ ap) * (Fm @ bp))).real / M

    M = 1 << max(0, (2 * L - 1).bit_length())
    y = oracle.hyena_1d(v[None], _ones((1, 1, L)), h[None, None])[0]
    np.testing.assert_allclose(y, naive_circular(h, v, M)[:L], rtol=1e-10, atol=1e-10)
    if L >= 2:
        wrapped = naive_circular(h, v, L)
        assert np.max(np.abs(wrapped - y)) > 1e-6


def test_geometric_filter_closed_form():
    """'The decay window': h_t = r^t, v = 1 gives c_t = (1 - r^(t+1)) / (1 - r)."""
    L, r = 200, 0.97
    t = np.arange(L)
    h = (r ** t)[None, None]
    y = oracle.hyena_1d(_ones((1, L)), _ones((1, 1, L)), h)[0]
    np.testing.assert_allclose(y, (1 - r ** (t + 1)) / (1 - r), rtol=1e-12)


def test_feedthrough_only():
    """'FFTConv': with h = 0 the operator is the gated skip x^n * D^n * z^{n-1}."""
    rng = np.random.default_rng(6)
    L = 33
    v = rng.standard_normal((2, L))
    gates = rng.standard_normal((2, 2, L))
    dskip = rng.standard_normal((2, 2))
    y = oracle.hyena_1d(v, gates, np.zeros((2, 2, L)), dskip)
    expect = gates[1] * dskip[1][:, None] * (gates[0] * dskip[0][:, None] * v)
    np.testing.assert_allclose(y, expect, rtol=1e-15)


def test_numpy_convolve_cross_check():
    """Library routine: numpy's direct convolution, gated, with feedthrough (order 1)."""
    rng = np.random.default_rng(7)
    R, L = 5, 700
    v = rng.standard_normal((R, L))
    gates = rng.standard_normal((1, R, L))
    h = rng.standard_normal((1, R, L)) * np.exp(-0.01 * np.arange(L))
    dskip = rng.standard_normal((1, R))
    y = oracle.hyena_1d(v, gates, h, dskip)
    for r in range(R):
        c = np.convolve(h[0, r], v[r])[:L]
        np.testing.assert_allclose(y[r], gates[0, r] * (c + dskip[0, r] * v[r]), rtol=1e-9, atol=1e-9)


def test_filter_index_and_threads():
    """Row r uses filter row fidx[r]; the thread count does not change any bit."""
    rng = np.random.default_rng(8)
    R, F, L, N = 12, 3, 40, 2
    v = rng.standard_normal((R, L))
    gates = rng.standard_normal((N, R, L))
    h = rng.standard_normal((N, F, L))
    dskip = rng.standard_normal((N, F))
    fidx = rng.integers(0, F, R)
    y = oracle.hyena_1d(v, gates, h, dskip, fidx, threads=1)
    for r in range(R):
        yr = oracle.hyena_1d(v[r:r + 1], gates[:, r:r + 1], h[:, fidx[r]:fidx[r] + 1], dskip[:, fidx[r]:fidx[r] + 1])
        np.testing.assert_array_equal(y[r], yr[0])
    np.testing.assert_array_equal(oracle.hyena_1d(v, gates, h, dskip, fidx, threads=7), y)


def test_bad_arguments_rejected():
    with pytest.raises(ValueError):
        oracle.hyena_1d(np.zeros((2, 8)), np.zeros((1, 2, 7)), np.zeros((1, 2, 8)))
    with pytest.raises(RuntimeError):
        oracle.hyena_1d(np.zeros((2, 8)), np.zeros((1, 2, 8)), np.zeros((1, 2, 8)), fidx=np.array([0, 5]))


# ---------------------------------------------------------------- 2D chain --

def test_2d_delta_kernel_is_identity():
    rng = np.random.default_rng(20)
    P, H, W = 2, 5, 7
    v = rng.standard_normal((P, H, W))
    gates = rng.standard_normal((1, P, H, W))
    k = np.zeros((1, P, 2 * H, 2 * W))
    k[:, :, H, W] = 1.0                               # offset (0, 0)
    dskip = rng.standard_normal((1, P))
    y = oracle.hyena_2d(v, gates, k, dskip)
    np.testing.assert_allclose(y, gates[0] * (1.0 + dskip[0][:, None, None]) * v, rtol=1e-15)


def test_2d_separable_kernel_matches_1d_convolutions():
    """A separable kernel a(oy) b(ox) gives non-causal 1D convolutions along each axis (numpy)."""
    rng = np.random.default_rng(21)
    H, W = 9, 6
    v = rng.standard_normal((1, H, W))
    a = rng.standard_normal(2 * H)                    # a[oy + H]
    b = rng.standard_normal(2 * W)                    # b[ox + W]
    k = np.outer(a, b)[None, None]
    y = oracle.hyena_2d(v, _ones((1, 1, H, W)), k)
    rows = np.stack([np.convolve(v[0, i], b)[W:W + W] for i in range(H)])            # along x
    expect = np.stack([np.convolve(rows[:, j], a)[H:H + H] for j in range(W)], axis=1)  # along y
    np.testing.assert_allclose(y[0], expect, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("N", [1, 2])
def test_2d_scipy_convolve2d_cross_check(N):
    """Library routine: scipy.signal.convolve2d (full) cropped at the zero offset, gated, chained."""
    rng = np.random.default_rng(22 + N)
    P, H, W = 3, 6, 5
    v = rng.standard_normal((P, H, W))
    gates = rng.standard_normal((N, P, H, W))
    k = rng.standard_normal((N, P, 2 * H, 2 * W))
    dskip = rng.standard_normal((N, P))
    y = oracle.hyena_2d(v, gates, k, dskip)
    for p in range(P):
        z = v[p]
        for n in range(N):
            full = scipy.signal.convolve2d(z, k[n, p])
            c = full[H:2 * H, W:2 * W]                # offset index oy + H -> output row i
            z = gates[n, p] * (c + dskip[n, p] * z)
        np.testing.assert_allclose(y[p], z, rtol=1e-11, atol=1e-11)


# -------------------------------------------------------- implicit filters --

def _onehot_net(width, fin, out, feat_index, a):
    """Weights under which the sine network collapses to sin(w_h sin(w0 a f)) for one feature f."""
    W1 = np.zeros((width, fin)); W1[0, feat_index] = a
    W2 = np.zeros((width, width)); W2[0, 0] = 1.0
    W3 = np.zeros((out, width)); W3[:, 0] = 1.0
    return W1, np.zeros(width), W2, np.zeros(width), W3, np.zeros(out)


@pytest.mark.parametrize("feat_index,fn", [
    (0, lambda t, L: t / L),
    (5, lambda t, L: np.cos(2 * np.pi * 3 * t / L)),     # features: t/L, cos1, sin1, cos2, sin2, cos3 ...
    (6, lambda t, L: np.sin(2 * np.pi * 3 * t / L)),
])
def test_implicit_1d_reduces_to_closed_form(feat_index, fn):
    L, N, D, K, width = 64, 2, 3, 4, 8
    a, w0, wh = 1.7, 1.3, 0.9
    alpha = np.linspace(0.0, 0.2, N * D).reshape(N, D)
    h = oracle.implicit_filter_1d(L, N, D, *_onehot_net(width, 1 + 2 * K, N * D, feat_index, a), alpha, K, w0, wh)
    t = np.arange(L)
    base = np.sin(wh * np.sin(w0 * a * fn(t, L)))
    for n in range(N):
        for d in range(D):
            np.testing.assert_allclose(h[n, d], np.exp(-alpha[n, d] * t) * base, rtol=1e-13, atol=1e-15)


def test_implicit_1d_window_only():
    """W3 = 0 leaves b3 under the window: h = b3 exp(-alpha t); at t = 0 the window is 1."""
    L, N, D, K, width = 32, 1, 4, 2, 8
    W1, b1, W2, b2, W3, _ = _onehot_net(width, 1 + 2 * K, N * D, 0, 1.0)
    b3 = np.array([0.5, -1.0, 2.0, 3.0])
    alpha = np.array([[0.0, 0.1, 0.5, 1.0]])
    h = oracle.implicit_filter_1d(L, N, D, W1, b1, W2, b2, np.zeros_like(W3), b3, alpha, K)
    np.testing.assert_allclose(h[0], b3[:, None] * np.exp(-alpha[0][:, None] * np.arange(L)), rtol=1e-14)
    np.testing.assert_array_equal(h[0, :, 0], b3)


@pytest.mark.parametrize("axis", [0, 1])
def test_implicit_2d_reduces_to_closed_form(axis):
    H, W, N, C, width = 4, 6, 1, 2, 8
    a, w0, wh = 0.8, 10.0, 1.0
    sigma = np.array([[0.5, 0.9]])
    k = oracle.implicit_filter_2d(H, W, N, C, *_onehot_net(width, 2, N * C, axis, a), sigma, w0, wh)
    oy = np.arange(-H, H) / H
    ox = np.arange(-W, W) / W
    py, px = np.meshgrid(oy, ox, indexing="ij")
    coord = py if axis == 0 else px
    for c in range(C):
        expect = np.exp(-(py ** 2 + px ** 2) / (2 * sigma[0, c] ** 2)) * np.sin(wh * np.sin(w0 * a * coord))
        np.testing.assert_allclose(k[0, c], expect, rtol=1e-13, atol=1e-15)
    # offset (0, 0) sits at [H, W] and has window 1 and coordinate 0
    np.testing.assert_array_equal(k[0, :, H, W], 0.0)


# Bias placement and hidden-weight orientation. The one-hot pins above run with
# zero biases and a symmetric W2, so they cannot tell sin(w0 (W1 g + b1)) from
# sin(w0 W1 g) + b1, nor a1 W2^T from a1 W2. The nets below can: a non-zero
# bias in the first unit of each hidden layer, and a W2 whose only entry sits
# off the diagonal (unit 0 of layer 1 feeds unit 1 of layer 2, which the head
# reads). The reading is the sine-network convention: each bias is added to
# the pre-activation and scaled by that layer's frequency together with it
# ("Hyena — Long Convolutions Math", "Implicit filters: an MLP over positions";
# "How HyenaND works", "1. An implicit filter").

def _biased_net(width, fin, out, feat_index, a, b1_0, b2_0):
    W1, b1, W2, b2, W3, b3 = _onehot_net(width, fin, out, feat_index, a)
    b1[0], b2[0] = b1_0, b2_0
    return W1, b1, W2, b2, W3, b3


def _offdiag_net(width, fin, out, feat_index, a, c):
    W1 = np.zeros((width, fin)); W1[0, feat_index] = a
    W2 = np.zeros((width, width)); W2[1, 0] = c       # layer-2 unit 1 reads layer-1 unit 0
    W3 = np.zeros((out, width)); W3[:, 1] = 1.0       # the head reads layer-2 unit 1
    return W1, np.zeros(width), W2, np.zeros(width), W3, np.zeros(out)


def _closed_biased(f, a, b1_0, b2_0, w0, wh):
    return np.sin(wh * (np.sin(w0 * (a * f + b1_0)) + b2_0))


def _closed_offdiag(f, a, c, w0, wh):
    return np.sin(wh * c * np.sin(w0 * a * f))


def _check_1d_bias(fn_1d):
    L, N, D, K, width = 48, 1, 2, 3, 8
    a, b1_0, b2_0, w0, wh = 1.3, 0.4, -0.7, 1.1, 0.8
    alpha = np.array([[0.0, 0.05]])
    h = fn_1d(L, N, D, *_biased_net(width, 1 + 2 * K, N * D, 0, a, b1_0, b2_0), alpha, K, w0, wh)
    t = np.arange(L)
    base = _closed_biased(t / L, a, b1_0, b2_0, w0, wh)
    for d in range(D):
        np.testing.assert_allclose(h[0, d], np.exp(-alpha[0, d] * t) * base, rtol=1e-13, atol=1e-15)


def _check_1d_offdiag(fn_1d):
    L, N, D, K, width = 48, 2, 1, 3, 8
    a, c, w0, wh = 1.9, 1.6, 0.7, 1.2
    alpha = np.array([[0.02], [0.0]])
    h = fn_1d(L, N, D, *_offdiag_net(width, 1 + 2 * K, N * D, 4, a, c), alpha, K, w0, wh)
    t = np.arange(L)
    base = _closed_offdiag(np.sin(2 * np.pi * 2 * t / L), a, c, w0, wh)   # feature 4 = sin(2 pi 2 t / L)
    for n in range(N):
        np.testing.assert_allclose(h[n, 0], np.exp(-alpha[n, 0] * t) * base, rtol=1e-13, atol=1e-15)


def _check_2d_bias_offdiag(fn_2d):
    H, W, N, C, width = 4, 4, 1, 2, 8
    a, b1_0, b2_0, c, w0, wh = 0.6, 0.3, 0.5, -1.4, 10.0, 1.0
    sigma = np.array([[0.5, 0.8]])
    oy = np.arange(-H, H) / H
    ox = np.arange(-W, W) / W
    py, px = np.meshgrid(oy, ox, indexing="ij")
    win = [np.exp(-(py ** 2 + px ** 2) / (2 * sigma[0, ch] ** 2)) for ch in range(C)]
    k = fn_2d(H, W, N, C, *_biased_net(width, 2, N * C, 1, a, b1_0, b2_0), sigma, w0, wh)
    for ch in range(C):
        np.testing.assert_allclose(k[0, ch], win[ch] * _closed_biased(px, a, b1_0, b2_0, w0, wh),
                                   rtol=1e-12, atol=1e-14)
    k = fn_2d(H, W, N, C, *_offdiag_net(width, 2, N * C, 0, a, c), sigma, w0, wh)
    for ch in range(C):
        np.testing.assert_allclose(k[0, ch], win[ch] * _closed_offdiag(py, a, c, w0, wh), rtol=1e-12, atol=1e-14)


def test_implicit_1d_bias_inside_the_frequency():
    """b1, b2 non-zero: h = window * sin(w_h (sin(w0 (a f + b1_0)) + b2_0))."""
    _check_1d_bias(oracle.implicit_filter_1d)


def test_implicit_1d_hidden_weight_orientation():
    """W2[1, 0] = c, head on unit 1: h = window * sin(w_h c sin(w0 a f)); W2 transposed gives 0."""
    _check_1d_offdiag(oracle.implicit_filter_1d)


def test_implicit_2d_bias_and_hidden_weight_orientation():
    _check_2d_bias_offdiag(oracle.implicit_filter_2d)


# Planted mistakes, in a copy of the network on the CPU: each must fail a pin above.
def _mlp_bias_outside(feat, W1, b1, W2, b2, W3, b3, omega0, omega_hidden):
    a1 = np.sin(omega0 * (feat @ W1.T)) + b1
    a2 = np.sin(omega_hidden * (a1 @ W2.T)) + b2
    return a2 @ W3.T + b3


def _mlp_w2_transposed(feat, W1, b1, W2, b2, W3, b3, omega0, omega_hidden):
    a1 = np.sin(omega0 * (feat @ W1.T + b1))
    a2 = np.sin(omega_hidden * (a1 @ W2 + b2))
    return a2 @ W3.T + b3


def _mlp_bias_unscaled(feat, W1, b1, W2, b2, W3, b3, omega0, omega_hidden):
    a1 = np.sin(omega0 * (feat @ W1.T) + b1)
    a2 = np.sin(omega_hidden * (a1 @ W2.T) + b2)
    return a2 @ W3.T + b3


@pytest.mark.parametrize("planted,check", [
    (_mlp_bias_outside, _check_1d_bias),
    (_mlp_bias_unscaled, _check_1d_bias),
    (_mlp_w2_transposed, _check_1d_offdiag),
    (_mlp_bias_outside, _check_2d_bias_offdiag),
    (_mlp_bias_unscaled, _check_2d_bias_offdiag),
    (_mlp_w2_transposed, _check_2d_bias_offdiag),
])
def test_implicit_pins_catch_planted_mistakes(monkeypatch, planted, check):
    import oracle.implicit as imp
    monkeypatch.setattr(imp, "_mlp", planted)
    fn = imp.implicit_filter_1d if check is not _check_2d_bias_offdiag else imp.implicit_filter_2d
    with pytest.raises(AssertionError):
        check(fn)


# ------------------------------------------------------------ gate sandwich --
# "How HyenaND works", "Putting it together: the HyenaND operator":
# Z = q ⊙ SiLU(k), H = K ∗ Z, O = H ⊙ SiLU(v).

def test_silu_special_values():
    s = oracle.silu(np.array([0.0, 1.0, -1.0, 40.0, -40.0, 800.0, -800.0]))
    assert s[0] == 0.0
    assert s[1] == pytest.approx(1.0 / (1.0 + np.exp(-1.0)), rel=1e-15)           # 0.7310585786300049
    assert s[2] == pytest.approx(-1.0 / (1.0 + np.exp(1.0)), rel=1e-15)
    assert s[3] == pytest.approx(40.0, rel=1e-15) and abs(s[4]) < 1e-15          # SiLU(x) -> x, -> 0
    assert s[5] == 800.0 and s[6] == 0.0 and np.all(np.isfinite(s))              # no overflow
    x = np.linspace(-12, 12, 2001)
    np.testing.assert_allclose(oracle.silu(x), x * scipy.special.expit(x), rtol=1e-14, atol=1e-300)


def test_gated_2d_delta_kernel_is_the_gates_alone():
    """K = δ at offset 0: y = SiLU(x) · (1 + Dskip) · q · SiLU(k), element by element."""
    rng = np.random.default_rng(41)
    P, H, W = 3, 5, 4
    q, k, x = rng.standard_normal((3, P, H, W))
    kern = np.zeros((1, P, 2 * H, 2 * W)); kern[0, :, H, W] = 1.0
    dsk = rng.standard_normal((1, P))
    y = oracle.hyena_gated(q, k, x[None], kern, dsk)
    sig = lambda a: a * scipy.special.expit(a)
    np.testing.assert_allclose(y, sig(x) * (1.0 + dsk[0][:, None, None]) * q * sig(k), rtol=1e-13, atol=1e-14)


def test_gated_2d_matches_scipy_with_both_gates():
    """O = (K ∗ (q ⊙ SiLU(k))) ⊙ SiLU(v) with scipy's full 2D convolution cropped at offset 0."""
    rng = np.random.default_rng(42)
    P, H, W = 2, 6, 7
    q, k, v = rng.standard_normal((3, P, H, W))
    kern = rng.standard_normal((1, P, 2 * H, 2 * W))
    y = oracle.hyena_gated(q, k, v[None], kern)
    sig = lambda a: a * scipy.special.expit(a)
    for p in range(P):
        c = scipy.signal.convolve2d(q[p] * sig(k[p]), kern[0, p])[H:2 * H, W:2 * W]
        np.testing.assert_allclose(y[p], c * sig(v[p]), rtol=1e-11, atol=1e-11)


def test_gated_saturated_gates_reduce_to_the_plain_operator():
    """k, x -> +inf make both SiLU gates the identity on k and x scaled out: with k = x = 50
    the sandwich equals 50 · 50 · (plain chain on q with unit gates)."""
    rng = np.random.default_rng(43)
    R, L = 3, 40
    q = rng.standard_normal((R, L))
    h = rng.standard_normal((1, R, L)) * np.exp(-0.1 * np.arange(L))
    y = oracle.hyena_gated(q, np.full((R, L), 50.0), np.full((1, R, L), 50.0), h)
    plain = oracle.hyena_1d(q, np.ones((1, R, L)), h)
    np.testing.assert_allclose(y, 2500.0 * plain, rtol=1e-13, atol=1e-13)
    # and k -> -inf closes the inner gate: the output is zero
    y0 = oracle.hyena_gated(q, np.full((R, L), -800.0), rng.standard_normal((1, R, L)), h)
    assert np.all(y0 == 0.0)


def test_order1_outputs_at_positions_match_the_chain_and_the_worked_example():
    """Single outputs by their own direct sums equal the full order-1 chain, and reproduce the
    worked example of 'Linear vs circular' (h = [1, .5, .25, .125], x = [1, 2, 0, 0])."""
    rng = np.random.default_rng(51)
    L = 300
    v, x, h = rng.standard_normal((3, L))
    d = 0.7
    full = oracle.hyena_1d(v[None], x[None, None], h[None, None], np.array([[d]]))[0]
    pos = [0, 1, 2, 150, 298, 299]
    np.testing.assert_allclose(oracle.hyena_1d_order1_at(v, x, h, d, pos), full[pos], rtol=1e-12, atol=1e-12)
    g = _read_golden("worked_example_causal_conv.txt")
    y = oracle.hyena_1d_order1_at(g["x"], np.ones(4), g["h"], None, range(4))
    np.testing.assert_array_equal(y, g["y_linear_causal"])


# ----------------------------------------------------------------- 3D chain --
# "How HyenaND works", "2. The convolution theorem (FFT)": the convolution on
# the native grid of a 3D volume.

def test_3d_delta_kernel_is_identity():
    rng = np.random.default_rng(61)
    P, Dz, H, W = 2, 3, 4, 5
    v = rng.standard_normal((P, Dz, H, W))
    k = np.zeros((1, P, 2 * Dz, 2 * H, 2 * W)); k[0, :, Dz, H, W] = 1.0
    np.testing.assert_array_equal(oracle.hyena_3d(v, _ones((1, P, Dz, H, W)), k), v)


def test_3d_separable_kernel_is_three_1d_convolutions():
    """k = a(oz) b(oy) c(ox): non-causal 1D convolutions along each axis (numpy.convolve)."""
    rng = np.random.default_rng(62)
    Dz, H, W = 4, 3, 5
    v = rng.standard_normal((1, Dz, H, W))
    a, b, c = rng.standard_normal(2 * Dz), rng.standard_normal(2 * H), rng.standard_normal(2 * W)
    k = np.einsum("i,j,l->ijl", a, b, c)[None, None]
    y = oracle.hyena_3d(v, _ones((1, 1, Dz, H, W)), k)
    t = np.apply_along_axis(lambda r: np.convolve(r, c)[W:2 * W], 2, v[0])
    t = np.apply_along_axis(lambda r: np.convolve(r, b)[H:2 * H], 1, t)
    t = np.apply_along_axis(lambda r: np.convolve(r, a)[Dz:2 * Dz], 0, t)
    np.testing.assert_allclose(y[0], t, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("N", [1, 2])
def test_3d_scipy_convolve_cross_check(N):
    """Library routine: scipy.signal.convolve (N-D, direct, full) cropped at the zero offset, gated, chained."""
    rng = np.random.default_rng(63 + N)
    P, Dz, H, W = 2, 3, 4, 3
    v = rng.standard_normal((P, Dz, H, W))
    gates = rng.standard_normal((N, P, Dz, H, W))
    k = rng.standard_normal((N, P, 2 * Dz, 2 * H, 2 * W))
    dskip = rng.standard_normal((N, P))
    y = oracle.hyena_3d(v, gates, k, dskip)
    for p in range(P):
        z = v[p]
        for n in range(N):
            full = scipy.signal.convolve(z, k[n, p], method="direct")
            c = full[Dz:2 * Dz, H:2 * H, W:2 * W]
            z = gates[n, p] * (c + dskip[n, p] * z)
        np.testing.assert_allclose(y[p], z, rtol=1e-11, atol=1e-11)


def test_3d_single_slice_reduces_to_2d():
    """Dz = 1: only offset oz = 0 touches the output, and the chain is the 2D one on that slice."""
    rng = np.random.default_rng(65)
    P, H, W = 3, 5, 4
    v = rng.standard_normal((P, 1, H, W))
    gates = rng.standard_normal((2, P, 1, H, W))
    k = rng.standard_normal((2, P, 2, 2 * H, 2 * W))
    dskip = rng.standard_normal((2, P))
    y3 = oracle.hyena_3d(v, gates, k, dskip)
    y2 = oracle.hyena_2d(v[:, 0], gates[:, :, 0], k[:, :, 1], dskip)
    np.testing.assert_allclose(y3[:, 0], y2, rtol=1e-13, atol=1e-13)


def test_3d_order1_voxels_match_the_chain():
    rng = np.random.default_rng(66)
    Dz, H, W = 3, 4, 5
    v, x = rng.standard_normal((2, Dz, H, W))
    k = rng.standard_normal((2 * Dz, 2 * H, 2 * W))
    full = oracle.hyena_3d(v[None], x[None, None], k[None, None], np.array([[0.4]]))[0]
    vox = [(0, 0, 0), (2, 3, 4), (1, 2, 0), (0, 3, 2)]
    got = oracle.hyena_3d_order1_at(v, x, k, 0.4, vox)
    np.testing.assert_allclose(got, [full[i] for i in vox], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("axis", [0, 1, 2])
def test_implicit_3d_reduces_to_closed_form(axis):
    """One coordinate through one unit per layer: K = Gaussian(|p|) sin(w_h sin(w0 a p_axis))."""
    Dz, H, W, N, C, width = 2, 3, 4, 1, 2, 8
    a, w0, wh = 0.7, 10.0, 1.0
    sigma = np.array([[0.5, 0.8]])
    k = oracle.implicit_filter_3d(Dz, H, W, N, C, *_onehot_net(width, 3, N * C, axis, a), sigma, w0, wh)
    pz, py, px = np.meshgrid(np.arange(-Dz, Dz) / Dz, np.arange(-H, H) / H, np.arange(-W, W) / W, indexing="ij")
    coord = (pz, py, px)[axis]
    for c in range(C):
        expect = np.exp(-(pz ** 2 + py ** 2 + px ** 2) / (2 * sigma[0, c] ** 2)) * np.sin(wh * np.sin(w0 * a * coord))
        np.testing.assert_allclose(k[0, c], expect, rtol=1e-13, atol=1e-15)
    np.testing.assert_array_equal(k[0, :, Dz, H, W], 0.0)     # offset 0: coordinate 0, window 1
