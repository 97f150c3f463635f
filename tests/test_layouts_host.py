"""Host-side checks of the kernels' shared-memory layouts and of the algebra of
their spectral step (CPU only). The address formulas are restated here from
csrc/cta_fft.cuh (maddr), csrc/kernels_1d_pair.cuh (swz2) and the pass plan
of csrc/fft_regs.cuh, and checked for the properties the kernels rely on:
every exchange of every Stockham pass is bank-conflict-free, and the
pairwise spectral step covers every bin exactly once with the right value."""
import numpy as np
import pytest


# ---------------------------------------------------------------- layouts --

def plan(L, LR):
    """Radices of the passes of a length-L FFT with largest radix 2^LR (the last one smaller)."""
    out, rr = [], L
    while rr % (1 << LR) == 0 and rr > 1:
        rr //= 1 << LR
        out.append(1 << LR)
    return out + ([rr] if rr > 1 else [])


def worst_ways(addrs, group, banks):
    """Largest number of distinct words one bank group serves within a hardware phase."""
    w = 1
    for h in range(0, len(addrs), group):
        seen = {}
        for a in addrs[h:h + group]:
            seen.setdefault(a % banks, set()).add(a)
        w = max(w, max(len(v) for v in seen.values()))
    return w


def stockham_accesses(L, E, T):
    """Yield, per (pass write or read), the element index touched by each of T lanes t."""
    LR = {16: 4, 8: 3}[E]
    P = plan(L, LR)
    ns = 1
    for p, R in enumerate(P):
        S = E // R
        if p < len(P) - 1:
            for s in range(S):
                for r in range(R):
                    yield [((t + s * T) // ns) * ns * R + (t + s * T) % ns + r * ns for t in range(T)]
        if p > 0:
            for q in range(E):
                yield [t + q * T for t in range(T)]
        ns *= R
    for q in range(E):   # natural-order loads and stores around the transform
        yield [t + q * T for t in range(T)]


def maddr(i, s, L, nsw):
    if nsw >= 16:
        return s * L + (i ^ (s & 31))
    par = bin((i >> 1) & 15).count("1") & 1
    return s * L + (i ^ (((2 * s) & 15) | par))


@pytest.mark.parametrize("L,E,nseq,elem", [
    (256, 16, 16, 8), (128, 16, 32, 8), (512, 16, 16, 8), (256, 16, 32, 8),   # cluster and staged kernels
    (512, 8, 8, 8), (256, 8, 8, 8), (128, 8, 8, 8), (64, 8, 8, 8),          # 2D cluster columns (radix 8)
    (512, 16, 8, 8),                                                         # staged 2D columns
    (256, 16, 8, 16), (128, 16, 16, 16), (256, 16, 32, 16),                 # lockstep pairs (16-byte elements)
])
def test_sequence_major_exchanges_are_conflict_free(L, E, nseq, elem):
    """Warps span nseq sequences at a common element (lane = s + nseq * t); 8-byte elements are
    served a half-warp at a time on 16 bank pairs, 16-byte elements a quarter-warp at a time on 8."""
    T = L // E
    group, banks = (16, 16) if elem == 8 else (8, 8)
    nsw = 32 if elem == 16 else nseq
    lanes = [(lane % nseq, lane // nseq) for lane in range(32)]
    worst = 1
    for t0 in range(0, T, 32 // nseq):
        for idx in stockham_accesses(L, E, T):
            addrs = [maddr(idx[(t0 + dt) % T], s, L, nsw) for (s, dt) in lanes if t0 + dt < T]
            worst = max(worst, worst_ways(addrs, group, banks))
    assert worst == 1, (L, E, nseq, elem, worst)


def test_old_eight_sequence_swizzle_would_conflict():
    """The plain XOR of the sequence index is not enough with 8 sequences per warp (negative control)."""
    L, E, nseq, T = 256, 16, 8, 16
    lanes = [(lane % nseq, lane // nseq) for lane in range(32)]
    worst = 1
    for idx in stockham_accesses(L, E, T):
        addrs = [s * L + (idx[dt] ^ (s & 31)) for (s, dt) in lanes]
        worst = max(worst, worst_ways(addrs, 16, 16))
    assert worst > 1


@pytest.mark.parametrize("MC", [256, 1024, 2048, 4096, 8192])
def test_pair_kernel_swizzle_is_conflict_free(MC):
    """swz2 (8-byte words, one sequence per thread group of MC/16 lanes) for every pass pattern."""
    swz2 = lambda i: i ^ ((i >> 4) & 15)
    E, T = 16, MC // 16
    worst = 1
    for idx in stockham_accesses(MC, E, T):
        addrs = [swz2(i) for i in idx]
        worst = max(worst, worst_ways(addrs, 16, 16))
    assert worst == 1


# ------------------------------------------------------ spectral algebra --

def test_pairwise_spectral_step_matches_per_bin():
    """Bins k and MC-k from one set of intermediates: Z'[MC-k] = conj(Ye - i Yo)."""
    rng = np.random.default_rng(7)
    MC = 128
    M = 2 * MC
    x = rng.standard_normal(M)
    H = rng.standard_normal(MC + 1) + 1j * rng.standard_normal(MC + 1)
    H[0], H[MC] = H[0].real, H[MC].real
    dsk = 0.7
    Z = np.fft.fft(x[0::2] + 1j * x[1::2])
    w = np.exp(-2j * np.pi * np.arange(MC) / M)

    def pieces(k):
        km = (MC - k) % MC
        Ek = (Z[k] + np.conj(Z[km])) / 2
        Ok = (Z[k] - np.conj(Z[km])) / 2j
        Xk, Xm = Ek + w[k] * Ok, np.conj(Ek - w[k] * Ok)
        Yk, Ym = Xk * (H[k] + dsk), Xm * (H[MC - k] + dsk)
        return (Yk + np.conj(Ym)) / 2, (Yk - np.conj(Ym)) * np.conj(w[k]) / 2

    per_bin = np.array([sum([pieces(k)[0], 1j * pieces(k)[1]]) for k in range(MC)])
    E, T = 16, MC // 16
    out = np.full(MC, np.nan, complex)
    for t in range(T):
        for q in list(range(E // 2)) + ([E // 2] if t == 0 else []):
            k = t + q * T
            Ye, Yo = pieces(k)
            out[k] = Ye + 1j * Yo
            km = (MC - k) % MC
            if km != k and not (t == 0 and q == E // 2):
                assert np.isnan(out[km]) or km == 0
                out[km] = np.conj(Ye - 1j * Yo)
    assert not np.isnan(out).any()
    np.testing.assert_allclose(out, per_bin, rtol=0, atol=1e-12)
    # and the whole step reproduces the convolution: inverse half-length FFT, unpack
    y = np.fft.ifft(out)
    yr = np.empty(M)
    yr[0::2], yr[1::2] = y.real, y.imag
    ref = np.fft.irfft(np.fft.rfft(x) * (H + dsk), M)
    np.testing.assert_allclose(yr, ref, rtol=0, atol=1e-10)


@pytest.mark.parametrize("MC,M1,NROW,twod", [(32768, 128, 16, False), (65536, 256, 16, False),
                                              (65536, 256, 8, False), (131072, 512, 32, True),
                                              (131072, 512, 8, True)])
def test_mirror_handoff_covers_every_bin_once(MC, M1, NROW, twod):
    """Row groups hold rows k1 and M1 - k1 (row 0's partner slot holds M1/2); each thread computes its
    registers q < E/2 and hands the mirror result over; the rest is its own mirror (t2 = 0)."""
    E, M2 = 16, MC // M1
    T2, HROW = M2 // E, NROW // 2

    def row_of_slot(g, r):
        base = g * HROW + (r % HROW)
        return base if r < HROW else (M1 // 2 if base == 0 else M1 - base)

    written, computed = {}, set()
    for g in range(M1 // NROW):
        for r in range(NROW):
            k1 = row_of_slot(g, r)
            rm = r if k1 in (0, M1 // 2) else (r + HROW if r < HROW else r - HROW)
            assert row_of_slot(g, rm) == (M1 - k1) % M1
            for t2 in range(T2):
                for q in range(E // 2):
                    k2 = t2 + q * T2
                    computed.add((g, r, k2))
                    if twod:
                        k2m = (M2 - k2) % M2
                    else:
                        k2m = ((MC - (k1 + M1 * k2)) % MC) // M1
                    written.setdefault((g, rm, k2m), []).append((g, r, k2))
                if (t2 == 0) and (twod or k1 == 0):
                    computed.add((g, r, t2 + (E // 2) * T2))
    for g in range(M1 // NROW):
        for r in range(NROW):
            for t2 in range(T2):
                for q in range(E // 2, E):
                    key = (g, r, t2 + q * T2)
                    if key not in computed:
                        assert len(written.get(key, [])) == 1, key
