// 2D (HyenaND-style) fused forward and kernel spectrum: one thread-block
// cluster per (batch, channel) plane.
//
// A real plane v[y][x] of H x W is zero-padded to 2H x 2W and packed along x,
// z[y][x'] = v[y][2x'] + i v[y][2x'+1], giving a complex [M1 = 2H][M2 = W]
// array. Its 2D DFT is the cluster four-step transform without the
// inter-stage twiddle (columns = y, rows = x'). Only y < H and x' < W/2 carry
// data, so both stages start from half-zero input and the inverse keeps only
// that quarter. The real-packing identity along x unpacks the spectrum with
// the 2D mirror bin Z[-ky][-kx'] and the twiddle W_{2W}^{kx'}.
//
// Convolution ("How HyenaND works", "2. The convolution theorem (FFT)"): the
// kernel on offsets o in [-H, H) x [-W, W) is placed cyclically (offset o at
// index o mod 2H, o mod 2W), so the cyclic product of the padded plane with it
// is the linear, non-causal convolution, read out on [0, H) x [0, W).
#pragma once
#include "kernels_1d_cluster.cuh"

namespace hyena {

struct Fwd2dArgs {
    const void *v;        // the convolution input; with the gate sandwich, q
    const void *k;        // gate sandwich only: the inner gate's key (z^0 = q SiLU(k))
    const void *gates[HYENA_MAX_ORDER];
    const c32 *K;         // [N, C, W + 1, 2H]: bin (ky, kx) at kx * 2H + ky
    const float *dskip;   // [N, C] or nullptr
    void *y;
    const c32 *tw;        // W_TWM^m
    int64_t planes;       // B * C
    int64_t C;
    int64_t B;
    int order;
    int *err;             // the plan's device error word (index checks of the debug build)
};

// Fused order-N 2D forward (planes visited c-major, b-minor). GATED: the
// gate sandwich, z^0 = q SiLU(k) formed at the load and SiLU applied to every
// gate x^n where it multiplies.
template <typename G, typename IO, bool GATED>
__global__ void __launch_bounds__(G::THREADS, G::MINB) hyena_fwd_2d_cluster(const Fwd2dArgs a) {
    using Ctx = ClusterCtx<G, false, true>;
    constexpr int E = G::E, M1 = G::M1, M2 = G::M2;
    constexpr int Hh = M1 / 2, Ww = M2;                 // plane extents
    constexpr int TWM = Ctx::TWM;
    extern __shared__ float smem[];
    Ctx cx(smem);
    const int64_t ord = (int64_t)blockIdx.x / G::C;
    const int64_t c = ord / a.B;
    const int64_t b = ord - c * a.B;
    const int64_t plane = b * a.C + c;
    const c32 wb = ldg_c(a.tw + cx.t2 * (TWM / (2 * M2)));   // W_{2 M2}^{t2}

    // Column-layout register q < E1 holds (y = t1 + q T1P, x' = n2); every
    // column of the column phase carries data (x' < W/2), and the registers
    // q < E1/2 hold the data rows y < H.
    constexpr int E1 = Ctx::E1;
    auto pos_of = [&](int q) -> int64_t { return (int64_t)(cx.t1 + q * Ctx::T1P) * Ww + 2 * cx.n2; };

    c32 v[E];
    {
        const IO *vp = reinterpret_cast<const IO *>(a.v) + plane * Hh * Ww;
        const IO *kp = reinterpret_cast<const IO *>(a.k) + plane * Hh * Ww;
#pragma unroll
        for (int q = 0; q < E1 / 2; ++q) {
            v[q] = load_pair<IO, true>(vp, pos_of(q), (int64_t)Hh * Ww);
            if constexpr (GATED) {
                const c32 kq = silu(load_pair<IO, true>(kp, pos_of(q), (int64_t)Hh * Ww));
                v[q] = mk(v[q].x * kq.x, v[q].y * kq.y);
            }
        }
#pragma unroll
        for (int q = E1 / 2; q < E; ++q) v[q] = mk(0.f, 0.f);
    }

    for (int n = 0; n < a.order; ++n) {
        const IO *gp = reinterpret_cast<const IO *>(a.gates[n]) + plane * Hh * Ww;
        typename io<IO>::pair_t g[E1 / 2];
#pragma unroll
        for (int q = 0; q < E1 / 2; ++q) g[q] = load_pair_raw<IO, true>(gp, pos_of(q), (int64_t)Hh * Ww);
        const float dsk = a.dskip ? __ldg(a.dskip + n * a.C + c) : 0.f;
        const c32 *Kp = a.K + ((int64_t)n * a.C + c) * (M1 * (M2 + 1));

        cx.template forward<true>(v, a.tw);
        cx.publish(v);
        // Spectral step, bins in pairs ((ky, kx), (-ky, -kx)): the mirror of register
        // q is register E-1-q of thread (rm, T2-t2) (register E-q when t2 = 0), so
        // each thread takes q < E/2 and returns the mirror result conj(Ye - i Yo) to
        // its owner; threads with t2 = 0 also take q = E/2 (kx = M2/2, whose mirror
        // is in the upper half of both owners).
        constexpr float s = 0.5f / (float)(M1 * M2);
        const int ky = cx.k1;
        const int kym = (M1 - ky) & (M1 - 1);
        const int z0 = opaque_zero();
        auto bin_pair = [&](int q, c32 Zk, c32 &Ye, c32 &Yo) __attribute__((always_inline)) {
            const int kx = cx.t2 + q * G::T2;
            const c32 Zm = cx.mirror_bin((M2 - kx) & (M2 - 1));
            const c32 Ek = mk(0.5f * (Zk.x + Zm.x), 0.5f * (Zk.y - Zm.y));
            const c32 Ok = mk(0.5f * (Zk.y + Zm.y), -0.5f * (Zk.x - Zm.x));
            const c32 w = mul(wb, w2e<E>(q, z0));            // W_{2 M2}^{kx}
            const c32 wO = mul(w, Ok);
            const c32 Xk = add(Ek, wO);                  // bin (ky, kx)
            const c32 Xm = conj(sub(Ek, wO));            // bin (-ky, M2 - kx)
            c32 Hk = ldg_c(Kp + (int64_t)kx * M1 + ky);              // lanes run along ky: coalesced
            c32 Hm = ldg_c(Kp + (int64_t)(M2 - kx) * M1 + kym);
            Hk.x += dsk;
            Hm.x += dsk;
            const c32 Yk = mul(Xk, Hk), Ym = mul(Xm, Hm);
            Ye = mk(s * (Yk.x + Ym.x), s * (Yk.y - Ym.y));
            const c32 Yd = mk(s * (Yk.x - Ym.x), s * (Yk.y + Ym.y));
            Yo = mul(Yd, conj(w));
        };
        const bool self_half = cx.t2 == 0;
        c32 vh = v[E / 2];
        if (self_half) {
            c32 Ye, Yo;
            bin_pair(E / 2, v[E / 2], Ye, Yo);
            vh = mk(Ye.x - Yo.y, Ye.y + Yo.x);
        }
#pragma unroll
        for (int q = 0; q < E / 2; ++q) {
            c32 Ye, Yo;
            bin_pair(q, v[q], Ye, Yo);
            v[q] = mk(Ye.x - Yo.y, Ye.y + Yo.x);              // Ye + i Yo       (bin (ky, kx))
            v[E / 2 + q] = mk(Ye.x + Yo.y, Yo.x - Ye.y);      // conj(Ye - i Yo) (bin (-ky, -kx))
            if ((q & 3) == 3) asm volatile("" ::: "memory");  // bound load hoisting (register pressure)
        }
        __syncthreads();                                // every mirror read done
#pragma unroll
        for (int q = 0; q < E / 2; ++q) cx.set_mirror_bin((M2 - (cx.t2 + q * G::T2)) & (M2 - 1), v[E / 2 + q]);
        __syncthreads();
#pragma unroll
        for (int q = E / 2; q < E; ++q) v[q] = cx.own_bin(q);
        if (self_half) v[E / 2] = vh;
        __syncthreads();                                // row buffer reads done before the inverse rewrites it
        cx.inverse(v, a.tw);
#pragma unroll
        for (int q = 0; q < E1 / 2; ++q) {
            c32 gq = io<IO>::unpack(g[q]);
            if constexpr (GATED) gq = silu(gq);
            v[q] = mk(gq.x * v[q].x, gq.y * v[q].y);
        }
#pragma unroll
        for (int q = E1 / 2; q < E; ++q) v[q] = mk(0.f, 0.f);
    }

    IO *yp = reinterpret_cast<IO *>(a.y) + plane * Hh * Ww;
#pragma unroll
    for (int q = 0; q < E1 / 2; ++q) store_pair<IO, true>(yp, pos_of(q), (int64_t)Hh * Ww, v[q]);
}

// 2D kernel spectra, stored kx-major ([W + 1][2H] per kernel: the spectral step's
// lanes run along ky). Kernel (n, c) starts at K + o * cs (o = n * C + c); row iy
// of its offset grid (offset oy = iy - H) starts at + iy * rs and holds 2W
// floats (ox = ix - W). In place (K == Kout, rs = 2W + 2, cs = 2H (2W + 2)) is
// allowed: every read precedes the first cluster barrier, every write follows it.
template <typename G>
__global__ void __launch_bounds__(G::THREADS, G::MINB)
    hyena_spectrum_2d_cluster(const float *K, int64_t rs, int64_t cs, c32 *Kout, const c32 *__restrict__ tw) {
    using Ctx = ClusterCtx<G, false, false>;
    constexpr int E = G::E, M1 = G::M1, M2 = G::M2;
    constexpr int Hh = M1 / 2, Ww = M2;
    constexpr int TWM = Ctx::TWM;
    extern __shared__ float smem[];
    Ctx cx(smem);
    const int64_t o = (int64_t)blockIdx.x / G::C;
    const float *Kp = K + o * cs;
    c32 v[E];
    const int ix = (2 * cx.n2 + Ww) & (2 * Ww - 1);    // cyclic column 2 n2 -> offset-grid column
#pragma unroll
    for (int q = 0; q < E; ++q) {
        const int iy = (cx.t1 + q * Ctx::T1P + Hh) & (M1 - 1);
        const float *rowp = Kp + iy * rs;
        v[q] = mk(rowp[ix], rowp[ix + 1]);
    }
    cx.template forward<false>(v, tw);                  // contains a cluster barrier after all reads
    cx.publish(v);
    const int ky = cx.k1;
    const int kym = (M1 - ky) & (M1 - 1);
    const c32 wb = ldg_c(tw + cx.t2 * (TWM / (2 * M2)));
    c32 *Ko = Kout + o * (M1 * (M2 + 1));
    const int z0 = opaque_zero();
#pragma unroll
    for (int q = 0; q < E; ++q) {
        const int kx = cx.t2 + q * G::T2;
        const c32 Zm = cx.mirror_bin((M2 - kx) & (M2 - 1));
        const c32 Zk = v[q];
        const c32 Ek = mk(0.5f * (Zk.x + Zm.x), 0.5f * (Zk.y - Zm.y));
        const c32 Ok = mk(0.5f * (Zk.y + Zm.y), -0.5f * (Zk.x - Zm.x));
        const c32 wO = mul(mul(wb, w2e<E>(q, z0)), Ok);
        Ko[(int64_t)kx * M1 + ky] = add(Ek, wO);
        if (kx == 0) Ko[(int64_t)M2 * M1 + kym] = conj(sub(Ek, wO));   // bin (-ky, M2)
    }
}

}  // namespace hyena
