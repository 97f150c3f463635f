// 2D (HyenaND-style) forward as staged kernels: the plane's transform travels
// through a device workspace between a column kernel (over y) and a row
// kernel (over the packed x axis), as in kernels_1d_staged.cuh for long rows.
//
// Packing as in kernels_2d.cuh: z[y][x'] = v[y][2x'] + i v[y][2x'+1] on the
// zero-padded [M1 = 2H][M2 = W] complex array; only y < H and x' < W/2 carry
// data. Per chunk of planes and order n:
//   column kernel: (n > 0) inverse column FFTs (length M1; only y < H is
//                  kept), gate x^n, then the forward column FFTs of the next
//                  order (half-zero input) into the workspace [ky][x' < W/2]
//                  (or the output y);
//   row kernel:    row FFTs (length M2, half-zero input), the spectral step
//                  (real-packing identity along x with the 2D mirror bin),
//                  inverse row FFTs of which only x' < W/2 is kept.
// The row kernel carries two planes in lockstep (c32x2); a CTA holds rows ky
// and M1 - ky, so every mirror bin is in the CTA and one thread computes a bin
// and its mirror.
#pragma once
#include "kernels_1d_staged.cuh"
#include "kernels_2d.cuh"

namespace hyena {

template <int H_>
struct Staged2dGeom {
    static constexpr int Hh = H_, Ww = H_;
    static constexpr int M1 = 2 * H_, M2 = H_, XW = H_ / 2;   // transform [M1][M2]; x' < XW carry data
    static constexpr int E = 16;
    static constexpr int NCOL = 8;                  // column kernel: 8 data columns per CTA (one plane)
    static constexpr int T1 = M1 / E;               // threads per column FFT
    static constexpr int CT = NCOL * T1;
    static constexpr int CGROUPS = XW / NCOL;
    static constexpr int NROW = 8, HROW = 4;        // row kernel: 8 rows (4 + mirrors), two planes
    static constexpr int T2 = M2 / E;
    static constexpr int RT = NROW * T2;
    static constexpr int RGROUPS = M1 / NROW;
    static constexpr int TWS = 1024;
    static constexpr size_t CSMEM = (size_t)NCOL * M1 * 8;
    static constexpr size_t RSMEM = (size_t)NROW * M2 * 16;
    static constexpr int64_t PLANE = (int64_t)M1 * XW;   // workspace complex64 per plane
    static_assert(XW % NCOL == 0 && M1 % NROW == 0, "groups must tile the plane");
    static_assert(TWS % M1 == 0 && TWS % M2 == 0, "sub-transform twiddles");
    static_assert(XW % RT == 0 || RT % XW == 0, "row copies");
};

struct Staged2dArgs {
    Fwd2dArgs f;      // operator arguments
    float2 *ws;       // workspace: chunk planes x [M1][XW] complex
    int64_t o0;       // visit index of the chunk's first plane (c-major, b-minor)
    int n;            // order
};

__device__ __forceinline__ int64_t visit_plane(const Fwd2dArgs &f, int64_t o, int64_t &c) {
    c = o / f.B;
    return (o - c * f.B) * f.C + c;
}

// MODE 0: load v, forward columns; 1: inverse columns, gate x^n, forward
// columns; 2: inverse columns, gate x^n, store y. GATED: the gate sandwich
// (z^0 = q SiLU(k) at the load, SiLU of every gate where it multiplies).
template <typename G, typename IO, int MODE, bool GATED>
__global__ void __launch_bounds__(G::CT, 3) hyena_staged2d_cols(const Staged2dArgs a) {
    constexpr int E = G::E, M1 = G::M1, XW = G::XW, T1 = G::T1, Hh = G::Hh, Ww = G::Ww;
    extern __shared__ float smem[];
    const int64_t lp = blockIdx.x / G::CGROUPS;      // plane within the chunk
    const int cgp = blockIdx.x % G::CGROUPS;
    const int j = threadIdx.x % G::NCOL, t1 = threadIdx.x / G::NCOL;
    const int xc = cgp * G::NCOL + j;                // data column x' < XW
    int64_t c;
    const int64_t plane = visit_plane(a.f, a.o0 + lp, c);
    // debug build: the plane exists (uniform over the CTA, so it may leave as a whole)
    if (!(check_index(a.f.err, plane, a.f.planes) && check_index(a.f.err, c, a.f.C))) return;
    float2 *wp = a.ws + lp * G::PLANE;
    const c32 *tws = a.f.tw + 2 * G::M2;             // W_1024 after the W_{2W} table
    const int64_t plane_elems = (int64_t)Hh * Ww;
    // register q holds row y = t1 + q T1 of column x'; rows y < H (q < E/2) carry data
    auto pos_of = [&](int q) -> int64_t { return (int64_t)(t1 + q * T1) * Ww + 2 * xc; };

    // The columns read their plane in sectors a row (2W bytes and more) apart,
    // which DRAM serves poorly. The CGROUPS CTAs of a plane cover all of it, so
    // each first brings 1/CGROUPS of the plane's input (v and, for the gate
    // sandwich, k; or this order's gate) into L2 with one bulk prefetch each.
    if (threadIdx.x < (MODE == 0 && GATED ? 2 : 1)) {
        const IO *in = MODE != 0 ? reinterpret_cast<const IO *>(a.f.gates[a.n])
                                 : reinterpret_cast<const IO *>(threadIdx.x ? a.f.k : a.f.v);
        const uintptr_t ps = reinterpret_cast<uintptr_t>(in + plane * plane_elems);
        const int64_t plane_bytes = plane_elems * (int64_t)sizeof(IO);
        const int64_t piece = ((plane_bytes + G::CGROUPS - 1) / G::CGROUPS + 15) & ~(int64_t)15;
        const int64_t off = (int64_t)cgp * piece;
        int64_t len = plane_bytes - off < piece ? plane_bytes - off : piece;
        len &= ~(int64_t)15;
        if ((ps & 15) == 0 && len > 0)
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(ps + off), "r"((uint32_t)len)
                         : "memory");
    }
    c32 v[E];
    if constexpr (MODE == 0) {
        const IO *vp = reinterpret_cast<const IO *>(a.f.v) + plane * plane_elems;
        const IO *kp = reinterpret_cast<const IO *>(a.f.k) + plane * plane_elems;
#pragma unroll
        for (int q = 0; q < E / 2; ++q) {
            v[q] = load_pair<IO, true>(vp, pos_of(q), plane_elems);
            if constexpr (GATED) {
                const c32 kq = silu(load_pair<IO, true>(kp, pos_of(q), plane_elems));
                v[q] = mk(v[q].x * kq.x, v[q].y * kq.y);
            }
        }
    } else {
        using P = typename io<IO>::pair_t;
        const IO *gp = reinterpret_cast<const IO *>(a.f.gates[a.n]) + plane * plane_elems;
        P g[E / 2];
#pragma unroll
        for (int q = 0; q < E / 2; ++q) g[q] = load_pair_raw<IO, true>(gp, pos_of(q), plane_elems);
        const uint64_t pol = MODE == 2 ? l2_stream() : l2_keep();
#pragma unroll
        for (int q = 0; q < E; ++q) {
            const float2 f = ld_pol(wp + (t1 + q * T1) * XW + xc, pol);   // ky = t1 + q T1
            v[q] = mk(f.x, f.y);
        }
        fft_cta<M1, E, +1, false, G::TWS, G::NCOL>(v, smem, nullptr, t1, tws, j);
#pragma unroll
        for (int q = 0; q < E / 2; ++q) {
            c32 gq = io<IO>::unpack(g[q]);
            if constexpr (GATED) gq = silu(gq);
            v[q] = mk(gq.x * v[q].x, gq.y * v[q].y);
        }
        if constexpr (MODE == 2) {
            IO *yp = reinterpret_cast<IO *>(a.f.y) + plane * plane_elems;
#pragma unroll
            for (int q = 0; q < E / 2; ++q) store_pair<IO, true>(yp, pos_of(q), plane_elems, v[q]);
            return;
        }
    }
    if constexpr (MODE != 2) {
#pragma unroll
        for (int q = E / 2; q < E; ++q) v[q] = mk(0.f, 0.f);
        fft_cta<M1, E, -1, true, G::TWS, G::NCOL>(v, smem, nullptr, t1, tws, j);
        const uint64_t keep = l2_keep();
#pragma unroll
        for (int q = 0; q < E; ++q) st_pol(wp + (t1 + q * T1) * XW + xc, make_float2(v[q].x, v[q].y), keep);
    }
}

template <typename G>
__global__ void __launch_bounds__(G::RT, 3) hyena_staged2d_rows_x2(const Staged2dArgs a, int64_t np) {
    constexpr int E = G::E, M1 = G::M1, M2 = G::M2, XW = G::XW, T2 = G::T2, RT = G::RT;
    constexpr int NROW = G::NROW, HROW = G::HROW;
    extern __shared__ float smem[];
    float4 *rowb = reinterpret_cast<float4 *>(smem);
    const int64_t lp = blockIdx.x / G::RGROUPS;      // plane pair within the chunk
    const int g = blockIdx.x % G::RGROUPS;
    const int r = threadIdx.x % NROW, t2 = threadIdx.x / NROW;
    const int ky = row_of_slot<G>(g, r);
    const int rm = (ky == 0 || ky == M1 / 2) ? r : (r < HROW ? r + HROW : r - HROW);   // slot of row M1 - ky
    const int kym = (M1 - ky) & (M1 - 1);
    const bool has1 = 2 * lp + 1 < np;
    int64_t c0, c1;
    (void)visit_plane(a.f, a.o0 + 2 * lp, c0);
    (void)visit_plane(a.f, a.o0 + 2 * lp + (has1 ? 1 : 0), c1);
    // debug build: the planes and their kernel spectra exist (uniform over the CTA)
    if (!(check_index(a.f.err, 2 * lp + (has1 ? 1 : 0), np) && check_index(a.f.err, c0, a.f.C) &&
          check_index(a.f.err, c1, a.f.C) && check_index(a.f.err, a.n, a.f.order)))
        return;
    float2 *w0 = a.ws + (2 * lp) * G::PLANE;
    float2 *w1 = a.ws + (2 * lp + (has1 ? 1 : 0)) * G::PLANE;
    const c32 *tws = a.f.tw + 2 * M2;
    // the debug build checks the slot index of every shared access
    auto ld = [&](int ad) -> c32x2 {
        if (!check_index(a.f.err, ad, NROW * M2)) return c32x2{f2(0.f, 0.f), f2(0.f, 0.f)};
        const float4 f = rowb[ad];
        return c32x2{f2(f.x, f.y), f2(f.z, f.w)};
    };
    auto st = [&](int ad, c32x2 x) {
        if (check_index(a.f.err, ad, NROW * M2)) rowb[ad] = make_float4(x.re.x, x.re.y, x.im.x, x.im.y);
    };

    // The kernel-spectrum bins of a row group lie 2H bins apart, which DRAM
    // serves poorly. The RGROUPS CTAs of a plane pair cover both planes'
    // spectra, so each first brings 1/RGROUPS of them (a contiguous run of
    // 16-byte blocks inside the channel's spectrum) into L2, one bulk prefetch
    // per channel.
    if (threadIdx.x < 2 && (threadIdx.x == 0 || c1 != c0)) {
        const uintptr_t ks = reinterpret_cast<uintptr_t>(
            a.f.K + ((int64_t)a.n * a.f.C + (threadIdx.x ? c1 : c0)) * (int64_t)(M1 * (M2 + 1)));
        const uintptr_t ke = ks + (uintptr_t)(M1 * (M2 + 1)) * 8;
        const uintptr_t piece = (((uintptr_t)(M1 * (M2 + 1)) * 8 + G::RGROUPS - 1) / G::RGROUPS + 15) & ~(uintptr_t)15;
        const uintptr_t b = (ks + (uintptr_t)g * piece + 15) & ~(uintptr_t)15;
        uintptr_t e = ks + (uintptr_t)(g + 1) * piece;
        e = (e < ke ? e : ke) & ~(uintptr_t)15;
        if (e > b)
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(b), "r"((uint32_t)(e - b)) : "memory");
    }
    // the group's rows of both planes (data columns x' < XW), coalesced
    const uint64_t keep = l2_keep();
#pragma unroll
    for (int sl = 0; sl < NROW; ++sl) {
        const int64_t base = (int64_t)row_of_slot<G>(g, sl) * XW;
#pragma unroll
        for (int x = threadIdx.x; x < XW; x += RT) {
            const float2 f0 = ld_pol(w0 + base + x, keep), f1 = ld_pol(w1 + base + x, keep);
            rowb[maddr<M2>(x, sl)] = make_float4(f0.x, f1.x, f0.y, f1.y);
        }
    }
    __syncthreads();
    c32x2 v[E];
#pragma unroll
    for (int q = 0; q < E; ++q) v[q] = q < E / 2 ? ld(maddr<M2>(t2 + q * T2, r)) : c32x2{f2(0.f, 0.f), f2(0.f, 0.f)};
    __syncthreads();
    fft_cta<M2, E, -1, true, G::TWS, NROW>(v, smem, nullptr, t2, tws, r);
#pragma unroll
    for (int q = 0; q < E; ++q) st(maddr<M2>(t2 + q * T2, r), v[q]);
    __syncthreads();

    // Spectral step on both planes, bins in pairs ((ky, kx), (-ky, -kx)): the
    // mirror of register q is register E-1-q of thread (rm, T2-t2) (register
    // E-q when t2 = 0), so each thread takes q < E/2 and returns the mirror
    // result; threads with t2 = 0 also take q = E/2 (kx = M2/2). The unpacking
    // is written without its factors 1/2, folded into the gain.
    const float dsk0 = a.f.dskip ? __ldg(a.f.dskip + a.n * a.f.C + c0) : 0.f;
    const float dsk1 = a.f.dskip ? __ldg(a.f.dskip + a.n * a.f.C + c1) : 0.f;
    const c32 *K0 = a.f.K + ((int64_t)a.n * a.f.C + c0) * (M1 * (M2 + 1));
    const c32 *K1 = a.f.K + ((int64_t)a.n * a.f.C + c1) * (M1 * (M2 + 1));
    const c32 wb = ldg_c(a.f.tw + t2);               // W_{2 M2}^{t2}
    constexpr float s = 0.25f / (float)(M1 * M2);
    const uint64_t once = l2_stream();
    const int z0 = opaque_zero();
    auto bin_pair = [&](int q, c32x2 Zk, c32x2 &Ye, c32x2 &Yo) __attribute__((always_inline)) {
        const int kx = t2 + q * T2;
        const int kxm = (M2 - kx) & (M2 - 1);
        const c32x2 Zm = ld(maddr<M2>(kxm, rm));
        const c32x2 E2{f2add(Zk.re, Zm.re), f2sub(Zk.im, Zm.im)};   // Zk + conj Zm
        const c32x2 O2{f2add(Zk.im, Zm.im), f2sub(Zm.re, Zk.re)};   // (Zk - conj Zm) / i
        const c32 w = mul(wb, w2e<E>(q, z0));                        // W_{2 M2}^{kx}
        const c32x2 wO = mul(O2, w);
        const c32x2 Xk = add(E2, wO);                                 // 2 X(ky, kx)
        const c32x2 Xm{f2sub(E2.re, wO.re), f2sub(wO.im, E2.im)};    // 2 X(-ky, M2 - kx)
        const int64_t ak = (int64_t)kx * M1 + ky, am = (int64_t)(M2 - kx) * M1 + kym;   // column-bin-major
        const c32 hk0 = ldc_pol(K0 + ak, once), hk1 = ldc_pol(K1 + ak, once);
        const c32 hm0 = ldc_pol(K0 + am, once), hm1 = ldc_pol(K1 + am, once);
        const c32x2 Hk{f2(s * (hk0.x + dsk0), s * (hk1.x + dsk1)), f2(s * hk0.y, s * hk1.y)};
        const c32x2 Hm{f2(s * (hm0.x + dsk0), s * (hm1.x + dsk1)), f2(s * hm0.y, s * hm1.y)};
        const c32x2 Yk = mul(Xk, Hk), Ym = mul(Xm, Hm);
        Ye = c32x2{f2add(Yk.re, Ym.re), f2sub(Yk.im, Ym.im)};       // Yk + conj Ym
        const c32x2 Yd{f2sub(Yk.re, Ym.re), f2add(Yk.im, Ym.im)};   // Yk - conj Ym
        Yo = mul(Yd, conj(w));
    };
    const bool self_half = t2 == 0;
    c32x2 vh = v[E / 2];
    if (self_half) {
        c32x2 Ye, Yo;
        bin_pair(E / 2, v[E / 2], Ye, Yo);
        vh = c32x2{f2sub(Ye.re, Yo.im), f2add(Ye.im, Yo.re)};
    }
#pragma unroll
    for (int q = 0; q < E / 2; ++q) {
        c32x2 Ye, Yo;
        bin_pair(q, v[q], Ye, Yo);
        v[q] = c32x2{f2sub(Ye.re, Yo.im), f2add(Ye.im, Yo.re)};             // Ye + i Yo       (bin (ky, kx))
        v[E / 2 + q] = c32x2{f2add(Ye.re, Yo.im), f2sub(Yo.re, Ye.im)};    // conj(Ye - i Yo) (bin (-ky, -kx))
        if ((q & 3) == 3) asm volatile("" ::: "memory");  // bound load hoisting (register pressure)
    }
    __syncthreads();                                      // every mirror read done
#pragma unroll
    for (int q = 0; q < E / 2; ++q) st(maddr<M2>((M2 - (t2 + q * T2)) & (M2 - 1), rm), v[E / 2 + q]);
    __syncthreads();
#pragma unroll
    for (int q = E / 2; q < E; ++q) v[q] = ld(maddr<M2>(t2 + q * T2, r));
    if (self_half) v[E / 2] = vh;
    __syncthreads();                                      // buffer reads done before the inverse rewrites it

    fft_cta<M2, E, +1, false, G::TWS, NROW>(v, smem, nullptr, t2, tws, r);
    // keep x' < XW (registers q < E/2), out through the buffer
#pragma unroll
    for (int q = 0; q < E / 2; ++q) st(maddr<M2>(t2 + q * T2, r), v[q]);
    __syncthreads();
#pragma unroll
    for (int sl = 0; sl < NROW; ++sl) {
        const int64_t base = (int64_t)row_of_slot<G>(g, sl) * XW;
#pragma unroll
        for (int x = threadIdx.x; x < XW; x += RT) {
            const float4 f = rowb[maddr<M2>(x, sl)];
            st_pol(w0 + base + x, make_float2(f.x, f.z), keep);
            if (has1) st_pol(w1 + base + x, make_float2(f.y, f.w), keep);
        }
    }
}

// ---------------------------------------------------------------------------
// 2D kernel spectra through the same two stages. The kernel on the offset grid
// is placed cyclically (offset o at index o mod 2H, o mod 2W), packed along x
// and transformed; every column and row carries data. The plan owns the
// scratch ([M1][M2] complex64 per kernel), so the spectrum may be computed in
// place: a chunk's column kernel reads all of its kernels before its row
// kernel writes their spectra.

struct Spec2dArgs {
    const float *K;    // kernel (n, c) at K + o * cs; row iy at + iy * rs, 2W floats (ox = ix - W)
    int64_t rs, cs;
    c32 *Kout;         // [W + 1][2H] complex per kernel, bin (ky, kx) at kx * 2H + ky
    const c32 *tw;     // W_{2W}, then W_1024
    float2 *ws;        // chunk kernels x [M1][M2]
    int64_t o0;        // first kernel of the chunk
    int64_t nk;        // kernels in the chunk
};

template <typename G>
__global__ void __launch_bounds__(G::CT, 3) hyena_staged2d_spec_cols(const Spec2dArgs a) {
    constexpr int E = G::E, M1 = G::M1, M2 = G::M2, T1 = G::T1, Hh = G::Hh, Ww = G::Ww;
    constexpr int CG = M2 / G::NCOL;                   // column groups: every column carries data
    extern __shared__ float smem[];
    const int64_t lk = blockIdx.x / CG;
    const int cgp = blockIdx.x % CG;
    const int j = threadIdx.x % G::NCOL, t1 = threadIdx.x / G::NCOL;
    const int xc = cgp * G::NCOL + j;
    const float *Kp = a.K + (a.o0 + lk) * a.cs;
    float2 *wp = a.ws + lk * (int64_t)M1 * M2;
    const int ix = (2 * xc + Ww) & (2 * Ww - 1);      // cyclic column 2 x' -> offset-grid column
    c32 v[E];
#pragma unroll
    for (int q = 0; q < E; ++q) {
        const int iy = (t1 + q * T1 + Hh) & (M1 - 1);
        const float *rowp = Kp + iy * a.rs;
        v[q] = mk(rowp[ix], rowp[ix + 1]);
    }
    fft_cta<M1, E, -1, false, G::TWS, G::NCOL>(v, smem, nullptr, t1, a.tw + 2 * M2, j);
    const uint64_t keep = l2_keep();
#pragma unroll
    for (int q = 0; q < E; ++q) st_pol(wp + (t1 + q * T1) * M2 + xc, make_float2(v[q].x, v[q].y), keep);
}

template <typename G>
__global__ void __launch_bounds__(G::RT, 3) hyena_staged2d_spec_rows_x2(const Spec2dArgs a) {
    constexpr int E = G::E, M1 = G::M1, M2 = G::M2, T2 = G::T2, RT = G::RT;
    constexpr int NROW = G::NROW, HROW = G::HROW;
    extern __shared__ float smem[];
    float4 *rowb = reinterpret_cast<float4 *>(smem);
    const int64_t lp = blockIdx.x / G::RGROUPS;      // kernel pair within the chunk
    const int g = blockIdx.x % G::RGROUPS;
    const int r = threadIdx.x % NROW, t2 = threadIdx.x / NROW;
    const int ky = row_of_slot<G>(g, r);
    const int rm = (ky == 0 || ky == M1 / 2) ? r : (r < HROW ? r + HROW : r - HROW);
    const int kym = (M1 - ky) & (M1 - 1);
    const bool has1 = 2 * lp + 1 < a.nk;
    const float2 *w0 = a.ws + (2 * lp) * (int64_t)M1 * M2;
    const float2 *w1 = a.ws + (2 * lp + (has1 ? 1 : 0)) * (int64_t)M1 * M2;
    auto ld = [&](int ad) -> c32x2 {
        const float4 f = rowb[ad];
        return c32x2{f2(f.x, f.y), f2(f.z, f.w)};
    };
    const uint64_t stream = l2_stream();              // the scratch is read once
#pragma unroll
    for (int sl = 0; sl < NROW; ++sl) {
        const int64_t base = (int64_t)row_of_slot<G>(g, sl) * M2;
#pragma unroll
        for (int x = threadIdx.x; x < M2; x += RT) {
            const float2 f0 = ld_pol(w0 + base + x, stream), f1 = ld_pol(w1 + base + x, stream);
            rowb[maddr<M2>(x, sl)] = make_float4(f0.x, f1.x, f0.y, f1.y);
        }
    }
    __syncthreads();
    c32x2 v[E];
#pragma unroll
    for (int q = 0; q < E; ++q) v[q] = ld(maddr<M2>(t2 + q * T2, r));
    __syncthreads();
    fft_cta<M2, E, -1, false, G::TWS, NROW>(v, smem, nullptr, t2, a.tw + 2 * M2, r);
#pragma unroll
    for (int q = 0; q < E; ++q) rowb[maddr<M2>(t2 + q * T2, r)] = make_float4(v[q].re.x, v[q].re.y, v[q].im.x, v[q].im.y);
    __syncthreads();
    // unpack along x: X(ky, kx) = E + W_{2 M2}^{kx} O with the mirror bin (-ky, -kx); bin
    // (-ky, M2) (the Nyquist column) is conj(E - W O) of kx = 0
    const c32 wb = ldg_c(a.tw + t2);
    c32 *K0 = a.Kout + (a.o0 + 2 * lp) * (int64_t)M1 * (M2 + 1);
    c32 *K1 = a.Kout + (a.o0 + 2 * lp + (has1 ? 1 : 0)) * (int64_t)M1 * (M2 + 1);
    const int z0 = opaque_zero();
#pragma unroll
    for (int q = 0; q < E; ++q) {
        const int kx = t2 + q * T2;
        const c32x2 Zk = v[q];
        const c32x2 Zm = ld(maddr<M2>((M2 - kx) & (M2 - 1), rm));
        const c32x2 E2{f2add(Zk.re, Zm.re), f2sub(Zk.im, Zm.im)};   // 2E
        const c32x2 O2{f2add(Zk.im, Zm.im), f2sub(Zm.re, Zk.re)};   // 2O
        const c32x2 wO = mul(O2, mul(wb, w2e<E>(q, z0)));
        const c32x2 X{f2mul(f2add(E2.re, wO.re), f2(0.5f, 0.5f)), f2mul(f2add(E2.im, wO.im), f2(0.5f, 0.5f))};
        const int64_t ak = (int64_t)kx * M1 + ky;
        K0[ak] = mk(X.re.x, X.im.x);
        if (has1) K1[ak] = mk(X.re.y, X.im.y);
        if (kx == 0) {
            const c32x2 N{f2mul(f2sub(E2.re, wO.re), f2(0.5f, 0.5f)), f2mul(f2sub(wO.im, E2.im), f2(0.5f, 0.5f))};
            const int64_t an = (int64_t)M2 * M1 + kym;
            K0[an] = mk(N.re.x, N.im.x);
            if (has1) K1[an] = mk(N.re.y, N.im.y);
        }
    }
}

}  // namespace hyena
