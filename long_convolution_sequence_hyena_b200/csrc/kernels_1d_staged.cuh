// 1D kernels for long rows as a staged four-step FFT: a column kernel and a
// row kernel per order exchange the row's transform through a device
// workspace instead of distributed shared memory. The workspace holds a
// chunk of rows small enough to stay in L2 between the launches; kernel
// boundaries are the only synchronisation, and every CTA is independent, so
// all SMs take CTAs (no cluster has to fit inside one GPC).
//
// Four-step split as in kernels_1d_cluster.cuh: MC = M1 * M2, element
// n = M2 n1 + n2; column FFTs of length M1 over n1, twiddle W_MC^{n2 k1},
// row FFTs of length M2 over n2, giving Z[k1 + M1 k2]. The workspace row is
// [k1][n2] (row-major in k1), complex64.
//
// Per chunk and order n:
//   column kernel: (n > 0) inverse column FFTs, gate x^n, then the forward
//                  column FFTs and twiddle of the next order (or the output);
//   row kernel:    row FFTs, spectral step of order n (bins k and MC-k from
//                  one thread; a row group holds rows k1 and M1-k1 together),
//                  inverse row FFTs and the conjugate twiddle.
#pragma once
#include "kernels_1d_cluster.cuh"

namespace hyena {

// ROWS: rows per CTA, 1 (complex values) or 2 (two rows in lockstep as c32x2;
// 16-byte shared elements).
template <int MC_, int M1_, int NCOL_, int NROW_, int ROWS_ = 1>
struct StagedGeom {
    static constexpr int MC = MC_, M1 = M1_, M2 = MC_ / M1_, E = 16, ROWS = ROWS_;
    static constexpr int NCOL = NCOL_;               // columns per column-kernel CTA
    static constexpr int NROW = NROW_;               // rows per row-kernel CTA (mirror pairs)
    static constexpr int HROW = NROW / 2;
    static constexpr int T1 = M1 / E, T2 = M2 / E;   // threads per column / row FFT
    static constexpr int CT = NCOL * T1;             // column-kernel threads
    static constexpr int RT = NROW * T2;             // row-kernel threads
    static constexpr int CGROUPS = M2 / NCOL;        // column CTAs per row
    static constexpr int RGROUPS = M1 / NROW;        // row CTAs per row
    static constexpr int TWS = 1024;                 // sub-transform twiddle table W_1024
    static constexpr size_t CSMEM = (size_t)NCOL * M1 * 8 * ROWS;
    static constexpr size_t RSMEM = (size_t)NROW * M2 * 8 * ROWS;
    // resident CTAs per SM the register budget is sized for (128-thread CTAs: 4,
    // at 128 registers, a few bytes of spills in some column instances, which
    // measured faster than 3 CTAs at up to 168 registers; larger CTAs: 128
    // registers per thread)
    static constexpr int CMINB = CT <= 128 ? 4 : 512 / CT;
    static constexpr int RMINB = RT <= 128 ? 4 : 512 / RT;
    static_assert(M2 % NCOL == 0 && M1 % NROW == 0 && NROW % 2 == 0, "groups must tile the row");
    static_assert((ROWS == 1 && NCOL >= 16 && NROW >= 16) || (ROWS == 2 && NCOL >= 8 && NROW >= 8),
                  "warps must span enough sequences for conflict-free exchanges");
    static_assert(TWS % M1 == 0 && TWS % M2 == 0, "sub-transform twiddles");
    static_assert(CT <= 1024 && RT <= 1024, "too many threads");
    static_assert(ROWS == 2 || RT == M2, "the row kernel copies one element of every row per thread");
    static_assert(M2 % RT == 0, "row copies tile the row");
};

struct StagedArgs {
    Fwd1dArgs f;      // operator arguments
    float2 *ws;       // workspace: chunk rows x MC complex, each [k1][n2]
    int64_t o0;       // visit index of the chunk's first row (visit order d-major, b-minor)
    int n;            // order: gate x^n (column kernel), spectrum H^n (row kernel)
};

// L2 eviction priorities. The chunk's workspace is written and read again by
// the next launch, so it is kept (evict_last); the spectrum rows are read once
// per launch and must not push it out (evict_first).
__device__ __forceinline__ uint64_t l2_keep() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_stream() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ float2 ld_pol(const float2 *ptr, uint64_t pol) {
    float2 v;
    asm volatile("ld.global.L2::cache_hint.v2.f32 {%0, %1}, [%2], %3;" : "=f"(v.x), "=f"(v.y) : "l"(ptr), "l"(pol));
    return v;
}
__device__ __forceinline__ c32 ldc_pol(const c32 *ptr, uint64_t pol) {   // read-only data
    float2 v;
    asm volatile("ld.global.nc.L2::cache_hint.v2.f32 {%0, %1}, [%2], %3;" : "=f"(v.x), "=f"(v.y) : "l"(ptr), "l"(pol));
    return mk(v.x, v.y);
}
__device__ __forceinline__ void st_pol(float2 *ptr, float2 v, uint64_t pol) {
    asm volatile("st.global.L2::cache_hint.v2.f32 [%0], {%1, %2}, %3;" ::"l"(ptr), "f"(v.x), "f"(v.y), "l"(pol)
                 : "memory");
}

// Flat row of visit index o (d-major, b-minor: the B rows of one channel run together).
__device__ __forceinline__ int64_t visit_row(const Fwd1dArgs &f, int64_t o, int64_t &d) {
    d = o / f.B;
    return (o - d * f.B) * f.D + d;
}

// ---------------------------------------------------------------------------
// The column and row kernels, each carrying two rows of the chunk in lockstep
// (c32x2: lane a = visit index o, lane b = o + 1). Butterflies, twiddle
// products and exchanges are one instruction for both rows; each lane reads
// its own gate, spectrum row and feedthrough. An odd row count leaves the last
// pair's lane b empty.
//
// MODE 0: first (load v, forward columns); 1: between orders (inverse columns,
// gate x^n, forward columns); 2: last (inverse columns, gate x^n, store y).

template <typename G, typename IO, bool EVEN, int MODE>
__global__ void __launch_bounds__(G::CT, G::CMINB) hyena_staged_cols_x2(const StagedArgs a, int64_t nr) {
    static_assert(G::ROWS == 2, "lockstep geometry");
    constexpr int E = G::E, M1 = G::M1, M2 = G::M2, T1 = G::T1, MC = G::MC, M = 2 * MC;
    extern __shared__ float smem[];
    const int64_t lp = blockIdx.x / G::CGROUPS;      // row pair within the chunk
    const int cgp = blockIdx.x % G::CGROUPS;
    const int j = threadIdx.x % G::NCOL, t1 = threadIdx.x / G::NCOL;
    const int n2 = cgp * G::NCOL + j;
    const bool has1 = 2 * lp + 1 < nr;
    int64_t d0, d1;
    const int64_t row0 = visit_row(a.f, a.o0 + 2 * lp, d0);
    const int64_t row1 = visit_row(a.f, a.o0 + 2 * lp + (has1 ? 1 : 0), d1);
    // debug build: the CTA's rows exist (uniform over the CTA, so it may leave as a whole)
    if (!(check_index(a.f.err, row0, a.f.rows) && check_index(a.f.err, row1, a.f.rows) &&
          check_index(a.f.err, 2 * lp + (has1 ? 1 : 0), nr)))
        return;
    const int64_t L = a.f.L;
    float2 *w0 = a.ws + (2 * lp) * MC;
    float2 *w1 = a.ws + (2 * lp + (has1 ? 1 : 0)) * MC;
    const c32 *tws = a.f.tw + M;                     // W_1024
    auto pos_of = [&](int q) -> int64_t { return 2 * ((int64_t)M2 * (t1 + q * T1) + n2); };

    // The columns read their input (v, or this order's gate) in sectors 1 KB and
    // more apart, which DRAM serves poorly. The chunk's rows are contiguous, so
    // each CTA first brings its share of its two rows (1/CGROUPS of each) into
    // L2 in one bulk prefetch per row; the column loads then meet L2.
    if (a.f.es == 1 && threadIdx.x < 2 && (threadIdx.x == 0 || has1)) {
        const IO *in = MODE == 0 ? reinterpret_cast<const IO *>(a.f.v)
                                 : reinterpret_cast<const IO *>(a.f.gates[a.n]);
        const uintptr_t row_start = reinterpret_cast<uintptr_t>(in + (threadIdx.x ? row1 : row0) * L);
        const int64_t row_bytes = L * (int64_t)sizeof(IO);
        const int64_t piece = ((row_bytes + G::CGROUPS - 1) / G::CGROUPS + 15) & ~(int64_t)15;
        const int64_t off = (int64_t)cgp * piece;
        int64_t len = row_bytes - off < piece ? row_bytes - off : piece;
        len &= ~(int64_t)15;   // whole 16-byte blocks inside the row
        if ((row_start & 15) == 0 && len > 0)
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(row_start + off), "r"((uint32_t)len)
                         : "memory");
    }
    c32x2 v[E];
    if constexpr (MODE == 0) {
        const IO *r0 = reinterpret_cast<const IO *>(a.f.v) + act_row_off(a.f, row0);
        const IO *r1 = reinterpret_cast<const IO *>(a.f.v) + act_row_off(a.f, row1);
#pragma unroll
        for (int q = 0; q < E / 2; ++q) {
            const c32 x0 = load_pair_s<IO, EVEN>(r0, pos_of(q), L, a.f.es);
            const c32 x1 = has1 ? load_pair_s<IO, EVEN>(r1, pos_of(q), L, a.f.es) : mk(0.f, 0.f);
            v[q] = c32x2{f2(x0.x, x1.x), f2(x0.y, x1.y)};
        }
    } else {
        using P = typename io<IO>::pair_t;
        const IO *g0 = reinterpret_cast<const IO *>(a.f.gates[a.n]) + act_row_off(a.f, row0);
        const IO *g1 = reinterpret_cast<const IO *>(a.f.gates[a.n]) + act_row_off(a.f, row1);
        P ga[E / 2], gb[E / 2];   // this order's gates, loaded while the inverse transform runs
#pragma unroll
        for (int q = 0; q < E / 2; ++q) {
            ga[q] = load_pair_raw_s<IO, EVEN>(g0, pos_of(q), L, a.f.es);
            gb[q] = load_pair_raw_s<IO, EVEN>(g1, pos_of(q), L, a.f.es);
        }
        // the last read of the chunk's workspace releases it (evict_first)
        const uint64_t pol = MODE == 2 ? l2_stream() : l2_keep();
#pragma unroll
        for (int q = 0; q < E; ++q) {
            const int ad = (t1 + q * T1) * M2 + n2;     // k1 = t1 + q T1
            if (!check_index(a.f.err, ad, MC)) {
                v[q] = c32x2{f2(0.f, 0.f), f2(0.f, 0.f)};
                continue;
            }
            const float2 f0 = ld_pol(w0 + ad, pol), f1 = ld_pol(w1 + ad, pol);
            v[q] = c32x2{f2(f0.x, f1.x), f2(f0.y, f1.y)};
        }
        fft_cta<M1, E, +1, false, G::TWS, G::NCOL>(v, smem, nullptr, t1, tws, j);
#pragma unroll
        for (int q = 0; q < E / 2; ++q) {
            const int64_t pos = pos_of(q);
            const c32 ca = io<IO>::unpack(ga[q]), cb = io<IO>::unpack(gb[q]);
            v[q] = c32x2{pos < L ? f2mul(v[q].re, f2(ca.x, cb.x)) : f2(0.f, 0.f),
                         pos + 1 < L ? f2mul(v[q].im, f2(ca.y, cb.y)) : f2(0.f, 0.f)};
        }
        if constexpr (MODE == 2) {
            IO *y0 = reinterpret_cast<IO *>(a.f.y) + act_row_off(a.f, row0);
            IO *y1 = reinterpret_cast<IO *>(a.f.y) + act_row_off(a.f, row1);
#pragma unroll
            for (int q = 0; q < E / 2; ++q) {
                store_pair_s<IO, EVEN>(y0, pos_of(q), L, a.f.es, mk(v[q].re.x, v[q].im.x));
                if (has1) store_pair_s<IO, EVEN>(y1, pos_of(q), L, a.f.es, mk(v[q].re.y, v[q].im.y));
            }
            return;
        }
    }
    if constexpr (MODE != 2) {
#pragma unroll
        for (int q = E / 2; q < E; ++q) v[q] = c32x2{f2(0.f, 0.f), f2(0.f, 0.f)};
        fft_cta<M1, E, -1, true, G::TWS, G::NCOL>(v, smem, nullptr, t1, tws, j);
        const c32 base = ldg_c(a.f.tw + ((2 * (int64_t)n2 * t1) & (M - 1)));
        const c32 step = ldg_c(a.f.tw + ((2 * (int64_t)n2 * T1) & (M - 1)));
        twiddle_powers<E, 1, 0>(v, step);
        const uint64_t keep = l2_keep();
#pragma unroll
        for (int q = 0; q < E; ++q) {
            const c32x2 r = mul(v[q], base);
            const int ad = (t1 + q * T1) * M2 + n2;
            if (!check_index(a.f.err, ad, MC)) continue;
            st_pol(w0 + ad, make_float2(r.re.x, r.im.x), keep);
            if (has1) st_pol(w1 + ad, make_float2(r.re.y, r.im.y), keep);
        }
    }
}

template <typename G>
__global__ void __launch_bounds__(G::RT, G::RMINB) hyena_staged_rows_x2(const StagedArgs a, int64_t nr) {
    static_assert(G::ROWS == 2, "lockstep geometry");
    constexpr int E = G::E, M1 = G::M1, M2 = G::M2, T2 = G::T2, MC = G::MC, M = 2 * MC;
    constexpr int NROW = G::NROW, HROW = G::HROW, RT = G::RT;
    extern __shared__ float smem[];
    float4 *rowb = reinterpret_cast<float4 *>(smem);
    const int64_t lp = blockIdx.x / G::RGROUPS;
    const int g = blockIdx.x % G::RGROUPS;
    const int r = threadIdx.x % NROW, t2 = threadIdx.x / NROW;
    const int k1 = row_of_slot<G>(g, r);
    const int rm = (k1 == 0 || k1 == M1 / 2) ? r : (r < HROW ? r + HROW : r - HROW);   // slot of row M1 - k1
    const bool has1 = 2 * lp + 1 < nr;
    int64_t d0, d1;
    (void)visit_row(a.f, a.o0 + 2 * lp, d0);
    (void)visit_row(a.f, a.o0 + 2 * lp + (has1 ? 1 : 0), d1);
    // debug build: the CTA's rows and their spectrum rows exist (uniform over the CTA)
    const int64_t hrows = (int64_t)a.f.order * a.f.hD;
    if (!(check_index(a.f.err, 2 * lp + (has1 ? 1 : 0), nr) && check_index(a.f.err, d0, a.f.D) &&
          check_index(a.f.err, d1, a.f.D) && check_index(a.f.err, (int64_t)a.n * a.f.hD + d1, hrows)))
        return;
    float2 *w0 = a.ws + (2 * lp) * MC;
    float2 *w1 = a.ws + (2 * lp + (has1 ? 1 : 0)) * MC;
    const c32 *tws = a.f.tw + M;
    // shared element (re a, re b, im a, im b); the debug build checks the slot index
    auto ld = [&](int ad) -> c32x2 {
        if (!check_index(a.f.err, ad, NROW * M2)) return c32x2{f2(0.f, 0.f), f2(0.f, 0.f)};
        const float4 f = rowb[ad];
        return c32x2{f2(f.x, f.y), f2(f.z, f.w)};
    };
    auto st = [&](int ad, c32x2 x) {
        if (check_index(a.f.err, ad, NROW * M2)) rowb[ad] = make_float4(x.re.x, x.re.y, x.im.x, x.im.y);
    };

    // The spectrum bins of a row group lie 2 KB apart in the channel's spectrum
    // row, which DRAM serves poorly. The RGROUPS CTAs of a row pair cover both
    // rows' spectra, so each first brings 1/RGROUPS of them (a contiguous run
    // of 16-byte blocks inside the row) into L2 with one bulk prefetch per row.
    if (threadIdx.x < 2 && (threadIdx.x == 0 || d1 != d0)) {
        const uintptr_t rs =
            reinterpret_cast<uintptr_t>(a.f.H + ((int64_t)a.n * a.f.hD + (threadIdx.x ? d1 : d0)) * (MC + 1));
        const uintptr_t re = rs + (uintptr_t)(MC + 1) * 8;
        const uintptr_t piece = (((uintptr_t)(MC + 1) * 8 + G::RGROUPS - 1) / G::RGROUPS + 15) & ~(uintptr_t)15;
        const uintptr_t b = (rs + (uintptr_t)g * piece + 15) & ~(uintptr_t)15;
        uintptr_t e = rs + (uintptr_t)(g + 1) * piece;
        e = (e < re ? e : re) & ~(uintptr_t)15;
        if (e > b)
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(b), "r"((uint32_t)(e - b)) : "memory");
    }
    // the group's rows of both lanes, coalesced, into the sequence-major buffer
    const uint64_t keep = l2_keep(), stream = l2_stream();
#pragma unroll
    for (int sl = 0; sl < NROW; ++sl) {
        const int64_t base = (int64_t)row_of_slot<G>(g, sl) * M2;
#pragma unroll
        for (int k2 = threadIdx.x; k2 < M2; k2 += RT) {
            const float2 f0 = ld_pol(w0 + base + k2, keep), f1 = ld_pol(w1 + base + k2, keep);
            rowb[maddr<M2>(k2, sl)] = make_float4(f0.x, f1.x, f0.y, f1.y);
        }
    }
    __syncthreads();
    c32x2 v[E];
#pragma unroll
    for (int q = 0; q < E; ++q) v[q] = ld(maddr<M2>(t2 + q * T2, r));
    __syncthreads();
    fft_cta<M2, E, -1, false, G::TWS, NROW>(v, smem, nullptr, t2, tws, r);
#pragma unroll
    for (int q = 0; q < E; ++q) st(maddr<M2>(t2 + q * T2, r), v[q]);
    __syncthreads();

    // spectral step on both lanes, bins in pairs (k, MC - k): the mirror of register q is
    // register E-1-q of thread (rm, T2-1-t2) (in row 0: of thread (0, T2-t2), and register
    // E-q when t2 = 0), so each thread takes q < E/2 and returns the mirror result
    // conj(Ye - i Yo) to its owner; bin (0, M2/2) is its own mirror;
    // the unpacking is written without its factors 1/2, folded into the gain
    const float dsk0 = a.f.dskip ? __ldg(a.f.dskip + a.n * a.f.hD + d0) : 0.f;
    const float dsk1 = a.f.dskip ? __ldg(a.f.dskip + a.n * a.f.hD + d1) : 0.f;
    const c32 *H0 = a.f.H + ((int64_t)a.n * a.f.hD + d0) * (MC + 1);
    const c32 *H1 = a.f.H + ((int64_t)a.n * a.f.hD + d1) * (MC + 1);
    const c32 wb = ldg_c(a.f.tw + k1 + M1 * t2);     // W_M^{k1 + M1 t2}
    constexpr float s = 0.25f / (float)MC;
    const int z0 = opaque_zero();
    auto bin_pair = [&](int q, c32x2 Zk, c32x2 &Ye, c32x2 &Yo) __attribute__((always_inline)) {
        const int k = k1 + M1 * (t2 + q * T2);
        const int km = (MC - k) & (MC - 1);
        const c32x2 Zm = ld(maddr<M2>(km / M1, rm));
        const c32x2 E2{f2add(Zk.re, Zm.re), f2sub(Zk.im, Zm.im)};   // Zk + conj Zm
        const c32x2 O2{f2add(Zk.im, Zm.im), f2sub(Zm.re, Zk.re)};   // (Zk - conj Zm) / i
        const c32 w = mul(wb, w2e<E>(q, z0));                        // W_M^k
        const c32x2 wO = mul(O2, w);
        const c32x2 Xk = add(E2, wO);
        const c32x2 Xm{f2sub(E2.re, wO.re), f2sub(wO.im, E2.im)};
        const c32 hk0 = ldc_pol(H0 + k, stream), hk1 = ldc_pol(H1 + k, stream);
        const c32 hm0 = ldc_pol(H0 + (MC - k), stream), hm1 = ldc_pol(H1 + (MC - k), stream);
        const c32x2 Hk{f2(s * (hk0.x + dsk0), s * (hk1.x + dsk1)), f2(s * hk0.y, s * hk1.y)};
        const c32x2 Hm{f2(s * (hm0.x + dsk0), s * (hm1.x + dsk1)), f2(s * hm0.y, s * hm1.y)};
        const c32x2 Yk = mul(Xk, Hk), Ym = mul(Xm, Hm);
        Ye = c32x2{f2add(Yk.re, Ym.re), f2sub(Yk.im, Ym.im)};       // Yk + conj Ym
        const c32x2 Yd{f2sub(Yk.re, Ym.re), f2add(Yk.im, Ym.im)};   // Yk - conj Ym
        Yo = mul(Yd, conj(w));
    };
    const bool self_half = k1 == 0 && t2 == 0;
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
        v[q] = c32x2{f2sub(Ye.re, Yo.im), f2add(Ye.im, Yo.re)};             // Ye + i Yo       (bin k)
        v[E / 2 + q] = c32x2{f2add(Ye.re, Yo.im), f2sub(Yo.re, Ye.im)};    // conj(Ye - i Yo) (bin MC - k)
        if ((q & 3) == 3) asm volatile("" ::: "memory");  // bound load hoisting (register pressure)
    }
    __syncthreads();                                      // every mirror read done
#pragma unroll
    for (int q = 0; q < E / 2; ++q) {
        const int k = k1 + M1 * (t2 + q * T2);
        st(maddr<M2>(((MC - k) & (MC - 1)) / M1, rm), v[E / 2 + q]);
    }
    __syncthreads();
#pragma unroll
    for (int q = E / 2; q < E; ++q) v[q] = ld(maddr<M2>(t2 + q * T2, r));
    if (self_half) v[E / 2] = vh;
    __syncthreads();                                      // buffer reads done before the inverse rewrites it

    fft_cta<M2, E, +1, false, G::TWS, NROW>(v, smem, nullptr, t2, tws, r);
    const c32 base = conj(ldg_c(a.f.tw + ((2 * (int64_t)t2 * k1) & (M - 1))));
    const c32 step = conj(ldg_c(a.f.tw + ((2 * (int64_t)T2 * k1) & (M - 1))));
    twiddle_powers<E, 1, 0>(v, step);
#pragma unroll
    for (int q = 0; q < E; ++q) st(maddr<M2>(t2 + q * T2, r), mul(v[q], base));
    __syncthreads();
#pragma unroll
    for (int sl = 0; sl < NROW; ++sl) {
        const int64_t base_ad = (int64_t)row_of_slot<G>(g, sl) * M2;
#pragma unroll
        for (int k2 = threadIdx.x; k2 < M2; k2 += RT) {
            const float4 f = rowb[maddr<M2>(k2, sl)];
            st_pol(w0 + base_ad + k2, make_float2(f.x, f.z), keep);
            if (has1) st_pol(w1 + base_ad + k2, make_float2(f.y, f.w), keep);
        }
    }
}

// ---------------------------------------------------------------------------
// Filter spectra of long rows through the same two stages, two filter rows in
// lockstep: the column kernel reads the taps (fp32, zero past L) and runs the
// forward column FFTs and twiddle; the row kernel runs the row FFTs and
// unpacks the packed spectrum into H[k] = E[k] + W_M^k O[k] (natural order,
// H[MC] = E[0] - O[0]). The scratch belongs to the plan, so the spectrum may
// be computed in place: a chunk's column kernel reads all of its rows before
// its row kernel writes their spectra.

struct Spec1dArgs {
    const float *h;    // filter row o at h + o * h_stride, L taps
    int64_t h_stride;
    int64_t L;
    c32 *Hout;         // [rows][MC + 1]
    const c32 *tw;     // W_M, then W_1024
    float2 *ws;        // chunk rows x MC complex, each [k1][n2]
    int64_t o0;        // first filter row of the chunk
    int64_t nr;        // rows in the chunk
};

template <typename G>
__global__ void __launch_bounds__(G::CT, G::CMINB) hyena_staged_spec_cols_x2(const Spec1dArgs a) {
    static_assert(G::ROWS == 2, "lockstep geometry");
    constexpr int E = G::E, M1 = G::M1, M2 = G::M2, T1 = G::T1, MC = G::MC, M = 2 * MC;
    extern __shared__ float smem[];
    const int64_t lp = blockIdx.x / G::CGROUPS;
    const int cgp = blockIdx.x % G::CGROUPS;
    const int j = threadIdx.x % G::NCOL, t1 = threadIdx.x / G::NCOL;
    const int n2 = cgp * G::NCOL + j;
    const bool has1 = 2 * lp + 1 < a.nr;
    const float *h0 = a.h + (a.o0 + 2 * lp) * a.h_stride;
    const float *h1 = a.h + (a.o0 + 2 * lp + (has1 ? 1 : 0)) * a.h_stride;
    float2 *w0 = a.ws + (2 * lp) * MC;
    float2 *w1 = a.ws + (2 * lp + (has1 ? 1 : 0)) * MC;
    c32x2 v[E];
#pragma unroll
    for (int q = 0; q < E / 2; ++q) {
        const int64_t pos = 2 * ((int64_t)M2 * (t1 + q * T1) + n2);
        const float a0 = pos < a.L ? h0[pos] : 0.f, b0 = pos + 1 < a.L ? h0[pos + 1] : 0.f;
        const float a1 = has1 && pos < a.L ? h1[pos] : 0.f, b1 = has1 && pos + 1 < a.L ? h1[pos + 1] : 0.f;
        v[q] = c32x2{f2(a0, a1), f2(b0, b1)};
    }
#pragma unroll
    for (int q = E / 2; q < E; ++q) v[q] = c32x2{f2(0.f, 0.f), f2(0.f, 0.f)};
    fft_cta<M1, E, -1, true, G::TWS, G::NCOL>(v, smem, nullptr, t1, a.tw + M, j);
    const c32 base = ldg_c(a.tw + ((2 * (int64_t)n2 * t1) & (M - 1)));
    const c32 step = ldg_c(a.tw + ((2 * (int64_t)n2 * T1) & (M - 1)));
    twiddle_powers<E, 1, 0>(v, step);
    const uint64_t keep = l2_keep();
#pragma unroll
    for (int q = 0; q < E; ++q) {
        const c32x2 r = mul(v[q], base);
        const int ad = (t1 + q * T1) * M2 + n2;
        st_pol(w0 + ad, make_float2(r.re.x, r.im.x), keep);
        if (has1) st_pol(w1 + ad, make_float2(r.re.y, r.im.y), keep);
    }
}

template <typename G>
__global__ void __launch_bounds__(G::RT, G::RMINB) hyena_staged_spec_rows_x2(const Spec1dArgs a) {
    static_assert(G::ROWS == 2, "lockstep geometry");
    constexpr int E = G::E, M1 = G::M1, M2 = G::M2, T2 = G::T2, MC = G::MC, M = 2 * MC;
    constexpr int NROW = G::NROW, HROW = G::HROW, RT = G::RT;
    extern __shared__ float smem[];
    float4 *rowb = reinterpret_cast<float4 *>(smem);
    const int64_t lp = blockIdx.x / G::RGROUPS;
    const int g = blockIdx.x % G::RGROUPS;
    const int r = threadIdx.x % NROW, t2 = threadIdx.x / NROW;
    const int k1 = row_of_slot<G>(g, r);
    const int rm = (k1 == 0 || k1 == M1 / 2) ? r : (r < HROW ? r + HROW : r - HROW);
    const bool has1 = 2 * lp + 1 < a.nr;
    const float2 *w0 = a.ws + (2 * lp) * MC;
    const float2 *w1 = a.ws + (2 * lp + (has1 ? 1 : 0)) * MC;
    auto ld = [&](int ad) -> c32x2 {
        const float4 f = rowb[ad];
        return c32x2{f2(f.x, f.y), f2(f.z, f.w)};
    };
    const uint64_t once = l2_stream();               // the scratch is read once
#pragma unroll
    for (int sl = 0; sl < NROW; ++sl) {
        const int64_t base = (int64_t)row_of_slot<G>(g, sl) * M2;
#pragma unroll
        for (int k2 = threadIdx.x; k2 < M2; k2 += RT) {
            const float2 f0 = ld_pol(w0 + base + k2, once), f1 = ld_pol(w1 + base + k2, once);
            rowb[maddr<M2>(k2, sl)] = make_float4(f0.x, f1.x, f0.y, f1.y);
        }
    }
    __syncthreads();
    c32x2 v[E];
#pragma unroll
    for (int q = 0; q < E; ++q) v[q] = ld(maddr<M2>(t2 + q * T2, r));
    __syncthreads();
    fft_cta<M2, E, -1, false, G::TWS, NROW>(v, smem, nullptr, t2, a.tw + M, r);
#pragma unroll
    for (int q = 0; q < E; ++q)
        rowb[maddr<M2>(t2 + q * T2, r)] = make_float4(v[q].re.x, v[q].re.y, v[q].im.x, v[q].im.y);
    __syncthreads();
    const c32 wb = ldg_c(a.tw + k1 + M1 * t2);      // W_M^{k1 + M1 t2}
    c32 *H0 = a.Hout + (a.o0 + 2 * lp) * (int64_t)(MC + 1);
    c32 *H1 = a.Hout + (a.o0 + 2 * lp + (has1 ? 1 : 0)) * (int64_t)(MC + 1);
    const int z0 = opaque_zero();
#pragma unroll
    for (int q = 0; q < E; ++q) {
        const int k = k1 + M1 * (t2 + q * T2);
        const int km = (MC - k) & (MC - 1);
        const c32x2 Zk = v[q];
        const c32x2 Zm = ld(maddr<M2>(km / M1, rm));
        const c32x2 E2{f2add(Zk.re, Zm.re), f2sub(Zk.im, Zm.im)};   // 2E
        const c32x2 O2{f2add(Zk.im, Zm.im), f2sub(Zm.re, Zk.re)};   // 2O
        const c32x2 wO = mul(O2, mul(wb, w2e<E>(q, z0)));
        const float2 half = f2(0.5f, 0.5f);
        const c32x2 X{f2mul(f2add(E2.re, wO.re), half), f2mul(f2add(E2.im, wO.im), half)};
        H0[k] = mk(X.re.x, X.im.x);
        if (has1) H1[k] = mk(X.re.y, X.im.y);
        if (k == 0) {                                  // Nyquist bin: E_0 - O_0, real
            const float2 ny = f2mul(f2sub(E2.re, O2.re), half);
            H0[MC] = mk(ny.x, 0.f);
            if (has1) H1[MC] = mk(ny.y, 0.f);
        }
    }
}

}  // namespace hyena
