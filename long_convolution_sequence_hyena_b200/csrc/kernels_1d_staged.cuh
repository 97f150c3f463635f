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

template <int MC_, int M1_, int NCOL_, int NROW_>
struct StagedGeom {
    static constexpr int MC = MC_, M1 = M1_, M2 = MC_ / M1_, E = 16;
    static constexpr int NCOL = NCOL_;               // columns per column-kernel CTA
    static constexpr int NROW = NROW_;               // rows per row-kernel CTA (mirror pairs)
    static constexpr int HROW = NROW / 2;
    static constexpr int T1 = M1 / E, T2 = M2 / E;   // threads per column / row FFT
    static constexpr int CT = NCOL * T1;             // column-kernel threads
    static constexpr int RT = NROW * T2;             // row-kernel threads
    static constexpr int CGROUPS = M2 / NCOL;        // column CTAs per row
    static constexpr int RGROUPS = M1 / NROW;        // row CTAs per row
    static constexpr int TWS = 1024;                 // sub-transform twiddle table W_1024
    static constexpr size_t CSMEM = (size_t)NCOL * M1 * 8;
    static constexpr size_t RSMEM = (size_t)NROW * M2 * 8;
    static_assert(M2 % NCOL == 0 && M1 % NROW == 0 && NROW % 2 == 0, "groups must tile the row");
    static_assert(NCOL >= 16 && NROW >= 16, "warps must span at least 16 sequences");
    static_assert(TWS % M1 == 0 && TWS % M2 == 0, "sub-transform twiddles");
    static_assert(CT <= 1024 && RT <= 1024, "too many threads");
};

struct StagedArgs {
    Fwd1dArgs f;      // operator arguments
    float2 *ws;       // workspace: chunk rows x MC complex, each [k1][n2]
    int64_t o0;       // visit index of the chunk's first row (visit order d-major, b-minor)
    int n;            // order: gate x^n (column kernel), spectrum H^n (row kernel)
};

// Flat row of visit index o (d-major, b-minor: the B rows of one channel run together).
__device__ __forceinline__ int64_t visit_row(const Fwd1dArgs &f, int64_t o, int64_t &d) {
    d = o / f.B;
    return (o - d * f.B) * f.D + d;
}

// MODE 0: first (load v, forward columns); 1: between orders (inverse columns,
// gate x^n, forward columns); 2: last (inverse columns, gate x^n, store y).
template <typename G, typename IO, bool EVEN, int MODE>
__global__ void __launch_bounds__(G::CT, 2) hyena_staged_cols(const StagedArgs a) {
    constexpr int E = G::E, M1 = G::M1, M2 = G::M2, T1 = G::T1, MC = G::MC, M = 2 * MC;
    extern __shared__ float smem[];
    const int64_t lr = blockIdx.x / G::CGROUPS;      // row within the chunk
    const int cgp = blockIdx.x % G::CGROUPS;
    const int j = threadIdx.x % G::NCOL, t1 = threadIdx.x / G::NCOL;
    const int n2 = cgp * G::NCOL + j;
    int64_t d;
    const int64_t row = visit_row(a.f, a.o0 + lr, d);
    const int64_t L = a.f.L;
    float2 *wrow = a.ws + lr * MC;
    const c32 *tws = a.f.tw + M;                     // W_1024
    // time-domain element (n1, n2) of register q is z[M2 (t1 + q T1) + n2] = x[pos], x[pos + 1]
    auto pos_of = [&](int q) -> int64_t { return 2 * ((int64_t)M2 * (t1 + q * T1) + n2); };

    c32 v[E];
    if constexpr (MODE == 0) {
        const IO *vrow = reinterpret_cast<const IO *>(a.f.v) + row * L;
#pragma unroll
        for (int q = 0; q < E / 2; ++q) v[q] = load_pair<IO, EVEN>(vrow, pos_of(q), L);
    } else {
        using P = typename io<IO>::pair_t;
        const IO *grow = reinterpret_cast<const IO *>(a.f.gates[a.n]) + row * L;
        P g[E / 2];   // this order's gate, loaded while the inverse transform runs
#pragma unroll
        for (int q = 0; q < E / 2; ++q) g[q] = load_pair_raw<IO, EVEN>(grow, pos_of(q), L);
#pragma unroll
        for (int q = 0; q < E; ++q) {
            const float2 f = wrow[(t1 + q * T1) * M2 + n2];   // k1 = t1 + q T1
            v[q] = mk(f.x, f.y);
        }
        fft_cta<M1, E, +1, false, G::TWS, G::NCOL>(v, smem, nullptr, t1, tws, j);
        // gate; registers q >= E/2 hold the zero padding (positions >= MC)
#pragma unroll
        for (int q = 0; q < E / 2; ++q) {
            const int64_t pos = pos_of(q);
            const c32 gq = io<IO>::unpack(g[q]);
            v[q] = mk(pos < L ? gq.x * v[q].x : 0.f, pos + 1 < L ? gq.y * v[q].y : 0.f);
        }
        if constexpr (MODE == 2) {
            IO *yrow = reinterpret_cast<IO *>(a.f.y) + row * L;
#pragma unroll
            for (int q = 0; q < E / 2; ++q) store_pair<IO, EVEN>(yrow, pos_of(q), L, v[q]);
            return;
        }
    }
    if constexpr (MODE != 2) {
#pragma unroll
        for (int q = E / 2; q < E; ++q) v[q] = mk(0.f, 0.f);
        fft_cta<M1, E, -1, true, G::TWS, G::NCOL>(v, smem, nullptr, t1, tws, j);
        // four-step twiddle W_MC^{n2 k1} = W_M^{2 n2 k1}, k1 = t1 + q T1
        const c32 base = ldg_c(a.f.tw + ((2 * (int64_t)n2 * t1) & (M - 1)));
        const c32 step = ldg_c(a.f.tw + ((2 * (int64_t)n2 * T1) & (M - 1)));
        twiddle_powers<E, 1, 0>(v, step);
#pragma unroll
        for (int q = 0; q < E; ++q) {
            const c32 r = mul(v[q], base);
            wrow[(t1 + q * T1) * M2 + n2] = make_float2(r.x, r.y);
        }
    }
}

template <typename G>
__global__ void __launch_bounds__(G::RT, 2) hyena_staged_rows(const StagedArgs a) {
    constexpr int E = G::E, M1 = G::M1, M2 = G::M2, T2 = G::T2, MC = G::MC, M = 2 * MC;
    constexpr int NROW = G::NROW, HROW = G::HROW;
    extern __shared__ float smem[];
    float2 *rowb = reinterpret_cast<float2 *>(smem);
    const int64_t lr = blockIdx.x / G::RGROUPS;
    const int g = blockIdx.x % G::RGROUPS;
    const int r = threadIdx.x % NROW, t2 = threadIdx.x / NROW;
    const int k1 = row_of_slot<G>(g, r);
    const int rm = (k1 == 0 || k1 == M1 / 2) ? r : (r < HROW ? r + HROW : r - HROW);   // slot of row M1 - k1
    int64_t d;
    (void)visit_row(a.f, a.o0 + lr, d);
    float2 *wrow = a.ws + lr * MC;
    const c32 *tws = a.f.tw + M;

    // the group's rows, coalesced, into the sequence-major buffer
    for (int e = threadIdx.x; e < NROW * M2; e += G::RT) {
        const int s = e / M2, k2 = e % M2;
        cp_async8(rowb + maddr<M2>(k2, s), wrow + (int64_t)row_of_slot<G>(g, s) * M2 + k2);
    }
    cp_async_commit();
    cp_async_wait_all();
    __syncthreads();
    c32 v[E];
#pragma unroll
    for (int q = 0; q < E; ++q) {
        const float2 f = rowb[maddr<M2>(t2 + q * T2, r)];
        v[q] = mk(f.x, f.y);
    }
    __syncthreads();
    fft_cta<M2, E, -1, false, G::TWS, NROW>(v, smem, nullptr, t2, tws, r);

    // publish the bins so that the mirror rows can read them
#pragma unroll
    for (int q = 0; q < E; ++q) rowb[maddr<M2>(t2 + q * T2, r)] = make_float2(v[q].x, v[q].y);
    __syncthreads();

    // Spectral step, bins in pairs (k, MC - k): the mirror of register q is
    // register E-1-q of thread (rm, T2-1-t2) (in row 0: of thread (0, T2-t2),
    // and register E-q when t2 = 0), so each thread takes q < E/2 and returns
    // the mirror result conj(Ye - i Yo) to its owner; bin (0, M2/2) is its own mirror.
    const float dsk = a.f.dskip ? __ldg(a.f.dskip + a.n * a.f.D + d) : 0.f;
    const c32 *Hrow = a.f.H + ((int64_t)a.n * a.f.D + d) * (MC + 1);
    const c32 wb = ldg_c(a.f.tw + k1 + M1 * t2);     // W_M^{k1 + M1 t2}
    constexpr float s = 0.5f / (float)MC;
    const int z0 = opaque_zero();
    auto bin_pair = [&](int q, c32 Zk, c32 &Ye, c32 &Yo) __attribute__((always_inline)) {
        const int k = k1 + M1 * (t2 + q * T2);
        const int km = (MC - k) & (MC - 1);
        const float2 mf = rowb[maddr<M2>(km / M1, rm)];
        const c32 Zm = mk(mf.x, mf.y);
        const c32 Ek = mk(0.5f * (Zk.x + Zm.x), 0.5f * (Zk.y - Zm.y));
        const c32 Ok = mk(0.5f * (Zk.y + Zm.y), -0.5f * (Zk.x - Zm.x));
        const c32 w = mul(wb, w2e<E>(q, z0));            // W_M^k
        const c32 wO = mul(w, Ok);
        const c32 Xk = add(Ek, wO);
        const c32 Xm = conj(sub(Ek, wO));
        c32 Hk = ldg_c(Hrow + k);
        c32 Hm = ldg_c(Hrow + (MC - k));
        Hk.x += dsk;
        Hm.x += dsk;
        const c32 Yk = mul(Xk, Hk), Ym = mul(Xm, Hm);
        Ye = mk(s * (Yk.x + Ym.x), s * (Yk.y - Ym.y));
        const c32 Yd = mk(s * (Yk.x - Ym.x), s * (Yk.y + Ym.y));
        Yo = mul(Yd, conj(w));
    };
    const bool self_half = k1 == 0 && t2 == 0;
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
        v[q] = mk(Ye.x - Yo.y, Ye.y + Yo.x);              // Ye + i Yo       (bin k)
        v[E / 2 + q] = mk(Ye.x + Yo.y, Yo.x - Ye.y);      // conj(Ye - i Yo) (bin MC - k)
        if ((q & 3) == 3) asm volatile("" ::: "memory");  // bound load hoisting (register pressure)
    }
    __syncthreads();                                      // every mirror read done
#pragma unroll
    for (int q = 0; q < E / 2; ++q) {
        const int k = k1 + M1 * (t2 + q * T2);
        rowb[maddr<M2>(((MC - k) & (MC - 1)) / M1, rm)] = make_float2(v[E / 2 + q].x, v[E / 2 + q].y);
    }
    __syncthreads();
#pragma unroll
    for (int q = E / 2; q < E; ++q) {
        const float2 f = rowb[maddr<M2>(t2 + q * T2, r)];
        v[q] = mk(f.x, f.y);
    }
    if (self_half) v[E / 2] = vh;
    __syncthreads();                                      // buffer reads done before the inverse rewrites it

    fft_cta<M2, E, +1, false, G::TWS, NROW>(v, smem, nullptr, t2, tws, r);
    // conjugate four-step twiddle, conj W_MC^{n2 k1}, n2 = t2 + q T2; out through the buffer
    const c32 base = conj(ldg_c(a.f.tw + ((2 * (int64_t)t2 * k1) & (M - 1))));
    const c32 step = conj(ldg_c(a.f.tw + ((2 * (int64_t)T2 * k1) & (M - 1))));
    twiddle_powers<E, 1, 0>(v, step);
#pragma unroll
    for (int q = 0; q < E; ++q) {
        const c32 o = mul(v[q], base);
        rowb[maddr<M2>(t2 + q * T2, r)] = make_float2(o.x, o.y);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < NROW * M2; e += G::RT) {
        const int sl = e / M2, k2 = e % M2;
        wrow[(int64_t)row_of_slot<G>(g, sl) * M2 + k2] = rowb[maddr<M2>(k2, sl)];
    }
}

}  // namespace hyena
