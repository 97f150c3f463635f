// 1D fused order-N forward and filter spectrum for padded lengths that are
// three times a power of two: M = 6 P, packed complex length MC = 3 P.
//
// "Hyena — Long Convolutions Math", "Linear vs circular" and "Counting the
// cost": the causal product only needs a transform of at least 2L points, and
// rounding 2L up to a power of two can nearly double the work; M = 3 2^j cuts
// the padding (2L = 6000: 6144 points instead of 8192).
//
// The MC-point transform is one radix-3 step and three P-point transforms
// (MC = 3 x P, element n = P s + n2, bin k = k1 + 3 k2):
//   forward:  y_{k1}[n2] = sum_s z[P s + n2] W_3^{s k1}        (radix 3, in registers)
//             y_{k1}[n2] *= W_MC^{n2 k1}                       (twiddle)
//             Z[k1 + 3 k2] = DFT_P(y_{k1})[k2]                  (three radix-16 Stockham FFTs)
//   inverse:  the same steps backwards with conjugate twiddles.
// A row takes three groups of T = P / E threads (E = 16 values per thread, 32
// at P = 4096); thread t of group s holds positions P s + t + q T (q < E) in
// the time domain and bins s + 3 (t + q T)
// in the frequency domain, so the gate stays in registers; the radix-3 step
// exchanges through shared memory, and the three P-point transforms run at
// once, each group on its own exchange region.
//
// The spectral step (real-input unpack, product with the filter gain plus the
// feedthrough, repack for the inverse, as in kernels_1d.cuh) needs each bin's
// mirror Z[MC - k]; all bins of the row are published in shared memory and
// every thread computes its own bins (each mirror pair is formed twice).
#pragma once
#include "kernels_1d.cuh"

namespace hyena {

template <int P>
struct MR3 {
    static constexpr int E = P >= 4096 ? 32 : 16;        // values per thread (32: at most 384 threads per row)
    static constexpr int T = P / E, MC = 3 * P, M = 2 * MC;
    static constexpr int GT = 3 * T;                      // threads per row: three groups of T
    static constexpr int RPC = GT >= 96 ? 1 : 96 / GT;    // rows per CTA
    static constexpr int THREADS = RPC * GT;
    static constexpr int SMEM_FLOATS = 2 * MC;            // per row: the row (re, im planes) or three FFT exchanges
    // resident CTAs per SM the register budget is sized for (about 170 registers per thread)
    static constexpr int MINB = THREADS >= 384 ? 1 : 384 / THREADS;
    static_assert(P >= 16 && (P & (P - 1)) == 0, "P is a power of two of at least 16");
    static_assert(THREADS <= 1024, "P up to 4096");
};

// Radix-3 DFT output k1: sum_s x_s W_3^{s k1}, W_3 = exp(DIR 2 pi i / 3).
template <int DIR>
__device__ __forceinline__ c32 dft3_out(c32 x0, c32 x1, c32 x2, int k1) {
    constexpr float h = 0.86602540378443864676f;   // sqrt(3) / 2
    const c32 s = add(x1, x2);
    if (k1 == 0) return add(x0, s);
    const c32 t = mk(x0.x - 0.5f * s.x, x0.y - 0.5f * s.y);
    const c32 u = rot90<DIR>(scale(sub(x1, x2), h));   // DIR i sqrt(3)/2 (x1 - x2)
    return k1 == 1 ? add(t, u) : sub(t, u);
}

// The row's radix-3 step through shared memory: every thread publishes its 16
// values of sub-sequence `s`, then takes output `s` (k1 = s forward, n1 = s
// inverse) of the 3-point DFTs at its positions. Ends with the buffer free.
template <int P, int DIR>
__device__ __forceinline__ void radix3_step(c32 (&v)[MR3<P>::E], float *rre, float *rim, int s, int t) {
    using G = MR3<P>;
    constexpr int E = G::E, T = G::T;
#pragma unroll
    for (int q = 0; q < E; ++q) {
        rre[P * s + t + q * T] = v[q].x;
        rim[P * s + t + q * T] = v[q].y;
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < E; ++q) {
        const int n2 = t + q * T;
        v[q] = dft3_out<DIR>(mk(rre[n2], rim[n2]), mk(rre[P + n2], rim[P + n2]), mk(rre[2 * P + n2], rim[2 * P + n2]),
                             s);
    }
    __syncthreads();
}

// Forward (DIR -1) or inverse (+1) MC-point transform. Thread (s, t) holds
// positions P s + t + q T in the time domain and bins s + 3 (t + q T) in the
// frequency domain. buf: 2 MC floats (the row, or three FFT exchanges of 2 P).
template <int P, int DIR>
__device__ __forceinline__ void fft_mr3(c32 (&v)[MR3<P>::E], float *buf, int s, int t, const c32 *__restrict__ tw) {
    using G = MR3<P>;
    constexpr int E = G::E, T = G::T, M = G::M, MC = G::MC;
    float *ere = buf + 2 * P * s, *eim = ere + P;   // this group's exchange region
    if constexpr (DIR < 0) {
        radix3_step<P, -1>(v, buf, buf + MC, s, t);
        if (s > 0) {
#pragma unroll
            for (int q = 0; q < E; ++q) v[q] = mul(v[q], ldg_c(tw + ((2 * s * (t + q * T)) % M)));   // W_MC^{n2 k1}
        }
        fft_cta<P, E, -1, false, M>(v, ere, eim, t, tw);
        __syncthreads();
    } else {
        fft_cta<P, E, +1, false, M>(v, ere, eim, t, tw);
        __syncthreads();
        if (s > 0) {
#pragma unroll
            for (int q = 0; q < E; ++q) v[q] = mul(v[q], conj(ldg_c(tw + ((2 * s * (t + q * T)) % M))));
        }
        radix3_step<P, +1>(v, buf, buf + MC, s, t);
    }
}

template <int P, typename IO, bool EVEN>
__global__ void __launch_bounds__(MR3<P>::THREADS, MR3<P>::MINB) hyena_fwd_1d_mr3(const Fwd1dArgs a) {
    using G = MR3<P>;
    constexpr int E = G::E, T = G::T, MC = G::MC, RPC = G::RPC;
    extern __shared__ float smem[];
    const int lrow = threadIdx.x / G::GT;
    const int gt = threadIdx.x - lrow * G::GT;
    const int s = gt / T, t = gt - s * T;          // sub-sequence and thread within it
    const int64_t ord = (int64_t)blockIdx.x * RPC + lrow;
    const bool active = ord < a.rows;
    const int64_t d = active ? ord / a.B : 0;
    const int64_t b = active ? ord - d * a.B : 0;
    const int64_t row = b * a.D + d;
    float *buf = smem + lrow * G::SMEM_FLOATS;
    float *pre = buf, *pim = buf + MC;
    const int64_t L = a.L;
    auto pos_of = [&](int q) -> int64_t { return 2 * ((int64_t)P * s + t + q * T); };

    c32 v[E];
    {
        const IO *vrow = reinterpret_cast<const IO *>(a.v) + act_row_off(a, row);
#pragma unroll
        for (int q = 0; q < E; ++q) v[q] = active ? load_pair_s<IO, EVEN>(vrow, pos_of(q), L, a.es) : mk(0.f, 0.f);
    }
    constexpr float sc = 0.5f / (float)MC;
    for (int n = 0; n < a.order; ++n) {
        const IO *grow = reinterpret_cast<const IO *>(a.gates[n]) + act_row_off(a, row);
        // this order's gate, loaded while the transforms run (16 values per thread; with 32 the
        // registers are needed for the transform and the gate is read where it multiplies)
        constexpr bool PRE = E == 16;
        typename io<IO>::pair_t g[PRE ? E : 1];
        if constexpr (PRE) {
#pragma unroll
            for (int q = 0; q < E; ++q)
                g[q] = active ? load_pair_raw_s<IO, EVEN>(grow, pos_of(q), L, a.es) : io<IO>::zero();
        }
        fft_mr3<P, -1>(v, buf, s, t, a.tw);
        // spectral step: every bin of the row in shared memory, each thread takes its own
#pragma unroll
        for (int q = 0; q < E; ++q) {
            const int k = s + 3 * (t + q * T);
            pre[k] = v[q].x;
            pim[k] = v[q].y;
        }
        __syncthreads();
        const float dsk = a.dskip ? __ldg(a.dskip + n * a.hD + d) : 0.f;
        const c32 *Hrow = a.H + ((int64_t)n * a.hD + d) * (MC + 1);
#pragma unroll
        for (int q = 0; q < E; ++q) {
            const int k = s + 3 * (t + q * T);
            const int km = (MC - k) % MC;
            const c32 Zk = v[q], Zm = mk(pre[km], pim[km]);
            const c32 Ek = mk(0.5f * (Zk.x + Zm.x), 0.5f * (Zk.y - Zm.y));
            const c32 Ok = mk(0.5f * (Zk.y + Zm.y), -0.5f * (Zk.x - Zm.x));
            const c32 w = ldg_c(a.tw + k);                  // W_M^k
            const c32 wO = mul(w, Ok);
            const c32 Xk = add(Ek, wO), Xm = conj(sub(Ek, wO));   // bins k and MC - k of the real row
            c32 Hk = ldg_c(Hrow + k), Hm = ldg_c(Hrow + (MC - k));
            Hk.x += dsk;
            Hm.x += dsk;
            const c32 Yk = mul(Xk, Hk), Ym = mul(Xm, Hm);
            const c32 Ye = mk(sc * (Yk.x + Ym.x), sc * (Yk.y - Ym.y));
            const c32 Yd = mk(sc * (Yk.x - Ym.x), sc * (Yk.y + Ym.y));
            const c32 Yo = mul(Yd, conj(w));
            v[q] = mk(Ye.x - Yo.y, Ye.y + Yo.x);             // Ye + i Yo
            if ((q & 3) == 3) asm volatile("" ::: "memory");  // bound load hoisting (register pressure)
        }
        __syncthreads();   // every mirror read done before the inverse reuses the buffer
        fft_mr3<P, +1>(v, buf, s, t, a.tw);
        // gate; positions >= L are cleared so the next order sees a zero-padded row
#pragma unroll
        for (int q = 0; q < E; ++q) {
            const int64_t pos = pos_of(q);
            c32 gq;
            if constexpr (PRE) gq = io<IO>::unpack(g[q]);
            else gq = active ? load_pair_s<IO, EVEN>(grow, pos, L, a.es) : mk(0.f, 0.f);
            v[q] = mk(pos < L ? gq.x * v[q].x : 0.f, pos + 1 < L ? gq.y * v[q].y : 0.f);
        }
    }
    if (active) {
        IO *yrow = reinterpret_cast<IO *>(a.y) + act_row_off(a, row);
#pragma unroll
        for (int q = 0; q < E; ++q) store_pair_s<IO, EVEN>(yrow, pos_of(q), L, a.es, v[q]);
    }
}

// Filter spectra for M = 6 P: Hout[o, k] = sum_t h[o, t] e^{-2 pi i k t / M}, k in [0, MC].
template <int P>
__global__ void __launch_bounds__(MR3<P>::THREADS, MR3<P>::MINB)
    hyena_spectrum_1d_mr3(const float *h, int64_t h_stride, int64_t L, c32 *Hout, int64_t nrows,
                          const c32 *__restrict__ tw) {
    using G = MR3<P>;
    constexpr int E = G::E, T = G::T, MC = G::MC, RPC = G::RPC;
    extern __shared__ float smem[];
    const int lrow = threadIdx.x / G::GT;
    const int gt = threadIdx.x - lrow * G::GT;
    const int s = gt / T, t = gt - s * T;
    const int64_t o = (int64_t)blockIdx.x * RPC + lrow;
    const bool active = o < nrows;
    float *buf = smem + lrow * G::SMEM_FLOATS;
    float *pre = buf, *pim = buf + MC;
    const float *hrow = h + (active ? o : 0) * h_stride;
    c32 v[E];
#pragma unroll
    for (int q = 0; q < E; ++q) {
        const int64_t pos = 2 * ((int64_t)P * s + t + q * T);
        v[q] = mk(active && pos < L ? hrow[pos] : 0.f, active && pos + 1 < L ? hrow[pos + 1] : 0.f);
    }
    // a row is read completely before the first barrier: in place (h == Hout) is allowed
    fft_mr3<P, -1>(v, buf, s, t, tw);
#pragma unroll
    for (int q = 0; q < E; ++q) {
        const int k = s + 3 * (t + q * T);
        pre[k] = v[q].x;
        pim[k] = v[q].y;
    }
    __syncthreads();
    c32 *Hrow = Hout + (active ? o : 0) * (MC + 1);
#pragma unroll
    for (int q = 0; q < E; ++q) {
        const int k = s + 3 * (t + q * T);
        const int km = (MC - k) % MC;
        const c32 Zk = v[q], Zm = mk(pre[km], pim[km]);
        const c32 Ek = mk(0.5f * (Zk.x + Zm.x), 0.5f * (Zk.y - Zm.y));
        const c32 Ok = mk(0.5f * (Zk.y + Zm.y), -0.5f * (Zk.x - Zm.x));
        if (active) {
            Hrow[k] = add(Ek, mul(ldg_c(tw + k), Ok));
            if (k == 0) Hrow[MC] = mk(Ek.x - Ok.x, 0.f);   // Nyquist bin: E_0 - O_0, real
        }
    }
}

}  // namespace hyena
