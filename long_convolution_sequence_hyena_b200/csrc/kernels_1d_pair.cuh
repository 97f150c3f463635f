// 1D fused order-N forward for two rows of one channel per thread group.
//
// Rows (b, d) and (b+1, d) share the filter, the feedthrough and every
// twiddle, so one thread group carries both in lockstep as packed fp32x2
// values (c32x2): every butterfly add, every multiply and every shared-memory
// access is one instruction for the two rows, and the spectrum row is staged
// once for both. The algorithm is the one of hyena_fwd_1d_cta (real-input
// packing into a half-length complex FFT, radix-16 Stockham passes, spectral
// step with the feedthrough as a constant gain, inverse, gate), applied lane
// by lane.
#pragma once
#include "kernels_1d.cuh"

namespace hyena {

// Swizzle of the pair exchange buffer (8-byte words): within every half-warp
// the 16 lanes hit 16 distinct 8-byte bank pairs for the consecutive reads and
// for the Stockham write patterns of every pass (checked on the CPU for
// MC = 256..8192). It only permutes within aligned blocks of 16 words.
__device__ __forceinline__ int swz2(int i) { return i ^ ((i >> 4) & 15); }

template <int LEN, int E, int DIR, bool HALF_IN, int p>
__device__ __forceinline__ void fft_pass_x2(c32x2 (&v)[E], float2 *__restrict__ sre, float2 *__restrict__ sim, int t,
                                            const c32 *__restrict__ tw) {
    constexpr int T = LEN / E;
    constexpr int P = num_passes(LEN);
    constexpr int R = pass_radix(LEN, p);
    constexpr int NS = pass_stride(LEN, p);
    constexpr int S = E / R;
    constexpr bool LAST = (p == P - 1);
    constexpr int TWM = 2 * LEN;
    if constexpr (p > 0) {
        __syncthreads();  // writes of pass p-1 visible
#pragma unroll
        for (int q = 0; q < E; ++q) {
            const int i = swz2(t + q * T);
            v[q] = c32x2{sre[i], sim[i]};
        }
        __syncthreads();  // every read done before pass p writes
    }
    static_for<S>([&](auto sc) __attribute__((always_inline)) {
        constexpr int s = decltype(sc)::value;
        const int j = t + s * T;
        const int k = j & (NS - 1);
        (void)k;
        if constexpr (NS > 1) {
            const float2 wf = __ldg(reinterpret_cast<const float2 *>(tw) + (size_t)k * (TWM / (NS * R)));
            twiddle_powers<R, S, s>(v, DIR > 0 ? mk(wf.x, -wf.y) : mk(wf.x, wf.y));
        }
        dftR<R, DIR, HALF_IN && p == 0, S, s>(v);
        if constexpr (!LAST) {
            const int base = (j / NS) * NS * R + k;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int i = swz2(base + r * NS);
                sre[i] = v[s + r * S].re;
                sim[i] = v[s + r * S].im;
            }
        }
    });
    if constexpr (!LAST) fft_pass_x2<LEN, E, DIR, false, p + 1>(v, sre, sim, t, tw);
}

// Length-LEN FFT of two rows in lockstep (natural order in and out; the
// table is W_{2 LEN}, the plan's table for M = 2 LEN).
template <int LEN, int E, int DIR, bool HALF_IN>
__device__ __forceinline__ void fft_cta_x2(c32x2 (&v)[E], float2 *sre, float2 *sim, int t,
                                           const c32 *__restrict__ tw) {
    fft_pass_x2<LEN, E, DIR, HALF_IN, 0>(v, sre, sim, t, tw);
}

// Spectral step for both rows (see spectral_product in kernels_1d.cuh). The
// unpacking is written without its factors 1/2; those and the 1/MC of the
// inverse are folded into the (shared) filter gain.
//
// Bins k and MC - k need the same intermediates: with A = Y[k], B = Y[MC-k],
// Ye ~ A + conj B and Yo ~ (A - conj B) conj(W_M^k), the packed inverse input
// is Ye + i Yo at k and conj(Ye - i Yo) at MC - k (W_M^{MC-k} = -conj W_M^k).
// Each thread therefore takes its bins k = t + qT with q < E/2 (thread 0 also
// k = MC/2, its own mirror) and produces both outputs; the mirror outputs
// reach their owners (thread T - t, register E-1-q) through shared memory.
template <int MC, int E>
__device__ __forceinline__ void spectral_product_x2(c32x2 (&v)[E], float2 *__restrict__ sre,
                                                    float2 *__restrict__ sim, int t, const c32 *Hs, float dsk,
                                                    c32 wt) {
    constexpr int T = MC / E;
#pragma unroll
    for (int q = 0; q < E; ++q) {
        sre[t + q * T] = v[q].re;
        sim[t + q * T] = v[q].im;
    }
    cp_async_wait_all();
    __syncthreads();
    constexpr float s = 0.25f / (float)MC;
    const int z0 = opaque_zero();
    // Ye and Yo of bin k from Z[k] (register) and Z[MC-k] (shared memory)
    auto bin_pair = [&](int q, c32x2 Zk, c32x2 &Ye, c32x2 &Yo) __attribute__((always_inline)) {
        const int k = t + q * T;
        const int km = (MC - k) & (MC - 1);
        const float2 mre = sre[km], mim = sim[km];
        // 2E = Zk + conj Zm, 2O = (Zk - conj Zm) / i
        const c32x2 E2{f2add(Zk.re, mre), f2sub(Zk.im, mim)};
        const c32x2 O2{f2add(Zk.im, mim), f2sub(mre, Zk.re)};
        const c32 w = mul(wt, w2e<E>(q, z0));          // W_M^{t + qT}
        const c32x2 wO = mul(O2, w);
        const c32x2 Xk = add(E2, wO);                   // 2 X[k]
        const c32x2 Xm{f2sub(E2.re, wO.re), f2sub(wO.im, E2.im)};   // 2 X[MC-k] = conj(2E - 2wO)
        c32 Hk = Hs[k], Hm = Hs[MC - k];
        Hk = mk(s * (Hk.x + dsk), s * Hk.y);
        Hm = mk(s * (Hm.x + dsk), s * Hm.y);
        const c32x2 Yk = mul(Xk, Hk), Ym = mul(Xm, Hm);
        Ye = c32x2{f2add(Yk.re, Ym.re), f2sub(Yk.im, Ym.im)};   // Yk + conj Ym
        const c32x2 Yd{f2sub(Yk.re, Ym.re), f2add(Yk.im, Ym.im)};   // Yk - conj Ym
        Yo = mul(Yd, conj(w));
    };
    c32x2 vh = v[E / 2];
    if (t == 0) {   // k = MC/2 is its own mirror
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
    }
    __syncthreads();   // every mirror read done
#pragma unroll
    for (int q = 0; q < E / 2; ++q) {
        const int km = (MC - (t + q * T)) & (MC - 1);
        sre[km] = v[E / 2 + q].re;
        sim[km] = v[E / 2 + q].im;
    }
    __syncthreads();
#pragma unroll
    for (int q = E / 2; q < E; ++q) {
        const int k = t + q * T;
        v[q] = c32x2{sre[k], sim[k]};
    }
    if (t == 0) v[E / 2] = vh;
    __syncthreads();
}

constexpr int pair_pairs_per_cta(int MC, int E) { return (MC / E) >= 128 ? 1 : 128 / (MC / E); }
constexpr int pair_threads(int MC, int E) { return pair_pairs_per_cta(MC, E) * (MC / E); }
// Resident CTAs per SM the register budget is sized for (128 threads: 3 -> 168
// registers; 256 threads: 2 -> 128; 512 threads: 1 -> 128).
#ifndef HYENA_PAIR_MINB_128
#define HYENA_PAIR_MINB_128 3
#endif
constexpr int pair_min_blocks(int MC, int E) {
    return pair_threads(MC, E) >= 512 ? 1 : (pair_threads(MC, E) >= 256 ? 2 : HYENA_PAIR_MINB_128);
}
// Shared bytes per row pair: exchange buffer (two float2 planes) + staged spectrum row.
// (rounded up to 16 bytes so every pair's region, and the gate stage after
// them, start 16-byte aligned)
constexpr size_t pair_smem_bytes_per_pair(int MC) { return ((size_t)MC * 16 + (size_t)(MC + 1) * 8 + 15) & ~(size_t)15; }
// Staging for one order's gates of both rows (E/2 element pairs per row and thread).
template <typename IO>
constexpr size_t pair_gate_stage_bytes(int MC, int E) {
    return (size_t)pair_threads(MC, E) * E * sizeof(typename io<IO>::pair_t);
}
// Gates are staged in shared memory (freeing registers) when the row length
// is even and the stage fits next to the buffers.
template <typename IO, bool EVEN>
constexpr bool pair_stage_gates(int MC, int E) {
    return EVEN && pair_pairs_per_cta(MC, E) * pair_smem_bytes_per_pair(MC) + pair_gate_stage_bytes<IO>(MC, E) <=
                       227 * 1024;
}
template <typename IO, bool EVEN>
constexpr size_t pair_smem_bytes(int MC, int E) {
    return pair_pairs_per_cta(MC, E) * pair_smem_bytes_per_pair(MC) +
           (pair_stage_gates<IO, EVEN>(MC, E) ? pair_gate_stage_bytes<IO>(MC, E) : 0);
}

// Fused order-N forward, one group of MC/E threads per pair of rows
// (b, d), (b+1, d); B must be even. Pairs are visited d-major so the B/2
// pairs that read the same spectrum row run together. NORD > 0 fixes the
// order at compile time (the chain is unrolled); NORD = 0 reads it from the
// arguments.
template <int MC, int E, typename IO, bool EVEN, int NORD>
__global__ void __launch_bounds__(pair_threads(MC, E), pair_min_blocks(MC, E))
    hyena_fwd_1d_pair(const Fwd1dArgs a) {
    constexpr int T = MC / E;
    constexpr int PPC = pair_pairs_per_cta(MC, E);
    extern __shared__ float4 smem4[];
    const int lp = threadIdx.x / T;
    const int t = threadIdx.x - lp * T;
    const int64_t npairs = a.rows / 2;
    const int64_t pidx = (int64_t)blockIdx.x * PPC + lp;
    const bool in_grid = pidx < npairs;
    const int64_t hb = a.B / 2;
    const int64_t d = in_grid ? pidx / hb : 0;
    const int64_t b0 = in_grid ? 2 * (pidx - d * hb) : 0;
    const int64_t row0 = b0 * a.D + d, row1 = row0 + a.D;
    const bool active = in_grid && check_index(a.err, row0, a.rows) && check_index(a.err, row1, a.rows) &&
                        check_index(a.err, d, a.D);
    unsigned char *base = reinterpret_cast<unsigned char *>(smem4) + lp * pair_smem_bytes_per_pair(MC);
    float2 *sre = reinterpret_cast<float2 *>(base);
    float2 *sim = sre + MC;
    c32 *Hs = reinterpret_cast<c32 *>(sim + MC);
    const int64_t L = a.L;
    const c32 wt = ldg_c(a.tw + t);                       // W_M^t

    c32x2 v[E];
    {
        const IO *r0 = reinterpret_cast<const IO *>(a.v) + row0 * L;
        const IO *r1 = reinterpret_cast<const IO *>(a.v) + row1 * L;
#pragma unroll
        for (int q = 0; q < E / 2; ++q) {
            const int64_t pos = 2 * (int64_t)(t + q * T);
            const c32 x0 = active ? load_pair<IO, EVEN>(r0, pos, L) : mk(0.f, 0.f);
            const c32 x1 = active ? load_pair<IO, EVEN>(r1, pos, L) : mk(0.f, 0.f);
            v[q] = c32x2{f2(x0.x, x1.x), f2(x0.y, x1.y)};
        }
#pragma unroll
        for (int q = E / 2; q < E; ++q) v[q] = c32x2{f2(0.f, 0.f), f2(0.f, 0.f)};
    }

    using P = typename io<IO>::pair_t;
    constexpr bool GST = pair_stage_gates<IO, EVEN>(MC, E);
    constexpr int NT = pair_threads(MC, E);
    P *gst = reinterpret_cast<P *>(reinterpret_cast<unsigned char *>(smem4) + PPC * pair_smem_bytes_per_pair(MC)) +
             threadIdx.x;   // thread-private slots gst[(2 q + row) * NT]
    const int norder = NORD > 0 ? NORD : a.order;
#pragma unroll
    for (int n = 0; n < norder; ++n) {   // unrolled only when the order is a constant
        const IO *g0 = reinterpret_cast<const IO *>(a.gates[n]) + row0 * L;
        const IO *g1 = reinterpret_cast<const IO *>(a.gates[n]) + row1 * L;
        P ga[GST ? 1 : E / 2], gb[GST ? 1 : E / 2];
        if constexpr (GST) {   // staged while the transforms run
#pragma unroll
            for (int q = 0; q < E / 2; ++q) {
                const int64_t pos = 2 * (int64_t)(t + q * T);
                if (active && pos < L) {
                    cp_async_n<sizeof(P)>(gst + (2 * q) * NT, g0 + pos);
                    cp_async_n<sizeof(P)>(gst + (2 * q + 1) * NT, g1 + pos);
                } else {
                    gst[(2 * q) * NT] = io<IO>::zero();
                    gst[(2 * q + 1) * NT] = io<IO>::zero();
                }
            }
        } else {
#pragma unroll
            for (int q = 0; q < E / 2; ++q) {
                const int64_t pos = 2 * (int64_t)(t + q * T);
                ga[q] = active ? load_pair_raw<IO, EVEN>(g0, pos, L) : io<IO>::zero();
                gb[q] = active ? load_pair_raw<IO, EVEN>(g1, pos, L) : io<IO>::zero();
            }
        }
        const int64_t hrow = check_index(a.err, (int64_t)n * a.hD + d, (int64_t)a.order * a.hD) ? n * a.hD + d : 0;
        const float dsk = a.dskip ? __ldg(a.dskip + hrow) : 0.f;
        const c32 *Hrow = a.H + hrow * (MC + 1);
        for (int i = t; i <= MC; i += T) cp_async8(Hs + i, Hrow + i);   // staged while the FFT runs
        cp_async_commit();

        // With 128 registers (256 threads and more), each stage takes its own
        // opaque copy of the thread index, so that the compiler recomputes the
        // stage's shared-memory addresses and twiddle indices instead of
        // keeping them live across the whole chain (which spills; ptxas -v).
        constexpr bool OPQ = pair_threads(MC, E) >= 256;
        int tf = t, ts = t, ti = t;
        if constexpr (OPQ) asm volatile("" : "+r"(tf));
        fft_cta_x2<MC, E, -1, true>(v, sre, sim, tf, a.tw);
        if constexpr (OPQ) asm volatile("" : "+r"(ts));
        spectral_product_x2<MC, E>(v, sre, sim, ts, Hs, dsk, wt);
        if constexpr (OPQ) asm volatile("" : "+r"(ti));
        fft_cta_x2<MC, E, +1, false>(v, sre, sim, ti, a.tw);

        // gate; positions >= L are cleared so the next order sees a zero-padded row
#pragma unroll
        for (int q = 0; q < E / 2; ++q) {
            const int64_t pos = 2 * (int64_t)(t + q * T);
            const c32 ca = io<IO>::unpack(GST ? gst[(2 * q) * NT] : ga[q]);
            const c32 cb = io<IO>::unpack(GST ? gst[(2 * q + 1) * NT] : gb[q]);
            const bool in0 = pos < L, in1 = pos + 1 < L;
            v[q] = c32x2{in0 ? f2mul(v[q].re, f2(ca.x, cb.x)) : f2(0.f, 0.f),
                         in1 ? f2mul(v[q].im, f2(ca.y, cb.y)) : f2(0.f, 0.f)};
        }
#pragma unroll
        for (int q = E / 2; q < E; ++q) v[q] = c32x2{f2(0.f, 0.f), f2(0.f, 0.f)};
    }

    if (active) {
        IO *y0 = reinterpret_cast<IO *>(a.y) + row0 * L;
        IO *y1 = reinterpret_cast<IO *>(a.y) + row1 * L;
#pragma unroll
        for (int q = 0; q < E / 2; ++q) {
            const int64_t pos = 2 * (int64_t)(t + q * T);
            store_pair<IO, EVEN>(y0, pos, L, mk(v[q].re.x, v[q].im.x));
            store_pair<IO, EVEN>(y1, pos, L, mk(v[q].re.y, v[q].im.y));
        }
    }
}

}  // namespace hyena

