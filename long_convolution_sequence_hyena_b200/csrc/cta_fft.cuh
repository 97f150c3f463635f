// CTA-level complex FFT of length MC over registers + a shared-memory exchange
// buffer, and the real-input packing used by the 1D kernels.
//
// Real-input packing (standard "two reals in one complex" identity): a real
// row x of length M = 2*MC is carried as z[n] = x[2n] + i x[2n+1], n < MC.
// With Z = DFT_MC(z):
//   E[k] = (Z[k] + conj Z[MC-k]) / 2,  O[k] = (Z[k] - conj Z[MC-k]) / (2i)
//   X[k] = E[k] + W_M^k O[k],  X[MC-k] = conj(E[k] - W_M^k O[k])          (X = DFT_M(x))
// and back, for a spectrum Y of a real row y:
//   Z'[k] = (Y[k] + conj Y[MC-k]) / 2 + i (Y[k] - conj Y[MC-k]) conj(W_M^k) / 2
//   IDFT_MC(Z')[n] * (1/MC) = y[2n] + i y[2n+1].
#pragma once
#include "fft_regs.cuh"

namespace hyena {

// One Stockham pass p of a length-MC FFT (see fft_regs.cuh for the layout).
// tw: W_M^m = exp(-2 pi i m / M), m in [0, M), M = 2*MC (forward sign).
template <int MC, int E, int DIR, bool HALF_IN, int p>
__device__ __forceinline__ void fft_pass(c32 (&v)[E], float *__restrict__ sre, float *__restrict__ sim, int t,
                                         const c32 *__restrict__ tw) {
    constexpr int T = MC / E;
    constexpr int P = num_passes(MC);
    constexpr int R = pass_radix(MC, p);
    constexpr int NS = pass_stride(MC, p);
    constexpr int S = E / R;
    constexpr bool LAST = (p == P - 1);
    if constexpr (p > 0) {
        constexpr int NSP = pass_stride(MC, p - 1);
        __syncthreads();  // writes of pass p-1 visible
#pragma unroll
        for (int q = 0; q < E; ++q) {
            const int i = swz<NSP>(t + q * T);
            v[q] = mk(sre[i], sim[i]);
        }
        __syncthreads();  // every read done before pass p writes
    }
    static_for<S>([&](auto sc) {
        constexpr int s = decltype(sc)::value;
        const int j = t + s * T;
        const int k = j & (NS - 1);
        (void)k;
        if constexpr (NS > 1) {
            const float2 wf = __ldg(reinterpret_cast<const float2 *>(tw) + (size_t)k * (2 * MC / (NS * R)));
            twiddle_powers<R, S, s>(v, DIR > 0 ? mk(wf.x, -wf.y) : mk(wf.x, wf.y));
        }
        dftR<R, DIR, HALF_IN && p == 0, S, s>(v);
        if constexpr (!LAST) {
            const int base = (j / NS) * NS * R + k;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int i = swz<NS>(base + r * NS);
                sre[i] = v[s + r * S].x;
                sim[i] = v[s + r * S].y;
            }
        }
    });
    if constexpr (!LAST) fft_pass<MC, E, DIR, false, p + 1>(v, sre, sim, t, tw);
}

// Full length-MC FFT in place on v (natural order in and out).
// HALF_IN: registers q >= E/2 hold zeros on entry (zero-padded input).
// On return every smem read of this FFT is complete in all threads of the CTA
// (the last exchange ends with a barrier), unless the FFT has a single pass.
template <int MC, int E, int DIR, bool HALF_IN>
__device__ __forceinline__ void fft_cta(c32 (&v)[E], float *sre, float *sim, int t, const c32 *__restrict__ tw) {
    fft_pass<MC, E, DIR, HALF_IN, 0>(v, sre, sim, t, tw);
}

}  // namespace hyena
