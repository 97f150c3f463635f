// Block-level complex FFT of length LEN over registers + a shared-memory
// exchange buffer, used by every kernel of the library.
//
// Two shared-memory layouts:
//  * NSEQ == 0: one sequence per buffer, contiguous; the Stockham write
//    pattern is made bank-conflict-free by swz<NS>() (see fft_regs.cuh).
//  * NSEQ  > 0: NSEQ sequences, sequence-major, interleaved complex (one
//    8-byte float2 per element, in the buffer passed as `sre`; `sim` is
//    unused), element i of sequence s at maddr<LEN, NSEQ>(i, s). Warps span
//    the sequence index with a common i, so the XOR puts each half-warp on
//    distinct 8-byte bank pairs; and lanes that span 32 consecutive i of one
//    sequence touch one contiguous 256-byte block (what a remote,
//    distributed-shared-memory store wants).
//
// Twiddles come from one table of W_TWM^m = exp(-2 pi i m / TWM), m < TWM,
// with TWM a multiple of LEN.
//
// Real-input packing used by the 1D kernels (the standard identity that
// carries a real sequence as a complex one of half the length): a real row x
// of length M = 2*MC is carried as z[n] = x[2n] + i x[2n+1], n < MC. With
// Z = DFT_MC(z):
//   E[k] = (Z[k] + conj Z[MC-k]) / 2,  O[k] = (Z[k] - conj Z[MC-k]) / (2i)
//   X[k] = E[k] + W_M^k O[k],  X[MC-k] = conj(E[k] - W_M^k O[k])          (X = DFT_M(x))
// and back, for a spectrum Y of a real row y:
//   Z'[k] = (Y[k] + conj Y[MC-k]) / 2 + i (Y[k] - conj Y[MC-k]) conj(W_M^k) / 2
//   IDFT_MC(Z')[n] * (1/MC) = y[2n] + i y[2n+1].
#pragma once
#include "fft_regs.cuh"

namespace hyena {

// Sequence-major address of element i of sequence s (sequences of length LEN >= 32).
// NSW: the number of sequences a warp spans at a common i. With 16 or more,
// each half-warp holds 16 sequences and XOR-ing the sequence index into i
// puts them on distinct 8-byte bank pairs. With 8, each half-warp holds 8
// sequences at two elements i, i' that differ in one bit among bits 0..4
// (every Stockham pattern of radix-8 and radix-16 passes): XOR-ing 2s into
// bits 1..3 and the parity of bits 1..4 of i into bit 0 separates them
// (checked on the CPU for lengths 64..512).
template <int LEN, int NSW = 32>
__device__ __forceinline__ int maddr(int i, int s) {
    static_assert(NSW == 8 || NSW >= 16, "sequence-major layout needs 8 or at least 16 sequences per warp");
    if constexpr (NSW >= 16) return s * LEN + (i ^ (s & 31));
    else return s * LEN + (i ^ (((2 * s) & 15) | (__popc((i >> 1) & 15) & 1)));
}

// Shared-memory element of a value type in the sequence-major layout: one
// 8-byte float2 per complex value, one 16-byte float4 (re a, re b, im a, im b)
// per pair of complex values.
template <typename V>
struct selem;
template <>
struct selem<c32> {
    using T = float2;
    __device__ __forceinline__ static c32 ld(const float2 &f) { return mk(f.x, f.y); }
    __device__ __forceinline__ static float2 st(c32 v) { return make_float2(v.x, v.y); }
};
template <>
struct selem<c32x2> {
    using T = float4;
    __device__ __forceinline__ static c32x2 ld(const float4 &f) { return c32x2{f2(f.x, f.y), f2(f.z, f.w)}; }
    __device__ __forceinline__ static float4 st(c32x2 v) { return make_float4(v.re.x, v.re.y, v.im.x, v.im.y); }
};

// Exchange address of element i. Sequence-major layouts with 16-byte
// elements (lockstep pairs) are read and written a quarter-warp (8 lanes) at
// a time; with 8 or more sequences per warp at a common i, the plain XOR of
// the sequence index already spreads those 8 over distinct 16-byte bank groups.
template <int NS, int NSEQ, int LEN, int EB = 8>
__device__ __forceinline__ int saddr(int i, int seq) {
    if constexpr (NSEQ == 0) return swz<NS>(i);
    else if constexpr (EB == 16) return maddr<LEN, 32>(i, seq);
    else return maddr<LEN, NSEQ>(i, seq);
}

// One Stockham pass p of a length-LEN FFT (register layout in fft_regs.cuh).
// V is c32, or c32x2 (two sequences in lockstep, sequence-major layout only).
template <int LEN, int E, int DIR, bool HALF_IN, int p, int TWM, int NSEQ, typename V>
__device__ __forceinline__ void fft_pass(V (&v)[E], float *__restrict__ sre, float *__restrict__ sim, int t,
                                         int seq, const c32 *__restrict__ tw) {
    using SE = selem<V>;
    constexpr int EB = (int)sizeof(typename SE::T);
    static_assert(NSEQ > 0 || sizeof(V) == sizeof(c32), "lockstep pairs need the sequence-major layout");
    static_assert(EB == 8 || NSEQ >= 8, "16-byte elements need at least 8 sequences per warp");
    constexpr int T = LEN / E;
    constexpr int LR = pass_lr(E);
    constexpr int P = num_passes(LEN, LR);
    constexpr int R = pass_radix(LEN, p, LR);
    constexpr int NS = pass_stride(LEN, p, LR);
    static_assert(NSEQ > 0 || LR == 4, "the contiguous swizzled layout assumes radix-16 passes");
    constexpr int S = E / R;
    constexpr bool LAST = (p == P - 1);
    static_assert(TWM % LEN == 0, "twiddle table must cover the transform");
    if constexpr (p > 0) {
        constexpr int NSP = pass_stride(LEN, p - 1, LR);
        __syncthreads();  // writes of pass p-1 visible
#pragma unroll
        for (int q = 0; q < E; ++q) {
            const int i = saddr<NSP, NSEQ, LEN, EB>(t + q * T, seq);
            if constexpr (NSEQ > 0) {
                v[q] = SE::ld(reinterpret_cast<const typename SE::T *>(sre)[i]);
            } else {
                v[q] = mk(sre[i], sim[i]);
            }
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
                const int i = saddr<NS, NSEQ, LEN, EB>(base + r * NS, seq);
                if constexpr (NSEQ > 0) {
                    reinterpret_cast<typename SE::T *>(sre)[i] = SE::st(v[s + r * S]);
                } else {
                    sre[i] = v[s + r * S].x;
                    sim[i] = v[s + r * S].y;
                }
            }
        }
    });
    if constexpr (!LAST) fft_pass<LEN, E, DIR, false, p + 1, TWM, NSEQ>(v, sre, sim, t, seq, tw);
}

// Full length-LEN FFT in place on v (natural order in and out).
// HALF_IN: registers q >= E/2 hold zeros on entry (zero-padded input).
// When the FFT has more than one pass, every shared-memory read it makes is
// complete in all threads of the block on return (the last exchange ends with
// a barrier).
template <int LEN, int E, int DIR, bool HALF_IN, int TWM = 2 * LEN, int NSEQ = 0, typename V>
__device__ __forceinline__ void fft_cta(V (&v)[E], float *sre, float *sim, int t, const c32 *__restrict__ tw,
                                        int seq = 0) {
    fft_pass<LEN, E, DIR, HALF_IN, 0, TWM, NSEQ>(v, sre, sim, t, seq, tw);
}

}  // namespace hyena
