// 1D kernels: the fused order-N forward (one CTA group per channel row) and the
// filter spectrum. Launch wrappers are declared in launch.h.
#pragma once
#include <cuda_bf16.h>

#include "check.cuh"
#include "cta_fft.cuh"
#include "hyena.h"

namespace hyena {

struct Fwd1dArgs {
    const void *v;
    const void *gates[HYENA_MAX_ORDER];
    const c32 *H;         // row (n, d) at H + (n hD + d) (MC + 1)
    const float *dskip;   // Dskip^n_d at dskip[n hD + d], or nullptr
    void *y;
    const c32 *tw;        // W_M^m, m in [0, M)
    int64_t rows;         // B * D
    int64_t L;
    int64_t D;
    int64_t B;
    int order;
    // channels between consecutive orders' rows of H and entries of dskip: D, or
    // the plan's channel count when a call covers a sub-range of the channels
    // (H and dskip then point at the range's first channel)
    int64_t hD;
    int *err;             // the plan's device error word (index checks of the debug build)
    // activation layout: es = 1 for [B, D, L] (a channel row is contiguous);
    // es = D for channels-last [B, L, D] (consecutive positions of a row are D
    // elements apart, and channel d of batch element b starts at b L D + d)
    int64_t es;
};

// Offset (elements) of flat row b * D + d in an activation tensor.
__device__ __forceinline__ int64_t act_row_off(const Fwd1dArgs &a, int64_t row) {
    if (a.es == 1) return row * a.L;
    const int64_t b = row / a.D;
    return b * a.L * a.D + (row - b * a.D);
}

constexpr int rows_per_cta(int MC, int E) { return (MC / E) >= 128 ? 1 : 128 / (MC / E); }

// ---- activation I/O: element pairs (x[2k], x[2k+1]) as one complex value ----
template <typename IO>
struct io;

template <>
struct io<float> {
    using pair_t = float2;
    __device__ __forceinline__ static c32 unpack(pair_t p) { return mk(p.x, p.y); }
    __device__ __forceinline__ static pair_t pack(c32 a) { return make_float2(a.x, a.y); }
    __device__ __forceinline__ static float to_f(float a) { return a; }
    __device__ __forceinline__ static float from_f(float a) { return a; }
    __device__ __forceinline__ static pair_t zero() { return make_float2(0.f, 0.f); }
};

template <>
struct io<__nv_bfloat16> {
    using pair_t = __nv_bfloat162;
    __device__ __forceinline__ static c32 unpack(pair_t p) {
        const float2 f = __bfloat1622float2(p);
        return mk(f.x, f.y);
    }
    __device__ __forceinline__ static pair_t pack(c32 a) { return __floats2bfloat162_rn(a.x, a.y); }
    __device__ __forceinline__ static float to_f(__nv_bfloat16 a) { return __bfloat162float(a); }
    __device__ __forceinline__ static __nv_bfloat16 from_f(float a) { return __float2bfloat16_rn(a); }
    __device__ __forceinline__ static pair_t zero() { return __floats2bfloat162_rn(0.f, 0.f); }
};

// SiLU(x) = x σ(x) = x / (1 + e^{-x}) for the gate sandwich of HyenaND
// ("How HyenaND works", "Putting it together: the HyenaND operator"), with the
// fast exponential and divide (a few ulp, far inside the fp32 tolerance). The
// exponent is clamped at 80 so that the divisor stays below 2^126, where the
// fast divide is defined; below x = -80 the result is x / (1 + e^80), whose
// magnitude is under 1e-32 (the exact value is smaller still).
__device__ __forceinline__ float silu(float x) { return __fdividef(x, 1.f + __expf(fminf(-x, 80.f))); }
__device__ __forceinline__ c32 silu(c32 a) { return mk(silu(a.x), silu(a.y)); }

// Load positions (pos, pos+1) of a row of length L, zero beyond L.
// EVEN: L is even, so the pair is either fully inside or fully outside and the
// pair load is aligned.
template <typename IO, bool EVEN>
__device__ __forceinline__ c32 load_pair(const IO *__restrict__ row, int64_t pos, int64_t L) {
    if constexpr (EVEN) {
        if (pos < L) return io<IO>::unpack(__ldg(reinterpret_cast<const typename io<IO>::pair_t *>(row + pos)));
        return mk(0.f, 0.f);
    } else {
        const float a = pos < L ? io<IO>::to_f(row[pos]) : 0.f;
        const float b = pos + 1 < L ? io<IO>::to_f(row[pos + 1]) : 0.f;
        return mk(a, b);
    }
}

// Raw (still packed) pair for prefetching: one register per pair in bf16.
template <typename IO, bool EVEN>
__device__ __forceinline__ typename io<IO>::pair_t load_pair_raw(const IO *__restrict__ row, int64_t pos, int64_t L) {
    using P = typename io<IO>::pair_t;
    if constexpr (EVEN) {
        if (pos < L) return __ldg(reinterpret_cast<const P *>(row + pos));
        return io<IO>::zero();
    } else {
        const c32 c = load_pair<IO, false>(row, pos, L);
        return io<IO>::pack(c);
    }
}

template <typename IO, bool EVEN>
__device__ __forceinline__ void store_pair(IO *__restrict__ row, int64_t pos, int64_t L, c32 val) {
    if constexpr (EVEN) {
        if (pos < L) *reinterpret_cast<typename io<IO>::pair_t *>(row + pos) = io<IO>::pack(val);
    } else {
        if (pos < L) row[pos] = io<IO>::from_f(val.x);
        if (pos + 1 < L) row[pos + 1] = io<IO>::from_f(val.y);
    }
}

// The same accesses for a row whose consecutive positions are es elements
// apart (es = 1: the contiguous forms above; channels-last: one element each).
template <typename IO, bool EVEN>
__device__ __forceinline__ c32 load_pair_s(const IO *__restrict__ row, int64_t pos, int64_t L, int64_t es) {
    if (es == 1) return load_pair<IO, EVEN>(row, pos, L);
    const float x0 = pos < L ? io<IO>::to_f(row[pos * es]) : 0.f;
    const float x1 = pos + 1 < L ? io<IO>::to_f(row[(pos + 1) * es]) : 0.f;
    return mk(x0, x1);
}
template <typename IO, bool EVEN>
__device__ __forceinline__ typename io<IO>::pair_t load_pair_raw_s(const IO *__restrict__ row, int64_t pos, int64_t L,
                                                                    int64_t es) {
    if (es == 1) return load_pair_raw<IO, EVEN>(row, pos, L);
    return io<IO>::pack(load_pair_s<IO, EVEN>(row, pos, L, es));
}
template <typename IO, bool EVEN>
__device__ __forceinline__ void store_pair_s(IO *__restrict__ row, int64_t pos, int64_t L, int64_t es, c32 val) {
    if (es == 1) return store_pair<IO, EVEN>(row, pos, L, val);
    if (pos < L) row[pos * es] = io<IO>::from_f(val.x);
    if (pos + 1 < L) row[(pos + 1) * es] = io<IO>::from_f(val.y);
}

__device__ __forceinline__ c32 ldg_c(const c32 *p) {
    const float2 f = __ldg(reinterpret_cast<const float2 *>(p));
    return mk(f.x, f.y);
}

// Asynchronous 8-byte global -> shared copy (bypasses registers).
__device__ __forceinline__ void cp_async8(void *smem_dst, const void *gmem_src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"((uint32_t)__cvta_generic_to_shared(smem_dst)),
                 "l"(gmem_src)
                 : "memory");
}
template <int BYTES>
__device__ __forceinline__ void cp_async_n(void *smem_dst, const void *gmem_src) {
    static_assert(BYTES == 4 || BYTES == 8 || BYTES == 16, "cp.async size");
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"((uint32_t)__cvta_generic_to_shared(smem_dst)),
                 "l"(gmem_src), "n"(BYTES)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Whether the fused CTA kernel stages each order's spectrum row in shared
// memory (it must fit next to the exchange buffer).
constexpr bool stage_spectrum(int MC) { return MC <= 8192; }
constexpr int fwd_threads(int MC, int E) { return rows_per_cta(MC, E) * (MC / E); }
constexpr int fwd_min_blocks(int MC, int E) {
    return fwd_threads(MC, E) >= 512 ? 1 : (fwd_threads(MC, E) >= 256 ? 2 : 4);
}
// Shared floats per row: exchange buffer (re, im planes) + staged spectrum row.
constexpr int fwd_smem_floats_per_row(int MC) { return 2 * MC + (stage_spectrum(MC) ? 2 * (MC + 1) : 0); }

// Spectral step of one order for a row held as packed complex spectrum Z
// (natural order in registers): unpack the real-row spectrum X, multiply by
// the filter gain plus the feedthrough (the feedthrough is the delta tap, whose
// spectrum is the constant Dskip), repack for the half-length inverse, and fold
// in the 1/2 of the repacking and the 1/MC of the inverse transform.
// Hs: the spectrum row staged in shared memory (cp.async group pending), or
// nullptr to read Hrow from global memory. wt = W_M^t.
//
// Bins k and MC - k need the same intermediates: with A = Y[k], B = Y[MC-k],
// Ye = (A + conj B)/2 and Yo = (A - conj B) conj(W_M^k)/2, the packed inverse
// input is Ye + i Yo at k and conj(Ye - i Yo) at MC - k (W_M^{MC-k} =
// -conj W_M^k). Each thread takes its bins k = t + qT with q < E/2 (thread 0
// also k = MC/2, its own mirror) and produces both; the mirror outputs reach
// their owners (thread T - t, register E-1-q) through shared memory.
template <int MC, int E>
__device__ __forceinline__ void spectral_product(c32 (&v)[E], float *__restrict__ sre, float *__restrict__ sim,
                                                 int t, const c32 *__restrict__ Hrow, const c32 *Hs, float dsk,
                                                 c32 wt) {
    constexpr int T = MC / E;
#pragma unroll
    for (int q = 0; q < E; ++q) {
        sre[t + q * T] = v[q].x;
        sim[t + q * T] = v[q].y;
    }
    if (Hs) cp_async_wait_all();
    __syncthreads();
    constexpr float s = 0.5f / (float)MC;
    const int z0 = opaque_zero();
    auto bin_pair = [&](int q, c32 Zk, c32 &Ye, c32 &Yo) __attribute__((always_inline)) {
        const int k = t + q * T;
        const int km = (MC - k) & (MC - 1);
        const c32 Zm = mk(sre[km], sim[km]);
        const c32 Ek = mk(0.5f * (Zk.x + Zm.x), 0.5f * (Zk.y - Zm.y));
        const c32 Ok = mk(0.5f * (Zk.y + Zm.y), -0.5f * (Zk.x - Zm.x));
        const c32 w = mul(wt, w2e<E>(q, z0));            // W_M^{t + qT} = W_M^t W_{2E}^q
        const c32 wO = mul(w, Ok);
        const c32 Xk = add(Ek, wO);
        const c32 Xm = conj(sub(Ek, wO));
        c32 Hk = Hs ? Hs[k] : ldg_c(Hrow + k);
        c32 Hm = Hs ? Hs[MC - k] : ldg_c(Hrow + (MC - k));
        Hk.x += dsk;
        Hm.x += dsk;
        const c32 Yk = mul(Xk, Hk), Ym = mul(Xm, Hm);
        Ye = mk(s * (Yk.x + Ym.x), s * (Yk.y - Ym.y));
        const c32 Yd = mk(s * (Yk.x - Ym.x), s * (Yk.y + Ym.y));
        Yo = mul(Yd, conj(w));
    };
    c32 vh = v[E / 2];
    if (t == 0) {   // k = MC/2 is its own mirror
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
    __syncthreads();   // every mirror read done
#pragma unroll
    for (int q = 0; q < E / 2; ++q) {
        const int km = (MC - (t + q * T)) & (MC - 1);
        sre[km] = v[E / 2 + q].x;
        sim[km] = v[E / 2 + q].y;
    }
    __syncthreads();
#pragma unroll
    for (int q = E / 2; q < E; ++q) {
        const int k = t + q * T;
        v[q] = mk(sre[k], sim[k]);
    }
    if (t == 0) v[E / 2] = vh;
    __syncthreads();
}

// Fused order-N forward, one group of MC/E threads per channel row.
// Grid: ceil(B*D / rows_per_cta) CTAs, rows visited d-major / b-minor so the B
// rows that read the same filter spectrum run at the same time (L2 reuse).
template <int MC, int E, typename IO, bool EVEN>
__global__ void __launch_bounds__(fwd_threads(MC, E), fwd_min_blocks(MC, E))
    hyena_fwd_1d_cta(const Fwd1dArgs a) {
    constexpr int T = MC / E;
    constexpr int RPC = rows_per_cta(MC, E);
    constexpr bool HS = stage_spectrum(MC);
    extern __shared__ float smem[];
    const int lrow = threadIdx.x / T;
    const int t = threadIdx.x - lrow * T;
    const int64_t ord = (int64_t)blockIdx.x * RPC + lrow;
    const bool in_grid = ord < a.rows;
    const int64_t d = in_grid ? ord / a.B : 0;
    const int64_t b = in_grid ? ord - d * a.B : 0;
    const int64_t row = b * a.D + d;
    const bool active = in_grid && check_index(a.err, row, a.rows) && check_index(a.err, d, a.D);
    float *sre = smem + lrow * fwd_smem_floats_per_row(MC);
    float *sim = sre + MC;
    c32 *Hs = HS ? reinterpret_cast<c32 *>(sim + MC) : nullptr;
    const int64_t L = a.L;
    const c32 wt = ldg_c(a.tw + t);                       // W_M^t

    c32 v[E];
    {
        const IO *vrow = reinterpret_cast<const IO *>(a.v) + act_row_off(a, row);
#pragma unroll
        for (int q = 0; q < E / 2; ++q)
            v[q] = active ? load_pair_s<IO, EVEN>(vrow, 2 * (int64_t)(t + q * T), L, a.es) : mk(0.f, 0.f);
#pragma unroll
        for (int q = E / 2; q < E; ++q) v[q] = mk(0.f, 0.f);
    }

    for (int n = 0; n < a.order; ++n) {
        const IO *grow = reinterpret_cast<const IO *>(a.gates[n]) + act_row_off(a, row);
        typename io<IO>::pair_t g[E / 2];
#pragma unroll
        for (int q = 0; q < E / 2; ++q)
            g[q] = active ? load_pair_raw_s<IO, EVEN>(grow, 2 * (int64_t)(t + q * T), L, a.es) : io<IO>::zero();
        const int64_t hrow = check_index(a.err, (int64_t)n * a.hD + d, (int64_t)a.order * a.hD) ? n * a.hD + d : 0;
        const float dsk = a.dskip ? __ldg(a.dskip + hrow) : 0.f;
        const c32 *Hrow = a.H + hrow * (MC + 1);
        if constexpr (HS) {  // stage the spectrum row while the forward FFT runs
            for (int i = t; i <= MC; i += T) cp_async8(Hs + i, Hrow + i);
            cp_async_commit();
        }

        fft_cta<MC, E, -1, true>(v, sre, sim, t, a.tw);
        spectral_product<MC, E>(v, sre, sim, t, Hrow, Hs, dsk, wt);
        fft_cta<MC, E, +1, false>(v, sre, sim, t, a.tw);

        // gate; positions >= L are cleared so the next order sees a zero-padded row
#pragma unroll
        for (int q = 0; q < E / 2; ++q) {
            const int64_t pos = 2 * (int64_t)(t + q * T);
            const c32 gq = io<IO>::unpack(g[q]);
            v[q] = mk(pos < L ? gq.x * v[q].x : 0.f, pos + 1 < L ? gq.y * v[q].y : 0.f);
        }
#pragma unroll
        for (int q = E / 2; q < E; ++q) v[q] = mk(0.f, 0.f);
    }

    if (active) {
        IO *yrow = reinterpret_cast<IO *>(a.y) + act_row_off(a, row);
#pragma unroll
        for (int q = 0; q < E / 2; ++q) store_pair_s<IO, EVEN>(yrow, 2 * (int64_t)(t + q * T), L, a.es, v[q]);
    }
}

// Spectrum of causal real filters: Hout[o, k] = sum_t h[o, t] e^{-2 pi i k t / M},
// k in [0, MC]. Input row o starts at h + o * h_stride (floats) and has L taps.
// May run in place (h_stride = 2 (MC + 1), h == Hout): a row is read completely
// before the first barrier, and only its own slot is written.
template <int MC, int E>
__global__ void __launch_bounds__(rows_per_cta(MC, E) * (MC / E))
    hyena_spectrum_1d(const float *h, int64_t h_stride, int64_t L, c32 *Hout, int64_t nrows,
                      const c32 *__restrict__ tw) {
    constexpr int T = MC / E;
    constexpr int RPC = rows_per_cta(MC, E);
    extern __shared__ float smem[];
    const int lrow = threadIdx.x / T;
    const int t = threadIdx.x - lrow * T;
    const int64_t o = (int64_t)blockIdx.x * RPC + lrow;
    const bool active = o < nrows;
    float *sre = smem + lrow * 2 * MC;
    float *sim = sre + MC;
    c32 v[E];
    const float *hrow = h + (active ? o : 0) * h_stride;
    // tap pairs as one 8-byte load where every row starts 8-byte aligned
    const bool pairs = ((reinterpret_cast<uintptr_t>(h) | (uintptr_t)(h_stride * 4)) & 7) == 0;
#pragma unroll
    for (int q = 0; q < E / 2; ++q) {
        const int64_t pos = 2 * (int64_t)(t + q * T);
        if (pairs && active && pos + 1 < L) {
            const float2 x = *reinterpret_cast<const float2 *>(hrow + pos);   // plain load: the row may be transformed in place
            v[q] = mk(x.x, x.y);
        } else {
            v[q] = mk(active && pos < L ? hrow[pos] : 0.f, active && pos + 1 < L ? hrow[pos + 1] : 0.f);
        }
    }
#pragma unroll
    for (int q = E / 2; q < E; ++q) v[q] = mk(0.f, 0.f);
    fft_cta<MC, E, -1, true>(v, sre, sim, t, tw);
#pragma unroll
    for (int q = 0; q < E; ++q) {
        sre[t + q * T] = v[q].x;
        sim[t + q * T] = v[q].y;
    }
    __syncthreads();
    c32 *Hrow = Hout + (active ? o : 0) * (MC + 1);
#pragma unroll
    for (int q = 0; q < E; ++q) {
        const int k = t + q * T;
        const int km = (MC - k) & (MC - 1);
        const c32 Zk = v[q];
        const c32 Zm = mk(sre[km], sim[km]);
        const c32 Ek = mk(0.5f * (Zk.x + Zm.x), 0.5f * (Zk.y - Zm.y));
        const c32 Ok = mk(0.5f * (Zk.y + Zm.y), -0.5f * (Zk.x - Zm.x));
        const c32 wO = mul(ldg_c(tw + k), Ok);
        if (active) {
            Hrow[k] = add(Ek, wO);
            if (k == 0) Hrow[MC] = mk(Ek.x - Ok.x, 0.f);  // Nyquist bin: E_0 - O_0, real
        }
    }
}

}  // namespace hyena
