// Register-resident FFT building blocks for sm_100a.
//
// A CTA-level complex FFT of length Mc is run as Stockham passes: each thread
// keeps E complex values in registers, performs radix-16 (or a final radix-2/4/8)
// butterflies on them, and the threads exchange data through shared memory
// between passes. Thread t holds element t + q*T in register q (T = Mc / E)
// both before the first pass and after the last one (natural order), so
// element-wise work (loads, gating, the spectral product) happens in registers.
//
// Shared memory holds the exchange buffer as two float planes (re, im). The
// write pattern of a pass with stride Ns = 16^p is made bank-conflict-free with
// an XOR swizzle of the low five index bits; reads of the next pass are
// consecutive per warp and stay conflict-free under the same swizzle.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace hyena {

// Compile-time loop: f(std::integral_constant<int, i>) for i = 0..N-1. Bodies that
// take register arrays by reference are marked always_inline: a lambda left
// out of line makes its captured array addressable, and the array then lives
// in local memory.
template <typename F, int... I>
__device__ __forceinline__ void static_for_impl(F &&f, std::integer_sequence<int, I...>) {
    (f(std::integral_constant<int, I>{}), ...);
}
template <int N, typename F>
__device__ __forceinline__ void static_for(F &&f) {
    static_for_impl(f, std::make_integer_sequence<int, N>{});
}

struct c32 {
    float x, y;
};

__device__ __forceinline__ c32 mk(float x, float y) { return c32{x, y}; }
__device__ __forceinline__ c32 add(c32 a, c32 b) { return c32{a.x + b.x, a.y + b.y}; }
__device__ __forceinline__ c32 sub(c32 a, c32 b) { return c32{a.x - b.x, a.y - b.y}; }
__device__ __forceinline__ c32 mul(c32 a, c32 b) {
    return c32{fmaf(a.x, b.x, -a.y * b.y), fmaf(a.x, b.y, a.y * b.x)};
}
__device__ __forceinline__ c32 conj(c32 a) { return c32{a.x, -a.y}; }
__device__ __forceinline__ c32 scale(c32 a, float s) { return c32{a.x * s, a.y * s}; }
// a * (DIR * i): multiply by +i (DIR = +1) or -i (DIR = -1)
template <int DIR>
__device__ __forceinline__ c32 rot90(c32 a) {
    return DIR > 0 ? c32{-a.y, a.x} : c32{a.y, -a.x};
}
// a + rot90(b) and a - rot90(b)
template <int DIR>
__device__ __forceinline__ c32 add_rot(c32 a, c32 b) { return add(a, rot90<DIR>(b)); }
template <int DIR>
__device__ __forceinline__ c32 sub_rot(c32 a, c32 b) { return sub(a, rot90<DIR>(b)); }

// Two complex values of two independent rows carried in lockstep: re = (row a,
// row b) real parts, im = imaginary parts. Every operation is one packed
// fp32x2 instruction per component, so two rows cost the instructions of one.
struct c32x2 {
    float2 re, im;
};
__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float2 f2add(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 f2sub(float2 a, float2 b) { return __ffma2_rn(b, f2(-1.f, -1.f), a); }
__device__ __forceinline__ float2 f2mul(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 f2fma(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ c32x2 add(c32x2 a, c32x2 b) { return c32x2{f2add(a.re, b.re), f2add(a.im, b.im)}; }
__device__ __forceinline__ c32x2 sub(c32x2 a, c32x2 b) { return c32x2{f2sub(a.re, b.re), f2sub(a.im, b.im)}; }
// both lanes times the same complex scalar w
__device__ __forceinline__ c32x2 mul(c32x2 a, c32 w) {
    return c32x2{f2fma(a.im, f2(-w.y, -w.y), f2mul(a.re, f2(w.x, w.x))),
                 f2fma(a.im, f2(w.x, w.x), f2mul(a.re, f2(w.y, w.y)))};
}
// lane-wise product of two pairs
__device__ __forceinline__ c32x2 mul(c32x2 a, c32x2 b) {
    return c32x2{f2fma(f2(-a.im.x, -a.im.y), b.im, f2mul(a.re, b.re)), f2fma(a.im, b.re, f2mul(a.re, b.im))};
}
// a complex scalar as the value type V (both lanes equal for pairs)
template <typename V>
__device__ __forceinline__ V bcast(c32 w);
template <>
__device__ __forceinline__ c32 bcast<c32>(c32 w) { return w; }
template <>
__device__ __forceinline__ c32x2 bcast<c32x2>(c32 w) { return c32x2{f2(w.x, w.x), f2(w.y, w.y)}; }

template <int DIR>
__device__ __forceinline__ c32x2 rot90(c32x2 a) {
    return DIR > 0 ? c32x2{f2mul(a.im, f2(-1.f, -1.f)), a.re} : c32x2{a.im, f2mul(a.re, f2(-1.f, -1.f))};
}
template <int DIR>
__device__ __forceinline__ c32x2 add_rot(c32x2 a, c32x2 b) {   // a + (DIR i) b
    return DIR > 0 ? c32x2{f2sub(a.re, b.im), f2add(a.im, b.re)} : c32x2{f2add(a.re, b.im), f2sub(a.im, b.re)};
}
template <int DIR>
__device__ __forceinline__ c32x2 sub_rot(c32x2 a, c32x2 b) {   // a - (DIR i) b
    return DIR > 0 ? c32x2{f2add(a.re, b.im), f2sub(a.im, b.re)} : c32x2{f2sub(a.re, b.im), f2add(a.im, b.re)};
}

// W_64^m = exp(-2 pi i m / 64), m = 0..63 (cos and sin of m pi / 32, rounded to
// float). Indexed with compile-time offsets, they become constant-bank operands.
__constant__ float2 c_w64[64] = {
    {1.000000000e+00f, -0.000000000e+00f},
    {9.951847267e-01f, -9.801714033e-02f},
    {9.807852804e-01f, -1.950903220e-01f},
    {9.569403357e-01f, -2.902846773e-01f},
    {9.238795325e-01f, -3.826834324e-01f},
    {8.819212643e-01f, -4.713967368e-01f},
    {8.314696123e-01f, -5.555702330e-01f},
    {7.730104534e-01f, -6.343932842e-01f},
    {7.071067812e-01f, -7.071067812e-01f},
    {6.343932842e-01f, -7.730104534e-01f},
    {5.555702330e-01f, -8.314696123e-01f},
    {4.713967368e-01f, -8.819212643e-01f},
    {3.826834324e-01f, -9.238795325e-01f},
    {2.902846773e-01f, -9.569403357e-01f},
    {1.950903220e-01f, -9.807852804e-01f},
    {9.801714033e-02f, -9.951847267e-01f},
    {6.123233996e-17f, -1.000000000e+00f},
    {-9.801714033e-02f, -9.951847267e-01f},
    {-1.950903220e-01f, -9.807852804e-01f},
    {-2.902846773e-01f, -9.569403357e-01f},
    {-3.826834324e-01f, -9.238795325e-01f},
    {-4.713967368e-01f, -8.819212643e-01f},
    {-5.555702330e-01f, -8.314696123e-01f},
    {-6.343932842e-01f, -7.730104534e-01f},
    {-7.071067812e-01f, -7.071067812e-01f},
    {-7.730104534e-01f, -6.343932842e-01f},
    {-8.314696123e-01f, -5.555702330e-01f},
    {-8.819212643e-01f, -4.713967368e-01f},
    {-9.238795325e-01f, -3.826834324e-01f},
    {-9.569403357e-01f, -2.902846773e-01f},
    {-9.807852804e-01f, -1.950903220e-01f},
    {-9.951847267e-01f, -9.801714033e-02f},
    {-1.000000000e+00f, -1.224646799e-16f},
    {-9.951847267e-01f, 9.801714033e-02f},
    {-9.807852804e-01f, 1.950903220e-01f},
    {-9.569403357e-01f, 2.902846773e-01f},
    {-9.238795325e-01f, 3.826834324e-01f},
    {-8.819212643e-01f, 4.713967368e-01f},
    {-8.314696123e-01f, 5.555702330e-01f},
    {-7.730104534e-01f, 6.343932842e-01f},
    {-7.071067812e-01f, 7.071067812e-01f},
    {-6.343932842e-01f, 7.730104534e-01f},
    {-5.555702330e-01f, 8.314696123e-01f},
    {-4.713967368e-01f, 8.819212643e-01f},
    {-3.826834324e-01f, 9.238795325e-01f},
    {-2.902846773e-01f, 9.569403357e-01f},
    {-1.950903220e-01f, 9.807852804e-01f},
    {-9.801714033e-02f, 9.951847267e-01f},
    {-1.836970199e-16f, 1.000000000e+00f},
    {9.801714033e-02f, 9.951847267e-01f},
    {1.950903220e-01f, 9.807852804e-01f},
    {2.902846773e-01f, 9.569403357e-01f},
    {3.826834324e-01f, 9.238795325e-01f},
    {4.713967368e-01f, 8.819212643e-01f},
    {5.555702330e-01f, 8.314696123e-01f},
    {6.343932842e-01f, 7.730104534e-01f},
    {7.071067812e-01f, 7.071067812e-01f},
    {7.730104534e-01f, 6.343932842e-01f},
    {8.314696123e-01f, 5.555702330e-01f},
    {8.819212643e-01f, 4.713967368e-01f},
    {9.238795325e-01f, 3.826834324e-01f},
    {9.569403357e-01f, 2.902846773e-01f},
    {9.807852804e-01f, 1.950903220e-01f},
    {9.951847267e-01f, 9.801714033e-02f}};

// A zero the compiler cannot see through: adding it to a constant-table index
// keeps the (cheap) constant loads inside loops instead of hoisting them into
// registers for the whole kernel.
__device__ __forceinline__ int opaque_zero() {
    int z;
    asm volatile("mov.u32 %0, 0;" : "=r"(z));
    return z;
}

// W_{2E}^q (E <= 32); z must be opaque_zero().
template <int E>
__device__ __forceinline__ c32 w2e(int q, int z) {
    const float2 f = c_w64[q * (32 / E) + z];
    return c32{f.x, f.y};
}

// cos / sin of k*pi/8 for the radix-16 internal twiddles (exact math constants)
#define HY_C1 0.92387953251128675613f  // cos(pi/8)
#define HY_S1 0.38268343236508977173f  // sin(pi/8)
#define HY_R2 0.70710678118654752440f  // sqrt(1/2)

// W_16^m = exp(DIR * 2 pi i m / 16) for the m that a 4x4 split needs.
template <int DIR, int m, typename V>
__device__ __forceinline__ V tw16(V a) {
    constexpr float s = (float)DIR;
    if constexpr (m == 0) return a;
    else if constexpr (m == 1) return mul(a, c32{HY_C1, s * HY_S1});
    else if constexpr (m == 2) return mul(a, c32{HY_R2, s * HY_R2});
    else if constexpr (m == 3) return mul(a, c32{HY_S1, s * HY_C1});
    else if constexpr (m == 4) return rot90<DIR>(a);
    else if constexpr (m == 6) return mul(a, c32{-HY_R2, s * HY_R2});
    else if constexpr (m == 9) return mul(a, c32{-HY_C1, -s * HY_S1});
    else return a;  // not reached
}

template <int DIR, int m, typename V>
__device__ __forceinline__ V tw8(V a) {
    constexpr float s = (float)DIR;
    if constexpr (m == 0) return a;
    else if constexpr (m == 1) return mul(a, c32{HY_R2, s * HY_R2});
    else if constexpr (m == 2) return rot90<DIR>(a);
    else return mul(a, c32{-HY_R2, s * HY_R2});  // m == 3
}

// In-place 4-point DFT, X[k] = sum_n a[n] W_4^{nk}, W_4 = exp(DIR 2 pi i / 4).
template <int DIR, typename V>
__device__ __forceinline__ void dft4(V &a0, V &a1, V &a2, V &a3) {
    V s02 = add(a0, a2), d02 = sub(a0, a2);
    V s13 = add(a1, a3), d13 = sub(a1, a3);
    a0 = add(s02, s13);
    a2 = sub(s02, s13);
    a1 = add_rot<DIR>(d02, d13);
    a3 = sub_rot<DIR>(d02, d13);
}

// 4-point DFT of (a0, a1, 0, 0).
template <int DIR, typename V>
__device__ __forceinline__ void dft4_half(V &a0, V &a1, V &a2, V &a3) {
    a2 = sub(a0, a1);
    a3 = sub_rot<DIR>(a0, a1);
    V t = a0;
    a0 = add(t, a1);
    a1 = add_rot<DIR>(t, a1);
}

template <typename V>
__device__ __forceinline__ void dft2(V &a0, V &a1) {
    V t = a0;
    a0 = add(t, a1);
    a1 = sub(t, a1);
}

// 16-point DFT on x[o + st*n], n = 0..15, result in natural order at the same
// positions. Split n = 4 n1 + n2, k = k1 + 4 k2. HALF: inputs n >= 8 are zero.
template <int DIR, bool HALF, int st, int o, typename V, int NR>
__device__ __forceinline__ void dft16(V (&x)[NR]) {
#define X(i) x[o + st * (i)]
    // DFT4 over n1 for each n2; result A[n2][k1] kept at position 4*k1 + n2
    if constexpr (HALF) {
        dft4_half<DIR>(X(0), X(4), X(8), X(12));
        dft4_half<DIR>(X(1), X(5), X(9), X(13));
        dft4_half<DIR>(X(2), X(6), X(10), X(14));
        dft4_half<DIR>(X(3), X(7), X(11), X(15));
    } else {
        dft4<DIR>(X(0), X(4), X(8), X(12));
        dft4<DIR>(X(1), X(5), X(9), X(13));
        dft4<DIR>(X(2), X(6), X(10), X(14));
        dft4<DIR>(X(3), X(7), X(11), X(15));
    }
    // twiddles W_16^{n2 k1}
    X(5) = tw16<DIR, 1>(X(5));
    X(6) = tw16<DIR, 2>(X(6));
    X(7) = tw16<DIR, 3>(X(7));
    X(9) = tw16<DIR, 2>(X(9));
    X(10) = tw16<DIR, 4>(X(10));
    X(11) = tw16<DIR, 6>(X(11));
    X(13) = tw16<DIR, 3>(X(13));
    X(14) = tw16<DIR, 6>(X(14));
    X(15) = tw16<DIR, 9>(X(15));
    // DFT4 over n2 for each k1: X[k1 + 4 k2] lands at position 4*k1 + k2
    dft4<DIR>(X(0), X(1), X(2), X(3));
    dft4<DIR>(X(4), X(5), X(6), X(7));
    dft4<DIR>(X(8), X(9), X(10), X(11));
    dft4<DIR>(X(12), X(13), X(14), X(15));
    // transpose 4x4 back to natural order
    V t;
    t = X(1); X(1) = X(4); X(4) = t;
    t = X(2); X(2) = X(8); X(8) = t;
    t = X(3); X(3) = X(12); X(12) = t;
    t = X(6); X(6) = X(9); X(9) = t;
    t = X(7); X(7) = X(13); X(13) = t;
    t = X(11); X(11) = X(14); X(14) = t;
#undef X
}

// 8-point DFT on x[o + st*n], n = 0..7 (split n = 2 n1 + n2, k = k1 + 4 k2).
// HALF: inputs n >= 4 are zero.
template <int DIR, bool HALF, int st, int o, typename V, int NR>
__device__ __forceinline__ void dft8(V (&x)[NR]) {
#define X(i) x[o + st * (i)]
    if constexpr (HALF) {
        dft4_half<DIR>(X(0), X(2), X(4), X(6));   // n2 = 0 -> A[0][k1] at 2*k1
        dft4_half<DIR>(X(1), X(3), X(5), X(7));   // n2 = 1 -> A[1][k1] at 2*k1 + 1
    } else {
        dft4<DIR>(X(0), X(2), X(4), X(6));
        dft4<DIR>(X(1), X(3), X(5), X(7));
    }
    X(3) = tw8<DIR, 1>(X(3));
    X(5) = tw8<DIR, 2>(X(5));
    X(7) = tw8<DIR, 3>(X(7));
    dft2(X(0), X(1));                    // X[k1 + 4 k2] at 2*k1 + k2
    dft2(X(2), X(3));
    dft2(X(4), X(5));
    dft2(X(6), X(7));
    V t;                                 // positions 2k1+k2 -> k1+4k2
    t = X(1); X(1) = X(2); X(2) = X(4); X(4) = t;
    t = X(3); X(3) = X(6); X(6) = X(5); X(5) = t;
#undef X
}

template <int DIR, int st, int o, typename V, int NR>
__device__ __forceinline__ void dft4r(V (&x)[NR]) {
    dft4<DIR>(x[o], x[o + st], x[o + 2 * st], x[o + 3 * st]);
}

template <int DIR, int st, int o, typename V, int NR>
__device__ __forceinline__ void dft2r(V (&x)[NR]) {
    dft2(x[o], x[o + st]);
}

template <int R, int DIR, bool HALF, int st, int o, typename V, int NR>
__device__ __forceinline__ void dftR(V (&x)[NR]) {
    if constexpr (R == 16) dft16<DIR, HALF, st, o>(x);
    else if constexpr (R == 8) dft8<DIR, HALF, st, o>(x);
    else if constexpr (R == 4) dft4r<DIR, st, o>(x);
    else dft2r<DIR, st, o>(x);
}

// Powers w^1..w^(R-1) of a twiddle applied to x[o + st*r]. Four running
// products p_i = w^i, w^(i+4), w^(i+8), w^(i+12) (each power at most four
// multiplications from w), applied as they are formed so that few powers are
// live at once.
template <int R, int st, int o, typename V, int NR>
__device__ __forceinline__ void twiddle_powers(V (&x)[NR], c32 w) {
    const V w1 = bcast<V>(w);
    if constexpr (R == 2) {
        x[o + st] = mul(x[o + st], w1);
    } else {
        V p1 = w1;
        V p2 = mul(w1, w1);
        V p3 = mul(p2, w1);
        x[o + st] = mul(x[o + st], p1);
        x[o + 2 * st] = mul(x[o + 2 * st], p2);
        x[o + 3 * st] = mul(x[o + 3 * st], p3);
        if constexpr (R >= 8) {
            const V w4 = mul(p2, p2);
            V p0 = w4;
#pragma unroll
            for (int g = 1; g < R / 4; ++g) {
                x[o + (4 * g) * st] = mul(x[o + (4 * g) * st], p0);
                p1 = mul(p1, w4);
                p2 = mul(p2, w4);
                p3 = mul(p3, w4);
                x[o + (4 * g + 1) * st] = mul(x[o + (4 * g + 1) * st], p1);
                x[o + (4 * g + 2) * st] = mul(x[o + (4 * g + 2) * st], p2);
                x[o + (4 * g + 3) * st] = mul(x[o + (4 * g + 3) * st], p3);
                if (g + 1 < R / 4) p0 = mul(p0, w4);
            }
        }
    }
}

// Swizzle of an exchange-buffer index written by a pass of stride Ns.
template <int NS>
__device__ __forceinline__ int swz(int i) {
    if constexpr (NS == 1) return i ^ ((i >> 5) & 15);
    else if constexpr (NS == 16) return i ^ (((i >> 8) & 1) << 4);
    else return i;
}

constexpr int ilog2(int v) { return v <= 1 ? 0 : 1 + ilog2(v >> 1); }
// Pass plan with passes of radix 2^LR (LR = 4: radix 16, the default; LR = 3
// when a thread holds only 8 values), then one pass for the remaining factor.
constexpr int num_passes(int Mc, int LR = 4) { return (ilog2(Mc) + LR - 1) / LR; }
constexpr int pass_radix(int Mc, int p, int LR = 4) {
    return (p < ilog2(Mc) / LR) ? (1 << LR) : (1 << (ilog2(Mc) % LR));
}
constexpr int pass_stride(int Mc, int p, int LR = 4) { return 1 << (LR * p); }  // Ns = (2^LR)^p
// log2 of the largest pass radix a thread holding E values can run
constexpr int pass_lr(int E) { return E >= 16 ? 4 : ilog2(E); }

}  // namespace hyena
