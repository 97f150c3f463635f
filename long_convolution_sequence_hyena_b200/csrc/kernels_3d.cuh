// 3D (HyenaND on a volume) forward and kernel spectrum as separable staged
// transforms through a device workspace.
//
// "How HyenaND works", "2. The convolution theorem (FFT)": the convolution of
// a volume with a global kernel runs on the native grid as a 3D FFT. A volume
// v [Dz][H][W] is zero-padded to [2Dz][2H][2W]; the kernel on offsets
// oz in [-Dz, Dz), oy in [-H, H), ox in [-W, W) is placed cyclically (offset o
// at index o mod 2Dz, ...), so the cyclic product read out on [0, Dz) x [0, H)
// x [0, W) is the linear, non-causal convolution (as in 2D).
//
// The transform is complex (the real volume enters with a zero imaginary
// part) and separable: one batched 1D FFT stage per axis, each stage a kernel
// of its own, through a workspace of [Dz][2H][2W] complex per volume. Only
// z < Dz and (in the x stage) y < H carry data, so no stage stores padding:
//   X: rows (z, y < H) of 2W points   [z][y][kx]          (input: the volume)
//   Y: columns (z, kx) of 2H points   [z][ky][kx]         (in place)
//   Z: columns (ky, kx) of 2Dz points, the spectral product (kernel spectrum
//      plus the feedthrough, scaled by 1/(8 Dz H W)) and the inverse, keeping
//      z < Dz                          [z][ky][kx]        (in place)
// then Y inverse (keeping y < H) and X inverse (keeping x < W, the real part),
// the gate, and the next order's X forward or the output. Per order: Z, Y
// inverse, X (inverse, gate, forward), Y forward.
//
// Every stage is a batch of NSEQ sequences per CTA in the sequence-major
// shared layout of cta_fft.cuh (128 threads; NSEQ x LEN = 2048 elements).
// The X stage moves whole rows through shared memory so that its global
// accesses are contiguous; the column stages give a warp consecutive columns,
// whose elements are contiguous in memory.
#pragma once
#include "kernels_1d.cuh"
#include "kernels_1d_staged.cuh"

namespace hyena {

struct Fwd3dArgs {
    const void *v;                         // [B, C, Dz, H, W] io (the gate sandwich: q)
    const void *k;                         // gate sandwich only: the inner gate's key
    const void *gates[HYENA_MAX_ORDER];
    const c32 *K;                          // [N, C, 2Dz, 2H, 2W] kernel spectra
    const float *dskip;                    // [N, C] or nullptr
    void *y;
    const c32 *tws;                        // W_1024^m
    float2 *ws;                            // chunk workspace: volumes x [Dz][2H][2W]
    int64_t o0, np;                        // first visit index and count of the chunk's volumes
    int64_t C, B;
    int Dz, H, W;
    int order, n;
};

constexpr int S3_ELEMS = 2048;             // elements per CTA in every stage
constexpr int S3_THREADS = 128;

template <int LEN>
struct Stage3 {
    static constexpr int E = 16, T = LEN / E, NSEQ = S3_ELEMS / LEN;
    static_assert(NSEQ * T == S3_THREADS, "128 threads per stage CTA");
    static_assert(LEN >= 32 && LEN <= 1024, "sequence-major layout needs LEN >= 32");
};

// Visit order c-major, b-minor (volumes sharing a kernel spectrum run together).
__device__ __forceinline__ int64_t visit_volume(const Fwd3dArgs &a, int64_t o, int64_t &c) {
    c = o / a.B;
    return (o - c * a.B) * a.C + c;
}

// X stage. MODE 0: volume -> forward rows; 1: inverse rows, gate x^n, forward
// rows; 2: inverse rows, gate x^n, store y. Rows are (volume, z, y < H).
template <int LX, typename IO, int MODE, bool GATED>
__global__ void __launch_bounds__(S3_THREADS) hyena_3d_x(const Fwd3dArgs a) {
    using S = Stage3<LX>;
    constexpr int E = S::E, T = S::T, NSEQ = S::NSEQ, W = LX / 2;
    __shared__ float2 buf[S3_ELEMS];           // sequence-major rows (maddr layout)
    __shared__ float gbuf[NSEQ * W];           // gate (or the first input) values, row-major
    const int tid = threadIdx.x;
    const int seq = tid % NSEQ, t = tid / NSEQ;
    const int64_t HW = (int64_t)a.H * W, V = (int64_t)a.Dz * HW;
    const int64_t rows_per_vol = (int64_t)a.Dz * a.H;
    const int64_t r0 = (int64_t)blockIdx.x * NSEQ;      // first row of the CTA (over the chunk)
    const int64_t nrows = a.np * rows_per_vol;
    const int64_t wsv = (int64_t)a.Dz * 2 * a.H * LX;   // workspace complex per volume
    // row r -> workspace row (volume lp, z, y) at lp wsv + (z 2H + y) LX; activation row at vol V + (z H + y) W
    auto ws_row = [&](int64_t r) -> float2 * {
        const int64_t lp = r / rows_per_vol, zy = r - lp * rows_per_vol;
        const int64_t z = zy / a.H, yy = zy - z * a.H;
        return a.ws + lp * wsv + (z * 2 * a.H + yy) * LX;
    };
    auto act_off = [&](int64_t r) -> int64_t {
        const int64_t lp = r / rows_per_vol, zy = r - lp * rows_per_vol;
        int64_t c;
        const int64_t vol = visit_volume(a, a.o0 + lp, c);
        return vol * V + zy * W;
    };
    // real values of the CTA's rows (x < W) from an activation tensor into gbuf
    auto load_real = [&](const void *src, bool silu_in) {
        for (int i = tid; i < NSEQ * W; i += S3_THREADS) {
            const int rl = i / W, x = i - rl * W;
            const int64_t r = r0 + rl;
            float val = 0.f;
            if (r < nrows) val = io<IO>::to_f(reinterpret_cast<const IO *>(src)[act_off(r) + x]);
            gbuf[i] = silu_in ? silu(val) : val;
        }
    };

    c32 v[E];
    if constexpr (MODE == 0) {
        load_real(a.v, false);
        __syncthreads();
#pragma unroll
        for (int q = 0; q < E / 2; ++q) v[q] = mk(gbuf[seq * W + t + q * T], 0.f);
        if constexpr (GATED) {   // z^0 = q SiLU(k)
            __syncthreads();
            load_real(a.k, true);
            __syncthreads();
#pragma unroll
            for (int q = 0; q < E / 2; ++q) v[q].x *= gbuf[seq * W + t + q * T];
        }
    } else {
        // the CTA's rows of the workspace, contiguous per row, into the shared layout
        for (int i = tid; i < NSEQ * LX; i += S3_THREADS) {
            const int rl = i / LX, kx = i - rl * LX;
            const int64_t r = r0 + rl;
            buf[maddr<LX, NSEQ>(kx, rl)] = r < nrows ? ws_row(r)[kx] : make_float2(0.f, 0.f);
        }
        load_real(a.gates[a.n], GATED);
        __syncthreads();
#pragma unroll
        for (int q = 0; q < E; ++q) {
            const float2 f = buf[maddr<LX, NSEQ>(t + q * T, seq)];
            v[q] = mk(f.x, f.y);
        }
        __syncthreads();
        fft_cta<LX, E, +1, false, 1024, NSEQ>(v, reinterpret_cast<float *>(buf), nullptr, t, a.tws, seq);
        // keep x < W (registers q < E/2), real part, times the gate
#pragma unroll
        for (int q = 0; q < E / 2; ++q) v[q] = mk(v[q].x * gbuf[seq * W + t + q * T], 0.f);
        if constexpr (MODE == 2) {
            __syncthreads();
#pragma unroll
            for (int q = 0; q < E / 2; ++q) gbuf[seq * W + t + q * T] = v[q].x;
            __syncthreads();
            for (int i = tid; i < NSEQ * W; i += S3_THREADS) {
                const int rl = i / W, x = i - rl * W;
                const int64_t r = r0 + rl;
                if (r < nrows) reinterpret_cast<IO *>(a.y)[act_off(r) + x] = io<IO>::from_f(gbuf[i]);
            }
        }
    }
    if constexpr (MODE != 2) {   // forward rows of this order's (or the next order's) input
#pragma unroll
        for (int q = E / 2; q < E; ++q) v[q] = mk(0.f, 0.f);
        __syncthreads();
        fft_cta<LX, E, -1, true, 1024, NSEQ>(v, reinterpret_cast<float *>(buf), nullptr, t, a.tws, seq);
        __syncthreads();
#pragma unroll
        for (int q = 0; q < E; ++q) buf[maddr<LX, NSEQ>(t + q * T, seq)] = make_float2(v[q].x, v[q].y);
        __syncthreads();
        for (int i = tid; i < NSEQ * LX; i += S3_THREADS) {
            const int rl = i / LX, kx = i - rl * LX;
            const int64_t r = r0 + rl;
            if (r < nrows) ws_row(r)[kx] = buf[maddr<LX, NSEQ>(kx, rl)];
        }
    }
}

// Y stage over columns (volume, z, kx), 2H points at stride 2W in the
// workspace. DIR -1: forward of rows y < H (the rest is padding); +1: inverse,
// keeping y < H.
template <int LY, int DIR>
__global__ void __launch_bounds__(S3_THREADS) hyena_3d_y(const Fwd3dArgs a) {
    using S = Stage3<LY>;
    constexpr int E = S::E, T = S::T, NSEQ = S::NSEQ;
    __shared__ float2 buf[S3_ELEMS];
    const int tid = threadIdx.x;
    const int seq = tid % NSEQ, t = tid / NSEQ;
    const int LX = 2 * a.W;
    const int64_t cols_per_vol = (int64_t)a.Dz * LX;
    const int64_t c = (int64_t)blockIdx.x * NSEQ + seq;   // column over the chunk
    const bool ok = c < a.np * cols_per_vol;
    const int64_t lp = ok ? c / cols_per_vol : 0, zk = ok ? c - lp * cols_per_vol : 0;
    const int64_t z = zk / LX, kx = zk - z * LX;
    float2 *col = a.ws + lp * ((int64_t)a.Dz * LY * LX) + z * LY * LX + kx;   // element y at col + y LX
    c32 v[E];
    constexpr int NIN = DIR < 0 ? E / 2 : E;
#pragma unroll
    for (int q = 0; q < E; ++q) {
        const float2 f = (q < NIN && ok) ? col[(int64_t)(t + q * T) * LX] : make_float2(0.f, 0.f);
        v[q] = mk(f.x, f.y);
    }
    fft_cta<LY, E, DIR, DIR < 0, 1024, NSEQ>(v, reinterpret_cast<float *>(buf), nullptr, t, a.tws, seq);
    constexpr int NOUT = DIR < 0 ? E : E / 2;
    if (ok) {
#pragma unroll
        for (int q = 0; q < NOUT; ++q) col[(int64_t)(t + q * T) * LX] = make_float2(v[q].x, v[q].y);
    }
}

// Z stage over columns (volume, ky, kx), 2Dz points at stride 2H 2W: forward
// (z < Dz carry data), the spectral product with order n's kernel spectrum
// plus the feedthrough (the delta tap's spectrum is the constant Dskip), the
// inverse; z < Dz is written back.
template <int LZ>
__global__ void __launch_bounds__(S3_THREADS) hyena_3d_z(const Fwd3dArgs a) {
    using S = Stage3<LZ>;
    constexpr int E = S::E, T = S::T, NSEQ = S::NSEQ;
    __shared__ float2 buf[S3_ELEMS];
    const int tid = threadIdx.x;
    const int seq = tid % NSEQ, t = tid / NSEQ;
    const int64_t plane = (int64_t)2 * a.H * 2 * a.W;     // one z slice of the workspace
    const int64_t c = (int64_t)blockIdx.x * NSEQ + seq;   // column (volume, ky, kx) over the chunk
    const bool ok = c < a.np * plane;
    const int64_t lp = ok ? c / plane : 0, kk = ok ? c - lp * plane : 0;
    int64_t ch;
    (void)visit_volume(a, a.o0 + lp, ch);
    float2 *col = a.ws + lp * ((int64_t)a.Dz * plane) + kk;           // element z at col + z plane
    const c32 *Kc = a.K + ((int64_t)a.n * a.C + ch) * ((int64_t)LZ * plane) + kk;   // bin kz at Kc + kz plane
    c32 v[E];
#pragma unroll
    for (int q = 0; q < E; ++q) {
        const float2 f = (q < E / 2 && ok) ? col[(int64_t)(t + q * T) * plane] : make_float2(0.f, 0.f);
        v[q] = mk(f.x, f.y);
    }
    fft_cta<LZ, E, -1, true, 1024, NSEQ>(v, reinterpret_cast<float *>(buf), nullptr, t, a.tws, seq);
    const float s = 1.f / (float)((int64_t)LZ * plane);
    const float dsk = a.dskip ? __ldg(a.dskip + a.n * a.C + ch) : 0.f;
#pragma unroll
    for (int q = 0; q < E; ++q) {
        c32 h = ok ? ldg_c(Kc + (int64_t)(t + q * T) * plane) : mk(0.f, 0.f);
        h = mk(s * (h.x + dsk), s * h.y);
        v[q] = mul(v[q], h);
    }
    __syncthreads();   // the forward's last shared reads are done before the inverse writes
    fft_cta<LZ, E, +1, false, 1024, NSEQ>(v, reinterpret_cast<float *>(buf), nullptr, t, a.tws, seq);
    if (ok) {
#pragma unroll
        for (int q = 0; q < E / 2; ++q) col[(int64_t)(t + q * T) * plane] = make_float2(v[q].x, v[q].y);
    }
}

// ---------------------------------------------------------------- spectra --
// Kernel spectra K^ = 3D DFT of the kernel placed cyclically, written in
// natural order [2Dz][2H][2W] into the output, which the Y and Z stages then
// transform in place. Input kernel o at Kin + o * cs, offset-grid element
// (iz, iy, ix) (offset iz - Dz, ...) at [(iz 2H + iy) 2W + ix].
struct Spec3dArgs {
    const float *Kin;
    int64_t cs;           // floats between input kernels
    c32 *Kout;            // [n][2Dz][2H][2W]
    const c32 *tws;
    int64_t n;            // kernels
    int Dz, H, W;
};

template <int LX>
__global__ void __launch_bounds__(S3_THREADS) hyena_3d_spec_x(const Spec3dArgs a) {
    using S = Stage3<LX>;
    constexpr int E = S::E, T = S::T, NSEQ = S::NSEQ, W = LX / 2;
    __shared__ float2 buf[S3_ELEMS];
    const int tid = threadIdx.x;
    const int seq = tid % NSEQ, t = tid / NSEQ;
    const int64_t rows_per_k = (int64_t)2 * a.Dz * 2 * a.H;
    const int64_t r0 = (int64_t)blockIdx.x * NSEQ;
    const int64_t nrows = a.n * rows_per_k;
    // cyclic row (kernel o, iz, iy) holds offset-grid row ((iz + Dz) mod 2Dz, (iy + H) mod 2H),
    // and cyclic element ix the offset-grid element (ix + W) mod 2W
    for (int i = tid; i < NSEQ * LX; i += S3_THREADS) {
        const int rl = i / LX, ix = i - rl * LX;
        const int64_t r = r0 + rl;
        float val = 0.f;
        if (r < nrows) {
            const int64_t o = r / rows_per_k, zy = r - o * rows_per_k;
            const int64_t iz = zy / (2 * a.H), iy = zy - iz * 2 * a.H;
            const int64_t sz = (iz + a.Dz) % (2 * a.Dz), sy = (iy + a.H) % (2 * a.H), sx = (ix + W) % LX;
            val = a.Kin[o * a.cs + (sz * 2 * a.H + sy) * LX + sx];
        }
        buf[maddr<LX, NSEQ>(ix, rl)] = make_float2(val, 0.f);
    }
    __syncthreads();
    c32 v[E];
#pragma unroll
    for (int q = 0; q < E; ++q) {
        const float2 f = buf[maddr<LX, NSEQ>(t + q * T, seq)];
        v[q] = mk(f.x, f.y);
    }
    __syncthreads();
    fft_cta<LX, E, -1, false, 1024, NSEQ>(v, reinterpret_cast<float *>(buf), nullptr, t, a.tws, seq);
    __syncthreads();
#pragma unroll
    for (int q = 0; q < E; ++q) buf[maddr<LX, NSEQ>(t + q * T, seq)] = make_float2(v[q].x, v[q].y);
    __syncthreads();
    for (int i = tid; i < NSEQ * LX; i += S3_THREADS) {
        const int rl = i / LX, kx = i - rl * LX;
        const int64_t r = r0 + rl;
        if (r < nrows) {
            const float2 f = buf[maddr<LX, NSEQ>(kx, rl)];
            a.Kout[r * LX + kx] = mk(f.x, f.y);
        }
    }
}

// Y (AXIS 1) or Z (AXIS 2) forward over full columns of the spectrum, in place.
template <int LEN, int AXIS>
__global__ void __launch_bounds__(S3_THREADS) hyena_3d_spec_col(const Spec3dArgs a) {
    using S = Stage3<LEN>;
    constexpr int E = S::E, T = S::T, NSEQ = S::NSEQ;
    __shared__ float2 buf[S3_ELEMS];
    const int tid = threadIdx.x;
    const int seq = tid % NSEQ, t = tid / NSEQ;
    const int64_t LX = 2 * a.W, LYY = 2 * a.H, LZZ = 2 * a.Dz;
    const int64_t per_k = LZZ * LYY * LX;
    const int64_t cols_per_k = AXIS == 1 ? LZZ * LX : LYY * LX;
    const int64_t stride = AXIS == 1 ? LX : LYY * LX;
    const int64_t c = (int64_t)blockIdx.x * NSEQ + seq;
    const bool ok = c < a.n * cols_per_k;
    const int64_t o = ok ? c / cols_per_k : 0, rem = ok ? c - o * cols_per_k : 0;
    // Y: column (iz, kx) starts at iz 2H 2W + kx; Z: column (ky, kx) at ky 2W + kx
    const int64_t base = AXIS == 1 ? (rem / LX) * LYY * LX + rem % LX : rem;
    c32 *col = a.Kout + o * per_k + base;
    c32 v[E];
#pragma unroll
    for (int q = 0; q < E; ++q) v[q] = ok ? col[(int64_t)(t + q * T) * stride] : mk(0.f, 0.f);
    fft_cta<LEN, E, -1, false, 1024, NSEQ>(v, reinterpret_cast<float *>(buf), nullptr, t, a.tws, seq);
    if (ok) {
#pragma unroll
        for (int q = 0; q < E; ++q) col[(int64_t)(t + q * T) * stride] = v[q];
    }
}

}  // namespace hyena
