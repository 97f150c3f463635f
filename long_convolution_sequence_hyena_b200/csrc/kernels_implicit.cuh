// Implicit filter network: positional features -> two sine layers -> linear
// head -> window. One CTA per tile of 32 positions (one per lane); the hidden
// activations of the tile are computed once into shared memory and reused for
// every output channel.
//
// 1D ("Hyena — Long Convolutions Math", "Implicit filters: an MLP over
// positions", "The decay window"):
//   features of t: [t/L, cos(2 pi k t/L), sin(2 pi k t/L) for k = 1..K]
//   window: exp(-alpha[o] * t)
// 2D ("How HyenaND works", "1. An implicit filter"):
//   features of offset (oy, ox): (oy/H, ox/W), oy in [-H, H), ox in [-W, W)
//   window: exp(-(py^2 + px^2) / (2 sigma[o]^2))
#pragma once
#include "hyena.h"

namespace hyena {

constexpr int IMP_TP = 32;        // positions per CTA (one per lane)
constexpr int IMP_THREADS = 256;  // 8 warps; warp w handles outputs w, w+8, ...
constexpr int IMP_MAXW = 128;     // maximum width
constexpr int IMP_MAXF = 65;      // maximum input features (1 + 2K, K <= 32)

struct ImplicitArgs {
    hyena_implicit_params_t p;
    int ndim;
    int64_t L;                 // 1D length
    int64_t H, W;              // 2D half-extents (grid is 2H x 2W offsets)
    int64_t npos;              // L or 4 H W
    int64_t nout;              // N * channels
    float *out;                // output base
    int64_t out_stride;        // floats between output channels
    int64_t out_row_stride;    // 2D: floats between rows of one channel (>= 2W)
};

template <int WREG>
__global__ void __launch_bounds__(IMP_THREADS) hyena_implicit_filter_kernel(const ImplicitArgs a) {
    __shared__ float feat[IMP_TP][IMP_MAXF + 1];
    __shared__ float h1[IMP_TP][IMP_MAXW + 1];
    __shared__ float h2T[IMP_MAXW][IMP_TP];
    const int width = a.p.width;
    const int fin = a.ndim == 1 ? 1 + 2 * a.p.num_freqs : 2;
    const int64_t p0 = (int64_t)blockIdx.x * IMP_TP;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    // features
    for (int i = threadIdx.x; i < IMP_TP * fin; i += IMP_THREADS) {
        const int pl = i / fin, f = i - pl * fin;
        const int64_t pos = p0 + pl;
        float val = 0.f;
        if (pos < a.npos) {
            if (a.ndim == 1) {
                if (f == 0) {
                    val = (float)((double)pos / (double)a.L);
                } else {
                    const int64_t k = (f + 1) / 2;
                    // angle 2 pi k t / L, reduced exactly in integers first
                    const int64_t r = (k * pos) % a.L;
                    float s, c;
                    sincospif((float)(2.0 * (double)r / (double)a.L), &s, &c);
                    val = (f & 1) ? c : s;
                }
            } else {
                const int64_t iy = pos / (2 * a.W), ix = pos - iy * (2 * a.W);
                val = f == 0 ? (float)((double)(iy - a.H) / (double)a.H) : (float)((double)(ix - a.W) / (double)a.W);
            }
        }
        feat[pl][f] = val;
    }
    __syncthreads();
    // first sine layer
    for (int i = threadIdx.x; i < IMP_TP * width; i += IMP_THREADS) {
        const int pl = i / width, j = i - pl * width;
        float acc = __ldg(a.p.b1 + j);
        for (int f = 0; f < fin; ++f) acc = fmaf(__ldg(a.p.W1 + (int64_t)j * fin + f), feat[pl][f], acc);
        h1[pl][j] = sinf(a.p.omega0 * acc);
    }
    __syncthreads();
    // second sine layer, stored transposed for the head
    for (int i = threadIdx.x; i < IMP_TP * width; i += IMP_THREADS) {
        const int pl = i / width, j = i - pl * width;
        float acc = __ldg(a.p.b2 + j);
        for (int f = 0; f < width; ++f) acc = fmaf(__ldg(a.p.W2 + (int64_t)j * width + f), h1[pl][f], acc);
        h2T[j][pl] = sinf(a.p.omega_hidden * acc);
    }
    __syncthreads();

    // head + window: lane = position, warp-strided outputs
    const int64_t pos = p0 + lane;
    const bool ok = pos < a.npos;
    float act[WREG];
#pragma unroll
    for (int j = 0; j < WREG; ++j) act[j] = j < width ? h2T[j][lane] : 0.f;
    float py = 0.f, px = 0.f;
    int64_t off = pos;
    if (a.ndim == 2 && ok) {
        const int64_t iy = pos / (2 * a.W), ix = pos - iy * (2 * a.W);
        py = (float)((double)(iy - a.H) / (double)a.H);
        px = (float)((double)(ix - a.W) / (double)a.W);
        off = iy * a.out_row_stride + ix;
    }
    const float r2 = py * py + px * px;
    for (int64_t o = warp; o < a.nout; o += IMP_THREADS / 32) {
        const float4 *w3 = reinterpret_cast<const float4 *>(a.p.W3 + o * width);
        float acc = __ldg(a.p.b3 + o);
#pragma unroll
        for (int j4 = 0; j4 < WREG / 4; ++j4) {
            if (4 * j4 < width) {
                const float4 w = __ldg(w3 + j4);
                acc = fmaf(w.x, act[4 * j4], acc);
                acc = fmaf(w.y, act[4 * j4 + 1], acc);
                acc = fmaf(w.z, act[4 * j4 + 2], acc);
                acc = fmaf(w.w, act[4 * j4 + 3], acc);
            }
        }
        const float wp = __ldg(a.p.window + o);
        const float win = a.ndim == 1 ? expf(-wp * (float)pos) : expf(-r2 / (2.f * wp * wp));
        if (ok) a.out[o * a.out_stride + off] = win * acc;
    }
}

}  // namespace hyena
