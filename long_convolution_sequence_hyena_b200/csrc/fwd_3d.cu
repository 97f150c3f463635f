// 3D staged path: instantiations and the per-chunk launch sequence.
#include "kernels_3d.cuh"
#include "launch.h"

namespace hyena {

bool grid3d_supported(int64_t Dz, int64_t H, int64_t W) {
    auto ok = [](int64_t e) { return e == 16 || e == 32 || e == 64; };
    return ok(Dz) && ok(H) && ok(W);
}

int64_t grid3d_chunk_volumes(int64_t Dz, int64_t H, int64_t W) {
    // volumes whose workspaces ([Dz][2H][2W] complex64 each) fill 32 MB
    const int64_t r = ((int64_t)32 << 20) / (Dz * 2 * H * 2 * W * 8);
    return r < 1 ? 1 : r;
}

namespace {

template <typename IO, int MODE, bool G>
cudaError_t launch_x(const Fwd3dArgs &a, cudaStream_t st) {
    const int64_t rows = a.np * a.Dz * a.H;
    switch (2 * a.W) {
#define X_CASE(LX)                                                                                          \
    case LX:                                                                                                \
        hyena_3d_x<LX, IO, MODE, G><<<(unsigned)((rows + Stage3<LX>::NSEQ - 1) / Stage3<LX>::NSEQ),        \
                                      S3_THREADS, 0, st>>>(a);                                              \
        return launched();
        X_CASE(32) X_CASE(64) X_CASE(128)
#undef X_CASE
        default: return cudaErrorInvalidValue;
    }
}

template <int DIR>
cudaError_t launch_y(const Fwd3dArgs &a, cudaStream_t st) {
    const int64_t cols = a.np * a.Dz * 2 * a.W;
    switch (2 * a.H) {
#define Y_CASE(LY)                                                                                          \
    case LY:                                                                                                \
        hyena_3d_y<LY, DIR><<<(unsigned)((cols + Stage3<LY>::NSEQ - 1) / Stage3<LY>::NSEQ), S3_THREADS, 0,  \
                              st>>>(a);                                                                     \
        return launched();
        Y_CASE(32) Y_CASE(64) Y_CASE(128)
#undef Y_CASE
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_z(const Fwd3dArgs &a, cudaStream_t st) {
    const int64_t cols = a.np * 2 * a.H * 2 * a.W;
    switch (2 * a.Dz) {
#define Z_CASE(LZ)                                                                                          \
    case LZ:                                                                                                \
        hyena_3d_z<LZ><<<(unsigned)((cols + Stage3<LZ>::NSEQ - 1) / Stage3<LZ>::NSEQ), S3_THREADS, 0, st>>>(a); \
        return launched();
        Z_CASE(32) Z_CASE(64) Z_CASE(128)
#undef Z_CASE
        default: return cudaErrorInvalidValue;
    }
}

template <typename IO, bool G>
cudaError_t run_chunk(Fwd3dArgs a, cudaStream_t st) {
    cudaError_t e = launch_x<IO, 0, G>(a, st);
    if (e == cudaSuccess) e = launch_y<-1>(a, st);
    for (int n = 0; n < a.order && e == cudaSuccess; ++n) {
        a.n = n;
        e = launch_z(a, st);
        if (e == cudaSuccess) e = launch_y<+1>(a, st);
        if (e != cudaSuccess) break;
        if (n + 1 < a.order) {
            e = launch_x<IO, 1, G>(a, st);
            if (e == cudaSuccess) e = launch_y<-1>(a, st);
        } else {
            e = launch_x<IO, 2, G>(a, st);
        }
    }
    return e;
}

}  // namespace

cudaError_t launch_fwd_3d(const Fwd3dArgs &base, int64_t volumes, hyena_dtype_t dt, cudaStream_t st) {
    const int64_t chunk = grid3d_chunk_volumes(base.Dz, base.H, base.W);
    for (int64_t o0 = 0; o0 < volumes; o0 += chunk) {
        Fwd3dArgs a = base;
        a.o0 = o0;
        a.np = volumes - o0 < chunk ? volumes - o0 : chunk;
        const bool g = a.k != nullptr;
        const cudaError_t e = dt == HYENA_F32 ? (g ? run_chunk<float, true>(a, st) : run_chunk<float, false>(a, st))
                                              : (g ? run_chunk<__nv_bfloat16, true>(a, st)
                                                   : run_chunk<__nv_bfloat16, false>(a, st));
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_spec_3d(const float *K, int64_t cs, c32 *Kout, int64_t n, int Dz, int H, int W, const c32 *tws,
                           cudaStream_t st) {
    Spec3dArgs a;
    a.Kin = K;
    a.cs = cs;
    a.Kout = Kout;
    a.tws = tws;
    a.n = n;
    a.Dz = Dz;
    a.H = H;
    a.W = W;
    const int64_t rows = n * 2 * Dz * 2 * H, ycols = n * 2 * Dz * 2 * W, zcols = n * 2 * H * 2 * W;
    switch (2 * W) {
#define SX(LX) case LX: hyena_3d_spec_x<LX><<<(unsigned)((rows + Stage3<LX>::NSEQ - 1) / Stage3<LX>::NSEQ), S3_THREADS, 0, st>>>(a); note_launch(); break;
        SX(32) SX(64) SX(128)
#undef SX
        default: return cudaErrorInvalidValue;
    }
    switch (2 * H) {
#define SY(LY) case LY: hyena_3d_spec_col<LY, 1><<<(unsigned)((ycols + Stage3<LY>::NSEQ - 1) / Stage3<LY>::NSEQ), S3_THREADS, 0, st>>>(a); note_launch(); break;
        SY(32) SY(64) SY(128)
#undef SY
        default: return cudaErrorInvalidValue;
    }
    switch (2 * Dz) {
#define SZ(LZ) case LZ: hyena_3d_spec_col<LZ, 2><<<(unsigned)((zcols + Stage3<LZ>::NSEQ - 1) / Stage3<LZ>::NSEQ), S3_THREADS, 0, st>>>(a); note_launch(); break;
        SZ(32) SZ(64) SZ(128)
#undef SZ
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace hyena
