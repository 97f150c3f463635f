// 1D kernels for padded lengths M = 6 P (P = 16 .. 4096): instantiations and launch.
#include "kernels_1d_mr.cuh"
#include "launch.h"

namespace hyena {

bool mr3_supported(int64_t P) { return P >= 16 && P <= 4096 && (P & (P - 1)) == 0; }

namespace {

template <int P, typename IO, bool EVEN>
cudaError_t launch_t(const Fwd1dArgs &a, cudaStream_t st) {
    using G = MR3<P>;
    auto kern = hyena_fwd_1d_mr3<P, IO, EVEN>;
    const size_t sm = (size_t)G::RPC * G::SMEM_FLOATS * sizeof(float);
    if (sm > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
    }
    kern<<<(unsigned)((a.rows + G::RPC - 1) / G::RPC), G::THREADS, sm, st>>>(a);
    return launched();
}

template <int P>
cudaError_t launch_p(const Fwd1dArgs &a, hyena_dtype_t dt, bool even, cudaStream_t st) {
    if (dt == HYENA_F32) return even ? launch_t<P, float, true>(a, st) : launch_t<P, float, false>(a, st);
    return even ? launch_t<P, __nv_bfloat16, true>(a, st) : launch_t<P, __nv_bfloat16, false>(a, st);
}

template <int P>
cudaError_t launch_spec_p(const float *h, int64_t hs, int64_t L, c32 *Hout, int64_t nrows, const c32 *tw,
                          cudaStream_t st) {
    using G = MR3<P>;
    const size_t sm = (size_t)G::RPC * G::SMEM_FLOATS * sizeof(float);
    if (sm > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(hyena_spectrum_1d_mr3<P>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
    }
    hyena_spectrum_1d_mr3<P><<<(unsigned)((nrows + G::RPC - 1) / G::RPC), G::THREADS, sm, st>>>(h, hs, L, Hout,
                                                                                              nrows, tw);
    return launched();
}

}  // namespace

cudaError_t launch_fwd_1d_mr3(const Fwd1dArgs &a, int64_t P, hyena_dtype_t dt, bool even, cudaStream_t st) {
    switch (P) {
#define MR_CASE(PP) case PP: return launch_p<PP>(a, dt, even, st);
        MR_CASE(16) MR_CASE(32) MR_CASE(64) MR_CASE(128) MR_CASE(256) MR_CASE(512) MR_CASE(1024) MR_CASE(2048)
        MR_CASE(4096)
#undef MR_CASE
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_spec_1d_mr3(const float *h, int64_t h_stride, int64_t L, c32 *Hout, int64_t nrows, int64_t P,
                               const c32 *tw, cudaStream_t st) {
    switch (P) {
#define MR_CASE(PP) case PP: return launch_spec_p<PP>(h, h_stride, L, Hout, nrows, tw, st);
        MR_CASE(16) MR_CASE(32) MR_CASE(64) MR_CASE(128) MR_CASE(256) MR_CASE(512) MR_CASE(1024) MR_CASE(2048)
        MR_CASE(4096)
#undef MR_CASE
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace hyena
