// 1D single-CTA kernels: fused forward and filter spectrum instantiations.
#include "launch.h"

namespace hyena {

// Elements per thread for each half-length MC (threads per row = MC / E).
constexpr int e_for(int MC) { return MC >= 16384 ? 32 : 16; }

template <int MC>
size_t smem_1d() {
    return (size_t)rows_per_cta(MC, e_for(MC)) * 2 * MC * sizeof(float);
}
template <int MC>
size_t smem_fwd_1d() {
    return (size_t)rows_per_cta(MC, e_for(MC)) * fwd_smem_floats_per_row(MC) * sizeof(float);
}

template <int MC, typename IO, bool EVEN>
cudaError_t launch_fwd_1d_t(const Fwd1dArgs &a, cudaStream_t st) {
    constexpr int E = e_for(MC);
    constexpr int RPC = rows_per_cta(MC, E);
    auto kern = hyena_fwd_1d_cta<MC, E, IO, EVEN>;
    const size_t sm = smem_fwd_1d<MC>();
    if (sm > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
    }
    const int64_t grid = (a.rows + RPC - 1) / RPC;
    kern<<<(unsigned)grid, RPC * (MC / E), sm, st>>>(a);
    return launched();
}

template <int MC>
cudaError_t launch_fwd_1d_mc(const Fwd1dArgs &a, hyena_dtype_t dt, bool even, cudaStream_t st) {
    if (dt == HYENA_F32)
        return even ? launch_fwd_1d_t<MC, float, true>(a, st) : launch_fwd_1d_t<MC, float, false>(a, st);
    return even ? launch_fwd_1d_t<MC, __nv_bfloat16, true>(a, st) : launch_fwd_1d_t<MC, __nv_bfloat16, false>(a, st);
}

template <int MC>
cudaError_t launch_spec_1d_mc(const float *h, int64_t h_stride, int64_t L, c32 *Hout, int64_t nrows, const c32 *tw,
                              cudaStream_t st) {
    constexpr int E = e_for(MC);
    constexpr int RPC = rows_per_cta(MC, E);
    auto kern = hyena_spectrum_1d<MC, E>;
    const size_t sm = smem_1d<MC>();
    if (sm > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
    }
    const int64_t grid = (nrows + RPC - 1) / RPC;
    kern<<<(unsigned)grid, RPC * (MC / E), sm, st>>>(h, h_stride, L, Hout, nrows, tw);
    return launched();
}

#define HY_MC_SWITCH(MCV, CALL)     \
    switch (MCV) {                  \
        case 16: return CALL(16);   \
        case 32: return CALL(32);   \
        case 64: return CALL(64);   \
        case 128: return CALL(128); \
        case 256: return CALL(256); \
        case 512: return CALL(512); \
        case 1024: return CALL(1024); \
        case 2048: return CALL(2048); \
        case 4096: return CALL(4096); \
        case 8192: return CALL(8192); \
        case 16384: return CALL(16384); \
        default: return cudaErrorInvalidValue; \
    }

cudaError_t launch_fwd_1d(const Fwd1dArgs &a, int64_t MC, hyena_dtype_t dt, bool even, cudaStream_t st) {
#define HY_CALL(X) launch_fwd_1d_mc<X>(a, dt, even, st)
    HY_MC_SWITCH(MC, HY_CALL)
#undef HY_CALL
}

cudaError_t launch_spec_1d(const float *h, int64_t h_stride, int64_t L, c32 *Hout, int64_t nrows, int64_t MC,
                           const c32 *tw, cudaStream_t st) {
#define HY_CALL(X) launch_spec_1d_mc<X>(h, h_stride, L, Hout, nrows, tw, st)
    HY_MC_SWITCH(MC, HY_CALL)
#undef HY_CALL
}

}  // namespace hyena
