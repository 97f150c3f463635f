// 2D cluster kernels: fused forward and kernel spectrum instantiations.
#include "launch.h"
#include "cluster_launch.cuh"
#include "kernels_2d.cuh"

namespace hyena {

template <typename G>
cudaError_t launch_fwd_2d_g(const Fwd2dArgs &a, hyena_dtype_t dt, cudaStream_t st) {
    const bool gated = a.k != nullptr;
    if (dt == HYENA_F32)
        return gated ? launch_cluster<G>(hyena_fwd_2d_cluster<G, float, true>, a.planes, st, a)
                     : launch_cluster<G>(hyena_fwd_2d_cluster<G, float, false>, a.planes, st, a);
    return gated ? launch_cluster<G>(hyena_fwd_2d_cluster<G, __nv_bfloat16, true>, a.planes, st, a)
                 : launch_cluster<G>(hyena_fwd_2d_cluster<G, __nv_bfloat16, false>, a.planes, st, a);
}

cudaError_t launch_fwd_2d(const Fwd2dArgs &a, int64_t W, hyena_dtype_t dt, cudaStream_t st) {
    switch (W) {
        case 32: return launch_fwd_2d_g<G2_32>(a, dt, st);
        case 64: return launch_fwd_2d_g<G2_64>(a, dt, st);
        case 128: return launch_fwd_2d_g<G2_128>(a, dt, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_spec_2d(const float *K, int64_t rs, int64_t cs, c32 *Kout, int64_t n, int64_t W, const c32 *tw,
                           cudaStream_t st) {
    switch (W) {
        case 32: return launch_cluster<G2_32>(hyena_spectrum_2d_cluster<G2_32>, n, st, K, rs, cs, Kout, tw);
        case 64: return launch_cluster<G2_64>(hyena_spectrum_2d_cluster<G2_64>, n, st, K, rs, cs, Kout, tw);
        case 128: return launch_cluster<G2_128>(hyena_spectrum_2d_cluster<G2_128>, n, st, K, rs, cs, Kout, tw);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace hyena
