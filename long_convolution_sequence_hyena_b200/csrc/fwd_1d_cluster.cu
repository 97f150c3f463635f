// 1D cluster kernels: fused forward and filter spectrum instantiations
// (M = 262144; shorter long rows take the staged kernels).
#include "launch.h"
#include "cluster_launch.cuh"

namespace hyena {

// ------------------------------------------------------------- cluster paths
template <typename G>
cudaError_t launch_fwd_1d_cluster_g(const Fwd1dArgs &a, hyena_dtype_t dt, bool even, cudaStream_t st) {
    if (dt == HYENA_F32)
        return even ? launch_cluster<G>(hyena_fwd_1d_cluster<G, float, true>, a.rows, st, a)
                    : launch_cluster<G>(hyena_fwd_1d_cluster<G, float, false>, a.rows, st, a);
    return even ? launch_cluster<G>(hyena_fwd_1d_cluster<G, __nv_bfloat16, true>, a.rows, st, a)
                : launch_cluster<G>(hyena_fwd_1d_cluster<G, __nv_bfloat16, false>, a.rows, st, a);
}

bool cluster_path_supported(int64_t MC) { return MC == 131072; }

cudaError_t launch_fwd_1d_cluster(const Fwd1dArgs &a, int64_t MC, hyena_dtype_t dt, bool even, cudaStream_t st) {
    switch (MC) {
        case 131072: return launch_fwd_1d_cluster_g<G1_128K>(a, dt, even, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_spec_1d_cluster(const float *h, int64_t h_stride, int64_t L, c32 *Hout, int64_t nrows, int64_t MC,
                                   const c32 *tw, cudaStream_t st) {
    switch (MC) {
        case 131072:
            return launch_cluster<G1_128K>(hyena_spectrum_1d_cluster<G1_128K>, nrows, st, h, h_stride, L, Hout, tw);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace hyena
