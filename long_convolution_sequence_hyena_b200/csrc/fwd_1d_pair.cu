// 1D paired-row kernels (two rows of one channel per thread group, packed
// fp32x2): instantiations and launch.
#include "kernels_1d_pair.cuh"
#include "launch.h"

namespace hyena {

template <int MC, typename IO, bool EVEN>
cudaError_t launch_fwd_1d_pair_t(const Fwd1dArgs &a, cudaStream_t st) {
    constexpr int E = 16;
    constexpr int PPC = pair_pairs_per_cta(MC, E);
    // With 256 threads and more (128 registers), order 2 runs the unrolled
    // chain, which needs fewer registers than the loop (4.8 % faster at
    // MC = 8192). With 128 threads the loop is faster (the unrolled chain at
    // MC = 2048 was 19 % slower).
    auto kern = hyena_fwd_1d_pair<MC, E, IO, EVEN, 0>;
    if constexpr (pair_threads(MC, E) >= 256)
        if (a.order == 2) kern = hyena_fwd_1d_pair<MC, E, IO, EVEN, 2>;
    const size_t sm = pair_smem_bytes<IO, EVEN>(MC, E);
    if (sm > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
    }
    const int64_t npairs = a.rows / 2;
    const int64_t grid = (npairs + PPC - 1) / PPC;
    kern<<<(unsigned)grid, pair_threads(MC, E), sm, st>>>(a);
    return launched();
}

template <int MC>
cudaError_t launch_fwd_1d_pair_mc(const Fwd1dArgs &a, hyena_dtype_t dt, bool even, cudaStream_t st) {
    if (dt == HYENA_F32)
        return even ? launch_fwd_1d_pair_t<MC, float, true>(a, st) : launch_fwd_1d_pair_t<MC, float, false>(a, st);
    return even ? launch_fwd_1d_pair_t<MC, __nv_bfloat16, true>(a, st)
                : launch_fwd_1d_pair_t<MC, __nv_bfloat16, false>(a, st);
}

bool pair_path_supported(int64_t MC, int64_t B) { return B % 2 == 0 && MC >= 16 && MC <= 8192; }

cudaError_t launch_fwd_1d_pair(const Fwd1dArgs &a, int64_t MC, hyena_dtype_t dt, bool even, cudaStream_t st) {
    switch (MC) {
        case 16: return launch_fwd_1d_pair_mc<16>(a, dt, even, st);
        case 32: return launch_fwd_1d_pair_mc<32>(a, dt, even, st);
        case 64: return launch_fwd_1d_pair_mc<64>(a, dt, even, st);
        case 128: return launch_fwd_1d_pair_mc<128>(a, dt, even, st);
        case 256: return launch_fwd_1d_pair_mc<256>(a, dt, even, st);
        case 512: return launch_fwd_1d_pair_mc<512>(a, dt, even, st);
        case 1024: return launch_fwd_1d_pair_mc<1024>(a, dt, even, st);
        case 2048: return launch_fwd_1d_pair_mc<2048>(a, dt, even, st);
        case 4096: return launch_fwd_1d_pair_mc<4096>(a, dt, even, st);
        case 8192: return launch_fwd_1d_pair_mc<8192>(a, dt, even, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace hyena
