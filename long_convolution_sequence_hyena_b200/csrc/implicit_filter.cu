// Implicit filter network launch.
#include "launch.h"

namespace hyena {

cudaError_t launch_implicit(const ImplicitArgs &a, cudaStream_t st) {
    const int64_t grid = (a.npos + IMP_TP - 1) / IMP_TP;
    if (a.p.width <= 64)
        hyena_implicit_filter_kernel<64><<<(unsigned)grid, IMP_THREADS, 0, st>>>(a);
    else
        hyena_implicit_filter_kernel<128><<<(unsigned)grid, IMP_THREADS, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace hyena
