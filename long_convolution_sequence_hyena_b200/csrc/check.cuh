#pragma once
// Index checks of the HYENA_CHECK_BOUNDS debug build (libhyena_checked.so).
// Where compute-sanitizer cannot run, that build checks the indices the
// kernels compute before they use them: rows of the activation tensors and of
// the spectrum, offsets into the staged workspace and into shared memory. A
// failed check sets HYENA_DEVERR_BOUNDS in the plan's device error word (read
// with hyena_plan_device_errors) and the access it guards is skipped: nothing
// traps. In the normal build every check is the constant true.
#include <cuda_runtime.h>
#include <stdint.h>

#include "hyena.h"

namespace hyena {

// i in [0, n)?
__device__ __forceinline__ bool check_index(int *err, int64_t i, int64_t n) {
#ifdef HYENA_CHECK_BOUNDS
    if (i >= 0 && i < n) return true;
    if (err) atomicOr(err, HYENA_DEVERR_BOUNDS);
    return false;
#else
    (void)err;
    (void)i;
    (void)n;
    return true;
#endif
}

}  // namespace hyena
