#pragma once
// Count of the kernels this library has enqueued in the process, read through
// hyena_launch_count: every launch site notes its launches here.
#include <cuda_runtime.h>

namespace hyena {

void note_launch(int n = 1);
// Notes the launch just enqueued and returns its status.
inline cudaError_t launched() {
    note_launch(1);
    return cudaGetLastError();
}

}  // namespace hyena
