#pragma once
// Launch wrappers shared by the translation units of the library.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "hyena.h"
#include "kernels_1d.cuh"
#include "kernels_implicit.cuh"
#include "launch_count.h"

namespace hyena {

// 1D, single CTA group per row (MC <= 16384)
cudaError_t launch_fwd_1d(const Fwd1dArgs &a, int64_t MC, hyena_dtype_t dt, bool even, cudaStream_t st);
cudaError_t launch_spec_1d(const float *h, int64_t h_stride, int64_t L, c32 *Hout, int64_t nrows, int64_t MC,
                           const c32 *tw, cudaStream_t st);
// 1D, padded length M = 6 P (MC = 3 P, P a power of two, 16..4096): one row per thread group
bool mr3_supported(int64_t P);
cudaError_t launch_fwd_1d_mr3(const Fwd1dArgs &a, int64_t P, hyena_dtype_t dt, bool even, cudaStream_t st);
cudaError_t launch_spec_1d_mr3(const float *h, int64_t h_stride, int64_t L, c32 *Hout, int64_t nrows, int64_t P,
                               const c32 *tw, cudaStream_t st);
// 1D, two rows of one channel per thread group (B even, MC <= 8192)
bool pair_path_supported(int64_t MC, int64_t B);
cudaError_t launch_fwd_1d_pair(const Fwd1dArgs &a, int64_t MC, hyena_dtype_t dt, bool even, cudaStream_t st);
// 1D, one cluster per row (MC = 131072)
bool cluster_path_supported(int64_t MC);
cudaError_t launch_fwd_1d_cluster(const Fwd1dArgs &a, int64_t MC, hyena_dtype_t dt, bool even, cudaStream_t st);
cudaError_t launch_spec_1d_cluster(const float *h, int64_t h_stride, int64_t L, c32 *Hout, int64_t nrows, int64_t MC,
                                   const c32 *tw, cudaStream_t st);
// 1D, staged four-step through a workspace (MC in {32768, 65536}); chunks of
// staged_chunk_rows(MC) rows, two in flight on the plan's lanes; workspace
// staged_workspace_rows(MC, rows) * MC complex64
// Lanes (plan-owned streams) of the staged paths: a staged 1D forward keeps
// HYENA_STAGED_LANES chunks of HYENA_STAGED_CHUNK_MB of transforms in flight,
// one per lane; spectra and the 2D path use the first two.
#ifndef HYENA_STAGED_LANES
#define HYENA_STAGED_LANES 3
#endif
#ifndef HYENA_STAGED_CHUNK_MB
#define HYENA_STAGED_CHUNK_MB 16
#endif
static_assert(HYENA_STAGED_LANES >= 2 && HYENA_STAGED_LANES <= 8, "lane count");
struct StagedLanes {
    cudaStream_t lane[HYENA_STAGED_LANES];     // non-blocking streams owned by the plan
    cudaEvent_t fork, join[HYENA_STAGED_LANES];   // events of the calling operation only
};
// Fork n lanes off `st`, run(lanes, n), join them back into `st` (also after a
// failed launch, so that `st` never runs ahead of the lanes).
template <typename F>
cudaError_t run_on_lanes(cudaStream_t st, const StagedLanes &sl, int n, F &&run) {
    cudaError_t e = cudaEventRecord(sl.fork, st);
    for (int i = 0; i < n && e == cudaSuccess; ++i) e = cudaStreamWaitEvent(sl.lane[i], sl.fork, 0);
    if (e != cudaSuccess) return e;
    const cudaError_t le = run(sl.lane, n);
    for (int i = 0; i < n; ++i) {
        e = cudaEventRecord(sl.join[i], sl.lane[i]);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(st, sl.join[i], 0);
        if (e != cudaSuccess) return e;
    }
    return le;
}
bool staged_path_supported(int64_t MC);
int64_t staged_chunk_rows(int64_t MC);
int64_t staged_workspace_rows(int64_t MC, int64_t rows);
cudaError_t launch_fwd_1d_staged(const Fwd1dArgs &a, int64_t MC, float2 *ws, hyena_dtype_t dt, bool even,
                                 cudaStream_t st, const StagedLanes &lanes);
// The same launch sequence with an explicit chunk (rows per workspace slot) and
// lanes: chunk c runs on lanes[c % nst] in slot c % nst of ws (nst slots).
cudaError_t launch_fwd_1d_staged_chunks(const Fwd1dArgs &f, int64_t MC, float2 *ws, int64_t chunk, hyena_dtype_t dt,
                                        bool even, const cudaStream_t *lanes, int nst);
// 1D filter spectra through the staged kernels, with plan-owned scratch of
// staged_spec_scratch_bytes(MC)
size_t staged_spec_scratch_bytes(int64_t MC);
cudaError_t launch_spec_1d_staged(const float *h, int64_t h_stride, int64_t L, c32 *Hout, int64_t nrows, int64_t MC,
                                  const c32 *tw, float2 *scratch, cudaStream_t st, const StagedLanes &lanes);
// 2D staged (H = W = 256): chunks of staged2d_chunk_planes(W) planes, two in flight;
// workspace staged2d_workspace_planes(W, planes) * 2H * W/2 complex64
struct Fwd2dArgs;
bool staged2d_supported(int64_t W);
int64_t staged2d_chunk_planes(int64_t W);
int64_t staged2d_workspace_planes(int64_t W, int64_t planes);
cudaError_t launch_fwd_2d_staged(const Fwd2dArgs &f, int64_t W, float2 *ws, hyena_dtype_t dt, cudaStream_t st,
                                 const StagedLanes &lanes);
// 2D kernel spectra through the staged kernels, with plan-owned scratch of
// staged2d_spec_scratch_bytes(W) (two chunks of staged2d_spec_chunk(W) kernels)
size_t staged2d_spec_scratch_bytes(int64_t W);
cudaError_t launch_spec_2d_staged(const float *K, int64_t rs, int64_t cs, c32 *Kout, int64_t n, int64_t W,
                                  const c32 *tw, float2 *scratch, cudaStream_t st, const StagedLanes &lanes);
// 2D, one cluster per plane (H == W in {32, 64, 128})
struct Fwd2dArgs;
cudaError_t launch_fwd_2d(const Fwd2dArgs &a, int64_t W, hyena_dtype_t dt, cudaStream_t st);
cudaError_t launch_spec_2d(const float *K, int64_t rs, int64_t cs, c32 *Kout, int64_t n, int64_t W, const c32 *tw,
                           cudaStream_t st);
// 3D grids (Dz, H, W each 16, 32 or 64): separable staged transforms through a
// workspace of grid3d_chunk_volumes volumes of [Dz][2H][2W] complex64
struct Fwd3dArgs;
bool grid3d_supported(int64_t Dz, int64_t H, int64_t W);
int64_t grid3d_chunk_volumes(int64_t Dz, int64_t H, int64_t W);
cudaError_t launch_fwd_3d(const Fwd3dArgs &a, int64_t volumes, hyena_dtype_t dt, cudaStream_t st);
cudaError_t launch_spec_3d(const float *K, int64_t cs, c32 *Kout, int64_t n, int Dz, int H, int W, const c32 *tws,
                           cudaStream_t st);
// implicit filter network: width 64 with the head on the tensor cores
// (implicit_tc.cu), other widths on the CUDA cores; err: the plan's device
// error word (bounded waits that time out set it)
cudaError_t launch_implicit(const ImplicitArgs &a, int *err, cudaStream_t st);
bool implicit_tc_supported(const ImplicitArgs &a);
cudaError_t launch_implicit_tc(const ImplicitArgs &a, int *err, cudaStream_t st);

}  // namespace hyena
