// Plan object behind the opaque hyena_plan_t handle.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "hyena.h"

#define HYENA_MAX_L_1D 524288    // longest 1D sequence (M = 1048576)
#define HYENA_MAX_M_CTA 32768    // longest padded length the single-CTA path runs
#define HYENA_SUB_TWIDDLES 1024  // W_1024 table appended to the main one (cluster sub-transforms)

struct hyena_plan_s {
    int ndim = 1;
    int64_t D = 0;               // channels
    int order = 0;
    hyena_dtype_t dtype = HYENA_F32;
    int path = HYENA_PATH_CTA;
    int layout = HYENA_LAYOUT_BDL;   // activation layout (hyena_plan_set_layout)
    int device = 0;
    // 1D geometry
    int64_t L = 0;               // sequence length
    int64_t M = 0;               // padded real FFT length, next_pow2(2L) (at least 32)
    int64_t MC = 0;              // M / 2: length of the packed complex FFT
    int64_t P3 = 0;              // M = 6 P3 (a radix-3 length, HYENA_PLAN_RADIX3), else 0
    // 2D geometry
    int64_t Hh = 0, Ww = 0;      // grid extents (the transform is 2H x 2W)
    int64_t Dd = 0;              // 3D: depth (the transform is 2Dz x 2H x 2W)
    int64_t spectrum_elems = 0;  // complex bins per (order, channel)
    // device tables (owned)
    int64_t tw_len = 0;          // 1D: M; 2D: 2W
    float2 *tw = nullptr;        // W_tw_len^m, m in [0, tw_len), then W_1024^m, m in [0, 1024)
    // staged paths: two non-blocking streams; each call forks them off its
    // stream and joins them back with events of its own
    bool has_lanes = false;
    cudaStream_t lane[8] = {};   // the first HYENA_STAGED_LANES are created
    // staged spectra (1D long rows, 2D 256x256): scratch for two chunks of
    // transforms (owned). Chunk slot i is only ever used by lane i, and the
    // mutex keeps each call's launch sequence together on the lanes, so calls
    // from several threads run one after the other on the GPU.
    float2 *spec_ws = nullptr;
    std::mutex *spec_mu = nullptr;
    // device error word (owned): set by a kernel whose bounded wait timed out
    int *dev_err = nullptr;
};

namespace hyena {

// Rows of a staged 1D chunk (one lane's workspace slot) at packed length MC.
int64_t staged_chunk_rows(int64_t MC);
// Scratch a 1D forward over `rows` channel rows needs (0 off the staged path).
size_t workspace_bytes_1d(hyena_plan_t plan, int64_t rows);
// The 1D forward over channels [d0, d0 + dc) of one batch element of a
// [B, D, L] plan: v, the gates and y hold those dc rows; H and Dskip are the
// plan's whole tensors. Same kernels, so each row equals hyena_forward's.
hyena_status_t forward_channels_1d(hyena_plan_t plan, int64_t d0, int64_t dc, const void *v, const void *const *gates,
                                   const void *H, const float *Dskip, void *y, void *workspace, size_t ws_bytes,
                                   void *stream);

}  // namespace hyena
