// Implicit filter network: positional features -> two sine layers -> linear
// head -> window.
//
// 1D ("Hyena — Long Convolutions Math", "Implicit filters: an MLP over
// positions", "The decay window"):
//   features of t: [t/L, cos(2 pi k t/L), sin(2 pi k t/L) for k = 1..K]
//   window: exp(-alpha[o] * t)
// 2D ("How HyenaND works", "1. An implicit filter"):
//   features of offset (oy, ox): (oy/H, ox/W), oy in [-H, H), ox in [-W, W)
//   window: exp(-(py^2 + px^2) / (2 sigma[o]^2))
//
// One CTA per tile of IMP_TP positions and one slice of the outputs. Every
// layer is a dense contraction out[j][p] = sum_k W[j][k] in[k][p] over the
// tile's positions, computed as a register-blocked tiled product: each thread
// takes a 4-row x 4-position block of a 64 x 64 tile, with the weight tile in
// shared memory and the activations stored [unit][position].
#pragma once
#include "hyena.h"

namespace hyena {

constexpr int IMP_TP = 64;        // positions per CTA
constexpr int IMP_OT = 64;        // outputs per head tile
constexpr int IMP_THREADS = 256;  // 16 x 16 threads, each a 4 x 4 block of the 64 x 64 head tile
constexpr int IMP_MAXW = 128;     // maximum width
constexpr int IMP_MAXF = 65;      // maximum input features (1 + 2K, K <= 32)
constexpr int IMP_OSPLIT = 512;   // outputs per CTA slice (grid.y covers the rest)

struct ImplicitArgs {
    hyena_implicit_params_t p;
    int ndim;
    int64_t L;                 // 1D length
    int64_t H, W;              // 2D / 3D half-extents (grid is 2H x 2W offsets)
    int64_t Dz;                // 3D half-depth (grid is 2Dz x 2H x 2W offsets)
    int64_t npos;              // L or 4 H W
    int64_t nout;              // N * channels
    float *out;                // output base
    int64_t out_stride;        // floats between output channels
    int64_t out_row_stride;    // 2D: floats between rows of one channel (>= 2W)
};

struct ImplicitSmem {
    float act[2][IMP_MAXW][IMP_TP];     // activations [unit][position]; act[1] first holds the features
    float wt[IMP_MAXW][IMP_OT + 4];     // weight tile, transposed: [input][row] (a layer's 64 rows at a time)
};
static_assert(IMP_MAXF <= IMP_MAXW, "features are staged in an activation buffer");

// Defined in implicit_filter.cu (one translation unit).
__global__ void hyena_implicit_filter_kernel(const ImplicitArgs a);

}  // namespace hyena
