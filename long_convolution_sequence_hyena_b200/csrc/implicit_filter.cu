// Implicit filter network launch.
#include "launch.h"

namespace hyena {

// Thread (ty, tx) accumulates rows 4 ty..4 ty+3 of the weight tile (stored
// [input][row]) against positions 4 tx..4 tx+3 of in[k][IMP_TP]: per input k,
// one 16-byte load of weights and one of activations feed 16 FMAs.
__device__ __forceinline__ void tile_product(const ImplicitSmem &S, const float (*in)[IMP_TP], int K, int tx, int ty,
                                             float (&acc)[4][4]) {
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;
#pragma unroll 4
    for (int k = 0; k < K; ++k) {
        const float4 b = *reinterpret_cast<const float4 *>(&in[k][4 * tx]);
        const float4 w4 = *reinterpret_cast<const float4 *>(&S.wt[k][4 * ty]);
        const float wr[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            acc[r][0] = fmaf(wr[r], b.x, acc[r][0]);
            acc[r][1] = fmaf(wr[r], b.y, acc[r][1]);
            acc[r][2] = fmaf(wr[r], b.z, acc[r][2]);
            acc[r][3] = fmaf(wr[r], b.w, acc[r][3]);
        }
    }
}

// Weight rows [j0, j0 + IMP_OT) of W ([J][K], row-major) into the tile (zero past J).
__device__ __forceinline__ void load_weight_tile(ImplicitSmem &S, const float *__restrict__ W, int64_t j0, int64_t J,
                                                 int K, int tid) {
    for (int i = tid; i < IMP_OT * K; i += IMP_THREADS) {
        const int r = i / K, k = i - r * K;   // coalesced reads along k
        S.wt[k][r] = j0 + r < J ? __ldg(W + (j0 + r) * K + k) : 0.f;
    }
}

// out[j][p] = sin(omega (b[j] + sum_k W[j][k] in[k][p])), j < J (a sine layer).
// Ends with every write of out visible to the CTA.
__device__ __forceinline__ void sine_layer(ImplicitSmem &S, const float *__restrict__ W, const float *__restrict__ b,
                                           int K, int J, float omega, const float (*in)[IMP_TP],
                                           float (*out)[IMP_TP], int tid, int tx, int ty) {
    for (int j0 = 0; j0 < J; j0 += IMP_OT) {
        __syncthreads();   // earlier readers of the weight tile done; `in` complete
        load_weight_tile(S, W, j0, J, K, tid);
        __syncthreads();
        float acc[4][4];
        tile_product(S, in, K, tx, ty, acc);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int j = j0 + 4 * ty + r;
            if (j >= J) break;
            const float bias = __ldg(b + j);
#pragma unroll
            for (int c = 0; c < 4; ++c) out[j][4 * tx + c] = sinf(omega * (acc[r][c] + bias));
        }
    }
    __syncthreads();
}

__global__ void __launch_bounds__(IMP_THREADS) hyena_implicit_filter_kernel(const ImplicitArgs a) {
    extern __shared__ float4 imp_smem4[];
    ImplicitSmem &S = *reinterpret_cast<ImplicitSmem *>(imp_smem4);
    const int width = a.p.width;
    const int fin = a.ndim == 1 ? 1 + 2 * a.p.num_freqs : 2;
    const int64_t p0 = (int64_t)blockIdx.x * IMP_TP;
    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;

    // positional features, stored [feature][position] in the second activation buffer
    float (*feat)[IMP_TP] = S.act[1];
    for (int i = tid; i < IMP_TP * fin; i += IMP_THREADS) {
        const int f = i / IMP_TP, pl = i - f * IMP_TP;
        const int64_t pos = p0 + pl;
        float val = 0.f;
        if (pos < a.npos) {
            if (a.ndim == 1) {
                if (f == 0) {
                    val = (float)((double)pos / (double)a.L);
                } else {
                    const int64_t k = (f + 1) / 2;
                    const int64_t r = (k * pos) % a.L;   // angle 2 pi k t / L, reduced exactly first
                    float sv, cv;
                    sincospif((float)(2.0 * (double)r / (double)a.L), &sv, &cv);
                    val = (f & 1) ? cv : sv;
                }
            } else {
                const int64_t iy = pos / (2 * a.W), ix = pos - iy * (2 * a.W);
                val = f == 0 ? (float)((double)(iy - a.H) / (double)a.H) : (float)((double)(ix - a.W) / (double)a.W);
            }
        }
        feat[f][pl] = val;
    }
    // two sine layers: features -> act[0] -> act[1]
    sine_layer(S, a.p.W1, a.p.b1, fin, width, a.p.omega0, feat, S.act[0], tid, tx, ty);
    sine_layer(S, a.p.W2, a.p.b2, width, width, a.p.omega_hidden, S.act[0], S.act[1], tid, tx, ty);

    // head + window: thread (ty, tx) owns outputs 4 ty..4 ty+3 and positions 4 tx..4 tx+3 of a tile
    float wy[4], wx[4];                        // 2D window coordinates of this thread's positions
    int64_t off[4];
    bool ok[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int64_t pos = p0 + 4 * tx + c;
        ok[c] = pos < a.npos;
        wy[c] = wx[c] = 0.f;
        off[c] = pos;
        if (a.ndim == 2 && ok[c]) {
            const int64_t iy = pos / (2 * a.W), ix = pos - iy * (2 * a.W);
            wy[c] = (float)((double)(iy - a.H) / (double)a.H);
            wx[c] = (float)((double)(ix - a.W) / (double)a.W);
            off[c] = iy * a.out_row_stride + ix;
        }
    }
    const int64_t o_begin = (int64_t)blockIdx.y * IMP_OSPLIT;
    const int64_t o_end = o_begin + IMP_OSPLIT < a.nout ? o_begin + IMP_OSPLIT : a.nout;
    for (int64_t ob = o_begin; ob < o_end; ob += IMP_OT) {
        __syncthreads();   // previous tile's reads of the weight tile complete
        load_weight_tile(S, a.p.W3, ob, a.nout, width, tid);
        __syncthreads();
        float acc[4][4];
        tile_product(S, S.act[1], width, tx, ty, acc);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int64_t o = ob + 4 * ty + r;
            if (o >= o_end) break;
            const float bias = __ldg(a.p.b3 + o);
            const float wp = __ldg(a.p.window + o);
            // exp(-alpha t) (1D) or exp(-|p|^2 / (2 sigma^2)) (2D): one exponent scale per output
            const float esc = a.ndim == 1 ? -wp : -1.f / (2.f * wp * wp);
            float *orow = a.out + o * a.out_stride;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (!ok[c]) continue;
                const float e = a.ndim == 1 ? (float)(p0 + 4 * tx + c) : wy[c] * wy[c] + wx[c] * wx[c];
                orow[off[c]] = expf(esc * e) * (acc[r][c] + bias);
            }
        }
    }
}

cudaError_t launch_implicit(const ImplicitArgs &a, int *err, cudaStream_t st) {
    if (implicit_tc_supported(a)) return launch_implicit_tc(a, err, st);
    const size_t sm = sizeof(ImplicitSmem);
    cudaError_t e = cudaFuncSetAttribute(hyena_implicit_filter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((a.npos + IMP_TP - 1) / IMP_TP), (unsigned)((a.nout + IMP_OSPLIT - 1) / IMP_OSPLIT));
    hyena_implicit_filter_kernel<<<grid, IMP_THREADS, sm, st>>>(a);
    return launched();
}

}  // namespace hyena
