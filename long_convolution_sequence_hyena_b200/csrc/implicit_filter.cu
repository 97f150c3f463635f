// Implicit filter network launch.
#include "launch.h"

namespace hyena {

__global__ void __launch_bounds__(IMP_THREADS) hyena_implicit_filter_kernel(const ImplicitArgs a) {
    extern __shared__ float4 imp_smem4[];
    ImplicitSmem &S = *reinterpret_cast<ImplicitSmem *>(imp_smem4);
    const int width = a.p.width;
    const int fin = a.ndim == 1 ? 1 + 2 * a.p.num_freqs : 2;
    const int64_t p0 = (int64_t)blockIdx.x * IMP_TP;
    const int tid = threadIdx.x;

    // positional features
    for (int i = tid; i < IMP_TP * fin; i += IMP_THREADS) {
        const int pl = i / fin, f = i - pl * fin;
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
        S.u.in.feat[pl][f] = val;
    }
    __syncthreads();
    // first sine layer
    for (int i = tid; i < IMP_TP * width; i += IMP_THREADS) {
        const int pl = i / width, j = i - pl * width;
        float acc = __ldg(a.p.b1 + j);
        for (int f = 0; f < fin; ++f) acc = fmaf(__ldg(a.p.W1 + (int64_t)j * fin + f), S.u.in.feat[pl][f], acc);
        S.u.in.h1[pl][j] = sinf(a.p.omega0 * acc);
    }
    __syncthreads();
    // second sine layer, stored [unit][position] for the head
    for (int i = tid; i < IMP_TP * width; i += IMP_THREADS) {
        const int j = i / IMP_TP, pl = i - j * IMP_TP;
        float acc = __ldg(a.p.b2 + j);
        for (int f = 0; f < width; ++f) acc = fmaf(__ldg(a.p.W2 + (int64_t)j * width + f), S.u.in.h1[pl][f], acc);
        S.a2[j][pl] = sinf(a.p.omega_hidden * acc);
    }

    // head + window: thread (ty, tx) owns outputs 4 ty..4 ty+3 and positions 4 tx..4 tx+3 of a tile
    const int tx = tid & 15, ty = tid >> 4;
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
        __syncthreads();   // previous tile's reads of w3 (and the a2 writes above) complete
        for (int i = tid; i < IMP_OT * width; i += IMP_THREADS) {
            const int r = i / width, j = i - r * width;
            S.u.w3[r][j] = ob + r < a.nout ? __ldg(a.p.W3 + (ob + r) * width + j) : 0.f;
        }
        __syncthreads();
        float acc[4][4];
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;
        for (int j = 0; j < width; ++j) {
            const float4 b = *reinterpret_cast<const float4 *>(&S.a2[j][4 * tx]);
            float wv[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) wv[r] = S.u.w3[4 * ty + r][j];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                acc[r][0] = fmaf(wv[r], b.x, acc[r][0]);
                acc[r][1] = fmaf(wv[r], b.y, acc[r][1]);
                acc[r][2] = fmaf(wv[r], b.z, acc[r][2]);
                acc[r][3] = fmaf(wv[r], b.w, acc[r][3]);
            }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const int64_t o = ob + 4 * ty + r;
            if (o >= o_end) break;
            const float bias = __ldg(a.p.b3 + o);
            const float wp = __ldg(a.p.window + o);
            float *orow = a.out + o * a.out_stride;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                if (!ok[c]) continue;
                const int64_t pos = p0 + 4 * tx + c;
                const float win = a.ndim == 1 ? expf(-wp * (float)pos)
                                              : expf(-(wy[c] * wy[c] + wx[c] * wx[c]) / (2.f * wp * wp));
                orow[off[c]] = win * (acc[r][c] + bias);
            }
        }
    }
}

cudaError_t launch_implicit(const ImplicitArgs &a, cudaStream_t st) {
    const size_t sm = sizeof(ImplicitSmem);
    cudaError_t e = cudaFuncSetAttribute(hyena_implicit_filter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((a.npos + IMP_TP - 1) / IMP_TP), (unsigned)((a.nout + IMP_OSPLIT - 1) / IMP_OSPLIT));
    hyena_implicit_filter_kernel<<<grid, IMP_THREADS, sm, st>>>(a);
    return cudaGetLastError();
}

}  // namespace hyena
