// 2D staged path (H = W = 256): instantiations and the per-chunk launch sequence.
#include "kernels_2d_staged.cuh"
#include "launch.h"

namespace hyena {

using GS2_256 = Staged2dGeom<256>;

bool staged2d_supported(int64_t W) { return W == 256; }

int64_t staged2d_chunk_planes(int64_t W) {
    // planes whose transforms ([2H][W/2] complex64 each) fill 32 MB; two chunks in flight
    const int64_t r = ((int64_t)32 << 20) / (2 * W * (W / 2) * 8);
    return r < 1 ? 1 : r;
}

int64_t staged2d_workspace_planes(int64_t W, int64_t planes) {
    const int64_t r = staged2d_chunk_planes(W);
    return planes <= r ? planes : 2 * r;
}

template <typename G, typename IO, bool GATED>
cudaError_t launch_staged2d_io(const Fwd2dArgs &f, float2 *ws, int64_t chunk, const cudaStream_t *lanes, int nst) {
    cudaError_t e = cudaFuncSetAttribute(hyena_staged2d_rows_x2<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)G::RSMEM);
    if (e != cudaSuccess) return e;
    for (int64_t o0 = 0, c = 0; o0 < f.planes; o0 += chunk, ++c) {
        const int64_t np = (f.planes - o0) < chunk ? (f.planes - o0) : chunk;
        const cudaStream_t st = lanes[c % nst];
        Staged2dArgs a;
        a.f = f;
        a.ws = ws + (c % nst) * chunk * G::PLANE;
        a.o0 = o0;
        a.n = 0;
        const unsigned cgrid = (unsigned)(np * G::CGROUPS), rgrid = (unsigned)((np + 1) / 2 * G::RGROUPS);
        hyena_staged2d_cols<G, IO, 0, GATED><<<cgrid, G::CT, G::CSMEM, st>>>(a);
        for (int n = 0; n < f.order; ++n) {
            a.n = n;
            hyena_staged2d_rows_x2<G><<<rgrid, G::RT, G::RSMEM, st>>>(a, np);
            if (n + 1 < f.order)
                hyena_staged2d_cols<G, IO, 1, GATED><<<cgrid, G::CT, G::CSMEM, st>>>(a);
            else
                hyena_staged2d_cols<G, IO, 2, GATED><<<cgrid, G::CT, G::CSMEM, st>>>(a);
        }
        note_launch(2 * f.order + 1);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

int64_t staged2d_spec_chunk(int64_t W) { return W == 256 ? 16 : 0; }

size_t staged2d_spec_scratch_bytes(int64_t W) {
    return W == 256 ? (size_t)2 * staged2d_spec_chunk(W) * (2 * W) * W * sizeof(float2) : 0;
}

cudaError_t launch_spec_2d_staged(const float *K, int64_t rs, int64_t cs, c32 *Kout, int64_t n, int64_t W,
                                  const c32 *tw, float2 *scratch, cudaStream_t st, const StagedLanes &sl) {
    using G = GS2_256;
    if (W != 256) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(hyena_staged2d_spec_rows_x2<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)G::RSMEM);
    if (e != cudaSuccess) return e;
    const int64_t chunk = staged2d_spec_chunk(W);
    const int64_t per = (int64_t)G::M1 * G::M2;
    auto run = [&](const cudaStream_t *lanes, int nst) -> cudaError_t {
        for (int64_t o0 = 0, c = 0; o0 < n; o0 += chunk, ++c) {
            Spec2dArgs a;
            a.K = K;
            a.rs = rs;
            a.cs = cs;
            a.Kout = Kout;
            a.tw = tw;
            a.ws = scratch + (c % nst) * chunk * per;
            a.o0 = o0;
            a.nk = (n - o0) < chunk ? (n - o0) : chunk;
            const cudaStream_t s = lanes[c % nst];
            hyena_staged2d_spec_cols<G><<<(unsigned)(a.nk * (G::M2 / G::NCOL)), G::CT, G::CSMEM, s>>>(a);
            hyena_staged2d_spec_rows_x2<G><<<(unsigned)((a.nk + 1) / 2 * G::RGROUPS), G::RT, G::RSMEM, s>>>(a);
            note_launch(2);
            const cudaError_t le = cudaGetLastError();
            if (le != cudaSuccess) return le;
        }
        return cudaSuccess;
    };
    // always on the plan's lanes, one chunk too: scratch slot i is used by lane i only
    e = cudaEventRecord(sl.fork, st);
    for (int i = 0; i < 2 && e == cudaSuccess; ++i) e = cudaStreamWaitEvent(sl.lane[i], sl.fork, 0);
    if (e != cudaSuccess) return e;
    const cudaError_t le = run(sl.lane, 2);
    for (int i = 0; i < 2; ++i) {
        e = cudaEventRecord(sl.join[i], sl.lane[i]);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(st, sl.join[i], 0);
        if (e != cudaSuccess) return e;
    }
    return le;
}

cudaError_t launch_fwd_2d_staged(const Fwd2dArgs &f, int64_t W, float2 *ws, hyena_dtype_t dt, cudaStream_t st,
                                 const StagedLanes &sl) {
    if (W != 256) return cudaErrorInvalidValue;
    const int64_t chunk = staged2d_chunk_planes(W);
    auto run = [&](const cudaStream_t *lanes, int nst) -> cudaError_t {
        if (f.k)
            return dt == HYENA_F32 ? launch_staged2d_io<GS2_256, float, true>(f, ws, chunk, lanes, nst)
                                   : launch_staged2d_io<GS2_256, __nv_bfloat16, true>(f, ws, chunk, lanes, nst);
        return dt == HYENA_F32 ? launch_staged2d_io<GS2_256, float, false>(f, ws, chunk, lanes, nst)
                               : launch_staged2d_io<GS2_256, __nv_bfloat16, false>(f, ws, chunk, lanes, nst);
    };
    if (f.planes <= chunk) return run(&st, 1);
    return run_on_lanes(st, sl, 2, run);
}

}  // namespace hyena
