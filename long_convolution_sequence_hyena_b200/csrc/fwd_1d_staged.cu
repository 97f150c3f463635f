// 1D staged long-row path: instantiations and the per-chunk launch sequence.
#include "kernels_1d_staged.cuh"
#include "launch.h"

namespace hyena {

// two rows in lockstep per CTA; 128 threads (three or four CTAs per SM) up to
// M = 131072, then 256 and 512 threads for the longer columns and rows
using GS_32K = StagedGeom<32768, 128, 16, 8, 2>;    // M = 65536: columns of 128, rows of 256
using GS_64K = StagedGeom<65536, 256, 8, 8, 2>;     // M = 131072: 256 x 256
using GS_128K = StagedGeom<131072, 512, 8, 8, 2>;   // M = 262144: 512 x 256
using GS_256K = StagedGeom<262144, 512, 8, 8, 2>;   // M = 524288: 512 x 512
using GS_512K = StagedGeom<524288, 1024, 8, 8, 2>;  // M = 1048576: 1024 x 512

// Dynamic shared memory above the default 48 KB limit, for every kernel of a geometry.
template <typename G, typename IO, bool EVEN>
cudaError_t staged_smem_attrs() {
    cudaError_t e = cudaSuccess;
    if (G::CSMEM > 48 * 1024) {
        const int c = (int)G::CSMEM;
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(hyena_staged_cols_x2<G, IO, EVEN, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, c);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(hyena_staged_cols_x2<G, IO, EVEN, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, c);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(hyena_staged_cols_x2<G, IO, EVEN, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, c);
    }
    if (G::RSMEM > 48 * 1024 && e == cudaSuccess)
        e = cudaFuncSetAttribute(hyena_staged_rows_x2<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)G::RSMEM);
    return e;
}

int64_t staged_chunk_rows(int64_t MC) {
    // rows whose transforms (MC complex64 each) fill HYENA_STAGED_CHUNK_MB; one
    // chunk per lane is in flight at a time, which mostly stays in L2 between launches
    const int64_t r = ((int64_t)HYENA_STAGED_CHUNK_MB << 20) / (MC * 8);
    return r < 2 ? 2 : r & ~(int64_t)1;
}

int64_t staged_workspace_rows(int64_t MC, int64_t rows) {
    const int64_t r = staged_chunk_rows(MC);
    return rows <= r ? rows : HYENA_STAGED_LANES * r;
}

bool staged_path_supported(int64_t MC) {
    return MC == 32768 || MC == 65536 || MC == 131072 || MC == 262144 || MC == 524288;
}

// Chunk c runs on lane c % nst (a stream of its own) with its own workspace
// slot, so that two chunks' launch sequences overlap on the GPU.
template <typename G, typename IO, bool EVEN>
cudaError_t launch_staged_io(const Fwd1dArgs &f, float2 *ws, int64_t chunk, const cudaStream_t *lanes, int nst) {
    static_assert(G::ROWS == 2, "the launch sequence below runs the lockstep kernels");
    const cudaError_t ea = staged_smem_attrs<G, IO, EVEN>();
    if (ea != cudaSuccess) return ea;
    for (int64_t o0 = 0, c = 0; o0 < f.rows; o0 += chunk, ++c) {
        const int64_t nr = (f.rows - o0) < chunk ? (f.rows - o0) : chunk;
        const int64_t pairs = (nr + 1) / 2;
        const cudaStream_t st = lanes[c % nst];
        StagedArgs a;
        a.f = f;
        a.ws = ws + (c % nst) * chunk * G::MC;
        a.o0 = o0;
        a.n = 0;
        const unsigned cgrid = (unsigned)(pairs * G::CGROUPS), rgrid = (unsigned)(pairs * G::RGROUPS);
        hyena_staged_cols_x2<G, IO, EVEN, 0><<<cgrid, G::CT, G::CSMEM, st>>>(a, nr);
        for (int n = 0; n < f.order; ++n) {
            a.n = n;
            hyena_staged_rows_x2<G><<<rgrid, G::RT, G::RSMEM, st>>>(a, nr);
            if (n + 1 < f.order)
                hyena_staged_cols_x2<G, IO, EVEN, 1><<<cgrid, G::CT, G::CSMEM, st>>>(a, nr);
            else
                hyena_staged_cols_x2<G, IO, EVEN, 2><<<cgrid, G::CT, G::CSMEM, st>>>(a, nr);
        }
        note_launch(2 * f.order + 1);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template <typename G>
cudaError_t launch_staged_g(const Fwd1dArgs &f, float2 *ws, int64_t chunk, hyena_dtype_t dt, bool even,
                            const cudaStream_t *lanes, int nst) {
    if (dt == HYENA_F32)
        return even ? launch_staged_io<G, float, true>(f, ws, chunk, lanes, nst)
                    : launch_staged_io<G, float, false>(f, ws, chunk, lanes, nst);
    return even ? launch_staged_io<G, __nv_bfloat16, true>(f, ws, chunk, lanes, nst)
                : launch_staged_io<G, __nv_bfloat16, false>(f, ws, chunk, lanes, nst);
}

// Filter spectra: two chunks of 32 MB of transforms in flight, in plan-owned scratch.
int64_t staged_spec_chunk(int64_t MC) { return ((int64_t)32 << 20) / (MC * 8); }
size_t staged_spec_scratch_bytes(int64_t MC) { return (size_t)2 * staged_spec_chunk(MC) * MC * sizeof(float2); }

template <typename G>
cudaError_t launch_spec_staged_g(const Spec1dArgs &base, int64_t nrows, const cudaStream_t *lanes, int nst) {
    cudaError_t e = cudaFuncSetAttribute(hyena_staged_spec_rows_x2<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)G::RSMEM);
    if (e == cudaSuccess && G::CSMEM > 48 * 1024)
        e = cudaFuncSetAttribute(hyena_staged_spec_cols_x2<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)G::CSMEM);
    if (e != cudaSuccess) return e;
    const int64_t chunk = staged_spec_chunk(G::MC);
    for (int64_t o0 = 0, c = 0; o0 < nrows; o0 += chunk, ++c) {
        Spec1dArgs a = base;
        a.ws = base.ws + (c % nst) * chunk * G::MC;
        a.o0 = o0;
        a.nr = (nrows - o0) < chunk ? (nrows - o0) : chunk;
        const int64_t pairs = (a.nr + 1) / 2;
        const cudaStream_t s = lanes[c % nst];
        hyena_staged_spec_cols_x2<G><<<(unsigned)(pairs * G::CGROUPS), G::CT, G::CSMEM, s>>>(a);
        hyena_staged_spec_rows_x2<G><<<(unsigned)(pairs * G::RGROUPS), G::RT, G::RSMEM, s>>>(a);
        note_launch(2);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_spec_1d_staged(const float *h, int64_t h_stride, int64_t L, c32 *Hout, int64_t nrows, int64_t MC,
                                  const c32 *tw, float2 *scratch, cudaStream_t st, const StagedLanes &sl) {
    Spec1dArgs a;
    a.h = h;
    a.h_stride = h_stride;
    a.L = L;
    a.Hout = Hout;
    a.tw = tw;
    a.ws = scratch;
    a.o0 = 0;
    a.nr = 0;
    auto run = [&](const cudaStream_t *lanes, int nst) -> cudaError_t {
        switch (MC) {
            case 32768: return launch_spec_staged_g<GS_32K>(a, nrows, lanes, nst);
            case 65536: return launch_spec_staged_g<GS_64K>(a, nrows, lanes, nst);
            case 131072: return launch_spec_staged_g<GS_128K>(a, nrows, lanes, nst);
            case 262144: return launch_spec_staged_g<GS_256K>(a, nrows, lanes, nst);
            case 524288: return launch_spec_staged_g<GS_512K>(a, nrows, lanes, nst);
            default: return cudaErrorInvalidValue;
        }
    };
    // always on the plan's first two lanes, one chunk too: scratch slot i is used by lane i only
    return run_on_lanes(st, sl, 2, run);
}

cudaError_t launch_fwd_1d_staged_chunks(const Fwd1dArgs &f, int64_t MC, float2 *ws, int64_t chunk, hyena_dtype_t dt,
                                        bool even, const cudaStream_t *lanes, int nst) {
    switch (MC) {
        case 32768: return launch_staged_g<GS_32K>(f, ws, chunk, dt, even, lanes, nst);
        case 65536: return launch_staged_g<GS_64K>(f, ws, chunk, dt, even, lanes, nst);
        case 131072: return launch_staged_g<GS_128K>(f, ws, chunk, dt, even, lanes, nst);
        case 262144: return launch_staged_g<GS_256K>(f, ws, chunk, dt, even, lanes, nst);
        case 524288: return launch_staged_g<GS_512K>(f, ws, chunk, dt, even, lanes, nst);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_fwd_1d_staged(const Fwd1dArgs &f, int64_t MC, float2 *ws, hyena_dtype_t dt, bool even,
                                 cudaStream_t st, const StagedLanes &sl) {
    const int64_t chunk = staged_chunk_rows(MC);
    auto run = [&](const cudaStream_t *lanes, int nst) -> cudaError_t {
        return launch_fwd_1d_staged_chunks(f, MC, ws, chunk, dt, even, lanes, nst);
    };
    if (f.rows <= chunk) return run(&st, 1);   // one chunk: the caller's stream only
    const int64_t nchunks = (f.rows + chunk - 1) / chunk;
    return run_on_lanes(st, sl, (int)(nchunks < HYENA_STAGED_LANES ? nchunks : HYENA_STAGED_LANES), run);
}

}  // namespace hyena
