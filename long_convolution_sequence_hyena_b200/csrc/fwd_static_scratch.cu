// hyena_forward_no_alloc: the staged long-row forward with its scratch in a
// fixed device array of this library instead of a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run the
// operator: a plain C host program that links this library has no allocator
// of its own to hand a workspace from, and a process whose memory is owned by
// a framework's caching allocator, or a latency-bound loop in which a
// cudaMalloc (which may synchronise the device) is not acceptable, should not
// allocate per call either. For them this entry point needs only the plan,
// the inputs and the outputs.
//
// The scratch is one file-scope array of HYENA_STATIC_SCRATCH_BYTES per
// device; every device that loads the library holds it until the process
// exits. Rows run in chunks of as many rows as the array holds, through the
// same column and row kernels as hyena_forward on HYENA_PATH_STAGED.
#include <cuda_runtime.h>

#include <mutex>

#include "hyena.h"
#include "kernels_1d_staged.cuh"
#include "plan.h"

// The scratch array (complex64 elements). In host code `scratch` names a
// host-side stand-in, not device memory; its device address is looked up
// once per device, with that device current (scratch_address below).
static __device__ __align__(256) float2 scratch[HYENA_STATIC_SCRATCH_BYTES / sizeof(float2)];

namespace {

using namespace hyena;

constexpr size_t kScratchBytes = HYENA_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;
float2 *g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

cudaError_t scratch_address(int dev, float2 **out) {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = static_cast<float2 *>(p);
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

template <typename G, typename IO, bool EVEN>
cudaError_t run_chunks(const Fwd1dArgs &f, float2 *ws, int64_t chunk, cudaStream_t st) {
    for (int64_t o0 = 0; o0 < f.rows; o0 += chunk) {
        const int64_t nr = (f.rows - o0) < chunk ? (f.rows - o0) : chunk;
        StagedArgs a;
        a.f = f;
        a.ws = ws;
        a.o0 = o0;
        a.n = 0;
        hyena_staged_cols<G, IO, EVEN, 0><<<(unsigned)(nr * G::CGROUPS), G::CT, G::CSMEM, st>>>(a);
        for (int n = 0; n < f.order; ++n) {
            a.n = n;
            hyena_staged_rows<G><<<(unsigned)(nr * G::RGROUPS), G::RT, G::RSMEM, st>>>(a);
            if (n + 1 < f.order)
                hyena_staged_cols<G, IO, EVEN, 1><<<(unsigned)(nr * G::CGROUPS), G::CT, G::CSMEM, st>>>(a);
            else
                hyena_staged_cols<G, IO, EVEN, 2><<<(unsigned)(nr * G::CGROUPS), G::CT, G::CSMEM, st>>>(a);
        }
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template <typename G>
cudaError_t run_geom(const Fwd1dArgs &f, float2 *ws, int64_t chunk, hyena_dtype_t dt, bool even, cudaStream_t st) {
    if (dt == HYENA_F32)
        return even ? run_chunks<G, float, true>(f, ws, chunk, st) : run_chunks<G, float, false>(f, ws, chunk, st);
    return even ? run_chunks<G, __nv_bfloat16, true>(f, ws, chunk, st)
                : run_chunks<G, __nv_bfloat16, false>(f, ws, chunk, st);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" hyena_status_t hyena_forward_no_alloc(hyena_plan_t plan, int64_t batch, const void *v,
                                                 const void *const *gates, const void *H, const float *Dskip,
                                                 void *y, void *stream) {
    if (!plan || batch < 0) return HYENA_ERR_INVALID_ARG;
    if (plan->path != HYENA_PATH_STAGED || (plan->MC != 32768 && plan->MC != 65536)) return HYENA_ERR_UNSUPPORTED;
    // one row's transform (MC complex64) must fit the array: M <= kScratchBytes / 4
    const size_t row_bytes = (size_t)plan->MC * sizeof(float2);
    if (row_bytes > kScratchBytes) return HYENA_ERR_WORKSPACE;
    if (batch == 0) return HYENA_OK;
    if (!v || !gates || !H || !y) return HYENA_ERR_INVALID_ARG;
    for (int n = 0; n < plan->order; ++n)
        if (!gates[n] || !aligned16(gates[n])) return gates[n] ? HYENA_ERR_ALIGNMENT : HYENA_ERR_INVALID_ARG;
    if (!aligned16(v) || !aligned16(H) || !aligned16(y) || (Dskip && (reinterpret_cast<uintptr_t>(Dskip) & 3u)))
        return HYENA_ERR_ALIGNMENT;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return HYENA_ERR_CUDA;
    if (dev != plan->device) return HYENA_ERR_INVALID_ARG;
    if (dev < 0 || dev >= kMaxDevices) return HYENA_ERR_UNSUPPORTED;
    float2 *ws = nullptr;
    if (scratch_address(dev, &ws) != cudaSuccess) return HYENA_ERR_CUDA;

    Fwd1dArgs a = {};
    a.v = v;
    for (int n = 0; n < plan->order; ++n) a.gates[n] = gates[n];
    a.H = reinterpret_cast<const c32 *>(H);
    a.dskip = Dskip;
    a.y = y;
    a.tw = reinterpret_cast<const c32 *>(plan->tw);
    a.rows = batch * plan->D;
    a.L = plan->L;
    a.D = plan->D;
    a.B = batch;
    a.order = plan->order;
    const int64_t chunk = (int64_t)(kScratchBytes / row_bytes);
    const bool even = (plan->L % 2) == 0;
    cudaStream_t st = (cudaStream_t)stream;
    const cudaError_t e =
        plan->MC == 32768
            ? run_geom<StagedGeom<32768, 128, 32, 16>>(a, ws, chunk, plan->dtype, even, st)
            : run_geom<StagedGeom<65536, 256, 16, 16>>(a, ws, chunk, plan->dtype, even, st);
    return e == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;
}
