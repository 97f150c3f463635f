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
// exits. Rows run in chunks of as many rows as the array holds, one chunk
// after another on the caller's stream, through the same column and row
// kernels (and the same launch sequence per chunk) as hyena_forward on
// HYENA_PATH_STAGED, so each row's result is the same bit for bit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "hyena.h"
#include "launch.h"
#include "plan.h"

// The scratch array (complex64 elements). In host code `scratch` names a
// host-side stand-in, not device memory; its device address is looked up
// with the device current (scratch_address below).
static __device__ __align__(256) float2 scratch[HYENA_STATIC_SCRATCH_BYTES / sizeof(float2)];

namespace {

using namespace hyena;

constexpr size_t kScratchBytes = HYENA_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// The array's address is a property of the CUDA context the module was
// loaded into. It is cached per device together with the id of that context,
// and looked up again when the current context is another one (after a
// device reset, or when the primary context was released and created anew).
struct ScratchCache {
    unsigned long long ctx_id = 0;
    float2 *ptr = nullptr;
};
ScratchCache g_cache[kMaxDevices];
std::mutex g_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// The current context's id through the driver entry points the runtime hands
// out (the library links only the runtime). 0 when it cannot be had.
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(f);
        f = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(f);
        cudaGetLastError();
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of the array for device `dev` (current). The first call in a
// context looks it up with cudaGetSymbolAddress; later calls in the same
// context reuse it.
cudaError_t scratch_address(int dev, float2 **out) {
    std::lock_guard<std::mutex> lock(g_mu);
    ScratchCache &c = g_cache[dev];
    const unsigned long long id = current_context_id();
    if (!c.ptr || id == 0 || id != c.ctx_id) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, scratch);   // makes the context current if needed
        if (e != cudaSuccess) return e;
        c.ptr = static_cast<float2 *>(p);
        c.ctx_id = current_context_id();
    }
    *out = c.ptr;
    return cudaSuccess;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" hyena_status_t hyena_forward_no_alloc(hyena_plan_t plan, int64_t batch, const void *v,
                                                 const void *const *gates, const void *H, const float *Dskip,
                                                 void *y, void *stream) {
    if (!plan || batch < 0) return HYENA_ERR_INVALID_ARG;
    if (plan->path != HYENA_PATH_STAGED || !staged_path_supported(plan->MC)) return HYENA_ERR_UNSUPPORTED;
    // two rows' transforms (MC complex64 each) must fit the array: the kernels run rows in pairs
    const size_t row_bytes = (size_t)plan->MC * sizeof(float2);
    if (2 * row_bytes > kScratchBytes) return HYENA_ERR_WORKSPACE;
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
    a.hD = plan->D;
    a.B = batch;
    a.order = plan->order;
    a.es = plan->layout == HYENA_LAYOUT_BLD ? plan->D : 1;
    a.err = plan->dev_err;
    const int64_t chunk = (int64_t)(kScratchBytes / row_bytes) & ~(int64_t)1;   // whole row pairs
    cudaStream_t st = (cudaStream_t)stream;
    const cudaError_t e =
        launch_fwd_1d_staged_chunks(a, plan->MC, ws, chunk, plan->dtype, (plan->L % 2) == 0, &st, 1);
    return e == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;
}
