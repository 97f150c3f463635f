// Forward on host-resident activations: the batch is cut into stages of whole
// batch elements, or, for long 1D rows in the [B, D, L] layout, of channel
// ranges of one batch element (the operator is depthwise, so a channel range
// is an independent forward; one batch element of such rows holds hundreds of
// MB, and a stage per element would leave nothing to overlap at batch 1). A
// stage's inputs are copied to one of two device stage buffers on a copy-in
// stream, the stage runs the forward on the caller's stream, and its output
// is copied back on a copy-out stream. Two buffers let the copy-in of stage
// c+1, the forward of stage c and the copy-out of stage c-1 overlap
// (host-to-device and device-to-host copies use separate copy engines). The
// streams and events belong to the call, so that calls on one plan from
// several threads stay independent.
#include <cuda_runtime.h>

#include <cstdint>

#include "hyena.h"
#include "plan.h"

namespace {

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

struct HostStages {
    int64_t per_b = 0;   // elements of one batch element: D * L (1D) or C * H * W (2D)
    size_t io = 0;       // bytes per element
    int64_t bc = 0;      // batch elements per stage
    int64_t dc = 0;      // channels per stage: D (whole batch elements), or fewer
                         // when every batch element is split into channel ranges (bc = 1)
    size_t tensor = 0;   // bytes of one stage tensor, rounded up to 256
    size_t fwd_ws = 0;   // the forward's workspace for one stage
};

HostStages host_stages(hyena_plan_s *p, int64_t batch) {
    HostStages s;
    s.per_b = p->D * (p->ndim == 1 ? p->L : p->Hh * p->Ww);
    s.io = p->dtype == HYENA_F32 ? 4 : 2;
    s.dc = p->D;
    const size_t in_per_b = (size_t)(p->order + 1) * (size_t)s.per_b * s.io;
    // long rows: stages of about 16 MB of inputs, in whole chunks of the staged path
    const size_t split_target = (size_t)16 << 20;
    if (p->ndim == 1 && p->layout == HYENA_LAYOUT_BDL &&
        (p->path == HYENA_PATH_STAGED || p->path == HYENA_PATH_CLUSTER) && in_per_b > split_target) {
        const size_t in_per_ch = (size_t)(p->order + 1) * (size_t)p->L * s.io;
        const int64_t q = p->path == HYENA_PATH_STAGED ? hyena::staged_chunk_rows(p->MC) : 1;
        int64_t dc = (int64_t)(split_target / in_per_ch) / q * q;
        if (dc < q) dc = q;
        if (dc > p->D) dc = p->D;
        s.bc = 1;
        s.dc = dc;
        s.tensor = align256((size_t)dc * (size_t)p->L * s.io);
        s.fwd_ws = align256(hyena::workspace_bytes_1d(p, dc));
        return s;
    }
    const size_t target = (size_t)8 << 20;
    int64_t bc = (int64_t)((target + in_per_b - 1) / in_per_b);
    if (bc < 1) bc = 1;
    if (p->ndim == 1 && (bc & 1)) ++bc;   // even: two rows of a channel share a thread group
    if (bc > batch) bc = batch;
    s.bc = bc;
    s.tensor = align256((size_t)bc * (size_t)s.per_b * s.io);
    s.fwd_ws = align256(hyena_workspace_bytes(p, bc));
    return s;
}

// Page-locked (allocated or registered) host memory at both ends of the range.
bool pinned_range(const void *p, size_t bytes) {
    const char *c = static_cast<const char *>(p);
    const void *ends[2] = {c, c + bytes - 1};
    for (const void *e : ends) {
        cudaPointerAttributes at;
        if (cudaPointerGetAttributes(&at, e) != cudaSuccess) {
            cudaGetLastError();
            return false;
        }
        if (at.type != cudaMemoryTypeHost) return false;
    }
    return true;
}

bool overlaps(const void *a, const void *b, size_t bytes) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + bytes && y < x + bytes;
}

}  // namespace

extern "C" {

size_t hyena_forward_host_workspace_bytes(hyena_plan_t plan, int64_t batch) {
    if (!plan || batch <= 0) return 0;
    const HostStages s = host_stages(plan, batch);
    return 2 * (size_t)(plan->order + 2) * s.tensor + s.fwd_ws;
}

hyena_status_t hyena_forward_host(hyena_plan_t plan, int64_t batch, const void *v_host, const void *const *gates_host,
                                  const void *H, const float *Dskip, void *y_host, void *workspace, size_t ws_bytes,
                                  void *stream) {
    if (!plan || batch < 0) return HYENA_ERR_INVALID_ARG;
    if (batch == 0) return HYENA_OK;
    if (!v_host || !gates_host || !H || !y_host) return HYENA_ERR_INVALID_ARG;
    const int N = plan->order;
    for (int n = 0; n < N; ++n)
        if (!gates_host[n]) return HYENA_ERR_INVALID_ARG;
    if (!aligned16(H) || (Dskip && !aligned4(Dskip))) return HYENA_ERR_ALIGNMENT;
    const HostStages s = host_stages(plan, batch);
    const size_t need = hyena_forward_host_workspace_bytes(plan, batch);
    if (!workspace || ws_bytes < need) return HYENA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return HYENA_ERR_ALIGNMENT;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return HYENA_ERR_CUDA;
    if (dev != plan->device) return HYENA_ERR_INVALID_ARG;
    const size_t total = (size_t)batch * (size_t)s.per_b * s.io;
    if (!pinned_range(v_host, total) || !pinned_range(y_host, total)) return HYENA_ERR_INVALID_ARG;
    if (overlaps(y_host, v_host, total)) return HYENA_ERR_INVALID_ARG;
    for (int n = 0; n < N; ++n) {
        if (!pinned_range(gates_host[n], total)) return HYENA_ERR_INVALID_ARG;
        if (overlaps(y_host, gates_host[n], total)) return HYENA_ERR_INVALID_ARG;
    }

    cudaStream_t st = (cudaStream_t)stream, cin = nullptr, cout = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr, ev_in[2] = {nullptr, nullptr}, ev_comp[2] = {nullptr, nullptr},
                ev_out[2] = {nullptr, nullptr};
    auto release = [&]() {
        if (cin) cudaStreamDestroy(cin);
        if (cout) cudaStreamDestroy(cout);
        cudaEvent_t *evs[] = {&fork, &join, &ev_in[0], &ev_in[1], &ev_comp[0], &ev_comp[1], &ev_out[0], &ev_out[1]};
        for (cudaEvent_t *e : evs)
            if (*e) cudaEventDestroy(*e);
    };
    bool ok = cudaStreamCreateWithFlags(&cin, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&cout, cudaStreamNonBlocking) == cudaSuccess;
    cudaEvent_t *evs[] = {&fork, &join, &ev_in[0], &ev_in[1], &ev_comp[0], &ev_comp[1], &ev_out[0], &ev_out[1]};
    for (cudaEvent_t *e : evs) ok = ok && cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
        release();
        cudaGetLastError();
        return HYENA_ERR_CUDA;
    }

    // both copy streams start after the work already on the caller's stream
    cudaError_t e = cudaEventRecord(fork, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(cin, fork, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(cout, fork, 0);
    hyena_status_t status = e == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;

    char *base = static_cast<char *>(workspace);
    void *fwd_ws = s.fwd_ws ? base + 2 * (size_t)(N + 2) * s.tensor : nullptr;
    const char *vh = static_cast<const char *>(v_host);
    char *yh = static_cast<char *>(y_host);
    const bool split = s.dc < plan->D;
    const int64_t nsplit = split ? (plan->D + s.dc - 1) / s.dc : 1;   // channel ranges per batch element
    const int64_t nstage = split ? batch * nsplit : (batch + s.bc - 1) / s.bc;
    for (int64_t c = 0; c < nstage && status == HYENA_OK; ++c) {
        const int k = (int)(c & 1);
        int64_t b0, nb, d0 = 0, dcount = plan->D;
        if (split) {
            b0 = c / nsplit;
            nb = 1;
            d0 = (c % nsplit) * s.dc;
            dcount = (plan->D - d0) < s.dc ? (plan->D - d0) : s.dc;
        } else {
            b0 = c * s.bc;
            nb = (batch - b0) < s.bc ? (batch - b0) : s.bc;
        }
        const size_t row_elems = (size_t)(s.per_b / plan->D);   // L (1D) or H W (2D)
        const size_t bytes = (size_t)nb * (size_t)dcount * row_elems * s.io;
        const size_t off = ((size_t)b0 * (size_t)plan->D + (size_t)d0) * row_elems * s.io;
        // stage buffer k: v, x^1..x^N, y
        char *buf = base + (size_t)k * (size_t)(N + 2) * s.tensor;
        const void *gdev[HYENA_MAX_ORDER];
        for (int n = 0; n < N; ++n) gdev[n] = buf + (size_t)(1 + n) * s.tensor;
        char *ydev = buf + (size_t)(N + 1) * s.tensor;

        // copy-in: the buffer's inputs are free once the forward of stage c-2 is done
        if (c >= 2) e = cudaStreamWaitEvent(cin, ev_comp[k], 0);
        if (e == cudaSuccess) e = cudaMemcpyAsync(buf, vh + off, bytes, cudaMemcpyHostToDevice, cin);
        for (int n = 0; n < N && e == cudaSuccess; ++n)
            e = cudaMemcpyAsync(const_cast<void *>(gdev[n]), static_cast<const char *>(gates_host[n]) + off, bytes,
                                cudaMemcpyHostToDevice, cin);
        if (e == cudaSuccess) e = cudaEventRecord(ev_in[k], cin);
        // forward: after the copy-in, and once the copy-out of stage c-2 has read the output buffer
        if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ev_in[k], 0);
        if (e == cudaSuccess && c >= 2) e = cudaStreamWaitEvent(st, ev_out[k], 0);
        if (e != cudaSuccess) {
            status = HYENA_ERR_CUDA;
            break;
        }
        status = split ? hyena::forward_channels_1d(plan, d0, dcount, buf, gdev, H, Dskip, ydev, fwd_ws, s.fwd_ws, st)
                       : hyena_forward(plan, nb, buf, gdev, H, Dskip, ydev, fwd_ws, s.fwd_ws, st);
        if (status != HYENA_OK) break;
        e = cudaEventRecord(ev_comp[k], st);
        // copy-out
        if (e == cudaSuccess) e = cudaStreamWaitEvent(cout, ev_comp[k], 0);
        if (e == cudaSuccess) e = cudaMemcpyAsync(yh + off, ydev, bytes, cudaMemcpyDeviceToHost, cout);
        if (e == cudaSuccess) e = cudaEventRecord(ev_out[k], cout);
        if (e != cudaSuccess) status = HYENA_ERR_CUDA;
    }
    // join both copy streams back to the caller's stream, also after a failure,
    // so that nothing enqueued on it later runs ahead of them
    for (cudaStream_t cs : {cin, cout}) {
        e = cudaEventRecord(join, cs);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(st, join, 0);
        if (e != cudaSuccess) status = HYENA_ERR_CUDA;
    }
    release();
    return status;
}

}  // extern "C"
