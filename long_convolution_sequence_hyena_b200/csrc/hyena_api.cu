// C ABI of the Hyena operator library: plans, argument validation and kernel
// dispatch. See include/hyena.h for the contract of every entry point.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <new>
#include <utility>
#include <vector>

#include "hyena.h"
#include "kernels_2d.cuh"
#include "kernels_3d.cuh"
#include "launch.h"
#include "plan.h"

using namespace hyena;

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int64_t next_pow2(int64_t v) {
    int64_t p = 1;
    while (p < v) p <<= 1;
    return p;
}

// W_M^m = exp(-2 pi i m / M), m in [0, M), computed in double and rounded once.
std::vector<float2> twiddle_table(int64_t M) {
    std::vector<float2> t((size_t)M);
    for (int64_t m = 0; m < M; ++m) {
        const double ang = -2.0 * M_PI * (double)m / (double)M;
        t[(size_t)m] = make_float2((float)std::cos(ang), (float)std::sin(ang));
    }
    return t;
}

// Destroy the staged path's streams (those that were created).
// Resources a plan holds (device buffers, streams, host objects) are created
// and released through these helpers, which count them (the test hook
// hyena_debug_plan_resources reads the count) and can be made to fail
// (hyena_debug_fail_allocation), so that tests reach every unwind path of
// plan creation.
std::atomic<int64_t> g_plan_resources{0};
std::atomic<int> g_fail_countdown{0};   // the nth creation from now fails; 0: none

bool injected_failure() {
    int n = g_fail_countdown.load();
    while (n > 0)
        if (g_fail_countdown.compare_exchange_weak(n, n - 1)) return n == 1;
    return false;
}
bool res_dev_alloc(void **p, size_t bytes) {
    if (injected_failure()) return false;
    if (cudaMalloc(p, bytes) != cudaSuccess) {
        cudaGetLastError();
        *p = nullptr;
        return false;
    }
    ++g_plan_resources;
    return true;
}
bool res_dev_free(void *p) {
    if (!p) return true;
    --g_plan_resources;
    return cudaFree(p) == cudaSuccess;
}
bool res_stream_create(cudaStream_t *s) {
    if (injected_failure()) return false;
    if (cudaStreamCreateWithFlags(s, cudaStreamNonBlocking) != cudaSuccess) {
        cudaGetLastError();
        *s = nullptr;
        return false;
    }
    ++g_plan_resources;
    return true;
}
template <typename T, typename... A>
T *res_new(A &&...args) {
    if (injected_failure()) return nullptr;
    T *o = new (std::nothrow) T(std::forward<A>(args)...);
    if (o) ++g_plan_resources;
    return o;
}
template <typename T>
void res_delete(T *o) {
    if (!o) return;
    --g_plan_resources;
    delete o;
}

bool release_lanes(hyena_plan_s *p) {
    if (!p->has_lanes) return true;
    bool ok = true;
    for (int i = 0; i < HYENA_STAGED_LANES; ++i) {
        if (p->lane[i]) {
            --g_plan_resources;
            if (cudaStreamDestroy(p->lane[i]) != cudaSuccess) ok = false;
        }
        p->lane[i] = nullptr;
    }
    p->has_lanes = false;
    return ok;
}

// Everything a plan (or a plan under construction) holds, except the plan
// object itself; false if a CUDA release failed.
bool release_plan_resources(hyena_plan_s *p) {
    bool ok = release_lanes(p);
    ok = res_dev_free(p->spec_ws) && ok;
    ok = res_dev_free(p->dev_err) && ok;
    ok = res_dev_free(p->tw) && ok;
    res_delete(p->spec_mu);
    p->spec_ws = nullptr;
    p->dev_err = nullptr;
    p->tw = nullptr;
    p->spec_mu = nullptr;
    return ok;
}

// The plan's lanes with fork and join events that belong to one call, so
// that calls on one plan from several threads never wait on each other's
// event records. cudaEventDestroy returns at once; an event that a stream
// still waits on is released when the wait is over.
struct CallLanes {
    StagedLanes l;
    bool ok = false;
    explicit CallLanes(const hyena_plan_s *p) {
        l.fork = nullptr;
        for (int i = 0; i < HYENA_STAGED_LANES; ++i) {
            l.lane[i] = p->lane[i];
            l.join[i] = nullptr;
        }
        ok = cudaEventCreateWithFlags(&l.fork, cudaEventDisableTiming) == cudaSuccess;
        for (int i = 0; i < HYENA_STAGED_LANES && ok; ++i)
            ok = cudaEventCreateWithFlags(&l.join[i], cudaEventDisableTiming) == cudaSuccess;
        if (!ok) cudaGetLastError();
    }
    ~CallLanes() {
        if (l.fork) cudaEventDestroy(l.fork);
        for (int i = 0; i < HYENA_STAGED_LANES; ++i)
            if (l.join[i]) cudaEventDestroy(l.join[i]);
    }
    CallLanes(const CallLanes &) = delete;
    CallLanes &operator=(const CallLanes &) = delete;
};

hyena_status_t check_device(const hyena_plan_s *p) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return HYENA_ERR_CUDA;
    return dev == p->device ? HYENA_OK : HYENA_ERR_INVALID_ARG;
}

hyena_status_t check_implicit(const hyena_plan_s *p, const hyena_implicit_params_t *ip) {
    if (!ip->W1 || !ip->b1 || !ip->W2 || !ip->b2 || !ip->W3 || !ip->b3 || !ip->window) return HYENA_ERR_INVALID_ARG;
    if (ip->width < 4 || ip->width > IMP_MAXW || (ip->width & 3)) return HYENA_ERR_UNSUPPORTED;
    if (p->ndim == 1 && (ip->num_freqs < 0 || 1 + 2 * ip->num_freqs > IMP_MAXF)) return HYENA_ERR_UNSUPPORTED;
    if (p->ndim == 3 && ip->width != 64) return HYENA_ERR_UNSUPPORTED;   // 3D coordinates: tensor-core network only
    if (!aligned16(ip->W3)) return HYENA_ERR_ALIGNMENT;
    if (!std::isfinite(ip->omega0) || !std::isfinite(ip->omega_hidden)) return HYENA_ERR_INVALID_ARG;
    return HYENA_OK;
}

ImplicitArgs implicit_args(const hyena_plan_s *p, const hyena_implicit_params_t *ip, float *out, int64_t out_stride,
                           int64_t out_row_stride) {
    ImplicitArgs a;
    a.p = *ip;
    a.ndim = p->ndim;
    a.L = p->L;
    a.H = p->Hh;
    a.W = p->Ww;
    a.Dz = p->Dd;
    a.npos = p->ndim == 1 ? p->L : (p->ndim == 2 ? 4 * p->Hh * p->Ww : 8 * p->Dd * p->Hh * p->Ww);
    a.nout = (int64_t)p->order * p->D;
    a.out = out;
    a.out_stride = out_stride;
    a.out_row_stride = out_row_stride;
    return a;
}

}  // namespace

namespace hyena {
static std::atomic<int64_t> g_launches{0};
void note_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
}  // namespace hyena

extern "C" {

const char *hyena_status_string(hyena_status_t s) {
    switch (s) {
        case HYENA_OK: return "ok";
        case HYENA_ERR_INVALID_ARG: return "invalid argument";
        case HYENA_ERR_UNSUPPORTED: return "unsupported configuration";
        case HYENA_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
        case HYENA_ERR_WORKSPACE: return "workspace missing or too small";
        case HYENA_ERR_CUDA: return "CUDA error";
        case HYENA_ERR_NOMEM: return "out of memory";
    }
    return "unknown status";
}

hyena_status_t hyena_plan_create(hyena_plan_t *out, int ndim, const int64_t *shape, int64_t channels, int order,
                                 hyena_dtype_t io_dtype, int causal) {
    return hyena_plan_create_ex(out, ndim, shape, channels, order, io_dtype, causal, 0);
}

hyena_status_t hyena_plan_create_ex(hyena_plan_t *out, int ndim, const int64_t *shape, int64_t channels, int order,
                                    hyena_dtype_t io_dtype, int causal, int flags) {
    if (flags & ~HYENA_PLAN_RADIX3) return HYENA_ERR_INVALID_ARG;
    if (!out) return HYENA_ERR_INVALID_ARG;
    *out = nullptr;
    if (!shape || channels < 1 || order < 1 || order > HYENA_MAX_ORDER) return HYENA_ERR_INVALID_ARG;
    if (io_dtype != HYENA_F32 && io_dtype != HYENA_BF16) return HYENA_ERR_INVALID_ARG;
    if (ndim < 1 || ndim > 3) return HYENA_ERR_INVALID_ARG;
    for (int i = 0; i < ndim; ++i)
        if (shape[i] < 1) return HYENA_ERR_INVALID_ARG;
    if ((ndim == 1 && causal != 1) || (ndim >= 2 && causal != 0)) return HYENA_ERR_UNSUPPORTED;

    hyena_plan_s p;
    p.ndim = ndim;
    p.D = channels;
    p.order = order;
    p.dtype = io_dtype;
    if (ndim == 1) {
        p.L = shape[0];
        if (p.L > HYENA_MAX_L_1D) return HYENA_ERR_UNSUPPORTED;
        p.M = next_pow2(2 * p.L);
        if (p.M < 32) p.M = 32;  // smallest FFT the kernels run (extra zero padding is exact)
        if (flags & HYENA_PLAN_RADIX3) {
            // the smallest M = 6 P >= 2L, when it is below the power of two
            int64_t P = 16;
            while (6 * P < 2 * p.L) P <<= 1;
            if (6 * P < p.M && mr3_supported(P)) {
                p.M = 6 * P;
                p.P3 = P;
            }
        }
        p.MC = p.M / 2;
        p.path = p.M <= HYENA_MAX_M_CTA ? HYENA_PATH_CTA
                 : (staged_path_supported(p.MC) ? HYENA_PATH_STAGED : HYENA_PATH_CLUSTER);
        if (p.P3) p.path = HYENA_PATH_CTA;
        // test and measurement override: HYENA_FORCE_PATH=cta|staged|cluster picks a
        // kernel family that can run this length, or the plan is UNSUPPORTED
        if (const char *fp = p.P3 ? nullptr : std::getenv("HYENA_FORCE_PATH")) {
            if (!std::strcmp(fp, "cta")) {
                if (p.M > HYENA_MAX_M_CTA) return HYENA_ERR_UNSUPPORTED;
                p.path = HYENA_PATH_CTA;
            } else if (!std::strcmp(fp, "staged")) {
                if (!staged_path_supported(p.MC)) return HYENA_ERR_UNSUPPORTED;
                p.path = HYENA_PATH_STAGED;
            } else if (!std::strcmp(fp, "cluster")) {
                if (!cluster_path_supported(p.MC)) return HYENA_ERR_UNSUPPORTED;
                p.path = HYENA_PATH_CLUSTER;
            } else if (*fp) {
                return HYENA_ERR_INVALID_ARG;
            }
        }
        if (p.path == HYENA_PATH_CLUSTER && !cluster_path_supported(p.MC)) return HYENA_ERR_UNSUPPORTED;
        p.spectrum_elems = p.MC + 1;
        p.tw_len = p.M;
    } else if (ndim == 3) {
        p.Dd = shape[0];
        p.Hh = shape[1];
        p.Ww = shape[2];
        if (!grid3d_supported(p.Dd, p.Hh, p.Ww)) return HYENA_ERR_UNSUPPORTED;
        p.path = HYENA_PATH_3D;
        p.spectrum_elems = 8 * p.Dd * p.Hh * p.Ww;
        p.tw_len = 2 * p.Ww;
    } else {
        p.Hh = shape[0];
        p.Ww = shape[1];
        const bool ok = p.Hh == p.Ww && (p.Ww == 32 || p.Ww == 64 || p.Ww == 128 || p.Ww == 256);
        if (!ok) return HYENA_ERR_UNSUPPORTED;
        p.path = HYENA_PATH_2D;
        p.spectrum_elems = 2 * p.Hh * (p.Ww + 1);
        p.tw_len = 2 * p.Ww;
    }
    if (cudaGetDevice(&p.device) != cudaSuccess) return HYENA_ERR_CUDA;

    // main table W_tw_len, followed by W_1024 for the short sub-transforms of the cluster paths
    std::vector<float2> tw = twiddle_table(p.tw_len);
    {
        std::vector<float2> sub = twiddle_table(HYENA_SUB_TWIDDLES);
        tw.insert(tw.end(), sub.begin(), sub.end());
    }
    // every failure below releases what was created before it (release_plan_resources)
    auto fail = [&](hyena_status_t st) {
        release_plan_resources(&p);
        return st;
    };
    if (!res_dev_alloc(reinterpret_cast<void **>(&p.tw), sizeof(float2) * tw.size())) return fail(HYENA_ERR_NOMEM);
    if (cudaMemcpy(p.tw, tw.data(), sizeof(float2) * tw.size(), cudaMemcpyHostToDevice) != cudaSuccess)
        return fail(HYENA_ERR_CUDA);
    if (!res_dev_alloc(reinterpret_cast<void **>(&p.dev_err), 4 * sizeof(int))) return fail(HYENA_ERR_NOMEM);
    if (cudaMemset(p.dev_err, 0, 4 * sizeof(int)) != cudaSuccess) return fail(HYENA_ERR_CUDA);
    if (p.path == HYENA_PATH_STAGED || (p.path == HYENA_PATH_2D && staged2d_supported(p.Ww))) {
        p.has_lanes = true;
        for (int i = 0; i < HYENA_STAGED_LANES; ++i)
            if (!res_stream_create(&p.lane[i])) return fail(HYENA_ERR_CUDA);
        const size_t sb = p.path == HYENA_PATH_STAGED ? staged_spec_scratch_bytes(p.MC)
                                                      : staged2d_spec_scratch_bytes(p.Ww);
        if (!res_dev_alloc(reinterpret_cast<void **>(&p.spec_ws), sb)) return fail(HYENA_ERR_NOMEM);
        p.spec_mu = res_new<std::mutex>();
        if (!p.spec_mu) return fail(HYENA_ERR_NOMEM);
    }
    hyena_plan_s *heap = res_new<hyena_plan_s>(p);
    if (!heap) return fail(HYENA_ERR_NOMEM);
    *out = heap;
    return HYENA_OK;
}

hyena_status_t hyena_plan_destroy(hyena_plan_t plan) {
    if (!plan) return HYENA_OK;
    const bool ok = release_plan_resources(plan);
    res_delete(plan);
    return ok ? HYENA_OK : HYENA_ERR_CUDA;
}

hyena_status_t hyena_debug_fail_allocation(int nth) {
    if (nth < 0) return HYENA_ERR_INVALID_ARG;
    g_fail_countdown.store(nth);
    return HYENA_OK;
}

hyena_status_t hyena_debug_plan_resources(int64_t *count) {
    if (!count) return HYENA_ERR_INVALID_ARG;
    *count = g_plan_resources.load();
    return HYENA_OK;
}

hyena_status_t hyena_plan_set_layout(hyena_plan_t plan, int layout) {
    if (!plan || (layout != HYENA_LAYOUT_BDL && layout != HYENA_LAYOUT_BLD)) return HYENA_ERR_INVALID_ARG;
    if (plan->ndim != 1 && layout != HYENA_LAYOUT_BDL) return HYENA_ERR_UNSUPPORTED;
    plan->layout = layout;
    return HYENA_OK;
}

hyena_status_t hyena_plan_device_errors(hyena_plan_t plan, int *flags, int clear) {
    if (!plan) return HYENA_ERR_INVALID_ARG;
    int h[4] = {0, 0, 0, 0};
    if (cudaMemcpy(h, plan->dev_err, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return HYENA_ERR_CUDA;
    if (clear && cudaMemset(plan->dev_err, 0, sizeof(h)) != cudaSuccess) return HYENA_ERR_CUDA;
    if (flags) flags[0] = h[0];
    return h[0] ? HYENA_ERR_CUDA : HYENA_OK;
}

hyena_status_t hyena_launch_count(int64_t *count) {
    if (!count) return HYENA_ERR_INVALID_ARG;
    *count = hyena::g_launches.load(std::memory_order_relaxed);
    return HYENA_OK;
}

hyena_status_t hyena_plan_info(hyena_plan_t plan, int64_t *fft_len, int64_t *spectrum_elems, int *path) {
    if (!plan) return HYENA_ERR_INVALID_ARG;
    if (fft_len)
        *fft_len = plan->ndim == 1 ? plan->M
                                   : (plan->ndim == 2 ? 4 * plan->Hh * plan->Ww : 8 * plan->Dd * plan->Hh * plan->Ww);
    if (spectrum_elems) *spectrum_elems = plan->spectrum_elems;
    if (path) *path = plan->path;
    return HYENA_OK;
}

size_t hyena_workspace_bytes(hyena_plan_t plan, int64_t batch) {
    if (!plan || batch < 0) return 0;
    if (plan->path == HYENA_PATH_3D) {
        const int64_t c = grid3d_chunk_volumes(plan->Dd, plan->Hh, plan->Ww), vols = batch * plan->D;
        return (size_t)(vols < c ? vols : c) * (size_t)(plan->Dd * 4 * plan->Hh * plan->Ww) * sizeof(float2);
    }
    if (plan->path == HYENA_PATH_2D && staged2d_supported(plan->Ww))
        return (size_t)staged2d_workspace_planes(plan->Ww, batch * plan->D) * (size_t)(2 * plan->Hh) *
               (size_t)(plan->Ww / 2) * sizeof(float2);
    if (plan->path != HYENA_PATH_STAGED) return 0;
    return (size_t)staged_workspace_rows(plan->MC, batch * plan->D) * (size_t)plan->MC * sizeof(float2);
}

hyena_status_t hyena_implicit_filter(hyena_plan_t plan, const hyena_implicit_params_t *params, float *h_out,
                                     void *stream) {
    if (!plan || !params || !h_out) return HYENA_ERR_INVALID_ARG;
    hyena_status_t s = check_implicit(plan, params);
    if (s != HYENA_OK) return s;
    if (!aligned16(h_out)) return HYENA_ERR_ALIGNMENT;
    if ((s = check_device(plan)) != HYENA_OK) return s;
    const int64_t stride = plan->ndim == 1 ? plan->L
                           : (plan->ndim == 2 ? 4 * plan->Hh * plan->Ww : 8 * plan->Dd * plan->Hh * plan->Ww);
    ImplicitArgs a = implicit_args(plan, params, h_out, stride, 2 * plan->Ww);
    return launch_implicit(a, plan->dev_err, (cudaStream_t)stream) == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;
}

size_t hyena_filter_spectrum_workspace_bytes(hyena_plan_t plan) {
    if (!plan) return 0;
    if (plan->ndim == 1 && plan->path == HYENA_PATH_STAGED) return staged_spec_scratch_bytes(plan->MC);
    if (plan->ndim == 2 && staged2d_supported(plan->Ww)) return staged2d_spec_scratch_bytes(plan->Ww);
    return 0;
}

hyena_status_t hyena_filter_spectrum(hyena_plan_t plan, const float *h, const hyena_implicit_params_t *params,
                                     void *H_out, void *stream) {
    return hyena_filter_spectrum_ws(plan, h, params, H_out, nullptr, 0, stream);
}

hyena_status_t hyena_filter_spectrum_ws(hyena_plan_t plan, const float *h, const hyena_implicit_params_t *params,
                                        void *H_out, void *workspace, size_t ws_bytes, void *stream) {
    if (!plan || !H_out || (!h && !params)) return HYENA_ERR_INVALID_ARG;
    // the transforms' scratch: the caller's workspace, or (none given) the plan's,
    // whose lock then keeps each call's launch sequence together
    const size_t ws_need = hyena_filter_spectrum_workspace_bytes(plan);
    if (workspace && ws_bytes < ws_need) return HYENA_ERR_WORKSPACE;
    if (workspace && !aligned16(workspace)) return HYENA_ERR_ALIGNMENT;
    float2 *scratch = workspace ? reinterpret_cast<float2 *>(workspace) : plan->spec_ws;
    if (!aligned16(H_out) || (h && !aligned16(h))) return HYENA_ERR_ALIGNMENT;
    hyena_status_t s;
    if (!h && (s = check_implicit(plan, params)) != HYENA_OK) return s;
    if ((s = check_device(plan)) != HYENA_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    const int64_t nrows = (int64_t)plan->order * plan->D;
    c32 *Hc = reinterpret_cast<c32 *>(H_out);
    const c32 *tw = reinterpret_cast<const c32 *>(plan->tw);
    const float *src = h;
    cudaError_t e;
    if (plan->ndim == 3) {
        if (!h) return HYENA_ERR_UNSUPPORTED;   // 3D spectra from taps only (hyena_implicit_filter writes them)
        if (!aligned16(h)) return HYENA_ERR_ALIGNMENT;
        const int64_t V = plan->Dd * plan->Hh * plan->Ww;
        e = launch_spec_3d(h, 8 * V, Hc, nrows, (int)plan->Dd, (int)plan->Hh, (int)plan->Ww, tw + plan->tw_len, st);
        return e == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;
    }
    if (plan->ndim == 1) {
        int64_t src_stride = plan->L;
        if (!h) {
            // generate the taps inside each row's own output slot, then transform in place
            src_stride = 2 * (plan->MC + 1);
            ImplicitArgs a = implicit_args(plan, params, reinterpret_cast<float *>(H_out), src_stride, 0);
            if (launch_implicit(a, plan->dev_err, st) != cudaSuccess) return HYENA_ERR_CUDA;
            src = reinterpret_cast<const float *>(H_out);
        }
        if (plan->path == HYENA_PATH_STAGED) {
            CallLanes cl(plan);
            if (!cl.ok) return HYENA_ERR_CUDA;
            std::unique_lock<std::mutex> hold(*plan->spec_mu, std::defer_lock);
            if (!workspace) hold.lock();
            e = launch_spec_1d_staged(src, src_stride, plan->L, Hc, nrows, plan->MC, tw, scratch, st, cl.l);
        } else {
            e = plan->P3 ? launch_spec_1d_mr3(src, src_stride, plan->L, Hc, nrows, plan->P3, tw, st)
                : plan->path == HYENA_PATH_CTA
                    ? launch_spec_1d(src, src_stride, plan->L, Hc, nrows, plan->MC, tw, st)
                    : launch_spec_1d_cluster(src, src_stride, plan->L, Hc, nrows, plan->MC, tw, st);
        }
    } else {
        int64_t rs = 2 * plan->Ww, cs = 4 * plan->Hh * plan->Ww;
        if (!h) {
            // kernel rows written at the spectrum's row pitch inside each channel's slot
            rs = 2 * (plan->Ww + 1);
            cs = 2 * plan->Hh * rs;
            ImplicitArgs a = implicit_args(plan, params, reinterpret_cast<float *>(H_out), cs, rs);
            if (launch_implicit(a, plan->dev_err, st) != cudaSuccess) return HYENA_ERR_CUDA;
            src = reinterpret_cast<const float *>(H_out);
        }
        if (plan->spec_ws) {
            CallLanes cl(plan);
            if (!cl.ok) return HYENA_ERR_CUDA;
            std::unique_lock<std::mutex> hold(*plan->spec_mu, std::defer_lock);
            if (!workspace) hold.lock();
            e = launch_spec_2d_staged(src, rs, cs, Hc, nrows, plan->Ww, tw, scratch, st, cl.l);
        } else {
            e = launch_spec_2d(src, rs, cs, Hc, nrows, plan->Ww, tw, st);
        }
    }
    return e == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;
}

}  // extern "C"

namespace {

// The forward of both entry points: k == nullptr is the plain operator, else
// the gate sandwich (z^0 = v SiLU(k), SiLU of every gate). A 1D call may cover
// the channel range [d0, d0 + dc) of one batch element: v, the gates and y then
// hold those dc rows, while H and Dskip keep the whole plan's layout.
hyena_status_t forward_impl(hyena_plan_t plan, int64_t batch, const void *v, const void *k, const void *const *gates,
                            const void *H, const float *Dskip, void *y, void *workspace, size_t ws_bytes,
                            void *stream, int64_t d0 = 0, int64_t dc = -1) {
    if (dc < 0) dc = plan->D;
    if (!v || !gates || !H || !y) return HYENA_ERR_INVALID_ARG;
    if (k && !aligned16(k)) return HYENA_ERR_ALIGNMENT;
    for (int n = 0; n < plan->order; ++n)
        if (!gates[n]) return HYENA_ERR_INVALID_ARG;
    if (!aligned16(v) || !aligned16(H) || !aligned16(y) || (Dskip && !aligned4(Dskip))) return HYENA_ERR_ALIGNMENT;
    for (int n = 0; n < plan->order; ++n)
        if (!aligned16(gates[n])) return HYENA_ERR_ALIGNMENT;
    const size_t ws_need = dc == plan->D ? hyena_workspace_bytes(plan, batch) : hyena::workspace_bytes_1d(plan, batch * dc);
    if (ws_need && (!workspace || ws_bytes < ws_need)) return HYENA_ERR_WORKSPACE;
    if (ws_need && !aligned16(workspace)) return HYENA_ERR_ALIGNMENT;
    hyena_status_t s = check_device(plan);
    if (s != HYENA_OK) return s;

    if (plan->ndim == 3) {
        Fwd3dArgs a;
        std::memset(&a, 0, sizeof(a));
        a.v = v;
        a.k = k;
        for (int n = 0; n < plan->order; ++n) a.gates[n] = gates[n];
        a.K = reinterpret_cast<const c32 *>(H);
        a.dskip = Dskip;
        a.y = y;
        a.tws = reinterpret_cast<const c32 *>(plan->tw) + plan->tw_len;   // W_1024
        a.ws = reinterpret_cast<float2 *>(workspace);
        a.C = plan->D;
        a.B = batch;
        a.Dz = (int)plan->Dd;
        a.H = (int)plan->Hh;
        a.W = (int)plan->Ww;
        a.order = plan->order;
        return launch_fwd_3d(a, batch * plan->D, plan->dtype, (cudaStream_t)stream) == cudaSuccess ? HYENA_OK
                                                                                                  : HYENA_ERR_CUDA;
    }
    if (plan->ndim == 2) {
        Fwd2dArgs a;
        std::memset(&a, 0, sizeof(a));
        a.v = v;
        a.k = k;
        for (int n = 0; n < plan->order; ++n) a.gates[n] = gates[n];
        a.K = reinterpret_cast<const c32 *>(H);
        a.dskip = Dskip;
        a.y = y;
        a.tw = reinterpret_cast<const c32 *>(plan->tw);
        a.planes = batch * plan->D;
        a.C = plan->D;
        a.B = batch;
        a.order = plan->order;
        a.err = plan->dev_err;
        cudaError_t e2;
        if (staged2d_supported(plan->Ww)) {
            CallLanes cl(plan);
            if (!cl.ok) return HYENA_ERR_CUDA;
            e2 = launch_fwd_2d_staged(a, plan->Ww, reinterpret_cast<float2 *>(workspace), plan->dtype,
                                      (cudaStream_t)stream, cl.l);
        } else {
            e2 = launch_fwd_2d(a, plan->Ww, plan->dtype, (cudaStream_t)stream);
        }
        return e2 == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;
    }
    Fwd1dArgs a;
    std::memset(&a, 0, sizeof(a));
    a.v = v;
    for (int n = 0; n < plan->order; ++n) a.gates[n] = gates[n];
    a.H = reinterpret_cast<const c32 *>(H) + d0 * plan->spectrum_elems;
    a.dskip = Dskip ? Dskip + d0 : nullptr;
    a.y = y;
    a.tw = reinterpret_cast<const c32 *>(plan->tw);
    a.rows = batch * dc;
    a.L = plan->L;
    a.D = dc;
    a.hD = plan->D;
    a.B = batch;
    a.order = plan->order;
    a.es = plan->layout == HYENA_LAYOUT_BLD ? plan->D : 1;
    a.err = plan->dev_err;
    const bool even = (plan->L % 2) == 0;
    cudaError_t e;
    if (plan->path == HYENA_PATH_STAGED) {
        CallLanes cl(plan);
        if (!cl.ok) return HYENA_ERR_CUDA;
        e = launch_fwd_1d_staged(a, plan->MC, reinterpret_cast<float2 *>(workspace), plan->dtype, even,
                                 (cudaStream_t)stream, cl.l);
    } else if (plan->P3) {
        e = launch_fwd_1d_mr3(a, plan->P3, plan->dtype, even, (cudaStream_t)stream);
    } else if (plan->path == HYENA_PATH_CLUSTER)
        e = launch_fwd_1d_cluster(a, plan->MC, plan->dtype, even, (cudaStream_t)stream);
    else if (a.es == 1 && pair_path_supported(plan->MC, batch))
        e = launch_fwd_1d_pair(a, plan->MC, plan->dtype, even, (cudaStream_t)stream);
    else
        e = launch_fwd_1d(a, plan->MC, plan->dtype, even, (cudaStream_t)stream);
    return e == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;
}

}  // namespace

namespace hyena {

size_t workspace_bytes_1d(hyena_plan_t plan, int64_t rows) {
    if (plan->ndim != 1 || plan->path != HYENA_PATH_STAGED) return 0;
    return (size_t)staged_workspace_rows(plan->MC, rows) * (size_t)plan->MC * sizeof(float2);
}

hyena_status_t forward_channels_1d(hyena_plan_t plan, int64_t d0, int64_t dc, const void *v, const void *const *gates,
                                   const void *H, const float *Dskip, void *y, void *workspace, size_t ws_bytes,
                                   void *stream) {
    if (plan->ndim != 1 || plan->layout != HYENA_LAYOUT_BDL || d0 < 0 || dc <= 0 || d0 + dc > plan->D)
        return HYENA_ERR_INVALID_ARG;
    return forward_impl(plan, 1, v, nullptr, gates, H, Dskip, y, workspace, ws_bytes, stream, d0, dc);
}

}  // namespace hyena

extern "C" {

hyena_status_t hyena_forward(hyena_plan_t plan, int64_t batch, const void *v, const void *const *gates, const void *H,
                             const float *Dskip, void *y, void *workspace, size_t ws_bytes, void *stream) {
    if (!plan || batch < 0) return HYENA_ERR_INVALID_ARG;
    if (batch == 0) return HYENA_OK;  // nothing to read or write; pointers may be NULL
    return forward_impl(plan, batch, v, nullptr, gates, H, Dskip, y, workspace, ws_bytes, stream);
}

hyena_status_t hyena_forward_gated(hyena_plan_t plan, int64_t batch, const void *q, const void *k,
                                   const void *const *gates, const void *H, const float *Dskip, void *y,
                                   void *workspace, size_t ws_bytes, void *stream) {
    if (!plan || batch < 0) return HYENA_ERR_INVALID_ARG;
    if (plan->ndim == 1) return HYENA_ERR_UNSUPPORTED;
    if (batch == 0) return HYENA_OK;
    if (!k) return HYENA_ERR_INVALID_ARG;
    return forward_impl(plan, batch, q, k, gates, H, Dskip, y, workspace, ws_bytes, stream);
}

}  // extern "C"
