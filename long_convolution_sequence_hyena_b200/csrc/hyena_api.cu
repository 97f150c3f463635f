// C ABI of the Hyena operator library: plans, argument validation and kernel
// dispatch. See include/hyena.h for the contract of every entry point.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <new>
#include <vector>

#include "hyena.h"
#include "kernels_1d.cuh"
#include "kernels_1d_cluster.cuh"
#include "kernels_2d.cuh"
#include "kernels_implicit.cuh"
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

// ---------------------------------------------------------------- 1D dispatch
// Elements per thread for each half-length MC (threads per row = MC / E).
constexpr int e_for(int MC) { return MC >= 16384 ? 32 : 16; }

template <int MC>
size_t smem_1d() {
    return (size_t)rows_per_cta(MC, e_for(MC)) * 2 * MC * sizeof(float);
}

template <int MC, typename IO, bool EVEN>
cudaError_t launch_fwd_1d_t(const Fwd1dArgs &a, cudaStream_t st) {
    constexpr int E = e_for(MC);
    constexpr int RPC = rows_per_cta(MC, E);
    auto kern = hyena_fwd_1d_cta<MC, E, IO, EVEN>;
    const size_t sm = smem_1d<MC>();
    if (sm > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
    }
    const int64_t grid = (a.rows + RPC - 1) / RPC;
    kern<<<(unsigned)grid, RPC * (MC / E), sm, st>>>(a);
    return cudaGetLastError();
}

template <int MC>
cudaError_t launch_fwd_1d_mc(const Fwd1dArgs &a, hyena_dtype_t dt, bool even, cudaStream_t st) {
    if (dt == HYENA_F32)
        return even ? launch_fwd_1d_t<MC, float, true>(a, st) : launch_fwd_1d_t<MC, float, false>(a, st);
    return even ? launch_fwd_1d_t<MC, __nv_bfloat16, true>(a, st) : launch_fwd_1d_t<MC, __nv_bfloat16, false>(a, st);
}

template <int MC>
cudaError_t launch_spec_1d_mc(const float *h, int64_t h_stride, int64_t L, c32 *Hout, int64_t nrows, const c32 *tw,
                              cudaStream_t st) {
    constexpr int E = e_for(MC);
    constexpr int RPC = rows_per_cta(MC, E);
    auto kern = hyena_spectrum_1d<MC, E>;
    const size_t sm = smem_1d<MC>();
    if (sm > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
    }
    const int64_t grid = (nrows + RPC - 1) / RPC;
    kern<<<(unsigned)grid, RPC * (MC / E), sm, st>>>(h, h_stride, L, Hout, nrows, tw);
    return cudaGetLastError();
}

#define HY_MC_SWITCH(MCV, CALL)     \
    switch (MCV) {                  \
        case 16: return CALL(16);   \
        case 32: return CALL(32);   \
        case 64: return CALL(64);   \
        case 128: return CALL(128); \
        case 256: return CALL(256); \
        case 512: return CALL(512); \
        case 1024: return CALL(1024); \
        case 2048: return CALL(2048); \
        case 4096: return CALL(4096); \
        case 8192: return CALL(8192); \
        case 16384: return CALL(16384); \
        default: return cudaErrorInvalidValue; \
    }

cudaError_t launch_fwd_1d(const Fwd1dArgs &a, int64_t MC, hyena_dtype_t dt, bool even, cudaStream_t st) {
#define HY_CALL(X) launch_fwd_1d_mc<X>(a, dt, even, st)
    HY_MC_SWITCH(MC, HY_CALL)
#undef HY_CALL
}

cudaError_t launch_spec_1d(const float *h, int64_t h_stride, int64_t L, c32 *Hout, int64_t nrows, int64_t MC,
                           const c32 *tw, cudaStream_t st) {
#define HY_CALL(X) launch_spec_1d_mc<X>(h, h_stride, L, Hout, nrows, tw, st)
    HY_MC_SWITCH(MC, HY_CALL)
#undef HY_CALL
}

cudaError_t launch_implicit(const ImplicitArgs &a, cudaStream_t st) {
    const int64_t grid = (a.npos + IMP_TP - 1) / IMP_TP;
    if (a.p.width <= 64)
        hyena_implicit_filter_kernel<64><<<(unsigned)grid, IMP_THREADS, 0, st>>>(a);
    else
        hyena_implicit_filter_kernel<128><<<(unsigned)grid, IMP_THREADS, 0, st>>>(a);
    return cudaGetLastError();
}

// ------------------------------------------------------------- cluster paths
using G1_32K = ClusterGeom<32768, 4, 128, 16>;    // 1D, 32768 < M <= 65536
using G1_64K = ClusterGeom<65536, 8, 256, 16>;    // 1D, M = 131072
using G1_128K = ClusterGeom<131072, 8, 512, 32>;  // 1D, M = 262144
using G2_32 = ClusterGeom<2048, 1, 64, 16>;       // 2D, 32 x 32 grid (64 x 64 padded)
using G2_64 = ClusterGeom<8192, 2, 128, 16>;      // 2D, 64 x 64
using G2_128 = ClusterGeom<32768, 4, 256, 16>;    // 2D, 128 x 128
using G2_256 = ClusterGeom<131072, 8, 512, 32>;   // 2D, 256 x 256

template <typename G, typename Kern, typename... Args>
cudaError_t launch_cluster(Kern kern, int64_t units, cudaStream_t st, Args... args) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)G::SMEM);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(units * G::C), 1, 1);
    cfg.blockDim = dim3(G::THREADS, 1, 1);
    cfg.dynamicSmemBytes = G::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = G::C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, args...);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <typename G>
cudaError_t launch_fwd_1d_cluster_g(const Fwd1dArgs &a, hyena_dtype_t dt, bool even, cudaStream_t st) {
    if (dt == HYENA_F32)
        return even ? launch_cluster<G>(hyena_fwd_1d_cluster<G, float, true>, a.rows, st, a)
                    : launch_cluster<G>(hyena_fwd_1d_cluster<G, float, false>, a.rows, st, a);
    return even ? launch_cluster<G>(hyena_fwd_1d_cluster<G, __nv_bfloat16, true>, a.rows, st, a)
                : launch_cluster<G>(hyena_fwd_1d_cluster<G, __nv_bfloat16, false>, a.rows, st, a);
}

cudaError_t launch_fwd_1d_cluster(const Fwd1dArgs &a, int64_t MC, hyena_dtype_t dt, bool even, cudaStream_t st) {
    switch (MC) {
        case 32768: return launch_fwd_1d_cluster_g<G1_32K>(a, dt, even, st);
        case 65536: return launch_fwd_1d_cluster_g<G1_64K>(a, dt, even, st);
        case 131072: return launch_fwd_1d_cluster_g<G1_128K>(a, dt, even, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_spec_1d_cluster(const float *h, int64_t h_stride, int64_t L, c32 *Hout, int64_t nrows, int64_t MC,
                                   const c32 *tw, cudaStream_t st) {
    switch (MC) {
        case 32768: return launch_cluster<G1_32K>(hyena_spectrum_1d_cluster<G1_32K>, nrows, st, h, h_stride, L, Hout, tw);
        case 65536: return launch_cluster<G1_64K>(hyena_spectrum_1d_cluster<G1_64K>, nrows, st, h, h_stride, L, Hout, tw);
        case 131072:
            return launch_cluster<G1_128K>(hyena_spectrum_1d_cluster<G1_128K>, nrows, st, h, h_stride, L, Hout, tw);
        default: return cudaErrorInvalidValue;
    }
}

template <typename G>
cudaError_t launch_fwd_2d_g(const Fwd2dArgs &a, hyena_dtype_t dt, cudaStream_t st) {
    if (dt == HYENA_F32) return launch_cluster<G>(hyena_fwd_2d_cluster<G, float>, a.planes, st, a);
    return launch_cluster<G>(hyena_fwd_2d_cluster<G, __nv_bfloat16>, a.planes, st, a);
}

cudaError_t launch_fwd_2d(const Fwd2dArgs &a, int64_t W, hyena_dtype_t dt, cudaStream_t st) {
    switch (W) {
        case 32: return launch_fwd_2d_g<G2_32>(a, dt, st);
        case 64: return launch_fwd_2d_g<G2_64>(a, dt, st);
        case 128: return launch_fwd_2d_g<G2_128>(a, dt, st);
        case 256: return launch_fwd_2d_g<G2_256>(a, dt, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_spec_2d(const float *K, int64_t rs, int64_t cs, c32 *Kout, int64_t n, int64_t W, const c32 *tw,
                           cudaStream_t st) {
    switch (W) {
        case 32: return launch_cluster<G2_32>(hyena_spectrum_2d_cluster<G2_32>, n, st, K, rs, cs, Kout, tw);
        case 64: return launch_cluster<G2_64>(hyena_spectrum_2d_cluster<G2_64>, n, st, K, rs, cs, Kout, tw);
        case 128: return launch_cluster<G2_128>(hyena_spectrum_2d_cluster<G2_128>, n, st, K, rs, cs, Kout, tw);
        case 256: return launch_cluster<G2_256>(hyena_spectrum_2d_cluster<G2_256>, n, st, K, rs, cs, Kout, tw);
        default: return cudaErrorInvalidValue;
    }
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

hyena_status_t check_device(const hyena_plan_s *p) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return HYENA_ERR_CUDA;
    return dev == p->device ? HYENA_OK : HYENA_ERR_INVALID_ARG;
}

hyena_status_t check_implicit(const hyena_plan_s *p, const hyena_implicit_params_t *ip) {
    if (!ip->W1 || !ip->b1 || !ip->W2 || !ip->b2 || !ip->W3 || !ip->b3 || !ip->window) return HYENA_ERR_INVALID_ARG;
    if (ip->width < 4 || ip->width > IMP_MAXW || (ip->width & 3)) return HYENA_ERR_UNSUPPORTED;
    if (p->ndim == 1 && (ip->num_freqs < 0 || 1 + 2 * ip->num_freqs > IMP_MAXF)) return HYENA_ERR_UNSUPPORTED;
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
    a.npos = p->ndim == 1 ? p->L : 4 * p->Hh * p->Ww;
    a.nout = (int64_t)p->order * p->D;
    a.out = out;
    a.out_stride = out_stride;
    a.out_row_stride = out_row_stride;
    return a;
}

}  // namespace

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
    if (!out) return HYENA_ERR_INVALID_ARG;
    *out = nullptr;
    if (!shape || channels < 1 || order < 1 || order > HYENA_MAX_ORDER) return HYENA_ERR_INVALID_ARG;
    if (io_dtype != HYENA_F32 && io_dtype != HYENA_BF16) return HYENA_ERR_INVALID_ARG;
    if (ndim != 1 && ndim != 2) return HYENA_ERR_INVALID_ARG;
    for (int i = 0; i < ndim; ++i)
        if (shape[i] < 1) return HYENA_ERR_INVALID_ARG;
    if ((ndim == 1 && causal != 1) || (ndim == 2 && causal != 0)) return HYENA_ERR_UNSUPPORTED;

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
        p.MC = p.M / 2;
        p.path = p.M <= HYENA_MAX_M_CTA ? HYENA_PATH_CTA : HYENA_PATH_CLUSTER;
        p.spectrum_elems = p.MC + 1;
        p.tw_len = p.M;
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

    std::vector<float2> tw = twiddle_table(p.tw_len);
    if (cudaMalloc(&p.tw, sizeof(float2) * tw.size()) != cudaSuccess) {
        cudaGetLastError();
        return HYENA_ERR_NOMEM;
    }
    if (cudaMemcpy(p.tw, tw.data(), sizeof(float2) * tw.size(), cudaMemcpyHostToDevice) != cudaSuccess) {
        cudaFree(p.tw);
        return HYENA_ERR_CUDA;
    }
    hyena_plan_s *heap = new (std::nothrow) hyena_plan_s(p);
    if (!heap) {
        cudaFree(p.tw);
        return HYENA_ERR_NOMEM;
    }
    *out = heap;
    return HYENA_OK;
}

hyena_status_t hyena_plan_destroy(hyena_plan_t plan) {
    if (!plan) return HYENA_OK;
    hyena_status_t st = HYENA_OK;
    if (plan->tw && cudaFree(plan->tw) != cudaSuccess) st = HYENA_ERR_CUDA;
    delete plan;
    return st;
}

hyena_status_t hyena_plan_info(hyena_plan_t plan, int64_t *fft_len, int64_t *spectrum_elems, int *path) {
    if (!plan) return HYENA_ERR_INVALID_ARG;
    if (fft_len) *fft_len = plan->ndim == 1 ? plan->M : 4 * plan->Hh * plan->Ww;
    if (spectrum_elems) *spectrum_elems = plan->spectrum_elems;
    if (path) *path = plan->path;
    return HYENA_OK;
}

size_t hyena_workspace_bytes(hyena_plan_t plan, int64_t batch) {
    if (!plan || batch < 0) return 0;
    return 0;
}

hyena_status_t hyena_implicit_filter(hyena_plan_t plan, const hyena_implicit_params_t *params, float *h_out,
                                     void *stream) {
    if (!plan || !params || !h_out) return HYENA_ERR_INVALID_ARG;
    hyena_status_t s = check_implicit(plan, params);
    if (s != HYENA_OK) return s;
    if (!aligned16(h_out)) return HYENA_ERR_ALIGNMENT;
    if ((s = check_device(plan)) != HYENA_OK) return s;
    const int64_t stride = plan->ndim == 1 ? plan->L : 4 * plan->Hh * plan->Ww;
    ImplicitArgs a = implicit_args(plan, params, h_out, stride, 2 * plan->Ww);
    return launch_implicit(a, (cudaStream_t)stream) == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;
}

hyena_status_t hyena_filter_spectrum(hyena_plan_t plan, const float *h, const hyena_implicit_params_t *params,
                                     void *H_out, void *stream) {
    if (!plan || !H_out || (!h && !params)) return HYENA_ERR_INVALID_ARG;
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
    if (plan->ndim == 1) {
        int64_t src_stride = plan->L;
        if (!h) {
            // generate the taps inside each row's own output slot, then transform in place
            src_stride = 2 * (plan->MC + 1);
            ImplicitArgs a = implicit_args(plan, params, reinterpret_cast<float *>(H_out), src_stride, 0);
            if (launch_implicit(a, st) != cudaSuccess) return HYENA_ERR_CUDA;
            src = reinterpret_cast<const float *>(H_out);
        }
        e = plan->path == HYENA_PATH_CTA ? launch_spec_1d(src, src_stride, plan->L, Hc, nrows, plan->MC, tw, st)
                                         : launch_spec_1d_cluster(src, src_stride, plan->L, Hc, nrows, plan->MC, tw, st);
    } else {
        int64_t rs = 2 * plan->Ww, cs = 4 * plan->Hh * plan->Ww;
        if (!h) {
            // kernel rows written at the spectrum's row pitch inside each channel's slot
            rs = 2 * (plan->Ww + 1);
            cs = 2 * plan->Hh * rs;
            ImplicitArgs a = implicit_args(plan, params, reinterpret_cast<float *>(H_out), cs, rs);
            if (launch_implicit(a, st) != cudaSuccess) return HYENA_ERR_CUDA;
            src = reinterpret_cast<const float *>(H_out);
        }
        e = launch_spec_2d(src, rs, cs, Hc, nrows, plan->Ww, tw, st);
    }
    return e == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;
}

hyena_status_t hyena_forward(hyena_plan_t plan, int64_t batch, const void *v, const void *const *gates, const void *H,
                             const float *Dskip, void *y, void *workspace, size_t ws_bytes, void *stream) {
    (void)workspace;
    (void)ws_bytes;
    if (!plan || batch < 0) return HYENA_ERR_INVALID_ARG;
    if (batch == 0) return HYENA_OK;  // nothing to read or write; pointers may be NULL
    if (!v || !gates || !H || !y) return HYENA_ERR_INVALID_ARG;
    for (int n = 0; n < plan->order; ++n)
        if (!gates[n]) return HYENA_ERR_INVALID_ARG;
    if (!aligned16(v) || !aligned16(H) || !aligned16(y) || (Dskip && !aligned4(Dskip))) return HYENA_ERR_ALIGNMENT;
    for (int n = 0; n < plan->order; ++n)
        if (!aligned16(gates[n])) return HYENA_ERR_ALIGNMENT;
    hyena_status_t s = check_device(plan);
    if (s != HYENA_OK) return s;

    if (plan->ndim == 2) {
        Fwd2dArgs a;
        std::memset(&a, 0, sizeof(a));
        a.v = v;
        for (int n = 0; n < plan->order; ++n) a.gates[n] = gates[n];
        a.K = reinterpret_cast<const c32 *>(H);
        a.dskip = Dskip;
        a.y = y;
        a.tw = reinterpret_cast<const c32 *>(plan->tw);
        a.planes = batch * plan->D;
        a.C = plan->D;
        a.B = batch;
        a.order = plan->order;
        return launch_fwd_2d(a, plan->Ww, plan->dtype, (cudaStream_t)stream) == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;
    }
    Fwd1dArgs a;
    std::memset(&a, 0, sizeof(a));
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
    const bool even = (plan->L % 2) == 0;
    cudaError_t e = plan->path == HYENA_PATH_CTA
                        ? launch_fwd_1d(a, plan->MC, plan->dtype, even, (cudaStream_t)stream)
                        : launch_fwd_1d_cluster(a, plan->MC, plan->dtype, even, (cudaStream_t)stream);
    return e == cudaSuccess ? HYENA_OK : HYENA_ERR_CUDA;
}

}  // extern "C"
