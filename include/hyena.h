/*
 * hyena.h -- C ABI of the B200 (sm_100a) Hyena operator library (libhyena.so).
 *
 * The operator ("Hyena — Long Convolutions Math", "The Toeplitz picture";
 * "Hyena, Long Convolution, and Linear Attention", "The Hyena operator" and
 * "FFTConv: the O(L log L) primitive"):
 *
 *     z^0 = v
 *     z^n = x^n ⊙ ( h^n ∗ z^{n-1}  +  Dskip^n ⊙ z^{n-1} )      n = 1..N
 *     y   = z^N
 *
 * with ∗ a depthwise causal convolution along the sequence (1D) or a depthwise
 * linear, non-causal convolution over a grid ("How HyenaND works", "2. The
 * convolution theorem (FFT)"). Every convolution is computed by FFT on inputs
 * zero-padded to M = next_pow2(2L) (per grid axis in 2D), so the cyclic
 * product never wraps ("Hyena — Long Convolutions Math", "Linear vs circular").
 *
 * Conventions shared by every call
 *  - All tensor pointers are DEVICE pointers owned by the caller, contiguous
 *    and 16-byte aligned, unless a comment says "host".
 *  - Activation layout: 1D [B, D, L] (one channel row per (b, d); or [B, L, D],
 *    see hyena_plan_set_layout); 2D [B, C, H, W]; 3D [B, C, Dz, H, W]. io
 *    dtype is the plan's (fp32 or bf16); filters, spectra
 *    and Dskip are always fp32 / complex64 (interleaved re, im).
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream). Calls only
 *    enqueue work; none synchronises the host except plan create / destroy.
 *  - Arguments are validated on the host before anything is launched; a call
 *    that returns an error has launched nothing (HYENA_ERR_CUDA excepted: the
 *    launch itself failed). Nothing aborts the process.
 *  - Calls on one plan from several host threads are safe: a plan is read-only
 *    after creation, apart from the staged paths' streams and spectrum
 *    scratch, whose use every call orders on the GPU itself (each call forks
 *    and joins those streams with events of its own).
 */
#ifndef HYENA_H
#define HYENA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define HYENA_MAX_ORDER 8

#if defined(__GNUC__)
#define HYENA_API __attribute__((visibility("default")))
#else
#define HYENA_API
#endif

typedef struct hyena_plan_s *hyena_plan_t;

typedef enum { HYENA_F32 = 0, HYENA_BF16 = 1 } hyena_dtype_t;

typedef enum {
    HYENA_OK = 0,
    HYENA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad enum */
    HYENA_ERR_UNSUPPORTED = 2,   /* valid but outside what this library implements */
    HYENA_ERR_ALIGNMENT = 3,     /* a device pointer is not 16-byte aligned */
    HYENA_ERR_WORKSPACE = 4,     /* workspace missing or smaller than hyena_workspace_bytes */
    HYENA_ERR_CUDA = 5,          /* a CUDA runtime call or launch failed */
    HYENA_ERR_NOMEM = 6          /* host or device allocation failed (plan create only) */
} hyena_status_t;

/* Which kernel family a plan runs (hyena_plan_info). */
typedef enum {
    HYENA_PATH_CTA = 0,          /* 1D, M <= 32768: one CTA per row, all orders fused */
    HYENA_PATH_CLUSTER = 1,      /* 1D, M = 262144: a thread-block cluster per row */
    HYENA_PATH_2D = 2,           /* 2D grid (H = W = 256: column and row kernels through a workspace;
                                    smaller grids: a thread-block cluster per plane) */
    HYENA_PATH_STAGED = 3,       /* 1D, M from 65536 to 1048576: column and row kernels per order,
                                    the row's transform in a device workspace */
    HYENA_PATH_3D = 4            /* 3D grid: one batched 1D transform stage per axis through a
                                    device workspace */
} hyena_path_t;

/* Activation layout of a 1D plan (hyena_plan_set_layout). */
typedef enum {
    HYENA_LAYOUT_BDL = 0,        /* [B, D, L]: each channel row contiguous (the default) */
    HYENA_LAYOUT_BLD = 1         /* [B, L, D]: channels-last, the layout u ∈ R^{B×L×D} of the
                                    operator's statement ("Hyena, Long Convolution, and Linear
                                    Attention", "FFTConv: the O(L log L) primitive") */
} hyena_layout_t;

/*
 * Parameters of the implicit filter network, all DEVICE pointers to fp32.
 *
 * 1D ("Hyena — Long Convolutions Math", "Implicit filters: an MLP over
 * positions" and "The decay window"): positional features
 *   g(t) = [t/L, cos(2π·1·t/L), sin(2π·1·t/L), ..., cos(2π·K·t/L), sin(2π·K·t/L)]
 * (in = 1 + 2K, K = num_freqs), then
 *   a1 = sin(omega0 (W1 g + b1)), a2 = sin(omega_hidden (W2 a1 + b2)), o = W3 a2 + b3,
 *   h[n, d, t] = exp(-window[n*D + d] * t) * o[n*D + d]        (window = decay rates α ≥ 0)
 * 2D ("How HyenaND works", "1. An implicit filter"): coordinates
 *   p = (oy / H, ox / W), oy in [-H, H), ox in [-W, W)  (in = 2, num_freqs ignored),
 *   same two sine layers and head, K[n, c, oy + H, ox + W] =
 *   exp(-|p|^2 / (2 window[n*C + c]^2)) * o[n*C + c]           (window = Gaussian σ > 0)
 * 3D: p = (oz / Dz, oy / H, ox / W) (in = 3), K[n, c, oz + Dz, oy + H, ox + W]
 *   with the same Gaussian window of |p|^2; width 64 only.
 * Shapes: W1 [width, in], b1 [width], W2 [width, width], b2 [width],
 * W3 [N*D, width], b3 [N*D], window [N*D]; row-major. width <= 128 and a
 * multiple of 4; num_freqs <= 32. W3 must be 16-byte aligned.
 */
typedef struct {
    const float *W1, *b1, *W2, *b2, *W3, *b3;
    const float *window;
    int32_t width;
    int32_t num_freqs;
    float omega0;
    float omega_hidden;
} hyena_implicit_params_t;

/*
 * Create a plan.
 *   ndim      1 (sequence) or 2 (grid)
 *   shape     host array of ndim sizes: {L}, {H, W} or {Dz, H, W}; each >= 1.
 *             1D: L <= 524288. 2D: H == W, one of 32, 64, 128, 256.
 *             3D: Dz, H, W each 16, 32 or 64.
 *   channels  D (1D) or C (2D), >= 1
 *   order     N, 1..HYENA_MAX_ORDER
 *   io_dtype  storage type of v, the gates and y
 *   causal    must be 1 for ndim 1 and 0 for ndim 2 and 3
 * Allocates the plan's device twiddle tables on the current device (the plan
 * may only be used on that device) and synchronises. *out is NULL on error.
 */
HYENA_API hyena_status_t hyena_plan_create(hyena_plan_t *out, int ndim, const int64_t *shape, int64_t channels,
                                 int order, hyena_dtype_t io_dtype, int causal);

/*
 * Select the activation layout of v, the gates and y for every later forward
 * call on a 1D plan (hyena_forward, hyena_forward_host, hyena_forward_no_alloc).
 * With HYENA_LAYOUT_BLD the kernels read and write the [B, L, D] tensors in
 * place (no transpose pass): channel d of batch element b is the strided row
 * at b L D + d with stride D. Filters, spectra and Dskip keep their layouts.
 * 2D plans accept only HYENA_LAYOUT_BDL ([B, C, H, W]); another value returns
 * HYENA_ERR_UNSUPPORTED, an unknown one HYENA_ERR_INVALID_ARG. Call it before
 * the plan's first forward; it must not run concurrently with other calls on
 * the plan.
 */
HYENA_API hyena_status_t hyena_plan_set_layout(hyena_plan_t plan, int layout);

/*
 * Errors that kernels of this plan recorded on the device. A kernel that
 * waits on a barrier of its own (the tensor-core implicit network) bounds
 * every wait; when one runs out it records the event in a device word of the
 * plan, abandons the remaining work of that call and still exits cleanly, so
 * the context stays usable. This call copies that word to the host (it
 * synchronises with the device: call it after the work to check), stores it
 * in *flags if flags is not NULL, clears it when clear != 0, and returns
 * HYENA_ERR_CUDA if an error was recorded, HYENA_OK otherwise.
 */
HYENA_API hyena_status_t hyena_plan_device_errors(hyena_plan_t plan, int *flags, int clear);
/* Bits of the device error word: a bounded wait ran out; an index check of
 * the HYENA_CHECK_BOUNDS debug build (libhyena_checked.so) failed and the
 * access was skipped. */
#define HYENA_DEVERR_WAIT_TIMEOUT 1
#define HYENA_DEVERR_BOUNDS 4

/*
 * The number of kernels this library has enqueued in the calling process
 * since it was loaded, over all plans, threads and streams (a launch is
 * counted when it is enqueued, whether or not it has run yet). Reading it
 * before and after a call gives the kernels that call launched; it never
 * touches the device. *count must not be NULL (HYENA_ERR_INVALID_ARG).
 */
HYENA_API hyena_status_t hyena_launch_count(int64_t *count);

/*
 * Test hooks for the failure paths of plan creation (no effect on results).
 * hyena_debug_fail_allocation(n): the n-th resource that plan creation
 * creates from now on (device buffer, stream or host object, counted over all
 * threads) fails as if the device or host were out of memory; the plan call
 * then releases what it had created and returns HYENA_ERR_NOMEM (a stream:
 * HYENA_ERR_CUDA). n = 0 disarms it; n < 0 is HYENA_ERR_INVALID_ARG.
 * hyena_debug_plan_resources(&n): the number of such resources all live
 * plans hold; *count must not be NULL.
 */
HYENA_API hyena_status_t hyena_debug_fail_allocation(int nth);
HYENA_API hyena_status_t hyena_debug_plan_resources(int64_t *count);

/*
 * hyena_plan_create with options. flags is 0 (the same plan as
 * hyena_plan_create) or HYENA_PLAN_RADIX3: a 1D plan then pads to the smallest
 * M = 6 * 2^j >= 2L when that is below the power of two ("Hyena — Long
 * Convolutions Math", "Linear vs circular": any transform of at least 2L
 * points keeps the product causal; "Counting the cost": padding 2L up to a
 * power of two can nearly double the work), e.g. 6144 points instead of 8192
 * for L = 3000. Such plans (2^j from 16 to 4096, so L <= 12288) run one
 * channel row per thread group through a radix-3 step and three
 * power-of-two transforms; the spectrum has M/2 + 1 bins as for any 1D plan.
 * Other plans ignore the flag. Unknown flags return HYENA_ERR_INVALID_ARG.
 */
#define HYENA_PLAN_RADIX3 1
HYENA_API hyena_status_t hyena_plan_create_ex(hyena_plan_t *out, int ndim, const int64_t *shape, int64_t channels,
                                              int order, hyena_dtype_t io_dtype, int causal, int flags);

/* Free the plan's device tables (synchronises the device). NULL is accepted. */
HYENA_API hyena_status_t hyena_plan_destroy(hyena_plan_t plan);

/*
 * Geometry of a plan (any out-pointer may be NULL):
 *   fft_len        M (1D), 2H * 2W (2D) or 2Dz * 2H * 2W (3D): the padded transform size
 *   spectrum_elems complex64 elements of one (order, channel) spectrum:
 *                  M/2 + 1 (1D), 2H * (W + 1) (2D) or 2Dz * 2H * 2W (3D)
 *   path           a hyena_path_t
 */
HYENA_API hyena_status_t hyena_plan_info(hyena_plan_t plan, int64_t *fft_len, int64_t *spectrum_elems, int *path);

/*
 * Bytes of device workspace hyena_forward needs for `batch`. It is 0, except
 * on HYENA_PATH_STAGED, on 2D plans with H = W = 256 and on 3D plans. There,
 * rows (planes, volumes) run in chunks that keep their transforms in L2: 1D
 * rows with three chunks of 16 MB in flight, 2D planes with two of 32 MB, 3D
 * volumes one of 32 MB at a time. The workspace holds min(rows, lanes * chunk)
 * transforms: (M/2) * 8 bytes per 1D row, 2H * (W/2) * 8 bytes per plane,
 * Dz * 2H * 2W * 8 bytes per volume.
 */
HYENA_API size_t hyena_workspace_bytes(hyena_plan_t plan, int64_t batch);

/*
 * Evaluate the implicit filter network (see hyena_implicit_params_t) into
 * h_out: [N, D, L] (1D) or [N, C, 2H, 2W] (2D) fp32, device.
 */
HYENA_API hyena_status_t hyena_implicit_filter(hyena_plan_t plan, const hyena_implicit_params_t *params,
                                     float *h_out, void *stream);

/*
 * Filter spectra ("Hyena — Long Convolutions Math", "The convolution theorem":
 * FFT(h) is the filter's transfer function, one gain per frequency).
 *   h       1D: [N, D, L] causal taps 0..L-1 (zero-extended to M);
 *           2D: [N, C, 2H, 2W] kernel on the offset grid, element (oy, ox) at
 *           [oy + H, ox + W], oy in [-H, H), ox in [-W, W).
 *           May be NULL when params is given: the filters are then generated by
 *           the implicit network, inside H_out, with no other memory.
 *   params  implicit network, or NULL (then h must not be NULL)
 *           3D: [N, C, 2Dz, 2H, 2W] kernel on the offset grid, element
 *           (oz, oy, ox) at [oz + Dz, oy + H, ox + W]; h must not be NULL.
 *   H_out   1D: [N, D, M/2 + 1] complex64, bin k = sum_t h[t] e^{-2πi k t / M};
 *           2D: [N, C, W + 1, 2H] complex64, the 2D DFT of the kernel placed
 *           cyclically (offset o at index o mod 2H, o mod 2W), bins over the
 *           full row axis and the non-negative half of the column axis,
 *           stored column-bin-major: bin (ky, kx) at [kx][ky].
 *           3D: [N, C, 2Dz, 2H, 2W] complex64, the full 3D DFT of the kernel
 *           placed cyclically, bin (kz, ky, kx) at [kz][ky][kx].
 *           Unnormalised. Must not overlap h.
 * Plans on HYENA_PATH_STAGED (64 MiB) and 2D plans with H = W = 256 (32 MiB)
 * transform the filters in chunks through a device buffer that the plan
 * allocates at creation and owns. Those chunks run on the plan's own two
 * streams, forked from `stream` and joined back to it, so calls on one such
 * plan (from any stream or thread) run one after another on the GPU;
 * hyena_filter_spectrum_ws, with a workspace per caller, lets them overlap.
 */
HYENA_API hyena_status_t hyena_filter_spectrum(hyena_plan_t plan, const float *h, const hyena_implicit_params_t *params,
                                     void *H_out, void *stream);

/*
 * hyena_filter_spectrum with the transforms' scratch supplied by the caller:
 * workspace (device, 16-byte aligned) of at least
 * hyena_filter_spectrum_workspace_bytes(plan) bytes, or NULL for the plan's
 * own (then the same as hyena_filter_spectrum). With a workspace of its own
 * each call is independent of the others on the plan: calls from several
 * threads with separate workspaces overlap on the GPU (the plan's streams
 * carry them, each call with its own fork and join events). A workspace that
 * is too small is HYENA_ERR_WORKSPACE. Plans whose spectra need no scratch
 * (hyena_filter_spectrum_workspace_bytes = 0) ignore it.
 */
HYENA_API hyena_status_t hyena_filter_spectrum_ws(hyena_plan_t plan, const float *h,
                                                  const hyena_implicit_params_t *params, void *H_out,
                                                  void *workspace, size_t ws_bytes, void *stream);
HYENA_API size_t hyena_filter_spectrum_workspace_bytes(hyena_plan_t plan);

/*
 * The fused forward pass: all N orders in one launch per row, each row read
 * once from and written once to device memory.
 *   batch      B >= 0 (B = 0 launches nothing; the pointers are then not read)
 *   v          [B, D, L] or [B, C, H, W], io dtype
 *   gates      HOST array of N device pointers x^1..x^N, each shaped like v
 *   H          spectra from hyena_filter_spectrum
 *   Dskip      [N, D] fp32 feedthrough, or NULL for none
 *   y          output, shaped like v, io dtype; may alias v or a gate
 *              (each row is read completely before it is written)
 *   workspace  device scratch of at least hyena_workspace_bytes(plan, batch)
 *              bytes, or NULL when that is 0
 */
HYENA_API hyena_status_t hyena_forward(hyena_plan_t plan, int64_t batch, const void *v, const void *const *gates,
                             const void *H, const float *Dskip, void *y, void *workspace, size_t ws_bytes,
                             void *stream);

/*
 * The gate sandwich of HyenaND ("How HyenaND works", "How HyenaND stays
 * data-dependent: gating" and "Putting it together: the HyenaND operator"):
 * the inner gate Z = q ⊙ SiLU(k) is the convolution's input and every outer
 * gate passes through SiLU, SiLU(x) = x / (1 + e^{-x}):
 *
 *     z^0 = q ⊙ SiLU(k)
 *     z^n = SiLU(x^n) ⊙ ( K^n ∗ z^{n-1}  +  Dskip^n ⊙ z^{n-1} )     n = 1..N
 *     y   = z^N
 *
 * With one order, no Dskip and gates = {v} this is the page's
 * O = (K ∗ (q ⊙ SiLU(k))) ⊙ SiLU(v). Both gates are formed inside the
 * forward's first load and its gate multiplies (no extra pass over memory).
 *   q, k   [B, C, H, W] io dtype (device), in place of hyena_forward's v
 * The other arguments, the workspace and the aliasing rule (y may alias q, k
 * or a gate) are those of hyena_forward. 2D plans only; 1D plans return
 * HYENA_ERR_UNSUPPORTED.
 */
HYENA_API hyena_status_t hyena_forward_gated(hyena_plan_t plan, int64_t batch, const void *q, const void *k,
                                             const void *const *gates, const void *H, const float *Dskip,
                                             void *y, void *workspace, size_t ws_bytes, void *stream);

/* Static, human-readable name of a status code. */
HYENA_API const char *hyena_status_string(hyena_status_t status);

/*
 * hyena_forward for callers that cannot allocate device memory where they
 * run the operator: a plain C host program linked to this library, which has
 * no allocator of its own to hand out a workspace; a process whose device
 * memory belongs to a framework's caching allocator; a latency-bound loop in
 * which a cudaMalloc, which may synchronise the device, is not acceptable.
 * The pages cited at the top of this file have no counterpart of this call:
 * it changes only where the staged path's scratch lives, not what is
 * computed.
 *
 * Plans on HYENA_PATH_STAGED only (1D, M in {65536, 131072}); any other plan
 * returns HYENA_ERR_UNSUPPORTED. The other arguments are those of
 * hyena_forward, and so is the result.
 *
 * The scratch is one array of HYENA_STATIC_SCRATCH_BYTES in device memory,
 * per device, held from when the library is loaded until the process exits.
 * Rows run in chunks of HYENA_STATIC_SCRATCH_BYTES / (M/2 * 8) rows (32 rows
 * at M = 131072, 64 at M = 65536), one chunk after another on `stream`,
 * through the same kernels as hyena_forward, so y equals hyena_forward's bit
 * for bit; a plan whose two-row transform would not fit returns
 * HYENA_ERR_WORKSPACE. The first call in a CUDA context on a device looks up
 * the array's device address (cudaGetSymbolAddress, with that device
 * current): make that first call before any stream capture. The address is
 * kept with the context's id, so after a device reset (a new context) the
 * next call looks it up again. Nothing in the array has to start at zero (a
 * chunk's transforms are written before they are read), but every call on a
 * device uses the same array: calls whose kernels overlap on the GPU (on
 * different streams, or from different host threads) race; order them on one
 * stream or with events. This call allocates no memory.
 */
#define HYENA_STATIC_SCRATCH_BYTES (16u << 20)   /* 16 MiB */
HYENA_API hyena_status_t hyena_forward_no_alloc(hyena_plan_t plan, int64_t batch, const void *v,
                                                const void *const *gates, const void *H, const float *Dskip,
                                                void *y, void *stream);

/*
 * hyena_forward on activations that live in HOST memory: the call copies the
 * inputs to the device, runs the forward and copies y back, pipelined over
 * the batch so that the host-to-device copies of one stage, the forward of
 * the stage before and the device-to-host copy of the one before that
 * overlap. The pages cited at the top of this file have no counterpart of
 * this call: it moves data, and each stage computes exactly what
 * hyena_forward computes on its rows.
 *
 *   batch       B >= 0 (B = 0 copies and launches nothing)
 *   v_host      [B, D, L] or [B, C, H, W] io dtype, in PAGE-LOCKED host
 *               memory (cudaHostAlloc / cudaMallocHost, or registered with
 *               cudaHostRegister); pageable memory returns
 *               HYENA_ERR_INVALID_ARG, because a copy from the device into
 *               it would block the calling thread
 *   gates_host  HOST array of N pointers x^1..x^N, each page-locked and
 *               shaped like v_host
 *   H, Dskip    DEVICE pointers, as for hyena_forward
 *   y_host      output, page-locked host memory shaped like v_host; must not
 *               overlap v_host or a gate
 *   workspace   device scratch of at least
 *               hyena_forward_host_workspace_bytes(plan, batch) bytes,
 *               16-byte aligned: two stage buffers of inputs and outputs,
 *               then the forward's own workspace for one stage
 *
 * Stages are whole batch elements: as many as make about 8 MiB of input, at
 * most B; in 1D rounded up to an even count, so that two rows of one channel
 * share a thread group. On 1D plans of the staged and cluster paths (M of
 * 65536 and more) in the [B, D, L] layout whose batch element holds more than
 * 16 MiB of input, a stage is instead a range of channels of one batch
 * element: about 16 MiB of input, a whole number of the staged path's chunks
 * (32 rows at M = 131072), so that even B = 1 overlaps its copies with the
 * forward. Each stage's rows equal hyena_forward's bit for bit either way.
 * The copies run on two streams the call creates
 * and releases (cudaStreamDestroy returns at once, and the streams are freed
 * when their work is done). Every copy waits for the work enqueued on
 * `stream` before the call, and work enqueued on `stream` after the call
 * waits for all of them. The host buffers must stay valid, and y_host
 * unread, until then. Concurrent calls need one workspace each.
 */
HYENA_API size_t hyena_forward_host_workspace_bytes(hyena_plan_t plan, int64_t batch);
HYENA_API hyena_status_t hyena_forward_host(hyena_plan_t plan, int64_t batch, const void *v_host,
                                            const void *const *gates_host, const void *H, const float *Dskip,
                                            void *y_host, void *workspace, size_t ws_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* HYENA_H */
