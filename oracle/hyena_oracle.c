/*
 * Oracle for the order-N Hyena operator: plain, slow, fp64, CPU only.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's CPU
 * baseline leg may load this file's library. It shares no code, header, table
 * or constant with the CUDA library: it is the definition written out, with no
 * FFT, no blocking and no reordering beyond the sum the definition states.
 *
 * What it computes (citations are page title + section):
 *
 *  hyena_oracle_1d — the order-N Hyena recurrence
 *      z^0 = v
 *      z^n_t = x^n_t * ( sum_{tau=0..t} h^n_{t-tau} z^{n-1}_tau  +  D^n * z^{n-1}_t )
 *      y = z^N
 *    * the causal convolution y_t = sum_{tau<=t} h_{t-tau} x_tau:
 *      "Hyena — Long Convolutions Math", "The primitive: a causal convolution
 *      over the whole sequence";
 *    * the feedthrough b_d * u_{b,t,d} added to each convolution:
 *      "Hyena, Long Convolution, and Linear Attention", "FFTConv: the
 *      O(L log L) primitive";
 *    * the interleaving of convolutions and gates, v convolved first, gates
 *      x^1..x^N applied in order: "Hyena — Long Convolutions Math", "The
 *      Toeplitz picture" (y = x^2 ⊙ (h^2 ∗ (x^1 ⊙ (h^1 ∗ v)))), and
 *      "Hyena, Long Convolution, and Linear Attention", "The Hyena operator".
 *    Rows are depthwise-independent ("The primitive": channel c is convolved
 *    only with filter c), so a row carries its own filter index.
 *
 *  hyena_oracle_2d — the 2D (HyenaND-style) global convolution with gate
 *      c[i,j]   = sum_{i',j'} K[i-i', j-j'] * z[i',j']   (linear, non-causal)
 *      z^n[i,j] = x^n[i,j] * (c[i,j] + D^n * z^{n-1}[i,j])
 *    "How HyenaND works", "2. The convolution theorem (FFT)" (FFT on the native
 *    grid, zero padding, non-causal) and "How HyenaND stays data-dependent:
 *    gating". The kernel is stored on the offset grid [-H, H) x [-W, W),
 *    element (oy, ox) at index ((oy + H) * 2W + (ox + W)).
 *
 * Parity pins for both functions live in the CPU test suite.
 */
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <unistd.h>

typedef struct {
    int64_t row_begin, row_end;
    int64_t L, N, F, R;
    const double *v, *x, *h, *dskip;
    const int64_t *fidx;
    double *y;
} job1d_t;

/* One row of the order-N chain, exactly as written in the header comment. */
static void hyena_row_1d(const job1d_t *j, int64_t r, double *z, double *znew) {
    const int64_t L = j->L;
    const int64_t f = j->fidx[r];
    for (int64_t t = 0; t < L; ++t) z[t] = j->v[r * L + t];
    for (int64_t n = 0; n < j->N; ++n) {
        const double *h = j->h + (n * j->F + f) * L;      /* h^n for this channel */
        const double *xg = j->x + (n * j->R + r) * L;     /* gate x^n for this row */
        const double d = j->dskip ? j->dskip[n * j->F + f] : 0.0;
        for (int64_t t = 0; t < L; ++t) {
            double c = 0.0;
            for (int64_t tau = 0; tau <= t; ++tau) c += h[t - tau] * z[tau];
            znew[t] = xg[t] * (c + d * z[t]);
        }
        for (int64_t t = 0; t < L; ++t) z[t] = znew[t];
    }
    for (int64_t t = 0; t < L; ++t) j->y[r * L + t] = z[t];
}

static void *worker_1d(void *arg) {
    const job1d_t *j = (const job1d_t *)arg;
    double *z = (double *)malloc(sizeof(double) * (size_t)(2 * j->L));
    if (!z) return (void *)1;
    for (int64_t r = j->row_begin; r < j->row_end; ++r) hyena_row_1d(j, r, z, z + j->L);
    free(z);
    return NULL;
}

int hyena_oracle_num_threads(void) {
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

/*
 * R rows of length L, order N.
 *   v      [R, L]        conv input of order 1
 *   x      [N, R, L]     gates x^1..x^N
 *   h      [N, F, L]     filters (F filter rows per order)
 *   dskip  [N, F] or NULL (NULL means no feedthrough)
 *   fidx   [R]           filter row used by each data row
 *   y      [R, L]        output
 *   threads <= 0 means one per online CPU.
 * Returns 0, or -1 on bad arguments / allocation failure.
 */
int hyena_oracle_1d(int64_t R, int64_t L, int64_t N, int64_t F,
                    const double *v, const double *x, const double *h,
                    const double *dskip, const int64_t *fidx, double *y, int threads) {
    if (R < 0 || L < 0 || N < 1 || F < 1 || !v || !x || !h || !fidx || !y) return -1;
    for (int64_t r = 0; r < R; ++r)
        if (fidx[r] < 0 || fidx[r] >= F) return -1;
    if (R == 0 || L == 0) return 0;
    if (threads <= 0) threads = hyena_oracle_num_threads();
    if (threads > R) threads = (int)R;
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)threads);
    job1d_t *jobs = (job1d_t *)malloc(sizeof(job1d_t) * (size_t)threads);
    if (!tid || !jobs) { free(tid); free(jobs); return -1; }
    int rc = 0;
    for (int i = 0; i < threads; ++i) {
        job1d_t j = {R * i / threads, R * (i + 1) / threads, L, N, F, R, v, x, h, dskip, fidx, y};
        jobs[i] = j;
        if (pthread_create(&tid[i], NULL, worker_1d, &jobs[i]) != 0) { threads = i; rc = -1; break; }
    }
    for (int i = 0; i < threads; ++i) {
        void *ret = NULL;
        pthread_join(tid[i], &ret);
        if (ret) rc = -1;
    }
    free(tid);
    free(jobs);
    return rc;
}

typedef struct {
    int64_t p_begin, p_end;
    int64_t H, W, N, F, P;
    const double *v, *x, *k, *dskip;
    const int64_t *fidx;
    double *y;
} job2d_t;

/* One plane (one (batch, channel) pair) of the 2D chain. */
static void hyena_plane_2d(const job2d_t *j, int64_t p, double *z, double *znew) {
    const int64_t H = j->H, W = j->W, HW = H * W;
    const int64_t f = j->fidx[p];
    for (int64_t i = 0; i < HW; ++i) z[i] = j->v[p * HW + i];
    for (int64_t n = 0; n < j->N; ++n) {
        const double *K = j->k + (n * j->F + f) * (4 * HW);   /* [2H, 2W] offset grid */
        const double *xg = j->x + (n * j->P + p) * HW;
        const double d = j->dskip ? j->dskip[n * j->F + f] : 0.0;
        for (int64_t iy = 0; iy < H; ++iy)
            for (int64_t ix = 0; ix < W; ++ix) {
                double c = 0.0;
                for (int64_t sy = 0; sy < H; ++sy)
                    for (int64_t sx = 0; sx < W; ++sx) {
                        const int64_t oy = iy - sy, ox = ix - sx;   /* offset in (-H, H) x (-W, W) */
                        c += K[(oy + H) * (2 * W) + (ox + W)] * z[sy * W + sx];
                    }
                znew[iy * W + ix] = xg[iy * W + ix] * (c + d * z[iy * W + ix]);
            }
        for (int64_t i = 0; i < HW; ++i) z[i] = znew[i];
    }
    for (int64_t i = 0; i < HW; ++i) j->y[p * HW + i] = z[i];
}

static void *worker_2d(void *arg) {
    const job2d_t *j = (const job2d_t *)arg;
    double *z = (double *)malloc(sizeof(double) * (size_t)(2 * j->H * j->W));
    if (!z) return (void *)1;
    for (int64_t p = j->p_begin; p < j->p_end; ++p) hyena_plane_2d(j, p, z, z + j->H * j->W);
    free(z);
    return NULL;
}

/*
 * P planes of H x W, order N.
 *   v      [P, H, W]
 *   x      [N, P, H, W]
 *   k      [N, F, 2H, 2W]   kernels on the offset grid (see header comment)
 *   dskip  [N, F] or NULL
 *   fidx   [P]
 *   y      [P, H, W]
 */
int hyena_oracle_2d(int64_t P, int64_t H, int64_t W, int64_t N, int64_t F,
                    const double *v, const double *x, const double *k,
                    const double *dskip, const int64_t *fidx, double *y, int threads) {
    if (P < 0 || H < 0 || W < 0 || N < 1 || F < 1 || !v || !x || !k || !fidx || !y) return -1;
    for (int64_t p = 0; p < P; ++p)
        if (fidx[p] < 0 || fidx[p] >= F) return -1;
    if (P == 0 || H == 0 || W == 0) return 0;
    if (threads <= 0) threads = hyena_oracle_num_threads();
    if (threads > P) threads = (int)P;
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)threads);
    job2d_t *jobs = (job2d_t *)malloc(sizeof(job2d_t) * (size_t)threads);
    if (!tid || !jobs) { free(tid); free(jobs); return -1; }
    int rc = 0;
    for (int i = 0; i < threads; ++i) {
        job2d_t j = {P * i / threads, P * (i + 1) / threads, H, W, N, F, P, v, x, k, dskip, fidx, y};
        jobs[i] = j;
        if (pthread_create(&tid[i], NULL, worker_2d, &jobs[i]) != 0) { threads = i; rc = -1; break; }
    }
    for (int i = 0; i < threads; ++i) {
        void *ret = NULL;
        pthread_join(tid[i], &ret);
        if (ret) rc = -1;
    }
    free(tid);
    free(jobs);
    return rc;
}

/* ------------------------------------------------------------------------ 3D
 * The same gated global convolution on a 3D grid ("How HyenaND works", "2. The
 * convolution theorem (FFT)": in N dimensions the convolution runs on the
 * native grid, a 3D volume included). Kernel (n, f) lives on offsets
 * oz in [-Dz, Dz), oy in [-H, H), ox in [-W, W), stored [2Dz, 2H, 2W] with
 * offset (oz, oy, ox) at [oz + Dz, oy + H, ox + W]; the output at voxel
 * (iz, iy, ix) sums K(iz - sz, iy - sy, ix - sx) z(sz, sy, sx) over the grid.
 */
typedef struct {
    int64_t p_begin, p_end;
    int64_t Dz, H, W, N, F, P;
    const double *v, *x, *k, *dskip;
    const int64_t *fidx;
    double *y;
} job3d_t;

static void hyena_plane_3d(const job3d_t *j, int64_t p, double *z, double *znew) {
    const int64_t Dz = j->Dz, H = j->H, W = j->W, V = Dz * H * W;
    const int64_t f = j->fidx[p];
    for (int64_t i = 0; i < V; ++i) z[i] = j->v[p * V + i];
    for (int64_t n = 0; n < j->N; ++n) {
        const double *K = j->k + (n * j->F + f) * (8 * V);   /* [2Dz, 2H, 2W] offset grid */
        const double *xg = j->x + (n * j->P + p) * V;
        const double d = j->dskip ? j->dskip[n * j->F + f] : 0.0;
        for (int64_t iz = 0; iz < Dz; ++iz)
            for (int64_t iy = 0; iy < H; ++iy)
                for (int64_t ix = 0; ix < W; ++ix) {
                    double c = 0.0;
                    for (int64_t sz = 0; sz < Dz; ++sz)
                        for (int64_t sy = 0; sy < H; ++sy)
                            for (int64_t sx = 0; sx < W; ++sx) {
                                const int64_t oz = iz - sz, oy = iy - sy, ox = ix - sx;
                                c += K[((oz + Dz) * (2 * H) + (oy + H)) * (2 * W) + (ox + W)] *
                                     z[(sz * H + sy) * W + sx];
                            }
                    const int64_t o = (iz * H + iy) * W + ix;
                    znew[o] = xg[o] * (c + d * z[o]);
                }
        for (int64_t i = 0; i < V; ++i) z[i] = znew[i];
    }
    for (int64_t i = 0; i < V; ++i) j->y[p * V + i] = z[i];
}

static void *worker_3d(void *arg) {
    const job3d_t *j = (const job3d_t *)arg;
    const int64_t V = j->Dz * j->H * j->W;
    double *z = (double *)malloc(sizeof(double) * (size_t)(2 * V));
    if (!z) return (void *)1;
    for (int64_t p = j->p_begin; p < j->p_end; ++p) hyena_plane_3d(j, p, z, z + V);
    free(z);
    return NULL;
}

/*
 * P volumes of Dz x H x W, order N.
 *   v      [P, Dz, H, W]
 *   x      [N, P, Dz, H, W]
 *   k      [N, F, 2Dz, 2H, 2W]   kernels on the offset grid
 *   dskip  [N, F] or NULL
 *   fidx   [P]
 *   y      [P, Dz, H, W]
 */
int hyena_oracle_3d(int64_t P, int64_t Dz, int64_t H, int64_t W, int64_t N, int64_t F,
                    const double *v, const double *x, const double *k,
                    const double *dskip, const int64_t *fidx, double *y, int threads) {
    if (P < 0 || Dz < 0 || H < 0 || W < 0 || N < 1 || F < 1 || !v || !x || !k || !fidx || !y) return -1;
    for (int64_t p = 0; p < P; ++p)
        if (fidx[p] < 0 || fidx[p] >= F) return -1;
    if (P == 0 || Dz == 0 || H == 0 || W == 0) return 0;
    if (threads <= 0) threads = hyena_oracle_num_threads();
    if (threads > P) threads = (int)P;
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)threads);
    job3d_t *jobs = (job3d_t *)malloc(sizeof(job3d_t) * (size_t)threads);
    if (!tid || !jobs) { free(tid); free(jobs); return -1; }
    int rc = 0;
    for (int i = 0; i < threads; ++i) {
        job3d_t j = {P * i / threads, P * (i + 1) / threads, Dz, H, W, N, F, P, v, x, k, dskip, fidx, y};
        jobs[i] = j;
        if (pthread_create(&tid[i], NULL, worker_3d, &jobs[i]) != 0) { threads = i; rc = -1; break; }
    }
    for (int i = 0; i < threads; ++i) {
        void *ret = NULL;
        pthread_join(tid[i], &ret);
        if (ret) rc = -1;
    }
    free(tid);
    free(jobs);
    return rc;
}
