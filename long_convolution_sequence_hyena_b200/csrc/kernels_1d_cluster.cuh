// 1D kernels for long rows (32768 < M <= 262144): one thread-block cluster of
// C CTAs per channel row, the whole row resident in the cluster's shared
// memory across all N orders.
//
// The packed complex row of MC = M/2 points is transformed as a four-step FFT
// with MC = M1 * M2, element n = M2 * n1 + n2:
//   1. column FFTs of length M1 over n1 (each CTA owns M2/C columns);
//   2. twiddle W_MC^{n2 k1};
//   3. transpose through distributed shared memory (each CTA then owns M1/C
//      rows k1 with all n2);
//   4. row FFTs of length M2 over n2, giving Z[k1 + M1 k2].
// The spectral step reads the mirror bin Z[MC - k] from whichever CTA owns it
// (a DSMEM load), and the inverse runs the same steps backwards, ending in the
// column layout, so the gate and the next order's input stay in registers.
//
// Synchronisation is barrier.cluster only (no flag polling). With two
// buffers (column, row) a transpose needs one cluster barrier after it; with
// a single buffer (when two do not fit) also one before it.
#pragma once
#include <cooperative_groups.h>

#include "kernels_1d.cuh"

namespace hyena {

namespace cg = cooperative_groups;

template <int MC_, int C_, int M1_, int E_>
struct ClusterGeom {
    static constexpr int MC = MC_, C = C_, M1 = M1_, M2 = MC_ / M1_, E = E_;
    static constexpr int NCOL = M2 / C;          // columns per CTA (column phase)
    static constexpr int NROW = M1 / C;          // rows per CTA (row phase)
    static constexpr int T1 = M1 / E;            // threads per column FFT
    static constexpr int T2 = M2 / E;            // threads per row FFT
    static constexpr int THREADS = NCOL * T1;
    static constexpr int PER_CTA = MC / C;       // complex elements per CTA per buffer
    static constexpr bool TWO_BUF = 2 * PER_CTA * 8 <= 160 * 1024;
    static constexpr size_t SMEM = (TWO_BUF ? 2 : 1) * (size_t)PER_CTA * 8;
    static_assert(THREADS == NROW * T2, "both phases must use the same thread count");
    static_assert(NCOL >= 32 && NROW >= 32, "interleaved layouts need at least 32 sequences");
    static_assert(THREADS <= 1024, "too many threads");
};

// Distributed shared memory through 32-bit shared::cluster addresses.
__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ uint32_t dsmem_map(uint32_t local, int rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(rank));
    return remote;
}
__device__ __forceinline__ float dsmem_ld(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ void dsmem_st(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// Interleaved address of element i of sequence s (NSEQ sequences), matching saddr<.., NSEQ>.
template <int NSEQ>
__device__ __forceinline__ int iaddr(int i, int s) {
    return i * NSEQ + (s ^ (i & (NSEQ - 1)));
}

// Per-thread coordinates and buffers of one CTA of the cluster.
// TWID: apply the four-step twiddle W_MC^{n2 k1} between the two FFT stages
// (1D: one transform of length MC); without it the two stages are the two
// axes of a 2D transform of shape [M1][M2].
template <typename G, bool TWID = true>
struct ClusterCtx {
    // Twiddle table length: W_M, M = 2 MC (1D); for 2D the table must cover
    // both axes and the real-packing twiddle: W_{2 M2} with 2 M2 >= M1 (see the plan).
    static constexpr int TWM = TWID ? 2 * G::MC : (2 * G::M2 >= G::M1 ? 2 * G::M2 : G::M1);
    cg::cluster_group cluster;
    float *col_re, *col_im, *row_re, *row_im;
    int j, t1, n2;   // column phase: local column, FFT lane, global column
    int r, t2, k1;   // row phase: local row, FFT lane, global row

    __device__ __forceinline__ ClusterCtx(float *smem) : cluster(cg::this_cluster()) {
        const int crank = (int)cluster.block_rank();
        col_re = smem;
        col_im = col_re + G::PER_CTA;
        row_re = G::TWO_BUF ? col_im + G::PER_CTA : col_re;
        row_im = row_re + G::PER_CTA;
        const int tid = threadIdx.x;
        j = tid % G::NCOL;
        t1 = tid / G::NCOL;
        n2 = crank * G::NCOL + j;
        r = tid % G::NROW;
        t2 = tid / G::NROW;
        k1 = crank * G::NROW + r;
    }

    // Position (complex index) of column-layout register q: n = M2 * (t1 + q T1) + n2.
    __device__ __forceinline__ int64_t col_index(int q) const { return (int64_t)G::M2 * (t1 + q * G::T1) + n2; }
    // Bin of row-layout register q: k = k1 + M1 * (t2 + q T2).
    __device__ __forceinline__ int row_bin(int q) const { return k1 + G::M1 * (t2 + q * G::T2); }

    // Column layout (time domain) -> row layout (natural bins).
    // HALF_COL: the upper half of every column is zero (n1 >= M1/2);
    // HALF_ROW: the upper half of every row is zero after the first stage (n2 >= M2/2).
    template <bool HALF_COL = true, bool HALF_ROW = false>
    __device__ __forceinline__ void forward(c32 (&v)[G::E], const c32 *__restrict__ tw) {
        constexpr int E = G::E;
        fft_cta<G::M1, E, -1, HALF_COL, TWM, G::NCOL>(v, col_re, col_im, t1, tw, j);
        if constexpr (TWID) {
#pragma unroll
            for (int q = 0; q < E; ++q) {
                const int kk = t1 + q * G::T1;
                v[q] = mul(v[q], ldg_c(tw + ((2 * (int64_t)n2 * kk) & (TWM - 1))));
            }
        }
        if constexpr (!G::TWO_BUF) cluster.sync();    // every CTA done reading its buffer
#pragma unroll
        for (int q = 0; q < E; ++q) {
            const int kk = t1 + q * G::T1;
            const uint32_t ad = dsmem_map(smem_u32(row_re + iaddr<G::NROW>(n2, kk % G::NROW)), kk / G::NROW);
            dsmem_st(ad, v[q].x);
            dsmem_st(ad + 4 * G::PER_CTA, v[q].y);
        }
        cluster.sync();
#pragma unroll
        for (int q = 0; q < E; ++q) {
            const int ad = iaddr<G::NROW>(t2 + q * G::T2, r);
            v[q] = mk(row_re[ad], row_im[ad]);
        }
        __syncthreads();
        fft_cta<G::M2, E, -1, HALF_ROW, TWM, G::NROW>(v, row_re, row_im, t2, tw, r);
    }

    // Publish the row-layout spectrum so any CTA can read mirror bins (ends with a cluster barrier).
    __device__ __forceinline__ void publish(const c32 (&v)[G::E]) {
#pragma unroll
        for (int q = 0; q < G::E; ++q) {
            const int ad = iaddr<G::NROW>(t2 + q * G::T2, r);
            row_re[ad] = v[q].x;
            row_im[ad] = v[q].y;
        }
        cluster.sync();
    }

    // Published bin k (any CTA).
    __device__ __forceinline__ c32 bin(int k) {
        const int kr = k % G::M1, kc = k / G::M1;
        const int ad = iaddr<G::NROW>(kc, kr % G::NROW);
        const uint32_t ra = dsmem_map(smem_u32(row_re + ad), kr / G::NROW);
        return mk(dsmem_ld(ra), dsmem_ld(ra + 4 * G::PER_CTA));
    }

    // Row layout (bins) -> column layout (time domain, unscaled inverse).
    __device__ __forceinline__ void inverse(c32 (&v)[G::E], const c32 *__restrict__ tw) {
        constexpr int E = G::E;
        fft_cta<G::M2, E, +1, false, TWM, G::NROW>(v, row_re, row_im, t2, tw, r);
        if constexpr (TWID) {
#pragma unroll
            for (int q = 0; q < E; ++q) {
                const int nn = t2 + q * G::T2;
                v[q] = mul(v[q], conj(ldg_c(tw + ((2 * (int64_t)nn * k1) & (TWM - 1)))));
            }
        }
        if constexpr (!G::TWO_BUF) cluster.sync();
#pragma unroll
        for (int q = 0; q < E; ++q) {
            const int nn = t2 + q * G::T2;
            const uint32_t ad = dsmem_map(smem_u32(col_re + iaddr<G::NCOL>(k1, nn % G::NCOL)), nn / G::NCOL);
            dsmem_st(ad, v[q].x);
            dsmem_st(ad + 4 * G::PER_CTA, v[q].y);
        }
        cluster.sync();
#pragma unroll
        for (int q = 0; q < E; ++q) {
            const int ad = iaddr<G::NCOL>(t1 + q * G::T1, j);
            v[q] = mk(col_re[ad], col_im[ad]);
        }
        __syncthreads();
        fft_cta<G::M1, E, +1, false, TWM, G::NCOL>(v, col_re, col_im, t1, tw, j);
    }
};

// Fused order-N forward, one cluster per row (rows visited d-major, b-minor).
template <typename G, typename IO, bool EVEN>
__global__ void __launch_bounds__(G::THREADS, 1) hyena_fwd_1d_cluster(const Fwd1dArgs a) {
    constexpr int MC = G::MC, E = G::E;
    extern __shared__ float smem[];
    ClusterCtx<G> cx(smem);
    const int64_t ord = (int64_t)blockIdx.x / G::C;     // one cluster per row
    const int64_t d = ord / a.B;
    const int64_t b = ord - d * a.B;
    const int64_t row = b * a.D + d;
    const int64_t L = a.L;

    c32 v[E];
    {
        const IO *vrow = reinterpret_cast<const IO *>(a.v) + row * L;
#pragma unroll
        for (int q = 0; q < E / 2; ++q) v[q] = load_pair<IO, EVEN>(vrow, 2 * cx.col_index(q), L);
#pragma unroll
        for (int q = E / 2; q < E; ++q) v[q] = mk(0.f, 0.f);
    }

    for (int n = 0; n < a.order; ++n) {
        const IO *grow = reinterpret_cast<const IO *>(a.gates[n]) + row * L;
        typename io<IO>::pair_t g[E / 2];
#pragma unroll
        for (int q = 0; q < E / 2; ++q) g[q] = load_pair_raw<IO, EVEN>(grow, 2 * cx.col_index(q), L);
        const float dsk = a.dskip ? __ldg(a.dskip + n * a.D + d) : 0.f;
        const c32 *Hrow = a.H + ((int64_t)n * a.D + d) * (MC + 1);

        cx.forward(v, a.tw);
        cx.publish(v);
        constexpr float s = 0.5f / (float)MC;
#pragma unroll
        for (int q = 0; q < E; ++q) {
            const int k = cx.row_bin(q);
            const c32 Zm = cx.bin((MC - k) & (MC - 1));
            const c32 Zk = v[q];
            const c32 Ek = mk(0.5f * (Zk.x + Zm.x), 0.5f * (Zk.y - Zm.y));
            const c32 Ok = mk(0.5f * (Zk.y + Zm.y), -0.5f * (Zk.x - Zm.x));
            const c32 w = ldg_c(a.tw + k);
            const c32 wO = mul(w, Ok);
            const c32 Xk = add(Ek, wO);
            const c32 Xm = conj(sub(Ek, wO));
            c32 Hk = ldg_c(Hrow + k);
            c32 Hm = ldg_c(Hrow + (MC - k));
            Hk.x += dsk;
            Hm.x += dsk;
            const c32 Yk = mul(Xk, Hk), Ym = mul(Xm, Hm);
            const c32 Ye = mk(s * (Yk.x + Ym.x), s * (Yk.y - Ym.y));
            const c32 Yd = mk(s * (Yk.x - Ym.x), s * (Yk.y + Ym.y));
            const c32 Yo = mul(Yd, conj(w));
            v[q] = mk(Ye.x - Yo.y, Ye.y + Yo.x);
            if ((q & 3) == 3) asm volatile("" ::: "memory");  // bound load hoisting (register pressure)
        }
        cx.cluster.sync();                              // mirror reads done before buffers are rewritten
        cx.inverse(v, a.tw);

        // gate (registers q >= E/2 hold positions >= MC, i.e. padding)
#pragma unroll
        for (int q = 0; q < E / 2; ++q) {
            const int64_t pos = 2 * cx.col_index(q);
            const c32 gq = io<IO>::unpack(g[q]);
            v[q] = mk(pos < L ? gq.x * v[q].x : 0.f, pos + 1 < L ? gq.y * v[q].y : 0.f);
        }
#pragma unroll
        for (int q = E / 2; q < E; ++q) v[q] = mk(0.f, 0.f);
    }

    IO *yrow = reinterpret_cast<IO *>(a.y) + row * L;
#pragma unroll
    for (int q = 0; q < E / 2; ++q) store_pair<IO, EVEN>(yrow, 2 * cx.col_index(q), L, v[q]);
}

// Spectrum of long causal filters (same layout as hyena_spectrum_1d), one
// cluster per filter row. h row o starts at h + o * h_stride and has L taps.
// In place (h == Hout) is allowed: every CTA reads its part of the row before
// the first cluster barrier, and bins are written after the last one.
template <typename G>
__global__ void __launch_bounds__(G::THREADS, 1)
    hyena_spectrum_1d_cluster(const float *h, int64_t h_stride, int64_t L, c32 *Hout, const c32 *__restrict__ tw) {
    constexpr int MC = G::MC, E = G::E;
    extern __shared__ float smem[];
    ClusterCtx<G> cx(smem);
    const int64_t o = (int64_t)blockIdx.x / G::C;
    const float *hrow = h + o * h_stride;
    c32 v[E];
#pragma unroll
    for (int q = 0; q < E / 2; ++q) {
        const int64_t pos = 2 * cx.col_index(q);
        v[q] = mk(pos < L ? hrow[pos] : 0.f, pos + 1 < L ? hrow[pos + 1] : 0.f);
    }
#pragma unroll
    for (int q = E / 2; q < E; ++q) v[q] = mk(0.f, 0.f);
    cx.cluster.sync();                                  // whole row read before any bin is written
    cx.forward(v, tw);
    cx.publish(v);
    c32 *Hrow = Hout + o * (MC + 1);
    c32 outv[E];
    c32 nyq = mk(0.f, 0.f);
#pragma unroll
    for (int q = 0; q < E; ++q) {
        const int k = cx.row_bin(q);
        const c32 Zm = cx.bin((MC - k) & (MC - 1));
        const c32 Zk = v[q];
        const c32 Ek = mk(0.5f * (Zk.x + Zm.x), 0.5f * (Zk.y - Zm.y));
        const c32 Ok = mk(0.5f * (Zk.y + Zm.y), -0.5f * (Zk.x - Zm.x));
        outv[q] = add(Ek, mul(ldg_c(tw + k), Ok));
        if (k == 0) nyq = mk(Ek.x - Ok.x, 0.f);
    }
    cx.cluster.sync();                                  // all mirror reads done; no CTA touches DSMEM after this
#pragma unroll
    for (int q = 0; q < E; ++q) {
        const int k = cx.row_bin(q);
        Hrow[k] = outv[q];
        if (k == 0) Hrow[MC] = nyq;
    }
}

}  // namespace hyena
