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
// The spectral step reads the mirror bin Z[MC - k] from the same CTA (rows
// are assigned in mirror pairs), and the inverse runs the same steps
// backwards, ending in the column layout, so the gate and the next order's
// input stay in registers.
//
// Synchronisation is barrier.cluster only (no flag polling): one cluster
// barrier after each transpose, two per order. Rows are paired with their
// mirror rows inside one CTA, so the spectral step reads only local shared
// memory.
#pragma once
#include <cooperative_groups.h>

#include "kernels_1d.cuh"

namespace hyena {

namespace cg = cooperative_groups;

// MINB: CTAs resident per SM (the launch bounds); with 2, one cluster's
// barrier waits are covered by another cluster's work on the same SMs.
template <int MC_, int C_, int M1_, int E_, int MINB_ = 1>
struct ClusterGeom {
    static constexpr int MC = MC_, C = C_, M1 = M1_, M2 = MC_ / M1_, E = E_, MINB = MINB_;
    static constexpr int NCOL = M2 / C;          // columns per CTA (column phase)
    static constexpr int NROW = M1 / C;          // rows per CTA (row phase), in mirror pairs
    static constexpr int HROW = NROW / 2;        // rows k1 < M1/2 per CTA
    static constexpr int T1 = M1 / E;            // threads per column FFT
    static constexpr int T2 = M2 / E;            // threads per row FFT
    static constexpr int THREADS = NCOL * T1;
    static constexpr int PER_CTA = MC / C;       // complex elements per CTA per buffer
    // column buffer + row buffer + staging for one order's gates (E/2 element pairs per thread and row)
    static constexpr size_t GATE_STAGE = (size_t)THREADS * (E / 2) * 8;
    static constexpr size_t SMEM = 2 * (size_t)PER_CTA * 8 + GATE_STAGE;
    static_assert(THREADS == NROW * T2, "both phases must use the same thread count");
    static_assert(NCOL >= 16 && NROW >= 16, "warps must span at least 16 sequences");
    static_assert(M1 >= 32 && M2 >= 32, "sequence-major layouts need sequences of at least 32");
    static_assert(THREADS <= 1024, "too many threads");
    static_assert(SMEM <= 200 * 1024, "buffers must fit in shared memory");
    static_assert(MINB * (SMEM + 1024) <= 228 * 1024, "MINB CTAs must fit in one SM's shared memory");
    static_assert(MINB * THREADS <= 2048, "MINB CTAs must fit in one SM's thread slots");
};

// Distributed shared memory through 32-bit shared::cluster addresses.
__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ uint32_t dsmem_map(uint32_t local, int rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(rank));
    return remote;
}
__device__ __forceinline__ void dsmem_st(uint32_t addr, c32 v) {
    asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(v.x), "f"(v.y) : "memory");
}
// Cluster barrier that also orders shared::cluster memory (release / acquire).
__device__ __forceinline__ void cluster_sync_mem() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Rows of the row phase are held in mirror pairs: CTA c owns rows k1 in
// [c HROW, (c+1) HROW) (slots 0..HROW-1) and their mirrors M1 - k1 (slots
// HROW..NROW-1; the mirror slot of row 0 holds row M1/2). Every bin's mirror
// bin then lies in the same CTA, so the spectral step needs no DSMEM access.
template <typename G>
__device__ __forceinline__ int row_of_slot(int c, int r) {
    const int base = c * G::HROW + (r % G::HROW);
    if (r < G::HROW) return base;
    return base == 0 ? G::M1 / 2 : G::M1 - base;
}
template <typename G>
__device__ __forceinline__ void slot_of_row(int k1, int &c, int &r) {
    if (k1 < G::M1 / 2) {
        c = k1 / G::HROW;
        r = k1 % G::HROW;
    } else if (k1 == G::M1 / 2) {
        c = 0;
        r = G::HROW;
    } else {
        const int kb = G::M1 - k1;
        c = kb / G::HROW;
        r = G::HROW + kb % G::HROW;
    }
}

// Per-thread coordinates and buffers of one CTA of the cluster.
// TWID: apply the four-step twiddle W_MC^{n2 k1} between the two FFT stages
// (1D: one transform of length MC); without it the two stages are the two
// axes of a 2D transform of shape [M1][M2].
// HALFX: columns n2 >= M2/2 hold zeros on input and are not needed on output
// (2D, the zero-padded half of the x axis): they are neither transformed nor
// sent, and the M2/2 data columns are spread over all C CTAs (NCOLP = NCOL/2
// per CTA, twice the threads per column, E/2 values per thread), so that no
// CTA idles through the column phase.
template <typename G, bool TWID, bool HALFX>
struct ClusterCtx {
    using V = c32;
    using SE = selem<c32>;
    using ET = float2;
    static constexpr int NCOLP = HALFX ? G::NCOL / 2 : G::NCOL;   // columns per CTA, column phase
    static constexpr int T1P = G::THREADS / NCOLP;                // threads per column FFT
    static constexpr int E1 = G::M1 / T1P;                        // values per thread, column phase
    static_assert(NCOLP * T1P == G::THREADS && E1 * T1P == G::M1, "column phase must use every thread");
    static_assert(E1 == 8 || E1 == 16, "column FFTs run radix-8 or radix-16 passes");
    static_assert(NCOLP == 8 || NCOLP >= 16, "warps must span 8 or at least 16 columns");
    // Twiddle table length: 1D, W_M with M = 2 MC; 2D, W_{2 M2} with 2 M2 >= M1.
    // The plan appends W_1024 to it for the sub-transforms (kept L1-resident).
    static constexpr int TWM = TWID ? 2 * G::MC : (2 * G::M2 >= G::M1 ? 2 * G::M2 : G::M1);
    static constexpr int TWS = 1024;
    static_assert(TWS % G::M1 == 0 && TWS % G::M2 == 0, "sub-transform twiddles");
    ET *colb, *rowb;       // column and row buffers, interleaved complex, sequence-major
    int crank;
    int j, t1, n2;   // column phase: local column, FFT lane, global column
    int r, t2, k1;   // row phase: local slot, FFT lane, global row
    int rm;          // slot of the mirror row of k1

    __device__ __forceinline__ ClusterCtx(float *smem) {
        crank = (int)cg::this_cluster().block_rank();
        colb = reinterpret_cast<ET *>(smem);
        rowb = colb + G::PER_CTA;
        const int tid = threadIdx.x;
        j = tid % NCOLP;
        t1 = tid / NCOLP;
        n2 = crank * NCOLP + j;
        r = tid % G::NROW;
        t2 = tid / G::NROW;
        k1 = row_of_slot<G>(crank, r);
        rm = (k1 == 0 || k1 == G::M1 / 2) ? r : (r < G::HROW ? r + G::HROW : r - G::HROW);
    }

    // The column-phase registers: the first E1 of the E.
    __device__ __forceinline__ static V (&col_regs(V (&v)[G::E]))[E1] {
        if constexpr (E1 == G::E) return v;
        else return *reinterpret_cast<V (*)[E1]>(&v[0]);
    }

    // Complex index of column-layout register q: n = M2 * (t1 + q T1P) + n2.
    __device__ __forceinline__ int64_t col_index(int q) const { return (int64_t)G::M2 * (t1 + q * T1P) + n2; }

    // v[q] *= base * step^q, q = 0..E-1 (product tree of depth <= 4, then one multiply).
    __device__ __forceinline__ static void twiddle_ramp(V (&v)[G::E], c32 base, c32 step) {
        twiddle_powers<G::E, 1, 0>(v, step);
#pragma unroll
        for (int q = 0; q < G::E; ++q) v[q] = mul(v[q], base);
    }

    // Column layout (registers q < E1: time domain, upper half of every column
    // zero unless !HALF_COL) -> row layout (natural bins, register q = bin
    // k2 = t2 + q T2 of row k1).
    template <bool HALF_COL>
    __device__ __forceinline__ void forward(V (&v)[G::E], const c32 *__restrict__ tw) {
        constexpr int E = G::E;
        V (&vc)[E1] = col_regs(v);
        fft_cta<G::M1, E1, -1, HALF_COL, TWS, NCOLP>(vc, reinterpret_cast<float *>(colb), nullptr, t1, tw + TWM, j);
        if constexpr (TWID) {
            static_assert(E1 == E, "the four-step twiddle assumes one column layout");
            constexpr int M = 2 * G::MC;
            const c32 b = ldg_c(tw + ((2 * (int64_t)n2 * t1) & (M - 1)));
            const c32 st = ldg_c(tw + ((2 * (int64_t)n2 * T1P) & (M - 1)));
            twiddle_ramp(v, b, st);
        }
        {
            const int z = opaque_zero();   // recompute addresses per order rather than keep them live
#pragma unroll
            for (int q = 0; q < E1; ++q) {
                int dst, slot;
                slot_of_row<G>(t1 + q * T1P + z, dst, slot);
                dsmem_st(dsmem_map(smem_u32(rowb + maddr<G::M2>(n2, slot)), dst), vc[q]);
            }
        }
        cluster_sync_mem();
#pragma unroll
        for (int q = 0; q < E; ++q) {
            if (HALFX && q >= E / 2) {
                v[q] = SE::ld(ET{});
            } else {
                v[q] = SE::ld(rowb[maddr<G::M2>(t2 + q * G::T2, r)]);
            }
        }
        __syncthreads();
        fft_cta<G::M2, E, -1, HALFX, TWS, G::NROW>(v, reinterpret_cast<float *>(rowb), nullptr, t2, tw + TWM, r);
    }

    // Store the row-layout bins so the mirror bins can be read (ends with a CTA barrier).
    __device__ __forceinline__ void publish(const V (&v)[G::E]) {
#pragma unroll
        for (int q = 0; q < G::E; ++q) rowb[maddr<G::M2>(t2 + q * G::T2, r)] = SE::st(v[q]);
        __syncthreads();
    }
    // Published bin (mirror row, column k2m) from this CTA's own buffer.
    __device__ __forceinline__ V mirror_bin(int k2m) const { return SE::ld(rowb[maddr<G::M2>(k2m, rm)]); }
    // Hand a result to the owner of (mirror row, column k2m), after every mirror read.
    __device__ __forceinline__ void set_mirror_bin(int k2m, V val) { rowb[maddr<G::M2>(k2m, rm)] = SE::st(val); }
    // Row-layout register q from the buffer (results handed over by set_mirror_bin).
    __device__ __forceinline__ V own_bin(int q) const { return SE::ld(rowb[maddr<G::M2>(t2 + q * G::T2, r)]); }

    // Row layout (bins) -> column layout (time domain, unscaled inverse).
    // Must follow a CTA barrier after the last read of the published bins.
    __device__ __forceinline__ void inverse(V (&v)[G::E], const c32 *__restrict__ tw) {
        constexpr int E = G::E;
        fft_cta<G::M2, E, +1, false, TWS, G::NROW>(v, reinterpret_cast<float *>(rowb), nullptr, t2, tw + TWM, r);
        if constexpr (TWID) {
            constexpr int M = 2 * G::MC;
            const c32 b = conj(ldg_c(tw + ((2 * (int64_t)t2 * k1) & (M - 1))));
            const c32 st = conj(ldg_c(tw + ((2 * (int64_t)G::T2 * k1) & (M - 1))));
            twiddle_ramp(v, b, st);
        }
        const int z = opaque_zero();
#pragma unroll
        for (int q = 0; q < E; ++q) {
            // zero-padding half (nn >= M2/2 exactly when q >= E/2): never read back,
            // so the last row pass need not produce it
            if (HALFX && q >= E / 2) continue;
            const int nn = t2 + q * G::T2 + z;
            dsmem_st(dsmem_map(smem_u32(colb + maddr<G::M1, NCOLP>(k1, nn % NCOLP)), nn / NCOLP), v[q]);
        }
        cluster_sync_mem();
        V (&vc)[E1] = col_regs(v);
#pragma unroll
        for (int q = 0; q < E1; ++q) vc[q] = SE::ld(colb[maddr<G::M1, NCOLP>(t1 + q * T1P, j)]);
        __syncthreads();
        fft_cta<G::M1, E1, +1, false, TWS, NCOLP>(vc, reinterpret_cast<float *>(colb), nullptr, t1, tw + TWM, j);
    }
};

// Fused order-N forward, one cluster per row (rows visited d-major, b-minor).
template <typename G, typename IO, bool EVEN>
__global__ void __launch_bounds__(G::THREADS, G::MINB) hyena_fwd_1d_cluster(const Fwd1dArgs a) {
    constexpr int MC = G::MC, E = G::E, M1 = G::M1;
    extern __shared__ float smem[];
    ClusterCtx<G, true, false> cx(smem);
    const int64_t ord = (int64_t)blockIdx.x / G::C;     // one cluster per row
    const int64_t d = ord / a.B;
    const int64_t b = ord - d * a.B;
    const int64_t row = b * a.D + d;
    const int64_t L = a.L;
    const c32 wb = ldg_c(a.tw + cx.k1 + M1 * cx.t2);     // W_M^{k1 + M1 t2}

    c32 v[E];
    {
        const IO *vrow = reinterpret_cast<const IO *>(a.v) + act_row_off(a, row);
#pragma unroll
        for (int q = 0; q < E / 2; ++q) v[q] = load_pair_s<IO, EVEN>(vrow, 2 * cx.col_index(q), L, a.es);
#pragma unroll
        for (int q = E / 2; q < E; ++q) v[q] = mk(0.f, 0.f);
    }

    // this order's gates are staged in shared memory (thread-private slots)
    // while the transforms run, instead of occupying registers (contiguous rows
    // of even length; otherwise they are read where they multiply)
    using P = typename io<IO>::pair_t;
    P *gst = reinterpret_cast<P *>(smem + 4 * G::PER_CTA) + threadIdx.x;
    const bool stage = EVEN && a.es == 1;
    for (int n = 0; n < a.order; ++n) {
        const IO *grow = reinterpret_cast<const IO *>(a.gates[n]) + act_row_off(a, row);
        if (stage) {
#pragma unroll
            for (int q = 0; q < E / 2; ++q) {
                const int64_t pos = 2 * cx.col_index(q);
                if (pos < L) cp_async_n<sizeof(P)>(gst + q * G::THREADS, grow + pos);
                else gst[q * G::THREADS] = io<IO>::zero();
            }
            cp_async_commit();
        }
        const float dsk = a.dskip ? __ldg(a.dskip + n * a.hD + d) : 0.f;
        const c32 *Hrow = a.H + ((int64_t)n * a.hD + d) * (MC + 1);

        cx.template forward<true>(v, a.tw);
        cx.publish(v);
        // Spectral step, bins in pairs (k, MC - k): the mirror of register q is
        // register E-1-q of thread (rm, T2-1-t2) (in row 0: of thread (0, T2-t2),
        // and register E-q when t2 = 0), so each thread takes q < E/2 and returns
        // the mirror result conj(Ye - i Yo) to its owner; bin (0, M2/2) is its own mirror.
        constexpr float s = 0.5f / (float)MC;
        const int z0 = opaque_zero();
        auto bin_pair = [&](int q, c32 Zk, c32 &Ye, c32 &Yo) __attribute__((always_inline)) {
            const int k2 = cx.t2 + q * G::T2;
            const int k = cx.k1 + M1 * k2;
            const int km = (MC - k) & (MC - 1);
            const c32 Zm = cx.mirror_bin(km / M1);
            const c32 Ek = mk(0.5f * (Zk.x + Zm.x), 0.5f * (Zk.y - Zm.y));
            const c32 Ok = mk(0.5f * (Zk.y + Zm.y), -0.5f * (Zk.x - Zm.x));
            const c32 w = mul(wb, w2e<E>(q, z0));              // W_M^k, k = k1 + M1 (t2 + q T2)
            const c32 wO = mul(w, Ok);
            const c32 Xk = add(Ek, wO);
            const c32 Xm = conj(sub(Ek, wO));
            c32 Hk = ldg_c(Hrow + k);
            c32 Hm = ldg_c(Hrow + (MC - k));
            Hk.x += dsk;
            Hm.x += dsk;
            const c32 Yk = mul(Xk, Hk), Ym = mul(Xm, Hm);
            Ye = mk(s * (Yk.x + Ym.x), s * (Yk.y - Ym.y));
            const c32 Yd = mk(s * (Yk.x - Ym.x), s * (Yk.y + Ym.y));
            Yo = mul(Yd, conj(w));
        };
        const bool self_half = cx.k1 == 0 && cx.t2 == 0;
        c32 vh = v[E / 2];
        if (self_half) {
            c32 Ye, Yo;
            bin_pair(E / 2, v[E / 2], Ye, Yo);
            vh = mk(Ye.x - Yo.y, Ye.y + Yo.x);
        }
#pragma unroll
        for (int q = 0; q < E / 2; ++q) {
            c32 Ye, Yo;
            bin_pair(q, v[q], Ye, Yo);
            v[q] = mk(Ye.x - Yo.y, Ye.y + Yo.x);              // Ye + i Yo       (bin k)
            v[E / 2 + q] = mk(Ye.x + Yo.y, Yo.x - Ye.y);      // conj(Ye - i Yo) (bin MC - k)
            if ((q & 3) == 3) asm volatile("" ::: "memory");  // bound load hoisting (register pressure)
        }
        __syncthreads();                                // every mirror read done
#pragma unroll
        for (int q = 0; q < E / 2; ++q) {
            const int k = cx.k1 + M1 * (cx.t2 + q * G::T2);
            cx.set_mirror_bin(((MC - k) & (MC - 1)) / M1, v[E / 2 + q]);
        }
        __syncthreads();
#pragma unroll
        for (int q = E / 2; q < E; ++q) v[q] = cx.own_bin(q);
        if (self_half) v[E / 2] = vh;
        __syncthreads();                                // row buffer reads done before the inverse rewrites it
        cx.inverse(v, a.tw);

        // gate (registers q >= E/2 hold positions >= MC, i.e. padding)
        if (stage) cp_async_wait_all();
#pragma unroll
        for (int q = 0; q < E / 2; ++q) {
            const int64_t pos = 2 * cx.col_index(q);
            const c32 gq = stage ? io<IO>::unpack(gst[q * G::THREADS]) : load_pair_s<IO, false>(grow, pos, L, a.es);
            v[q] = mk(pos < L ? gq.x * v[q].x : 0.f, pos + 1 < L ? gq.y * v[q].y : 0.f);
        }
#pragma unroll
        for (int q = E / 2; q < E; ++q) v[q] = mk(0.f, 0.f);
    }

    IO *yrow = reinterpret_cast<IO *>(a.y) + act_row_off(a, row);
#pragma unroll
    for (int q = 0; q < E / 2; ++q) store_pair_s<IO, EVEN>(yrow, 2 * cx.col_index(q), L, a.es, v[q]);
}

// Spectrum of long causal filters (same layout as hyena_spectrum_1d), one
// cluster per filter row. h row o starts at h + o * h_stride and has L taps.
// In place (h == Hout) is allowed: every CTA reads its part of the row before
// the first cluster barrier, and bins are written after it.
template <typename G>
__global__ void __launch_bounds__(G::THREADS, G::MINB)
    hyena_spectrum_1d_cluster(const float *h, int64_t h_stride, int64_t L, c32 *Hout, const c32 *__restrict__ tw) {
    constexpr int MC = G::MC, E = G::E, M1 = G::M1;
    extern __shared__ float smem[];
    ClusterCtx<G, true, false> cx(smem);
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
    cx.template forward<true>(v, tw);                   // contains a cluster barrier after all reads
    cx.publish(v);
    const c32 wb = ldg_c(tw + cx.k1 + M1 * cx.t2);
    c32 *Hrow = Hout + o * (MC + 1);
    const int z0 = opaque_zero();
#pragma unroll
    for (int q = 0; q < E; ++q) {
        const int k = cx.k1 + M1 * (cx.t2 + q * G::T2);
        const int km = (MC - k) & (MC - 1);
        const c32 Zm = cx.mirror_bin(km / M1);
        const c32 Zk = v[q];
        const c32 Ek = mk(0.5f * (Zk.x + Zm.x), 0.5f * (Zk.y - Zm.y));
        const c32 Ok = mk(0.5f * (Zk.y + Zm.y), -0.5f * (Zk.x - Zm.x));
        Hrow[k] = add(Ek, mul(mul(wb, w2e<E>(q, z0)), Ok));
        if (k == 0) Hrow[MC] = mk(Ek.x - Ok.x, 0.f);  // Nyquist bin: E_0 - O_0, real
    }
}

}  // namespace hyena
