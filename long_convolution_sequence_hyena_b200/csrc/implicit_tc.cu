// Implicit filter network on the 5th-generation tensor cores (tcgen05.mma,
// accumulators in tensor memory), for networks of width 64.
//
// The network is the one of kernels_implicit.cuh ("Hyena — Long Convolutions
// Math", "Implicit filters: an MLP over positions" and "The decay window";
// "How HyenaND works", "1. An implicit filter"): positional features, two sine
// layers of width 64, a linear head to N*D outputs, the window. Two of its
// three layers are dense contractions over every position p: the second sine
// layer's pre-activation a1[p] W2^T (64 x 64) and the head a2[p] W3^T
// (64 x N*D, almost all of the work); both run on the tensor cores. The
// features and the first layer (1 + 2K or 2-3 inputs) stay on the CUDA cores.
//
// Precision: the filters must match an fp64 evaluation to fp32 accuracy, which
// one TF32 product (10-bit mantissa) cannot. Each operand is split as
// x = hi + lo with hi = x rounded to TF32 and lo = x - hi (exact in fp32), and
// each contraction accumulates hi*hi + hi*lo + lo*hi in fp32 (the dropped
// lo*lo term and the TF32 rounding of lo are about 2^-21 of the product).
//
// One CTA (256 threads, 8 warps) per tile of 128 positions and one slice of
// the outputs, two CTAs per SM (about 100 KB of shared memory each):
//   1. thread (p, part) forms the features of position p and units
//      [16 part, 16 part + 16) of the first sine layer, and writes them, split,
//      into the A tile (shared memory, the tensor core's K-major layout
//      without swizzle: 8 x 16-byte core matrices); W2, split, is the B tile;
//   2. one thread issues the 24 MMAs of the second layer (M 128, N 64, K 8:
//      eight K steps, three products) into tensor memory; the warps read the
//      pre-activations back (tcgen05.ld), add the bias, take the sine and
//      write the split result over the A tile;
//   3. per slice of 64 outputs: the CTA converts W3's rows into the B tile;
//      one thread issues 24 MMAs (N 64) into one of two accumulators; while
//      they run, the warps read the previous slice's accumulator, add the bias,
//      apply the window (constants per output staged in shared memory) and
//      store.
// Every wait on the mbarrier is bounded: on a timeout the kernel records an
// error in *err, skips the remaining MMAs and still frees its tensor memory.
#include <cuda_runtime.h>

#include <cstddef>

#include "launch.h"

namespace hyena {

namespace {

constexpr int TP = 128;            // positions per tile (the MMA's M)
constexpr int NT = 64;             // outputs per slice (the MMA's N)
constexpr int KW = 64;             // network width (the MMA's K over 8 steps)
constexpr int THREADS = 256;
constexpr int PARTS = THREADS / TP;      // threads per position (each takes KW / PARTS second-layer units)
constexpr int LBO = 16 * 128;      // bytes between K-adjacent core matrices (16 row groups of 128 B)
constexpr int SBO = 128;           // bytes between 8-row groups
constexpr int TMEM_COLS = 256;         // two head accumulators of 64 columns, then the second layer's 64
constexpr int L2COL = 2 * NT;          // first tensor-memory column of the second layer's accumulator
constexpr int SLICE_OUT = 512;         // outputs per CTA (grid.y covers the rest)

struct alignas(128) TcSmem {
    float a[2][TP * KW];           // A tile: hi, lo
    float b[2][KW * KW];           // B tile: hi, lo (W2, then slices of W3: NT <= KW rows)
    float b1[KW], b2[KW];
    float2 oc[NT];                 // per output of the slice: window exponent scale (log2 units), bias
    unsigned long long mbar;
    uint32_t tmem_base;
    alignas(16) float w1t[1][KW];  // first layer weights, transposed: [feature][unit] (fin rows follow; read as float4)
};
static_assert(offsetof(TcSmem, w1t) % 16 == 0 && offsetof(TcSmem, a) % 16 == 0 && offsetof(TcSmem, b) % 16 == 0,
              "16-byte accesses to the tiles and the first-layer weights");
static_assert(NT <= KW, "the B tile holds W2 and the head slices");

__device__ __forceinline__ uint32_t saddr(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

// x rounded to TF32 (round to nearest, ties away), as an fp32 bit pattern whose low 13 bits are zero
__device__ __forceinline__ float tf32_hi(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return __uint_as_float(r);
}

// Byte offset of element (row, k) in a K-major tile without swizzle: core matrices
// of 8 rows x 4 elements (16 bytes per row), 8-row groups SBO apart, K chunks LBO apart.
__device__ __forceinline__ int core_off(int row, int kc) { return kc * LBO + (row >> 3) * SBO + (row & 7) * 16; }

// Shared-memory matrix descriptor (K-major, no swizzle): start address, leading
// byte offset (between K-adjacent core matrices), stride byte offset (between
// 8-row groups), descriptor version 1, layout type 0.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, int lbo = LBO) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((SBO >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;
    return d;
}

// Instruction descriptor: fp32 accumulator, TF32 A and B, both K-major, M = TP, N as given.
constexpr uint32_t idesc_n(int n) {
    return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(TP >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}

// The 24 MMAs of one contraction over K = 64: eight K steps (two core
// matrices each), products hi*hi, hi*lo, lo*hi. Issued by one thread.
__device__ __forceinline__ void mma_split_k64(uint32_t d, uint32_t ah, uint32_t al, uint32_t bh, uint32_t bl,
                                              int lbo_b, uint32_t idesc) {
#pragma unroll
    for (int ks = 0; ks < KW / 8; ++ks) {
        const uint32_t ka = (uint32_t)(2 * ks * LBO), kb = (uint32_t)(2 * ks * lbo_b);
        mma_tf32(d, smem_desc(ah + ka), smem_desc(bh + kb, lbo_b), idesc, ks > 0);
        mma_tf32(d, smem_desc(ah + ka), smem_desc(bl + kb, lbo_b), idesc, 1);
        mma_tf32(d, smem_desc(al + ka), smem_desc(bh + kb, lbo_b), idesc, 1);
    }
}

__device__ __forceinline__ void mma_commit(unsigned long long *mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(saddr(mbar))
                 : "memory");
}

// Bounded wait for the mbarrier's phase `parity` to complete; false on timeout.
__device__ __forceinline__ bool mbar_wait(unsigned long long *mbar, uint32_t parity) {
    for (int i = 0; i < (1 << 22); ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(saddr(mbar)), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

// sin x for the sine layers: Cody and Waite's reduction x = 2 pi k + r, with
// 2 pi split into 6.28125 (8 significant bits, so k * 6.28125 is exact for
// the k that occur) and 2 pi - 6.28125, then the hardware sine __sinf on
// r in [-pi, pi], where its absolute error is below 2^-21.4. Arguments of
// magnitude 8192 and more, far outside what the layers produce, go to sinf.
__device__ __noinline__ float sin_large(float x) { return sinf(x); }   // kept out of the hot code
__device__ __forceinline__ float sin_layer(float x) {
    if (fabsf(x) >= 8192.f) return sin_large(x);
    const float k = rintf(x * 0.159154943091895336f);   // x / (2 pi)
    float r = fmaf(-k, 6.28125f, x);
    r = fmaf(-k, 1.93530717958647692e-3f, r);
    return __sinf(r);
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Rows [o0, o0 + n) of a row-major [*][64] fp32 matrix as a split K-major B tile.
__device__ __forceinline__ void load_b_tile(TcSmem &S, const float *__restrict__ Wm, int64_t o0, int n, int64_t oend,
                                            int tid) {
    unsigned char *bhi = reinterpret_cast<unsigned char *>(S.b[0]);
    unsigned char *blo = reinterpret_cast<unsigned char *>(S.b[1]);
    for (int i = tid; i < n * (KW / 4); i += THREADS) {
        const int o = i % n, kc = i / n;          // consecutive threads: consecutive rows of one K chunk
        const int64_t og = o0 + o;
        float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
        if (og < oend) w = __ldg(reinterpret_cast<const float4 *>(Wm + og * KW) + kc);
        const float4 h4 = make_float4(tf32_hi(w.x), tf32_hi(w.y), tf32_hi(w.z), tf32_hi(w.w));
        const int off = kc * (n / 8) * SBO + (o >> 3) * SBO + (o & 7) * 16;   // K chunks n/8 row groups apart
        *reinterpret_cast<float4 *>(bhi + off) = h4;
        *reinterpret_cast<float4 *>(blo + off) = make_float4(w.x - h4.x, w.y - h4.y, w.z - h4.z, w.w - h4.w);
    }
}

// The head's B tile in two steps, so that the global loads of the next slice
// overlap the current one: fetch_w3 reads rows [o0, o0 + NT) of W3 (zero past
// oend) into registers, store_w3 writes them split into the B tile.
constexpr int B_PER_THREAD = NT * (KW / 4) / THREADS;   // float4 per thread
__device__ __forceinline__ void fetch_w3(const float *__restrict__ Wm, int64_t o0, int64_t oend, int tid,
                                         float4 (&w)[B_PER_THREAD]) {
#pragma unroll
    for (int j = 0; j < B_PER_THREAD; ++j) {
        const int i = tid + j * THREADS, o = i % NT, kc = i / NT;
        const int64_t og = o0 + o;
        w[j] = og < oend ? __ldg(reinterpret_cast<const float4 *>(Wm + og * KW) + kc) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
}
__device__ __forceinline__ void store_w3(TcSmem &S, const float4 (&w)[B_PER_THREAD], int tid) {
    unsigned char *bhi = reinterpret_cast<unsigned char *>(S.b[0]);
    unsigned char *blo = reinterpret_cast<unsigned char *>(S.b[1]);
#pragma unroll
    for (int j = 0; j < B_PER_THREAD; ++j) {
        const int i = tid + j * THREADS, o = i % NT, kc = i / NT;
        const float4 h4 = make_float4(tf32_hi(w[j].x), tf32_hi(w[j].y), tf32_hi(w[j].z), tf32_hi(w[j].w));
        const int off = kc * (NT / 8) * SBO + (o >> 3) * SBO + (o & 7) * 16;
        *reinterpret_cast<float4 *>(bhi + off) = h4;
        *reinterpret_cast<float4 *>(blo + off) =
            make_float4(w[j].x - h4.x, w[j].y - h4.y, w[j].z - h4.z, w[j].w - h4.w);
    }
}

// 32 consecutive accumulator columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&r)[32]) {
    uint32_t u[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
          "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15]),
          "=r"(u[16]), "=r"(u[17]), "=r"(u[18]), "=r"(u[19]), "=r"(u[20]), "=r"(u[21]), "=r"(u[22]), "=r"(u[23]),
          "=r"(u[24]), "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]), "=r"(u[30]), "=r"(u[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = __uint_as_float(u[i]);
}

// NDIM: the grid's dimension (1, 2 or 3), fixed per instance so that each holds
// only its own feature and window code.
template <int NDIM>
__global__ void __launch_bounds__(THREADS, 2) hyena_implicit_tc_kernel(const ImplicitArgs a, int *err) {
    extern __shared__ float4 tc_smem4[];
    TcSmem &S = *reinterpret_cast<TcSmem *>(tc_smem4);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int fin = NDIM == 1 ? 1 + 2 * a.p.num_freqs : NDIM;
    const int64_t p0 = (int64_t)blockIdx.x * TP;

    // first-layer weights and biases, W2 as the B tile, the barrier and tensor memory
    for (int i = tid; i < KW * fin; i += THREADS) S.w1t[0][(i % fin) * KW + i / fin] = __ldg(a.p.W1 + i);
    if (tid < KW) {
        S.b1[tid] = __ldg(a.p.b1 + tid);
        S.b2[tid] = __ldg(a.p.b2 + tid);
    }
    load_b_tile(S, a.p.W2, 0, KW, KW, tid);
    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(saddr(&S.mbar)));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(saddr(&S.tmem_base)),
                     "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    unsigned char *ahi = reinterpret_cast<unsigned char *>(S.a[0]);
    unsigned char *alo = reinterpret_cast<unsigned char *>(S.a[1]);
    const uint32_t sah = saddr(S.a[0]), sal = saddr(S.a[1]), sbh = saddr(S.b[0]), sbl = saddr(S.b[1]);
    bool ok = true;
    uint32_t phase = 0;
    auto wait_mma = [&]() {
        if (ok && !mbar_wait(&S.mbar, phase)) {
            ok = false;
            atomicOr(err, HYENA_DEVERR_WAIT_TIMEOUT);
        }
        phase ^= 1;
        tc_fence_after();
    };

    // 1. features and first-layer units [16 part, 16 part + 16) of position p, split into the A tile
    {
        const int p = tid & (TP - 1), part = tid / TP;
        const int64_t pos = p0 + p;
        const bool in = pos < a.npos;
        float a1[KW / PARTS];
#pragma unroll
        for (int j = 0; j < KW / PARTS; ++j) a1[j] = 0.f;
        // adds feature f (value fv) times its first-layer weights to this thread's units
        auto add_feature = [&](int f, float fv) __attribute__((always_inline)) {
            const float4 *wrow = reinterpret_cast<const float4 *>(S.w1t[0] + f * KW + (KW / PARTS) * part);
#pragma unroll
            for (int j4 = 0; j4 < KW / PARTS / 4; ++j4) {
                const float4 w = wrow[j4];
                a1[4 * j4] = fmaf(w.x, fv, a1[4 * j4]);
                a1[4 * j4 + 1] = fmaf(w.y, fv, a1[4 * j4 + 1]);
                a1[4 * j4 + 2] = fmaf(w.z, fv, a1[4 * j4 + 2]);
                a1[4 * j4 + 3] = fmaf(w.w, fv, a1[4 * j4 + 3]);
            }
        };
        if constexpr (NDIM == 1) {
            // [t/L, cos(2 pi k t/L), sin(2 pi k t/L) for k = 1..K]: the angle's turns
            // (k t mod L) / L advance by t per frequency, kept exact in integers
            // (t < L <= 2^19, so k t fits in 32 bits)
            const int Li = (int)a.L, t = in ? (int)pos : 0;
            add_feature(0, in ? __fdiv_rn((float)t, (float)Li) : 0.f);
            int rk = 0;
#pragma unroll 1
            for (int k = 1; 2 * k < fin; ++k) {
                rk += t;
                if (rk >= Li) rk -= Li;
                float sv = 0.f, cv = 0.f;
                if (in) sincospif(__fdiv_rn((float)(2 * rk), (float)Li), &sv, &cv);
                add_feature(2 * k - 1, cv);
                add_feature(2 * k, sv);
            }
        } else {
#pragma unroll 1
            for (int f = 0; f < fin; ++f) {
                float fv = 0.f;
                if (in) {   // offsets on grids of at most 2^21 points: 32-bit index arithmetic
                    const int W2 = 2 * (int)a.W, Hi = (int)a.H, Wi = (int)a.W, pi = (int)pos;
                    if constexpr (NDIM == 2) {
                        const int iy = pi / W2, ix = pi - iy * W2;
                        fv = f == 0 ? __fdiv_rn((float)(iy - Hi), (float)Hi) : __fdiv_rn((float)(ix - Wi), (float)Wi);
                    } else {   // 3D: (oz / Dz, oy / H, ox / W) on the offset grid [2Dz][2H][2W]
                        const int hw = 2 * Hi * W2, Dzi = (int)a.Dz;
                        const int iz = pi / hw, rem = pi - iz * hw;
                        const int iy = rem / W2, ix = rem - iy * W2;
                        fv = f == 0 ? __fdiv_rn((float)(iz - Dzi), (float)Dzi)
                                    : (f == 1 ? __fdiv_rn((float)(iy - Hi), (float)Hi) : __fdiv_rn((float)(ix - Wi), (float)Wi));
                    }
                }
                add_feature(f, fv);
            }
        }
#pragma unroll
        for (int c = 0; c < KW / PARTS / 4; ++c) {   // 4 units per 16-byte core-matrix row
            const int kc = (KW / PARTS / 4) * part + c;
            float hi[4], lo[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float v = in ? sin_layer(a.p.omega0 * (a1[4 * c + u] + S.b1[4 * kc + u])) : 0.f;
                hi[u] = tf32_hi(v);
                lo[u] = v - hi[u];
            }
            const int off = core_off(p, kc);
            *reinterpret_cast<float4 *>(ahi + off) = make_float4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<float4 *>(alo + off) = make_float4(lo[0], lo[1], lo[2], lo[3]);
        }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // the tensor core sees the tiles
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // 2. second layer on the tensor cores: pre-activations of 64 units -> tensor memory
    if (tid == 0) {
        mma_split_k64(tmem + L2COL, sah, sal, sbh, sbl, (KW / 8) * SBO, idesc_n(KW));
        mma_commit(&S.mbar);
    }
    wait_mma();
    {
        constexpr int UPW = KW / (THREADS / 128);   // units per warp: 32
        const int q = warp & 3, cq = warp >> 2;      // lane quarter (positions), unit group
        const int p = 32 * q + lane;
        float r[UPW];
        tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(L2COL + UPW * cq), r);
        const bool in = p0 + p < a.npos;
#pragma unroll
        for (int c = 0; c < UPW / 4; ++c) {
            const int kc = (UPW / 4) * cq + c;
            float hi[4], lo[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float v = in ? sin_layer(a.p.omega_hidden * (r[4 * c + u] + S.b2[4 * kc + u])) : 0.f;
                hi[u] = tf32_hi(v);
                lo[u] = v - hi[u];
            }
            const int off = core_off(p, kc);
            *reinterpret_cast<float4 *>(ahi + off) = make_float4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<float4 *>(alo + off) = make_float4(lo[0], lo[1], lo[2], lo[3]);
        }
    }

    // 3. head slices
    const int64_t o_begin = (int64_t)blockIdx.y * SLICE_OUT;
    const int64_t o_end = o_begin + SLICE_OUT < a.nout ? o_begin + SLICE_OUT : a.nout;
    const int nslices = (int)((o_end - o_begin + NT - 1) / NT);
    const int q = warp & 3, cq = warp >> 2;            // TMEM lane quarter, column quarter
    const int prow = 32 * q + lane;                    // this thread's position in the epilogue
    const int64_t ppos = p0 + prow;
    float we = 0.f;                                    // window exponent argument: t (1D) or |p|^2 (2D, 3D)
    int64_t poff = ppos;
    if constexpr (NDIM == 1) {
        we = (float)ppos;
    } else if (NDIM == 2) {
        if (ppos < a.npos) {
        const int W2 = 2 * (int)a.W, Hi = (int)a.H, Wi = (int)a.W, pi = (int)ppos;
        const int iy = pi / W2, ix = pi - iy * W2;
        const float py = __fdiv_rn((float)(iy - Hi), (float)Hi), px = __fdiv_rn((float)(ix - Wi), (float)Wi);
        we = py * py + px * px;
        poff = (int64_t)iy * a.out_row_stride + ix;
        }
    } else if (ppos < a.npos) {   // 3D: output [2Dz][2H][2W] contiguous per channel
        const int W2 = 2 * (int)a.W, Hi = (int)a.H, Wi = (int)a.W, Dzi = (int)a.Dz, pi = (int)ppos;
        const int hw = 2 * Hi * W2;
        const int iz = pi / hw, rem = pi - iz * hw;
        const int iy = rem / W2, ix = rem - iy * W2;
        const float pz = __fdiv_rn((float)(iz - Dzi), (float)Dzi);
        const float py = __fdiv_rn((float)(iy - Hi), (float)Hi), px = __fdiv_rn((float)(ix - Wi), (float)Wi);
        we = pz * pz + py * py + px * px;
    }
    static_assert(NT / (THREADS / 128) == 32, "each warp reads 32 accumulator columns");
    auto epilogue = [&](int s) {
        float r[32];
        tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)((s & 1) * NT + 32 * cq), r);
        if (ppos >= a.npos) return;
        const int64_t ob = o_begin + (int64_t)s * NT + 32 * cq;
        float *dst = a.out + ob * a.out_stride + poff;
#pragma unroll 8
        for (int c = 0; c < 32; ++c) {
            if (ob + c >= o_end) break;
            const float2 k = S.oc[32 * cq + c];   // (window exponent scale in log2 units, bias)
            *dst = exp2f(k.x * we) * (r[c] + k.y);
            dst += a.out_stride;
        }
    };
    // The B tile is free: the second layer's MMAs have completed. Slice s's W3
    // rows are fetched while slice s - 1's MMAs and slice s - 2's epilogue run,
    // and written into the B tile once slice s - 1's MMAs are done.
    float4 wb[B_PER_THREAD];
    if (nslices > 0) {
        fetch_w3(a.p.W3, o_begin, o_end, tid, wb);
        store_w3(S, wb, tid);
    }
#pragma unroll 1
    for (int s = 0; s < nslices; ++s) {
        // slice s's window scales and biases; the epilogue of slice s - 1 still
        // reads S.oc: they are written after the barrier below
        const int64_t os = o_begin + (int64_t)s * NT;
        float2 oc_new = make_float2(0.f, 0.f);
        if (tid < NT && os + tid < o_end) {
            const float wp = __ldg(a.p.window + os + tid);
            // exp(-alpha t) (1D) or exp(-|p|^2 / (2 sigma^2)) (2D, 3D), as 2^(scale * arg)
            const float esc = NDIM == 1 ? -wp : -1.f / (2.f * wp * wp);
            oc_new = make_float2(esc * 1.4426950408889634f, __ldg(a.p.b3 + os + tid));
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0 && ok) {
            mma_split_k64(tmem + (uint32_t)((s & 1) * NT), sah, sal, sbh, sbl, (NT / 8) * SBO, idesc_n(NT));
            mma_commit(&S.mbar);
        }
        if (s + 1 < nslices) fetch_w3(a.p.W3, os + NT, o_end, tid, wb);   // in flight during the epilogue
        if (s > 0) epilogue(s - 1);   // overlaps the MMAs of slice s
        __syncthreads();              // every read of S.oc for slice s - 1 done
        if (tid < NT) S.oc[tid] = oc_new;
        wait_mma();                   // slice s complete (or abandoned): the B tile is free
        if (s + 1 < nslices) store_w3(S, wb, tid);
        __syncthreads();              // S.oc updated (the next iteration fences the B tile)
    }
    if (nslices > 0 && ok) epilogue(nslices - 1);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
}

}  // namespace

bool implicit_tc_supported(const ImplicitArgs &a) { return a.p.width == KW; }

size_t implicit_tc_smem_bytes(int fin) { return sizeof(TcSmem) + (size_t)(fin - 1) * KW * sizeof(float) + 128; }

cudaError_t launch_implicit_tc(const ImplicitArgs &a, int *err, cudaStream_t st) {
    const int sm = (int)implicit_tc_smem_bytes(a.ndim == 1 ? 1 + 2 * a.p.num_freqs : a.ndim);
    auto kern = a.ndim == 1 ? hyena_implicit_tc_kernel<1> : (a.ndim == 2 ? hyena_implicit_tc_kernel<2>
                                                                          : hyena_implicit_tc_kernel<3>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((a.npos + TP - 1) / TP), (unsigned)((a.nout + SLICE_OUT - 1) / SLICE_OUT));
    kern<<<grid, THREADS, sm, st>>>(a, err);
    return launched();
}

}  // namespace hyena
