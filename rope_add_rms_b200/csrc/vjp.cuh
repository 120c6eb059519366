// vjp.cuh -- gradients of rms_norm and layer_norm (vector-Jacobian products).
//
// Definitions: docs.rs nuvec-core 0.5.0, Enum FastOp, variants RmsNormVjp (gradients of
// rms_norm with respect to x and w) and LayerNormVjp (with respect to x, w and b).
//   RmsNorm:   r = 1/sqrt(mean(x^2) + eps), y = x r w
//              dx_j = r w_j g_j - x_j r^3 (sum_k g_k w_k x_k) / D,  dw_j = sum_rows g_j x_j r
//   LayerNorm: xh = (x - mean) r, a = w g
//              dx_j = r (a_j - mean(a) - xh_j mean(a xh)),  dw_j = sum_rows g_j xh_j,
//              db_j = sum_rows g_j
//
// dx is row-local.  dw and db are column sums over all rows: kernel 1 runs one wave of
// `parts` CTAs (as many as are resident on the GPU at once), CTA p walking rows p,
// p + parts, ...  Each thread owns VPT 16-byte vectors of every row it visits and keeps
// the float32 partial column sums of those elements in registers; with VPT = 1 it loads
// the next row's x and g before reducing the current one, so two rows per thread are in
// flight.  At the end each CTA writes its partials to the caller's workspace [parts, D]
// (one slice per sum), and kernel 2 adds them per column in double, in a fixed order
// (deterministic), rounding once to the I/O type.
//
// Precision: the gradients are differences of terms that can cancel, and their bar is an
// absolute error of 2^-16 times the sum of the terms' magnitudes.  Everything here is
// float32 with rounding errors a few float32 ulps of those magnitudes:
//   RmsNormVjp:   r and v = r^2 sum(g w x) / D, then dx = r (g w - x v).
//   LayerNormVjp: two passes over the registers.  Pass 1 sums x and a, giving a first mean
//   m1 (off by up to ~2^-20 |mean|) and mean(a).  Pass 2 sums c' = x - m1, c'^2 and a c';
//   d = sum c' / D corrects the mean to m1 + d, exact to rounding of the spread rather
//   than of |mean|, so rows whose mean dwarfs their spread keep full accuracy:
//   c = c' - d,  var = sum c'^2 / D - d^2,  sum a c = sum a c' - d sum a.
#pragma once

#include "common.cuh"
#include "rms.cuh"

namespace nvn {

struct VjpArgs {
    const void* x;
    const void* w;   // NULL: w = 1, no dw
    const void* g;   // upstream gradient [rows, D]
    void* dx;
    float* part;     // workspace: [nsum][parts][D] float32 partials (NULL: no column sums)
    int64_t rows;
    int D;
    int nvec;
    int parts;       // CTAs of kernel 1 (= partial rows per sum)
    int want_dw;
    int want_db;
    float eps;
    int G;           // vjp_narrow_kernel: threads of a row group (a power of two <= 32)
};

// CTA size bound of kernel 1 by vectors per thread: one thread per vector up to 1024
// vectors a row (64 registers a thread); 2 or 4 vectors a thread at up to 512 threads
// (128 registers).
constexpr int vjp_max_threads(int vpt) { return vpt == 1 ? 1024 : 512; }

// Warp sums of N (2 or 3) values at once: the first levels of the butterfly halve the set
// of sums each lane carries (a lane keeps one half and sends the other to its partner),
// so N sums cost 5 (N = 2) or 6 (N = 3) shuffles rather than 5 N.  On return lane l holds
// the warp total of sum l / kLanesPerSum<N> (N = 3: lanes 24-31 hold a zero pad sum);
// lanes holding the same sum hold bit-identical values.
template <int N>
constexpr int kLanesPerSum = N == 2 ? 16 : 8;

template <int N>
__device__ __forceinline__ float warp_sums(const float (&v)[N]) {
    static_assert(N >= 2 && N <= 4, "two to four sums");
    const int lane = threadIdx.x & 31;
    float keep;
    if constexpr (N == 2) {
        const bool hi = lane & 16;
        keep = hi ? v[1] : v[0];
        keep += __shfl_xor_sync(0xFFFFFFFFu, hi ? v[0] : v[1], 16);
    } else {
        // four slots (the fourth a zero pad when N = 3)
        const float v3 = N == 4 ? v[N - 1] : 0.f;
        const bool b4 = lane & 16, b3 = lane & 8;
        float k0 = b4 ? v[2] : v[0], k1 = b4 ? v3 : v[1];
        k0 += __shfl_xor_sync(0xFFFFFFFFu, b4 ? v[0] : v[2], 16);
        k1 += __shfl_xor_sync(0xFFFFFFFFu, b4 ? v[1] : v3, 16);
        keep = b3 ? k1 : k0;
        keep += __shfl_xor_sync(0xFFFFFFFFu, b3 ? k0 : k1, 8);
    }
#pragma unroll
    for (int off = kLanesPerSum<N> / 2; off >= 1; off >>= 1)
        keep += __shfl_xor_sync(0xFFFFFFFFu, keep, off);
    return keep;
}

template <int N>
struct CtaSums {
    float part[N][32];  // per-warp partials
    float tot[N];
};

// Sum of N floats across the CTA; every thread receives the totals.  Each warp reduces
// its own values, warp 0 reduces the warps' partials the same way and publishes the
// totals: two barriers, a fixed order of additions (the same totals in every thread and
// on every run).  One CtaSums may be reused by consecutive calls.
template <int N>
__device__ __forceinline__ void cta_sum(float (&v)[N], CtaSums<N>& b) {
    constexpr int L = kLanesPerSum<N>;
    const int lane = threadIdx.x & 31;
    const int wid = threadIdx.x >> 5;
    const bool writer = (lane & (L - 1)) == 0 && lane / L < N;
    const float s = warp_sums<N>(v);
    if (writer) b.part[lane / L][wid] = s;
    __syncthreads();
    if (wid == 0) {
        const bool in = lane < (int)(blockDim.x >> 5);
        float p[N];
#pragma unroll
        for (int i = 0; i < N; ++i) p[i] = in ? b.part[i][lane] : 0.f;
        const float t = warp_sums<N>(p);
        if (writer) b.tot[lane / L] = t;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = b.tot[i];
}

// This thread's x and g vectors of `row` (zeros past the row's end or past the last row).
template <typename T, int VPT>
__device__ __forceinline__ void load_xg(const VjpArgs& a, int64_t row, V16 (&xv)[VPT],
                                        V16 (&gv)[VPT]) {
    const bool live = row < a.rows;
    const size_t roff = (size_t)row * (size_t)a.nvec * 16;
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
        const int v = threadIdx.x + k * blockDim.x;
        const bool in = live && v < a.nvec;
        xv[k] = in ? ld_stream(static_cast<const char*>(a.x) + roff + (size_t)v * 16)
                   : zeros_vec<T>();
        gv[k] = in ? ld_stream(static_cast<const char*>(a.g) + roff + (size_t)v * 16)
                   : zeros_vec<T>();
    }
}

template <typename T>
__device__ __forceinline__ V16 load_w(const VjpArgs& a, int k) {
    const int v = threadIdx.x + k * blockDim.x;
    return (a.w && v < a.nvec) ? ld_param(static_cast<const char*>(a.w) + (size_t)v * 16)
                               : ones_vec<T>();
}

// Rows of kernel 1: CTA p takes rows p, p + parts, ...  With VPT <= 2 two register sets
// alternate, so row i + 1's loads are in flight while row i is reduced and written (and no
// register copy waits on them); with VPT = 4 each row is loaded where it is used.
template <int VPT, typename Row>
__device__ __forceinline__ void walk_rows(const VjpArgs& a, Row&& row_step) {
    using T = typename Row::T;
    if constexpr (VPT <= 2) {
        V16 xa[VPT], ga[VPT], xb[VPT], gb[VPT];
        load_xg<T, VPT>(a, blockIdx.x, xa, ga);
        const int64_t step = a.parts;
        for (int64_t row = blockIdx.x; row < a.rows; row += 2 * step) {
            load_xg<T, VPT>(a, row + step, xb, gb);
            row_step(row, xa, ga);
            if (row + step >= a.rows) break;
            load_xg<T, VPT>(a, row + 2 * step, xa, ga);
            row_step(row + step, xb, gb);
        }
    } else {
        for (int64_t row = blockIdx.x; row < a.rows; row += a.parts) {
            V16 xv[VPT], gv[VPT];
            load_xg<T, VPT>(a, row, xv, gv);
            row_step(row, xv, gv);
        }
    }
}

// The element work runs on float32 pairs (packed FFMA2 / FADD2 / FMUL2, IEEE per lane):
// each of a thread's row sums is two interleaved chains, added at the end.
__device__ __forceinline__ float2 splat2(float v) { return make_float2(v, v); }

// Column partial sums of a thread's elements, NSUM sums (dw, db) of VPT * NP float pairs:
// in registers, or for VPT = 4 -- where registers would spill -- in the thread's own slots
// of dynamic shared memory, [NSUM][VPT * NP][blockDim.x] (consecutive threads, consecutive
// slots).  Measured on layer_norm_vjp bf16 D = 16384: 147 us against 170 us in registers;
// slower for VPT <= 2, which keep registers.
template <int VPT, int NP, int NSUM>
struct ColAcc {
    static constexpr bool kShared = VPT >= 4;
    float2 r[kShared ? 1 : NSUM][kShared ? 1 : VPT * NP];
    float2* s;

    __device__ __forceinline__ void init(float2* smem) {
        s = smem;
#pragma unroll
        for (int j = 0; j < NSUM; ++j)
#pragma unroll
            for (int i = 0; i < VPT * NP; ++i) at(j, i) = splat2(0.f);
    }
    __device__ __forceinline__ float2& at(int j, int i) {
        if constexpr (kShared)
            return s[(j * VPT * NP + i) * blockDim.x + threadIdx.x];
        else
            return r[j][i];
    }
    // dynamic shared memory bytes for a CTA of `threads`
    __host__ __device__ static constexpr size_t smem_bytes(int threads) {
        return kShared ? (size_t)NSUM * VPT * NP * threads * sizeof(float2) : 0;
    }
};

// ---- RmsNormVjp, kernel 1 ---------------------------------------------------------------
template <typename TT, int VPT>
struct RmsVjpRow {
    using T = TT;
    using E = Elem<T>;
    static constexpr int VEC = E::kVec;
    static constexpr int NP = VEC / 2;  // float pairs per vector
    const VjpArgs& a;
    const float2 (&wf)[VPT][NP];
    ColAcc<VPT, NP, 1>& acc;
    CtaSums<2>& red;
    float invD;

    __device__ __forceinline__ void operator()(int64_t row, const V16 (&xv)[VPT],
                                               const V16 (&gv)[VPT]) const {
        // sum x^2 (the scale) and sum g w x (the projection); bfloat16 pairs consumed packed
        // (x x and g x exact products, (g x) w exact too: 8 + 8 + 8 significant bits)
        float2 s0 = splat2(0.f), s1 = splat2(0.f);
#pragma unroll
        for (int k = 0; k < VPT; ++k)
#pragma unroll
            for (int e = 0; e < VEC; e += 2) {
                if constexpr (sizeof(T) == 2) {
                    s0 = bf16x2_mac(xv[k].u[e / 2], xv[k].u[e / 2], s0);
                    s1 = fma2(bf16x2_mac(gv[k].u[e / 2], xv[k].u[e / 2], splat2(0.f)),
                              wf[k][e / 2], s1);
                } else {
                    const float2 x2 = E::get2(xv[k], e);
                    const float2 u2 = mul2(E::get2(gv[k], e), wf[k][e / 2]);
                    s0 = fma2(x2, x2, s0);
                    s1 = fma2(u2, x2, s1);
                }
            }
        float s[2] = {__fadd_rn(s0.x, s0.y), __fadd_rn(s1.x, s1.y)};
        cta_sum<2>(s, red);
        const float r = rsqrtf(__fmaf_rn(s[0], invD, a.eps));
        const float vr = __fmul_rn(__fmul_rn(r, r), __fmul_rn(s[1], invD));
        const float2 r2 = splat2(r), nv2 = splat2(-vr);
        const size_t roff = (size_t)row * (size_t)a.nvec * 16;
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = threadIdx.x + k * blockDim.x;
            if (v < a.nvec) {
                V16 o;
#pragma unroll
                for (int e = 0; e < VEC; e += 2) {
                    const float2 x2 = E::get2(xv[k], e);
                    const float2 g2 = E::get2(gv[k], e);
                    const float2 u2 = mul2(g2, wf[k][e / 2]);
                    E::put2(o, e, mul2(r2, fma2(x2, nv2, u2)));        // r (g w - x v)
                    float2& ac = acc.at(0, k * NP + e / 2);
                    ac = fma2(mul2(g2, x2), r2, ac);
                }
                st_stream(static_cast<char*>(a.dx) + roff + (size_t)v * 16, o);
            }
        }
    }
};

template <typename T, int VPT>
__device__ __forceinline__ void load_wf(const VjpArgs& a, float2 (&wf)[VPT][Elem<T>::kVec / 2]) {
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
        const V16 w = load_w<T>(a, k);
#pragma unroll
        for (int e = 0; e < Elem<T>::kVec; e += 2) wf[k][e / 2] = Elem<T>::get2(w, e);
    }
}

template <typename T, int VPT>
__global__ void __launch_bounds__(vjp_max_threads(VPT)) rms_vjp_kernel(const VjpArgs a) {
    pdl_wait();
    pdl_release();
    constexpr int NP = Elem<T>::kVec / 2;
    __shared__ CtaSums<2> red;
    extern __shared__ float2 acc_smem[];
    float2 wf[VPT][NP];
    load_wf<T, VPT>(a, wf);
    ColAcc<VPT, NP, 1> acc;
    acc.init(acc_smem);
    walk_rows<VPT>(a, RmsVjpRow<T, VPT>{a, wf, acc, red, 1.f / (float)a.D});
    if (a.want_dw) {
        float* out = a.part + (size_t)blockIdx.x * a.D;
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = threadIdx.x + k * blockDim.x;
            if (v < a.nvec)
#pragma unroll
                for (int i = 0; i < NP; ++i)
                    reinterpret_cast<float2*>(out)[v * NP + i] = acc.at(0, k * NP + i);
        }
    }
}

// ---- RmsNormVjp, kernel 1, two rows per reduction -------------------------------------------
// The same arithmetic as RmsVjpRow, but each CTA reduces the sums of two rows at once (four
// values in one butterfly and one cta_sum): half the barriers per row.  Rows p, p + parts,
// p + 2 parts, ... are taken in pairs; while one pair is reduced and written, the next
// pair's loads are in flight (four register sets).
template <typename TT, int VPT>
struct RmsVjpPair {
    using T = TT;
    using E = Elem<T>;
    static constexpr int VEC = E::kVec;
    static constexpr int NP = VEC / 2;
    const VjpArgs& a;
    const float2 (&wf)[VPT][NP];
    ColAcc<VPT, NP, 1>& acc;
    CtaSums<4>& red;
    float invD;

    __device__ __forceinline__ void sums(const V16 (&xv)[VPT], const V16 (&gv)[VPT], float& ss,
                                         float& sp) const {
        float2 s0 = splat2(0.f), s1 = splat2(0.f);
#pragma unroll
        for (int k = 0; k < VPT; ++k)
#pragma unroll
            for (int e = 0; e < VEC; e += 2) {
                if constexpr (sizeof(T) == 2) {
                    s0 = bf16x2_mac(xv[k].u[e / 2], xv[k].u[e / 2], s0);
                    s1 = fma2(bf16x2_mac(gv[k].u[e / 2], xv[k].u[e / 2], splat2(0.f)),
                              wf[k][e / 2], s1);
                } else {
                    const float2 x2 = E::get2(xv[k], e);
                    const float2 u2 = mul2(E::get2(gv[k], e), wf[k][e / 2]);
                    s0 = fma2(x2, x2, s0);
                    s1 = fma2(u2, x2, s1);
                }
            }
        ss = __fadd_rn(s0.x, s0.y);
        sp = __fadd_rn(s1.x, s1.y);
    }
    __device__ __forceinline__ void write(int64_t row, const V16 (&xv)[VPT], const V16 (&gv)[VPT],
                                          float ss, float sp) const {
        const float r = rsqrtf(__fmaf_rn(ss, invD, a.eps));
        const float vr = __fmul_rn(__fmul_rn(r, r), __fmul_rn(sp, invD));
        const float2 r2 = splat2(r), nv2 = splat2(-vr);
        const bool live = row < a.rows;
        const size_t roff = (size_t)row * (size_t)a.nvec * 16;
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = threadIdx.x + k * blockDim.x;
            if (v < a.nvec) {
                V16 o;
#pragma unroll
                for (int e = 0; e < VEC; e += 2) {
                    const float2 x2 = E::get2(xv[k], e);
                    const float2 g2 = E::get2(gv[k], e);
                    const float2 u2 = mul2(g2, wf[k][e / 2]);
                    E::put2(o, e, mul2(r2, fma2(x2, nv2, u2)));        // r (g w - x v)
                    float2& ac = acc.at(0, k * NP + e / 2);
                    ac = fma2(mul2(g2, x2), r2, ac);  // a row past the end holds zeros
                }
                if (live) st_stream(static_cast<char*>(a.dx) + roff + (size_t)v * 16, o);
            }
        }
    }
    __device__ __forceinline__ void operator()(int64_t r0, const V16 (&x0)[VPT], const V16 (&g0)[VPT],
                                               int64_t r1, const V16 (&x1)[VPT],
                                               const V16 (&g1)[VPT]) const {
        float s[4];
        sums(x0, g0, s[0], s[1]);
        sums(x1, g1, s[2], s[3]);
        cta_sum<4>(s, red);
        write(r0, x0, g0, s[0], s[1]);
        write(r1, x1, g1, s[2], s[3]);
    }
};

template <int VPT, typename Pair>
__device__ __forceinline__ void walk_row_pairs(const VjpArgs& a, Pair&& pair_step) {
    using T = typename Pair::T;
    V16 xa[VPT], ga[VPT], xb[VPT], gb[VPT], xc[VPT], gc[VPT], xd[VPT], gd[VPT];
    const int64_t step = a.parts;
    load_xg<T, VPT>(a, blockIdx.x, xa, ga);
    load_xg<T, VPT>(a, blockIdx.x + step, xb, gb);
    for (int64_t row = blockIdx.x; row < a.rows; row += 4 * step) {
        load_xg<T, VPT>(a, row + 2 * step, xc, gc);
        load_xg<T, VPT>(a, row + 3 * step, xd, gd);
        pair_step(row, xa, ga, row + step, xb, gb);
        if (row + 2 * step >= a.rows) break;
        load_xg<T, VPT>(a, row + 4 * step, xa, ga);
        load_xg<T, VPT>(a, row + 5 * step, xb, gb);
        pair_step(row + 2 * step, xc, gc, row + 3 * step, xd, gd);
    }
}

// CTAs of at most 512 threads: the four register sets need up to 128 registers.
constexpr int kVjpPairsMaxThreads = 512;

template <typename T, int VPT>
__global__ void __launch_bounds__(kVjpPairsMaxThreads) rms_vjp_pairs_kernel(const VjpArgs a) {
    pdl_wait();
    pdl_release();
    constexpr int NP = Elem<T>::kVec / 2;
    __shared__ CtaSums<4> red;
    extern __shared__ float2 acc_smem[];
    float2 wf[VPT][NP];
    load_wf<T, VPT>(a, wf);
    ColAcc<VPT, NP, 1> acc;
    acc.init(acc_smem);
    walk_row_pairs<VPT>(a, RmsVjpPair<T, VPT>{a, wf, acc, red, 1.f / (float)a.D});
    if (a.want_dw) {
        float* out = a.part + (size_t)blockIdx.x * a.D;
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = threadIdx.x + k * blockDim.x;
            if (v < a.nvec)
#pragma unroll
                for (int i = 0; i < NP; ++i)
                    reinterpret_cast<float2*>(out)[v * NP + i] = acc.at(0, k * NP + i);
        }
    }
}

// ---- LayerNormVjp, kernel 1 ---------------------------------------------------------------
template <typename TT, int VPT>
struct LayerVjpRow {
    using T = TT;
    using E = Elem<T>;
    static constexpr int VEC = E::kVec;
    static constexpr int NP = VEC / 2;
    const VjpArgs& a;
    V16 (&wv)[VPT];         // VPT <= 2: held for the whole walk; VPT = 4: reloaded per row
    ColAcc<VPT, NP, 2>& acc;  // sums: 0 dw, 1 db
    CtaSums<2>& red1;       // pass 1
    CtaSums<3>& red2;       // pass 2
    float invD;

    __device__ __forceinline__ void operator()(int64_t row, const V16 (&xv)[VPT],
                                               const V16 (&gv)[VPT]) const {
        if (VPT > 2)
#pragma unroll
            for (int k = 0; k < VPT; ++k) wv[k] = load_w<T>(a, k);
        // bfloat16 pairs are consumed packed (bf16x2_mac: the same single roundings as the
        // float32 arithmetic on the unpacked values, without the unpacking)
        constexpr bool kPacked = sizeof(T) == 2;
        // pass 1: sum x and sum a (a = w g)
        float2 p0 = splat2(0.f), p1 = splat2(0.f);
#pragma unroll
        for (int k = 0; k < VPT; ++k)
#pragma unroll
            for (int e = 0; e < VEC; e += 2) {
                if constexpr (kPacked) {
                    p0 = bf16x2_mac(xv[k].u[e / 2], kBf16x2One, p0);
                    p1 = bf16x2_mac(wv[k].u[e / 2], gv[k].u[e / 2], p1);
                } else {
                    p0 = add2(p0, E::get2(xv[k], e));
                    p1 = add2(p1, mul2(E::get2(wv[k], e), E::get2(gv[k], e)));
                }
            }
        float p[2] = {__fadd_rn(p0.x, p0.y), __fadd_rn(p1.x, p1.y)};
        cta_sum<2>(p, red1);
        const float m1 = __fmul_rn(p[0], invD);
        const float ma = __fmul_rn(p[1], invD);
        const float2 nm1 = splat2(-m1);
        // pass 2: sum c', sum c'^2 and sum a c' around m1 (c' = x - m1)
        float2 q0 = splat2(0.f), q1 = splat2(0.f), q2 = splat2(0.f);
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = threadIdx.x + k * blockDim.x;
            if (v < a.nvec)   // c' of a padding lane would be -m1
#pragma unroll
                for (int e = 0; e < VEC; e += 2) {
                    float2 cp, a2;
                    if constexpr (kPacked) {
                        cp = bf16x2_mac(xv[k].u[e / 2], kBf16x2One, nm1);
                        a2 = bf16x2_mac(wv[k].u[e / 2], gv[k].u[e / 2], splat2(0.f));
                    } else {
                        cp = add2(E::get2(xv[k], e), nm1);
                        a2 = mul2(E::get2(wv[k], e), E::get2(gv[k], e));
                    }
                    q0 = add2(q0, cp);
                    q1 = fma2(cp, cp, q1);
                    q2 = fma2(a2, cp, q2);
                }
        }
        float q[3] = {__fadd_rn(q0.x, q0.y), __fadd_rn(q1.x, q1.y), __fadd_rn(q2.x, q2.y)};
        cta_sum<3>(q, red2);
        const float dm = __fmul_rn(q[0], invD);                             // mean = m1 + dm
        const float var = fmaxf(__fmaf_rn(q[1], invD, -__fmul_rn(dm, dm)), 0.f);
        const float r = rsqrtf(__fadd_rn(var, a.eps));
        // dx = r (a - mean(a) - c B) with B = r^2 sum(a c) / D and c = c' - dm, evaluated as
        // r a + (c' (-r B) + (r B dm - r mean(a))), and xhat = c r as c' r - dm r: each
        // rounding relative to one of the terms, two packed fmas a pair for dx and one for
        // xhat
        const float B = __fmul_rn(__fmul_rn(r, r), __fmul_rn(__fmaf_rn(-dm, p[1], q[2]), invD));
        const float rB = __fmul_rn(r, B);
        const float2 r2 = splat2(r), nrB = splat2(-rB),
                     k0 = splat2(__fmaf_rn(rB, dm, -__fmul_rn(r, ma))),
                     ndmr = splat2(-__fmul_rn(dm, r));
        const size_t roff = (size_t)row * (size_t)a.nvec * 16;
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = threadIdx.x + k * blockDim.x;
            if (v < a.nvec) {
                V16 o;
#pragma unroll
                for (int e = 0; e < VEC; e += 2) {
                    const float2 g2 = E::get2(gv[k], e);
                    float2 a2, cp;  // cp = c' = x - m1
                    if constexpr (kPacked) {
                        a2 = bf16x2_mac(wv[k].u[e / 2], gv[k].u[e / 2], splat2(0.f));
                        cp = bf16x2_mac(xv[k].u[e / 2], kBf16x2One, nm1);
                    } else {
                        a2 = mul2(E::get2(wv[k], e), g2);
                        cp = add2(E::get2(xv[k], e), nm1);
                    }
                    E::put2(o, e, fma2(r2, a2, fma2(cp, nrB, k0)));
                    float2& aw = acc.at(0, k * NP + e / 2);
                    float2& ab = acc.at(1, k * NP + e / 2);
                    aw = fma2(g2, fma2(cp, r2, ndmr), aw);
                    ab = add2(ab, g2);
                }
                st_stream(static_cast<char*>(a.dx) + roff + (size_t)v * 16, o);
            }
        }
    }
};

template <typename T, int VPT>
__global__ void __launch_bounds__(vjp_max_threads(VPT)) layer_vjp_kernel(const VjpArgs a) {
    pdl_wait();
    pdl_release();
    constexpr int NP = Elem<T>::kVec / 2;
    __shared__ CtaSums<2> red1;
    __shared__ CtaSums<3> red2;
    extern __shared__ float2 acc_smem[];
    V16 wv[VPT];
    if (VPT <= 2)
#pragma unroll
        for (int k = 0; k < VPT; ++k) wv[k] = load_w<T>(a, k);
    ColAcc<VPT, NP, 2> acc;
    acc.init(acc_smem);
    walk_rows<VPT>(a, LayerVjpRow<T, VPT>{a, wv, acc, red1, red2, 1.f / (float)a.D});
    if (a.part) {
        float2* outw = reinterpret_cast<float2*>(a.part + (size_t)blockIdx.x * a.D);
        float2* outb = reinterpret_cast<float2*>(a.part + ((size_t)a.parts + blockIdx.x) * a.D);
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = threadIdx.x + k * blockDim.x;
            if (v < a.nvec)
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                    if (a.want_dw) outw[v * NP + i] = acc.at(0, k * NP + i);
                    if (a.want_db) outb[v * NP + i] = acc.at(1, k * NP + i);
                }
        }
    }
}

// ---- generic kernel 1: any D, any alignment ----------------------------------------------------
// One CTA per partial row p, walking rows p, p + parts, ...: scalar accesses, three passes
// over the row (x and g are re-read from global memory / L1), row statistics in double.
// The CTA's column partial sums live in its own row of the workspace, updated in place
// after each row (it is the only writer of that row).  dx may be x or g: each thread reads
// index j in every pass before it writes index j in the last one, and the passes of a row
// are separated by the barriers of the reductions.
template <int N>
__device__ __forceinline__ void cta_sum_f64(double (&v)[N], double (*buf)[32]) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int i = 0; i < N; ++i) {
        v[i] = warp_sum(v[i]);
        if (lane == 0) buf[i][wid] = v[i];
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < N; ++i) {
        double t = 0.0;
        for (int k = 0; k < nw; ++k) t += buf[i][k];
        v[i] = t;
    }
    __syncthreads();  // the buffer may be reused at once
}

template <typename T, bool LAYER>
__global__ void __launch_bounds__(256) vjp_generic_kernel(const VjpArgs a) {
    pdl_wait();
    pdl_release();
    using E = Elem<T>;
    __shared__ double buf[3][32];
    const int D = a.D;
    const double invD = 1.0 / (double)D;
    float* pdw = a.part ? a.part + (size_t)blockIdx.x * D : nullptr;
    float* pdb = (a.part && LAYER) ? a.part + ((size_t)a.parts + blockIdx.x) * D : nullptr;
    bool first = true;
    for (int64_t row = blockIdx.x; row < a.rows; row += a.parts, first = false) {
        const int64_t r0 = row * (int64_t)D;
        double mean = 0.0;
        if constexpr (LAYER) {
            double s[1] = {0.0};
            for (int j = threadIdx.x; j < D; j += blockDim.x) s[0] += (double)E::load1(a.x, r0 + j);
            cta_sum_f64<1>(s, buf);
            mean = s[0] * invD;
        }
        // RMS: sum x^2, sum g w x.  Layer: sum c^2, sum a, sum a c with c = x - mean, a = w g.
        double s[3] = {0.0, 0.0, 0.0};
        for (int j = threadIdx.x; j < D; j += blockDim.x) {
            const double x = (double)E::load1(a.x, r0 + j) - mean;
            const double wj = a.w ? (double)E::load1(a.w, j) : 1.0;
            const double u = wj * (double)E::load1(a.g, r0 + j);
            s[0] = fma(x, x, s[0]);
            if constexpr (LAYER) {
                s[1] += u;
                s[2] = fma(u, x, s[2]);
            } else {
                s[1] = fma(u, x, s[1]);
            }
        }
        cta_sum_f64<3>(s, buf);
        const double r = 1.0 / sqrt(s[0] * invD + (double)a.eps);
        // RMS: dx = r (u - x v), v = r^2 sum(u x) / D.
        // Layer: dx = r (u - mean(a) - xh mean(a xh)), xh = c r, mean(a xh) = r sum(a c) / D.
        const double ma = LAYER ? s[1] * invD : 0.0;
        const double k = LAYER ? r * r * s[2] * invD : r * r * s[1] * invD;
        for (int j = threadIdx.x; j < D; j += blockDim.x) {
            const double x = (double)E::load1(a.x, r0 + j) - mean;
            const double gj = (double)E::load1(a.g, r0 + j);
            const double wj = a.w ? (double)E::load1(a.w, j) : 1.0;
            E::store1(a.dx, r0 + j, (float)(r * (wj * gj - ma - x * k)));
            if (pdw) {
                const float c = (float)(gj * x * r);
                pdw[j] = first ? c : __fadd_rn(pdw[j], c);
            }
            if constexpr (LAYER)
                if (pdb) pdb[j] = first ? (float)gj : __fadd_rn(pdb[j], (float)gj);
        }
    }
}

// ---- narrow rows: at most 64 vectors a row --------------------------------------------------
// A row of the kernels above takes at least a warp and pays CTA-wide reductions; a row of
// 128 bfloat16 features then leaves half of its warp idle.  Here a CTA of 256 threads holds
// R = 256 / G row groups of G threads (a power of two up to 32, VPT vectors a thread); each
// group walks its own rows (virtual part p = blockIdx.x R + group, rows p, p + gridDim.x R,
// ...), reduces with shuffles over its own lanes only (no barrier), and keeps its column
// partial sums in registers, with the next row's x and g loading into a second register set
// meanwhile.  At the end the CTA adds its groups' partials in shared memory
// in group order -- one partial row per CTA, as kernel 2 expects.  The arithmetic of a row
// is that of RmsVjpRow / LayerVjpRow (the same roundings; the sums differ only in the order
// of their additions).
template <typename T, int VPT, bool LAYER>
__global__ void __launch_bounds__(256) vjp_narrow_kernel(const VjpArgs a) {
    pdl_wait();
    pdl_release();
    using E = Elem<T>;
    constexpr int VEC = E::kVec;
    constexpr int NP = VEC / 2;
    constexpr int NSUM = LAYER ? 2 : 1;
    constexpr bool kPacked = sizeof(T) == 2;
    extern __shared__ float2 comb[];  // [R][nvec * NP]: the groups' partials of one sum
    const int G = a.G;
    const int R = blockDim.x / G;
    const int grp = threadIdx.x / G;
    const int t = threadIdx.x - grp * G;
    const int64_t step = (int64_t)gridDim.x * R;
    const float invD = 1.f / (float)a.D;

    V16 wv[VPT];
    float2 acc[NSUM][VPT * NP];
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
        const int v = t + k * G;
        wv[k] = (a.w != nullptr && v < a.nvec)
                    ? ld_param(static_cast<const char*>(a.w) + (size_t)v * 16)
                    : ones_vec<T>();
#pragma unroll
        for (int i = 0; i < NP; ++i)
#pragma unroll
            for (int j = 0; j < NSUM; ++j) acc[j][k * NP + i] = splat2(0.f);
    }

    // the groups of one warp step together while the warp's first group has a row (the
    // others then have one too, or take part as inactive rows): the shuffles are warp-wide
    const int gpw = G < 32 ? 32 / G : 1;
    const int first = grp / gpw * gpw;
    // the next row's x and g load into a second register set before this row is reduced
    auto load = [&](int64_t row, V16 (&xo)[VPT], V16 (&go)[VPT]) {
        const size_t off = (size_t)row * (size_t)a.nvec * 16;
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = t + k * G;
            const bool in = row < a.rows && v < a.nvec;
            xo[k] = in ? ld_stream(static_cast<const char*>(a.x) + off + (size_t)v * 16)
                       : zeros_vec<T>();
            go[k] = in ? ld_stream(static_cast<const char*>(a.g) + off + (size_t)v * 16)
                       : zeros_vec<T>();
        }
    };
    V16 xn[VPT], gn[VPT];
    load((int64_t)blockIdx.x * R + grp, xn, gn);
    for (int64_t r0 = (int64_t)blockIdx.x * R + first; r0 < a.rows; r0 += step) {
        const int64_t row = r0 + (grp - first);
        const bool live = row < a.rows;
        const size_t roff = (size_t)row * (size_t)a.nvec * 16;
        V16 xv[VPT], gv[VPT];
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            xv[k] = xn[k];
            gv[k] = gn[k];
        }
        load(row + step, xn, gn);
        if constexpr (!LAYER) {
            float2 s0 = splat2(0.f), s1 = splat2(0.f);
#pragma unroll
            for (int k = 0; k < VPT; ++k)
#pragma unroll
                for (int e = 0; e < VEC; e += 2) {
                    const float2 w2 = E::get2(wv[k], e);
                    if constexpr (kPacked) {
                        s0 = bf16x2_mac(xv[k].u[e / 2], xv[k].u[e / 2], s0);
                        s1 = fma2(bf16x2_mac(gv[k].u[e / 2], xv[k].u[e / 2], splat2(0.f)), w2,
                                  s1);
                    } else {
                        const float2 x2 = E::get2(xv[k], e);
                        const float2 u2 = mul2(E::get2(gv[k], e), w2);
                        s0 = fma2(x2, x2, s0);
                        s1 = fma2(u2, x2, s1);
                    }
                }
            const float ss = group_sum(__fadd_rn(s0.x, s0.y), G);
            const float sp = group_sum(__fadd_rn(s1.x, s1.y), G);
            const float r = rsqrtf(__fmaf_rn(ss, invD, a.eps));
            const float vr = __fmul_rn(__fmul_rn(r, r), __fmul_rn(sp, invD));
            const float2 r2 = splat2(r), nv2 = splat2(-vr);
#pragma unroll
            for (int k = 0; k < VPT; ++k) {
                const int v = t + k * G;
                if (live && v < a.nvec) {
                    V16 o;
#pragma unroll
                    for (int e = 0; e < VEC; e += 2) {
                        const float2 x2 = E::get2(xv[k], e);
                        const float2 g2 = E::get2(gv[k], e);
                        const float2 u2 = mul2(g2, E::get2(wv[k], e));
                        E::put2(o, e, mul2(r2, fma2(x2, nv2, u2)));  // r (g w - x v)
                        acc[0][k * NP + e / 2] = fma2(mul2(g2, x2), r2, acc[0][k * NP + e / 2]);
                    }
                    st_stream(static_cast<char*>(a.dx) + roff + (size_t)v * 16, o);
                }
            }
        } else {
            // pass 1: sum x and sum a (a = w g), a first mean m1
            float2 p0 = splat2(0.f), p1 = splat2(0.f);
#pragma unroll
            for (int k = 0; k < VPT; ++k)
#pragma unroll
                for (int e = 0; e < VEC; e += 2) {
                    if constexpr (kPacked) {
                        p0 = bf16x2_mac(xv[k].u[e / 2], kBf16x2One, p0);
                        p1 = bf16x2_mac(wv[k].u[e / 2], gv[k].u[e / 2], p1);
                    } else {
                        p0 = add2(p0, E::get2(xv[k], e));
                        p1 = add2(p1, mul2(E::get2(wv[k], e), E::get2(gv[k], e)));
                    }
                }
            const float m1 = __fmul_rn(group_sum(__fadd_rn(p0.x, p0.y), G), invD);
            const float sa = group_sum(__fadd_rn(p1.x, p1.y), G);
            const float ma = __fmul_rn(sa, invD);
            const float2 nm1 = splat2(-m1);
            // pass 2: sum c', sum c'^2 and sum a c' around m1 (c' = x - m1)
            float2 q0 = splat2(0.f), q1 = splat2(0.f), q2 = splat2(0.f);
#pragma unroll
            for (int k = 0; k < VPT; ++k) {
                if (t + k * G < a.nvec)  // c' of a padding lane would be -m1
#pragma unroll
                    for (int e = 0; e < VEC; e += 2) {
                        float2 cp, a2;
                        if constexpr (kPacked) {
                            cp = bf16x2_mac(xv[k].u[e / 2], kBf16x2One, nm1);
                            a2 = bf16x2_mac(wv[k].u[e / 2], gv[k].u[e / 2], splat2(0.f));
                        } else {
                            cp = add2(E::get2(xv[k], e), nm1);
                            a2 = mul2(E::get2(wv[k], e), E::get2(gv[k], e));
                        }
                        q0 = add2(q0, cp);
                        q1 = fma2(cp, cp, q1);
                        q2 = fma2(a2, cp, q2);
                    }
            }
            const float c0 = group_sum(__fadd_rn(q0.x, q0.y), G);
            const float c1 = group_sum(__fadd_rn(q1.x, q1.y), G);
            const float c2 = group_sum(__fadd_rn(q2.x, q2.y), G);
            const float dm = __fmul_rn(c0, invD);  // mean = m1 + dm
            const float var = fmaxf(__fmaf_rn(c1, invD, -__fmul_rn(dm, dm)), 0.f);
            const float r = rsqrtf(__fadd_rn(var, a.eps));
            const float B = __fmul_rn(__fmul_rn(r, r), __fmul_rn(__fmaf_rn(-dm, sa, c2), invD));
            const float rB = __fmul_rn(r, B);
            const float2 r2 = splat2(r), nrB = splat2(-rB),
                         k0 = splat2(__fmaf_rn(rB, dm, -__fmul_rn(r, ma))),
                         ndmr = splat2(-__fmul_rn(dm, r));
#pragma unroll
            for (int k = 0; k < VPT; ++k) {
                const int v = t + k * G;
                if (live && v < a.nvec) {
                    V16 o;
#pragma unroll
                    for (int e = 0; e < VEC; e += 2) {
                        const float2 g2 = E::get2(gv[k], e);
                        float2 a2, cp;
                        if constexpr (kPacked) {
                            a2 = bf16x2_mac(wv[k].u[e / 2], gv[k].u[e / 2], splat2(0.f));
                            cp = bf16x2_mac(xv[k].u[e / 2], kBf16x2One, nm1);
                        } else {
                            a2 = mul2(E::get2(wv[k], e), g2);
                            cp = add2(E::get2(xv[k], e), nm1);
                        }
                        E::put2(o, e, fma2(r2, a2, fma2(cp, nrB, k0)));
                        float2& aw = acc[0][k * NP + e / 2];
                        float2& ab = acc[NSUM - 1][k * NP + e / 2];
                        aw = fma2(g2, fma2(cp, r2, ndmr), aw);
                        ab = add2(ab, g2);
                    }
                    st_stream(static_cast<char*>(a.dx) + roff + (size_t)v * 16, o);
                }
            }
        }
    }

    if (a.part == nullptr) return;
    // the groups' partials, added per column in group order
    const int ncol = a.nvec * NP;  // float pairs of a row
#pragma unroll
    for (int j = 0; j < NSUM; ++j) {
        const bool want = j == 0 ? a.want_dw : a.want_db;
        if (!want) continue;  // uniform over the CTA
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = t + k * G;
            if (v < a.nvec)
#pragma unroll
                for (int i = 0; i < NP; ++i) comb[(size_t)grp * ncol + v * NP + i] = acc[j][k * NP + i];
        }
        __syncthreads();
        float2* out = reinterpret_cast<float2*>(a.part + ((size_t)j * a.parts + blockIdx.x) * a.D);
        for (int c = threadIdx.x; c < ncol; c += blockDim.x) {
            float2 sum = comb[c];
            for (int q = 1; q < R; ++q) sum = add2(sum, comb[(size_t)q * ncol + c]);
            out[c] = sum;
        }
        __syncthreads();
    }
}

// ---- kernel 2: column sums of the partials --------------------------------------------------
// out[y][j] = sum_{p < parts} part[first + y][p][j] in double, y = blockIdx.y.
// A CTA of nw = blockDim.x / 32 warps owns 32 columns.  Warp w adds the contiguous run of
// parts [w per, (w + 1) per) in order, per = ceil(parts / nw), with up to kReduceBatch loads
// in flight per lane; the host picks nw = ceil(parts / kReduceBatch) (at most 32), so a warp
// waits for one batch of loads.  After one barrier warp 0 adds the warps' sums in warp
// order.  The order is fixed, so the result does not depend on timing.
constexpr int kReduceBatch = 16;
constexpr int kReduceMaxWarps = 32;

struct ReduceArgs {
    const float* part;  // [nsum][parts][D]
    void* out[2];       // [D] for sums first, first + 1
    int first;          // slice of the first sum reduced (0: dw, 1: db)
    int parts;
    int D;
};

// warps per CTA of vjp_reduce_kernel for `parts` partial rows
__host__ __device__ constexpr int reduce_warps(int parts) {
    return parts <= kReduceBatch ? 1
           : (parts + kReduceBatch - 1) / kReduceBatch > kReduceMaxWarps
               ? kReduceMaxWarps
               : (parts + kReduceBatch - 1) / kReduceBatch;
}

template <typename T>
__global__ void __launch_bounds__(kReduceMaxWarps * 32) vjp_reduce_kernel(const ReduceArgs a) {
    pdl_wait();
    pdl_release();
    __shared__ double sw[kReduceMaxWarps][32];
    const int lane = threadIdx.x & 31;
    const int w = threadIdx.x >> 5;
    const int nw = blockDim.x >> 5;
    const int j = blockIdx.x * 32 + lane;
    const float* part =
        a.part ? a.part + (size_t)(a.first + blockIdx.y) * a.parts * a.D : nullptr;
    const int per = (a.parts + nw - 1) / nw;
    const int p0 = min(w * per, a.parts);
    const int p1 = min(p0 + per, a.parts);
    double s = 0.0;
    if (j < a.D && part) {
        const float* col = part + (size_t)p0 * a.D + j;
        int n = p1 - p0;
        for (; n >= kReduceBatch; n -= kReduceBatch, col += (size_t)kReduceBatch * a.D) {
            float v[kReduceBatch];
#pragma unroll
            for (int i = 0; i < kReduceBatch; ++i) v[i] = col[(size_t)i * a.D];
#pragma unroll
            for (int i = 0; i < kReduceBatch; ++i) s += (double)v[i];
        }
        float v[kReduceBatch];
#pragma unroll
        for (int i = 0; i < kReduceBatch; ++i) v[i] = i < n ? col[(size_t)i * a.D] : 0.f;
#pragma unroll
        for (int i = 0; i < kReduceBatch; ++i)
            if (i < n) s += (double)v[i];
    }
    sw[w][lane] = s;
    __syncthreads();
    if (w == 0 && j < a.D) {
        double t = sw[0][lane];
        for (int i = 1; i < nw; ++i) t += sw[i][lane];
        Elem<T>::store1(blockIdx.y ? a.out[1] : a.out[0], j, __double2float_rn(t));
    }
}

}  // namespace nvn
