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
};

// Largest CTA of kernel 1: one thread per vector for VPT = 1 up to 1024 vectors a row.
constexpr int kVjpThreads = 1024;

// Sum of N floats across the CTA with one barrier: warp butterflies, one partial per warp
// in `buf`, then every warp reduces the partials itself with the same butterfly, so all
// threads end with bit-identical totals.  `buf` holds N x 32 floats.
template <int N>
__device__ __forceinline__ void cta_sum(float (&v)[N], float (*buf)[32]) {
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = warp_sum(v[i]);
    const int nw = blockDim.x >> 5;
    if (nw == 1) return;
    const int lane = threadIdx.x & 31;
    if (lane == 0)
#pragma unroll
        for (int i = 0; i < N; ++i) buf[i][threadIdx.x >> 5] = v[i];
    __syncthreads();
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = warp_sum(lane < nw ? buf[i][lane] : 0.f);
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

// ---- RmsNormVjp, kernel 1 ---------------------------------------------------------------
template <typename T, int VPT>
__global__ void __launch_bounds__(kVjpThreads) rms_vjp_kernel(const VjpArgs a) {
    pdl_wait();
    pdl_release();
    using E = Elem<T>;
    constexpr int VEC = E::kVec;
    constexpr bool kAhead = VPT == 1;  // next row in flight
    __shared__ float red[2][2][32];
    const int G = blockDim.x;
    const int t = threadIdx.x;
    const float invD = 1.f / (float)a.D;

    V16 wv[VPT];
    float acc[VPT][VEC];
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
        wv[k] = load_w<T>(a, k);
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[k][e] = 0.f;
    }
    V16 xv[VPT], gv[VPT];
    if (kAhead) load_xg<T, VPT>(a, blockIdx.x, xv, gv);

    int it = 0;
    for (int64_t row = blockIdx.x; row < a.rows; row += a.parts, ++it) {
        V16 xn[VPT], gn[VPT];
        if (kAhead)
            load_xg<T, VPT>(a, row + a.parts, xn, gn);
        else
            load_xg<T, VPT>(a, row, xv, gv);
        // sum x^2 (the scale) and sum g w x (the projection)
        float s[2] = {0.f, 0.f};
#pragma unroll
        for (int k = 0; k < VPT; ++k)
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                const float xf = E::get(xv[k], e);
                s[0] = __fmaf_rn(xf, xf, s[0]);
                s[1] = __fmaf_rn(__fmul_rn(E::get(gv[k], e), E::get(wv[k], e)), xf, s[1]);
            }
        cta_sum<2>(s, red[it & 1]);
        const float r = rsqrtf(__fmaf_rn(s[0], invD, a.eps));
        const float vr = __fmul_rn(__fmul_rn(r, r), __fmul_rn(s[1], invD));
        const size_t roff = (size_t)row * (size_t)a.nvec * 16;
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = t + k * G;
            if (v < a.nvec) {
                V16 o;
#pragma unroll
                for (int e = 0; e < VEC; e += 2) {
                    float d[2];
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const float xf = E::get(xv[k], e + q);
                        const float gf = E::get(gv[k], e + q);
                        const float u = __fmul_rn(gf, E::get(wv[k], e + q));
                        d[q] = __fmul_rn(r, __fmaf_rn(-xf, vr, u));   // r (g w - x v)
                        acc[k][e + q] = __fmaf_rn(__fmul_rn(gf, xf), r, acc[k][e + q]);
                    }
                    E::put2(o, e, d[0], d[1]);
                }
                st_stream(static_cast<char*>(a.dx) + roff + (size_t)v * 16, o);
            }
        }
        if (kAhead)
#pragma unroll
            for (int k = 0; k < VPT; ++k) {
                xv[k] = xn[k];
                gv[k] = gn[k];
            }
    }
    if (a.want_dw) {
        float* out = a.part + (size_t)blockIdx.x * a.D;
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = t + k * G;
            if (v < a.nvec)
#pragma unroll
                for (int e = 0; e < VEC; ++e) out[v * VEC + e] = acc[k][e];
        }
    }
}

// ---- LayerNormVjp, kernel 1 ---------------------------------------------------------------
template <typename T, int VPT>
__global__ void __launch_bounds__(kVjpThreads) layer_vjp_kernel(const VjpArgs a) {
    pdl_wait();
    pdl_release();
    using E = Elem<T>;
    constexpr int VEC = E::kVec;
    constexpr bool kAhead = VPT == 1;  // next row in flight; w kept in registers
    __shared__ float red[2][3][32];    // [pass][sum][warp]
    const int G = blockDim.x;
    const int t = threadIdx.x;
    const float invD = 1.f / (float)a.D;

    V16 wv[VPT];
    float accw[VPT][VEC], accb[VPT][VEC];
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
        if (kAhead) wv[k] = load_w<T>(a, k);
#pragma unroll
        for (int e = 0; e < VEC; ++e) accw[k][e] = accb[k][e] = 0.f;
    }
    V16 xv[VPT], gv[VPT];
    if (kAhead) load_xg<T, VPT>(a, blockIdx.x, xv, gv);

    for (int64_t row = blockIdx.x; row < a.rows; row += a.parts) {
        V16 xn[VPT], gn[VPT];
        if (kAhead) {
            load_xg<T, VPT>(a, row + a.parts, xn, gn);
        } else {
            load_xg<T, VPT>(a, row, xv, gv);
#pragma unroll
            for (int k = 0; k < VPT; ++k) wv[k] = load_w<T>(a, k);
        }
        // pass 1: sum x and sum a (a = w g)
        float p[2] = {0.f, 0.f};
#pragma unroll
        for (int k = 0; k < VPT; ++k)
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                p[0] = __fadd_rn(p[0], E::get(xv[k], e));
                p[1] = __fadd_rn(p[1], __fmul_rn(E::get(wv[k], e), E::get(gv[k], e)));
            }
        cta_sum<2>(p, red[0]);
        const float m1 = __fmul_rn(p[0], invD);
        const float ma = __fmul_rn(p[1], invD);
        // pass 2: sum c', sum c'^2 and sum a c' around m1 (c' = x - m1)
        float q[3] = {0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = t + k * G;
            if (v < a.nvec)   // c' of a padding lane would be -m1
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    const float cp = __fsub_rn(E::get(xv[k], e), m1);
                    const float af = __fmul_rn(E::get(wv[k], e), E::get(gv[k], e));
                    q[0] = __fadd_rn(q[0], cp);
                    q[1] = __fmaf_rn(cp, cp, q[1]);
                    q[2] = __fmaf_rn(af, cp, q[2]);
                }
        }
        cta_sum<3>(q, red[1]);
        const float dm = __fmul_rn(q[0], invD);                             // mean = m1 + dm
        const float var = fmaxf(__fmaf_rn(q[1], invD, -__fmul_rn(dm, dm)), 0.f);
        const float r = rsqrtf(__fadd_rn(var, a.eps));
        // dx = r (a - mean(a) - c B) with B = r^2 sum(a c) / D
        const float B = __fmul_rn(__fmul_rn(r, r), __fmul_rn(__fmaf_rn(-dm, p[1], q[2]), invD));
        const size_t roff = (size_t)row * (size_t)a.nvec * 16;
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = t + k * G;
            if (v < a.nvec) {
                V16 o;
#pragma unroll
                for (int e = 0; e < VEC; e += 2) {
                    float d[2];
#pragma unroll
                    for (int q2 = 0; q2 < 2; ++q2) {
                        const float xf = E::get(xv[k], e + q2);
                        const float gf = E::get(gv[k], e + q2);
                        const float af = __fmul_rn(E::get(wv[k], e + q2), gf);
                        const float c = __fsub_rn(__fsub_rn(xf, m1), dm);
                        d[q2] = __fmul_rn(r, __fmaf_rn(-c, B, __fsub_rn(af, ma)));
                        accw[k][e + q2] = __fmaf_rn(gf, __fmul_rn(c, r), accw[k][e + q2]);
                        accb[k][e + q2] = __fadd_rn(accb[k][e + q2], gf);
                    }
                    E::put2(o, e, d[0], d[1]);
                }
                st_stream(static_cast<char*>(a.dx) + roff + (size_t)v * 16, o);
            }
        }
        if (kAhead)
#pragma unroll
            for (int k = 0; k < VPT; ++k) {
                xv[k] = xn[k];
                gv[k] = gn[k];
            }
    }
    if (a.part) {
        float* outw = a.part + (size_t)blockIdx.x * a.D;
        float* outb = a.part + ((size_t)a.parts + blockIdx.x) * a.D;
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = t + k * G;
            if (v < a.nvec)
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    if (a.want_dw) outw[v * VEC + e] = accw[k][e];
                    if (a.want_db) outb[v * VEC + e] = accb[k][e];
                }
        }
    }
}

// ---- kernel 2: column sums of the partials --------------------------------------------------
// out[j] = sum_{p < parts} part[p][j] in double.  A CTA owns 32 columns; warp w adds parts
// w, w + 8, w + 16, ... in that order, then lane j of warp 0 adds the 8 warp sums in warp
// order: a fixed order, so the result does not depend on timing.
constexpr int kReduceWarps = 8;

template <typename T>
__global__ void __launch_bounds__(kReduceWarps * 32) vjp_reduce_kernel(const float* part,
                                                                       int parts, int D,
                                                                       void* out) {
    pdl_wait();
    pdl_release();
    __shared__ double sw[kReduceWarps][32];
    const int lane = threadIdx.x & 31;
    const int w = threadIdx.x >> 5;
    const int j = blockIdx.x * 32 + lane;
    double s = 0.0;
    if (j < D) {
#pragma unroll 4
        for (int p = w; p < parts; p += kReduceWarps) s += (double)part[(size_t)p * D + j];
    }
    sw[w][lane] = s;
    __syncthreads();
    if (w == 0 && j < D) {
        double tot = 0.0;
#pragma unroll
        for (int i = 0; i < kReduceWarps; ++i) tot += sw[i][lane];
        Elem<T>::store1(out, j, __double2float_rn(tot));
    }
}

}  // namespace nvn
