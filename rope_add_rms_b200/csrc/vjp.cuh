// vjp.cuh -- gradients of rms_norm and layer_norm (vector-Jacobian products).
//
// Definitions: docs.rs nuvec-core 0.5.0, Enum FastOp, variants RmsNormVjp ("the
// gradients of RmsNorm for x and w") and LayerNormVjp ("... for x, w and b").
//   RmsNorm:   r = 1/sqrt(mean(x^2) + eps), y = x r w
//              dx_j = r w_j g_j - x_j r^3 (sum_k g_k w_k x_k) / D,  dw_j = sum_rows g_j x_j r
//   LayerNorm: xh = (x - mean) r, a = w g
//              dx_j = r (a_j - mean(a) - xh_j mean(a xh)),  dw_j = sum_rows g_j xh_j,
//              db_j = sum_rows g_j
//
// dx is row-local.  dw and db are column sums over all rows: kernel 1 runs a grid of
// `parts` CTAs, each walking rows blockIdx.x, blockIdx.x + parts, ... and keeping the
// float32 partial sums of its own columns in registers; it writes them to the caller's
// workspace [parts, D] (one slice per sum).  Kernel 2 adds the partials of each column
// in double, in a fixed order (deterministic), and rounds once to the I/O type.
//
// Precision: the row sums that feed a cancelling difference (sum g w x and the
// statistics) are accumulated in double from exact float32 products; the per-element
// difference is evaluated with fma against double-float row constants.  The float32
// rounding that remains is a small multiple of 2^-24 times the magnitude of the terms
// that cancel.
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

// Sum of two doubles across the CTA (one row per CTA); `buf` holds 2 x 32 doubles.
__device__ __forceinline__ void cta_sum2(double& a, double& b, double (*buf)[32]) {
    a = warp_sum(a);
    b = warp_sum(b);
    const int nw = blockDim.x >> 5;
    if (nw > 1) {
        if ((threadIdx.x & 31) == 0) {
            buf[0][threadIdx.x >> 5] = a;
            buf[1][threadIdx.x >> 5] = b;
        }
        __syncthreads();
        a = 0.0;
        b = 0.0;
        for (int i = 0; i < nw; ++i) {
            a += buf[0][i];
            b += buf[1][i];
        }
    }
}

__device__ __forceinline__ void split_f64(double v, float& hi, float& lo) {
    hi = __double2float_rn(v);
    lo = __double2float_rn(v - (double)hi);
}

// ---- RmsNormVjp, kernel 1 ---------------------------------------------------------------
template <typename T, int VPT>
__global__ void __launch_bounds__(512) rms_vjp_kernel(const VjpArgs a) {
    pdl_wait();
    pdl_release();
    using E = Elem<T>;
    constexpr int VEC = E::kVec;
    __shared__ double red[2][2][32];
    const int G = blockDim.x;
    const int t = threadIdx.x;
    const double invD = 1.0 / (double)a.D;

    V16 wv[VPT];
    float acc[VPT][VEC];
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
        const int v = t + k * G;
        wv[k] = (a.w && v < a.nvec) ? ld_param(static_cast<const char*>(a.w) + (size_t)v * 16)
                                    : ones_vec<T>();
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[k][e] = 0.f;
    }

    int it = 0;
    for (int64_t row = blockIdx.x; row < a.rows; row += a.parts, ++it) {
        const size_t roff = (size_t)row * (size_t)a.nvec * 16;
        V16 xv[VPT], gv[VPT];
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = t + k * G;
            const bool in = v < a.nvec;
            xv[k] = in ? ld_stream(static_cast<const char*>(a.x) + roff + (size_t)v * 16) : zeros_vec<T>();
            gv[k] = in ? ld_stream(static_cast<const char*>(a.g) + roff + (size_t)v * 16) : zeros_vec<T>();
        }
        // sum x^2 (the scale) and sum g w x (the projection), both in double; g w x is
        // an exact float32 product for bfloat16 data
        double ss = 0.0, c = 0.0;
#pragma unroll
        for (int k = 0; k < VPT; ++k)
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                const float xf = E::get(xv[k], e);
                ss += (double)__fmul_rn(xf, xf);
                c += (double)__fmul_rn(__fmul_rn(E::get(gv[k], e), E::get(wv[k], e)), xf);
            }
        cta_sum2(ss, c, red[it & 1]);
        const double r = rsqrt(ss * invD + (double)a.eps);
        float v_hi, v_lo;
        split_f64(r * r * c * invD, v_hi, v_lo);
        const float rf = __double2float_rn(r);
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
                        float tt = __fmaf_rn(-xf, v_hi, u);   // u - x v, v = v_hi + v_lo
                        tt = __fmaf_rn(-xf, v_lo, tt);
                        d[q] = __fmul_rn(rf, tt);
                        acc[k][e + q] = __fmaf_rn(__fmul_rn(gf, xf), rf, acc[k][e + q]);
                    }
                    E::put2(o, e, d[0], d[1]);
                }
                st_stream(static_cast<char*>(a.dx) + roff + (size_t)v * 16, o);
            }
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
__global__ void __launch_bounds__(512) layer_vjp_kernel(const VjpArgs a) {
    pdl_wait();
    pdl_release();
    using E = Elem<T>;
    constexpr int VEC = E::kVec;
    __shared__ double red[4][2][32];
    const int G = blockDim.x;
    const int t = threadIdx.x;
    const double invD = 1.0 / (double)a.D;

    V16 wv[VPT];
    float accw[VPT][VEC], accb[VPT][VEC];
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
        const int v = t + k * G;
        wv[k] = (a.w && v < a.nvec) ? ld_param(static_cast<const char*>(a.w) + (size_t)v * 16)
                                    : ones_vec<T>();
#pragma unroll
        for (int e = 0; e < VEC; ++e) accw[k][e] = accb[k][e] = 0.f;
    }

    int it = 0;
    for (int64_t row = blockIdx.x; row < a.rows; row += a.parts, ++it) {
        const size_t roff = (size_t)row * (size_t)a.nvec * 16;
        V16 xv[VPT], gv[VPT];
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = t + k * G;
            const bool in = v < a.nvec;
            xv[k] = in ? ld_stream(static_cast<const char*>(a.x) + roff + (size_t)v * 16) : zeros_vec<T>();
            gv[k] = in ? ld_stream(static_cast<const char*>(a.g) + roff + (size_t)v * 16) : zeros_vec<T>();
        }
        // statistics: sum x, sum x^2; projections: sum a, sum a x (a = w g); all double,
        // from exact float32 products for bfloat16 data
        double s1 = 0.0, s2 = 0.0, sa = 0.0, sax = 0.0;
#pragma unroll
        for (int k = 0; k < VPT; ++k)
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                const float xf = E::get(xv[k], e);
                const float af = __fmul_rn(E::get(wv[k], e), E::get(gv[k], e));
                const double xd = (double)xf;
                s1 += xd;
                s2 = fma(xd, xd, s2);
                sa += (double)af;
                sax = fma((double)af, xd, sax);
            }
        cta_sum2(s1, s2, red[(it & 1) * 2]);
        cta_sum2(sa, sax, red[(it & 1) * 2 + 1]);
        const double mean = s1 * invD;
        const double var = fmax(s2 * invD - mean * mean, 0.0);
        const double r = rsqrt(var + (double)a.eps);
        // dx = r (a - C - x K) with K = r^2 (sum a x - mean sum a) / D, C = sum a / D - mean K
        const double K = r * r * (sax - mean * sa) * invD;
        const double C = sa * invD - mean * K;
        float K_hi, K_lo, C_hi, C_lo;
        split_f64(K, K_hi, K_lo);
        split_f64(C, C_hi, C_lo);
        const float rf = __double2float_rn(r);
        const float mf = __double2float_rn(mean);
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
                        const float af = __fmul_rn(E::get(wv[k], e + q), gf);
                        float tt = __fmaf_rn(-xf, K_hi, af);
                        tt = __fsub_rn(tt, C_hi);
                        tt = __fmaf_rn(-xf, K_lo, tt);
                        tt = __fsub_rn(tt, C_lo);
                        d[q] = __fmul_rn(rf, tt);
                        const float xh = __fmul_rn(__fsub_rn(xf, mf), rf);
                        accw[k][e + q] = __fmaf_rn(gf, xh, accw[k][e + q]);
                        accb[k][e + q] = __fadd_rn(accb[k][e + q], gf);
                    }
                    E::put2(o, e, d[0], d[1]);
                }
                st_stream(static_cast<char*>(a.dx) + roff + (size_t)v * 16, o);
            }
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
// out[j] = sum_{p < parts} part[p][j], added in double in the order p = 0, 1, ...
template <typename T>
__global__ void __launch_bounds__(256) vjp_reduce_kernel(const float* part, int parts, int D,
                                                         void* out) {
    pdl_wait();
    pdl_release();
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= D) return;
    double s = 0.0;
    for (int p = 0; p < parts; ++p) s += (double)part[(size_t)p * D + j];
    Elem<T>::store1(out, j, __double2float_rn(s));
}

}  // namespace nvn
