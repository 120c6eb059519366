// layer.cuh -- layer_norm kernels.
//
// Definition: docs.rs nuvec-core 0.5.0, Enum FastOp, variant LayerNorm:
// y = (x - mean) / sqrt(var + eps) * w + b over the last axis, w and b 1-D or the
// scalars 1 and 0; var is the population variance.
//
// Precision: the output y = a + b with a = (x - mean) * rstd * w can cancel (a close
// to -b).  A float32 error in mean or rstd is an absolute error of about 2^-24 |a| in
// y, which exceeds half a bfloat16 ulp of y whenever |y| < 2^-15 |a|: thousands of
// elements of a [16384, 8192] batch.  So the statistics (sum, centred sum of
// squares) and the output are formed in double precision; only the final value is
// rounded to the I/O type.
#pragma once

#include "common.cuh"
#include "rms.cuh"

namespace nvn {

template <typename T>
__device__ __forceinline__ void store_out(void* p, int64_t i, double v);

template <>
__device__ __forceinline__ void store_out<float>(void* p, int64_t i, double v) {
    static_cast<float*>(p)[i] = __double2float_rn(v);
}
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(void* p, int64_t i, double v) {
    static_cast<__nv_bfloat16*>(p)[i] = __double2bfloat16(v);
}

// Pack two doubles into the I/O vector at elements e, e + 1 (each rounded once).
template <typename T>
__device__ __forceinline__ void put2_f64(V16& v, int e, double a, double b);

template <>
__device__ __forceinline__ void put2_f64<float>(V16& v, int e, double a, double b) {
    v.u[e] = __float_as_uint(__double2float_rn(a));
    v.u[e + 1] = __float_as_uint(__double2float_rn(b));
}
template <>
__device__ __forceinline__ void put2_f64<__nv_bfloat16>(V16& v, int e, double a, double b) {
    const __nv_bfloat16 lo = __double2bfloat16(a);
    const __nv_bfloat16 hi = __double2bfloat16(b);
    v.u[e >> 1] = (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
}

// Sum of a double across the row's G threads (G a multiple of 32).
__device__ __forceinline__ double row_sum_f64(double v, double* buf, int slot, int wpr) {
    v = warp_sum(v);
    if (wpr > 1) {
        if ((threadIdx.x & 31) == 0) buf[threadIdx.x >> 5] = v;
        __syncthreads();
        v = 0.0;
        const int w0 = slot * wpr;
        for (int i = 0; i < wpr; ++i) v += buf[w0 + i];
    }
    return v;
}

// ---- register path ------------------------------------------------------------------
template <typename T, int VPT>
__global__ void __launch_bounds__(layer_max_threads(VPT)) layer_rows_kernel(const RowArgs a) {
    pdl_wait();
    pdl_release();
    using E = Elem<T>;
    constexpr int VEC = E::kVec;
    const int G = a.G;
    const int slot = threadIdx.x / G;
    const int t = threadIdx.x - slot * G;
    const int wpr = G >> 5;
    // four buffers: (mean, variance) x iteration parity
    __shared__ double red[4][32];

    V16 wv[VPT], bv[VPT];
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
        const int v = t + k * G;
        const bool in = v < a.nvec;
        wv[k] = (a.w != nullptr && in) ? ld_param(static_cast<const char*>(a.w) + (size_t)v * 16)
                                       : ones_vec<T>();
        bv[k] = (a.b != nullptr && in) ? ld_param(static_cast<const char*>(a.b) + (size_t)v * 16)
                                       : zeros_vec<T>();
    }
    const double Dd = (double)a.D;
    const double eps = (double)a.eps;

    int it = 0;
    for (int64_t base = (int64_t)blockIdx.x * a.rows_per_cta; base < a.rows;
         base += (int64_t)gridDim.x * a.rows_per_cta, ++it) {
        const int64_t row = base + slot;
        const bool active = row < a.rows;
        const size_t roff = (size_t)row * (size_t)a.D * sizeof(T);

        V16 xv[VPT];
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = t + k * G;
            if (active && v < a.nvec)
                xv[k] = ld_stream(static_cast<const char*>(a.x) + roff + (size_t)v * 16);
        }

        double s1 = 0.0;
#pragma unroll
        for (int k = 0; k < VPT; ++k)
            if (active && t + k * G < a.nvec)
#pragma unroll
                for (int e = 0; e < VEC; ++e) s1 += (double)E::get(xv[k], e);
        const double mean = row_sum_f64(s1, red[(it & 1) * 2], slot, wpr) / Dd;

        double s2 = 0.0;
#pragma unroll
        for (int k = 0; k < VPT; ++k)
            if (active && t + k * G < a.nvec)
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    const double d = (double)E::get(xv[k], e) - mean;
                    s2 = fma(d, d, s2);
                }
        const double var = row_sum_f64(s2, red[(it & 1) * 2 + 1], slot, wpr) / Dd;
        const double rstd = 1.0 / sqrt(var + eps);

#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = t + k * G;
            if (active && v < a.nvec) {
                V16 o;
#pragma unroll
                for (int e = 0; e < VEC; e += 2) {
                    const double d0 = (double)E::get(xv[k], e) - mean;
                    const double d1 = (double)E::get(xv[k], e + 1) - mean;
                    const double y0 = fma(d0, rstd * (double)E::get(wv[k], e), (double)E::get(bv[k], e));
                    const double y1 =
                        fma(d1, rstd * (double)E::get(wv[k], e + 1), (double)E::get(bv[k], e + 1));
                    put2_f64<T>(o, e, y0, y1);
                }
                st_stream(static_cast<char*>(a.y) + roff + (size_t)v * 16, o);
            }
        }
    }
}

// ---- generic path ---------------------------------------------------------------------
// Any D and alignment: one CTA per row; three scalar passes over the row (sum, centred
// sum of squares, output).  y may be x: each thread reads index j in every pass before
// it writes index j in the last one.
template <typename T>
__global__ void __launch_bounds__(256) layer_generic_kernel(const RowArgs a) {
    pdl_wait();
    pdl_release();
    using E = Elem<T>;
    __shared__ double red[4][32];
    const int wpr = blockDim.x >> 5;
    int it = 0;
    for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x, ++it) {
        const int64_t r0 = row * (int64_t)a.D;
        double s1 = 0.0;
        for (int j = threadIdx.x; j < a.D; j += blockDim.x) s1 += (double)E::load1(a.x, r0 + j);
        const double mean = row_sum_f64(s1, red[(it & 1) * 2], 0, wpr) / (double)a.D;
        double s2 = 0.0;
        for (int j = threadIdx.x; j < a.D; j += blockDim.x) {
            const double d = (double)E::load1(a.x, r0 + j) - mean;
            s2 = fma(d, d, s2);
        }
        const double var = row_sum_f64(s2, red[(it & 1) * 2 + 1], 0, wpr) / (double)a.D;
        const double rstd = 1.0 / sqrt(var + (double)a.eps);
        for (int j = threadIdx.x; j < a.D; j += blockDim.x) {
            const double d = (double)E::load1(a.x, r0 + j) - mean;
            const double wj = a.w ? (double)E::load1(a.w, j) : 1.0;
            const double bj = a.b ? (double)E::load1(a.b, j) : 0.0;
            store_out<T>(a.y, r0 + j, fma(d, rstd * wj, bj));
        }
    }
}

}  // namespace nvn
