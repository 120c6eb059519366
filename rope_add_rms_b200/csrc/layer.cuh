// layer.cuh -- layer_norm kernels.
//
// Definition: docs.rs nuvec-core 0.5.0, Enum FastOp, variant LayerNorm:
// y = (x - mean) / sqrt(var + eps) * w + b for every row (last axis), with the
// population variance; w and b are length-D vectors, or absent and standing for 1 and 0.
//
// Precision: the output y = a + b with a = (x - mean) * rstd * w can cancel (a close
// to -b).  A float32 error in mean or rstd is an absolute error of about 2^-24 |a| in
// y, which exceeds half a bfloat16 ulp of y whenever |y| < 2^-15 |a|: thousands of
// elements of a [16384, 8192] batch.  So the statistics (sum, centred sum of
// squares) and the output are formed in double precision; only the final value is
// rounded to the I/O type.
#pragma once

#include <type_traits>

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

// Recompute one output vector in double precision, y = (x - mean) * (rstd * w) + b,
// rounded (via float32) to the I/O type.  Called for the rare vectors holding an
// element that fails the float32 error test.
template <typename T>
__device__ __forceinline__ V16 layer_vector_f64(V16 xv, V16 wv, V16 bv, double mean, double rstd) {
    using E = Elem<T>;
    V16 o;
#pragma unroll 1
    for (int e = 0; e < E::kVec; e += 2) {
        const double y0 = fma((double)E::get(xv, e) - mean, rstd * (double)E::get(wv, e),
                              (double)E::get(bv, e));
        const double y1 = fma((double)E::get(xv, e + 1) - mean, rstd * (double)E::get(wv, e + 1),
                              (double)E::get(bv, e + 1));
        E::put2(o, e, __double2float_rn(y0), __double2float_rn(y1));
    }
    return o;
}

// ---- register path ------------------------------------------------------------------
// Conversions between float32 and double run at a quarter of the double-add rate on
// B200, so each element is widened once: the statistics are the double sums S1 = sum x
// and S2 = sum x^2 (exact for bfloat16 rows of ordinary range), var = S2/D - mean^2.
// When mean^2 > 2^20 var the one-pass form could lose bits, and the row (every thread
// of the CTA holds the same row, so the branch is CTA-uniform) redoes the centred sum
// sum (x - mean)^2 in double.
//
// The output is formed in float32 with A = rstd * w and y = fma(d, A, b), where d is
// x - mean_hi (one subtraction) or, for rows whose mean is large against their
// spread, (x - mean_hi) - mean_lo with mean = mean_hi + mean_lo.  d and A each carry
// at most ~2^-23 relative error, plus the absolute error of the mean kept, m = |mean_lo|
// (one subtraction) or 2^-48 |mean| (two); so the error of y is below
// 2^-22 |d A| + m |A| + 2^-24 |y|, and since |d A| <= |y| + |b| it stays under half a
// bfloat16 step (2^-9 |y|) whenever |y| > 2^-11 |b| + 2^10 m |A| (a factor-2 margin on
// each term).  The kernel tests a whole vector at once against the largest such bound
// over the thread's columns (|A| <= rstd max|w|, |b| <= max|b|): only a near
// cancellation of d A against b fails it -- about one vector in a thousand -- and those
// vectors are recomputed in double.
// MAXT bounds the CTA: 128 (256) lets the compiler keep the 8-vector form under 85
// registers, six (three) CTAs = 24 warps per SM -- measured 13 % faster on bf16
// [16384, 8192] than four CTAs at 128 registers; wider rows use 512 threads.
// NARROW: G < 32, several rows to a warp -- slot-width sums and a warp-wide vote for the
// centred pass, in their own instantiation so the wide rows keep plain warp sums.
template <typename T, int VPT, int MAXT = layer_max_threads(VPT), bool NARROW = false>
__global__ void __launch_bounds__(MAXT, MAXT <= 256 ? 768 / MAXT : 1)
    layer_rows_kernel(const RowArgs a) {
    pdl_wait();
    pdl_release();
    using E = Elem<T>;
    constexpr int VEC = E::kVec;
    const int G = a.G;
    const int slot = threadIdx.x / G;
    const int t = threadIdx.x - slot * G;
    const int wpr = G >> 5;
    // [parity][S1, S2][warp]; a row spanning several warps is alone in its CTA
    __shared__ double red[2][2][32];

    const double invD = 1.0 / (double)a.D;
    const double eps = (double)a.eps;
    constexpr bool kPRegs = weights_in_regs(VPT);
    V16 wv[VPT], bv[VPT];
    // largest |w| and 2^-11 |b| over this thread's columns: the per-vector error test
    // below bounds every element's test term by them
    float wmax = 0.f, bmax = 0.f;
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
        const int v = t + k * G;
        const bool in = v < a.nvec;
        wv[k] = (a.w && in) ? ld_param(static_cast<const char*>(a.w) + (size_t)v * 16) : ones_vec<T>();
        bv[k] = (a.b && in) ? ld_param(static_cast<const char*>(a.b) + (size_t)v * 16) : zeros_vec<T>();
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            wmax = fmaxf(wmax, fabsf(E::get(wv[k], e)));
            bmax = fmaxf(bmax, fabsf(E::get(bv[k], e)));
        }
    }
    bmax *= 0x1p-11f;

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
            xv[k] = (active && v < a.nvec)
                        ? ld_stream(static_cast<const char*>(a.x) + roff + (size_t)v * 16)
                        : zeros_vec<T>();
        }

        // two independent accumulator chains per sum
        double s1 = 0.0, s2 = 0.0, s1b = 0.0, s2b = 0.0;
#pragma unroll
        for (int k = 0; k < VPT; ++k)
#pragma unroll
            for (int e = 0; e < VEC; e += 2) {
                const double x0 = (double)E::get(xv[k], e);
                const double x1 = (double)E::get(xv[k], e + 1);
                s1 += x0;
                s1b += x1;
                s2 = fma(x0, x0, s2);
                s2b = fma(x1, x1, s2b);
            }
        s1 += s1b;
        s2 += s2b;
        if constexpr (NARROW) {
            s1 = group_sum(s1, G);
            s2 = group_sum(s2, G);
        } else {
            s1 = warp_sum(s1);
            s2 = warp_sum(s2);
        }
        // bfloat16: the row's loads have landed, so ask L2 for this slot's next row (one bulk
        // prefetch of the whole row from this GPU's own memory, nothing to wait on).
        // Measured: [65536, 1024] 70.3 -> 65.0 us, [131072, 512] 82.4 -> 72.1 us; float32
        // rows gain nothing ([65536, 1024] 95.4 -> 99.1 us) and go without.
        if constexpr (sizeof(T) == 2) {
            const int64_t next = row + (int64_t)gridDim.x * a.rows_per_cta;
            if (t == 0 && next < a.rows)
                prefetch_l2(static_cast<const char*>(a.x) + (size_t)next * (size_t)a.D * sizeof(T),
                            (uint32_t)((size_t)a.D * sizeof(T)));
        }
        if (wpr > 1) {
            double* b1 = red[it & 1][0];
            double* b2 = red[it & 1][1];
            if ((threadIdx.x & 31) == 0) {
                b1[threadIdx.x >> 5] = s1;
                b2[threadIdx.x >> 5] = s2;
            }
            __syncthreads();
            s1 = 0.0;
            s2 = 0.0;
            for (int i = 0; i < wpr; ++i) {
                s1 += b1[i];
                s2 += b2[i];
            }
        }
        const double mean = s1 * invD;
        double var = s2 * invD - mean * mean;
        // centred second pass: uniform over a row's threads, and with several rows to a warp
        // taken by the whole warp when any of its rows needs it (its shuffles are warp-wide),
        // each row keeping its own result only if it asked for it
        const bool centre = !(var > ldexp(mean * mean, -20));
        bool centre_warp = centre;
        if constexpr (NARROW) centre_warp = __any_sync(0xFFFFFFFFu, centre);
        if (centre_warp) {
            double c2 = 0.0;
#pragma unroll
            for (int k = 0; k < VPT; ++k)
                if (t + k * G < a.nvec)
#pragma unroll
                    for (int e = 0; e < VEC; ++e) {
                        const double dd = (double)E::get(xv[k], e) - mean;
                        c2 = fma(dd, dd, c2);
                    }
            if constexpr (NARROW)
                c2 = group_sum(c2, G);
            else
                c2 = warp_sum(c2);
            if (wpr > 1) {
                __syncthreads();  // every thread has read red[it & 1] above
                double* b1 = red[it & 1][0];
                if ((threadIdx.x & 31) == 0) b1[threadIdx.x >> 5] = c2;
                __syncthreads();
                c2 = 0.0;
                for (int i = 0; i < wpr; ++i) c2 += b1[i];
            }
            if (centre) var = c2 * invD;
        }
        const double rstd = rsqrt(var + eps);
        const float mu_hi = __double2float_rn(mean);
        const float mu_lo = __double2float_rn(mean - (double)mu_hi);
        const float rf = __double2float_rn(rstd);
        // d = x - mean_hi, and for rows whose mean is large against their spread
        // (two_sub) also - mean_lo; kmu is the matching mean-error term of the test
        const bool two_sub = 0x1p10f * fabsf(mu_lo) * rf > 0x1p-16f;
        const float kmu = two_sub ? 0x1p-37f * fabsf(mu_hi) : 0x1p10f * fabsf(mu_lo);
        const float2 rf2 = make_float2(rf, rf);
        const float2 nhi2 = make_float2(-mu_hi, -mu_hi);
        const float2 nlo2 = make_float2(-mu_lo, -mu_lo);  // used when two_sub
        // kmu |A| + 2^-11 |b| <= kmu rf wmax + bmax =: tmax for every element of the thread
        const float tmax = __fmaf_rn(__fmul_rn(kmu, rf), wmax, bmax);

        // the output loop, compiled twice: with the second subtraction of the mean
        // (two_sub) and without it, chosen once per row (CTA-uniform)
        auto output = [&](auto two) {
            constexpr bool TWO = decltype(two)::value;
#pragma unroll
            for (int k = 0; k < VPT; ++k) {
                const int v = t + k * G;
                if (active && v < a.nvec) {
                    if constexpr (!kPRegs) {
                        wv[k] = a.w ? ld_param(static_cast<const char*>(a.w) + (size_t)v * 16) : ones_vec<T>();
                        bv[k] = a.b ? ld_param(static_cast<const char*>(a.b) + (size_t)v * 16) : zeros_vec<T>();
                    }
                    V16 o;
                    float ymin = INFINITY;
#pragma unroll
                    for (int e = 0; e < VEC; e += 2) {
                        const float2 w2 = E::get2(wv[k], e);
                        const float2 b2 = E::get2(bv[k], e);
                        const float2 A2 = mul2(rf2, w2);
                        const float2 d2 = TWO ? add2(add2(E::get2(xv[k], e), nhi2), nlo2)
                                                  : add2(E::get2(xv[k], e), nhi2);
                        const float2 y2 = fma2(d2, A2, b2);
                        ymin = fminf(ymin, fminf(fabsf(y2.x), fabsf(y2.y)));
                        E::put2(o, e, y2);
                    }
                    // the vector passes when its smallest |y| clears the thread's bound (a NaN
                    // y is skipped by fminf and kept: the double form gives NaN too)
                    if (!(ymin > tmax)) o = layer_vector_f64<T>(xv[k], wv[k], bv[k], mean, rstd);
                    st_stream(static_cast<char*>(a.y) + roff + (size_t)v * 16, o);
                }
            }
        };
        if (two_sub)
            output(std::true_type{});
        else
            output(std::false_type{});
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
