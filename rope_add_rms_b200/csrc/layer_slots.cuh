// layer_slots.cuh -- bfloat16 layer_norm with the row in registers, several rows per CTA
// sharing one float32 table of w and b in shared memory.
//
// Definition: docs.rs nuvec-core 0.5.0, Enum FastOp, variant LayerNorm:
// y = (x - mean) / sqrt(var + eps) * w + b over the last axis, population variance.
//
// The arithmetic is that of layer_rows_kernel (layer.cuh): double statistics from one
// widening per element, a float32 output with the per-vector error test, and a double
// recomputation of the rare vectors that fail it.  What changes is the instruction count per
// element, which bounds that kernel (about 20 lane instructions per element, half of them
// unpacking bfloat16 pairs into float32 registers):
//   - x is never unpacked: sm_100 converts a bfloat16 half of a register straight to double
//     (cvt.f64.bf16) for the statistics, and its mixed-precision fma (fma.rn.f32.bf16,
//     bfloat16 factors, float32 addend and result) forms d = x - mean_hi in one rounding
//     from the packed register, as the float32 subtraction did;
//   - w and b are read as float32 from a table in shared memory, filled once per CTA and
//     shared by the CTA's row slots (16-byte words, word q of every vector contiguous, so
//     the lanes of a warp read consecutive words);
//   - a CTA holds `slots` rows at a time (G threads each); a row's cross-warp reduction
//     uses a named barrier of its slot alone, and rows narrower than a warp (G = 2, 4, 8 or
//     16) share warps, reducing over their own lanes;
//   - prefetching form (PREFETCH): once a row's loads have landed (after its warp sums, before
//     the cross-warp step), one thread of the slot asks L2 for the slot's next row
//     (cp.async.bulk.prefetch.L2, one bulk prefetch of the whole row from this GPU's own
//     memory; no shared memory, no registers, nothing to wait on), so that row's loads find
//     it in L2 instead of waiting on DRAM.  Issued at the start of the row instead, the
//     prefetch competed with that row's own loads: bf16 [16384, 8192] 98.7 against 95.6 us,
//     [8192, 16384] 105.9 against 99.9 us.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "layer.cuh"

namespace nvn {

// The statistics of a bfloat16 pair: both halves widened to double and accumulated at once
// (s1 += lo, s1b += hi, s2 += lo^2, s2b += hi^2), in one block so that each conversion is
// consumed where it is made.
__device__ __forceinline__ void bf16x2_stats(uint32_t u, double& s1, double& s1b, double& s2,
                                             double& s2b) {
    asm("{\n\t.reg .b16 l, h;\n\t.reg .f64 a, b;\n\tmov.b32 {l, h}, %4;\n\t"
        "cvt.f64.bf16 a, l;\n\tcvt.f64.bf16 b, h;\n\t"
        "add.rn.f64 %0, %0, a;\n\tadd.rn.f64 %1, %1, b;\n\t"
        "fma.rn.f64 %2, a, a, %2;\n\tfma.rn.f64 %3, b, b, %3;\n}"
        : "+d"(s1), "+d"(s1b), "+d"(s2), "+d"(s2b)
        : "r"(u));
}

// The centred square sum of a bfloat16 pair: c2 += (lo - m)^2 + (hi - m)^2 in double.
__device__ __forceinline__ void bf16x2_centred(uint32_t u, double m, double& c2) {
    asm("{\n\t.reg .b16 l, h;\n\t.reg .f64 a, b;\n\tmov.b32 {l, h}, %1;\n\t"
        "cvt.f64.bf16 a, l;\n\tcvt.f64.bf16 b, h;\n\t"
        "sub.rn.f64 a, a, %2;\n\tsub.rn.f64 b, b, %2;\n\t"
        "fma.rn.f64 %0, a, a, %0;\n\tfma.rn.f64 %0, b, b, %0;\n}"
        : "+d"(c2)
        : "r"(u), "d"(m));
}

// (lo - m, hi - m) for the bfloat16 halves of u, each the float32 difference rounded once:
// fma with the bfloat16 factor 1 (0x3F80).
__device__ __forceinline__ float2 bf16x2_minus(uint32_t u, float m) {
    float lo, hi;
    asm("{\n\t.reg .b16 l, h, one;\n\tmov.b32 {l, h}, %2;\n\tmov.b16 one, 0x3F80;\n\t"
        "fma.rn.f32.bf16 %0, l, one, %3;\n\tfma.rn.f32.bf16 %1, h, one, %3;\n}"
        : "=f"(lo), "=f"(hi)
        : "r"(u), "f"(-m));
    return make_float2(lo, hi);
}

__device__ __forceinline__ void slot_bar(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Bytes of dynamic shared memory: the table (nvec vectors x 8 elements x (w, b) float32).
__host__ __device__ constexpr size_t slots_table_bytes(int nvec) {
    return (size_t)nvec * 8u * 2u * sizeof(float);
}
// CTA sizes the kernel is built for: 768 threads (24 warps, up to 80 registers) and 1024
// (32 warps, up to 64 registers).
constexpr int kSlotsMaxThreads = 1024;

// Launch: blockDim.x = a.G * a.rows_per_cta, a multiple of 32 (rows_per_cta = slots <= 15
// when G > 32; G a multiple of 32 or a power of two up to 16),
// dynamic shared memory = slots_table_bytes(a.nvec); persistent grid.
// NARROW: G < 32, several rows to a warp (slot-width sums, a warp-wide vote for the
// centred pass).  The wide form keeps plain warp sums: compiled into one kernel, the narrow
// code cost the wide rows 3 % on bf16 [16384, 8192].
template <int VPT, bool PREFETCH, int MAXT, bool NARROW = false>
__global__ void __launch_bounds__(MAXT, 1) layer_slots_kernel(const RowArgs a) {
    pdl_wait();
    pdl_release();
    using T = __nv_bfloat16;
    using E = Elem<T>;
    constexpr int VEC = 8;
    extern __shared__ float4 tab[];  // [4][nvec]: w 0-3, w 4-7, b 0-3, b 4-7
    __shared__ double red[2][MAXT / 32][3];

    const int G = a.G;
    const int slots = a.rows_per_cta;
    const int slot = threadIdx.x / G;
    const int t = threadIdx.x - slot * G;
    const int wpr = G >> 5;
    const int gw = G < 32 ? G : 32;  // lanes of a row within a warp
    const int warp = threadIdx.x >> 5;
    const int nvec = a.nvec;
    const uint32_t row_bytes = (uint32_t)nvec * 16u;
    const int64_t row_step = (int64_t)gridDim.x * slots;

    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
        const V16 wv = a.w ? ld_param(static_cast<const char*>(a.w) + (size_t)v * 16) : ones_vec<T>();
        const V16 bv = a.b ? ld_param(static_cast<const char*>(a.b) + (size_t)v * 16) : zeros_vec<T>();
        tab[v] = make_float4(E::get(wv, 0), E::get(wv, 1), E::get(wv, 2), E::get(wv, 3));
        tab[nvec + v] = make_float4(E::get(wv, 4), E::get(wv, 5), E::get(wv, 6), E::get(wv, 7));
        tab[2 * nvec + v] = make_float4(E::get(bv, 0), E::get(bv, 1), E::get(bv, 2), E::get(bv, 3));
        tab[3 * nvec + v] = make_float4(E::get(bv, 4), E::get(bv, 5), E::get(bv, 6), E::get(bv, 7));
    }
    __syncthreads();

    // the largest |w| and 2^-11 |b| over this thread's columns (bounds of the error test)
    float wmax = 0.f, bmax = 0.f;
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
        const int v = t + k * G;
        if (v < nvec) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const float4 w4 = tab[q * nvec + v], b4 = tab[(2 + q) * nvec + v];
                wmax = fmaxf(wmax, fmaxf(fmaxf(fabsf(w4.x), fabsf(w4.y)), fmaxf(fabsf(w4.z), fabsf(w4.w))));
                bmax = fmaxf(bmax, fmaxf(fmaxf(fabsf(b4.x), fabsf(b4.y)), fmaxf(fabsf(b4.z), fabsf(b4.w))));
            }
        }
    }
    bmax *= 0x1p-11f;

    const double invD = 1.0 / (double)a.D;
    const double eps = (double)a.eps;
    const int bar_id = 1 + slot;
    int it = 0;
    for (int64_t base = (int64_t)blockIdx.x * slots; base < a.rows;
         base += (int64_t)gridDim.x * slots, ++it) {
        const int64_t row = base + slot;
        const bool active = row < a.rows;
        const char* xrow = static_cast<const char*>(a.x) + (size_t)row * (size_t)nvec * 16;
        char* yrow = static_cast<char*>(a.y) + (size_t)row * (size_t)nvec * 16;

        V16 xv[VPT];
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = t + k * G;
            xv[k] = (active && v < nvec) ? ld_stream(xrow + (size_t)v * 16) : zeros_vec<T>();
        }
        // eight accumulator chains (two sets of four, alternating by word): the double
        // adds are latency-bound chains, so more of them run side by side
        double s1 = 0.0, s2 = 0.0, s1b = 0.0, s2b = 0.0;
        double t1 = 0.0, t2 = 0.0, t1b = 0.0, t2b = 0.0;
#pragma unroll
        for (int k = 0; k < VPT; ++k)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                if (q & 1)
                    bf16x2_stats(xv[k].u[q], t1, t1b, t2, t2b);
                else
                    bf16x2_stats(xv[k].u[q], s1, s1b, s2, s2b);
            }
        if constexpr (NARROW) {
            s1 = group_sum((s1 + s1b) + (t1 + t1b), gw);
            s2 = group_sum((s2 + s2b) + (t2 + t2b), gw);
        } else {
            s1 = warp_sum((s1 + s1b) + (t1 + t1b));
            s2 = warp_sum((s2 + s2b) + (t2 + t2b));
        }
        // the row's loads have landed: ask L2 for the slot's next row (see the header)
        if constexpr (PREFETCH) {
            if (t == 0 && row + row_step < a.rows)
                prefetch_l2(static_cast<const char*>(a.x) + (size_t)(row + row_step) * row_bytes,
                            row_bytes);
        }
        double(*rb)[3] = red[it & 1];
        if (wpr > 1) {
            if ((threadIdx.x & 31) == 0) {
                rb[warp][0] = s1;
                rb[warp][1] = s2;
            }
            slot_bar(bar_id, G);
            s1 = 0.0;
            s2 = 0.0;
            for (int i = 0; i < wpr; ++i) {
                s1 += rb[slot * wpr + i][0];
                s2 += rb[slot * wpr + i][1];
            }
        }
        const double mean = s1 * invD;
        double var = s2 * invD - mean * mean;
        // centred second pass: uniform over a slot, and for slots narrower than a warp
        // taken by the whole warp when any of its slots needs it (its shuffles are
        // warp-wide), each slot keeping its own result only if it asked for it
        const bool centre = !(var > ldexp(mean * mean, -20));
        bool centre_warp = centre;
        if constexpr (NARROW) centre_warp = __any_sync(0xFFFFFFFFu, centre);
        if (centre_warp) {
            // centred second pass (uniform over the slot's threads)
            double c2 = 0.0;
#pragma unroll
            for (int k = 0; k < VPT; ++k)
                if (t + k * G < nvec)
#pragma unroll
                    for (int q = 0; q < 4; ++q) bf16x2_centred(xv[k].u[q], mean, c2);
            if constexpr (NARROW)
                c2 = group_sum(c2, gw);
            else
                c2 = warp_sum(c2);
            if (wpr > 1) {
                if ((threadIdx.x & 31) == 0) rb[warp][2] = c2;
                slot_bar(bar_id, G);
                c2 = 0.0;
                for (int i = 0; i < wpr; ++i) c2 += rb[slot * wpr + i][2];
            }
            if (centre) var = c2 * invD;
        }
        const double rstd = rsqrt(var + eps);
        const float mu_hi = __double2float_rn(mean);
        const float mu_lo = __double2float_rn(mean - (double)mu_hi);
        const float rf = __double2float_rn(rstd);
        const bool two_sub = 0x1p10f * fabsf(mu_lo) * rf > 0x1p-16f;
        const float kmu = two_sub ? 0x1p-37f * fabsf(mu_hi) : 0x1p10f * fabsf(mu_lo);
        const float2 rf2 = make_float2(rf, rf);
        const float2 nlo2 = make_float2(-mu_lo, -mu_lo);  // used when two_sub
        const float tmax = __fmaf_rn(__fmul_rn(kmu, rf), wmax, bmax);

        // the table offset of this thread's columns, opaque to the compiler on every row so
        // that it reloads w and b from shared memory per row instead of keeping all of them
        // live in registers across the loop (which would spill)
        int t_row = t;
        asm volatile("" : "+r"(t_row));
        auto output = [&](auto two) {
            constexpr bool TWO = decltype(two)::value;
#pragma unroll
            for (int k = 0; k < VPT; ++k) {
                const int v = t_row + k * G;
                if (active && v < nvec) {
                    V16 o;
                    float ymin = INFINITY;
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const float4 w4 = tab[q * nvec + v], b4 = tab[(2 + q) * nvec + v];
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int wi = 2 * q + h;  // word of the vector: elements 2wi, 2wi+1
                            const float2 w2 = h ? make_float2(w4.z, w4.w) : make_float2(w4.x, w4.y);
                            const float2 b2 = h ? make_float2(b4.z, b4.w) : make_float2(b4.x, b4.y);
                            float2 d2 = bf16x2_minus(xv[k].u[wi], mu_hi);
                            if (TWO) d2 = add2(d2, nlo2);
                            const float2 y2 = fma2(d2, mul2(rf2, w2), b2);
                            ymin = fminf(ymin, fminf(fabsf(y2.x), fabsf(y2.y)));
                            E::put2(o, 2 * wi, y2);
                        }
                    }
                    if (!(ymin > tmax)) {
                        // rare: recompute the vector in double from the exact mean
                        const float* tf = reinterpret_cast<const float*>(tab);
#pragma unroll
                        for (int e = 0; e < VEC; e += 2) {
                            const size_t wi = ((size_t)(e >> 2) * nvec + v) * 4 + (e & 3);
                            const size_t bi = wi + (size_t)8 * nvec;
                            const double y0 = fma((double)E::get(xv[k], e) - mean,
                                                  rstd * (double)tf[wi], (double)tf[bi]);
                            const double y1 = fma((double)E::get(xv[k], e + 1) - mean,
                                                  rstd * (double)tf[wi + 1], (double)tf[bi + 1]);
                            E::put2(o, e, __double2float_rn(y0), __double2float_rn(y1));
                        }
                    }
                    st_stream(yrow + (size_t)v * 16, o);
                }
            }
        };
        if (two_sub)
            output(std::true_type{});
        else
            output(std::false_type{});
    }
}

}  // namespace nvn
