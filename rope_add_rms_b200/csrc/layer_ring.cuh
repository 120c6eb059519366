// layer_ring.cuh -- layer_norm over a ring of shared-memory row stages, one row per group
// of warps.
//
// Definition: docs.rs nuvec-core 0.5.0, Enum FastOp, variant LayerNorm:
// y = (x - mean) / sqrt(var + eps) * w + b over the last axis, population variance.
//
// Why this shape.  The op reads x and writes y (two HBM streams) but needs, per element,
// a double-precision contribution to the row statistics (a near-cancelling output needs
// the exact mean, see layer.cuh) and a float32 output with an error test.  When the row
// lives in registers, a warp cannot load its next row while it reduces and writes the
// current one, so the bytes in flight per SM follow the compute phases.  Here:
//   - the CTA's rows stream through a ring of `stages` shared-memory buffers, each
//     filled by one plain 1-D bulk copy (cp.async.bulk, non-multicast, from this GPU's
//     own memory) completing on the stage's mbarrier; a stage is refilled with the row
//     `stages` places later as soon as the warps that read it are done, so rows keep
//     arriving while others are reduced;
//   - the CTA's warps form `groups` row groups of R warps; group g takes the CTA's rows
//     g, g + groups, ...; its row reduction uses a named barrier of the group alone (no
//     CTA-wide barrier in the loop), and the last of its warps to finish a row refills
//     that row's stage (an atomic count per stage, no waiting).  `stages` is a multiple of
//     `groups`, so row k's stage k mod stages belongs to group k mod groups alone and the
//     group waits on each of its stages' phases in order (a parity wait never sees an
//     older phase meant for someone else);
//   - w and b are unpacked once per CTA into a float32 table in shared memory, laid out
//     so the lanes of a warp read consecutive 16-byte words (no bank conflicts), so no
//     per-element conversion of w or b remains (rows wider than the table read w and b
//     from global memory, L1-resident, in the I/O type).
// Arithmetic per element: the statistics widen x once to double (S1 = sum x,
// S2 = sum x^2, double sums), the output is packed float32 with the error test of
// layer.cuh, and vectors failing the test are recomputed in double from the exact mean.
//
// Every wait on a stage's mbarrier is bounded (~1 s).  If it runs out, the group learns it
// at its row barrier (a reducing barrier over the group), counts a fault and stops; the
// other groups then wait at most as long for the rows it no longer refills and stop too;
// at the end one thread waits (bounded) for the copies still in flight before the CTA
// exits.  A correct launch never gets there: every stage receives exactly the bytes its
// barrier expects.
#pragma once

#include "common.cuh"
#include "layer.cuh"
#include "staged.cuh"

namespace nvn {

struct RingArgs {
    int R;        // warps per row group
    int groups;   // row groups per CTA
    int stages;   // ring buffers (rows resident in shared memory): a multiple of groups,
                  // at least 2 x groups, so that each buffer serves one group
    int wb_smem;  // 1: w and b as a float32 table in shared memory
};

// Dynamic shared memory: [stages x row_bytes][table: w and b of each 16-byte vector as
// float32, in 16-byte words (bf16: w 0-3, w 4-7, b 0-3, b 4-7; float32: w, b), word q of
// every vector contiguous][mbarriers: stages x 8][last row issued per stage: stages x 8]
// [warps done per stage: stages x 4][reduction: groups x 2 x R x 3 doubles][fault flag]
__host__ __device__ inline size_t ring_table_bytes(int nvec, int vec_elems) {
    return (size_t)nvec * (size_t)vec_elems * 2u * sizeof(float);
}
__host__ __device__ inline size_t ring_smem_bytes(int nvec, int vec_elems, const RingArgs& r) {
    const size_t row = (size_t)nvec * 16u;
    size_t b = (size_t)r.stages * row;
    if (r.wb_smem) b += ring_table_bytes(nvec, vec_elems);
    b += (size_t)r.stages * 16u + (size_t)r.stages * 4u;
    b = (b + 7u) & ~(size_t)7u;
    b += (size_t)r.groups * 2u * (size_t)r.R * 3u * sizeof(double);
    b += 16u;
    return b;
}

__device__ __forceinline__ void named_bar(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Barrier over `nthreads` threads that also ORs a predicate across them.
__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool pred) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %3, 0;\n\t"
        "bar.red.or.pred q, %1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n}"
        : "=r"(out)
        : "r"(id), "r"(nthreads), "r"((uint32_t)pred)
        : "memory");
    return out != 0;
}

// w and b of vector v as float32 (wf[0..VEC), bf[0..VEC)), from the table or from global
// memory.
template <typename T, bool WB>
__device__ __forceinline__ void ring_wb(const RowArgs& a, const float* table, int nvec, int v,
                                        float* wf, float* bf) {
    using E = Elem<T>;
    constexpr int VEC = E::kVec;
    if constexpr (WB) {
        // four 16-byte words per vector of bf16 (w 0-3, w 4-7, b 0-3, b 4-7); for float32
        // vectors two (w 0-3, b 0-3)
        constexpr int Q = VEC / 4;  // words of w per vector
#pragma unroll
        for (int q = 0; q < Q; ++q) {
            const float4 wq = reinterpret_cast<const float4*>(table)[(size_t)q * nvec + v];
            const float4 bq = reinterpret_cast<const float4*>(table)[(size_t)(Q + q) * nvec + v];
            wf[4 * q + 0] = wq.x; wf[4 * q + 1] = wq.y; wf[4 * q + 2] = wq.z; wf[4 * q + 3] = wq.w;
            bf[4 * q + 0] = bq.x; bf[4 * q + 1] = bq.y; bf[4 * q + 2] = bq.z; bf[4 * q + 3] = bq.w;
        }
    } else {
        const V16 wv = a.w ? ld_param(static_cast<const char*>(a.w) + (size_t)v * 16) : ones_vec<T>();
        const V16 bv = a.b ? ld_param(static_cast<const char*>(a.b) + (size_t)v * 16) : zeros_vec<T>();
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            wf[e] = E::get(wv, e);
            bf[e] = E::get(bv, e);
        }
    }
}

// One output vector recomputed in double from the exact mean and rstd:
// y = (x - mean) * (rstd * w) + b, rounded once (via float32) to the I/O type.  Rare (a
// near cancellation), so kept out of line.
template <typename T, bool WB>
__device__ __noinline__ V16 ring_vector_f64(V16 xv, const RowArgs& a, const float* table,
                                            int nvec, int v, double mean, double rstd) {
    using E = Elem<T>;
    float wf[E::kVec], bf[E::kVec];
    ring_wb<T, WB>(a, table, nvec, v, wf, bf);
    V16 o;
#pragma unroll
    for (int e = 0; e < E::kVec; e += 2) {
        const double y0 =
            fma((double)E::get(xv, e) - mean, rstd * (double)wf[e], (double)bf[e]);
        const double y1 =
            fma((double)E::get(xv, e + 1) - mean, rstd * (double)wf[e + 1], (double)bf[e + 1]);
        E::put2(o, e, __double2float_rn(y0), __double2float_rn(y1));
    }
    return o;
}

template <typename T, bool WB>
__global__ void __launch_bounds__(512) layer_ring_kernel(const RowArgs a, const RingArgs rg) {
    pdl_wait();
    pdl_release();
    using E = Elem<T>;
    constexpr int VEC = E::kVec;
    extern __shared__ __align__(128) unsigned char smem[];

    const int R = rg.R, NG = rg.groups, S = rg.stages;
    const int nvec = a.nvec;
    const uint32_t row_bytes = (uint32_t)nvec * 16u;
    unsigned char* stage0 = smem;
    float* table = reinterpret_cast<float*>(smem + (size_t)S * row_bytes);
    unsigned char* tail = smem + (size_t)S * row_bytes + (WB ? ring_table_bytes(nvec, VEC) : 0);
    const uint32_t bar0 = smem_addr(tail);
    long long* last_issued = reinterpret_cast<long long*>(tail + (size_t)S * 8u);
    int* counts = reinterpret_cast<int*>(tail + (size_t)S * 16u);
    double* red = reinterpret_cast<double*>(
        smem + (((size_t)(tail - smem) + (size_t)S * 20u + 7u) & ~(size_t)7u));
    int* faulted = reinterpret_cast<int*>(red + (size_t)NG * 2 * R * 3);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = warp / R, wg = warp - g * R;
    const int GT = 32 * R;            // threads of a row group
    const int t = wg * 32 + lane;     // thread within the group
    const int64_t first = blockIdx.x, stride = gridDim.x;
    const int64_t nmine = first < a.rows ? (a.rows - 1 - first) / stride + 1 : 0;

    auto issue = [&](int64_t k) {
        const int s = (int)(k % S);
        const uint32_t bar = bar0 + 8u * (uint32_t)s;
        last_issued[s] = k;
        mbar_arrive_expect_tx(bar, row_bytes);
        bulk_load(smem_addr(stage0 + (size_t)s * row_bytes),
                  static_cast<const char*>(a.x) + (size_t)(first + k * stride) * row_bytes, row_bytes,
                  bar);
    };
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(bar0 + 8u * (uint32_t)s, 1);
            counts[s] = 0;
            last_issued[s] = -1;
        }
        *faulted = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
        for (int64_t k = 0; k < nmine && k < S; ++k) issue(k);
    }
    // the float32 table of w and b (while the first copies are in flight)
    if constexpr (WB) {
        constexpr int Q = VEC / 4;
        for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
            const V16 wv = a.w ? ld_param(static_cast<const char*>(a.w) + (size_t)v * 16) : ones_vec<T>();
            const V16 bv = a.b ? ld_param(static_cast<const char*>(a.b) + (size_t)v * 16) : zeros_vec<T>();
#pragma unroll
            for (int q = 0; q < Q; ++q) {
                reinterpret_cast<float4*>(table)[(size_t)q * nvec + v] =
                    make_float4(E::get(wv, 4 * q), E::get(wv, 4 * q + 1), E::get(wv, 4 * q + 2),
                                E::get(wv, 4 * q + 3));
                reinterpret_cast<float4*>(table)[(size_t)(Q + q) * nvec + v] =
                    make_float4(E::get(bv, 4 * q), E::get(bv, 4 * q + 1), E::get(bv, 4 * q + 2),
                                E::get(bv, 4 * q + 3));
            }
        }
    }
    __syncthreads();

    // the largest |w| and 2^-11 |b| over this thread's columns (bounds of the error test)
    float wmax = 0.f, bmax = 0.f;
    for (int v = t; v < nvec; v += GT) {
        float wf[VEC], bf[VEC];
        ring_wb<T, WB>(a, table, nvec, v, wf, bf);
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            wmax = fmaxf(wmax, fabsf(wf[e]));
            bmax = fmaxf(bmax, fabsf(bf[e]));
        }
    }
    bmax *= 0x1p-11f;

    const double invD = 1.0 / (double)a.D;
    const double eps = (double)a.eps;
    const int bar_id = 1 + g;
    bool bad = false;
    int j = 0;  // rows done by this group
    for (int64_t k = g; k < nmine; k += NG, ++j) {
        const int s = (int)(k % S);
        const unsigned char* stg = stage0 + (size_t)s * row_bytes;
        if (!mbar_wait_bounded(bar0 + 8u * (uint32_t)s, (uint32_t)((k / S) & 1))) bad = true;

        double s1 = 0.0, s2 = 0.0, s1b = 0.0, s2b = 0.0;
        if (!bad) {
#pragma unroll 4
            for (int v = t; v < nvec; v += GT) {
                const V16 xv = ld_shared16(stg + (size_t)v * 16);
#pragma unroll
                for (int e = 0; e < VEC; e += 2) {
                    const double x0 = (double)E::get(xv, e);
                    const double x1 = (double)E::get(xv, e + 1);
                    s1 += x0;
                    s1b += x1;
                    s2 = fma(x0, x0, s2);
                    s2b = fma(x1, x1, s2b);
                }
            }
        }
        s1 = warp_sum(s1 + s1b);
        s2 = warp_sum(s2 + s2b);
        double* rb = red + ((size_t)(g * 2 + (j & 1)) * R) * 3;
        if (R > 1) {
            if (lane == 0) {
                rb[wg * 3 + 0] = s1;
                rb[wg * 3 + 1] = s2;
            }
            bad = named_bar_or(bar_id, GT, bad);
        } else {
            bad = __any_sync(0xFFFFFFFFu, bad);
        }
        if (bad) break;
        if (R > 1) {
            s1 = 0.0;
            s2 = 0.0;
            for (int i = 0; i < R; ++i) {
                s1 += rb[i * 3 + 0];
                s2 += rb[i * 3 + 1];
            }
        }
        const double mean = s1 * invD;
        double var = s2 * invD - mean * mean;
        if (!(var > ldexp(mean * mean, -20))) {
            // centred second pass (uniform over the group)
            double c2 = 0.0;
            for (int v = t; v < nvec; v += GT) {
                const V16 xv = ld_shared16(stg + (size_t)v * 16);
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    const double dd = (double)E::get(xv, e) - mean;
                    c2 = fma(dd, dd, c2);
                }
            }
            c2 = warp_sum(c2);
            if (R > 1) {
                if (lane == 0) rb[wg * 3 + 2] = c2;
                named_bar(bar_id, GT);
                c2 = 0.0;
                for (int i = 0; i < R; ++i) c2 += rb[i * 3 + 2];
            }
            var = c2 * invD;
        }
        const double rstd = rsqrt(var + eps);
        const float mu_hi = __double2float_rn(mean);
        const float mu_lo = __double2float_rn(mean - (double)mu_hi);
        const float rf = __double2float_rn(rstd);
        const bool two_sub = 0x1p10f * fabsf(mu_lo) * rf > 0x1p-16f;
        const float kmu = two_sub ? 0x1p-37f * fabsf(mu_hi) : 0x1p10f * fabsf(mu_lo);
        const float2 rf2 = make_float2(rf, rf);
        const float2 nhi2 = make_float2(-mu_hi, -mu_hi);
        const float nlo = two_sub ? -mu_lo : 0.f;
        const float2 nlo2 = make_float2(nlo, nlo);
        const float tmax = __fmaf_rn(__fmul_rn(kmu, rf), wmax, bmax);
        const int64_t row = first + k * stride;
        char* yrow = static_cast<char*>(a.y) + (size_t)row * row_bytes;

        auto output = [&](auto two) {
            constexpr bool TWO = decltype(two)::value;
#pragma unroll 2
            for (int v = t; v < nvec; v += GT) {
                const V16 xv = ld_shared16(stg + (size_t)v * 16);
                float wf[VEC], bf[VEC];
                ring_wb<T, WB>(a, table, nvec, v, wf, bf);
                V16 o;
                float ymin = INFINITY;
#pragma unroll
                for (int e = 0; e < VEC; e += 2) {
                    const float2 w2 = make_float2(wf[e], wf[e + 1]);
                    const float2 b2 = make_float2(bf[e], bf[e + 1]);
                    const float2 A2 = mul2(rf2, w2);
                    const float2 d2 = TWO ? add2(add2(E::get2(xv, e), nhi2), nlo2)
                                          : add2(E::get2(xv, e), nhi2);
                    const float2 y2 = fma2(d2, A2, b2);
                    ymin = fminf(ymin, fminf(fabsf(y2.x), fabsf(y2.y)));
                    E::put2(o, e, y2);
                }
                if (!(ymin > tmax)) o = ring_vector_f64<T, WB>(xv, a, table, nvec, v, mean, rstd);
                st_stream(yrow + (size_t)v * 16, o);
            }
        };
        if (two_sub)
            output(std::true_type{});
        else
            output(std::false_type{});

        // this warp is done with stage s; the group's last warp to get here refills it
        // (the count only grows: R arrivals per row held by the stage)
        __syncwarp();
        if (lane == 0) {
            __threadfence_block();
            if ((atomicAdd(&counts[s], 1) + 1) % R == 0 && k + S < nmine) {
                __threadfence_block();
                fence_proxy_async_smem();
                issue(k + S);
            }
        }
    }

    if (bad && t == 0) atomicExch(faulted, 1);
    __syncthreads();
    if (*faulted && threadIdx.x == 0) {
        // count the fault; let every copy still in flight land before the CTA leaves
        atomicAdd(&nvn_fault_count, 1u);
        for (int s = 0; s < S; ++s)  // a completed phase returns at once
            if (last_issued[s] >= 0)
                mbar_wait_bounded(bar0 + 8u * (uint32_t)s, (uint32_t)((last_issued[s] / S) & 1));
    }
}

}  // namespace nvn
