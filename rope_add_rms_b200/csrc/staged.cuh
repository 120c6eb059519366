// staged.cuh -- persistent rms_norm / add_rms_norm with rows staged in shared memory by
// bulk asynchronous copies (the Blackwell/Hopper copy engine, cp.async.bulk).
//
// Why: the op is HBM-bound, and the register path keeps only a CTA's own row in flight
// per thread group, which left DRAM about two thirds busy.  Here one thread per CTA
// keeps `stages` whole rows of x (and r) in flight into a ring of shared-memory
// buffers; the CTA's threads consume the ring in order.  A full row of a 4096-wide
// bfloat16 add_rms_norm is 16 KB, so a few stages give each SM 64-200 KB of reads in
// flight regardless of register occupancy.
//
// Per row k of this CTA (rows blockIdx.x, blockIdx.x + gridDim.x, ...):
//   wait full[k % S] -> read x, r from the stage into registers -> h = RNE(x + r),
//   store h, sum of squares -> CTA reduction (one barrier, __syncthreads_or: after it
//   every thread has consumed the stage, and all know whether any wait ran out) ->
//   thread 0 refills the stage with row k + S -> y = h*inv*w, store y.
// The copies are plain (non-multicast) 1-D bulk copies from this GPU's own memory into
// the issuing CTA's shared memory.
//
// Every wait on an mbarrier is bounded (about one second of %globaltimer).  If a wait
// runs out, every thread of the CTA learns it at the row's barrier, the CTA counts a
// fault in nvn_fault_count (read by nv_fault_count()), stops consuming rows, waits (again
// bounded) for the copies it has in flight and returns.  A correct launch never gets there: the bytes expected per stage equal the
// bytes copied into it.
#pragma once

#include "common.cuh"
#include "layer.cuh"
#include "rms.cuh"

namespace nvn {

// Timed-out bounded waits since load (or the last reset); see nv_fault_count().
__device__ unsigned int nvn_fault_count;

constexpr uint64_t kWaitLimitNs = 1000000000ull;  // ~1 s per wait

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
// 1-D bulk copy global -> this CTA's shared memory, completion counted on `bar`.
// dst, src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Wait for phase `parity` of `bar`; false once ~limit_ns have passed (or after an
// iteration cap, whichever comes first).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 1; i < (1u << 28); ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63u) == 0 && global_ns() - t0 > kWaitLimitNs) return false;
    }
    return false;
}

// Check of the bounded wait itself: each CTA waits on an mbarrier that nothing arrives on
// (its first phase never completes), so every thread gives up after ~kWaitLimitNs, and
// the CTA counts one fault, as a staged kernel does when its copies never land.  No copy
// is in flight, so the CTA may leave at once.
__global__ void __launch_bounds__(32) bounded_wait_selftest_kernel() {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_addr(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        fence_mbar_init();
    }
    __syncthreads();
    const bool ok = mbar_wait_bounded(b, 0);
    if (__syncthreads_count(ok ? 0 : 1) > 0 && threadIdx.x == 0) atomicAdd(&nvn_fault_count, 1u);
}

__device__ __forceinline__ V16 ld_shared16(const unsigned char* p) {
    const uint4 t = *reinterpret_cast<const uint4*>(p);
    return V16{{t.x, t.y, t.z, t.w}};
}

// Launch: blockDim.x = G threads (multiple of 32) handle one row at a time; dynamic
// shared memory = stages * (ADD ? 2 : 1) * row_bytes + stages * 8 (mbarriers).
template <typename T, int VPT, bool ADD>
__global__ void __launch_bounds__(512) rms_staged_kernel(const RowArgs a, const int stages) {
    pdl_wait();
    pdl_release();
    using E = Elem<T>;
    constexpr int VEC = E::kVec;
    constexpr int NT = ADD ? 2 : 1;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ float red[2][32];

    const int G = blockDim.x;
    const int t = threadIdx.x;
    const int wpr = G >> 5;
    const uint32_t row_bytes = (uint32_t)a.nvec * 16u;
    const uint32_t stage_bytes = NT * row_bytes;
    const uint32_t sbase = smem_addr(smem);
    const uint32_t bbase = sbase + (uint32_t)stages * stage_bytes;
    const int64_t first = blockIdx.x;
    const int64_t stride = gridDim.x;
    const int64_t nmine = first < a.rows ? (a.rows - 1 - first) / stride + 1 : 0;

    if (t == 0) {
        for (int s = 0; s < stages; ++s) mbar_init(bbase + 8u * s, 1);
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    __syncthreads();

    auto issue = [&](int64_t k) {
        const int s = (int)(k % stages);
        const int64_t row = first + k * stride;
        const uint32_t bar = bbase + 8u * s;
        const uint32_t dst = sbase + (uint32_t)s * stage_bytes;
        mbar_arrive_expect_tx(bar, stage_bytes);
        bulk_load(dst, static_cast<const char*>(a.x) + (size_t)row * row_bytes, row_bytes, bar);
        if constexpr (ADD)
            bulk_load(dst + row_bytes, static_cast<const char*>(a.r) + (size_t)row * row_bytes,
                      row_bytes, bar);
    };
    if (t == 0)
        for (int64_t k = 0; k < nmine && k < stages; ++k) issue(k);

    constexpr bool kWRegs = weights_in_regs(VPT);
    V16 wv[VPT];
    if constexpr (kWRegs) {
#pragma unroll
        for (int kk = 0; kk < VPT; ++kk) {
            const int v = t + kk * G;
            wv[kk] = (a.w != nullptr && v < a.nvec)
                         ? ld_param(static_cast<const char*>(a.w) + (size_t)v * 16)
                         : ones_vec<T>();
        }
    }
    const float invD = 1.0f / (float)a.D;

    int64_t k = 0;
    for (; k < nmine; ++k) {
        const int s = (int)(k % stages);
        const uint32_t parity = (uint32_t)((k / stages) & 1);
        const bool bad = !mbar_wait_bounded(bbase + 8u * s, parity);
        const int64_t row = first + k * stride;
        const size_t roff = (size_t)row * row_bytes;
        const unsigned char* stg = smem + (size_t)s * stage_bytes;

        V16 hv[VPT];
        V16 rv[VPT];
#pragma unroll
        for (int kk = 0; kk < VPT; ++kk) {
            const int v = t + kk * G;
            if (v < a.nvec) {
                hv[kk] = ld_shared16(stg + (size_t)v * 16);
                if constexpr (ADD) rv[kk] = ld_shared16(stg + row_bytes + (size_t)v * 16);
            }
        }
        float ss = 0.f;
#pragma unroll
        for (int kk = 0; kk < VPT; ++kk) {
            const int v = t + kk * G;
            if (v < a.nvec) {
                if constexpr (ADD) {
#pragma unroll
                    for (int e = 0; e < VEC; e += 2) {
                        const float s0 = __fadd_rn(E::get(hv[kk], e), E::get(rv[kk], e));
                        const float s1 = __fadd_rn(E::get(hv[kk], e + 1), E::get(rv[kk], e + 1));
                        E::put2(hv[kk], e, s0, s1);
                    }
                    st_stream(static_cast<char*>(a.h) + roff + (size_t)v * 16, hv[kk]);
                }
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    const float f = E::get(hv[kk], e);
                    ss = fmaf(f, f, ss);
                }
            }
        }
        ss = warp_sum(ss);
        float* buf = red[k & 1];
        if ((t & 31) == 0) buf[t >> 5] = ss;
        // every thread has consumed stage s; a wait that ran out anywhere stops every thread
        if (__syncthreads_or(bad ? 1 : 0)) break;
        if (t == 0 && k + stages < nmine) {
            fence_proxy_async_smem();
            issue(k + stages);
        }
        ss = 0.f;
        for (int i = 0; i < wpr; ++i) ss += buf[i];
        const float inv = rsqrtf(__fmaf_rn(ss, invD, a.eps));
#pragma unroll
        for (int kk = 0; kk < VPT; ++kk) {
            const int v = t + kk * G;
            if (v < a.nvec) {
                if constexpr (!kWRegs)
                    wv[kk] = a.w != nullptr
                                 ? ld_param(static_cast<const char*>(a.w) + (size_t)v * 16)
                                 : ones_vec<T>();
                V16 o;
#pragma unroll
                for (int e = 0; e < VEC; e += 2) {
                    const float y0 =
                        __fmul_rn(__fmul_rn(E::get(hv[kk], e), inv), E::get(wv[kk], e));
                    const float y1 =
                        __fmul_rn(__fmul_rn(E::get(hv[kk], e + 1), inv), E::get(wv[kk], e + 1));
                    E::put2(o, e, y0, y1);
                }
                st_stream(static_cast<char*>(a.y) + roff + (size_t)v * 16, o);
            }
        }
    }

    if (k < nmine) {  // a wait ran out: count it, let the copies in flight land, leave
        if (t == 0) {
            atomicAdd(&nvn_fault_count, 1u);
            for (int64_t j = k; j < nmine && j < k + stages; ++j)
                mbar_wait_bounded(bbase + 8u * (uint32_t)(j % stages),
                                  (uint32_t)((j / stages) & 1));
        }
    }
}

// ---- layer_norm, staged ------------------------------------------------------------
// Same arithmetic as layer_rows_kernel (double statistics from one widening per
// element, float32 output with the error test and the double recompute), but the row
// lives in a shared-memory stage filled by a bulk copy instead of in registers: each
// thread reads its vectors from the stage in the statistics pass and again in the
// output pass.  Registers then hold no row data across the reduction, so more warps fit
// per SM, and the copies of the next `stages - 1` rows are in flight meanwhile.  Two
// barriers per row: the reduction's, and one after the output pass that frees the stage.
template <typename T, int VPT>
__global__ void __launch_bounds__(512) layer_staged_kernel(const RowArgs a, const int stages) {
    pdl_wait();
    pdl_release();
    using E = Elem<T>;
    constexpr int VEC = E::kVec;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ double red[2][3][16];

    const int G = blockDim.x;
    const int t = threadIdx.x;
    const int wpr = G >> 5;
    const uint32_t row_bytes = (uint32_t)a.nvec * 16u;
    const uint32_t sbase = smem_addr(smem);
    const uint32_t bbase = sbase + (uint32_t)stages * row_bytes;
    const int64_t first = blockIdx.x;
    const int64_t stride = gridDim.x;
    const int64_t nmine = first < a.rows ? (a.rows - 1 - first) / stride + 1 : 0;

    if (t == 0) {
        for (int s = 0; s < stages; ++s) mbar_init(bbase + 8u * s, 1);
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    __syncthreads();
    auto issue = [&](int64_t k) {
        const int s = (int)(k % stages);
        const int64_t row = first + k * stride;
        const uint32_t bar = bbase + 8u * s;
        mbar_arrive_expect_tx(bar, row_bytes);
        bulk_load(sbase + (uint32_t)s * row_bytes,
                  static_cast<const char*>(a.x) + (size_t)row * row_bytes, row_bytes, bar);
    };
    if (t == 0)
        for (int64_t k = 0; k < nmine && k < stages; ++k) issue(k);

    const double invD = 1.0 / (double)a.D;
    const double eps = (double)a.eps;
    // largest |w| and 2^-11 |b| over this thread's columns (bounds of the error test)
    float wmax = 0.f, bmax = 0.f;
#pragma unroll
    for (int kk = 0; kk < VPT; ++kk) {
        const int v = t + kk * G;
        if (v < a.nvec) {
            const V16 wv = a.w ? ld_param(static_cast<const char*>(a.w) + (size_t)v * 16)
                               : ones_vec<T>();
            const V16 bv = a.b ? ld_param(static_cast<const char*>(a.b) + (size_t)v * 16)
                               : zeros_vec<T>();
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                wmax = fmaxf(wmax, fabsf(E::get(wv, e)));
                bmax = fmaxf(bmax, fabsf(E::get(bv, e)));
            }
        }
    }
    bmax *= 0x1p-11f;

    int64_t k = 0;
    for (; k < nmine; ++k) {
        const int s = (int)(k % stages);
        const bool bad = !mbar_wait_bounded(bbase + 8u * s, (uint32_t)((k / stages) & 1));
        const unsigned char* stg = smem + (size_t)s * row_bytes;
        const int64_t row = first + k * stride;
        const size_t roff = (size_t)row * row_bytes;

        double s1 = 0.0, s2 = 0.0, s1b = 0.0, s2b = 0.0;
#pragma unroll
        for (int kk = 0; kk < VPT; ++kk) {
            const int v = t + kk * G;
            if (v < a.nvec) {
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
        double(*buf)[16] = red[k & 1];
        if ((t & 31) == 0) {
            buf[0][t >> 5] = s1;
            buf[1][t >> 5] = s2;
        }
        if (__syncthreads_or(bad ? 1 : 0)) break;  // the same decision in every thread
        s1 = 0.0;
        s2 = 0.0;
        for (int i = 0; i < wpr; ++i) {
            s1 += buf[0][i];
            s2 += buf[1][i];
        }
        const double mean = s1 * invD;
        double var = s2 * invD - mean * mean;
        if (!(var > ldexp(mean * mean, -20))) {   // CTA-uniform: one row per CTA
            double c2 = 0.0;
#pragma unroll
            for (int kk = 0; kk < VPT; ++kk) {
                const int v = t + kk * G;
                if (v < a.nvec) {
                    const V16 xv = ld_shared16(stg + (size_t)v * 16);
#pragma unroll
                    for (int e = 0; e < VEC; ++e) {
                        const double dd = (double)E::get(xv, e) - mean;
                        c2 = fma(dd, dd, c2);
                    }
                }
            }
            c2 = warp_sum(c2);
            if ((t & 31) == 0) buf[2][t >> 5] = c2;
            __syncthreads();
            c2 = 0.0;
            for (int i = 0; i < wpr; ++i) c2 += buf[2][i];
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
#pragma unroll
        for (int kk = 0; kk < VPT; ++kk) {
            const int v = t + kk * G;
            if (v < a.nvec) {
                const V16 xv = ld_shared16(stg + (size_t)v * 16);
                const V16 wv = a.w ? ld_param(static_cast<const char*>(a.w) + (size_t)v * 16)
                                   : ones_vec<T>();
                const V16 bv = a.b ? ld_param(static_cast<const char*>(a.b) + (size_t)v * 16)
                                   : zeros_vec<T>();
                V16 o;
                float ymin = INFINITY;
#pragma unroll
                for (int e = 0; e < VEC; e += 2) {
                    const float2 w2 = E::get2(wv, e);
                    const float2 b2 = E::get2(bv, e);
                    const float2 A2 = mul2(rf2, w2);
                    const float2 d2 = add2(add2(E::get2(xv, e), nhi2), nlo2);
                    const float2 y2 = fma2(d2, A2, b2);
                    ymin = fminf(ymin, fminf(fabsf(y2.x), fabsf(y2.y)));
                    E::put2(o, e, y2);
                }
                if (!(ymin > tmax)) o = layer_vector_f64<T>(xv, wv, bv, mean, rstd);
                st_stream(static_cast<char*>(a.y) + roff + (size_t)v * 16, o);
            }
        }
        __syncthreads();  // every thread is done with stage s
        if (t == 0 && k + stages < nmine) {
            fence_proxy_async_smem();
            issue(k + stages);
        }
    }

    if (k < nmine && t == 0) {  // a wait ran out: count it, let the copies in flight land
        atomicAdd(&nvn_fault_count, 1u);
        for (int64_t j = k; j < nmine && j < k + stages; ++j)
            mbar_wait_bounded(bbase + 8u * (uint32_t)(j % stages), (uint32_t)((j / stages) & 1));
    }
}

}  // namespace nvn
