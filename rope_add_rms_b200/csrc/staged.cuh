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
//   store h, sum of squares -> CTA reduction (one __syncthreads: after it every thread
//   has consumed the stage) -> thread 0 refills the stage with row k + S -> y = h*inv*w,
//   store y.
// The copies are plain (non-multicast) 1-D bulk copies from this GPU's own memory into
// the issuing CTA's shared memory.
//
// Every wait on an mbarrier is bounded (about one second of %globaltimer).  If a wait
// runs out, the CTA counts a fault in nvn_fault_count (read by nv_fault_count()),
// stops consuming rows, waits (again bounded) for the copies it has in flight and
// returns.  A correct launch never gets there: the bytes expected per stage equal the
// bytes copied into it.
#pragma once

#include "common.cuh"
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
    __shared__ int abort_flag;

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
        abort_flag = 0;
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
        if (!mbar_wait_bounded(bbase + 8u * s, parity)) abort_flag = 1;
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
        __syncthreads();  // every thread has consumed stage s; abort_flag is settled
        if (abort_flag) break;
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

}  // namespace nvn
