// allreduce.cuh -- the reduction half of an all-reduce fused with add_rms_norm.
//
// Definition: miniVLLM Layers page, section Linear layers, RowParallelLinear (the forward
// pass of a tensor-parallel decoder's row-parallel layer sums the ranks' partial outputs
// with an all_reduce), followed by the fused residual add + RMSNorm of the same page,
// section LayerNorm, and docs.rs nuvec-core 0.5.0, Enum FastOp, variant AddRmsNorm.
//   x = sum over the nparts partial tensors, in part order, in double, rounded once to the
//       I/O type (the exact sum for bfloat16 parts of ordinary range);
//   h = x + r in float32 rounded to the I/O type;  y = h * rsqrt(mean(h^2) + eps) * w.
// The partial tensors are whatever the caller points at: copies gathered into this GPU's
// memory (an all-gather), or other GPUs' buffers mapped into this process.  Each element
// of every part is read once and x is never re-read, so one pass reads (nparts + 1) rows
// and writes two or three.
//
// One-shot form over peers' memory: each rank keeps its partial in its own buffer, which
// the other ranks have mapped (CUDA IPC).  After producing the partial of step `epoch`, a
// rank publishes that epoch into a flag slot of every rank (tp_publish_kernel: a
// system-scope fence, then a release store per rank); the fused kernel of every rank first
// waits until all flags of its own array have reached the epoch (acquire loads, bounded to
// about a second, one thread per CTA), then reads the peers' partials directly with plain
// loads -- no copy, no multicast.  A wait that runs out counts a fault (nv_fault_count)
// and the CTA leaves without touching its rows.
#pragma once

#include "common.cuh"
#include "rms.cuh"
#include "staged.cuh"

namespace nvn {

constexpr int kMaxParts = 8;

__device__ __forceinline__ long long ld_acquire_sys(const long long* p) {
    long long v;
    asm volatile("ld.acquire.sys.global.s64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_sys(long long* p, long long v) {
    asm volatile("st.release.sys.global.s64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Wait until flags[0..n) all reach `epoch`; false once ~kWaitLimitNs have passed (or after
// an iteration cap).  One thread.
__device__ __forceinline__ bool wait_flags(const long long* flags, int n, long long epoch) {
    const uint64_t t0 = global_ns();
    uint32_t i = 0;
    for (int p = 0; p < n; ++p) {
        while (ld_acquire_sys(flags + p) < epoch) {
            if (++i >= (1u << 26)) return false;
            if ((i & 63u) == 0 && global_ns() - t0 > kWaitLimitNs) return false;
            __nanosleep(64);
        }
    }
    return true;
}

struct PublishArgs {
    long long* flags[kMaxParts];  // every rank's flag array (this rank's own, and mapped)
    int world;
    int rank;
    long long epoch;
};

// Publish `epoch` in slot `rank` of every rank's flag array, after everything queued
// before on the stream (the partial) is complete and visible system-wide.
__global__ void __launch_bounds__(32) tp_publish_kernel(const PublishArgs a) {
    pdl_wait();
    if (threadIdx.x != 0) return;
    __threadfence_system();
    for (int p = 0; p < a.world; ++p) st_release_sys(a.flags[p] + a.rank, a.epoch);
}

struct ReduceNormArgs {
    const void* parts[kMaxParts];
    int nparts;
    const void* r;
    const void* w;
    void* y;
    void* h;
    void* x_out;  // NULL: x is not written
    int64_t rows;
    int D;
    int nvec;     // 16-byte vectors per row (register path)
    int G;        // threads per row (register path)
    float eps;
    const long long* flags;  // NULL, or this rank's flag array [nparts]: wait for `epoch`
    long long epoch;
};

// The one-shot form's wait (a no-op without flags): false when this CTA must leave.
__device__ __forceinline__ bool peers_ready(const ReduceNormArgs& a) {
    if (!a.flags) return true;
    bool ok = true;
    if (threadIdx.x == 0) ok = wait_flags(a.flags, a.nparts, a.epoch);
    if (__syncthreads_or(ok ? 0 : 1)) {
        if (threadIdx.x == 0) atomicAdd(&nvn_fault_count, 1u);
        return false;
    }
    return true;
}

template <typename T>
__device__ __forceinline__ float round_io(double v);
template <>
__device__ __forceinline__ float round_io<float>(double v) {
    return __double2float_rn(v);
}
template <>
__device__ __forceinline__ float round_io<__nv_bfloat16>(double v) {
    return __bfloat162float(__double2bfloat16(v));  // one rounding, to nearest even
}

// Register path: one row per CTA of G threads, thread t holding vectors t, t + G, ...
template <typename T, int VPT>
__global__ void __launch_bounds__(1024) allreduce_rms_rows_kernel(const ReduceNormArgs a) {
    pdl_wait();
    pdl_release();
    if (!peers_ready(a)) return;
    using E = Elem<T>;
    constexpr int VEC = E::kVec;
    __shared__ float red[2][32];
    const int G = a.G;
    const int t = threadIdx.x;
    const float invD = 1.0f / (float)a.D;
    int it = 0;
    for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x, ++it) {
        const size_t roff = (size_t)row * (size_t)a.nvec * 16;
        V16 hv[VPT];
        float ss = 0.f;
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = t + k * G;
            if (v >= a.nvec) continue;
            const size_t off = roff + (size_t)v * 16;
            const V16 rv = ld_stream(static_cast<const char*>(a.r) + off);
            V16 pv[kMaxParts];
#pragma unroll
            for (int p = 0; p < kMaxParts; ++p)
                if (p < a.nparts) pv[p] = ld_stream(static_cast<const char*>(a.parts[p]) + off);
            double acc[VEC];
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[e] = 0.0;
#pragma unroll
            for (int p = 0; p < kMaxParts; ++p)
                if (p < a.nparts)
#pragma unroll
                    for (int e = 0; e < VEC; ++e) acc[e] += (double)E::get(pv[p], e);
            V16 xv;
#pragma unroll
            for (int e = 0; e < VEC; e += 2) {
                const float x0 = round_io<T>(acc[e]), x1 = round_io<T>(acc[e + 1]);
                E::put2(xv, e, x0, x1);
                E::put2(hv[k], e, __fadd_rn(x0, E::get(rv, e)), __fadd_rn(x1, E::get(rv, e + 1)));
            }
            if (a.x_out) st_stream(static_cast<char*>(a.x_out) + off, xv);
            st_stream(static_cast<char*>(a.h) + off, hv[k]);
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                const float f = E::get(hv[k], e);
                ss = fmaf(f, f, ss);
            }
        }
        ss = warp_sum(ss);
        const int nw = blockDim.x >> 5;
        if (nw > 1) {
            float* buf = red[it & 1];
            if ((t & 31) == 0) buf[t >> 5] = ss;
            __syncthreads();
            ss = 0.f;
            for (int i = 0; i < nw; ++i) ss += buf[i];
        }
        const float inv = rsqrtf(__fmaf_rn(ss, invD, a.eps));
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = t + k * G;
            if (v >= a.nvec) continue;
            const V16 wv = a.w ? ld_param(static_cast<const char*>(a.w) + (size_t)v * 16)
                               : ones_vec<T>();
            V16 o;
#pragma unroll
            for (int e = 0; e < VEC; e += 2)
                E::put2(o, e, __fmul_rn(__fmul_rn(E::get(hv[k], e), inv), E::get(wv, e)),
                        __fmul_rn(__fmul_rn(E::get(hv[k], e + 1), inv), E::get(wv, e + 1)));
            st_stream(static_cast<char*>(a.y) + roff + (size_t)v * 16, o);
        }
    }
}

// Any D and alignment: one CTA per row, scalar accesses; h is written in the first pass
// and read back (by the thread that wrote it) in the second.
template <typename T>
__global__ void __launch_bounds__(256) allreduce_rms_generic_kernel(const ReduceNormArgs a) {
    pdl_wait();
    pdl_release();
    if (!peers_ready(a)) return;
    using E = Elem<T>;
    __shared__ float red[2][32];
    const int nw = blockDim.x >> 5;
    int it = 0;
    for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x, ++it) {
        const int64_t r0 = row * (int64_t)a.D;
        float ss = 0.f;
        for (int j = threadIdx.x; j < a.D; j += blockDim.x) {
            double acc = 0.0;
            for (int p = 0; p < a.nparts; ++p) acc += (double)E::load1(a.parts[p], r0 + j);
            const float x = round_io<T>(acc);
            if (a.x_out) E::store1(a.x_out, r0 + j, x);
            const float h = E::round(__fadd_rn(x, E::load1(a.r, r0 + j)));
            E::store1(a.h, r0 + j, h);
            ss = fmaf(h, h, ss);
        }
        ss = warp_sum(ss);
        float* buf = red[it & 1];
        if ((threadIdx.x & 31) == 0) buf[threadIdx.x >> 5] = ss;
        __syncthreads();
        ss = 0.f;
        for (int i = 0; i < nw; ++i) ss += buf[i];
        const float inv = rsqrtf(__fmaf_rn(ss, 1.0f / (float)a.D, a.eps));
        for (int j = threadIdx.x; j < a.D; j += blockDim.x) {
            const float h = E::load1(a.h, r0 + j);
            const float wj = a.w ? E::load1(a.w, j) : 1.f;
            E::store1(a.y, r0 + j, __fmul_rn(__fmul_rn(h, inv), wj));
        }
    }
}

}  // namespace nvn
