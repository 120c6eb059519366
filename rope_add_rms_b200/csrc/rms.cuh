// rms.cuh -- rms_norm and add_rms_norm kernels.
//
// Definitions: docs.rs nuvec-core 0.5.0, Enum FastOp, variants RmsNorm
// (y = x / sqrt(mean(x^2) + eps) * w) and AddRmsNorm (h = x + r, then RmsNorm of h);
// miniVLLM Layers page, LayerNorm.forward with a residual (returns y and the updated
// residual h).  h is the float32 sum rounded once to the I/O type and y normalises
// that rounded h.
#pragma once

#include "common.cuh"

namespace nvn {

struct RowArgs {
    const void* x;
    const void* r;  // residual (add_rms_norm) -- unused otherwise
    const void* w;  // NULL: w = 1
    const void* b;  // layer_norm bias, NULL: b = 0
    void* y;
    void* h;        // updated residual (add_rms_norm)
    int64_t rows;
    int D;          // row length in elements
    int nvec;       // 16-byte vectors per row (register path)
    int G;          // threads per row (multiple of 32)
    int rows_per_cta;
    float eps;
};

// ---- register path ------------------------------------------------------------------
// G threads share one row (a multiple of 32, or for narrow rows a power of two up to 16,
// several rows to a warp); thread t holds vectors t, t + G, ..., t + (VPT-1) G of the
// row in registers (coalesced: consecutive threads read consecutive 16-byte vectors).
// All loads of a row are issued before any arithmetic; the sum of squares is reduced
// with warp shuffles and, when a row spans several warps, one shared-memory step.
// The CTA walks its rows in a grid-stride loop, so the per-column weights stay in
// registers for the whole launch.
// Largest CTA the register kernels are built for (more vectors per thread, fewer threads).
__host__ __device__ constexpr int rms_max_threads(int vpt) { return vpt >= 4 ? 512 : 1024; }
__host__ __device__ constexpr int layer_max_threads(int vpt) { return vpt >= 2 ? 512 : 1024; }
// With few vectors per thread the weights stay in registers for the whole launch; with
// more, they are re-read per row from L1 (every row of the CTA uses the same D values).
__host__ __device__ constexpr bool weights_in_regs(int vpt) { return vpt <= 2; }

template <typename T, int VPT, bool ADD>
__global__ void __launch_bounds__(rms_max_threads(VPT)) rms_rows_kernel(const RowArgs a) {
    pdl_wait();
    pdl_release();
    using E = Elem<T>;
    constexpr int VEC = E::kVec;
    const int G = a.G;
    const int slot = threadIdx.x / G;
    const int t = threadIdx.x - slot * G;
    const int wpr = G >> 5;  // warps per row
    __shared__ float red[2][32];

    constexpr bool kWRegs = weights_in_regs(VPT);
    V16 wv[VPT];
    if constexpr (kWRegs) {
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = t + k * G;
            wv[k] = (a.w != nullptr && v < a.nvec)
                        ? ld_param(static_cast<const char*>(a.w) + (size_t)v * 16)
                        : ones_vec<T>();
        }
    }
    const float invD = 1.0f / (float)a.D;

    int it = 0;
    for (int64_t base = (int64_t)blockIdx.x * a.rows_per_cta; base < a.rows;
         base += (int64_t)gridDim.x * a.rows_per_cta, ++it) {
        const int64_t row = base + slot;
        const bool active = row < a.rows;
        const size_t roff = (size_t)row * (size_t)a.D * sizeof(T);

        V16 hv[VPT];
        V16 rv[VPT];
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = t + k * G;
            if (active && v < a.nvec) {
                hv[k] = ld_stream(static_cast<const char*>(a.x) + roff + (size_t)v * 16);
                if constexpr (ADD)
                    rv[k] = ld_stream(static_cast<const char*>(a.r) + roff + (size_t)v * 16);
            }
        }

        float ss = 0.f;
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = t + k * G;
            if (active && v < a.nvec) {
                if constexpr (ADD) {
#pragma unroll
                    for (int e = 0; e < VEC; e += 2) {
                        const float s0 = __fadd_rn(E::get(hv[k], e), E::get(rv[k], e));
                        const float s1 = __fadd_rn(E::get(hv[k], e + 1), E::get(rv[k], e + 1));
                        E::put2(hv[k], e, s0, s1);  // h rounded once to the I/O type
                    }
                    st_stream(static_cast<char*>(a.h) + roff + (size_t)v * 16, hv[k]);
                }
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    const float f = E::get(hv[k], e);
                    ss = fmaf(f, f, ss);
                }
            }
        }

        ss = group_sum(ss, G < 32 ? G : 32);  // a row of fewer than 32 lanes: its own lanes
        if (wpr > 1) {
            float* buf = red[it & 1];
            if ((threadIdx.x & 31) == 0) buf[threadIdx.x >> 5] = ss;
            __syncthreads();
            ss = 0.f;
            const int w0 = slot * wpr;
            for (int i = 0; i < wpr; ++i) ss += buf[w0 + i];
        }
        const float inv = rsqrtf(__fmaf_rn(ss, invD, a.eps));

#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int v = t + k * G;
            if (active && v < a.nvec) {
                if constexpr (!kWRegs)
                    wv[k] = a.w != nullptr
                                ? ld_param(static_cast<const char*>(a.w) + (size_t)v * 16)
                                : ones_vec<T>();
                V16 o;
#pragma unroll
                for (int e = 0; e < VEC; e += 2) {
                    const float y0 = __fmul_rn(__fmul_rn(E::get(hv[k], e), inv), E::get(wv[k], e));
                    const float y1 =
                        __fmul_rn(__fmul_rn(E::get(hv[k], e + 1), inv), E::get(wv[k], e + 1));
                    E::put2(o, e, y0, y1);
                }
                st_stream(static_cast<char*>(a.y) + roff + (size_t)v * 16, o);
            }
        }
    }
}

// ---- generic path ---------------------------------------------------------------------
// Any D and any element alignment: one CTA per row, scalar accesses.  Pass 1 forms
// (and for add_rms_norm stores) h and its sum of squares; pass 2 re-reads h (or x)
// -- the same thread touches the same index in both passes -- and writes y.
template <typename T, bool ADD>
__global__ void __launch_bounds__(256) rms_generic_kernel(const RowArgs a) {
    pdl_wait();
    pdl_release();
    using E = Elem<T>;
    __shared__ float red[2][32];
    const int nw = blockDim.x >> 5;
    int it = 0;
    for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x, ++it) {
        const int64_t r0 = row * (int64_t)a.D;
        float ss = 0.f;
        for (int j = threadIdx.x; j < a.D; j += blockDim.x) {
            float hv;
            if constexpr (ADD) {
                hv = E::round(__fadd_rn(E::load1(a.x, r0 + j), E::load1(a.r, r0 + j)));
                E::store1(a.h, r0 + j, hv);
            } else {
                hv = E::load1(a.x, r0 + j);
            }
            ss = fmaf(hv, hv, ss);
        }
        ss = warp_sum(ss);
        float* buf = red[it & 1];
        if ((threadIdx.x & 31) == 0) buf[threadIdx.x >> 5] = ss;
        __syncthreads();
        ss = 0.f;
        for (int i = 0; i < nw; ++i) ss += buf[i];
        const float inv = rsqrtf(__fmaf_rn(ss, 1.0f / (float)a.D, a.eps));
        for (int j = threadIdx.x; j < a.D; j += blockDim.x) {
            const float hv = ADD ? E::load1(a.h, r0 + j) : E::load1(a.x, r0 + j);
            const float wj = a.w ? E::load1(a.w, j) : 1.f;
            E::store1(a.y, r0 + j, __fmul_rn(__fmul_rn(hv, inv), wj));
        }
    }
}

}  // namespace nvn
