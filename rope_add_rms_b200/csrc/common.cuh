// common.cuh -- element types, 16-byte vector I/O and reductions shared by the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace nvn {

// ---- element types ---------------------------------------------------------------
// A 16-byte vector of the I/O type, kept as four 32-bit words: 8 bfloat16 or 4 float32.
struct V16 {
    uint32_t u[4];
};

template <typename T>
struct Elem;

template <>
struct Elem<float> {
    static constexpr int kVec = 4;  // elements per 16-byte vector
    static constexpr int kSize = 4;
    __device__ __forceinline__ static float get(const V16& v, int e) {
        return __uint_as_float(v.u[e]);
    }
    // round-to-nearest-even into the I/O type; float32 needs no rounding
    __device__ __forceinline__ static void put2(V16& v, int e, float a, float b) {
        v.u[e] = __float_as_uint(a);
        v.u[e + 1] = __float_as_uint(b);
    }
    __device__ __forceinline__ static float load1(const void* p, int64_t i) {
        return static_cast<const float*>(p)[i];
    }
    __device__ __forceinline__ static void store1(void* p, int64_t i, float v) {
        static_cast<float*>(p)[i] = v;
    }
    __device__ __forceinline__ static float round(float v) { return v; }
    // elements e, e + 1 (e even) as a float pair, and back
    __device__ __forceinline__ static float2 get2(const V16& v, int e) {
        return make_float2(__uint_as_float(v.u[e]), __uint_as_float(v.u[e + 1]));
    }
    __device__ __forceinline__ static void put2(V16& v, int e, float2 p) { put2(v, e, p.x, p.y); }
};

template <>
struct Elem<__nv_bfloat16> {
    static constexpr int kVec = 8;
    static constexpr int kSize = 2;
    // element e of the vector: the 16-bit pattern moved to the top of a binary32 (exact)
    __device__ __forceinline__ static float get(const V16& v, int e) {
        uint32_t w = v.u[e >> 1];
        return __uint_as_float((e & 1) ? (w & 0xFFFF0000u) : (w << 16));
    }
    // elements e and e + 1 (e even), each rounded once to nearest even
    __device__ __forceinline__ static void put2(V16& v, int e, float a, float b) {
        __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
        v.u[e >> 1] = *reinterpret_cast<uint32_t*>(&p);
    }
    __device__ __forceinline__ static float load1(const void* p, int64_t i) {
        return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
    }
    __device__ __forceinline__ static void store1(void* p, int64_t i, float v) {
        static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
    }
    __device__ __forceinline__ static float round(float v) {
        return __bfloat162float(__float2bfloat16_rn(v));
    }
    __device__ __forceinline__ static float2 get2(const V16& v, int e) {
        const uint32_t w = v.u[e >> 1];
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
    }
    __device__ __forceinline__ static void put2(V16& v, int e, float2 p) { put2(v, e, p.x, p.y); }
};

// Bulk prefetch of `bytes` (a multiple of 16) at global address p (16-byte aligned) into L2.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// ---- packed float32 pairs (Blackwell FFMA2 / FADD2 / FMUL2; IEEE per lane) ------------
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 neg2(float2 a) { return make_float2(-a.x, -a.y); }

// ---- bfloat16 pairs consumed packed (sm_100 mixed-precision fma) ----------------------
// (lo(u) lo(v) + c.x, hi(u) hi(v) + c.y): each a float32 fma of the bfloat16 halves of two
// packed words -- the exact product plus c, rounded once, as the float32 fma of the unpacked
// values would give -- with no unpacking.
__device__ __forceinline__ float2 bf16x2_mac(uint32_t u, uint32_t v, float2 c) {
    float lo, hi;
    asm("{\n\t.reg .b16 ul, uh, vl, vh;\n\tmov.b32 {ul, uh}, %2;\n\tmov.b32 {vl, vh}, %3;\n\t"
        "fma.rn.f32.bf16 %0, ul, vl, %4;\n\tfma.rn.f32.bf16 %1, uh, vh, %5;\n}"
        : "=f"(lo), "=f"(hi)
        : "r"(u), "r"(v), "f"(c.x), "f"(c.y));
    return make_float2(lo, hi);
}
constexpr uint32_t kBf16x2One = 0x3F803F80u;  // (1, 1)

// ---- 16-byte global memory access -------------------------------------------------
// Streaming loads (read once: evict-first) and stores for the row data; plain cached
// loads for the per-column parameters that every row reuses.
__device__ __forceinline__ V16 ld_stream(const void* p) {
    uint4 t = __ldcs(static_cast<const uint4*>(p));
    return V16{{t.x, t.y, t.z, t.w}};
}
__device__ __forceinline__ V16 ld_param(const void* p) {
    uint4 t = __ldg(static_cast<const uint4*>(p));
    return V16{{t.x, t.y, t.z, t.w}};
}
__device__ __forceinline__ void st_stream(void* p, const V16& v) {
    __stcs(static_cast<uint4*>(p), make_uint4(v.u[0], v.u[1], v.u[2], v.u[3]));
}

// A vector whose every element is 1 in the I/O type (stands in for a NULL weight).
template <typename T>
__device__ __forceinline__ V16 ones_vec() {
    if constexpr (sizeof(T) == 4) {
        const uint32_t one = 0x3F800000u;
        return V16{{one, one, one, one}};
    } else {
        const uint32_t one2 = 0x3F803F80u;
        return V16{{one2, one2, one2, one2}};
    }
}
template <typename T>
__device__ __forceinline__ V16 zeros_vec() {
    return V16{{0u, 0u, 0u, 0u}};
}

// ---- programmatic dependent launch ---------------------------------------------------
// Every kernel starts with pdl_wait() before it touches global memory: when it was
// launched with programmatic stream serialization after a kernel that lets dependents
// start early, this blocks until that kernel has completed and its memory is visible;
// otherwise it returns at once.  pdl_release() lets the next such kernel in the stream
// be scheduled while this one still runs (that kernel waits in its own pdl_wait()).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- reductions ---------------------------------------------------------------------
// Butterfly sum over aligned groups of `width` lanes (width a power of two <= 32).
template <typename F>
__device__ __forceinline__ F group_sum(F v, int width) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1)
        if (off < width) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
    return v;
}
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
    return v;
}

}  // namespace nvn
