// nvnorm_api.cu -- the C ABI of libnvnorm.so: argument validation, kernel-variant
// selection and launch.  Declarations and the contract of every entry point are in
// include/nvnorm.h.
#include <cuda.h>  // CUresult / CUdeviceptr for the driver range query (no libcuda link)
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <utility>

#include "nvnorm.h"

#include "allreduce.cuh"
#include "common.cuh"
#include "layer.cuh"
#include "layer_ring.cuh"
#include "layer_slots.cuh"
#include "rms.cuh"
#include "rope.cuh"
#include "staged.cuh"
#include "vjp.cuh"

namespace {

using namespace nvn;

constexpr int kVersion = 200;  // 0.2.0 (nv_plan gained `stages`)
constexpr int kMaxSelftestCtas = 64;  // nv_selftest_bounded_wait: one resident wave

// ---- error reporting ------------------------------------------------------------------
thread_local char g_msg[512] = "";

nv_status fail(nv_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
    return st;
}

nv_status cuda_fail(cudaError_t e, const char* what) {
    return fail(NV_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// ---- device facts, cached per device ---------------------------------------------------
struct DevInfo {
    int sms = 0;
    int smem_optin = 0;   // largest dynamic + static shared memory one CTA may use
    int smem_per_sm = 0;
    bool ready = false;
};
constexpr int kMaxDevices = 64;
DevInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

nv_status current_device(int* dev, DevInfo* info) {
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (*dev < 0 || *dev >= kMaxDevices) return fail(NV_ERR_UNSUPPORTED, "device %d", *dev);
    // each thread keeps its own copy of the (immutable) facts: no lock after the first call
    thread_local DevInfo tl_dev[kMaxDevices];
    if (tl_dev[*dev].ready) {
        *info = tl_dev[*dev];
        return NV_OK;
    }
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DevInfo& d = g_dev[*dev];
    if (!d.ready) {
        e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, *dev);
        if (e == cudaSuccess)
            e = cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, *dev);
        if (e == cudaSuccess)
            e = cudaDeviceGetAttribute(&d.smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor,
                                       *dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
        d.ready = true;
    }
    tl_dev[*dev] = d;
    *info = d;
    return NV_OK;
}

// ---- pointer checks ----------------------------------------------------------------------
// Driver entry points, fetched through the runtime so the library needs no libcuda link.
template <typename F>
F driver_fn(const char* name) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    F fn = nullptr;
    if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        fn = reinterpret_cast<F>(p);
    cudaGetLastError();
    return fn;
}

// cuPointerGetAttributes answers every question the check asks (memory type, device,
// managed or not, the allocation's range) in one driver call per pointer.
using AttrsFn = CUresult (*)(unsigned int, CUpointer_attribute*, void**, CUdeviceptr);
AttrsFn attrs_fn() {
    static AttrsFn fn = driver_fn<AttrsFn>("cuPointerGetAttributes");
    return fn;
}

// cuMemGetAddressRange, for the checks of peers' parts and of page-locked host buffers.
using RangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);
RangeFn range_fn() {
    static RangeFn fn = driver_fn<RangeFn>("cuMemGetAddressRange");
    return fn;
}

struct Buf {
    const void* p;
    size_t bytes;
    const char* name;
    bool output;
    bool row_input;  // an output may be the very same buffer as a row input
};

// The buffer must be device (or managed) memory of the current device and lie inside
// one allocation.
nv_status check_pointer(const Buf& b, int dev) {
    AttrsFn fn = attrs_fn();
    if (!fn) return fail(NV_ERR_CUDA, "the driver does not provide cuPointerGetAttributes");
    unsigned int mtype = 0;
    int ordinal = -1;
    uint64_t managed = 0;  // the driver writes a bool into the first byte
    CUdeviceptr base = 0;
    size_t size = 0;
    CUpointer_attribute which[5] = {CU_POINTER_ATTRIBUTE_MEMORY_TYPE,
                                    CU_POINTER_ATTRIBUTE_DEVICE_ORDINAL,
                                    CU_POINTER_ATTRIBUTE_IS_MANAGED,
                                    CU_POINTER_ATTRIBUTE_RANGE_START_ADDR,
                                    CU_POINTER_ATTRIBUTE_RANGE_SIZE};
    void* out[5] = {&mtype, &ordinal, &managed, &base, &size};
    // an address the driver does not know comes back as success with empty attributes
    if (fn(5, which, out, (CUdeviceptr)(uintptr_t)b.p) != CUDA_SUCCESS || mtype == 0)
        return fail(NV_ERR_INVALID_ARG, "%s (%p) is not a CUDA pointer", b.name, b.p);
    const bool is_managed = (managed & 0xFFu) != 0;
    if (!is_managed && mtype != CU_MEMORYTYPE_DEVICE)
        return fail(NV_ERR_INVALID_ARG, "%s (%p) is not device memory", b.name, b.p);
    if (!is_managed && ordinal != dev)
        return fail(NV_ERR_INVALID_ARG, "%s (%p) belongs to device %d, current device is %d",
                    b.name, b.p, ordinal, dev);
    if (size == 0)
        return fail(NV_ERR_INVALID_ARG, "%s (%p): allocation not found", b.name, b.p);
    const uintptr_t lo = (uintptr_t)b.p;
    if (lo + b.bytes > (uintptr_t)base + size)
        return fail(NV_ERR_INVALID_ARG,
                    "%s (%p): %zu bytes run past the end of its allocation (%zu bytes at %p)",
                    b.name, b.p, b.bytes, size, (void*)(uintptr_t)base);
    return NV_OK;
}

// Process-wide switch for the driver queries of check_pointer (nv_set_pointer_checks).
std::atomic<int> g_pointer_checks{1};

nv_status check_buffers(const Buf* bufs, int n, int dev) {
    if (g_pointer_checks.load(std::memory_order_relaxed)) {
        for (int i = 0; i < n; ++i) {
            if (!bufs[i].p) continue;
            nv_status st = check_pointer(bufs[i], dev);
            if (st != NV_OK) return st;
        }
    }
    // an output may not overlap anything, except that it may be exactly a row input
    for (int i = 0; i < n; ++i) {
        if (!bufs[i].p || !bufs[i].output) continue;
        const uintptr_t a0 = (uintptr_t)bufs[i].p, a1 = a0 + bufs[i].bytes;
        for (int j = 0; j < n; ++j) {
            if (j == i || !bufs[j].p) continue;
            const uintptr_t b0 = (uintptr_t)bufs[j].p, b1 = b0 + bufs[j].bytes;
            if (a0 >= b1 || b0 >= a1) continue;
            if (a0 == b0 && bufs[i].bytes == bufs[j].bytes && bufs[j].row_input) continue;
            return fail(NV_ERR_INVALID_ARG, "output %s overlaps %s", bufs[i].name, bufs[j].name);
        }
    }
    return NV_OK;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

size_t elem_size(nv_dtype dt) { return dt == NV_F32 ? 4 : 2; }

nv_status check_common(int64_t rows, int64_t D, float eps, nv_dtype dt, bool check_eps = true) {
    if (dt == NV_F16) return fail(NV_ERR_UNSUPPORTED, "dtype NV_F16 is not supported");
    if (dt != NV_F32 && dt != NV_BF16) return fail(NV_ERR_INVALID_ARG, "unknown dtype %d", (int)dt);
    if (rows < 0) return fail(NV_ERR_INVALID_ARG, "rows = %lld < 0", (long long)rows);
    if (D < 1) return fail(NV_ERR_INVALID_ARG, "D = %lld < 1", (long long)D);
    if (D > (int64_t)1 << 30) return fail(NV_ERR_UNSUPPORTED, "D = %lld > 2^30", (long long)D);
    if (check_eps && (!std::isfinite(eps) || eps < 0.f))
        return fail(NV_ERR_INVALID_ARG, "eps = %g must be finite and >= 0", (double)eps);
    const size_t s = elem_size(dt);
    if ((uint64_t)rows > (uint64_t)INT64_MAX / ((uint64_t)D * s))
        return fail(NV_ERR_INVALID_ARG, "rows * D overflows");
    return NV_OK;
}

// ---- plans --------------------------------------------------------------------------------
enum Op { OP_RMS = 0, OP_ADD = 1, OP_LAYER = 2, OP_ROPE = 3 };

int pow2_ceil(int v) {
    int p = 1;
    while (p < v) p <<= 1;
    return p;
}

// Largest vectors-per-thread the register kernels are instantiated for, and the
// largest CTA each instance is built for.
int max_vpt(Op) { return 8; }
int max_threads(Op op, int vpt) {
    return op == OP_LAYER ? layer_max_threads(vpt) : rms_max_threads(vpt);
}

// Register-path shape: VPT vectors per thread, G threads per row.
// Automatic choice (measured on B200 over D = 1024..16384, bf16 and fp32): four
// 16-byte vectors per thread and tensor -- enough loads in flight per thread while
// keeping several CTAs per SM -- unless the row would then need more threads than
// the kernel is built for; short rows use fewer vectors so a warp is not mostly idle.
bool rows_shape(Op op, int nvec, int vpt_req, int g_req, int* vpt, int* G,
                bool narrow_rows = false) {
    int v = vpt_req;
    if (v == 0) {
        v = 0;
        // layer_norm does more arithmetic per element and gains from longer rows per
        // thread (eight vectors); the rms kernels from more threads (four)
        const int pref = op == OP_LAYER ? 8 : 4;
        if (narrow_rows && (op == OP_RMS || op == OP_LAYER) && nvec <= 128) {
            // rms_norm and layer_norm rows of up to 128 vectors: four (rms_norm) or eight
            // (layer_norm, more arithmetic a row) vectors a thread, rows narrower than a
            // warp sharing warps.  Measured at 2^25-2^26 elements, CTAs of 128 threads:
            //   rms_norm bf16 D = 64 44.4 us, 128 41.4, 256 42.0, 512 42.1 (one vector a
            //   thread 57-69 us);
            //   layer_norm f32 D = 128 48.6 us, 256 48.6, 512 47.7 (four vectors 58.3,
            //   58.7, 56.6; one or two vectors at 32 threads a row 73.0, 70.3)
            v = std::min(op == OP_LAYER ? 8 : 4, pow2_ceil(nvec));
        } else if (nvec <= 32 * pref) {
            v = std::max(1, pow2_ceil((nvec + 31) / 32));
        } else {
            for (int c = pref; c <= max_vpt(op); c *= 2)
                if ((nvec + c - 1) / c <= max_threads(op, c)) { v = c; break; }
        }
        if (v == 0) return false;
    }
    if (v != 1 && v != 2 && v != 4 && v != 8) return false;
    if (v > max_vpt(op)) return false;
    int g = g_req;
    // register-path (narrow_rows) rows of at most 16 x v vectors: a power of two of threads,
    // several rows to a warp (their reductions run over the row's own lanes); every other
    // row takes whole warps
    const bool sub = narrow_rows;
    if (g == 0) {
        const int n = (nvec + v - 1) / v;
        g = (sub && n <= 16) ? pow2_ceil(std::max(n, 1)) : (n + 31) / 32 * 32;
    }
    const bool sub_ok = sub && g >= 1 && g <= 16 && (g & (g - 1)) == 0;
    if ((!sub_ok && (g % 32 != 0 || g < 32)) || g > max_threads(op, v)) return false;
    if ((int64_t)g * v < nvec) return false;
    *vpt = v;
    *G = g;
    return true;
}

// Staged path: shared memory of one CTA for `stages` rows in flight.
size_t staged_smem(Op op, int64_t D, nv_dtype dt, int stages) {
    const size_t stage = (size_t)(op == OP_ADD ? 2 : 1) * (size_t)D * elem_size(dt);
    return (size_t)stages * (stage + 8);
}
constexpr int kStaticSmemReserve = 2048;  // static shared memory + per-CTA system use

// Slots path shape (bfloat16 layer_norm): VPT vectors a thread (8, or 4 for narrow rows),
// G threads a row (a multiple of 32, or a power of two up to 16), as many row slots as make
// 768 threads (24 warps per SM, one CTA per SM),
// at most 15 when a row spans several warps (one named barrier each); the float32 w/b table
// (64 bytes a vector) must fit the shared memory.
bool slots_shape(int nvec, const nv_plan& req, const DevInfo* di, nv_plan* out) {
    nv_plan p = req;
    // threads a row: a multiple of 32, or a power of two up to 16 when that covers the row
    // (several rows to a warp)
    const auto threads = [nvec](int vv) {
        const int n = (nvec + vv - 1) / vv;
        int p2 = 1;
        while (p2 < n) p2 *= 2;
        return n <= 16 ? p2 : (n + 31) / 32 * 32;
    };
    const auto lanes = [&](int vv) { return threads(vv) * vv; };
    // vectors a thread, measured on B200 (bf16, 2^26-2^27 elements, the prefetch after the
    // warp sums): 8 in CTAs of 768 threads from 256 vectors a row on (D = 4096: 51.9 us
    // against 52.7 with 4 in CTAs of 1024 threads); below, the first of 4, 8, 6 and 3 that
    // covers the row with no idle lane (D = 256, 512, 1024 take 4: 53.6, 54.2, 48.3 us;
    // D = 384, 768, 1536 take 6: 50.2, 50.1, 47.9 us, against 57.3, 57.1, 54.2 with 8 and
    // 55.8, 52.3, 57.1 with 3), else whichever of 4 and 8 leaves fewer lanes idle, 8 on a tie
    int v = p.vec_per_thread ? p.vec_per_thread
                             : nvec >= 256 ? 8
                             : lanes(4) == nvec ? 4
                             : lanes(8) == nvec ? 8
                             : lanes(6) == nvec ? 6
                             : lanes(3) == nvec ? 3
                             : lanes(8) <= lanes(4) ? 8 : 4;
    if (v != 3 && v != 4 && v != 6 && v != 8) return false;
    int g = p.threads_per_row ? p.threads_per_row : threads(v);
    if (g < 1 || (g % 32 && (g > 16 || (g & (g - 1)))) || (int64_t)g * v < nvec ||
        g > kSlotsMaxThreads)
        return false;
    // 768 threads (24 warps, 80 registers) unless asked for more rows per CTA
    int slots = p.rows_per_cta ? p.rows_per_cta : 768 / g;
    if (g > 32) slots = std::min(slots, 15);
    // whole warps only: the row sums and the centred pass's vote are warp-wide shuffles
    if (slots < 1 || slots * g > kSlotsMaxThreads || (g > 32 && slots > 15) ||
        (slots * g) % 32 != 0)
        return false;
    const size_t optin = (size_t)(di ? di->smem_optin : 232448) - kStaticSmemReserve;
    if (slots_table_bytes(nvec) > optin) return false;
    if (p.ctas_per_sm > 1) return false;  // one table per SM
    // stages: 1 (and 0, automatic) = each slot prefetches its next row into L2 once its
    // current row has landed (one bulk prefetch a row), -1 = no prefetch.  Measured, bf16:
    // D = 1024 48.1 against 53.9 us, D = 2048 49.5 against 51.5, D = 4096 52.6 against 56.8
    if (p.stages != 0 && p.stages != 1 && p.stages != -1) return false;
    p.stages = p.stages == 0 ? 1 : p.stages;
    p.vec_per_thread = v;
    p.threads_per_row = g;
    p.rows_per_cta = slots;
    p.ctas_per_sm = 1;
    *out = p;
    return true;
}

// Ring path shape (layer_norm): R warps per row group so that a thread holds about eight
// 16-byte vectors of a row; 16 warps per CTA in row groups; then as many row buffers as
// the shared memory holds (at most 32) in a multiple of the group count, at least two per
// group, with w and b as a float32 table when it takes at most 64 KB.  Requested fields
// are kept.  The multiple matters for correctness: row k uses buffer k mod stages and
// belongs to group k mod groups, so each buffer serves one group only, and that group
// waits on the buffer's phases strictly in order -- a parity wait can never be answered by
// the completion of an earlier phase meant for another group.
bool ring_shape(int nvec, int vecw, const nv_plan& p, const DevInfo* di, RingArgs* out) {
    RingArgs r{};
    if (p.vec_per_thread != 0) return false;
    if (p.threads_per_row != 0) {
        if (p.threads_per_row % 32 != 0 || p.threads_per_row < 32 || p.threads_per_row > 256)
            return false;
        r.R = p.threads_per_row / 32;
    } else {
        r.R = std::min(8, std::max(1, (nvec + 255) / 256));
    }
    const int optin = di ? di->smem_optin : 232448;
    const int per_sm = di ? di->smem_per_sm : 233472;
    const int cps = p.ctas_per_sm > 0 ? p.ctas_per_sm : 1;
    const int64_t budget = std::min(optin, per_sm / cps) - kStaticSmemReserve;
    const int64_t row = (int64_t)nvec * 16;
    const int64_t table = (int64_t)ring_table_bytes(nvec, vecw);
    const int want_groups = p.rows_per_cta > 0 ? p.rows_per_cta : std::max(1, 16 / r.R);
    if (want_groups * r.R > 16) return false;  // CTAs of at most 512 threads
    // fixed bytes besides the buffers and the table (barriers, counts, reduction slots)
    auto fixed = [&](int groups, int stages) {
        RingArgs t{r.R, groups, stages, 0};
        return (int64_t)ring_smem_bytes(nvec, vecw, t) - (int64_t)stages * row;
    };
    for (int wb = 1; wb >= 0; --wb) {
        if (wb && table > 64 * 1024) continue;
        const int64_t room = budget - (wb ? table : 0) - fixed(want_groups, 32);
        int64_t smax = std::min<int64_t>(room / row, 32);
        int groups = want_groups;
        if (p.stages > 0) {
            if (p.stages > smax || p.stages % groups != 0 || p.stages < 2 * groups) continue;
            smax = p.stages;
        } else {
            if (p.rows_per_cta == 0) groups = (int)std::min<int64_t>(groups, smax / 2);
            if (groups < 1) continue;
            smax = smax / groups * groups;
        }
        if (smax < 2 * groups) continue;
        r.groups = groups;
        r.stages = (int)smax;
        r.wb_smem = wb;
        *out = r;
        return true;
    }
    return false;
}

nv_status make_plan(Op op, int64_t rows, int64_t D, nv_dtype dt, bool aligned, const nv_plan* req,
                    nv_plan* out, const DevInfo* di = nullptr) {
    nv_plan p{};
    if (req) p = *req;
    const int vecw = 16 / (int)elem_size(dt);
    const bool vec_ok = aligned && D % vecw == 0 && D / vecw <= 8192;
    const int nvec = vec_ok ? (int)(D / vecw) : 0;
    if (p.path == NV_PATH_AUTO) {
        int v = 0, g = 0;
        nv_plan sp{};
        // bfloat16 layer_norm: the slots kernel for rows of 8 vectors or more, whenever its
        // w/b table fits.  Measured against the register kernel on B200 (2^26 elements):
        // D = 64 58.4 against 368.1 us (2 threads a row), D = 128 55.5 against 188.6 (4),
        // D = 256 53.6 against 101.3, D = 512 54.2 against 71.8, D = 768 56.3 against
        // 77.6, D = 1024 48.1 against 64.6, D = 1536 54.1 against 67.0, D = 2048..16384
        // 10-20 % faster
        if (op == OP_LAYER && dt == NV_BF16 && vec_ok && nvec >= 8 && p.vec_per_thread == 0 &&
            p.threads_per_row == 0 && p.rows_per_cta == 0 && slots_shape(nvec, p, di, &sp))
            p.path = NV_PATH_SLOTS;
        else
            p.path = vec_ok && rows_shape(op, nvec, p.vec_per_thread, p.threads_per_row, &v, &g,
                                          true)
                         ? NV_PATH_ROWS
                         : NV_PATH_GENERIC;
    }
    if (p.path == NV_PATH_ROWS) {
        if (!vec_ok) return fail(NV_ERR_UNSUPPORTED, "register path needs D %% %d == 0 and "
                                 "16-byte aligned pointers", vecw);
        int vpt = 0, G = 0;
        if (!rows_shape(op, nvec, p.vec_per_thread, p.threads_per_row, &vpt, &G, true))
            return fail(NV_ERR_UNSUPPORTED, "no register-path shape for D = %lld (vpt %d, G %d)",
                        (long long)D, p.vec_per_thread, p.threads_per_row);
        p.vec_per_thread = vpt;
        p.threads_per_row = G;
        // CTAs of at least 128 threads; a layer_norm row spanning several warps is alone
        if (p.rows_per_cta == 0)
            p.rows_per_cta = (op == OP_LAYER && G > 32) ? 1 : std::max(1, 128 / G);
        // whole warps only (a row of fewer than 32 lanes reduces with warp-wide shuffles)
        if (p.rows_per_cta * G > max_threads(op, vpt) || p.rows_per_cta < 1 ||
            (G < 32 && (p.rows_per_cta * G) % 32 != 0))
            return fail(NV_ERR_UNSUPPORTED, "rows_per_cta %d x G %d", p.rows_per_cta, G);
        if (op == OP_LAYER && G > 32 && p.rows_per_cta != 1)
            return fail(NV_ERR_UNSUPPORTED, "layer_norm: a row spanning several warps is alone "
                        "in its CTA (rows_per_cta must be 1)");
    } else if (p.path == NV_PATH_GENERIC) {
        p.vec_per_thread = 0;
        p.threads_per_row = 256;
        p.rows_per_cta = 1;
    } else if (p.path == NV_PATH_STAGED) {
        if (!vec_ok) return fail(NV_ERR_UNSUPPORTED, "staged path needs D %% %d == 0 and "
                                 "16-byte aligned pointers", vecw);
        int vpt = 0, G = 0;
        if (!rows_shape(op, nvec, p.vec_per_thread, p.threads_per_row, &vpt, &G) || G > 512)
            return fail(NV_ERR_UNSUPPORTED, "no staged shape for D = %lld (vpt %d, G %d)",
                        (long long)D, p.vec_per_thread, p.threads_per_row);
        p.vec_per_thread = vpt;
        p.threads_per_row = G;
        const int optin = di ? di->smem_optin : 232448;
        const int per_sm = di ? di->smem_per_sm : 233472;
        if (p.ctas_per_sm == 0) p.ctas_per_sm = 1;
        const int budget = std::min(optin, per_sm / p.ctas_per_sm) - kStaticSmemReserve;
        const size_t one = staged_smem(op, D, dt, 1);
        if (p.rows_per_cta == 0) p.rows_per_cta = (int)std::min<size_t>(8, budget / one);
        if (p.rows_per_cta < 2 || staged_smem(op, D, dt, p.rows_per_cta) > (size_t)budget)
            return fail(NV_ERR_UNSUPPORTED, "staged path: %d stages of %zu bytes do not fit "
                        "%d bytes of shared memory", p.rows_per_cta, one, budget);
    } else if (p.path == NV_PATH_SLOTS && op == OP_LAYER) {
        if (!vec_ok || dt != NV_BF16)
            return fail(NV_ERR_UNSUPPORTED, "slots path: bfloat16 layer_norm with D %% 8 == 0 "
                        "and 16-byte aligned pointers");
        if (!slots_shape(nvec, p, di, &p))
            return fail(NV_ERR_UNSUPPORTED, "slots path: no shape for D = %lld (vpt %d, G %d, "
                        "slots %d)", (long long)D, p.vec_per_thread, p.threads_per_row,
                        p.rows_per_cta);
    } else if (p.path == NV_PATH_RING && op == OP_LAYER) {
        if (!vec_ok) return fail(NV_ERR_UNSUPPORTED, "ring path needs D %% %d == 0 and "
                                 "16-byte aligned pointers", vecw);
        RingArgs rg{};
        if (!ring_shape(nvec, vecw, p, di, &rg))
            return fail(NV_ERR_UNSUPPORTED, "ring path: no shape for D = %lld (group %d threads, "
                        "%d groups, %d stages)", (long long)D, p.threads_per_row, p.rows_per_cta,
                        p.stages);
        p.vec_per_thread = 0;
        p.threads_per_row = 32 * rg.R;
        p.rows_per_cta = rg.groups;
        p.stages = rg.stages;
        if (p.ctas_per_sm == 0) p.ctas_per_sm = 1;
    } else {
        return fail(NV_ERR_UNSUPPORTED, "path %d is not available for this op", p.path);
    }
    if (p.path != NV_PATH_RING && p.path != NV_PATH_SLOTS && p.stages != 0)
        return fail(NV_ERR_UNSUPPORTED, "stages is for the ring and slots paths only");
    if (p.ctas_per_sm < 0) return fail(NV_ERR_INVALID_ARG, "ctas_per_sm < 0");
    (void)rows;
    *out = p;
    return NV_OK;
}

// ---- launching -----------------------------------------------------------------------------
template <typename K>
int occupancy(K kernel, int block, size_t smem) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, block, smem) != cudaSuccess) {
        cudaGetLastError();
        n = 1;
    }
    return std::max(n, 1);
}

int64_t grid_for(int64_t units, int sms, int per_sm) {
    return std::max<int64_t>(1, std::min<int64_t>(units, (int64_t)sms * per_sm));
}

// Launch with programmatic stream serialization allowed (unless the plan asks for a
// plain launch): the kernel may be scheduled while the preceding kernel of the stream
// finishes, and waits for it in pdl_wait() before touching global memory.
thread_local bool g_pdl = true;

template <typename... KArgs, typename... Args>
nv_status launch_kernel(void (*kernel)(KArgs...), dim3 grid, int block, size_t smem,
                        cudaStream_t s, Args&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = dim3((unsigned)block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = g_pdl ? 1 : 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return NV_OK;
}

// ctas_per_sm == 0: one CTA per unit of work (the hardware scheduler balances the
// tail); > 0: a persistent grid of that many CTAs per SM looping over the units.
template <typename K>
nv_status launch(K kernel, int64_t units, int block, size_t smem, int ctas_per_sm,
                 const DevInfo& di, cudaStream_t s, const RowArgs& a) {
    const int64_t grid =
        ctas_per_sm > 0 ? grid_for(units, di.sms, ctas_per_sm) : std::min<int64_t>(units, INT32_MAX);
    (void)smem;
    return launch_kernel(kernel, grid, block, smem, s, a);
}

template <typename K>
nv_status launch_staged(K kernel, const nv_plan& p, size_t smem, const DevInfo& di,
                        cudaStream_t s, const RowArgs& a) {
    cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    const int64_t grid = grid_for(a.rows, di.sms, p.ctas_per_sm);
    return launch_kernel(kernel, grid, p.threads_per_row, smem, s, a, p.rows_per_cta);
}

template <typename T, bool ADD>
nv_status run_rms(const nv_plan& p, const DevInfo& di, cudaStream_t s, RowArgs a) {
    if (p.path == NV_PATH_GENERIC)
        return launch(rms_generic_kernel<T, ADD>, a.rows, 256, 0, p.ctas_per_sm, di, s, a);
    if (p.path == NV_PATH_STAGED) {
        const size_t smem = staged_smem(ADD ? OP_ADD : OP_RMS, a.D,
                                        sizeof(T) == 4 ? NV_F32 : NV_BF16, p.rows_per_cta);
        switch (p.vec_per_thread) {
            case 1: return launch_staged(rms_staged_kernel<T, 1, ADD>, p, smem, di, s, a);
            case 2: return launch_staged(rms_staged_kernel<T, 2, ADD>, p, smem, di, s, a);
            case 4: return launch_staged(rms_staged_kernel<T, 4, ADD>, p, smem, di, s, a);
            case 8: return launch_staged(rms_staged_kernel<T, 8, ADD>, p, smem, di, s, a);
        }
        return fail(NV_ERR_UNSUPPORTED, "vec_per_thread %d", p.vec_per_thread);
    }
    a.G = p.threads_per_row;
    a.rows_per_cta = p.rows_per_cta;
    const int block = a.G * a.rows_per_cta;
    const int64_t units = (a.rows + a.rows_per_cta - 1) / a.rows_per_cta;
    switch (p.vec_per_thread) {
        case 1: return launch(rms_rows_kernel<T, 1, ADD>, units, block, 0, p.ctas_per_sm, di, s, a);
        case 2: return launch(rms_rows_kernel<T, 2, ADD>, units, block, 0, p.ctas_per_sm, di, s, a);
        case 4: return launch(rms_rows_kernel<T, 4, ADD>, units, block, 0, p.ctas_per_sm, di, s, a);
        case 8: return launch(rms_rows_kernel<T, 8, ADD>, units, block, 0, p.ctas_per_sm, di, s, a);
    }
    return fail(NV_ERR_UNSUPPORTED, "vec_per_thread %d", p.vec_per_thread);
}

template <typename T>
nv_status run_layer(const nv_plan& p, const DevInfo& di, cudaStream_t s, RowArgs a) {
    if (p.path == NV_PATH_GENERIC)
        return launch(layer_generic_kernel<T>, a.rows, 256, 0, p.ctas_per_sm, di, s, a);
    if (p.path == NV_PATH_SLOTS) {
        if constexpr (sizeof(T) == 2) {
            a.G = p.threads_per_row;
            a.rows_per_cta = p.rows_per_cta;
            const bool pf = p.stages == 1;
            const size_t smem = slots_table_bytes(a.nvec);
            const bool big = a.G * a.rows_per_cta > 768;
            auto pick = [&](auto vpt) {
                constexpr int V = decltype(vpt)::value;
                if (a.G < 32)  // several rows to a warp: the narrow form
                    return big ? (pf ? layer_slots_kernel<V, true, 1024, true>
                                     : layer_slots_kernel<V, false, 1024, true>)
                               : (pf ? layer_slots_kernel<V, true, 768, true>
                                     : layer_slots_kernel<V, false, 768, true>);
                return big ? (pf ? layer_slots_kernel<V, true, 1024> : layer_slots_kernel<V, false, 1024>)
                           : (pf ? layer_slots_kernel<V, true, 768> : layer_slots_kernel<V, false, 768>);
            };
            auto kern = p.vec_per_thread == 8   ? pick(std::integral_constant<int, 8>{})
                        : p.vec_per_thread == 6 ? pick(std::integral_constant<int, 6>{})
                        : p.vec_per_thread == 3 ? pick(std::integral_constant<int, 3>{})
                                                : pick(std::integral_constant<int, 4>{});
            cudaError_t e =
                cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
            const int64_t units = (a.rows + a.rows_per_cta - 1) / a.rows_per_cta;
            const int64_t grid = grid_for(units, di.sms, 1);
            return launch_kernel(kern, grid, a.G * a.rows_per_cta, smem, s, a);
        } else {
            return fail(NV_ERR_UNSUPPORTED, "slots path: bfloat16 only");
        }
    }
    if (p.path == NV_PATH_RING) {
        constexpr int vecw = 16 / sizeof(T);
        RingArgs rg{};
        if (!ring_shape(a.nvec, vecw, p, &di, &rg))
            return fail(NV_ERR_UNSUPPORTED, "ring path: no shape");
        const size_t smem = ring_smem_bytes(a.nvec, vecw, rg);
        auto kern = rg.wb_smem ? layer_ring_kernel<T, true> : layer_ring_kernel<T, false>;
        cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        const int64_t grid = grid_for(a.rows, di.sms, std::max(1, p.ctas_per_sm));
        return launch_kernel(kern, grid, 32 * rg.R * rg.groups, smem, s, a, rg);
    }
    if (p.path == NV_PATH_STAGED) {
        const size_t smem = staged_smem(OP_LAYER, a.D, sizeof(T) == 4 ? NV_F32 : NV_BF16,
                                        p.rows_per_cta);
        switch (p.vec_per_thread) {
            case 1: return launch_staged(layer_staged_kernel<T, 1>, p, smem, di, s, a);
            case 2: return launch_staged(layer_staged_kernel<T, 2>, p, smem, di, s, a);
            case 4: return launch_staged(layer_staged_kernel<T, 4>, p, smem, di, s, a);
            case 8: return launch_staged(layer_staged_kernel<T, 8>, p, smem, di, s, a);
        }
        return fail(NV_ERR_UNSUPPORTED, "vec_per_thread %d", p.vec_per_thread);
    }
    a.G = p.threads_per_row;
    a.rows_per_cta = p.rows_per_cta;
    const int block = a.G * a.rows_per_cta;
    const int64_t units = (a.rows + a.rows_per_cta - 1) / a.rows_per_cta;
    // persistent by default: each CTA takes the bounds of its columns' w and b once and
    // walks many rows (measured 4% faster than one CTA per row on bf16 [16384, 8192])
    auto go = [&](auto kern) {
        const int per_sm = p.ctas_per_sm > 0 ? p.ctas_per_sm : occupancy(kern, block, 0);
        return launch(kern, units, block, 0, std::max(per_sm, 1), di, s, a);
    };
    const bool nar = a.G < 32;  // several rows to a warp: the narrow form
    switch (p.vec_per_thread) {
        case 1: return nar ? go(layer_rows_kernel<T, 1, layer_max_threads(1), true>)
                           : go(layer_rows_kernel<T, 1>);
        case 2: return nar ? go(layer_rows_kernel<T, 2, layer_max_threads(2), true>)
                           : go(layer_rows_kernel<T, 2>);
        case 4: return nar ? go(layer_rows_kernel<T, 4, layer_max_threads(4), true>)
                           : go(layer_rows_kernel<T, 4>);
        case 8:
            if (nar)
                return block <= 128 ? go(layer_rows_kernel<T, 8, 128, true>)
                       : block <= 256 ? go(layer_rows_kernel<T, 8, 256, true>)
                                      : go(layer_rows_kernel<T, 8, layer_max_threads(8), true>);
            return block <= 128   ? go(layer_rows_kernel<T, 8, 128>)
                   : block <= 256 ? go(layer_rows_kernel<T, 8, 256>)
                                  : go(layer_rows_kernel<T, 8>);
    }
    return fail(NV_ERR_UNSUPPORTED, "vec_per_thread %d", p.vec_per_thread);
}

nv_status row_dispatch(Op op, const nv_plan& p, const DevInfo& di, nv_dtype dt, cudaStream_t cs,
                       const RowArgs& a);

nv_status row_op(Op op, const void* x, const void* r, const void* w, const void* b, void* y,
                 void* h, int64_t rows, int64_t D, float eps, nv_dtype dt, nv_stream_t stream,
                 const nv_plan* req) {
    nv_status st = check_common(rows, D, eps, dt);
    if (st != NV_OK) return st;
    if (rows == 0) return NV_OK;
    const size_t s = elem_size(dt);
    const size_t nbytes = (size_t)rows * (size_t)D * s;
    const size_t pbytes = (size_t)D * s;
    if (!x) return fail(NV_ERR_INVALID_ARG, "x is NULL");
    if (!y) return fail(NV_ERR_INVALID_ARG, "y is NULL");
    if (op == OP_ADD && !r) return fail(NV_ERR_INVALID_ARG, "r is NULL");
    if (op == OP_ADD && !h) return fail(NV_ERR_INVALID_ARG, "h is NULL");
    if (op == OP_ADD && y == h) return fail(NV_ERR_INVALID_ARG, "y and h are the same buffer");

    int dev = 0;
    DevInfo di;
    st = current_device(&dev, &di);
    if (st != NV_OK) return st;
    const Buf bufs[] = {
        {x, nbytes, "x", false, true},
        {op == OP_ADD ? r : nullptr, nbytes, "r", false, true},
        {w, pbytes, "w", false, false},
        {op == OP_LAYER ? b : nullptr, pbytes, "b", false, false},
        {y, nbytes, "y", true, false},
        {op == OP_ADD ? h : nullptr, nbytes, "h", true, false},
    };
    st = check_buffers(bufs, 6, dev);
    if (st != NV_OK) return st;

    bool al = aligned16(x) && aligned16(y) && (!w || aligned16(w));
    if (op == OP_ADD) al = al && aligned16(r) && aligned16(h);
    if (op == OP_LAYER) al = al && (!b || aligned16(b));
    nv_plan p;
    st = make_plan(op, rows, D, dt, al, req, &p, &di);
    if (st != NV_OK) return st;
    g_pdl = p.launch != NV_LAUNCH_PLAIN;

    RowArgs a{};
    a.x = x;
    a.r = r;
    a.w = w;
    a.b = b;
    a.y = y;
    a.h = h;
    a.rows = rows;
    a.D = (int)D;
    a.nvec = (int)(D * (int64_t)s / 16);
    a.eps = eps;
    return row_dispatch(op, p, di, dt, reinterpret_cast<cudaStream_t>(stream), a);
}

nv_status row_dispatch(Op op, const nv_plan& p, const DevInfo& di, nv_dtype dt, cudaStream_t cs,
                       const RowArgs& a) {
    const bool bf = dt == NV_BF16;
    switch (op) {
        case OP_RMS:
            return bf ? run_rms<__nv_bfloat16, false>(p, di, cs, a) : run_rms<float, false>(p, di, cs, a);
        case OP_ADD:
            return bf ? run_rms<__nv_bfloat16, true>(p, di, cs, a) : run_rms<float, true>(p, di, cs, a);
        case OP_LAYER:
            return bf ? run_layer<__nv_bfloat16>(p, di, cs, a) : run_layer<float>(p, di, cs, a);
        default:
            return fail(NV_ERR_INVALID_ARG, "op %d", (int)op);
    }
}

// ---- norm_rope -------------------------------------------------------------------------------
struct RopePlan {
    bool rows;
    bool pairs;  // two vectors per lane: rope_pairs_kernel
    int depth;   // > 0: rope_pairs_async_kernel with this many rounds in flight
    int lpr;
    int bt;
    int64_t n_chunks;
};

template <typename T, bool TRAD, int HV, int PART>
nv_status launch_rope_async(cudaStream_t s, const RopeArgs& a, int depth) {
    const size_t smem = (size_t)a.half * sizeof(float4) +
                        (size_t)Elem<T>::kVec / 2 * (size_t)HV * sizeof(float4) +
                        rope_async_ring_bytes(depth);
    auto kern = depth == 4   ? rope_pairs_async_kernel<T, TRAD, HV, 4, PART>
                : depth == 6 ? rope_pairs_async_kernel<T, TRAD, HV, 6, PART>
                : depth == 2 ? rope_pairs_async_kernel<T, TRAD, HV, 2, PART>
                : depth == 5 ? rope_pairs_async_kernel<T, TRAD, HV, 5, PART>
                             : rope_pairs_async_kernel<T, TRAD, HV, 3, PART>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    }
    return launch_kernel(kern, a.L * a.n_chunks, kRopeThreads, smem, s, a);
}

template <typename T, bool TRAD>
nv_status launch_rope_rows(const DevInfo& di, cudaStream_t s, const RopeArgs& a, bool pairs,
                           int depth) {
    // dims < D (the plan only takes the pairs kernels there at 4, 8 or 16 lanes per row):
    // PART 1 while fewer than half the lanes of a row rotate, else 2
    const int part = a.dims == a.D ? 0 : (2 * (a.half / Elem<T>::kVec) < a.nvec / 2 ? 1 : 2);
    if (depth > 0) {
        const int hv = a.nvec / 2;
        if (part == 1)
            return hv == 8    ? launch_rope_async<T, TRAD, 8, 1>(s, a, depth)
                   : hv == 16 ? launch_rope_async<T, TRAD, 16, 1>(s, a, depth)
                              : launch_rope_async<T, TRAD, 4, 1>(s, a, depth);
        if (part == 2)
            return hv == 8    ? launch_rope_async<T, TRAD, 8, 2>(s, a, depth)
                   : hv == 16 ? launch_rope_async<T, TRAD, 16, 2>(s, a, depth)
                              : launch_rope_async<T, TRAD, 4, 2>(s, a, depth);
        return hv == 8    ? launch_rope_async<T, TRAD, 8, 0>(s, a, depth)
               : hv == 16 ? launch_rope_async<T, TRAD, 16, 0>(s, a, depth)
                          : launch_rope_async<T, TRAD, 4, 0>(s, a, depth);
    }
    // the pairs kernel keeps its lanes' weights after the table: VEC/2 records per lane
    const size_t smem = (size_t)a.half * sizeof(float4) +
                        (pairs ? (size_t)Elem<T>::kVec / 2 * (size_t)(a.nvec / 2) * sizeof(float4)
                               : 0);
    // the pairs kernel with lanes per row fixed at compile time where hvec is 4, 8 or 16
    const int hv = pairs && a.lpr == a.nvec / 2 ? a.nvec / 2 : 0;
    auto kern = !pairs                ? rope_rows_kernel<T, TRAD>
                : part == 1 && hv == 8  ? rope_pairs_kernel<T, TRAD, 8, 1>
                : part == 1 && hv == 16 ? rope_pairs_kernel<T, TRAD, 16, 1>
                : part == 1             ? rope_pairs_kernel<T, TRAD, 4, 1>
                : part == 2 && hv == 8  ? rope_pairs_kernel<T, TRAD, 8, 2>
                : part == 2 && hv == 16 ? rope_pairs_kernel<T, TRAD, 16, 2>
                : part == 2             ? rope_pairs_kernel<T, TRAD, 4, 2>
                : hv == 8               ? rope_pairs_kernel<T, TRAD, 8>
                : hv == 16              ? rope_pairs_kernel<T, TRAD, 16>
                : hv == 4               ? rope_pairs_kernel<T, TRAD, 4>
                                        : rope_pairs_kernel<T, TRAD, 0>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
    }
    (void)di;
    return launch_kernel(kern, a.L * a.n_chunks, kRopeThreads, smem, s, a);
}

template <typename T>
nv_status launch_rope_generic(const DevInfo& di, int ctas_per_sm, cudaStream_t s,
                              const RopeArgs& a) {
    auto kern = rope_generic_kernel<T>;
    const int per_sm = ctas_per_sm > 0 ? ctas_per_sm : occupancy(kern, 128, 0);
    return launch_kernel(kern, grid_for(a.BH * a.L, di.sms, per_sm), 128, 0, s, a);
}

nv_status rope_plan(int64_t rows, int64_t L, int64_t D, int dims, bool trad, nv_dtype dt,
                    bool aligned, int sms, const nv_plan* req, nv_plan* out, RopePlan* rp) {
    nv_plan p{};
    if (req) p = *req;
    const int vecw = 16 / (int)elem_size(dt);
    const int64_t nvec = D / vecw;
    const bool vec_ok = aligned && D % vecw == 0 && nvec <= 32 &&
                        (trad || (dims / 2) % vecw == 0);
    // two vectors per lane (both halves of the rotation, or two vectors of interleaved
    // pairs), an even number of vectors; with dims < D the rotated features fill an even
    // number of whole vectors (halves: dims / 2 of them on each side) and the lanes per row
    // are 4, 8 or 16 (the kernels with the lanes fixed at compile time)
    const int64_t hv_all = nvec / 2;
    const bool part_ok = (trad ? dims % (2 * vecw) == 0 : (dims / 2) % vecw == 0) &&
                         (hv_all == 4 || hv_all == 8 || hv_all == 16);
    const bool pairs_ok = aligned && D % vecw == 0 && nvec % 2 == 0 && nvec / 2 <= 32 &&
                          (dims == D || part_ok);
    if (p.path == NV_PATH_AUTO) p.path = (vec_ok || pairs_ok) ? NV_PATH_ROWS : NV_PATH_GENERIC;
    rp->rows = p.path == NV_PATH_ROWS;
    rp->pairs = rp->rows && pairs_ok && p.vec_per_thread != 1;
    // stages: rounds of rows in flight per lane group through the shared-memory ring of
    // rope_pairs_async_kernel (2..6; two vectors per lane of 4, 8 or 16 lanes), -1: the
    // register kernel, 0: automatic.  Measured on [8, 32, 2048, 128]:
    //   dims == D, bfloat16: 2 rounds, 45.4-45.7 us (register kernel 48.2, 3 rounds 45.8);
    //   dims == D, float32:  the register kernel, 86.8 us (the ring 87.0-87.5);
    //   dims < D,  bfloat16: 3 rounds, 45.9 / 47.6 / 47.8 us at dims 32 / 64 / 96 (2 rounds
    //                        46.7 / 48.3 / 48.2, register kernel 57-61);
    //   dims < D,  float32:  4 rounds, 87.6-88.6 us (register kernel 104-107).
    const int hv = (int)(nvec / 2);
    const bool ring_ok = rp->pairs && (hv == 4 || hv == 8 || hv == 16);
    if (p.stages != 0 && p.stages != -1 &&
        (!(p.stages >= 2 && p.stages <= 6) || !ring_ok || p.vec_per_thread == 1))
        return fail(NV_ERR_UNSUPPORTED, "norm_rope stages = %d: 2 to 6 rounds of the "
                    "two-vectors-per-lane kernel at 4, 8 or 16 lanes per row, or -1", p.stages);
    const bool part = dims < D;
    const int auto_depth = !ring_ok ? 0 : part ? (dt == NV_BF16 ? 3 : 4) : (dt == NV_BF16 ? 2 : 0);
    rp->depth = p.stages > 0 ? p.stages : (p.stages == 0 ? auto_depth : 0);
    if (p.path == NV_PATH_ROWS) {
        if (!vec_ok && !rp->pairs)
            return fail(NV_ERR_UNSUPPORTED, "norm_rope register path needs D %% %d == 0, "
                        "D <= %d, 16-byte alignment and (halves) dims/2 %% %d == 0",
                        vecw, 32 * vecw, vecw);
        const int lanes_needed = rp->pairs ? (int)(nvec / 2) : (int)nvec;
        const int lpr = pow2_ceil(std::max(lanes_needed, 1));
        const int slots = kRopeThreads / lpr;
        const int64_t BH = rows / L;
        int64_t bt = p.rows_per_cta;
        if (bt <= 0) {
            const int64_t target = (rows + 8LL * sms - 1) / (8LL * sms);
            bt = std::max<int64_t>(slots * (rp->pairs ? 3 : 4), std::min<int64_t>(target, 256));
            bt = std::min<int64_t>(bt, std::max<int64_t>(BH, 1));
        }
        rp->lpr = lpr;
        rp->bt = (int)bt;
        rp->n_chunks = (BH + bt - 1) / bt;
        if (L * rp->n_chunks >= ((int64_t)1 << 31))
            return fail(NV_ERR_UNSUPPORTED, "norm_rope grid too large");
        p.vec_per_thread = rp->pairs ? 2 : 1;
        p.threads_per_row = lpr;
        p.rows_per_cta = (int)bt;
        p.stages = rp->depth > 0 ? rp->depth : -1;
    } else if (p.path == NV_PATH_GENERIC) {
        p.vec_per_thread = 0;
        p.threads_per_row = 128;
        p.rows_per_cta = 1;
    } else {
        return fail(NV_ERR_UNSUPPORTED, "path %d is not available for norm_rope", p.path);
    }
    *out = p;
    return NV_OK;
}

nv_status rope_op(const void* x, const void* w, const float* freqs, void* y, int64_t rows,
                  int64_t L, int64_t y_len, int64_t D, int32_t dims, int32_t traditional,
                  float base, float scale, int64_t offset, int32_t forward, int32_t normalize,
                  float eps, nv_dtype dt, nv_stream_t stream, const nv_plan* req) {
    nv_status st = check_common(rows, D, eps, dt, normalize != 0);
    if (st != NV_OK) return st;
    if (L < 1) return fail(NV_ERR_INVALID_ARG, "L = %lld < 1", (long long)L);
    if (rows % L != 0)
        return fail(NV_ERR_INVALID_ARG, "rows = %lld is not a multiple of L = %lld",
                    (long long)rows, (long long)L);
    if (dims <= 0 || dims % 2 != 0 || dims > D)
        return fail(NV_ERR_INVALID_ARG, "dims = %d must be even with 0 < dims <= D = %lld", dims,
                    (long long)D);
    if (!freqs && (!(base > 0.f) || !std::isfinite(base)))
        return fail(NV_ERR_INVALID_ARG, "base = %g must be finite and > 0", (double)base);
    if (!std::isfinite(scale)) return fail(NV_ERR_INVALID_ARG, "scale must be finite");
    if (offset < 0) return fail(NV_ERR_INVALID_ARG, "offset = %lld < 0", (long long)offset);
    if (offset > ((int64_t)1 << 52) - L)
        return fail(NV_ERR_INVALID_ARG, "offset + L must stay below 2^52");
    if (y_len < 0) return fail(NV_ERR_INVALID_ARG, "y_len = %lld < 0", (long long)y_len);
    if (y_len > 0 && y_len < offset + L)
        return fail(NV_ERR_INVALID_ARG, "cache length y_len = %lld < offset + L = %lld",
                    (long long)y_len, (long long)(offset + L));
    if (rows == 0) return NV_OK;
    if (!x) return fail(NV_ERR_INVALID_ARG, "x is NULL");
    if (!y) return fail(NV_ERR_INVALID_ARG, "y is NULL");

    int dev = 0;
    DevInfo di;
    st = current_device(&dev, &di);
    if (st != NV_OK) return st;
    const size_t s = elem_size(dt);
    const size_t nbytes = (size_t)rows * (size_t)D * s;
    const bool cache = y_len > 0;
    const size_t ybytes = cache ? (size_t)(rows / L) * (size_t)y_len * (size_t)D * s : nbytes;
    const Buf bufs[] = {
        // a cache has another layout than x: then y may not even alias x
        {x, nbytes, "x", false, !cache},
        {normalize ? w : nullptr, (size_t)D * s, "w", false, false},
        {freqs, (size_t)(dims / 2) * sizeof(float), "freqs", false, false},
        {y, ybytes, "y", true, false},
    };
    st = check_buffers(bufs, 4, dev);
    if (st != NV_OK) return st;

    const bool al = aligned16(x) && aligned16(y) && (!w || !normalize || aligned16(w));
    nv_plan p;
    RopePlan rp{};
    st = rope_plan(rows, L, D, dims, traditional != 0, dt, al, di.sms, req, &p, &rp);
    if (st != NV_OK) return st;
    g_pdl = p.launch != NV_LAUNCH_PLAIN;

    RopeArgs a{};
    a.x = x;
    a.w = normalize ? w : nullptr;
    a.y = y;
    a.BH = rows / L;
    a.L = L;
    a.offset = offset;
    a.n_chunks = rp.n_chunks;
    a.D = (int)D;
    a.nvec = (int)(D * (int64_t)s / 16);
    a.dims = dims;
    a.half = dims / 2;
    a.lpr = rp.lpr;
    a.bt = rp.bt;
    a.base = base;
    a.log2_base = freqs ? 0.0 : std::log2((double)base);
    a.scale = scale;
    a.eps = eps;
    a.normalize = normalize != 0;
    a.traditional = traditional != 0;
    a.freqs = freqs;
    a.forward = forward != 0;
    a.y_len = cache ? y_len : L;
    a.y_off = cache ? offset : 0;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const bool bf = dt == NV_BF16;
    if (rp.rows) {
        if (traditional)
            return bf ? launch_rope_rows<__nv_bfloat16, true>(di, cs, a, rp.pairs, rp.depth)
                      : launch_rope_rows<float, true>(di, cs, a, rp.pairs, rp.depth);
        return bf ? launch_rope_rows<__nv_bfloat16, false>(di, cs, a, rp.pairs, rp.depth)
                  : launch_rope_rows<float, false>(di, cs, a, rp.pairs, rp.depth);
    }
    return bf ? launch_rope_generic<__nv_bfloat16>(di, p.ctas_per_sm, cs, a)
              : launch_rope_generic<float>(di, p.ctas_per_sm, cs, a);
}

// ---- all-reduce of partial sums + add_rms_norm ---------------------------------------------
// A part may live on another GPU (mapped into this process): it must be device memory of
// some device and lie inside one allocation; the other buffers belong to the current one.
nv_status check_part(const void* p, size_t bytes, int i) {
    cudaPointerAttributes at;
    cudaError_t e = cudaPointerGetAttributes(&at, p);
    if (e != cudaSuccess || (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged)) {
        cudaGetLastError();
        return fail(NV_ERR_INVALID_ARG, "parts[%d] (%p) is not device memory", i, p);
    }
    RangeFn fn = range_fn();
    if (fn) {
        CUdeviceptr base = 0;
        size_t size = 0;
        if (fn(&base, &size, (CUdeviceptr)(uintptr_t)p) == CUDA_SUCCESS &&
            (uintptr_t)p + bytes > (uintptr_t)base + size)
            return fail(NV_ERR_INVALID_ARG, "parts[%d] (%p): %zu bytes run past the end of its "
                        "allocation", i, p, bytes);
    }
    return NV_OK;
}

nv_status allreduce_add_rms_norm(const void* const* parts, int32_t nparts, const void* r,
                                 const void* w, void* y, void* h, void* x_out, int64_t rows,
                                 int64_t D, float eps, nv_dtype dt, nv_stream_t stream,
                                 const int64_t* flags = nullptr, int64_t epoch = 0) {
    nv_status st = check_common(rows, D, eps, dt);
    if (st != NV_OK) return st;
    if (nparts < 1 || nparts > kMaxParts)
        return fail(NV_ERR_INVALID_ARG, "nparts = %d must be 1..%d", nparts, kMaxParts);
    if (flags && epoch < 1)
        return fail(NV_ERR_INVALID_ARG, "epoch = %lld must be >= 1", (long long)epoch);
    if (flags && ((uintptr_t)flags & 7u))
        return fail(NV_ERR_INVALID_ARG, "flags must be 8-byte aligned");
    if (rows == 0) return NV_OK;
    if (!parts) return fail(NV_ERR_INVALID_ARG, "parts is NULL");
    for (int i = 0; i < nparts; ++i)
        if (!parts[i]) return fail(NV_ERR_INVALID_ARG, "parts[%d] is NULL", i);
    if (!r) return fail(NV_ERR_INVALID_ARG, "r is NULL");
    if (!y) return fail(NV_ERR_INVALID_ARG, "y is NULL");
    if (!h) return fail(NV_ERR_INVALID_ARG, "h is NULL");
    const size_t s = elem_size(dt);
    const size_t nbytes = (size_t)rows * (size_t)D * s;
    int dev = 0;
    DevInfo di;
    st = current_device(&dev, &di);  // first, as in every entry: no usable device is NV_ERR_CUDA
    if (st != NV_OK) return st;
    for (int i = 0; i < nparts; ++i) {
        st = check_part(parts[i], nbytes, i);
        if (st != NV_OK) return st;
    }
    // outputs may be exactly a row input (h over r, x_out over a part), nothing else
    Buf bufs[kMaxParts + 5];
    int nb = 0;
    bufs[nb++] = {r, nbytes, "r", false, true};
    bufs[nb++] = {w, (size_t)D * s, "w", false, false};
    bufs[nb++] = {y, nbytes, "y", true, false};
    bufs[nb++] = {h, nbytes, "h", true, false};
    bufs[nb++] = {x_out, nbytes, "x_out", true, false};
    bufs[nb++] = {flags, (size_t)nparts * sizeof(int64_t), "flags", false, false};
    st = check_buffers(bufs, nb, dev);
    if (st != NV_OK) return st;
    for (int i = 0; i < nparts; ++i) {  // parts are inputs: only x_out may be one of them
        const uintptr_t p0 = (uintptr_t)parts[i], p1 = p0 + nbytes;
        const void* outs[] = {y, h, x_out};
        const char* names[] = {"y", "h", "x_out"};
        for (int o = 0; o < 3; ++o) {
            if (!outs[o]) continue;
            const uintptr_t o0 = (uintptr_t)outs[o], o1 = o0 + nbytes;
            if (o0 >= p1 || p0 >= o1) continue;
            if (o == 2 && o0 == p0) continue;
            return fail(NV_ERR_INVALID_ARG, "output %s overlaps parts[%d]", names[o], i);
        }
    }

    ReduceNormArgs a{};
    for (int i = 0; i < nparts; ++i) a.parts[i] = parts[i];
    a.nparts = nparts;
    a.r = r;
    a.w = w;
    a.y = y;
    a.h = h;
    a.x_out = x_out;
    a.rows = rows;
    a.D = (int)D;
    a.eps = eps;
    a.flags = reinterpret_cast<const long long*>(flags);
    a.epoch = epoch;
    g_pdl = true;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const bool bf = dt == NV_BF16;
    const int vecw = 16 / (int)s;
    bool al = aligned16(r) && aligned16(y) && aligned16(h) && (!w || aligned16(w)) &&
              (!x_out || aligned16(x_out)) && D % vecw == 0;
    for (int i = 0; i < nparts; ++i) al = al && aligned16(parts[i]);
    const int64_t nvec = D / vecw;
    const int64_t grid = std::min<int64_t>(rows, INT32_MAX);
    if (al && nvec <= 2048) {
        const int vpt = nvec <= 1024 ? 1 : 2;
        a.nvec = (int)nvec;
        a.G = (int)(((nvec + vpt - 1) / vpt + 31) / 32 * 32);
        if (vpt == 1)
            return bf ? launch_kernel(allreduce_rms_rows_kernel<__nv_bfloat16, 1>, grid, a.G, 0, cs, a)
                      : launch_kernel(allreduce_rms_rows_kernel<float, 1>, grid, a.G, 0, cs, a);
        return bf ? launch_kernel(allreduce_rms_rows_kernel<__nv_bfloat16, 2>, grid, a.G, 0, cs, a)
                  : launch_kernel(allreduce_rms_rows_kernel<float, 2>, grid, a.G, 0, cs, a);
    }
    return bf ? launch_kernel(allreduce_rms_generic_kernel<__nv_bfloat16>, grid, 256, 0, cs, a)
              : launch_kernel(allreduce_rms_generic_kernel<float>, grid, 256, 0, cs, a);
}

// ---- host-resident rows: copies and compute pipelined over row chunks ---------------------
// A three-stage pipeline over row chunks, one internal stream per stage: stream IN copies
// chunk after chunk of x and r to the device, stream COMPUTE runs add_rms_norm on chunk k
// once IN has recorded it, stream OUT copies chunk k's y and h back once COMPUTE has
// recorded it.  No stage waits on a later one, so uploads run back to back while the
// downloads of earlier chunks proceed: the PCIe link works in both directions at once.
// The stages start after the work already queued on the caller's stream and the caller's
// stream waits for all of them, so the call is ordered like any other launch on `stream`.
constexpr int kPipeStreams = 3;  // IN, COMPUTE, OUT
constexpr int kPipeMaxChunks = 64;

struct Pipe {
    cudaStream_t s[kPipeStreams] = {};
    cudaEvent_t start = nullptr;
    cudaEvent_t done[kPipeStreams] = {};
    cudaEvent_t in[kPipeMaxChunks] = {};    // chunk k is on the device
    cudaEvent_t comp[kPipeMaxChunks] = {};  // chunk k's outputs are written
};
Pipe g_pipe[kMaxDevices];
std::mutex g_pipe_mu;  // guards creation and the enqueue sequence (events are reused)

nv_status pipe_for(int dev, Pipe** out) {
    Pipe& pp = g_pipe[dev];
    if (!pp.start) {
        cudaError_t e = cudaEventCreateWithFlags(&pp.start, cudaEventDisableTiming);
        for (int i = 0; e == cudaSuccess && i < kPipeStreams; ++i) {
            e = cudaStreamCreateWithFlags(&pp.s[i], cudaStreamNonBlocking);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&pp.done[i], cudaEventDisableTiming);
        }
        for (int k = 0; e == cudaSuccess && k < kPipeMaxChunks; ++k) {
            e = cudaEventCreateWithFlags(&pp.in[k], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&pp.comp[k], cudaEventDisableTiming);
        }
        if (e != cudaSuccess) {
            pp = Pipe{};  // a later call retries; objects made so far are left to the context
            return cuda_fail(e, "creating the pipeline streams");
        }
    }
    *out = &pp;
    return NV_OK;
}

// Page-locked host memory (cudaHostAlloc or cudaHostRegister) holding `bytes` bytes.
nv_status check_host(const void* p, size_t bytes, const char* name) {
    cudaPointerAttributes at;
    cudaError_t e = cudaPointerGetAttributes(&at, p);
    if (e != cudaSuccess || at.type != cudaMemoryTypeHost) {
        cudaGetLastError();
        return fail(NV_ERR_INVALID_ARG, "%s (%p) is not page-locked host memory", name, p);
    }
    RangeFn fn = range_fn();
    if (fn && at.devicePointer) {
        CUdeviceptr base = 0;
        size_t size = 0;
        if (fn(&base, &size, (CUdeviceptr)(uintptr_t)at.devicePointer) == CUDA_SUCCESS &&
            (uintptr_t)at.devicePointer + bytes > (uintptr_t)base + size)
            return fail(NV_ERR_INVALID_ARG, "%s (%p): %zu bytes run past the end of its "
                        "page-locked allocation", name, p, bytes);
    }
    return NV_OK;
}

nv_status add_rms_norm_host(const void* x_host, const void* r_host, const void* w,
                            void* y_host, void* h_host, void* x_dev, void* r_dev, void* y_dev,
                            void* h_dev, int64_t rows, int64_t D, float eps, nv_dtype dt,
                            int64_t chunk_rows, nv_stream_t stream) {
    nv_status st = check_common(rows, D, eps, dt);
    if (st != NV_OK) return st;
    if (chunk_rows < 0) return fail(NV_ERR_INVALID_ARG, "chunk_rows = %lld < 0", (long long)chunk_rows);
    if (rows == 0) return NV_OK;
    const void* ptrs[] = {x_host, r_host, y_host, h_host, x_dev, r_dev, y_dev, h_dev};
    const char* names[] = {"x_host", "r_host", "y_host", "h_host", "x_dev", "r_dev", "y_dev", "h_dev"};
    for (int i = 0; i < 8; ++i)
        if (!ptrs[i]) return fail(NV_ERR_INVALID_ARG, "%s is NULL", names[i]);
    if (y_dev == h_dev || y_host == h_host)
        return fail(NV_ERR_INVALID_ARG, "y and h are the same buffer");
    const size_t s = elem_size(dt);
    const size_t nbytes = (size_t)rows * (size_t)D * s;
    int dev = 0;
    DevInfo di;
    st = current_device(&dev, &di);  // first, as in every entry: no usable device is NV_ERR_CUDA
    if (st != NV_OK) return st;
    for (int i = 0; i < 4; ++i) {
        st = check_host(ptrs[i], nbytes, names[i]);
        if (st != NV_OK) return st;
    }
    // host outputs: each may be exactly its own row input (chunk k is read before it is
    // written, and no other chunk touches its rows), otherwise disjoint from the rest
    const struct { const void* p; bool out; const void* may_equal; } hb[] = {
        {x_host, false, nullptr}, {r_host, false, nullptr},
        {y_host, true, x_host}, {h_host, true, r_host}};
    for (int i = 0; i < 4; ++i) {
        if (!hb[i].out) continue;
        const uintptr_t a0 = (uintptr_t)hb[i].p, a1 = a0 + nbytes;
        for (int j = 0; j < 4; ++j) {
            if (j == i || hb[j].p == hb[i].may_equal) continue;
            const uintptr_t b0 = (uintptr_t)hb[j].p, b1 = b0 + nbytes;
            if (a0 < b1 && b0 < a1)
                return fail(NV_ERR_INVALID_ARG, "host output %s overlaps %s", names[i],
                            names[j]);
        }
    }

    const Buf bufs[] = {
        {x_dev, nbytes, "x_dev", false, true},  {r_dev, nbytes, "r_dev", false, true},
        {w, (size_t)D * s, "w", false, false},  {y_dev, nbytes, "y_dev", true, false},
        {h_dev, nbytes, "h_dev", true, false},
    };
    st = check_buffers(bufs, 5, dev);
    if (st != NV_OK) return st;
    int64_t chunk =
        chunk_rows > 0 ? chunk_rows : std::max<int64_t>(1, (rows + 7) / 8);  // ~8 chunks
    chunk = std::max(chunk, (rows + kPipeMaxChunks - 1) / kPipeMaxChunks);  // <= 64 chunks
    const int64_t row_bytes = D * (int64_t)s;
    bool al = aligned16(x_dev) && aligned16(r_dev) && aligned16(y_dev) && aligned16(h_dev) &&
              (!w || aligned16(w)) && (chunk * row_bytes) % 16 == 0;
    nv_plan p;
    st = make_plan(OP_ADD, std::min(rows, chunk), D, dt, al, nullptr, &p, &di);
    if (st != NV_OK) return st;
    g_pdl = true;

    std::lock_guard<std::mutex> lk(g_pipe_mu);
    Pipe* pp = nullptr;
    st = pipe_for(dev, &pp);
    if (st != NV_OK) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaEventRecord(pp->start, cs);
    for (int i = 0; e == cudaSuccess && i < kPipeStreams; ++i)
        e = cudaStreamWaitEvent(pp->s[i], pp->start, 0);
    if (e != cudaSuccess) return cuda_fail(e, "pipeline start");
    const int64_t nchunks = (rows + chunk - 1) / chunk;
    cudaStream_t s_in = pp->s[0], s_comp = pp->s[1], s_out = pp->s[2];
    for (int64_t k = 0; k < nchunks; ++k) {
        const int64_t r0 = k * chunk, n = std::min(chunk, rows - r0);
        const size_t off = (size_t)r0 * (size_t)row_bytes, len = (size_t)n * (size_t)row_bytes;
        auto at = [off](const void* base) {
            return static_cast<char*>(const_cast<void*>(base)) + off;
        };
        e = cudaMemcpyAsync(at(x_dev), at(x_host), len, cudaMemcpyHostToDevice, s_in);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(at(r_dev), at(r_host), len, cudaMemcpyHostToDevice, s_in);
        if (e == cudaSuccess) e = cudaEventRecord(pp->in[k], s_in);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s_comp, pp->in[k], 0);
        if (e != cudaSuccess) return cuda_fail(e, "pipeline: copy in");
        RowArgs a{};
        a.x = at(x_dev);
        a.r = at(r_dev);
        a.w = w;
        a.y = at(y_dev);
        a.h = at(h_dev);
        a.rows = n;
        a.D = (int)D;
        a.nvec = (int)(row_bytes / 16);
        a.eps = eps;
        st = row_dispatch(OP_ADD, p, di, dt, s_comp, a);
        if (st != NV_OK) return st;
        e = cudaEventRecord(pp->comp[k], s_comp);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s_out, pp->comp[k], 0);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(at(y_host), at(y_dev), len, cudaMemcpyDeviceToHost, s_out);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(at(h_host), at(h_dev), len, cudaMemcpyDeviceToHost, s_out);
        if (e != cudaSuccess) return cuda_fail(e, "pipeline: copy out");
    }
    for (int i = 0; e == cudaSuccess && i < kPipeStreams; ++i) {
        e = cudaEventRecord(pp->done[i], pp->s[i]);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, pp->done[i], 0);
    }
    if (e != cudaSuccess) return cuda_fail(e, "pipeline end");
    return NV_OK;
}

// ---- backward (vjp) -------------------------------------------------------------------------
// Partial rows kept for the column sums: enough CTAs to fill the GPU at every D (up to
// 148 SMs x 32 CTAs for the narrowest rows) while the workspace stays <= 8 MiB per sum
// at D <= 4096 (512 x D x 4 bytes beyond that).
int vjp_parts_cap(int64_t D) {
    return (int)std::max<int64_t>(512, ((int64_t)1 << 21) / std::max<int64_t>(D, 1));
}

int vjp_parts(int64_t rows, int64_t D) {
    return (int)std::min<int64_t>(rows, vjp_parts_cap(D));
}

// Vectors per thread for the vjp kernels (measured on B200, bf16, 2^26 elements):
// rms_norm_vjp runs one thread per vector up to 1024 vectors a row; layer_norm_vjp, with
// five row sums and two reductions a row, is faster with 2 vectors a thread from 129
// vectors on (fewer warps per row to reduce).  4 vectors a thread up to 2048.
int vjp_vpt(Op op, int nvec) {
    if (nvec <= (op == OP_LAYER ? 128 : vjp_max_threads(1))) return 1;
    if (op == OP_LAYER && (nvec + 1) / 2 <= vjp_max_threads(2)) return 2;
    if ((nvec + 3) / 4 <= vjp_max_threads(4)) return 4;
    return 0;
}

size_t vjp_workspace(Op op, int64_t rows, int64_t D) {
    return (size_t)(op == OP_LAYER ? 2 : 1) * (size_t)vjp_parts(rows, D) * (size_t)D *
           sizeof(float);
}

// Kernel 1 runs one wave: `parts` = min(rows, cap, SMs x resident CTAs per SM), so no
// SM idles through a partial second wave.
template <typename T>
nv_status run_vjp(Op op, VjpArgs a, int vpt, int cap, const DevInfo& di, cudaStream_t s,
                  void* dw, void* db) {
    const int G = vpt == 0 ? 256 : ((a.nvec + vpt - 1) / vpt + 31) / 32 * 32;
    // rms_norm_vjp with one vector a thread and CTAs of at most 512 threads reduces two rows
    // at a time (half the barriers per row)
    const bool pairs = op == OP_RMS && vpt == 1 && G <= kVjpPairsMaxThreads;
    auto k1 = vpt == 0 ? (op == OP_RMS ? vjp_generic_kernel<T, false> : vjp_generic_kernel<T, true>)
              : pairs ? rms_vjp_pairs_kernel<T, 1>
              : op == OP_RMS
                  ? (vpt == 1 ? rms_vjp_kernel<T, 1>
                              : vpt == 2 ? rms_vjp_kernel<T, 2> : rms_vjp_kernel<T, 4>)
                  : (vpt == 1 ? layer_vjp_kernel<T, 1>
                              : vpt == 2 ? layer_vjp_kernel<T, 2> : layer_vjp_kernel<T, 4>);
    nv_status st = NV_OK;
    // narrow rows: row groups of a power-of-two G <= 32 threads, several to a CTA of 256,
    // each reducing with shuffles alone (vjp_narrow_kernel), one vector a thread up to 16
    // vectors a row, two above.  Taken where it measured faster than the kernels above
    // (bf16, 2^26 elements, the same box):
    //   rms_norm_vjp   D = 64 206.0 -> 86.2 us, 128 111.5 -> 87.1 (256 and 512 stay: 75.9
    //                  and 71.7 against 93.5 and 104.5 at two and four vectors a thread);
    //   layer_norm_vjp D = 64 366.9 -> 94.5 us, 128 191.1 -> 100.4, 256 103.5 -> 79.5,
    //                  512 100.6 -> 83.8
    const bool narrow = vpt != 0 && (a.nvec <= 16 || (op == OP_LAYER && a.nvec <= 64));
    if (narrow && a.rows > 0) {
        const int nvpt = a.nvec <= 16 ? 1 : 2;
        a.G = pow2_ceil(std::max(1, (a.nvec + nvpt - 1) / nvpt));
        constexpr int kThreads = 256;
        constexpr int NP = Elem<T>::kVec / 2;
        const int R = kThreads / a.G;
        const size_t smem = (size_t)R * (size_t)a.nvec * NP * sizeof(float2);
        auto kn = op == OP_RMS ? (nvpt == 1 ? vjp_narrow_kernel<T, 1, false>
                                            : vjp_narrow_kernel<T, 2, false>)
                               : (nvpt == 1 ? vjp_narrow_kernel<T, 1, true>
                                            : vjp_narrow_kernel<T, 2, true>);
        if (smem > 48 * 1024) {
            cudaError_t e =
                cudaFuncSetAttribute(kn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        }
        const int64_t wave = (int64_t)di.sms * occupancy(kn, kThreads, smem);
        const int64_t groups_needed = (a.rows + R - 1) / R;
        a.parts = (int)std::min<int64_t>(std::min<int64_t>(groups_needed, cap), wave);
        st = launch_kernel(kn, a.parts, kThreads, smem, s, a);
        if (st != NV_OK) return st;
    } else if (a.rows > 0) {
        // VPT = 4 keeps its column partial sums in shared memory (ColAcc)
        constexpr int NP = Elem<T>::kVec / 2;
        const size_t smem = vpt < 4 ? 0
                            : op == OP_RMS ? ColAcc<4, NP, 1>::smem_bytes(G)
                                           : ColAcc<4, NP, 2>::smem_bytes(G);
        if (smem > 48 * 1024) {
            cudaError_t e =
                cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
        }
        const int64_t wave = (int64_t)di.sms * occupancy(k1, G, smem);
        a.parts = (int)std::min<int64_t>(std::min<int64_t>(a.rows, cap), wave);
        st = launch_kernel(k1, a.parts, G, smem, s, a);
        if (st != NV_OK) return st;
    }
    if (!dw && !db) return st;
    // one launch for dw and db: blockIdx.y picks the sum
    ReduceArgs r{};
    r.part = a.part;
    r.parts = a.rows > 0 ? a.parts : 0;
    r.D = a.D;
    r.first = dw ? 0 : 1;
    r.out[0] = dw ? dw : db;
    r.out[1] = db;
    const dim3 grid((unsigned)((a.D + 31) / 32), (dw && db) ? 2u : 1u);
    return launch_kernel(vjp_reduce_kernel<T>, grid, reduce_warps(r.parts) * 32, 0, s, r);
}

nv_status vjp_op(Op op, const void* x, const void* w, const void* g, void* dx, void* dw, void* db,
                 void* ws, size_t ws_bytes, int64_t rows, int64_t D, float eps, nv_dtype dt,
                 nv_stream_t stream) {
    nv_status st = check_common(rows, D, eps, dt);
    if (st != NV_OK) return st;
    if ((dw != nullptr) != (w != nullptr))
        return fail(NV_ERR_INVALID_ARG, "dw must be given exactly when w is (w = NULL is the "
                    "scalar 1, which has no gradient)");
    const size_t s = elem_size(dt);
    const int vecw = 16 / (int)s;
    // the register kernels need whole 16-byte vectors (and aligned pointers, below); any
    // other row goes to the generic kernel
    const bool vec_ok = D % vecw == 0 && vjp_vpt(op, (int)(D / vecw)) != 0;
    const bool sums = dw || db;
    const size_t need = sums ? vjp_workspace(op, rows, D) : 0;
    if (sums && rows > 0) {
        if (!ws) return fail(NV_ERR_INVALID_ARG, "workspace is NULL (%zu bytes needed)", need);
        if (ws_bytes < need)
            return fail(NV_ERR_INVALID_ARG, "workspace of %zu bytes < %zu needed", ws_bytes, need);
    }
    if (rows > 0) {
        if (!x) return fail(NV_ERR_INVALID_ARG, "x is NULL");
        if (!g) return fail(NV_ERR_INVALID_ARG, "g is NULL");
        if (!dx) return fail(NV_ERR_INVALID_ARG, "dx is NULL");
    }
    if (rows == 0 && !sums) return NV_OK;

    int dev = 0;
    DevInfo di;
    st = current_device(&dev, &di);
    if (st != NV_OK) return st;
    const size_t nbytes = (size_t)rows * (size_t)D * s;
    const Buf bufs[] = {
        {rows ? x : nullptr, nbytes, "x", false, true},
        {rows ? g : nullptr, nbytes, "g", false, true},
        {w, (size_t)D * s, "w", false, false},
        {rows ? dx : nullptr, nbytes, "dx", true, false},
        {dw, (size_t)D * s, "dw", true, false},
        {db, (size_t)D * s, "db", true, false},
        {(sums && rows) ? ws : nullptr, need, "workspace", true, false},
    };
    st = check_buffers(bufs, 7, dev);
    if (st != NV_OK) return st;
    const bool al = (!rows || (aligned16(x) && aligned16(g) && aligned16(dx))) &&
                    (!w || aligned16(w));

    VjpArgs a{};
    a.x = x;
    a.w = w;
    a.g = g;
    a.dx = dx;
    a.part = (sums && rows) ? static_cast<float*>(ws) : nullptr;
    a.rows = rows;
    a.D = (int)D;
    a.nvec = (int)(D / vecw);
    a.parts = 0;  // set from the occupancy in run_vjp
    a.want_dw = dw != nullptr;
    a.want_db = db != nullptr;
    a.eps = eps;
    g_pdl = true;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const int vpt = (vec_ok && al) ? vjp_vpt(op, a.nvec) : 0;  // 0: the generic kernel
    const int cap = vjp_parts_cap(D);
    return dt == NV_BF16 ? run_vjp<__nv_bfloat16>(op, a, vpt, cap, di, cs, dw, db)
                         : run_vjp<float>(op, a, vpt, cap, di, cs, dw, db);
}

// ---- rms_norm_vjp without caller-provided workspace -------------------------------------------
// Scratch for the dw partials of nv_rms_norm_vjp_static: a fixed array in device memory
// that every GPU loading the library holds until the process exits.  Host code must not
// use the symbol as an address; the device address comes from cudaGetSymbolAddress.
constexpr int64_t kStaticScratchFloats = (int64_t)1 << 20;  // 4 MiB
constexpr int64_t kStaticMaxD = 16384;
static __device__ __align__(256) float nvn_static_scratch[kStaticScratchFloats];

// The address is looked up once per device and context: a device reset tears down the
// primary context (and the module holding the array), and the next context loads it anew.
struct StaticSlot {
    CUcontext ctx = nullptr;
    float* ptr = nullptr;
};
StaticSlot g_static_scratch[kMaxDevices];
std::mutex g_static_mu;

using CtxFn = CUresult (*)(CUcontext*);

// Device address of the scratch array on the current device (and context), fetched on the
// first call there.
nv_status static_scratch(int dev, float** out) {
    static CtxFn ctx_fn = driver_fn<CtxFn>("cuCtxGetCurrent");
    if (!ctx_fn) return fail(NV_ERR_CUDA, "the driver does not provide cuCtxGetCurrent");
    CUcontext ctx = nullptr;
    if (ctx_fn(&ctx) != CUDA_SUCCESS) ctx = nullptr;
    std::lock_guard<std::mutex> lk(g_static_mu);
    StaticSlot& slot = g_static_scratch[dev];
    if (!slot.ptr || !ctx || slot.ctx != ctx) {
        // the lookup also makes the runtime's context current if nothing has yet
        void* p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, nvn_static_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
        if (ctx_fn(&ctx) != CUDA_SUCCESS || !ctx)
            return fail(NV_ERR_CUDA, "no current CUDA context on device %d", dev);
        slot.ptr = static_cast<float*>(p);
        slot.ctx = ctx;
    }
    *out = slot.ptr;
    return NV_OK;
}

nv_status rms_vjp_static(const void* x, const void* w, const void* g, void* dx, void* dw,
                         int64_t rows, int64_t D, float eps, nv_dtype dt, nv_stream_t stream) {
    nv_status st = check_common(rows, D, eps, dt);
    if (st != NV_OK) return st;
    if (D > kStaticMaxD)
        return fail(NV_ERR_UNSUPPORTED, "nv_rms_norm_vjp_static: D = %lld exceeds %lld, the "
                    "widest row its fixed %lld-float scratch is sized for", (long long)D,
                    (long long)kStaticMaxD, (long long)kStaticScratchFloats);
    if ((dw != nullptr) != (w != nullptr))
        return fail(NV_ERR_INVALID_ARG, "dw must be given exactly when w is (w = NULL is the "
                    "scalar 1, which has no gradient)");
    const size_t s = elem_size(dt);
    const int vecw = 16 / (int)s;
    if (D % vecw != 0 || vjp_vpt(OP_RMS, (int)(D / vecw)) == 0)
        return fail(NV_ERR_UNSUPPORTED, "vjp needs D %% %d == 0 and D <= %d", vecw,
                    2048 * vecw);
    if (rows > 0 && (!x || !g || !dx))
        return fail(NV_ERR_INVALID_ARG, "x, g and dx must not be NULL");
    if (rows == 0 && !dw) return NV_OK;

    int dev = 0;
    DevInfo di;
    st = current_device(&dev, &di);
    if (st != NV_OK) return st;
    float* scratch = nullptr;
    if (dw) {
        st = static_scratch(dev, &scratch);
        if (st != NV_OK) return st;
    }
    const size_t nbytes = (size_t)rows * (size_t)D * s;
    const Buf bufs[] = {
        {rows ? x : nullptr, nbytes, "x", false, true},
        {rows ? g : nullptr, nbytes, "g", false, true},
        {w, (size_t)D * s, "w", false, false},
        {rows ? dx : nullptr, nbytes, "dx", true, false},
        {dw, (size_t)D * s, "dw", true, false},
    };
    st = check_buffers(bufs, 5, dev);
    if (st != NV_OK) return st;
    if (!((!rows || (aligned16(x) && aligned16(g) && aligned16(dx))) && (!w || aligned16(w))))
        return fail(NV_ERR_UNSUPPORTED, "vjp needs 16-byte aligned x, g, dx and w");

    VjpArgs a{};
    a.x = x;
    a.w = w;
    a.g = g;
    a.dx = dx;
    a.rows = rows;
    a.D = (int)D;
    a.nvec = (int)(D / vecw);
    // as many partial rows as the scratch holds (at least 64 at the widest D)
    const int cap = (int)std::min<int64_t>(vjp_parts_cap(D), kStaticScratchFloats / D);
    a.parts = 0;
    a.part = (dw && rows) ? scratch : nullptr;
    a.want_dw = dw != nullptr;
    a.want_db = 0;
    a.eps = eps;
    g_pdl = true;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const int vpt = vjp_vpt(OP_RMS, a.nvec);
    return dt == NV_BF16 ? run_vjp<__nv_bfloat16>(OP_RMS, a, vpt, cap, di, cs, dw, nullptr)
                         : run_vjp<float>(OP_RMS, a, vpt, cap, di, cs, dw, nullptr);
}

}  // namespace

// ---- exported C ABI -------------------------------------------------------------------------
extern "C" {

nv_status nv_rms_norm_ex(const void* x, const void* w, void* y, int64_t rows, int64_t D,
                         float eps, nv_dtype dt, nv_stream_t stream, const nv_plan* plan) {
    return row_op(OP_RMS, x, nullptr, w, nullptr, y, nullptr, rows, D, eps, dt, stream, plan);
}

nv_status nv_rms_norm(const void* x, const void* w, void* y, int64_t rows, int64_t D, float eps,
                      nv_dtype dt, nv_stream_t stream) {
    return nv_rms_norm_ex(x, w, y, rows, D, eps, dt, stream, nullptr);
}

nv_status nv_add_rms_norm_ex(const void* x, const void* r, const void* w, void* y, void* h,
                             int64_t rows, int64_t D, float eps, nv_dtype dt, nv_stream_t stream,
                             const nv_plan* plan) {
    return row_op(OP_ADD, x, r, w, nullptr, y, h, rows, D, eps, dt, stream, plan);
}

nv_status nv_add_rms_norm(const void* x, const void* r, const void* w, void* y, void* h,
                          int64_t rows, int64_t D, float eps, nv_dtype dt, nv_stream_t stream) {
    return nv_add_rms_norm_ex(x, r, w, y, h, rows, D, eps, dt, stream, nullptr);
}

nv_status nv_layer_norm_ex(const void* x, const void* w, const void* b, void* y, int64_t rows,
                           int64_t D, float eps, nv_dtype dt, nv_stream_t stream,
                           const nv_plan* plan) {
    return row_op(OP_LAYER, x, nullptr, w, b, y, nullptr, rows, D, eps, dt, stream, plan);
}

nv_status nv_layer_norm(const void* x, const void* w, const void* b, void* y, int64_t rows,
                        int64_t D, float eps, nv_dtype dt, nv_stream_t stream) {
    return nv_layer_norm_ex(x, w, b, y, rows, D, eps, dt, stream, nullptr);
}

nv_status nv_norm_rope_ex(const void* x, const void* w, void* y, int64_t rows, int64_t L,
                          int64_t D, int32_t dims, int32_t traditional, float base, float scale,
                          int64_t offset, int32_t normalize, float eps, nv_dtype dt,
                          nv_stream_t stream, const nv_plan* plan) {
    return rope_op(x, w, nullptr, y, rows, L, 0, D, dims, traditional, base, scale, offset, 1,
                   normalize, eps, dt, stream, plan);
}

nv_status nv_rope_ex(const void* x, const void* w, const float* freqs, void* y, int64_t rows,
                     int64_t L, int64_t y_len, int64_t D, int32_t dims, int32_t traditional,
                     float base, float scale, int64_t offset, int32_t forward, int32_t normalize,
                     float eps, nv_dtype dt, nv_stream_t stream, const nv_plan* plan) {
    return rope_op(x, w, freqs, y, rows, L, y_len, D, dims, traditional, base, scale, offset,
                   forward, normalize, eps, dt, stream, plan);
}

nv_status nv_rope(const void* x, const void* w, const float* freqs, void* y, int64_t rows,
                  int64_t L, int64_t y_len, int64_t D, int32_t dims, int32_t traditional,
                  float base, float scale, int64_t offset, int32_t forward, int32_t normalize,
                  float eps, nv_dtype dt, nv_stream_t stream) {
    return rope_op(x, w, freqs, y, rows, L, y_len, D, dims, traditional, base, scale, offset,
                   forward, normalize, eps, dt, stream, nullptr);
}

nv_status nv_norm_rope(const void* x, const void* w, void* y, int64_t rows, int64_t L, int64_t D,
                       int32_t dims, int32_t traditional, float base, float scale, int64_t offset,
                       int32_t normalize, float eps, nv_dtype dt, nv_stream_t stream) {
    return nv_norm_rope_ex(x, w, y, rows, L, D, dims, traditional, base, scale, offset, normalize,
                           eps, dt, stream, nullptr);
}

nv_status nv_describe_plan(int32_t op, int64_t rows, int64_t D, nv_dtype dt, nv_plan* plan) {
    if (!plan) return fail(NV_ERR_INVALID_ARG, "plan is NULL");
    nv_status st = check_common(rows, D, 0.f, dt);
    if (st != NV_OK) return st;
    if (op < 0 || op > 3) return fail(NV_ERR_INVALID_ARG, "op %d", op);
    if (op == OP_ROPE) {
        RopePlan rp{};
        // position count unknown here: describe one position holding every row
        return rope_plan(rows, 1, D, (int)(D - D % 2), false, dt, true, 148, nullptr, plan, &rp);
    }
    return make_plan((Op)op, rows, D, dt, true, nullptr, plan);
}

nv_status nv_rope_llama3_freqs(int32_t dims, float base, float factor, float low_freq_factor,
                               float high_freq_factor, int64_t original_max_position,
                               float* freqs) {
    if (dims < 2 || dims % 2 != 0)
        return fail(NV_ERR_INVALID_ARG, "dims = %d must be even and >= 2", dims);
    if (!(base > 0.f) || !std::isfinite(base))
        return fail(NV_ERR_INVALID_ARG, "base = %g must be finite and > 0", (double)base);
    if (!(factor >= 1.f) || !std::isfinite(factor))
        return fail(NV_ERR_INVALID_ARG, "factor = %g must be finite and >= 1", (double)factor);
    if (!(low_freq_factor > 0.f) || !(high_freq_factor > low_freq_factor) ||
        !std::isfinite(high_freq_factor))
        return fail(NV_ERR_INVALID_ARG, "need 0 < low_freq_factor (%g) < high_freq_factor (%g)",
                    (double)low_freq_factor, (double)high_freq_factor);
    if (original_max_position <= 0)
        return fail(NV_ERR_INVALID_ARG, "original_max_position = %lld must be > 0",
                    (long long)original_max_position);
    if (!freqs) return fail(NV_ERR_INVALID_ARG, "freqs is NULL");
    const double orig = (double)original_max_position, f = factor;
    const double short_wave = orig / high_freq_factor;  // shorter: unchanged
    const double long_wave = orig / low_freq_factor;    // longer: divided by factor
    const double pi2 = 2.0 * 3.14159265358979323846;
    for (int32_t i = 0; i < dims / 2; ++i) {
        const double th = std::pow((double)base, -2.0 * (double)i / (double)dims);
        const double lambda = pi2 / th;
        double out;
        if (lambda < short_wave) {
            out = th;
        } else if (lambda > long_wave) {
            out = th / f;
        } else {  // blend linearly in orig / lambda between the two thresholds
            const double t = (orig / lambda - low_freq_factor) /
                             ((double)high_freq_factor - (double)low_freq_factor);
            out = (1.0 - t) * (th / f) + t * th;
        }
        freqs[i] = (float)out;
    }
    return NV_OK;
}

nv_status nv_rope_yarn_freqs(int32_t dims, float base, float factor,
                             int64_t original_max_position, float alpha, float beta,
                             float* freqs, float* mscale) {
    if (dims < 2 || dims % 2 != 0)
        return fail(NV_ERR_INVALID_ARG, "dims = %d must be even and >= 2", dims);
    if (!(base > 0.f) || !std::isfinite(base))
        return fail(NV_ERR_INVALID_ARG, "base = %g must be finite and > 0", (double)base);
    if (!(factor >= 1.f) || !std::isfinite(factor))
        return fail(NV_ERR_INVALID_ARG, "factor = %g must be finite and >= 1", (double)factor);
    if (!(alpha > 0.f) || !(beta > alpha) || !std::isfinite(beta))
        return fail(NV_ERR_INVALID_ARG, "need 0 < alpha (%g) < beta (%g)", (double)alpha,
                    (double)beta);
    if (original_max_position <= 0)
        return fail(NV_ERR_INVALID_ARG, "original_max_position = %lld must be > 0",
                    (long long)original_max_position);
    if (!freqs) return fail(NV_ERR_INVALID_ARG, "freqs is NULL");
    const double ctx = (double)original_max_position, s = factor;
    const double per_turn = 1.0 / (2.0 * 3.14159265358979323846);
    for (int32_t i = 0; i < dims / 2; ++i) {
        const double th = std::pow((double)base, -2.0 * (double)i / (double)dims);
        const double turns = ctx * th * per_turn;  // rotations of pair i over the context
        double out;
        if (turns > beta) {
            out = th;                                 // fast pairs: extrapolate
        } else if (turns < alpha) {
            out = th / s;                             // slow pairs: interpolate
        } else {
            const double g = (turns - alpha) / ((double)beta - (double)alpha);
            out = th / s + g * (th - th / s);
        }
        freqs[i] = (float)out;
    }
    if (mscale) *mscale = (float)(1.0 + 0.1 * std::log(s));
    return NV_OK;
}

nv_status nv_rope_suscaled_freqs(int32_t dims, float base, const float* short_factors,
                                 const float* long_factors, int64_t seq_len,
                                 int64_t max_position, int64_t original_max_position,
                                 float* freqs, float* mscale) {
    if (dims < 2 || dims % 2 != 0)
        return fail(NV_ERR_INVALID_ARG, "dims = %d must be even and >= 2", dims);
    if (!(base > 0.f) || !std::isfinite(base))
        return fail(NV_ERR_INVALID_ARG, "base = %g must be finite and > 0", (double)base);
    if (original_max_position < 2)
        return fail(NV_ERR_INVALID_ARG, "original_max_position = %lld must be >= 2",
                    (long long)original_max_position);
    if (max_position < 1)
        return fail(NV_ERR_INVALID_ARG, "max_position = %lld must be >= 1", (long long)max_position);
    if (seq_len < 0) return fail(NV_ERR_INVALID_ARG, "seq_len = %lld < 0", (long long)seq_len);
    if (!short_factors || !long_factors)
        return fail(NV_ERR_INVALID_ARG, "short_factors and long_factors must not be NULL");
    if (!freqs) return fail(NV_ERR_INVALID_ARG, "freqs is NULL");
    // the long factors once the sequence runs past the original context
    const float* lam = seq_len > original_max_position ? long_factors : short_factors;
    for (int32_t i = 0; i < dims / 2; ++i)
        if (!(lam[i] > 0.f) || !std::isfinite(lam[i]))
            return fail(NV_ERR_INVALID_ARG, "factor %d = %g must be finite and > 0", i,
                        (double)lam[i]);
    for (int32_t i = 0; i < dims / 2; ++i) {
        const double th = 1.0 / std::pow((double)base, 2.0 * (double)i / (double)dims);
        freqs[i] = (float)(th / (double)lam[i]);
    }
    if (mscale) {
        const double ratio = (double)max_position / (double)original_max_position;
        *mscale = ratio > 1.0
                      ? (float)std::sqrt(1.0 + std::log(ratio) / std::log((double)original_max_position))
                      : 1.f;
    }
    return NV_OK;
}

nv_status nv_allreduce_add_rms_norm(const void* const* parts, int32_t nparts, const void* r,
                                    const void* w, void* y, void* h, void* x_out, int64_t rows,
                                    int64_t D, float eps, nv_dtype dt, nv_stream_t stream) {
    return allreduce_add_rms_norm(parts, nparts, r, w, y, h, x_out, rows, D, eps, dt, stream);
}

nv_status nv_allreduce_add_rms_norm_peers(const void* const* parts, int32_t nparts,
                                          const void* r, const void* w, void* y, void* h,
                                          void* x_out, int64_t rows, int64_t D, float eps,
                                          nv_dtype dt, const int64_t* flags, int64_t epoch,
                                          nv_stream_t stream) {
    if (!flags) return fail(NV_ERR_INVALID_ARG, "flags is NULL");
    return allreduce_add_rms_norm(parts, nparts, r, w, y, h, x_out, rows, D, eps, dt, stream,
                                  flags, epoch);
}

nv_status nv_tp_publish(int64_t* const* flags, int32_t world, int32_t rank, int64_t epoch,
                        nv_stream_t stream) {
    if (world < 1 || world > kMaxParts)
        return fail(NV_ERR_INVALID_ARG, "world = %d must be 1..%d", world, kMaxParts);
    if (rank < 0 || rank >= world)
        return fail(NV_ERR_INVALID_ARG, "rank = %d outside 0..%d", rank, world - 1);
    if (epoch < 1) return fail(NV_ERR_INVALID_ARG, "epoch = %lld must be >= 1", (long long)epoch);
    if (!flags) return fail(NV_ERR_INVALID_ARG, "flags is NULL");
    PublishArgs a{};
    for (int p = 0; p < world; ++p) {
        if (!flags[p]) return fail(NV_ERR_INVALID_ARG, "flags[%d] is NULL", p);
        if ((uintptr_t)flags[p] & 7u)
            return fail(NV_ERR_INVALID_ARG, "flags[%d] must be 8-byte aligned", p);
        a.flags[p] = reinterpret_cast<long long*>(flags[p]);
    }
    int dev = 0;
    DevInfo di;
    nv_status st = current_device(&dev, &di);
    if (st != NV_OK) return st;
    for (int p = 0; p < world; ++p) {
        st = check_part(flags[p], (size_t)world * sizeof(int64_t), p);
        if (st != NV_OK) return st;
    }
    a.world = world;
    a.rank = rank;
    a.epoch = epoch;
    g_pdl = true;
    return launch_kernel(tp_publish_kernel, 1, 32, 0, reinterpret_cast<cudaStream_t>(stream), a);
}

nv_status nv_ipc_export(const void* ptr, void* handle, uint64_t* offset) {
    if (!ptr || !handle || !offset)
        return fail(NV_ERR_INVALID_ARG, "ptr, handle and offset must not be NULL");
    RangeFn fn = range_fn();
    if (!fn) return fail(NV_ERR_CUDA, "the driver does not provide cuMemGetAddressRange");
    CUdeviceptr base = 0;
    size_t size = 0;
    if (fn(&base, &size, (CUdeviceptr)(uintptr_t)ptr) != CUDA_SUCCESS)
        return fail(NV_ERR_INVALID_ARG, "ptr (%p): allocation not found", ptr);
    cudaIpcMemHandle_t hd;
    cudaError_t e = cudaIpcGetMemHandle(&hd, (void*)(uintptr_t)base);
    if (e != cudaSuccess) return cuda_fail(e, "cudaIpcGetMemHandle");
    static_assert(sizeof(hd) == NV_IPC_HANDLE_BYTES, "IPC handle size");
    std::memcpy(handle, &hd, sizeof(hd));
    *offset = (uint64_t)((uintptr_t)ptr - (uintptr_t)base);
    return NV_OK;
}

nv_status nv_ipc_import(const void* handle, uint64_t offset, void** ptr) {
    if (!handle || !ptr) return fail(NV_ERR_INVALID_ARG, "handle and ptr must not be NULL");
    cudaIpcMemHandle_t hd;
    std::memcpy(&hd, handle, sizeof(hd));
    void* base = nullptr;
    cudaError_t e = cudaIpcOpenMemHandle(&base, hd, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) return cuda_fail(e, "cudaIpcOpenMemHandle");
    *ptr = static_cast<char*>(base) + offset;
    return NV_OK;
}

nv_status nv_ipc_close(void* ptr, uint64_t offset) {
    if (!ptr) return fail(NV_ERR_INVALID_ARG, "ptr is NULL");
    cudaError_t e = cudaIpcCloseMemHandle(static_cast<char*>(ptr) - offset);
    if (e != cudaSuccess) return cuda_fail(e, "cudaIpcCloseMemHandle");
    return NV_OK;
}

nv_status nv_add_rms_norm_host(const void* x_host, const void* r_host, const void* w,
                               void* y_host, void* h_host, void* x_dev, void* r_dev, void* y_dev,
                               void* h_dev, int64_t rows, int64_t D, float eps, nv_dtype dt,
                               int64_t chunk_rows, nv_stream_t stream) {
    return add_rms_norm_host(x_host, r_host, w, y_host, h_host, x_dev, r_dev, y_dev, h_dev, rows,
                             D, eps, dt, chunk_rows, stream);
}

nv_status nv_rms_norm_vjp_static(const void* x, const void* w, const void* g, void* dx, void* dw,
                                 int64_t rows, int64_t D, float eps, nv_dtype dt,
                                 nv_stream_t stream) {
    return rms_vjp_static(x, w, g, dx, dw, rows, D, eps, dt, stream);
}

size_t nv_norm_vjp_workspace_size(int32_t op, int64_t rows, int64_t D) {
    if ((op != OP_RMS && op != OP_LAYER) || rows <= 0 || D <= 0) return 0;
    return vjp_workspace((Op)op, rows, D);
}

nv_status nv_rms_norm_vjp(const void* x, const void* w, const void* g, void* dx, void* dw,
                          void* workspace, size_t workspace_bytes, int64_t rows, int64_t D,
                          float eps, nv_dtype dt, nv_stream_t stream) {
    return vjp_op(OP_RMS, x, w, g, dx, dw, nullptr, workspace, workspace_bytes, rows, D, eps, dt,
                  stream);
}

nv_status nv_layer_norm_vjp(const void* x, const void* w, const void* g, void* dx, void* dw,
                            void* db, void* workspace, size_t workspace_bytes, int64_t rows,
                            int64_t D, float eps, nv_dtype dt, nv_stream_t stream) {
    return vjp_op(OP_LAYER, x, w, g, dx, dw, db, workspace, workspace_bytes, rows, D, eps, dt,
                  stream);
}

const char* nv_status_string(nv_status status) {
    switch (status) {
        case NV_OK: return "NV_OK";
        case NV_ERR_INVALID_ARG: return "NV_ERR_INVALID_ARG";
        case NV_ERR_UNSUPPORTED: return "NV_ERR_UNSUPPORTED";
        case NV_ERR_CUDA: return "NV_ERR_CUDA";
    }
    return "NV_STATUS_UNKNOWN";
}

const char* nv_last_error(void) { return g_msg; }

nv_status nv_fault_count(uint32_t* count, int32_t reset) {
    if (!count) return fail(NV_ERR_INVALID_ARG, "count is NULL");
    cudaError_t e = cudaMemcpyFromSymbol(count, nvn::nvn_fault_count, sizeof(uint32_t));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyFromSymbol");
    if (reset) {
        const uint32_t zero = 0;
        e = cudaMemcpyToSymbol(nvn::nvn_fault_count, &zero, sizeof(uint32_t));
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyToSymbol");
    }
    return NV_OK;
}

nv_status nv_selftest_bounded_wait(int32_t ctas, nv_stream_t stream) {
    if (ctas < 1 || ctas > kMaxSelftestCtas)
        return fail(NV_ERR_INVALID_ARG, "ctas = %d outside 1..%d", ctas, kMaxSelftestCtas);
    bounded_wait_selftest_kernel<<<ctas, 32, 0, (cudaStream_t)stream>>>();
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "bounded_wait_selftest_kernel launch");
    return NV_OK;
}

int32_t nv_version(void) { return kVersion; }

nv_status nv_set_pointer_checks(int32_t enabled, int32_t* previous) {
    const int old = g_pointer_checks.exchange(enabled ? 1 : 0);
    if (previous) *previous = old;
    return NV_OK;
}

}  // extern "C"
