/*
 * Host cost of one call through the C ABI, from plain C (no Python, no ctypes): the time
 * the calling thread spends inside nv_rms_norm / nv_add_rms_norm per call (argument and
 * pointer checks, plan, launch), and the device time per call of the same calls run back
 * to back on one stream.  For decode-sized batches (a few rows) the host cost is the
 * whole story: when it exceeds the kernel time the stream runs dry between calls.
 *
 *   host_cost OP ROWS D DTYPE ITERS [nochecks]     OP: rms | add;  DTYPE: bf16 | f32
 *
 * With `nochecks` the library's per-pointer driver queries are turned off first
 * (nv_set_pointer_checks(0)): the host cost of a caller that vouches for its pointers.
 *
 * Prints one JSON object: {"op", "rows", "D", "dtype", "iters", "host_us_per_call",
 * "device_us_per_call", "empty_launch_us"}: the host time inside one call; the device time
 * per call with all calls queued before the first runs (no host gaps between them); and
 * the host time of a cudaMemsetAsync of 16 bytes on the same stream, the cheapest enqueue
 * the runtime offers, for scale.  Exit status 0 on success.
 */
#define _POSIX_C_SOURCE 199309L
#include <cuda_runtime_api.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include <time.h>

#include "nvnorm.h"

#define CK(call)                                                                          \
    do {                                                                                  \
        cudaError_t e_ = (call);                                                          \
        if (e_ != cudaSuccess) {                                                          \
            fprintf(stderr, "%s: %s\n", #call, cudaGetErrorString(e_));                   \
            return 2;                                                                     \
        }                                                                                 \
    } while (0)

/* Holds the stream until the main thread has queued every call (bounded: ~10 s). */
static volatile int gate;
static void CUDART_CB hold(void* arg) {
    (void)arg;
    struct timespec t = {0, 100000};
    for (int i = 0; i < 100000 && !__atomic_load_n(&gate, __ATOMIC_ACQUIRE); ++i)
        nanosleep(&t, NULL);
}

static double now_us(void) {
    struct timespec t;
    clock_gettime(CLOCK_MONOTONIC, &t);
    return (double)t.tv_sec * 1e6 + (double)t.tv_nsec * 1e-3;
}

int main(int argc, char** argv) {
    if (argc != 6 && argc != 7) {
        fprintf(stderr, "usage: %s rms|add ROWS D bf16|f32 ITERS [nochecks]\n", argv[0]);
        return 1;
    }
    const int checks = !(argc == 7 && strcmp(argv[6], "nochecks") == 0);
    nv_set_pointer_checks(checks, NULL);
    const int add = strcmp(argv[1], "add") == 0;
    const int64_t rows = atoll(argv[2]), D = atoll(argv[3]);
    const int bf = strcmp(argv[4], "bf16") == 0;
    const int iters = atoi(argv[5]);
    if (rows < 1 || D < 1 || iters < 1) return 1;
    const nv_dtype dt = bf ? NV_BF16 : NV_F32;
    const size_t bytes = (size_t)rows * (size_t)D * (bf ? 2u : 4u);
    void *x, *r, *w, *y, *h, *m;
    CK(cudaMalloc(&x, bytes));
    CK(cudaMalloc(&r, bytes));
    CK(cudaMalloc(&y, bytes));
    CK(cudaMalloc(&h, bytes));
    CK(cudaMalloc(&w, (size_t)D * 4u));
    CK(cudaMalloc(&m, 16));
    CK(cudaMemset(x, 0, bytes));
    CK(cudaMemset(r, 0, bytes));
    CK(cudaMemset(w, 0, (size_t)D * 4u));
    cudaStream_t st;
    CK(cudaStreamCreate(&st));
    cudaEvent_t e0, e1;
    CK(cudaEventCreate(&e0));
    CK(cudaEventCreate(&e1));

    nv_status s = NV_OK;
    for (int i = 0; i < 20 && s == NV_OK; ++i)  /* warm: first-call set-up, caches */
        s = add ? nv_add_rms_norm(x, r, w, y, h, rows, D, 1e-6f, dt, st)
                : nv_rms_norm(x, w, y, rows, D, 1e-6f, dt, st);
    if (s != NV_OK) {
        fprintf(stderr, "%s: %s\n", nv_status_string(s), nv_last_error());
        return 3;
    }
    CK(cudaStreamSynchronize(st));

    /* host time inside the calls (the device runs them behind) */
    const double t0 = now_us();
    for (int i = 0; i < iters; ++i)
        s |= add ? nv_add_rms_norm(x, r, w, y, h, rows, D, 1e-6f, dt, st)
                 : nv_rms_norm(x, w, y, rows, D, 1e-6f, dt, st);
    const double t1 = now_us();
    CK(cudaStreamSynchronize(st));
    if (s != NV_OK) return 3;

    /* device time per call: the stream is held by a host function until every call is
     * queued, then runs them back to back between two events (no host gaps) */
    gate = 0;
    CK(cudaLaunchHostFunc(st, hold, NULL));
    CK(cudaEventRecord(e0, st));
    for (int i = 0; i < iters; ++i)
        s |= add ? nv_add_rms_norm(x, r, w, y, h, rows, D, 1e-6f, dt, st)
                 : nv_rms_norm(x, w, y, rows, D, 1e-6f, dt, st);
    CK(cudaEventRecord(e1, st));
    __atomic_store_n(&gate, 1, __ATOMIC_RELEASE);
    CK(cudaStreamSynchronize(st));
    if (s != NV_OK) return 3;
    float span_ms = 0.f;
    CK(cudaEventElapsedTime(&span_ms, e0, e1));

    /* for scale: the host time of the cheapest enqueue, a 16-byte memset */
    const double m0 = now_us();
    for (int i = 0; i < iters; ++i) CK(cudaMemsetAsync(m, 0, 16, st));
    const double m1 = now_us();
    CK(cudaStreamSynchronize(st));

    printf("{\"op\": \"%s\", \"rows\": %lld, \"D\": %lld, \"dtype\": \"%s\", \"iters\": %d, "
           "\"pointer_checks\": %d, "
           "\"host_us_per_call\": %.3f, \"device_us_per_call\": %.3f, "
           "\"empty_launch_us\": %.3f}\n",
           add ? "add_rms_norm" : "rms_norm", (long long)rows, (long long)D, bf ? "bf16" : "f32",
           iters, checks, (t1 - t0) / iters, 1e3 * span_ms / iters, (m1 - m0) / iters);
    return 0;
}
