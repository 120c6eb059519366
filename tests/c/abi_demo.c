/*
 * A plain C (C99) client of libnvnorm.so: no C++, no torch, only the CUDA runtime for
 * device memory and a stream.  It reads x, r and w (bfloat16 bit patterns) from a file,
 * runs add_rms_norm, then rms_norm and layer_norm on its output y, and writes y, h, the
 * rms_norm output and the layer_norm output to another file; it also checks that an
 * invalid argument is rejected with a message.  Used by tests/test_c_program.py.
 *
 *   abi_demo ROWS D IN_FILE OUT_FILE      (exit status 0 on success)
 */
#include <cuda_runtime_api.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "nvnorm.h"

#define CK(call)                                                                          \
    do {                                                                                  \
        cudaError_t e_ = (call);                                                          \
        if (e_ != cudaSuccess) {                                                          \
            fprintf(stderr, "%s: %s\n", #call, cudaGetErrorString(e_));                   \
            return 2;                                                                     \
        }                                                                                 \
    } while (0)

#define NV(call)                                                                          \
    do {                                                                                  \
        nv_status s_ = (call);                                                            \
        if (s_ != NV_OK) {                                                                \
            fprintf(stderr, "%s: %s: %s\n", #call, nv_status_string(s_), nv_last_error()); \
            return 3;                                                                     \
        }                                                                                 \
    } while (0)

int main(int argc, char** argv) {
    if (argc != 5) {
        fprintf(stderr, "usage: %s ROWS D IN_FILE OUT_FILE\n", argv[0]);
        return 1;
    }
    const int64_t rows = atoll(argv[1]), D = atoll(argv[2]);
    const size_t n = (size_t)(rows * D), bytes = n * sizeof(uint16_t), wbytes = D * sizeof(uint16_t);
    uint16_t* host = (uint16_t*)malloc(2 * bytes + wbytes);
    uint16_t* out = (uint16_t*)malloc(4 * bytes);
    if (!host || !out) return 1;
    FILE* f = fopen(argv[3], "rb");
    if (!f || fread(host, 1, 2 * bytes + wbytes, f) != 2 * bytes + wbytes) return 1;
    fclose(f);

    void *x, *r, *w, *y, *h, *z, *u;
    CK(cudaMalloc(&x, bytes));
    CK(cudaMalloc(&r, bytes));
    CK(cudaMalloc(&w, wbytes));
    CK(cudaMalloc(&y, bytes));
    CK(cudaMalloc(&h, bytes));
    CK(cudaMalloc(&z, bytes));
    CK(cudaMalloc(&u, bytes));
    cudaStream_t st;
    CK(cudaStreamCreate(&st));
    CK(cudaMemcpyAsync(x, host, bytes, cudaMemcpyHostToDevice, st));
    CK(cudaMemcpyAsync(r, host + n, bytes, cudaMemcpyHostToDevice, st));
    CK(cudaMemcpyAsync(w, host + 2 * n, wbytes, cudaMemcpyHostToDevice, st));

    NV(nv_add_rms_norm(x, r, w, y, h, rows, D, 1e-5f, NV_BF16, st));
    NV(nv_rms_norm(y, w, z, rows, D, 1e-6f, NV_BF16, st));
    NV(nv_layer_norm(y, w, NULL, u, rows, D, 1e-5f, NV_BF16, st));

    /* an invalid argument is rejected on the host, with a message, before any launch */
    if (nv_rms_norm(x, w, z, rows, 0, 1e-6f, NV_BF16, st) != NV_ERR_INVALID_ARG ||
        strlen(nv_last_error()) == 0) {
        fprintf(stderr, "D = 0 was not rejected\n");
        return 4;
    }

    CK(cudaMemcpyAsync(out, y, bytes, cudaMemcpyDeviceToHost, st));
    CK(cudaMemcpyAsync(out + n, h, bytes, cudaMemcpyDeviceToHost, st));
    CK(cudaMemcpyAsync(out + 2 * n, z, bytes, cudaMemcpyDeviceToHost, st));
    CK(cudaMemcpyAsync(out + 3 * n, u, bytes, cudaMemcpyDeviceToHost, st));
    CK(cudaStreamSynchronize(st));
    f = fopen(argv[4], "wb");
    if (!f || fwrite(out, 1, 4 * bytes, f) != 4 * bytes) return 1;
    fclose(f);
    printf("abi_demo: version %d, %lld x %lld ok\n", (int)nv_version(), (long long)rows,
           (long long)D);
    return 0;
}
