/*
 * c_abi_client.c -- a plain C caller of libpararnn_b200 (no Python, no torch):
 * reads a problem from binary files, runs the Newton forward and the adjoint
 * backward through the C ABI on the GPU, and writes H, dL/dpx and dL/da back
 * to binary files.  Built and run by tests/test_gpu_c_client.py, which
 * writes the inputs and checks the outputs against the fp64 oracle.
 *
 *   c_abi_client DIR cell B T D K
 *   DIR/px.f32 (B,T,G,D), DIR/w.f32 (G,D), DIR/g.f32 (B,T,S,D) in;
 *   DIR/H.f32 (B,T,S,D), DIR/dpx.f32 (B,T,G,D), DIR/da.f32 (G,D) out.
 * Exit status 0 on success; otherwise the failing call and its message go to
 * stderr.
 */
#include <cuda_runtime.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "pararnn_b200.h"

static void* read_file(const char* dir, const char* name, size_t bytes) {
    char path[4096];
    snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE* f = fopen(path, "rb");
    if (!f) return NULL;
    void* buf = malloc(bytes ? bytes : 1);
    size_t got = buf ? fread(buf, 1, bytes, f) : 0;
    fclose(f);
    if (got != bytes) {
        free(buf);
        return NULL;
    }
    return buf;
}

static int write_file(const char* dir, const char* name, const void* buf, size_t bytes) {
    char path[4096];
    snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE* f = fopen(path, "wb");
    if (!f) return -1;
    size_t put = fwrite(buf, 1, bytes, f);
    fclose(f);
    return put == bytes ? 0 : -1;
}

#define CHECK_CUDA(x)                                                              \
    do {                                                                           \
        cudaError_t e_ = (x);                                                      \
        if (e_ != cudaSuccess) {                                                   \
            fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_));               \
            return 2;                                                              \
        }                                                                          \
    } while (0)

#define CHECK_PARARNN(x)                                                           \
    do {                                                                           \
        pararnn_status s_ = (x);                                                   \
        if (s_ != PARARNN_OK) {                                                    \
            fprintf(stderr, "%s: %s (%s)\n", #x, pararnn_status_string(s_),       \
                    pararnn_last_error());                                         \
            return 3;                                                              \
        }                                                                          \
    } while (0)

int main(int argc, char** argv) {
    if (argc != 7) {
        fprintf(stderr, "usage: %s DIR cell B T D K\n", argv[0]);
        return 1;
    }
    const char* dir = argv[1];
    const pararnn_cell cell = (pararnn_cell)atoi(argv[2]);
    const int64_t B = atoll(argv[3]), T = atoll(argv[4]), D = atoll(argv[5]);
    const int K = atoi(argv[6]);
    const int G = pararnn_num_gates(cell), S = pararnn_state_width(cell);
    if (G < 0 || B < 1 || T < 1 || D < 1) {
        fprintf(stderr, "bad problem\n");
        return 1;
    }
    const size_t n_px = (size_t)(B * T * G * D), n_h = (size_t)(B * T * S * D), n_w = (size_t)(G * D);
    float* px = (float*)read_file(dir, "px.f32", n_px * sizeof(float));
    float* w = (float*)read_file(dir, "w.f32", n_w * sizeof(float));
    float* g = (float*)read_file(dir, "g.f32", n_h * sizeof(float));
    if (!px || !w || !g) {
        fprintf(stderr, "cannot read the inputs from %s\n", dir);
        return 1;
    }
    const size_t ws_bytes = pararnn_workspace_bytes(cell, B, T, D, K);
    if (ws_bytes == 0) {
        fprintf(stderr, "pararnn_workspace_bytes: %s\n", pararnn_last_error());
        return 3;
    }
    float *d_px, *d_w, *d_g, *d_H, *d_dpx, *d_da;
    void* d_ws;
    CHECK_CUDA(cudaMalloc((void**)&d_px, n_px * sizeof(float)));
    CHECK_CUDA(cudaMalloc((void**)&d_w, n_w * sizeof(float)));
    CHECK_CUDA(cudaMalloc((void**)&d_g, n_h * sizeof(float)));
    CHECK_CUDA(cudaMalloc((void**)&d_H, n_h * sizeof(float)));
    CHECK_CUDA(cudaMalloc((void**)&d_dpx, n_px * sizeof(float)));
    CHECK_CUDA(cudaMalloc((void**)&d_da, n_w * sizeof(float)));
    CHECK_CUDA(cudaMalloc(&d_ws, ws_bytes));
    cudaStream_t stream;
    CHECK_CUDA(cudaStreamCreate(&stream));
    CHECK_CUDA(cudaMemcpyAsync(d_px, px, n_px * sizeof(float), cudaMemcpyHostToDevice, stream));
    CHECK_CUDA(cudaMemcpyAsync(d_w, w, n_w * sizeof(float), cudaMemcpyHostToDevice, stream));
    CHECK_CUDA(cudaMemcpyAsync(d_g, g, n_h * sizeof(float), cudaMemcpyHostToDevice, stream));
    /* the workspace holds whatever cudaMalloc left there: the library clears what it reads */
    CHECK_PARARNN(pararnn_newton_forward(cell, B, T, D, PARARNN_F32, d_px, d_w, NULL, K, d_H, d_ws, ws_bytes, NULL,
                                         stream));
    CHECK_PARARNN(pararnn_status_sync(d_ws, stream));
    CHECK_PARARNN(pararnn_newton_backward(cell, B, T, D, PARARNN_F32, d_px, d_w, NULL, d_H, d_g, d_dpx,
                                          cell == PARARNN_CELL_LINEAR ? NULL : d_da, NULL, d_ws, ws_bytes, stream));
    CHECK_PARARNN(pararnn_status_sync(d_ws, stream));
    float* H = (float*)malloc(n_h * sizeof(float));
    float* dpx = (float*)malloc(n_px * sizeof(float));
    float* da = (float*)calloc(n_w, sizeof(float));
    if (!H || !dpx || !da) return 1;
    CHECK_CUDA(cudaMemcpy(H, d_H, n_h * sizeof(float), cudaMemcpyDeviceToHost));
    CHECK_CUDA(cudaMemcpy(dpx, d_dpx, n_px * sizeof(float), cudaMemcpyDeviceToHost));
    if (cell != PARARNN_CELL_LINEAR) CHECK_CUDA(cudaMemcpy(da, d_da, n_w * sizeof(float), cudaMemcpyDeviceToHost));
    if (write_file(dir, "H.f32", H, n_h * sizeof(float)) || write_file(dir, "dpx.f32", dpx, n_px * sizeof(float)) ||
        write_file(dir, "da.f32", da, n_w * sizeof(float))) {
        fprintf(stderr, "cannot write the outputs to %s\n", dir);
        return 1;
    }
    cudaFree(d_px);
    cudaFree(d_w);
    cudaFree(d_g);
    cudaFree(d_H);
    cudaFree(d_dpx);
    cudaFree(d_da);
    cudaFree(d_ws);
    cudaStreamDestroy(stream);
    free(px);
    free(w);
    free(g);
    free(H);
    free(dpx);
    free(da);
    return 0;
}
