// unroll.cu -- the sequential unroll of the diagonal cells on the GPU:
// h_t = f(h_{t-1}, x_t) step by step, one thread per (batch row, channel).
//
// The pages' sequential_apply (pararnn-torch page, API overview /
// Quickstart: the one-step recurrence newton_apply reproduces), written for
// the GPU so that the Newton forward can be timed against the sequential
// recurrence on the same device and the same inputs.  Every channel is an
// independent recurrence, so a warp runs 32 neighbouring channels in step:
// each step's pre-activation loads are coalesced across the warp, and the
// loads of the next kAhead steps are issued before the current step's
// arithmetic (they do not depend on the state), so only the recurrence's own
// dependent chain -- a few multiply-adds and two or three exponentials and
// reciprocals per step -- sets the time per step.  With B * D channels the
// device holds B * D threads: a problem with few channels and long
// sequences leaves most of the GPU idle, which is what Newton's parallelism
// over T is for.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "cells.cuh"
#include "common.cuh"
#include "pararnn_b200.h"

namespace pararnn {
void set_last_error(const char* msg);   // pararnn_abi.cu
bool pointer_on_device(const void* p);  // pararnn_abi.cu

namespace ur {

constexpr int kThreads = 128;
constexpr int kAhead = 8;  // steps of pre-activations loaded ahead

struct Params {
    const void* px;    // (B,T,G,D)
    const float* w;    // (G,D) or null
    const float* h0;   // (B,S,D) or null
    float* H;          // (B,T,S,D)
    unsigned* status;  // workspace header word 0
    int64_t B, T, D;
};

template <class Cell, typename PxT>
__global__ void __launch_bounds__(kThreads) unroll_kernel(const Params pr) {
    constexpr int G = Cell::G, S = Cell::S;
    const int64_t c = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const bool valid = c < pr.B * pr.D;
    const int64_t b = valid ? c / pr.D : 0, d = valid ? c - b * pr.D : 0;
    const PxT* px = static_cast<const PxT*>(pr.px);
    float w[G], h[S];
#pragma unroll
    for (int g = 0; g < G; ++g) w[g] = (valid && pr.w) ? pr.w[g * pr.D + d] : 0.0f;
#pragma unroll
    for (int s = 0; s < S; ++s) h[s] = (valid && pr.h0) ? pr.h0[(b * S + s) * pr.D + d] : 0.0f;
    // a ring of the next kAhead steps' pre-activations
    float ring[kAhead][G];
    auto load = [&](int64_t t, float (&p)[G]) {
#pragma unroll
        for (int g = 0; g < G; ++g)
            p[g] = (valid && t < pr.T) ? PxTraits<PxT>::cvt(px[((b * pr.T + t) * G + g) * pr.D + d]) : 0.0f;
    };
#pragma unroll
    for (int i = 0; i < kAhead; ++i) load(i, ring[i]);
    bool bad = false;
    for (int64_t t0 = 0; t0 < pr.T; t0 += kAhead) {
#pragma unroll
        for (int i = 0; i < kAhead; ++i) {
            const int64_t t = t0 + i;
            if (t < pr.T) {
                float f[S], A[S * S], beta[S];
                Cell::elem(ring[i], w, h, f, A, beta);
#pragma unroll
                for (int s = 0; s < S; ++s) {
                    h[s] = f[s];
                    if (valid) pr.H[((b * pr.T + t) * S + s) * pr.D + d] = f[s];
                    bad |= !isfinite(f[s]);
                }
            }
            load(t + kAhead, ring[i]);  // the step kAhead later reuses this slot
        }
    }
    if (__any_sync(0xffffffffu, bad && valid) && (threadIdx.x & 31) == 0) atomicOr(pr.status, kStatusNonFinite);
}

pararnn_status fail(pararnn_status st, const char* msg) {
    set_last_error(msg);
    return st;
}

template <class Cell, typename PxT>
pararnn_status launch(const Params& pr, cudaStream_t st) {
    const int64_t n = pr.B * pr.D;
    unroll_kernel<Cell, PxT><<<(unsigned)((n + kThreads - 1) / kThreads), kThreads, 0, st>>>(pr);
    return cudaGetLastError() == cudaSuccess ? PARARNN_OK : fail(PARARNN_ECUDA, "pararnn_unroll: kernel launch failed");
}

}  // namespace ur
}  // namespace pararnn

using namespace pararnn;

extern "C" pararnn_status pararnn_unroll(pararnn_cell cell, int64_t B, int64_t T, int64_t D, pararnn_dtype px_dtype,
                                         const void* preacts, const float* diag_w, const float* h0, float* H_out,
                                         void* workspace, size_t ws_bytes, void* stream) {
    set_last_error("");
    const int G = pararnn_num_gates(cell);
    if (G < 0) return ur::fail(PARARNN_EINVAL, "pararnn_unroll: unknown cell");
    if (B < 0 || T < 0 || D < 0 || B * D >= (int64_t(1) << 37))
        return ur::fail(PARARNN_EINVAL, "pararnn_unroll: bad sizes");
    if (px_dtype != PARARNN_F32 && px_dtype != PARARNN_BF16)
        return ur::fail(PARARNN_EINVAL, "pararnn_unroll: unknown pre-activation dtype");
    if (!workspace || ws_bytes < 256 || !pointer_on_device(workspace))
        return ur::fail(PARARNN_EINVAL, "pararnn_unroll: workspace of at least 256 bytes of device memory required");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(workspace, 0, 256, st) != cudaSuccess)
        return ur::fail(PARARNN_ECUDA, "pararnn_unroll: workspace reset failed");
    if (B == 0 || T == 0 || D == 0) return PARARNN_OK;
    const size_t esz = px_dtype == PARARNN_F32 ? 4 : 2;
    if (!preacts || !H_out || !pointer_on_device(preacts) || !pointer_on_device(H_out) ||
        (diag_w && !pointer_on_device(diag_w)) || (h0 && !pointer_on_device(h0)))
        return ur::fail(PARARNN_EINVAL, "pararnn_unroll: a pointer is null or not device memory");
    if ((reinterpret_cast<uintptr_t>(preacts) % esz) || (reinterpret_cast<uintptr_t>(H_out) & 3) ||
        (diag_w && (reinterpret_cast<uintptr_t>(diag_w) & 3)) || (h0 && (reinterpret_cast<uintptr_t>(h0) & 3)))
        return ur::fail(PARARNN_EINVAL, "pararnn_unroll: pointer not aligned to its element size");
    ur::Params pr;
    memset(&pr, 0, sizeof pr);
    pr.px = preacts;
    pr.w = cell == PARARNN_CELL_LINEAR ? nullptr : diag_w;
    pr.h0 = h0;
    pr.H = H_out;
    pr.status = static_cast<unsigned*>(workspace);
    pr.B = B;
    pr.T = T;
    pr.D = D;
    typedef __nv_bfloat16 bf16;
    const bool bf = px_dtype == PARARNN_BF16;
    if (cell == PARARNN_CELL_LINEAR) return bf ? ur::launch<CellLinear, bf16>(pr, st) : ur::launch<CellLinear, float>(pr, st);
    if (cell == PARARNN_CELL_DIAG_GRU) return bf ? ur::launch<CellGRU, bf16>(pr, st) : ur::launch<CellGRU, float>(pr, st);
    return bf ? ur::launch<CellLSTM, bf16>(pr, st) : ur::launch<CellLSTM, float>(pr, st);
}
