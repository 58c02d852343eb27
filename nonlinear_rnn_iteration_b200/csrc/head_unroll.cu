// head_unroll.cu -- the sequential unroll of the head-wise GRU on the GPU:
// s_t = f(s_{t-1}, x_t) step by step, one thread block per (batch row, head).
//
// This is the pages' sequential_apply for ParaGRU(mix='head') (pararnn-torch
// page, API overview / Quickstart: the one-step recurrence that newton_apply
// must reproduce), written for the GPU so that the Newton scan of
// head_gru.cu can be timed against it on the same problem.  With a dense
// d x d recurrent block per head, one step costs 3 d^2 multiply-adds, the
// Newton scan's d x d x d products per step cost 2 d^3 (2/3 d times more),
// and a problem with few long sequences gives the scan its parallelism.  A
// problem with many sequences and d = 64 (B * n_heads thread blocks of
// 4 d threads each) is the opposite case.
//
// Cell, one head of width d, state s, gates (z, r, c):
//     z = sig(p_z + U_z s),  r = sig(p_r + U_r s),  n = U_c s,
//     c = tanh(p_c + r * n), s' = (1 - z) * s + z * c.
// Thread (row i, quarter q) of a block holds columns q*d/4 .. q*d/4+d/4-1 of
// row i of U_z, U_r and U_c in registers for the whole sequence; per step it
// forms its part of the three dot products with s_{t-1} (read from shared
// memory), the four threads of a row sum theirs with two shuffles, each of
// them evaluates the gates, and the first writes s_t to shared memory and to
// H.  Pre-activations arrive in chunks of kSteps steps by cp.async, one chunk
// ahead.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "common.cuh"
#include "pararnn_b200.h"

namespace pararnn {
void set_last_error(const char* msg);   // pararnn_abi.cu
bool pointer_on_device(const void* p);  // pararnn_abi.cu

namespace hu {

constexpr int kSteps = 32;  // steps per pre-activation chunk
constexpr int kTPR = 4;     // threads per row

struct Params {
    const void* px;    // (B,T,3,D)
    const float* U;    // (3,nh,d,d)
    const float* h0;   // (B,D) or null
    float* H;          // (B,T,D)
    unsigned* status;  // workspace header word 0
    int64_t B, T, D;
    int nh;
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

template <int DH, typename PxT>
struct Smem {
    alignas(16) PxT px[2][kSteps][3][DH];  // two chunks in turn
    float s[2][DH];                        // s_{t-1}, s_t in turn
};

// Copy the pre-activations of steps t0 .. t0+kSteps-1 (those below T) of one
// (batch row, head) into a chunk buffer: rows of d values, 16 bytes per copy.
// A row of d values starts at element ((b T + t) 3 + g) D + head d, a multiple
// of d, so with a 16-byte aligned base every copy is aligned.
template <int DH, typename PxT>
__device__ __forceinline__ void load_chunk(PxT (&dst)[kSteps][3][DH], const Params& pr, int64_t b, int head,
                                           int64_t t0) {
    constexpr int PER_ROW = DH * (int)sizeof(PxT) / 16;  // 16-byte pieces per gate row
    constexpr int N = kSteps * 3 * PER_ROW;
    const PxT* px = static_cast<const PxT*>(pr.px);
    for (int i = threadIdx.x; i < N; i += DH * kTPR) {
        const int st = i / (3 * PER_ROW), rem = i - st * (3 * PER_ROW), g = rem / PER_ROW, piece = rem - g * PER_ROW;
        const int64_t t = t0 + st;
        if (t < pr.T)
            cp_async16(reinterpret_cast<unsigned char*>(&dst[st][g][0]) + piece * 16,
                       reinterpret_cast<const unsigned char*>(px + ((b * pr.T + t) * 3 + g) * pr.D +
                                                              (int64_t)head * DH) +
                           piece * 16);
    }
}

template <int DH, typename PxT>
__global__ void __launch_bounds__(DH * kTPR) head_unroll_kernel(const Params pr) {
    constexpr int CPT = DH / kTPR;  // columns per thread
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Smem<DH, PxT>& sm = *reinterpret_cast<Smem<DH, PxT>*>(smem_raw);
    const int seq = blockIdx.x;
    const int64_t b = seq / pr.nh;
    const int head = seq - (int)(b * pr.nh);
    const int i = threadIdx.x / kTPR, q = threadIdx.x % kTPR;
    const int64_t col0 = (int64_t)head * DH;

    // this thread's columns of row i of U_z, U_r, U_c
    float uz[CPT], ur[CPT], uc[CPT];
    const int64_t ublk = (int64_t)DH * DH;
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
        const int64_t o = ((int64_t)head * DH + i) * DH + q * CPT + j;
        uz[j] = pr.U[0 * pr.nh * ublk + o];
        ur[j] = pr.U[1 * pr.nh * ublk + o];
        uc[j] = pr.U[2 * pr.nh * ublk + o];
    }
    if (q == 0) sm.s[0][i] = pr.h0 ? pr.h0[b * pr.D + col0 + i] : 0.0f;
    load_chunk<DH, PxT>(sm.px[0], pr, b, head, 0);
    cp_async_commit();
    bool bad = false;
    const int64_t nch = (pr.T + kSteps - 1) / kSteps;
    for (int64_t c = 0; c < nch; ++c) {
        // the next chunk streams in while this one is used
        if (c + 1 < nch) load_chunk<DH, PxT>(sm.px[(c + 1) & 1], pr, b, head, (c + 1) * kSteps);
        cp_async_commit();
        cp_async_wait_one();
        __syncthreads();
        const int nst = (int)((pr.T - c * kSteps) < kSteps ? (pr.T - c * kSteps) : kSteps);
        for (int st = 0; st < nst; ++st) {
            const int64_t t = c * kSteps + st;
            const float* sp = sm.s[t & 1];
            float az = 0.0f, ar = 0.0f, an = 0.0f;
#pragma unroll
            for (int j = 0; j < CPT; ++j) {
                const float sj = sp[q * CPT + j];
                az = __fmaf_rn(uz[j], sj, az);
                ar = __fmaf_rn(ur[j], sj, ar);
                an = __fmaf_rn(uc[j], sj, an);
            }
#pragma unroll
            for (int o = 1; o < kTPR; o <<= 1) {
                az += __shfl_xor_sync(0xffffffffu, az, o);
                ar += __shfl_xor_sync(0xffffffffu, ar, o);
                an += __shfl_xor_sync(0xffffffffu, an, o);
            }
            const float pz = PxTraits<PxT>::cvt(sm.px[c & 1][st][0][i]);
            const float prr = PxTraits<PxT>::cvt(sm.px[c & 1][st][1][i]);
            const float pc = PxTraits<PxT>::cvt(sm.px[c & 1][st][2][i]);
            const float z = sigmoid_f(pz + az);
            const float r = sigmoid_f(prr + ar);
            const float cc = tanh_f(__fmaf_rn(r, an, pc));
            const float si = sp[i];
            const float sn = __fmaf_rn(z, cc - si, si);  // (1 - z) s + z c
            if (q == 0) {
                sm.s[(t + 1) & 1][i] = sn;
                pr.H[(b * pr.T + t) * pr.D + col0 + i] = sn;
                bad |= !isfinite(sn);
            }
            __syncthreads();
        }
    }
    if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(pr.status, kStatusNonFinite);
}

pararnn_status fail(pararnn_status st, const char* msg) {
    set_last_error(msg);
    return st;
}

template <int DH, typename PxT>
pararnn_status launch(const Params& pr, cudaStream_t st) {
    auto kern = head_unroll_kernel<DH, PxT>;
    const size_t smem = sizeof(Smem<DH, PxT>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return fail(PARARNN_ECUDA, "pararnn_head_gru_unroll: shared-memory attribute failed");
    kern<<<(unsigned)(pr.B * pr.nh), DH * kTPR, smem, st>>>(pr);
    e = cudaGetLastError();
    return e == cudaSuccess ? PARARNN_OK : fail(PARARNN_ECUDA, "pararnn_head_gru_unroll: kernel launch failed");
}

}  // namespace hu
}  // namespace pararnn

using namespace pararnn;

extern "C" pararnn_status pararnn_head_gru_unroll(int64_t B, int64_t T, int64_t D, int n_heads,
                                                  pararnn_dtype px_dtype, const void* preacts, const float* U,
                                                  const float* h0, float* H_out, void* workspace, size_t ws_bytes,
                                                  void* stream) {
    set_last_error("");
    if (B < 0 || T < 0 || D < 0 || n_heads < 1 || D % n_heads != 0)
        return hu::fail(PARARNN_EINVAL, "pararnn_head_gru_unroll: bad sizes (D must be a multiple of n_heads)");
    const int64_t d = D / n_heads;
    if (D > 0 && d != 16 && d != 32 && d != 64)
        return hu::fail(PARARNN_EINVAL, "pararnn_head_gru_unroll: head width must be 16, 32 or 64");
    if (B * n_heads >= (int64_t(1) << 31) || B * T >= (int64_t(1) << 40))
        return hu::fail(PARARNN_EINVAL, "pararnn_head_gru_unroll: problem too large");
    if (px_dtype != PARARNN_F32 && px_dtype != PARARNN_BF16)
        return hu::fail(PARARNN_EINVAL, "pararnn_head_gru_unroll: unknown pre-activation dtype");
    if (!workspace || ws_bytes < 256 || !pointer_on_device(workspace))
        return hu::fail(PARARNN_EINVAL, "pararnn_head_gru_unroll: workspace of at least 256 bytes of device memory "
                                        "required");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(workspace, 0, 256, st);
    if (e != cudaSuccess) return hu::fail(PARARNN_ECUDA, "pararnn_head_gru_unroll: workspace reset failed");
    if (B == 0 || T == 0 || D == 0) return PARARNN_OK;
    if (!preacts || !U || !H_out || !pointer_on_device(preacts) || !pointer_on_device(U) ||
        !pointer_on_device(H_out) || (h0 && !pointer_on_device(h0)))
        return hu::fail(PARARNN_EINVAL, "pararnn_head_gru_unroll: a pointer is null or not device memory");
    if ((reinterpret_cast<uintptr_t>(preacts) & 15) || (reinterpret_cast<uintptr_t>(U) & 3) ||
        (reinterpret_cast<uintptr_t>(H_out) & 3) || (h0 && (reinterpret_cast<uintptr_t>(h0) & 3)))
        return hu::fail(PARARNN_EINVAL, "pararnn_head_gru_unroll: preacts must be 16-byte aligned, the rest 4-byte");
    hu::Params pr;
    memset(&pr, 0, sizeof pr);
    pr.px = preacts;
    pr.U = U;
    pr.h0 = h0;
    pr.H = H_out;
    pr.status = static_cast<unsigned*>(workspace);
    pr.B = B;
    pr.T = T;
    pr.D = D;
    pr.nh = n_heads;
    const bool bf = px_dtype == PARARNN_BF16;
    typedef __nv_bfloat16 bf16;
    if (d == 64) return bf ? hu::launch<64, bf16>(pr, st) : hu::launch<64, float>(pr, st);
    if (d == 32) return bf ? hu::launch<32, bf16>(pr, st) : hu::launch<32, float>(pr, st);
    return bf ? hu::launch<16, bf16>(pr, st) : hu::launch<16, float>(pr, st);
}
