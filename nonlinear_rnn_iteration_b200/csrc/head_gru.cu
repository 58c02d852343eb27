// head_gru.cu -- Newton forward of the head-wise GRU (block-diagonal
// recurrent weights: ParaGRU(mix='head', n_heads) on the pararnn-torch page,
// Models / Usage, "block-diagonal A").
//
// Cell, one head of width d (D = n_heads * d), state s, gates (z, r, c):
//     z = sig(p_z + U_z s),  r = sig(p_r + U_r s),  n = U_c s,
//     c = tanh(p_c + r * n), f = (1 - z) * s + z * c          (* elementwise)
// Jacobian (dense d x d):
//     A = diag(1 - z) + diag(alpha) U_z + diag(beta) U_r + diag(gamma) U_c,
//     alpha = (c - s) z (1 - z), beta = z (1 - c^2) n r (1 - r), gamma = z (1 - c^2) r.
// Newton on F(H)_t = h_t - f(h_{t-1}, x_t) from the warm start
// h^(0)_t = f(0, x_t) (Method section): each iteration solves the block
// lower-bidiagonal system delta_t = A_t delta_{t-1} - F_t (delta_{-1} = 0) and
// sets h^(k+1) = h^(k) + delta.  The solve is an associative scan whose
// elements are (A_t, -F_t) with dense d x d blocks, done in three launches
// per iteration over chunks of kChunk steps of one (batch row, head):
//   A. per chunk: the product P = A_{t1-1} ... A_{t0} (one d x d x d product
//      per step) and the chunk's delta from a zero carry, q;
//   B. per (batch row, head): the carries, carry_{c+1} = P_c carry_c + q_c;
//   C. per chunk: re-walk from its carry, delta_t = A_t delta_{t-1} - F_t
//      (A_t applied as the sum above, never formed), and write h^(k+1).
// No block waits on another, so there is no look-back and nothing to time
// out.  All arithmetic is float32; pre-activations f32 or bf16.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"
#include "pararnn_b200.h"

namespace pararnn {
void set_last_error(const char* msg);       // pararnn_abi.cu
bool pointer_on_device(const void* p);      // pararnn_abi.cu

namespace hg {

constexpr int kThreads = 256;
constexpr int kChunk = 32;  // steps per chunk
constexpr int kMaxK = 64;

struct Params {
    const void* px;     // (B,T,3,D)
    const float* U;     // (3,nh,d,d)
    const float* h0;    // (B,D) or null
    const float* Hold;  // h^(k) (B,T,D); null at k = 0 (the warm start is evaluated in place)
    float* Hnew;        // h^(k+1) (B,T,D)
    float* P;           // [nSeq][nChunks][d][d]
    float* q;           // [nSeq][nChunks][d]
    float* carry;       // [nSeq][nChunks][d]: delta just before each chunk
    float* resid;       // K+1 floats or null
    unsigned* status;   // workspace header word 0
    int64_t B, T, D;
    int nh, k, nChunks;
};

template <typename PxT>
__device__ __forceinline__ float ldp(const PxT* p) { return PxTraits<PxT>::cvt(*p); }

// Shared state of one chunk walk: the head's weights transposed,
// UT[g][j][i] = U_g[i][j] (so that thread i reads consecutive words), and the
// per-step vectors.
template <int DH>
struct Walk {
    float UT[3][DH][DH];
    float px[3][DH];      // p_z, p_r, p_c of the step
    float sprev[DH];      // h^(k)_{t-1}
    float scur[DH];       // h^(k)_t
    float u[3][DH];       // U_g s_prev
    float v[3][DH];       // U_g delta_{t-1} (re-walk)
    float dz[DH], al[DH], be[DH], ga[DH], F[DH];
    float del[2][DH];     // delta_{t-1}, delta_t
};

template <int DH>
__device__ void load_weights(Walk<DH>& w, const float* U, int nh, int h) {
    for (int idx = threadIdx.x; idx < 3 * DH * DH; idx += kThreads) {
        const int g = idx / (DH * DH), rem = idx - g * DH * DH, i = rem / DH, j = rem - i * DH;
        w.UT[g][j][i] = U[((int64_t)(g * nh + h) * DH + i) * DH + j];
    }
}

// h^(k) of row t of this head into dst (all d values): the iterate buffer, or
// the warm start f(0, x_t) = sig(p_z) tanh(p_c) at k = 0; h0 (or 0) at t = -1.
template <int DH, typename PxT>
__device__ __forceinline__ void iterate_row(const Params& pr, int64_t b, int h, int64_t t, float* dst) {
    const int i = threadIdx.x;
    if (i >= DH) return;
    const int64_t c = (int64_t)h * DH + i;
    if (t < 0) {
        dst[i] = pr.h0 ? pr.h0[b * pr.D + c] : 0.0f;
    } else if (pr.Hold) {
        dst[i] = pr.Hold[(b * pr.T + t) * pr.D + c];
    } else {
        const PxT* x = static_cast<const PxT*>(pr.px) + (b * pr.T + t) * 3 * pr.D + c;
        dst[i] = sigmoid_f(ldp(x)) * tanh_f(ldp(x + 2 * pr.D));
    }
}

// The cell at (s_prev, x_t) for row t: gates, f, F = h^(k)_t - f, and the
// Jacobian's row factors.  Returns |F| of this thread's row (0 for others).
template <int DH, typename PxT>
__device__ __forceinline__ float linearise(Walk<DH>& w, const Params& pr, int64_t b, int h, int64_t t, bool with_v) {
    const int tid = threadIdx.x;
    // pre-activations and the iterate at row t
    if (tid < 3 * DH) {
        const int g = tid / DH, i = tid - g * DH;
        w.px[g][i] = ldp(static_cast<const PxT*>(pr.px) + ((b * pr.T + t) * 3 + g) * pr.D + (int64_t)h * DH + i);
    }
    iterate_row<DH, PxT>(pr, b, h, t, w.scur);
    // U_g s_prev (and U_g delta_{t-1} for the re-walk)
    if (tid < 3 * DH) {
        const int g = tid / DH, i = tid - g * DH;
        float acc = 0.0f, acc2 = 0.0f;
#pragma unroll 8
        for (int j = 0; j < DH; ++j) {
            const float uw = w.UT[g][j][i];
            acc = __fmaf_rn(uw, w.sprev[j], acc);
            if (with_v) acc2 = __fmaf_rn(uw, w.del[0][j], acc2);
        }
        w.u[g][i] = acc;
        if (with_v) w.v[g][i] = acc2;
    }
    __syncthreads();
    float aF = 0.0f;
    if (tid < DH) {
        const int i = tid;
        const float s = w.sprev[i];
        const float z = sigmoid_f(w.px[0][i] + w.u[0][i]);
        const float r = sigmoid_f(w.px[1][i] + w.u[1][i]);
        const float n = w.u[2][i];
        const float c = tanh_f(__fmaf_rn(r, n, w.px[2][i]));
        const float f = __fmaf_rn(z, c - s, s);
        const float zc = z * __fmaf_rn(-c, c, 1.0f);  // z (1 - c^2)
        w.dz[i] = 1.0f - z;
        w.al[i] = (c - s) * (z - z * z);
        w.be[i] = zc * n * (r - r * r);
        w.ga[i] = zc * r;
        w.F[i] = w.scur[i] - f;
        aF = fabsf(w.F[i]);
    }
    __syncthreads();
    return aF;
}

// max over the block into *resid: a warp max, then one atomic per warp
// (a NaN wins, so a non-finite residual stays visible)
__device__ __forceinline__ void block_max_resid(float v, float* resid) {
    for (int o = 16; o > 0; o >>= 1) v = nanmax_f(v, __shfl_xor_sync(0xffffffffu, v, o));
    if ((threadIdx.x & 31) == 0 && (v > 0.0f || v != v)) atomic_max_nonneg(resid, v);
}

// ---- A: the chunk's Jacobian product and its delta from a zero carry -----
// (or, with kResidOnly, just max |F(h^(k))| over the chunk)
template <int DH, typename PxT, bool kResidOnly>
struct SmemA {
    Walk<DH> w;
    float AT[DH][DH];     // A_t transposed: AT[m][i] = A_t[i][m]
    float Pm[2][DH][DH];  // running product, row-major
};

template <int DH, typename PxT, bool kResidOnly>
__global__ void __launch_bounds__(kThreads) head_chunk_kernel(const Params pr) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto& sm = *reinterpret_cast<SmemA<DH, PxT, kResidOnly>*>(smem_raw);
    Walk<DH>& w = sm.w;
    const int tid = threadIdx.x;
    const int64_t task = blockIdx.x;
    const int64_t seq = task / pr.nChunks;
    const int chunk = (int)(task - seq * pr.nChunks);
    const int64_t b = seq / pr.nh;
    const int h = (int)(seq - b * pr.nh);
    const int64_t t0 = (int64_t)chunk * kChunk;
    const int64_t t1 = t0 + kChunk < pr.T ? t0 + kChunk : pr.T;

    load_weights<DH>(w, pr.U, pr.nh, h);
    iterate_row<DH, PxT>(pr, b, h, t0 - 1, w.sprev);
    if (tid < DH) w.del[0][tid] = 0.0f;
    __syncthreads();

    // thread tile of the product: TM x TM entries of P
    constexpr int TM = DH / 16;
    const int i0 = (tid / 16) * TM, j0 = (tid % 16) * TM;
    int cur = 0;
    float rmax = 0.0f;
    for (int64_t t = t0; t < t1; ++t) {
        rmax = nanmax_f(rmax, linearise<DH, PxT>(w, pr, b, h, t, false));
        if constexpr (!kResidOnly) {
            // A_t, transposed
            for (int idx = tid; idx < DH * DH; idx += kThreads) {
                const int m = idx / DH, i = idx - m * DH;  // AT[m][i] = A[i][m]
                float a = (i == m) ? w.dz[i] : 0.0f;
                a = __fmaf_rn(w.al[i], w.UT[0][m][i], a);
                a = __fmaf_rn(w.be[i], w.UT[1][m][i], a);
                a = __fmaf_rn(w.ga[i], w.UT[2][m][i], a);
                sm.AT[m][i] = a;
            }
            __syncthreads();
            // delta_t = A_t delta_{t-1} - F_t
            if (tid < DH) {
                float acc = -w.F[tid];
#pragma unroll 8
                for (int m = 0; m < DH; ++m) acc = __fmaf_rn(sm.AT[m][tid], w.del[0][m], acc);
                w.del[1][tid] = acc;
            }
            // P <- A_t P (P = A_t at the chunk's first step)
            if (t == t0) {
#pragma unroll
                for (int a = 0; a < TM; ++a)
#pragma unroll
                    for (int c = 0; c < TM; ++c) sm.Pm[cur][i0 + a][j0 + c] = sm.AT[j0 + c][i0 + a];
            } else {
                float acc[TM][TM];
#pragma unroll
                for (int a = 0; a < TM; ++a)
#pragma unroll
                    for (int c = 0; c < TM; ++c) acc[a][c] = 0.0f;
#pragma unroll 4
                for (int m = 0; m < DH; ++m) {
                    float av[TM], pv[TM];
#pragma unroll
                    for (int a = 0; a < TM; ++a) av[a] = sm.AT[m][i0 + a];
#pragma unroll
                    for (int c = 0; c < TM; ++c) pv[c] = sm.Pm[cur][m][j0 + c];
#pragma unroll
                    for (int a = 0; a < TM; ++a)
#pragma unroll
                        for (int c = 0; c < TM; ++c) acc[a][c] = __fmaf_rn(av[a], pv[c], acc[a][c]);
                }
#pragma unroll
                for (int a = 0; a < TM; ++a)
#pragma unroll
                    for (int c = 0; c < TM; ++c) sm.Pm[cur ^ 1][i0 + a][j0 + c] = acc[a][c];
                cur ^= 1;
            }
        }
        __syncthreads();
        if (tid < DH) {
            w.sprev[tid] = w.scur[tid];
            if constexpr (!kResidOnly) w.del[0][tid] = w.del[1][tid];
        }
        __syncthreads();
    }
    if (pr.resid) block_max_resid(rmax, pr.resid + pr.k);
    if constexpr (!kResidOnly) {
        float* Pout = pr.P + task * DH * DH;
        for (int idx = tid; idx < DH * DH; idx += kThreads) Pout[idx] = (&sm.Pm[cur][0][0])[idx];
        if (tid < DH) pr.q[task * DH + tid] = w.del[0][tid];
    }
}

// ---- B: the carries of one (batch row, head), chunk after chunk ----------
template <int DH>
__global__ void __launch_bounds__(64) head_carry_kernel(const Params pr) {
    __shared__ float x[2][DH];
    const int64_t seq = blockIdx.x;
    const int i = threadIdx.x;
    if (i < DH) x[0][i] = 0.0f;  // delta_{-1} = 0: h0 is given, not solved for
    __syncthreads();
    int cur = 0;
    for (int c = 0; c < pr.nChunks; ++c) {
        const int64_t task = seq * pr.nChunks + c;
        if (i < DH) {
            pr.carry[task * DH + i] = x[cur][i];
            const float* Prow = pr.P + (task * DH + i) * DH;
            float acc = pr.q[task * DH + i];
#pragma unroll 8
            for (int m = 0; m < DH; ++m) acc = __fmaf_rn(Prow[m], x[cur][m], acc);
            x[cur ^ 1][i] = acc;
        }
        __syncthreads();
        cur ^= 1;
    }
}

// ---- C: re-walk each chunk from its carry and write h^(k+1) --------------
template <int DH, typename PxT>
__global__ void __launch_bounds__(kThreads) head_walk_kernel(const Params pr) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Walk<DH>& w = *reinterpret_cast<Walk<DH>*>(smem_raw);
    const int tid = threadIdx.x;
    const int64_t task = blockIdx.x;
    const int64_t seq = task / pr.nChunks;
    const int chunk = (int)(task - seq * pr.nChunks);
    const int64_t b = seq / pr.nh;
    const int h = (int)(seq - b * pr.nh);
    const int64_t t0 = (int64_t)chunk * kChunk;
    const int64_t t1 = t0 + kChunk < pr.T ? t0 + kChunk : pr.T;

    load_weights<DH>(w, pr.U, pr.nh, h);
    iterate_row<DH, PxT>(pr, b, h, t0 - 1, w.sprev);
    if (tid < DH) w.del[0][tid] = pr.carry[task * DH + tid];
    __syncthreads();
    bool bad = false;
    for (int64_t t = t0; t < t1; ++t) {
        linearise<DH, PxT>(w, pr, b, h, t, true);
        if (tid < DH) {
            const int i = tid;
            float d = __fmaf_rn(w.dz[i], w.del[0][i], -w.F[i]);
            d = __fmaf_rn(w.al[i], w.v[0][i], d);
            d = __fmaf_rn(w.be[i], w.v[1][i], d);
            d = __fmaf_rn(w.ga[i], w.v[2][i], d);
            const float hn = w.scur[i] + d;
            pr.Hnew[(b * pr.T + t) * pr.D + (int64_t)h * DH + i] = hn;
            bad |= !isfinite(hn);
            w.del[1][i] = d;
        }
        __syncthreads();
        if (tid < DH) {
            w.sprev[tid] = w.scur[tid];
            w.del[0][tid] = w.del[1][tid];
        }
        __syncthreads();
    }
    if (__any_sync(0xffffffffu, bad) && (tid & 31) == 0) atomicOr(pr.status, kStatusNonFinite);
}

// ---- host side --------------------------------------------------------------

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Plan {
    int d = 0, nChunks = 0;
    int64_t nSeq = 0;
    size_t off_h = 0, off_P = 0, off_q = 0, off_c = 0, total = 0;
};

// workspace: 256-byte header (status word) | second iterate buffer (K >= 2)
// | chunk products P | chunk deltas q | chunk carries
bool make_plan(int64_t B, int64_t T, int64_t D, int nh, int K, Plan& pl) {
    if (B < 0 || T < 0 || D < 0 || nh < 1 || D % nh != 0) return false;
    const int64_t d = D / nh;
    if (d != 16 && d != 32 && d != 64) return false;
    if (B * T >= (int64_t(1) << 31) || (double)B * T * D > 4.0e12) return false;
    pl.d = (int)d;
    pl.nChunks = (int)((T + kChunk - 1) / kChunk);
    pl.nSeq = B * nh;
    const size_t ntask = (size_t)pl.nSeq * pl.nChunks;
    pl.off_h = 256;
    pl.off_P = align256(pl.off_h + (K >= 2 ? (size_t)B * T * D * sizeof(float) : 0));
    pl.off_q = align256(pl.off_P + ntask * d * d * sizeof(float));
    pl.off_c = align256(pl.off_q + ntask * d * sizeof(float));
    pl.total = align256(pl.off_c + ntask * d * sizeof(float));
    return true;
}

template <class Kern>
cudaError_t set_smem(Kern k, size_t bytes) {
    return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int DH, typename PxT>
cudaError_t launch_all(const Plan& pl, Params pr, float* H_out, float* Hbuf, int K, cudaStream_t st) {
    const size_t smemA = sizeof(SmemA<DH, PxT, false>), smemR = sizeof(SmemA<DH, PxT, true>);
    const size_t smemC = sizeof(Walk<DH>);
    cudaError_t e = set_smem(head_chunk_kernel<DH, PxT, false>, smemA);
    if (e == cudaSuccess) e = set_smem(head_chunk_kernel<DH, PxT, true>, smemR);
    if (e == cudaSuccess) e = set_smem(head_walk_kernel<DH, PxT>, smemC);
    if (e != cudaSuccess) return e;
    const unsigned ntask = (unsigned)(pl.nSeq * pl.nChunks);
    for (int k = 0; k < K; ++k) {
        // iterate k lives in X_k, X_j = H_out when K - j is even, else the
        // workspace buffer, so that h^(K) lands in H_out
        pr.k = k;
        pr.Hold = k == 0 ? nullptr : (((K - k) % 2 == 0) ? H_out : Hbuf);
        pr.Hnew = ((K - (k + 1)) % 2 == 0) ? H_out : Hbuf;
        head_chunk_kernel<DH, PxT, false><<<ntask, kThreads, smemA, st>>>(pr);
        head_carry_kernel<DH><<<(unsigned)pl.nSeq, 64, 0, st>>>(pr);
        head_walk_kernel<DH, PxT><<<ntask, kThreads, smemC, st>>>(pr);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (pr.resid) {
        // the residual of the final iterate
        pr.k = K;
        pr.Hold = H_out;
        head_chunk_kernel<DH, PxT, true><<<ntask, kThreads, smemR, st>>>(pr);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

pararnn_status fail(pararnn_status st, const char* msg) {
    set_last_error(msg);
    return st;
}

}  // namespace hg
}  // namespace pararnn

using namespace pararnn;

extern "C" size_t pararnn_head_gru_workspace_bytes(int64_t B, int64_t T, int64_t D, int n_heads, int K) {
    hg::Plan pl;
    if (K < 1 || K > hg::kMaxK || !hg::make_plan(B, T, D, n_heads, K, pl)) return 0;
    return pl.total;
}

extern "C" pararnn_status pararnn_head_gru_forward(int64_t B, int64_t T, int64_t D, int n_heads,
                                                   pararnn_dtype px_dtype, const void* preacts, const float* U,
                                                   const float* h0, int K, float* H_out, void* workspace,
                                                   size_t ws_bytes, float* resid_hist, void* stream) {
    hg::Plan pl;
    if (K < 1 || K > hg::kMaxK) return hg::fail(PARARNN_EINVAL, "pararnn_head_gru_forward: K must be in 1..64");
    if (!hg::make_plan(B, T, D, n_heads, K, pl))
        return hg::fail(PARARNN_EINVAL,
                        "pararnn_head_gru_forward: need B, T, D >= 0, D = n_heads * d with d in {16, 32, 64}, "
                        "and B*T below 2^31");
    if (px_dtype != PARARNN_F32 && px_dtype != PARARNN_BF16)
        return hg::fail(PARARNN_EINVAL, "pararnn_head_gru_forward: unknown pre-activation dtype");
    if (!workspace || ws_bytes < pl.total)
        return hg::fail(PARARNN_EINVAL, "pararnn_head_gru_forward: workspace missing or smaller than "
                                        "pararnn_head_gru_workspace_bytes()");
    if (!pointer_on_device(workspace) || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return hg::fail(PARARNN_EINVAL, "pararnn_head_gru_forward: workspace must be 256-byte aligned device memory");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    cudaError_t e = cudaMemsetAsync(ws, 0, 256, st);
    if (e != cudaSuccess) return hg::fail(PARARNN_ECUDA, "pararnn_head_gru_forward: header reset failed");
    if (B == 0 || T == 0 || D == 0) {
        if (resid_hist && pointer_on_device(resid_hist)) cudaMemsetAsync(resid_hist, 0, sizeof(float) * (K + 1), st);
        return PARARNN_OK;
    }
    const size_t esz = px_dtype == PARARNN_BF16 ? 2 : 4;
    if (!preacts || !U || !H_out || !pointer_on_device(preacts) || !pointer_on_device(U) ||
        !pointer_on_device(H_out) || (h0 && !pointer_on_device(h0)) ||
        (resid_hist && !pointer_on_device(resid_hist)))
        return hg::fail(PARARNN_EINVAL, "pararnn_head_gru_forward: a required pointer is null or not device memory");
    if ((reinterpret_cast<uintptr_t>(preacts) % esz) || (reinterpret_cast<uintptr_t>(U) & 3) ||
        (reinterpret_cast<uintptr_t>(H_out) & 3) || (h0 && (reinterpret_cast<uintptr_t>(h0) & 3)) ||
        (resid_hist && (reinterpret_cast<uintptr_t>(resid_hist) & 3)))
        return hg::fail(PARARNN_EINVAL, "pararnn_head_gru_forward: misaligned pointer");
    if (resid_hist) {
        e = cudaMemsetAsync(resid_hist, 0, sizeof(float) * (K + 1), st);
        if (e != cudaSuccess) return hg::fail(PARARNN_ECUDA, "pararnn_head_gru_forward: resid_hist reset failed");
    }
    hg::Params pr;
    pr.px = preacts;
    pr.U = U;
    pr.h0 = h0;
    pr.Hold = nullptr;
    pr.Hnew = H_out;
    pr.P = reinterpret_cast<float*>(ws + pl.off_P);
    pr.q = reinterpret_cast<float*>(ws + pl.off_q);
    pr.carry = reinterpret_cast<float*>(ws + pl.off_c);
    pr.resid = resid_hist;
    pr.status = reinterpret_cast<unsigned*>(ws);
    pr.B = B;
    pr.T = T;
    pr.D = D;
    pr.nh = n_heads;
    pr.k = 0;
    pr.nChunks = pl.nChunks;
    float* Hbuf = reinterpret_cast<float*>(ws + pl.off_h);
    const bool bf = px_dtype == PARARNN_BF16;
    switch (pl.d) {
        case 16: e = bf ? hg::launch_all<16, __nv_bfloat16>(pl, pr, H_out, Hbuf, K, st)
                        : hg::launch_all<16, float>(pl, pr, H_out, Hbuf, K, st); break;
        case 32: e = bf ? hg::launch_all<32, __nv_bfloat16>(pl, pr, H_out, Hbuf, K, st)
                        : hg::launch_all<32, float>(pl, pr, H_out, Hbuf, K, st); break;
        default: e = bf ? hg::launch_all<64, __nv_bfloat16>(pl, pr, H_out, Hbuf, K, st)
                        : hg::launch_all<64, float>(pl, pr, H_out, Hbuf, K, st); break;
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        return hg::fail(PARARNN_ECUDA, "pararnn_head_gru_forward: kernel launch failed");
    }
    return PARARNN_OK;
}
