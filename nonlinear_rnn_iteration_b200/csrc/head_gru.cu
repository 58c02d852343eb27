// head_gru.cu -- Newton forward and adjoint of the head-wise GRU (block-diagonal
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
//      per step; on the fifth-generation tensor cores for d = 64, with
//      mma.sync for d = 16 and 32), the chunk's delta from a zero carry, q,
//      and each step's row factors for C;
//   B. per (batch row, head): the carries, carry_{c+1} = P_c carry_c + q_c;
//   C. per chunk: re-walk from its carry, delta_t = A_t delta_{t-1} - F_t
//      (A_t applied as the sum above from the stored factors, never
//      formed), and write h^(k+1).
// No block waits on another, so there is no look-back and nothing to time
// out.  All arithmetic is float32; pre-activations f32 or bf16.  The adjoint
// (pararnn_head_gru_backward) runs the same three launches on the propagated
// adjoint, its carries and re-walk in reverse time (its d = 64 chunk pass
// forms prefix products forward in time within the chunk), plus a
// fixed-order reduction for dL/dU (see "the adjoint" below).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "common.cuh"
#include "pararnn_b200.h"
#include "tma.cuh"

namespace pararnn {
void set_last_error(const char* msg);       // pararnn_abi.cu
bool pointer_on_device(const void* p);      // pararnn_abi.cu

namespace hg {

constexpr int kThreads = 256;
constexpr int kChunk = 128;  // steps per chunk
constexpr int kMaxK = 64;
// row factors stored per step: forward h^(k)_t, F_t, 1 - z, alpha, beta,
// gamma; backward 1 - z, alpha, beta, z (1 - c^2), gamma
constexpr int kNF = 6;
constexpr int kNB = 5;

struct Params {
    const void* px;     // (B,T,3,D)
    const float* U;     // (3,nh,d,d)
    const float* h0;    // (B,D) or null
    const float* Hold;  // h^(k) (B,T,D); null at k = 0 (the warm start is evaluated in place)
    float* Hnew;        // h^(k+1) (B,T,D)
    float* P;           // [nSeq][nChunks][d][d]
    float* q;           // [nSeq][nChunks][d]
    float* carry;       // [nSeq][nChunks][d]: delta just before each chunk
    float* L;           // [nSeq][T][kNF or kNB][d]: each step's row factors, formed by the chunk
                        // kernel for the Jacobian rows and read back by the walk
    float* resid;       // K+1 floats or null
    unsigned* status;   // workspace header word 0
    // backward only
    const float* G;     // dL/dH (B,T,D)
    float* dpx;         // dL/dpx (B,T,3,D)
    float* ec;          // lambda * gamma (B,T,D): the factor of dL/dU_c
    float* dh0;         // dL/dh0 (B,D) or null
    int64_t B, T, D;
    int nh, k, nChunks;
};

template <typename PxT>
__device__ __forceinline__ float ldp(const PxT* p) { return PxTraits<PxT>::cvt(*p); }

// Thread layout of a chunk walk: row i of the head is handled by TPR
// consecutive threads (qt = 0..TPR-1); thread qt owns the SEG columns
// m = qt + TPR*s of row i of U_z, U_r, U_c, kept in registers for the whole
// chunk.  A row's dot products are summed over its TPR threads with
// shuffles, and every thread of the row then evaluates the row's gates (the
// redundancy is cheaper than another round through shared memory).  Vectors
// over the head's state live in shared memory in the permuted order
// vpos(m) = (m % TPR) * SEGP + m / TPR, so a thread's SEG elements are
// contiguous.  With 4 threads per row (d = 64) each thread's segment is
// padded by 4 floats (SEGP = 20), so that the four 16-byte loads of a
// row's threads fall on four different bank groups; the narrower heads'
// segments already do.
template <int DH>
struct Geo {
    static constexpr int TPR = kThreads / DH;
    static constexpr int SEG = DH / TPR;
    static constexpr int SEGP = SEG + (SEG == 16 ? 4 : 0);  // padded segment
    static constexpr int VLEN = TPR * SEGP;                 // floats of a permuted vector
    static_assert(TPR * SEG == DH && TPR <= 32, "one row's threads share a warp");
    static __device__ __forceinline__ int vpos(int m) { return (m % TPR) * SEGP + m / TPR; }
};

template <int DH>
__device__ __forceinline__ float row_sum(float v) {
#pragma unroll
    for (int o = Geo<DH>::TPR / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// The head's recurrent weights owned by this thread.
template <int DH>
struct RowU {
    float z[Geo<DH>::SEG], r[Geo<DH>::SEG], c[Geo<DH>::SEG];
    __device__ __forceinline__ void load(const float* U, int nh, int h, int i, int qt) {
        constexpr int SEG = Geo<DH>::SEG, TPR = Geo<DH>::TPR;
        const int64_t hs = (int64_t)DH * DH;
#pragma unroll
        for (int s = 0; s < SEG; ++s) {
            const int m = qt + TPR * s;
            z[s] = __ldg(U + (0 * nh + h) * hs + (int64_t)i * DH + m);
            r[s] = __ldg(U + ((int64_t)1 * nh + h) * hs + (int64_t)i * DH + m);
            c[s] = __ldg(U + ((int64_t)2 * nh + h) * hs + (int64_t)i * DH + m);
        }
    }
};

// The inputs of one step for row i: pre-activations and h^(k)_t.
struct StepIn {
    float pz, pr, pc, s;
};

template <int DH, typename PxT>
__device__ __forceinline__ StepIn load_step(const Params& pr, int64_t b, int h, int i, int64_t t) {
    StepIn in;
    const int64_t c = (int64_t)h * DH + i;
    const PxT* x = static_cast<const PxT*>(pr.px) + (b * pr.T + t) * 3 * pr.D + c;
    in.pz = ldp(x);
    in.pr = ldp(x + pr.D);
    in.pc = ldp(x + 2 * pr.D);
    // h^(k)_t: the iterate buffer, or the warm start f(0, x_t) = sig(p_z) tanh(p_c)
    in.s = pr.Hold ? pr.Hold[(b * pr.T + t) * pr.D + c] : sigmoid_f(in.pz) * tanh_f(in.pc);
    return in;
}

// h^(k)_{t0-1} of row i: h0 (or 0) before the sequence, else as load_step
template <int DH, typename PxT>
__device__ __forceinline__ float iterate_before(const Params& pr, int64_t b, int h, int i, int64_t t0) {
    if (t0 == 0) return pr.h0 ? pr.h0[b * pr.D + (int64_t)h * DH + i] : 0.0f;
    return load_step<DH, PxT>(pr, b, h, i, t0 - 1).s;
}

// The cell's row i at (s_prev, x_t), given the row's pre-activation sums
// u_g = (U_g s_prev)_i: F = h^(k)_t - f and the Jacobian's row factors.
struct RowLin {
    float F, dz, al, be, ga;
};

__device__ __forceinline__ RowLin row_linearise(const StepIn& in, float sp, float uz, float ur, float uc) {
    RowLin o;
    const float z = sigmoid_f(in.pz + uz);
    const float r = sigmoid_f(in.pr + ur);
    const float c = tanh_f(__fmaf_rn(r, uc, in.pc));
    const float f = __fmaf_rn(z, c - sp, sp);
    const float zc = z * __fmaf_rn(-c, c, 1.0f);  // z (1 - c^2)
    o.F = in.s - f;
    o.dz = 1.0f - z;
    o.al = (c - sp) * (z - z * z);
    o.be = zc * uc * (r - r * r);
    o.ga = zc * r;
    return o;
}

// step t's forward row factors of row i, for the walk
template <int DH>
__device__ __forceinline__ void store_row_factors(const Params& pr, int64_t seq, int64_t t, int i, float s,
                                                  const RowLin& L) {
    float* o = pr.L + ((seq * pr.T + t) * kNF) * DH + i;
    o[0] = s;
    o[DH] = L.F;
    o[2 * DH] = L.dz;
    o[3 * DH] = L.al;
    o[4 * DH] = L.be;
    o[5 * DH] = L.ga;
}

// max over the block into *resid: a warp max, then one atomic per warp
// (a NaN wins, so a non-finite residual stays visible)
__device__ __forceinline__ void block_max_resid(float v, float* resid) {
    for (int o = 16; o > 0; o >>= 1) v = nanmax_f(v, __shfl_xor_sync(0xffffffffu, v, o));
    if ((threadIdx.x & 31) == 0 && (v > 0.0f || v != v)) atomic_max_nonneg(resid, v);
}

// ---- A: the chunk's Jacobian product and its delta from a zero carry -----
// (or, with kResidOnly, just max |F(h^(k))| over the chunk).  This is the
// kernel for head widths 16 and 32 (and the residual-only pass of every
// width); width 64 runs head_chunk_tc_kernel below.
//
// The product P <- A_t P (d x d x d per step) runs on the tensor cores with
// mma.sync m16n8k8 in TF32.  TF32 keeps 10 mantissa bits, so each operand is
// kept as a TF32 head and a TF32 remainder, x = x_hi + x_lo, and the product
// accumulates a_lo b_hi + a_hi b_lo + a_hi b_hi in float32 (the lo * lo term
// is below float32 rounding): float32 accuracy from three TF32 products.
// The running product is split once, by the thread that produces it, and
// stored as {hi, lo} pairs (each of its elements is read by several warps);
// the Jacobian is stored as float and split when its fragment is loaded.
// Rows are padded (d + 4 pairs, d + 8 floats), which puts each warp's (or
// half-warp's, for 64-bit pairs) fragment loads on distinct banks.
constexpr int kPad = 4;
constexpr int kPadA = 8;

template <int DH>
struct SmemA {
    float AT[2][DH][DH + kPadA];  // A_t transposed (AT[m][i] = A_t[i][m]), two steps in turn
    uint2 Pm[2][DH][DH + kPad];   // running product, row-major, {hi, lo} TF32 pairs
    float sv[2][Geo<DH>::VLEN];   // h^(k) rows, permuted (vpos), two steps in turn
    float dv[2][Geo<DH>::VLEN];   // delta rows, permuted, two steps in turn
};

__device__ __forceinline__ uint2 split_tf32(float x) {
    uint32_t h, l;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(h) : "f"(x));
    const float r = x - __uint_as_float(h);
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(l) : "f"(r));
    return make_uint2(h, l);
}

__device__ __forceinline__ void mma_tf32(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Pout = A Pin, with A given transposed (AT[m][i] = A[i][m]) -- or, with
// kLeftT = false, Pout = AT Pin; all three d x d
// {hi, lo} arrays with row stride d + kPad.  The 16 x 8 output tiles are
// spread over the 8 warps, the tiles of one warp sharing their rows (and so
// their A fragments).  Fragment layout of m16n8k8 (lane = 4 g + t): A rows g
// and g+8, columns t and t+4; B rows t and t+4, column g; C rows g and g+8,
// columns 2t and 2t+1.
template <int DH, bool kLeftT = true>
__device__ __forceinline__ void matmul_tf32x3(const float (*AT)[DH + kPadA], const uint2 (*Pin)[DH + kPad],
                                              uint2 (*Pout)[DH + kPad]) {
    constexpr int MT = DH / 16, NT = DH / 8;             // 16-row and 8-column tiles
    constexpr int WPM = (kThreads / 32) / MT;            // warps per row of tiles
    constexpr int NPW = NT / WPM > 0 ? NT / WPM : 1;     // column tiles per warp
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int mt = warp % MT, nt0 = (warp / MT) * NPW;
    if (nt0 >= NT) return;
    const int r0 = mt * 16 + g;
    float c[NPW][4];
#pragma unroll
    for (int n = 0; n < NPW; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) c[n][e] = 0.0f;
#pragma unroll 2
    for (int ks = 0; ks < DH / 8; ++ks) {
        const int k0 = ks * 8 + t;
        // kLeftT: the left factor is the transpose of AT (A[r][k] = AT[k][r]);
        // otherwise AT itself, row-major (the backward's A^T)
        const uint2 a0 = split_tf32(kLeftT ? AT[k0][r0] : AT[r0][k0]);
        const uint2 a1 = split_tf32(kLeftT ? AT[k0][r0 + 8] : AT[r0 + 8][k0]);
        const uint2 a2 = split_tf32(kLeftT ? AT[k0 + 4][r0] : AT[r0][k0 + 4]);
        const uint2 a3 = split_tf32(kLeftT ? AT[k0 + 4][r0 + 8] : AT[r0 + 8][k0 + 4]);
        const uint32_t ahi[4] = {a0.x, a1.x, a2.x, a3.x}, alo[4] = {a0.y, a1.y, a2.y, a3.y};
#pragma unroll
        for (int n = 0; n < NPW; ++n) {
            const int col = (nt0 + n) * 8 + g;
            const uint2 b0 = Pin[k0][col], b1 = Pin[k0 + 4][col];
            mma_tf32(c[n], alo, b0.x, b1.x);
            mma_tf32(c[n], ahi, b0.y, b1.y);
            mma_tf32(c[n], ahi, b0.x, b1.x);
        }
    }
#pragma unroll
    for (int n = 0; n < NPW; ++n) {
        const int col = (nt0 + n) * 8 + 2 * t;
        Pout[r0][col] = split_tf32(c[n][0]);
        Pout[r0][col + 1] = split_tf32(c[n][1]);
        Pout[r0 + 8][col] = split_tf32(c[n][2]);
        Pout[r0 + 8][col + 1] = split_tf32(c[n][3]);
    }
}

// One block barrier per step, and the product of step t shares its barrier
// interval with the row work of step t+1 (A_{t+1} depends on the known
// iterate only, not on the product), so the tensor and FMA/ALU pipes work
// side by side.  Step t's row work reads sv/dv[p] (h^(k)_{t-1}, delta_{t-1})
// and writes AT[p] = A_t and sv/dv[p ^ 1], p = (t - t0) & 1; the product of
// step t reads AT[p] and Pm[cur] and writes Pm[cur ^ 1].  Every buffer is
// rewritten only after a barrier that all readers of its previous contents
// have passed.
template <int DH, typename PxT, bool kResidOnly>
__global__ void __launch_bounds__(kThreads, 2) head_chunk_kernel(const Params pr) {
    using Gm = Geo<DH>;
    constexpr int TPR = Gm::TPR, SEG = Gm::SEG, SEGP = Gm::SEGP;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto& sm = *reinterpret_cast<SmemA<DH>*>(smem_raw);
    const int tid = threadIdx.x, i = tid / TPR, qt = tid % TPR;
    const int64_t task = blockIdx.x;
    const int64_t seq = task / pr.nChunks;
    const int chunk = (int)(task - seq * pr.nChunks);
    const int64_t b = seq / pr.nh;
    const int h = (int)(seq - b * pr.nh);
    const int64_t t0 = (int64_t)chunk * kChunk;
    const int64_t t1 = t0 + kChunk < pr.T ? t0 + kChunk : pr.T;

    RowU<DH> U;
    U.load(pr.U, pr.nh, h, i, qt);
    const float s_before = iterate_before<DH, PxT>(pr, b, h, i, t0);
    if (qt == 0) {
        sm.sv[0][Gm::vpos(i)] = s_before;
        sm.dv[0][Gm::vpos(i)] = 0.0f;
    }
    if constexpr (!kResidOnly)
        for (int idx = tid; idx < DH * DH; idx += kThreads)
            sm.Pm[0][idx / DH][idx % DH] = make_uint2(idx / DH == idx % DH ? __float_as_uint(1.0f) : 0u, 0u);
    float rmax = 0.0f;

    // the row work of step t: row i of A_t into AT[p], the row factors for
    // the walk, and the next rows of the iterate and of delta
    // (delta_t = A_t delta_{t-1} - F_t)
    auto row_step = [&](const StepIn& in, int p, int64_t t) {
        float uz = 0.0f, ur = 0.0f, uc = 0.0f;
#pragma unroll
        for (int s = 0; s < SEG; ++s) {
            const float x = sm.sv[p][qt * SEGP + s];
            uz = __fmaf_rn(U.z[s], x, uz);
            ur = __fmaf_rn(U.r[s], x, ur);
            uc = __fmaf_rn(U.c[s], x, uc);
        }
        uz = row_sum<DH>(uz);
        ur = row_sum<DH>(ur);
        uc = row_sum<DH>(uc);
        const float sp = sm.sv[p][Gm::vpos(i)];
        const RowLin L = row_linearise(in, sp, uz, ur, uc);
        if (qt == 0) rmax = nanmax_f(rmax, fabsf(L.F));
        if constexpr (!kResidOnly) {
            if (qt == 0) store_row_factors<DH>(pr, seq, t, i, in.s, L);
            float dp = 0.0f;
#pragma unroll
            for (int s = 0; s < SEG; ++s) {
                const int m = qt + TPR * s;
                float a = __fmaf_rn(L.al, U.z[s], (m == i) ? L.dz : 0.0f);
                a = __fmaf_rn(L.be, U.r[s], a);
                a = __fmaf_rn(L.ga, U.c[s], a);
                sm.AT[p][m][i] = a;
                dp = __fmaf_rn(a, sm.dv[p][qt * SEGP + s], dp);
            }
            dp = row_sum<DH>(dp);
            if (qt == 0) sm.dv[p ^ 1][Gm::vpos(i)] = dp - L.F;
        }
        if (qt == 0) sm.sv[p ^ 1][Gm::vpos(i)] = in.s;
    };

    StepIn nxt = load_step<DH, PxT>(pr, b, h, i, t0);
    __syncthreads();
    {
        const StepIn in = nxt;
        if (t0 + 1 < t1) nxt = load_step<DH, PxT>(pr, b, h, i, t0 + 1);
        row_step(in, 0, t0);
    }
    __syncthreads();
    int p = 0, cur = 0;
    for (int64_t t = t0; t < t1; ++t) {
        if constexpr (!kResidOnly) matmul_tf32x3<DH>(sm.AT[p], sm.Pm[cur], sm.Pm[cur ^ 1]);
        if (t + 1 < t1) {
            const StepIn in = nxt;
            if (t + 2 < t1) nxt = load_step<DH, PxT>(pr, b, h, i, t + 2);
            row_step(in, p ^ 1, t + 1);
        }
        __syncthreads();
        cur ^= 1;
        p ^= 1;
    }
    if (pr.resid) block_max_resid(rmax, pr.resid + pr.k);
    if constexpr (!kResidOnly) {
        float* Pout = pr.P + task * DH * DH;
        for (int idx = tid; idx < DH * DH; idx += kThreads) {
            const uint2 v = sm.Pm[cur][idx / DH][idx % DH];
            Pout[idx] = __uint_as_float(v.x) + __uint_as_float(v.y);
        }
        // delta at the chunk's last step: written to dv[(t1 - t0) & 1]
        if (qt == 0) pr.q[task * DH + i] = sm.dv[p][Gm::vpos(i)];
    }
}

// ---- A on the fifth-generation tensor cores (head width 64) -------------
// The chunk work of head_chunk_kernel, with the product P <- A_t P issued as
// tcgen05.mma (kind::tf32, M = N = 64, K = 8 per instruction) and formed
// transposed, P^T <- P^T A_t^T, so that both operands are K-major: operands
// in shared memory, the accumulators in tensor memory.  One chunk
// per block, two blocks per SM: the blocks run unsynchronised, so one's
// tensor-core work overlaps the other's tensor-memory epilogue and barrier.
// The head/remainder split is kept (x = x_hi + x_lo; a_lo b_hi, a_hi b_lo and
// a_hi b_hi, each accumulated over K in float32 in tensor memory by its own
// issuing thread, summed in the epilogue): the head is rounded to
// TF32 with cvt.rna, the remainder stored as float (its low bits are below
// float32 rounding of the product).
//
// Operand layout (no swizzle; "core matrices" of 8 rows of 16 bytes), one
// for both: row i, K index m of a 64 x 64 operand at float (m / 4) * 256 +
// (i / 8) * 32 + (i % 8) * 4 + m % 4, i.e. 8-row groups 128 bytes apart
// (stride byte offset) and 4-column K chunks 1024 bytes apart (leading byte
// offset).  The right operand A_t^T (K x N) is stored as its N rows, which
// are the rows of A_t: row i of A_t is row i of the operand.  The left
// operand P^T has row n = column n of P.  Both are written by the threads
// that produce them with conflict-free stores: a warp's Jacobian rows fill
// whole 128-byte lines, and each eight threads of the epilogue write eight
// consecutive 16-byte core rows.
//
// With M = 64, row r of the accumulator is tensor-memory lane
// 32 (r / 16) + r % 16.  Warp w reads lanes 32 (w % 4) .. +15 of columns
// 32 (w / 4) .. +31 with one 16x32bx2 load: threads 0-15 get the first 16
// columns, threads 16-31 the next 16.
//
// One block barrier per step, as in head_chunk_kernel: after it the issuing
// threads start the product of step t; all threads form the Jacobian rows of
// step t+1 meanwhile, then wait for the product (mbarrier signalled by each
// issuer's tcgen05.commit), move it from tensor memory into the P operand,
// fence the generic-proxy writes for the tensor cores, and meet at the next
// barrier.
namespace tc {

constexpr int kD = 64;
constexpr uint32_t kTmemCols = 256;  // forward: three 64-column accumulators, one per split term
constexpr uint32_t kTmemColsB = 64;  // backward: one accumulator
constexpr uint64_t kWaitNs = 1000000000ull;  // 1 s: far beyond one step's product

struct Smem {
    float Ahi[2][kD * kD];  // A_t, K-major, two steps in turn
    float Alo[2][kD * kD];
    float Phi[kD * kD];     // running product P^T, K-major
    float Plo[kD * kD];
    float sv[2][Geo<kD>::VLEN];  // h^(k) rows, permuted (vpos), two steps in turn
    float dv[2][Geo<kD>::VLEN];  // delta rows, permuted, two steps in turn
    uint64_t bar;           // the product of this step is done
    uint32_t tmem;          // tensor-memory base address from tcgen05.alloc
    int abort;              // a wait ran out: stop issuing, keep the barrier count
};

__device__ __forceinline__ int a_idx(int i, int m) { return (m >> 2) * 256 + (i >> 3) * 32 + (i & 7) * 4 + (m & 3); }

// shared-memory matrix descriptor: start, leading and stride byte offsets
// (each >> 4), descriptor version 1, no swizzle
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// instruction descriptor: f32 accumulator, A and B TF32, both K-major,
// N = 64, M = 64.  (With B MN-major and no swizzle the TF32 product came out
// zero on sm_100a, so every operand here is K-major: the products are formed
// transposed, the running product as the left operand.)
constexpr uint32_t kIdesc = (1u << 4) | (2u << 7) | (2u << 10) | ((64u >> 3) << 17) | ((64u >> 4) << 24);

__device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t b, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d), "l"(a), "l"(b), "r"(kIdesc), "r"(accumulate));
}

__device__ __forceinline__ void commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// generic-proxy shared-memory writes made visible to the tensor cores
__device__ __forceinline__ void fence_operands() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void sync_block() {
    fence_operands();
    fence_before();
    __syncthreads();
    fence_after();
}

// 16 lanes x 16 columns twice (the second half 16 columns on), and the
// wait for the load in the same statement so no use can move above it
__device__ __forceinline__ void load_acc(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16], 16;\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
}

// the three accumulators (64 columns apart) of a thread's 16 columns,
// summed as (lo.hi + hi.lo) + hi.hi
__device__ __forceinline__ void load_acc3(uint32_t taddr, float (&v)[16]) {
    float w[16];
    load_acc(taddr, v);
    load_acc(taddr + 64u, w);
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] += w[j];
    load_acc(taddr + 128u, w);
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] += w[j];
}

__device__ __forceinline__ float tf32_head(float x) {
    uint32_t h;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(h) : "f"(x));
    return __uint_as_float(h);
}

}  // namespace tc

template <typename PxT>
__global__ void __launch_bounds__(kThreads, 2) head_chunk_tc_kernel(const Params pr) {
    using Gm = Geo<tc::kD>;
    constexpr int TPR = Gm::TPR, SEG = Gm::SEG, SEGP = Gm::SEGP, DH = tc::kD;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto& sm = *reinterpret_cast<tc::Smem*>(smem_raw);
    volatile int& abort_flag = sm.abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, i = tid / TPR, qt = tid % TPR;
    const int64_t task = blockIdx.x;
    const int64_t seq = task / pr.nChunks;
    const int chunk = (int)(task - seq * pr.nChunks);
    const int64_t b = seq / pr.nh;
    const int h = (int)(seq - b * pr.nh);
    const int64_t t0 = (int64_t)chunk * kChunk;
    const int64_t t1 = t0 + kChunk < pr.T ? t0 + kChunk : pr.T;

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem)),
                     "r"(tc::kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        mbar_init(&sm.bar, 3);  // one arrival per issuing thread
        abort_flag = 0;
        mbar_fence_init();
    }
    RowU<DH> U;
    U.load(pr.U, pr.nh, h, i, qt);
    const float s_before = iterate_before<DH, PxT>(pr, b, h, i, t0);
    if (qt == 0) {
        sm.sv[0][Gm::vpos(i)] = s_before;
        sm.dv[0][Gm::vpos(i)] = 0.0f;
    }
    // P^T = I
    for (int idx = tid; idx < DH * DH; idx += kThreads) {
        const int k = idx / DH, n = idx % DH;
        sm.Phi[tc::a_idx(n, k)] = k == n ? 1.0f : 0.0f;
        sm.Plo[tc::a_idx(n, k)] = 0.0f;
    }
    float rmax = 0.0f;

    // the row work of step t: row i of A_t (split) into A[p], the row factors
    // for the walk, and the next rows of the iterate and of delta
    // (delta_t = A_t delta_{t-1} - F_t)
    auto row_step = [&](const StepIn& in, int p, int64_t t) {
        float uz = 0.0f, ur = 0.0f, uc = 0.0f;
#pragma unroll
        for (int s = 0; s < SEG; ++s) {
            const float x = sm.sv[p][qt * SEGP + s];
            uz = __fmaf_rn(U.z[s], x, uz);
            ur = __fmaf_rn(U.r[s], x, ur);
            uc = __fmaf_rn(U.c[s], x, uc);
        }
        uz = row_sum<DH>(uz);
        ur = row_sum<DH>(ur);
        uc = row_sum<DH>(uc);
        const float sp = sm.sv[p][Gm::vpos(i)];
        const RowLin L = row_linearise(in, sp, uz, ur, uc);
        if (qt == 0) {
            rmax = nanmax_f(rmax, fabsf(L.F));
            store_row_factors<DH>(pr, seq, t, i, in.s, L);
        }
        float* ahi = sm.Ahi[p];
        float* alo = sm.Alo[p];
        float dp = 0.0f;
#pragma unroll
        for (int s = 0; s < SEG; ++s) {
            const int m = qt + TPR * s;
            float a = __fmaf_rn(L.al, U.z[s], (m == i) ? L.dz : 0.0f);
            a = __fmaf_rn(L.be, U.r[s], a);
            a = __fmaf_rn(L.ga, U.c[s], a);
            const float hi = tc::tf32_head(a);
            ahi[tc::a_idx(i, m)] = hi;
            alo[tc::a_idx(i, m)] = a - hi;
            dp = __fmaf_rn(a, sm.dv[p][qt * SEGP + s], dp);
        }
        dp = row_sum<DH>(dp);
        if (qt == 0) {
            sm.dv[p ^ 1][Gm::vpos(i)] = dp - L.F;
            sm.sv[p ^ 1][Gm::vpos(i)] = in.s;
        }
    };

    StepIn nxt = load_step<DH, PxT>(pr, b, h, i, t0);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = sm.tmem;
    {
        const StepIn in = nxt;
        if (t0 + 1 < t1) nxt = load_step<DH, PxT>(pr, b, h, i, t0 + 1);
        row_step(in, 0, t0);
    }
    tc::sync_block();

    // epilogue geometry: this thread's row and columns of the accumulator
    const int eq = warp & 3;
    const int ek = 16 * eq + (lane & 15);              // product row
    const int en = 32 * (warp >> 2) + 16 * (lane >> 4);  // first of 16 columns
    const uint32_t taddr = tmem + ((uint32_t)(32 * eq) << 16) + (uint32_t)(32 * (warp >> 2));

    int p = 0;
    for (int64_t t = t0; t < t1; ++t) {
        const uint32_t par = (uint32_t)((t - t0) & 1);
        if ((tid == 0 || tid == 96 || tid == 192) && !abort_flag) {
            // P_t^T = P_{t-1}^T A_t^T: the left operand is P^T (rows n, K
            // index k), the right one A_t with its rows as the N index.  One
            // split term per issuing thread (threads of warps 0, 3 and 6),
            // each into its own accumulator: one thread issuing all 24 MMAs
            // delayed its warp's row work, and the block's barrier with it.
            // K step ks starts 2048 bytes further on in both operands: 128 in
            // the descriptors' start-address field (no carry out of it)
            const int term = tid / 96;  // 0: P_hi A_lo, 1: P_lo A_hi, 2: P_hi A_hi
            const uint64_t da = tc::sdesc(smem_u32(term == 1 ? sm.Plo : sm.Phi), 1024, 128);
            const uint64_t db = tc::sdesc(smem_u32(term == 0 ? sm.Alo[p] : sm.Ahi[p]), 1024, 128);
            const uint32_t d = tmem + 64u * (uint32_t)term;
#pragma unroll
            for (int ks = 0; ks < DH / 8; ++ks) {
                const uint64_t ko = (uint64_t)ks * 128u;
                tc::mma(d, da + ko, db + ko, ks > 0 ? 1u : 0u);
            }
            tc::commit(&sm.bar);
        }
        if (t + 1 < t1) {
            const StepIn in = nxt;
            if (t + 2 < t1) nxt = load_step<DH, PxT>(pr, b, h, i, t + 2);
            row_step(in, p ^ 1, t + 1);
        }
        // wait for the product (bounded), then move it out of tensor memory
        if (!abort_flag) {
            uint64_t start = 0;
            while (!mbar_try_wait(&sm.bar, par)) {
                const uint64_t now = globaltimer_ns();
                if (start == 0) {
                    start = now | 1;
                } else if (now - start > tc::kWaitNs) {
                    if (lane == 0) atomicOr(pr.status, kStatusTimeout);
                    abort_flag = 1;
                    break;
                }
            }
        }
        tc::fence_after();
        float v[16];
        tc::load_acc3(taddr, v);
        if (t + 1 < t1) {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                float4 hv, lv;
                hv.x = tc::tf32_head(v[4 * g + 0]);
                hv.y = tc::tf32_head(v[4 * g + 1]);
                hv.z = tc::tf32_head(v[4 * g + 2]);
                hv.w = tc::tf32_head(v[4 * g + 3]);
                lv.x = v[4 * g + 0] - hv.x;
                lv.y = v[4 * g + 1] - hv.y;
                lv.z = v[4 * g + 2] - hv.z;
                lv.w = v[4 * g + 3] - hv.w;
                const int o = tc::a_idx(ek, en + 4 * g);
                *reinterpret_cast<float4*>(sm.Phi + o) = hv;
                *reinterpret_cast<float4*>(sm.Plo + o) = lv;
            }
        } else {
            // row ek of P^T is column ek of P (row-major in the workspace)
            float* Pout = pr.P + task * DH * DH + (int64_t)en * DH + ek;
#pragma unroll
            for (int j = 0; j < 16; ++j) Pout[(int64_t)j * DH] = v[j];
        }
        tc::sync_block();
        p ^= 1;
    }
    if (pr.resid) block_max_resid(rmax, pr.resid + pr.k);
    // delta at the chunk's last step: written to dv[(t1 - t0) & 1]
    if (qt == 0) pr.q[task * DH + i] = sm.dv[p][Gm::vpos(i)];
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(tc::kTmemCols)
                     : "memory");
}

// ---- B: the carries of one (batch row, head), chunk after chunk ----------
// Thread i keeps row i of the next chunk's P in registers while it applies
// the current one, so each chunk costs one dependent step, not a load's
// latency.  The forward runs the chunks in time order from delta_{-1} = 0
// (h0 is given, not solved for); the backward (kReverse) runs them from the
// end, from mu_T = 0.
template <int DH, bool kReverse = false>
__global__ void __launch_bounds__(64) head_carry_kernel(const Params pr) {
    __shared__ float x[2][DH];
    const int64_t seq = blockIdx.x;
    const int i = threadIdx.x;
    const bool act = i < DH;
    if (act) x[0][i] = 0.0f;
    float4 row[DH / 4];
    float qv = 0.0f;
    auto fetch = [&](int k) {
        const int c = kReverse ? pr.nChunks - 1 - k : k;
        const int64_t task = seq * pr.nChunks + c;
        const float4* Prow = reinterpret_cast<const float4*>(pr.P + (task * DH + i) * DH);
#pragma unroll
        for (int m = 0; m < DH / 4; ++m) row[m] = Prow[m];
        qv = pr.q[task * DH + i];
    };
    if (act) fetch(0);
    __syncthreads();
    int cur = 0;
    for (int c = 0; c < pr.nChunks; ++c) {
        float4 r[DH / 4];
        float qc = qv;
#pragma unroll
        for (int m = 0; m < DH / 4; ++m) r[m] = row[m];
        if (act && c + 1 < pr.nChunks) fetch(c + 1);
        if (act) {
            const int cc = kReverse ? pr.nChunks - 1 - c : c;
            pr.carry[(seq * pr.nChunks + cc) * DH + i] = x[cur][i];
            float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int m = 0; m < DH / 4; ++m) {
                acc[0] = __fmaf_rn(r[m].x, x[cur][4 * m], acc[0]);
                acc[1] = __fmaf_rn(r[m].y, x[cur][4 * m + 1], acc[1]);
                acc[2] = __fmaf_rn(r[m].z, x[cur][4 * m + 2], acc[2]);
                acc[3] = __fmaf_rn(r[m].w, x[cur][4 * m + 3], acc[3]);
            }
            x[cur ^ 1][i] = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + qc;
        }
        __syncthreads();
        cur ^= 1;
    }
}

// ---- C: re-walk each chunk from its carry and write h^(k+1) --------------
// delta_t = A_t delta_{t-1} - F_t with A_t applied as
// diag(1-z) + diag(alpha) U_z + diag(beta) U_r + diag(gamma) U_c.  The row
// factors (h^(k)_t, F_t, 1 - z, alpha, beta, gamma) are the ones the chunk
// kernel formed for the Jacobian rows, so per step the walk does only the
// dependent chain: three dot products with delta_{t-1} and the update.  One
// block barrier per step, delta double-buffered.  The row's first thread,
// the only one that combines the factors, loads them four steps ahead into
// one of four register sets that take turns with the steps (the loop body
// is unrolled four times so that a set is consumed before it is reloaded
// and no register copy waits on a load in flight).

template <int DH>
__global__ void __launch_bounds__(kThreads, 2) head_walk_kernel(const Params pr) {
    using Gm = Geo<DH>;
    constexpr int TPR = Gm::TPR, SEG = Gm::SEG, SEGP = Gm::SEGP;
    __shared__ float dv[2][Gm::VLEN];  // delta rows, permuted, two steps in turn
    const int tid = threadIdx.x, i = tid / TPR, qt = tid % TPR;
    const int64_t task = blockIdx.x;
    const int64_t seq = task / pr.nChunks;
    const int chunk = (int)(task - seq * pr.nChunks);
    const int64_t b = seq / pr.nh;
    const int h = (int)(seq - b * pr.nh);
    const int64_t t0 = (int64_t)chunk * kChunk;
    const int64_t t1 = t0 + kChunk < pr.T ? t0 + kChunk : pr.T;

    RowU<DH> U;
    U.load(pr.U, pr.nh, h, i, qt);
    auto load_f = [&](int64_t t, float (&f)[kNF]) {
        const float* src = pr.L + ((seq * pr.T + t) * kNF) * DH + i;
#pragma unroll
        for (int j = 0; j < kNF; ++j) f[j] = src[j * DH];
    };
    float fa[kNF], fb[kNF], fc[kNF], fd[kNF];
    if (qt == 0) {
        dv[0][Gm::vpos(i)] = pr.carry[task * DH + i];
        load_f(t0, fa);
        if (t0 + 1 < t1) load_f(t0 + 1, fb);
        if (t0 + 2 < t1) load_f(t0 + 2, fc);
        if (t0 + 3 < t1) load_f(t0 + 3, fd);
    }
    __syncthreads();
    int par = 0;
    bool bad = false;
    auto step = [&](int64_t t, float (&f)[kNF]) {
        float vz = 0.0f, vr = 0.0f, vc = 0.0f;
#pragma unroll
        for (int s = 0; s < SEG; ++s) {
            const float y = dv[par][qt * SEGP + s];
            vz = __fmaf_rn(U.z[s], y, vz);
            vr = __fmaf_rn(U.r[s], y, vr);
            vc = __fmaf_rn(U.c[s], y, vc);
        }
        vz = row_sum<DH>(vz);
        vr = row_sum<DH>(vr);
        vc = row_sum<DH>(vc);
        if (qt == 0) {
            const float dprev = dv[par][Gm::vpos(i)];
            float d = __fmaf_rn(f[2], dprev, -f[1]);  // (1 - z) delta_{t-1} - F_t
            d = __fmaf_rn(f[3], vz, d);
            d = __fmaf_rn(f[4], vr, d);
            d = __fmaf_rn(f[5], vc, d);
            const float hn = f[0] + d;
            pr.Hnew[(b * pr.T + t) * pr.D + (int64_t)h * DH + i] = hn;
            bad |= !isfinite(hn);
            dv[par ^ 1][Gm::vpos(i)] = d;
            if (t + 4 < t1) load_f(t + 4, f);
        }
        __syncthreads();
        par ^= 1;
    };
    for (int64_t t = t0; t < t1; t += 4) {
        step(t, fa);
        if (t + 1 < t1) step(t + 1, fb);
        if (t + 2 < t1) step(t + 2, fc);
        if (t + 3 < t1) step(t + 3, fd);
    }
    if (__any_sync(0xffffffffu, bad) && (tid & 31) == 0) atomicOr(pr.status, kStatusNonFinite);
}

// ==== the adjoint ===========================================================
// At the trajectory H, with g_t = dL/dH_t, the kernels scan the propagated
// adjoint mu_t = A_t^T lambda_t in reverse time:
//     mu_t = A_t^T (g_t + mu_{t+1}),  mu_T = 0,  lambda_t = g_t + mu_{t+1},
// so that each element needs only its own row's Jacobian (the same reading
// as the diagonal cells' backward), and dL/dh0 = mu_0.  Then
//     dL/dp_z = lambda * alpha, dL/dp_r = lambda * beta, dL/dp_c = lambda * z (1 - c^2),
//     dL/dU_g = sum_{b,t} (lambda * f_g) h_{t-1}^T,  f = alpha, beta, gamma.
// Launches: the chunk kernel (Q = A_{t0}^T ... A_{t1-1}^T on the tensor cores
// and the chunk's mu from a zero carry), the carry kernel in reverse chunk
// order, the walk kernel (lambda, dL/dpx, lambda * gamma, mu, dL/dh0) and a
// fixed-order reduction of the outer products for dL/dU.

// Per-step inputs of the backward row work for row i: pre-activations,
// g_t[i], and the state two rows back (the one the next row work needs).
struct BStepIn {
    float pz, pr, pc, g, s2;
};

template <int DH, typename PxT>
__device__ __forceinline__ BStepIn load_bstep(const Params& pr, int64_t b, int h, int i, int64_t t) {
    BStepIn in;
    const int64_t c = (int64_t)h * DH + i;
    const PxT* x = static_cast<const PxT*>(pr.px) + (b * pr.T + t) * 3 * pr.D + c;
    in.pz = ldp(x);
    in.pr = ldp(x + pr.D);
    in.pc = ldp(x + 2 * pr.D);
    in.g = pr.G[(b * pr.T + t) * pr.D + c];
    const int64_t t2 = t - 2;
    in.s2 = t2 >= 0 ? pr.Hold[(b * pr.T + t2) * pr.D + c] : (t2 == -1 && pr.h0 ? pr.h0[b * pr.D + c] : 0.0f);
    return in;
}

// the state just before row t (h_{t-1}, h0 at t = 0)
template <int DH>
__device__ __forceinline__ float state_before(const Params& pr, int64_t b, int h, int i, int64_t t) {
    const int64_t c = (int64_t)h * DH + i;
    if (t >= 1) return pr.Hold[(b * pr.T + t - 1) * pr.D + c];
    return pr.h0 ? pr.h0[b * pr.D + c] : 0.0f;
}

template <int DH>
struct SmemB {
    float AT[2][DH][DH + kPadA];  // AT[m][i] = A_t[i][m] = (A_t^T)[m][i], two steps in turn
    uint2 Pm[2][DH][DH + kPad];   // the running product of transposed Jacobians ({hi, lo} pairs)
    float sv[2][Geo<DH>::VLEN];   // h_{t-1} rows for the row work (permuted)
    float gv[2][Geo<DH>::VLEN];   // g_t rows (permuted)
    float mv[2][Geo<DH>::VLEN];   // mu rows (permuted)
};

// step t's backward row factors of row i, for the walk
template <int DH>
__device__ __forceinline__ void store_brow_factors(const Params& pr, int64_t seq, int64_t t, int i, float dz, float al,
                                                   float be, float zc, float ga) {
    float* o = pr.L + ((seq * pr.T + t) * kNB) * DH + i;
    o[0] = dz;
    o[DH] = al;
    o[2 * DH] = be;
    o[3 * DH] = zc;
    o[4 * DH] = ga;
}

// The backward's row work for step t, parity p: the gates at (h_{t-1}, x_t),
// row i of A_t into AT[p], the row factors for the walk, g_t into gv, and
// h_{t-2} into sv[p ^ 1] for the next (earlier) step's row work.
template <int DH>
__device__ __forceinline__ void bwd_row_work(SmemB<DH>& sm, const RowU<DH>& U, const BStepIn& in, int p, int i,
                                             int qt, const Params& pr, int64_t seq, int64_t t) {
    constexpr int TPR = Geo<DH>::TPR, SEG = Geo<DH>::SEG, SEGP = Geo<DH>::SEGP;
    float uz = 0.0f, ur = 0.0f, uc = 0.0f;
#pragma unroll
    for (int s = 0; s < SEG; ++s) {
        const float x = sm.sv[p][qt * SEGP + s];
        uz = __fmaf_rn(U.z[s], x, uz);
        ur = __fmaf_rn(U.r[s], x, ur);
        uc = __fmaf_rn(U.c[s], x, uc);
    }
    uz = row_sum<DH>(uz);
    ur = row_sum<DH>(ur);
    uc = row_sum<DH>(uc);
    const float sp = sm.sv[p][Geo<DH>::vpos(i)];
    const float z = sigmoid_f(in.pz + uz);
    const float r = sigmoid_f(in.pr + ur);
    const float c = tanh_f(__fmaf_rn(r, uc, in.pc));
    const float zc = z * __fmaf_rn(-c, c, 1.0f);
    const float dz = 1.0f - z, al = (c - sp) * (z - z * z), be = zc * uc * (r - r * r), ga = zc * r;
#pragma unroll
    for (int s = 0; s < SEG; ++s) {
        const int m = qt + TPR * s;
        float a = __fmaf_rn(al, U.z[s], (m == i) ? dz : 0.0f);
        a = __fmaf_rn(be, U.r[s], a);
        a = __fmaf_rn(ga, U.c[s], a);
        sm.AT[p][m][i] = a;
    }
    if (qt == 0) {
        const int vi = Geo<DH>::vpos(i);
        sm.gv[p][vi] = in.g;
        sm.sv[p ^ 1][vi] = in.s2;
        store_brow_factors<DH>(pr, seq, t, i, dz, al, be, zc, ga);
    }
}

// mu_t[m] = sum_i AT[p][m][i] (g_t[i] + mu_{t+1}[i]) for thread (m, qt)
template <int DH>
__device__ __forceinline__ float bwd_mu(const SmemB<DH>& sm, int p, int m, int qt) {
    constexpr int TPR = Geo<DH>::TPR, SEG = Geo<DH>::SEG, SEGP = Geo<DH>::SEGP;
    float acc = 0.0f;
#pragma unroll
    for (int s = 0; s < SEG; ++s) {
        const int i = qt + TPR * s;
        const float lam = sm.gv[p][qt * SEGP + s] + sm.mv[p ^ 1][qt * SEGP + s];
        acc = __fmaf_rn(sm.AT[p][m][i], lam, acc);
    }
    return row_sum<DH>(acc);
}

// ---- backward A: the chunk's product of transposed Jacobians -------------
// Steps run from t1-1 down to t0 (r = t1-1-t, p = r & 1); as in the forward
// chunk kernel the product of step t and mu_t share a barrier interval with
// the row work of step t-1.  (Head widths 16 and 32; 64 runs
// head_bwd_tc_kernel.)
template <int DH, typename PxT>
__global__ void __launch_bounds__(kThreads, 2) head_bwd_kernel(const Params pr) {
    using Gm = Geo<DH>;
    constexpr int TPR = Gm::TPR;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto& sm = *reinterpret_cast<SmemB<DH>*>(smem_raw);
    const int tid = threadIdx.x, i = tid / TPR, qt = tid % TPR;
    const int64_t task = blockIdx.x;
    const int64_t seq = task / pr.nChunks;
    const int chunk = (int)(task - seq * pr.nChunks);
    const int64_t b = seq / pr.nh;
    const int h = (int)(seq - b * pr.nh);
    const int64_t t0 = (int64_t)chunk * kChunk;
    const int64_t t1 = t0 + kChunk < pr.T ? t0 + kChunk : pr.T;

    RowU<DH> U;
    U.load(pr.U, pr.nh, h, i, qt);
    if (qt == 0) {
        sm.sv[0][Gm::vpos(i)] = state_before<DH>(pr, b, h, i, t1 - 1);
        sm.mv[1][Gm::vpos(i)] = 0.0f;  // mu_{t1} for the chunk's own product
    }
    for (int idx = tid; idx < DH * DH; idx += kThreads)
        sm.Pm[0][idx / DH][idx % DH] = make_uint2(idx / DH == idx % DH ? __float_as_uint(1.0f) : 0u, 0u);
    BStepIn nxt = load_bstep<DH, PxT>(pr, b, h, i, t1 - 1);
    __syncthreads();
    {
        const BStepIn in = nxt;
        if (t1 - 2 >= t0) nxt = load_bstep<DH, PxT>(pr, b, h, i, t1 - 2);
        bwd_row_work<DH>(sm, U, in, 0, i, qt, pr, seq, t1 - 1);
    }
    __syncthreads();
    int p = 0, cur = 0;
    for (int64_t t = t1 - 1; t >= t0; --t) {
        matmul_tf32x3<DH, false>(sm.AT[p], sm.Pm[cur], sm.Pm[cur ^ 1]);
        const float mu = bwd_mu<DH>(sm, p, i, qt);  // thread (m = i, qt)
        if (qt == 0) sm.mv[p][Gm::vpos(i)] = mu;
        if (t - 1 >= t0) {
            const BStepIn in = nxt;
            if (t - 2 >= t0) nxt = load_bstep<DH, PxT>(pr, b, h, i, t - 2);
            bwd_row_work<DH>(sm, U, in, p ^ 1, i, qt, pr, seq, t - 1);
        }
        __syncthreads();
        cur ^= 1;
        p ^= 1;
    }
    float* Pout = pr.P + task * DH * DH;
    for (int idx = tid; idx < DH * DH; idx += kThreads) {
        const uint2 v = sm.Pm[cur][idx / DH][idx % DH];
        Pout[idx] = __uint_as_float(v.x) + __uint_as_float(v.y);
    }
    // mu at the chunk's first step: written to mv[p ^ 1] by the last iteration
    if (qt == 0) pr.q[task * DH + i] = sm.mv[p ^ 1][Gm::vpos(i)];
}

// ---- backward C: re-walk each chunk from its carry -----------------------
// From mu_{t1} (the carry) down to t0: lambda_t = g_t + mu_{t+1},
// dL/dpx_t = lambda_t (alpha, beta, z (1 - c^2)), lambda_t gamma (the factor
// of dL/dU_c), and mu_t = A_t^T lambda_t applied without forming A_t:
//     mu_t = (1 - z) lambda + U_z^T (alpha lambda) + U_r^T (beta lambda)
//            + U_c^T (gamma lambda),
// with the row factors the product kernel stored.  Thread (m, qt) keeps
// column m of U_z, U_r, U_c (rows k = qt + TPR s) in registers; the row's
// first thread owns lambda_m and mu_m.  One block barrier per step, the
// scaled vectors double-buffered.
template <int DH>
struct ColU {
    float z[Geo<DH>::SEG], r[Geo<DH>::SEG], c[Geo<DH>::SEG];
    __device__ __forceinline__ void load(const float* U, int nh, int h, int m, int qt) {
        constexpr int SEG = Geo<DH>::SEG, TPR = Geo<DH>::TPR;
        const int64_t hs = (int64_t)DH * DH;
#pragma unroll
        for (int s = 0; s < SEG; ++s) {
            const int k = qt + TPR * s;
            z[s] = __ldg(U + (0 * nh + h) * hs + (int64_t)k * DH + m);
            r[s] = __ldg(U + ((int64_t)1 * nh + h) * hs + (int64_t)k * DH + m);
            c[s] = __ldg(U + ((int64_t)2 * nh + h) * hs + (int64_t)k * DH + m);
        }
    }
};

template <int DH>
__global__ void __launch_bounds__(kThreads, 2) head_bwd_walk_kernel(const Params pr) {
    using Gm = Geo<DH>;
    constexpr int TPR = Gm::TPR, SEG = Gm::SEG, SEGP = Gm::SEGP;
    __shared__ float wv[2][3][Gm::VLEN];  // alpha lambda, beta lambda, gamma lambda (permuted), two steps in turn
    const int tid = threadIdx.x, i = tid / TPR, qt = tid % TPR;
    const int64_t task = blockIdx.x;
    const int64_t seq = task / pr.nChunks;
    const int chunk = (int)(task - seq * pr.nChunks);
    const int64_t b = seq / pr.nh;
    const int h = (int)(seq - b * pr.nh);
    const int64_t t0 = (int64_t)chunk * kChunk;
    const int64_t t1 = t0 + kChunk < pr.T ? t0 + kChunk : pr.T;
    const int64_t col = (int64_t)h * DH + i;

    ColU<DH> UT;
    UT.load(pr.U, pr.nh, h, i, qt);
    // the row factors and g of step t (read by the row's first thread only)
    auto load_f = [&](int64_t t, float (&f)[kNB + 1]) {
        const float* src = pr.L + ((seq * pr.T + t) * kNB) * DH + i;
#pragma unroll
        for (int j = 0; j < kNB; ++j) f[j] = src[j * DH];
        f[kNB] = pr.G[(b * pr.T + t) * pr.D + col];
    };
    // four register sets of factors, taking turns with the steps (as in the
    // forward walk)
    float fa[kNB + 1], fb[kNB + 1], fc[kNB + 1], fd[kNB + 1];
    float mu = 0.0f;  // mu_{t+1} of row i (first thread of the row)
    if (qt == 0) {
        mu = pr.carry[task * DH + i];
        load_f(t1 - 1, fa);
        if (t1 - 2 >= t0) load_f(t1 - 2, fb);
        if (t1 - 3 >= t0) load_f(t1 - 3, fc);
        if (t1 - 4 >= t0) load_f(t1 - 4, fd);
    }
    int par = 0;
    bool bad = false;
    auto step = [&](int64_t t, float (&f)[kNB + 1]) {
        float dzl = 0.0f;
        if (qt == 0) {
            const float lam = f[kNB] + mu;
            const int64_t o = ((b * pr.T + t) * 3) * pr.D + col;
            const float d0 = lam * f[1], d1 = lam * f[2], d2 = lam * f[3];
            pr.dpx[o] = d0;
            pr.dpx[o + pr.D] = d1;
            pr.dpx[o + 2 * pr.D] = d2;
            pr.ec[(b * pr.T + t) * pr.D + col] = lam * f[4];
            bad |= !(isfinite(d0) && isfinite(d1) && isfinite(d2));
            const int vi = Gm::vpos(i);
            wv[par][0][vi] = f[1] * lam;
            wv[par][1][vi] = f[2] * lam;
            wv[par][2][vi] = f[4] * lam;
            dzl = f[0] * lam;
            if (t - 4 >= t0) load_f(t - 4, f);
        }
        __syncthreads();
        float sz = 0.0f, sr = 0.0f, sc = 0.0f;
#pragma unroll
        for (int s = 0; s < SEG; ++s) {
            sz = __fmaf_rn(UT.z[s], wv[par][0][qt * SEGP + s], sz);
            sr = __fmaf_rn(UT.r[s], wv[par][1][qt * SEGP + s], sr);
            sc = __fmaf_rn(UT.c[s], wv[par][2][qt * SEGP + s], sc);
        }
        sz = row_sum<DH>(sz);
        sr = row_sum<DH>(sr);
        sc = row_sum<DH>(sc);
        if (qt == 0) {
            mu = ((dzl + sz) + sr) + sc;  // mu_t
            if (t == 0 && pr.dh0) pr.dh0[b * pr.D + col] = mu;
        }
        par ^= 1;
    };
    for (int64_t t = t1 - 1; t >= t0; t -= 4) {
        step(t, fa);
        if (t - 1 >= t0) step(t - 1, fb);
        if (t - 2 >= t0) step(t - 2, fc);
        if (t - 3 >= t0) step(t - 3, fd);
    }
    if (__any_sync(0xffffffffu, bad) && (tid & 31) == 0) atomicOr(pr.status, kStatusNonFinite);
}

// ---- backward A on the fifth-generation tensor cores (head width 64) ------
// The chunk work of head_bwd_kernel for head width 64, run forward in time
// over the chunk.  The prefix products R_t = A_{t0}^T ... A_t^T
// (R_t = R_{t-1} A_t^T, R_{t0-1} = I) are formed on tcgen05 with the operand
// layout of head_chunk_tc_kernel: R is the left operand, A_t^T the right one
// stored as the rows of A_t, so the Jacobian rows are formed and stored as in
// the forward.  The chunk's product is R_{t1-1} = A_{t0}^T ... A_{t1-1}^T,
// and its adjoint from a zero carry is mu_{t0} = sum_t R_t g_t.  The
// epilogue threads hold R_t after step t's product: each adds its 16
// columns' share R_t[ek][n] g_t[n] to a float32 register, and the four
// shares of a row are summed after the last step.  No thread forms
// A_t^T lambda from shared memory.
namespace tc {


struct SmemB {
    float Ahi[2][kD * kD];  // A_t, K-major (rows of A_t as the N index), two steps in turn
    float Alo[2][kD * kD];
    float Phi[kD * kD];     // R_{t-1}, K-major
    float Plo[kD * kD];
    float gv[2][kD];        // g_t, two steps in turn
    float red[kD];          // the second half of each row's mu shares
    float sv[2][Geo<kD>::VLEN];  // h_{t-1} rows for the row work (permuted)
    uint64_t bar;
    uint32_t tmem;
    int abort;
};

// the bounded wait for a commit (1 s, then the timeout bit and no further MMA)
__device__ __forceinline__ void wait_bar(const Params& pr, uint64_t* bar, uint32_t par, volatile int& abort_flag,
                                         int lane) {
    if (abort_flag) return;
    uint64_t start = 0;
    while (!mbar_try_wait(bar, par)) {
        const uint64_t now = globaltimer_ns();
        if (start == 0) {
            start = now | 1;
        } else if (now - start > kWaitNs) {
            if (lane == 0) atomicOr(pr.status, kStatusTimeout);
            abort_flag = 1;
            return;
        }
    }
}

}  // namespace tc

// Per-step inputs of the forward-in-time backward row work for row i:
// pre-activations, g_t[i] and h_t[i] (the state the next step needs).
struct BStepF {
    float pz, pr, pc, g, s;
};

template <int DH, typename PxT>
__device__ __forceinline__ BStepF load_bstepf(const Params& pr, int64_t b, int h, int i, int64_t t) {
    BStepF in;
    const int64_t c = (int64_t)h * DH + i;
    const PxT* x = static_cast<const PxT*>(pr.px) + (b * pr.T + t) * 3 * pr.D + c;
    in.pz = ldp(x);
    in.pr = ldp(x + pr.D);
    in.pc = ldp(x + 2 * pr.D);
    in.g = pr.G[(b * pr.T + t) * pr.D + c];
    in.s = pr.Hold[(b * pr.T + t) * pr.D + c];
    return in;
}

template <typename PxT>
__global__ void __launch_bounds__(kThreads, 2) head_bwd_tc_kernel(const Params pr) {
    using Gm = Geo<tc::kD>;
    constexpr int TPR = Gm::TPR, SEG = Gm::SEG, SEGP = Gm::SEGP, DH = tc::kD;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto& sm = *reinterpret_cast<tc::SmemB*>(smem_raw);
    volatile int& abort_flag = sm.abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, i = tid / TPR, qt = tid % TPR;
    const int64_t task = blockIdx.x;
    const int64_t seq = task / pr.nChunks;
    const int chunk = (int)(task - seq * pr.nChunks);
    const int64_t b = seq / pr.nh;
    const int h = (int)(seq - b * pr.nh);
    const int64_t t0 = (int64_t)chunk * kChunk;
    const int64_t t1 = t0 + kChunk < pr.T ? t0 + kChunk : pr.T;

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm.tmem)),
                     "r"(tc::kTmemColsB)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        mbar_init(&sm.bar, 1);
        abort_flag = 0;
        mbar_fence_init();
    }
    RowU<DH> U;
    U.load(pr.U, pr.nh, h, i, qt);
    if (qt == 0) sm.sv[0][Gm::vpos(i)] = state_before<DH>(pr, b, h, i, t0);
    // R = I
    for (int idx = tid; idx < DH * DH; idx += kThreads) {
        const int k = idx / DH, n = idx % DH;
        sm.Phi[tc::a_idx(n, k)] = k == n ? 1.0f : 0.0f;
        sm.Plo[tc::a_idx(n, k)] = 0.0f;
    }

    // the row work of step t, parity p: the gates at (h_{t-1}, x_t), row i of
    // A_t (split) into A[p], g_t into gv[p], the row factors for the walk,
    // and h_t into sv[p ^ 1] for the next step
    auto row_step = [&](const BStepF& in, int p, int64_t t) {
        float uz = 0.0f, ur = 0.0f, uc = 0.0f;
#pragma unroll
        for (int s = 0; s < SEG; ++s) {
            const float x = sm.sv[p][qt * SEGP + s];
            uz = __fmaf_rn(U.z[s], x, uz);
            ur = __fmaf_rn(U.r[s], x, ur);
            uc = __fmaf_rn(U.c[s], x, uc);
        }
        uz = row_sum<DH>(uz);
        ur = row_sum<DH>(ur);
        uc = row_sum<DH>(uc);
        const float sp = sm.sv[p][Gm::vpos(i)];
        const float z = sigmoid_f(in.pz + uz);
        const float r = sigmoid_f(in.pr + ur);
        const float c = tanh_f(__fmaf_rn(r, uc, in.pc));
        const float zc = z * __fmaf_rn(-c, c, 1.0f);
        const float dz = 1.0f - z, al = (c - sp) * (z - z * z), be = zc * uc * (r - r * r), ga = zc * r;
        float* ahi = sm.Ahi[p];
        float* alo = sm.Alo[p];
#pragma unroll
        for (int s = 0; s < SEG; ++s) {
            const int m = qt + TPR * s;
            float a = __fmaf_rn(al, U.z[s], (m == i) ? dz : 0.0f);
            a = __fmaf_rn(be, U.r[s], a);
            a = __fmaf_rn(ga, U.c[s], a);
            const float hi = tc::tf32_head(a);
            ahi[tc::a_idx(i, m)] = hi;
            alo[tc::a_idx(i, m)] = a - hi;
        }
        if (qt == 0) {
            sm.gv[p][i] = in.g;
            sm.sv[p ^ 1][Gm::vpos(i)] = in.s;
            store_brow_factors<DH>(pr, seq, t, i, dz, al, be, zc, ga);
        }
    };

    BStepF nxt = load_bstepf<DH, PxT>(pr, b, h, i, t0);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = sm.tmem;
    {
        const BStepF in = nxt;
        if (t0 + 1 < t1) nxt = load_bstepf<DH, PxT>(pr, b, h, i, t0 + 1);
        row_step(in, 0, t0);
    }
    tc::sync_block();

    // epilogue geometry, as in the forward
    const int eq = warp & 3;
    const int ek = 16 * eq + (lane & 15);
    const int en = 32 * (warp >> 2) + 16 * (lane >> 4);
    const uint32_t taddr = tmem + ((uint32_t)(32 * eq) << 16) + (uint32_t)(32 * (warp >> 2));

    // descriptors: K step ks starts 2048 bytes further on in each operand
    // (128 in the start-address field)
    const uint64_t dph = tc::sdesc(smem_u32(sm.Phi), 1024, 128), dpl = tc::sdesc(smem_u32(sm.Plo), 1024, 128);
    float mu = 0.0f;  // this thread's share of mu_{t0}[ek]: columns en .. en+15
    int p = 0;
    for (int64_t t = t0; t < t1; ++t) {
        const uint32_t par = (uint32_t)((t - t0) & 1);
        if (tid == 0 && !abort_flag) {
            // R_t = R_{t-1} A_t^T
            const uint64_t dah = tc::sdesc(smem_u32(sm.Ahi[p]), 1024, 128);
            const uint64_t dal = tc::sdesc(smem_u32(sm.Alo[p]), 1024, 128);
#pragma unroll
            for (int ks = 0; ks < DH / 8; ++ks) {
                const uint64_t ko = (uint64_t)ks * 128u;
                tc::mma(tmem, dph + ko, dal + ko, ks > 0 ? 1u : 0u);
                tc::mma(tmem, dpl + ko, dah + ko, 1u);
                tc::mma(tmem, dph + ko, dah + ko, 1u);
            }
            tc::commit(&sm.bar);
        }
        if (t + 1 < t1) {
            const BStepF in = nxt;
            if (t + 2 < t1) nxt = load_bstepf<DH, PxT>(pr, b, h, i, t + 2);
            row_step(in, p ^ 1, t + 1);
        }
        tc::wait_bar(pr, &sm.bar, par, abort_flag, lane);
        tc::fence_after();
        float v[16];
        tc::load_acc(taddr, v);
        {
            // this thread's share of R_t g_t
            const float4* gq = reinterpret_cast<const float4*>(sm.gv[p] + en);
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                const float4 gg = gq[g];
                mu = __fmaf_rn(v[4 * g + 0], gg.x, mu);
                mu = __fmaf_rn(v[4 * g + 1], gg.y, mu);
                mu = __fmaf_rn(v[4 * g + 2], gg.z, mu);
                mu = __fmaf_rn(v[4 * g + 3], gg.w, mu);
            }
        }
        // R_t into the left operand for the next step's products
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            float4 hv, lv;
            hv.x = tc::tf32_head(v[4 * g + 0]);
            hv.y = tc::tf32_head(v[4 * g + 1]);
            hv.z = tc::tf32_head(v[4 * g + 2]);
            hv.w = tc::tf32_head(v[4 * g + 3]);
            lv.x = v[4 * g + 0] - hv.x;
            lv.y = v[4 * g + 1] - hv.y;
            lv.z = v[4 * g + 2] - hv.z;
            lv.w = v[4 * g + 3] - hv.w;
            const int o = tc::a_idx(ek, en + 4 * g);
            *reinterpret_cast<float4*>(sm.Phi + o) = hv;
            *reinterpret_cast<float4*>(sm.Plo + o) = lv;
        }
        if (t + 1 == t1) {
            // R_{t1-1}: the chunk's product A_{t0}^T ... A_{t1-1}^T, row-major
            float* Pout = pr.P + task * DH * DH + (int64_t)ek * DH + en;
#pragma unroll
            for (int g = 0; g < 4; ++g)
                *reinterpret_cast<float4*>(Pout + 4 * g) = make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
        }
        tc::sync_block();
        p ^= 1;
    }
    // the four shares of row ek: lanes l and l + 16, then warps w and w + 4
    mu += __shfl_xor_sync(0xffffffffu, mu, 16);
    if (warp >= 4 && lane < 16) sm.red[ek] = mu;
    tc::fence_before();
    __syncthreads();
    if (warp < 4 && lane < 16) pr.q[task * DH + ek] = mu + sm.red[ek];
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(tc::kTmemColsB)
                     : "memory");
}

// ---- dL/dU: outer products summed in a fixed order -------------------------
// part[split][g][h] = sum over the split's rows (b, t) of e_g[b,t] h_{t-1}^T
// (e_z = dL/dp_z, e_r = dL/dp_r, e_c = lambda * gamma), rows in increasing
// (b, t) order; the reduce kernel sums the splits in order.  A block takes
// one split of the rows for one head and all three gates, so each row of
// h_{t-1} is loaded once for the three products; batches of kURows rows are
// double-buffered in shared memory with cp.async (16-byte copies when every
// source row is 16-byte aligned, else 4-byte ones), the next batch in flight
// while the current one is multiplied.
constexpr int kURows = 32;

template <int DH>
struct SmemU {
    float E[2][3][kURows][DH];  // e_z, e_r, e_c rows, two batches in turn
    float S[2][kURows][DH];     // h_{t-1} rows
};

template <int kBytes>
__device__ __forceinline__ void cp_async(void* dst, const void* src) {
    if constexpr (kBytes == 16)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
    else
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

template <int DH, int kVec>
__global__ void __launch_bounds__(kThreads, 2) head_dU_kernel(const Params pr, int64_t rows_per_split, float* part) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto& sm = *reinterpret_cast<SmemU<DH>*>(smem_raw);
    constexpr int TM = DH / 16;
    constexpr int QPR = DH / kVec;  // copies per row and array
    const int tid = threadIdx.x, i0 = (tid / 16) * TM, j0 = (tid % 16) * TM;
    const int split = blockIdx.x, h = blockIdx.y;
    const int64_t nrows = pr.B * pr.T;
    const int64_t r0 = split * rows_per_split;
    const int64_t r1 = r0 + rows_per_split < nrows ? r0 + rows_per_split : nrows;
    float acc[3][TM][TM];
#pragma unroll
    for (int g = 0; g < 3; ++g)
#pragma unroll
        for (int a = 0; a < TM; ++a)
#pragma unroll
            for (int c = 0; c < TM; ++c) acc[g][a][c] = 0.0f;

    // start the copies of rows rb .. rb + kURows - 1 into buffer `buf`
    auto issue = [&](int64_t rb, int buf) {
        for (int idx = tid; idx < kURows * 4 * QPR; idx += kThreads) {
            const int rr = idx / (4 * QPR), rem = idx - rr * (4 * QPR), arr = rem / QPR, q = rem - arr * QPR;
            const int64_t row = rb + rr;
            float* dst = arr < 3 ? &sm.E[buf][arr][rr][q * kVec] : &sm.S[buf][rr][q * kVec];
            const float* src = nullptr;
            if (row < r1) {
                const int64_t bb = row / pr.T, t = row - bb * pr.T, c = (int64_t)h * DH + q * kVec;
                if (arr < 2)
                    src = pr.dpx + ((bb * pr.T + t) * 3 + arr) * pr.D + c;
                else if (arr == 2)
                    src = pr.ec + (bb * pr.T + t) * pr.D + c;
                else
                    src = t >= 1 ? pr.Hold + (bb * pr.T + t - 1) * pr.D + c : (pr.h0 ? pr.h0 + bb * pr.D + c : nullptr);
            }
            if (src) {
                cp_async<kVec * 4>(dst, src);
            } else {
#pragma unroll
                for (int v = 0; v < kVec; ++v) dst[v] = 0.0f;
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    int buf = 0;
    if (r0 < r1) issue(r0, 0);
    for (int64_t rb = r0; rb < r1; rb += kURows, buf ^= 1) {
        if (rb + kURows < r1) {
            issue(rb + kURows, buf ^ 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
#pragma unroll 4
        for (int rr = 0; rr < kURows; ++rr) {
            float sw[TM];
#pragma unroll
            for (int c = 0; c < TM; ++c) sw[c] = sm.S[buf][rr][j0 + c];
#pragma unroll
            for (int g = 0; g < 3; ++g) {
                float ev[TM];
#pragma unroll
                for (int a = 0; a < TM; ++a) ev[a] = sm.E[buf][g][rr][i0 + a];
#pragma unroll
                for (int a = 0; a < TM; ++a)
#pragma unroll
                    for (int c = 0; c < TM; ++c) acc[g][a][c] = __fmaf_rn(ev[a], sw[c], acc[g][a][c]);
            }
        }
        __syncthreads();  // the buffer is refilled by the next batch's copies
    }
#pragma unroll
    for (int g = 0; g < 3; ++g) {
        float* out = part + ((int64_t)split * 3 * gridDim.y + (int64_t)g * gridDim.y + h) * DH * DH;
#pragma unroll
        for (int a = 0; a < TM; ++a)
#pragma unroll
            for (int c = 0; c < TM; ++c) out[(i0 + a) * DH + j0 + c] = acc[g][a][c];
    }
}

__global__ void head_dU_reduce_kernel(const float* part, int nsplit, int64_t n, float* dU) {
    const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= n) return;
    float acc = 0.0f;
    for (int sp = 0; sp < nsplit; ++sp) acc += part[sp * n + k];
    dU[k] = acc;
}

// ---- host side --------------------------------------------------------------

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Plan {
    int d = 0, nChunks = 0;
    int64_t nSeq = 0;
    size_t off_h = 0, off_P = 0, off_q = 0, off_c = 0, off_L = 0, total = 0;
};

// workspace: 256-byte header (status word) | second iterate buffer (K >= 2)
// | chunk products P | chunk deltas q | chunk carries | row factors
// (kNF per element; the backward's plan sizes kNB)
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
    pl.off_L = align256(pl.off_c + ntask * d * sizeof(float));
    pl.total = align256(pl.off_L + (size_t)B * T * D * kNF * sizeof(float));
    return true;
}

template <class Kern>
cudaError_t set_smem(Kern k, size_t bytes) {
    return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int DH, typename PxT>
cudaError_t launch_all(const Plan& pl, Params pr, float* H_out, float* Hbuf, int K, cudaStream_t st) {
    // head width 64: the products on tcgen05; narrower heads (tcgen05.mma
    // has no M below 64) on mma.sync
    constexpr bool kTc = DH == tc::kD;
    const size_t smemA = kTc ? sizeof(tc::Smem) : sizeof(SmemA<DH>), smemR = sizeof(SmemA<DH>);
    cudaError_t e;
    if constexpr (kTc)
        e = set_smem(head_chunk_tc_kernel<PxT>, smemA);
    else
        e = set_smem(head_chunk_kernel<DH, PxT, false>, smemA);
    if (e == cudaSuccess) e = set_smem(head_chunk_kernel<DH, PxT, true>, smemR);
    if (e != cudaSuccess) return e;
    const unsigned ntask = (unsigned)(pl.nSeq * pl.nChunks);
    for (int k = 0; k < K; ++k) {
        // iterate k lives in X_k, X_j = H_out when K - j is even, else the
        // workspace buffer, so that h^(K) lands in H_out
        pr.k = k;
        pr.Hold = k == 0 ? nullptr : (((K - k) % 2 == 0) ? H_out : Hbuf);
        pr.Hnew = ((K - (k + 1)) % 2 == 0) ? H_out : Hbuf;
        if constexpr (kTc)
            head_chunk_tc_kernel<PxT><<<ntask, kThreads, smemA, st>>>(pr);
        else
            head_chunk_kernel<DH, PxT, false><<<ntask, kThreads, smemA, st>>>(pr);
        head_carry_kernel<DH><<<(unsigned)pl.nSeq, 64, 0, st>>>(pr);
        head_walk_kernel<DH><<<ntask, kThreads, 0, st>>>(pr);
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

struct BPlan {
    int d = 0, nChunks = 0, nsplit = 0;
    int64_t nSeq = 0, rows_per_split = 0;
    size_t off_P = 0, off_q = 0, off_c = 0, off_ec = 0, off_L = 0, off_part = 0, total = 0;
};

// backward workspace: 256-byte header (status word) | chunk products Q |
// chunk mus q | chunk carries | lambda * gamma (B,T,D) | row factors (kNB
// per element) | dL/dU split partials
bool make_bplan(int64_t B, int64_t T, int64_t D, int nh, BPlan& pl) {
    Plan fp;
    if (!make_plan(B, T, D, nh, 1, fp)) return false;
    pl.d = fp.d;
    pl.nChunks = fp.nChunks;
    pl.nSeq = fp.nSeq;
    const size_t ntask = (size_t)pl.nSeq * pl.nChunks, d = pl.d;
    const int64_t rows = B * T;
    // splits of at least 256 rows, at most 64, and about one wave of
    // blocks (two per SM on the 148 SMs) over the heads
    pl.nsplit = (int)(rows > 0 ? (rows + 255) / 256 : 1);
    if (pl.nsplit > 64) pl.nsplit = 64;
    const int wave = nh < 296 ? 296 / nh : 1;
    if (pl.nsplit > wave) pl.nsplit = wave;
    pl.rows_per_split = rows > 0 ? (rows + pl.nsplit - 1) / pl.nsplit : 1;
    pl.off_P = 256;
    pl.off_q = align256(pl.off_P + ntask * d * d * sizeof(float));
    pl.off_c = align256(pl.off_q + ntask * d * sizeof(float));
    pl.off_ec = align256(pl.off_c + ntask * d * sizeof(float));
    pl.off_L = align256(pl.off_ec + (size_t)B * T * D * sizeof(float));
    pl.off_part = align256(pl.off_L + (size_t)B * T * D * kNB * sizeof(float));
    pl.total = align256(pl.off_part + (size_t)pl.nsplit * 3 * nh * d * d * sizeof(float));
    return true;
}

template <int DH, typename PxT>
cudaError_t launch_bwd(const BPlan& pl, const Params& pr, float* dU, cudaStream_t st) {
    // head width 64: the products on tcgen05, as in the forward
    constexpr bool kTc = DH == tc::kD;
    const size_t smemP = kTc ? sizeof(tc::SmemB) : sizeof(SmemB<DH>);
    cudaError_t e;
    if constexpr (kTc)
        e = set_smem(head_bwd_tc_kernel<PxT>, smemP);
    else
        e = set_smem(head_bwd_kernel<DH, PxT>, smemP);
    if (e != cudaSuccess) return e;
    const unsigned ntask = (unsigned)(pl.nSeq * pl.nChunks);
    if constexpr (kTc)
        head_bwd_tc_kernel<PxT><<<ntask, kThreads, smemP, st>>>(pr);
    else
        head_bwd_kernel<DH, PxT><<<ntask, kThreads, smemP, st>>>(pr);
    head_carry_kernel<DH, true><<<(unsigned)pl.nSeq, 64, 0, st>>>(pr);
    head_bwd_walk_kernel<DH><<<ntask, kThreads, 0, st>>>(pr);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (dU) {
        float* part = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(pr.status) + pl.off_part);
        // 16-byte copies need every source row 16-byte aligned: the
        // workspace's lambda * gamma always is, dL/dpx, H and h0 are checked
        const bool vec = ((reinterpret_cast<uintptr_t>(pr.dpx) | reinterpret_cast<uintptr_t>(pr.Hold) |
                           reinterpret_cast<uintptr_t>(pr.h0)) & 15) == 0;
        const size_t smemU = sizeof(SmemU<DH>);
        const dim3 grid((unsigned)pl.nsplit, (unsigned)pr.nh);
        if (vec) {
            if ((e = set_smem(head_dU_kernel<DH, 4>, smemU)) != cudaSuccess) return e;
            head_dU_kernel<DH, 4><<<grid, kThreads, smemU, st>>>(pr, pl.rows_per_split, part);
        } else {
            if ((e = set_smem(head_dU_kernel<DH, 1>, smemU)) != cudaSuccess) return e;
            head_dU_kernel<DH, 1><<<grid, kThreads, smemU, st>>>(pr, pl.rows_per_split, part);
        }
        const int64_t n = (int64_t)3 * pr.nh * DH * DH;
        head_dU_reduce_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(part, pl.nsplit, n, dU);
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
    memset(&pr, 0, sizeof pr);
    pr.px = preacts;
    pr.U = U;
    pr.h0 = h0;
    pr.Hold = nullptr;
    pr.Hnew = H_out;
    pr.P = reinterpret_cast<float*>(ws + pl.off_P);
    pr.q = reinterpret_cast<float*>(ws + pl.off_q);
    pr.carry = reinterpret_cast<float*>(ws + pl.off_c);
    pr.L = reinterpret_cast<float*>(ws + pl.off_L);
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

extern "C" size_t pararnn_head_gru_backward_workspace_bytes(int64_t B, int64_t T, int64_t D, int n_heads) {
    hg::BPlan pl;
    if (!hg::make_bplan(B, T, D, n_heads, pl)) return 0;
    return pl.total;
}

extern "C" pararnn_status pararnn_head_gru_backward(int64_t B, int64_t T, int64_t D, int n_heads,
                                                    pararnn_dtype px_dtype, const void* preacts, const float* U,
                                                    const float* h0, const float* H, const float* dL_dH,
                                                    float* dL_dpx, float* dL_dU, float* dL_dh0, void* workspace,
                                                    size_t ws_bytes, void* stream) {
    hg::BPlan pl;
    if (!hg::make_bplan(B, T, D, n_heads, pl))
        return hg::fail(PARARNN_EINVAL,
                        "pararnn_head_gru_backward: need B, T, D >= 0, D = n_heads * d with d in {16, 32, 64}, "
                        "and B*T below 2^31");
    if (px_dtype != PARARNN_F32 && px_dtype != PARARNN_BF16)
        return hg::fail(PARARNN_EINVAL, "pararnn_head_gru_backward: unknown pre-activation dtype");
    if (!workspace || ws_bytes < pl.total)
        return hg::fail(PARARNN_EINVAL, "pararnn_head_gru_backward: workspace missing or smaller than "
                                        "pararnn_head_gru_backward_workspace_bytes()");
    if (!pointer_on_device(workspace) || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return hg::fail(PARARNN_EINVAL, "pararnn_head_gru_backward: workspace must be 256-byte aligned device memory");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    cudaError_t e = cudaMemsetAsync(ws, 0, 256, st);
    if (e != cudaSuccess) return hg::fail(PARARNN_ECUDA, "pararnn_head_gru_backward: header reset failed");
    const int d = pl.d;
    if (B == 0 || T == 0 || D == 0) {
        // nothing flows back: dL/dU (and dL/dh0) are zero
        if (dL_dU && pointer_on_device(dL_dU)) cudaMemsetAsync(dL_dU, 0, sizeof(float) * 3 * n_heads * d * d, st);
        if (dL_dh0 && pointer_on_device(dL_dh0)) cudaMemsetAsync(dL_dh0, 0, sizeof(float) * B * D, st);
        return PARARNN_OK;
    }
    const size_t esz = px_dtype == PARARNN_BF16 ? 2 : 4;
    const void* need[] = {preacts, U, H, dL_dH, dL_dpx};
    for (const void* q : need)
        if (!q || !pointer_on_device(q))
            return hg::fail(PARARNN_EINVAL, "pararnn_head_gru_backward: a required pointer is null or not device memory");
    const void* opt[] = {h0, dL_dU, dL_dh0};
    for (const void* q : opt)
        if (q && (!pointer_on_device(q) || (reinterpret_cast<uintptr_t>(q) & 3)))
            return hg::fail(PARARNN_EINVAL, "pararnn_head_gru_backward: h0, dL_dU or dL_dh0 is not aligned device memory");
    if ((reinterpret_cast<uintptr_t>(preacts) % esz) || (reinterpret_cast<uintptr_t>(U) & 3) ||
        (reinterpret_cast<uintptr_t>(H) & 3) || (reinterpret_cast<uintptr_t>(dL_dH) & 3) ||
        (reinterpret_cast<uintptr_t>(dL_dpx) & 3))
        return hg::fail(PARARNN_EINVAL, "pararnn_head_gru_backward: misaligned pointer");
    hg::Params pr;
    memset(&pr, 0, sizeof pr);
    pr.px = preacts;
    pr.U = U;
    pr.h0 = h0;
    pr.Hold = H;
    pr.G = dL_dH;
    pr.dpx = dL_dpx;
    pr.dh0 = dL_dh0;
    pr.P = reinterpret_cast<float*>(ws + pl.off_P);
    pr.q = reinterpret_cast<float*>(ws + pl.off_q);
    pr.carry = reinterpret_cast<float*>(ws + pl.off_c);
    pr.ec = reinterpret_cast<float*>(ws + pl.off_ec);
    pr.L = reinterpret_cast<float*>(ws + pl.off_L);
    pr.status = reinterpret_cast<unsigned*>(ws);
    pr.B = B;
    pr.T = T;
    pr.D = D;
    pr.nh = n_heads;
    pr.nChunks = pl.nChunks;
    const bool bf = px_dtype == PARARNN_BF16;
    switch (d) {
        case 16: e = bf ? hg::launch_bwd<16, __nv_bfloat16>(pl, pr, dL_dU, st) : hg::launch_bwd<16, float>(pl, pr, dL_dU, st); break;
        case 32: e = bf ? hg::launch_bwd<32, __nv_bfloat16>(pl, pr, dL_dU, st) : hg::launch_bwd<32, float>(pl, pr, dL_dU, st); break;
        default: e = bf ? hg::launch_bwd<64, __nv_bfloat16>(pl, pr, dL_dU, st) : hg::launch_bwd<64, float>(pl, pr, dL_dU, st); break;
    }
    if (e != cudaSuccess) {
        cudaGetLastError();
        return hg::fail(PARARNN_ECUDA, "pararnn_head_gru_backward: kernel launch failed");
    }
    return PARARNN_OK;
}
