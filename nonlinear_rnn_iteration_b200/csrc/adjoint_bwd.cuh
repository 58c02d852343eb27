// adjoint_bwd.cuh -- the backward pass: a reverse-time scan for the adjoint
// state and the gradient epilogue, fused in one kernel, plus a fixed-order
// reduction of the per-tile weight-gradient partials.
//
// At the trajectory H (the forward's output), with g_t = dL/dH_t:
//     lambda_t = g_t + A_{t+1}^T lambda_{t+1},   lambda_{T-1} = g_{T-1},
//     A_{t+1} = df/dh at (h_t, x_{t+1}),
// which is the scan of the elements (M_t, g_t), M_t = A_{t+1}^T, in reverse
// time under the same operator as the forward (pararnn-torch PyPI page,
// Method section: the backward follows the paper's adjoint; this is the plain
// adjoint of the lower-bidiagonal system F(H) = 0).  Then
//     dL/dp_g[t]  = lambda_t . df/dp_g   at (h_{t-1}, x_t)
//     dL/da_g     = sum_{b,t} lambda_t . df/da_g
//     dL/dh0      = A_0^T lambda_0.
// dL/da is summed within a tile in a fixed order, written per tile, and
// reduced over tiles in a fixed order by a second kernel: no floating-point
// atomics, so the result does not depend on scheduling (Compatibility
// section: the packed VJP is deterministic).
#pragma once

#include "cells.cuh"
#include "common.cuh"
#include "lookback.cuh"

namespace pararnn {

struct BwdParams {
    const void* px;     // (B,T,G,D)
    const float* w;     // (G,D) or null
    const float* h0;    // (B,S,D) or null
    const float* H;     // (B,T,S,D)
    const float* dLdH;  // (B,T,S,D)
    float* dLdpx;       // (B,T,G,D)
    float* dLdh0;       // (B,S,D) or null
    float* part;        // per-tile dL/da partials [nTiles][G][W]
    int64_t B, T, D;
    int64_t nCG, nChunks;
    LookbackCtx lb;     // nSlots = 1
};

template <class Cell, typename PxT, class Sh>
__global__ void __launch_bounds__(Sh::NT) adjoint_bwd_kernel(const BwdParams prm) {
    constexpr int G = Sh::G, S = Sh::S, NA = Sh::NA, V = Sh::V, R = Sh::R, NS = Cell::NSENS;
    constexpr int TPW = Sh::TPW, NSUB = Sh::NSUB, W = Sh::W, L = Sh::L, LC = Sh::LC, NT = Sh::NT;
    constexpr int CPL = W / 32;
    static_assert(G * W <= NT, "one thread per (gate, channel) in the partial reduction");

    __shared__ float s_agg[NSUB][NA][W];    // indexed by position in the reverse scan
    __shared__ float s_carry[NSUB][S][W];
    __shared__ float s_edge[NSUB][S][W];    // each sub-chunk's last state h
    __shared__ float s_firstA[NSUB][S * S][W];  // each sub-chunk's first-row Jacobian
    __shared__ float s_da[NSUB][G][W];
    __shared__ unsigned s_ticket;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sub = warp * TPW + lane / LC;
    const int rs = NSUB - 1 - sub;  // this sub-chunk's position in the reverse scan
    const int cc = (lane % LC) * V;

    if (tid == 0) s_ticket = atomicAdd(prm.lb.status + 1, 1u);
    __syncthreads();
    const int64_t tile = s_ticket;
    const int64_t pos = tile / prm.lb.nGroups;
    const int64_t gid = tile - pos * prm.lb.nGroups;
    const int64_t chunk = prm.nChunks - 1 - pos;
    const int64_t b = gid / prm.nCG;
    const int64_t d0 = (gid - b * prm.nCG) * W;
    const int64_t t0 = chunk * L;
    const int64_t tb = t0 + (int64_t)sub * R;
    const int64_t T = prm.T, D = prm.D;
    const bool cvalid = d0 + cc < D;
    const PxT* px = static_cast<const PxT*>(prm.px);

    float w[V][G];
#pragma unroll
    for (int v = 0; v < V; ++v)
#pragma unroll
        for (int g = 0; g < G; ++g) w[v][g] = (prm.w && cvalid) ? __ldg(prm.w + g * D + d0 + cc + v) : 0.0f;

    // ---- loads: pre-activations, states, upstream gradients ----
    float p[R][G][V], hs[R][S][V], gr[R][S][V];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int64_t t = tb + r;
        const bool ok = t < T && cvalid;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            if (ok) load_row<V>(px + ((b * T + t) * G + g) * D + d0 + cc, p[r][g]);
            else
#pragma unroll
                for (int v = 0; v < V; ++v) p[r][g][v] = 0.0f;
        }
#pragma unroll
        for (int s = 0; s < S; ++s) {
            if (ok) {
                load_row<V>(prm.H + ((b * T + t) * S + s) * D + d0 + cc, hs[r][s]);
                load_row<V>(prm.dLdH + ((b * T + t) * S + s) * D + d0 + cc, gr[r][s]);
            } else {
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    hs[r][s][v] = 0.0f;
                    gr[r][s][v] = 0.0f;
                }
            }
        }
    }
#pragma unroll
    for (int s = 0; s < S; ++s)
#pragma unroll
        for (int v = 0; v < V; ++v) s_edge[sub][s][cc + v] = hs[R - 1][s][v];
    __syncthreads();

    // ---- linearisation at (h_{t-1}, x_t) for every row ----
    float sp[S][V];
#pragma unroll
    for (int v = 0; v < V; ++v)
#pragma unroll
        for (int s = 0; s < S; ++s) {
            float x = 0.0f;
            if (sub > 0) x = s_edge[sub - 1][s][cc + v];
            else if (cvalid && t0 > 0) x = prm.H[((b * T + t0 - 1) * S + s) * D + d0 + cc + v];
            else if (cvalid && prm.h0) x = prm.h0[(b * S + s) * D + d0 + cc + v];
            sp[s][v] = x;
        }
    float jA[R][S * S][V], sens[R][NS][V];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int v = 0; v < V; ++v) {
            float pv[G], wv[G], spv[S], A[S * S], se[NS];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                pv[g] = p[r][g][v];
                wv[g] = w[v][g];
            }
#pragma unroll
            for (int s = 0; s < S; ++s) spv[s] = sp[s][v];
            Cell::bwd(pv, wv, spv, A, se);
#pragma unroll
            for (int a = 0; a < S * S; ++a) jA[r][a][v] = A[a];
#pragma unroll
            for (int n = 0; n < NS; ++n) sens[r][n][v] = se[n];
#pragma unroll
            for (int s = 0; s < S; ++s) sp[s][v] = hs[r][s][v];
        }
#pragma unroll
    for (int a = 0; a < S * S; ++a)
#pragma unroll
        for (int v = 0; v < V; ++v) s_firstA[sub][a][cc + v] = jA[0][a][v];

    // the last sub-chunk also needs A at the first row of the next tile
    float nextA[S * S][V];
    if (sub == NSUB - 1) {
        const int64_t tn = t0 + L;
#pragma unroll
        for (int v = 0; v < V; ++v) {
            float A[S * S];
#pragma unroll
            for (int a = 0; a < S * S; ++a) A[a] = 0.0f;
            if (tn < T && cvalid) {
                float pv[G], wv[G], spv[S], se[NS];
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    pv[g] = PxTraits<PxT>::cvt(px[((b * T + tn) * G + g) * D + d0 + cc + v]);
                    wv[g] = w[v][g];
                }
#pragma unroll
                for (int s = 0; s < S; ++s) spv[s] = hs[R - 1][s][v];
                Cell::bwd(pv, wv, spv, A, se);
            }
#pragma unroll
            for (int a = 0; a < S * S; ++a) nextA[a][v] = A[a];
        }
    }
    __syncthreads();

    // ---- reverse-scan elements (M_t, g_t), M_t = A_{t+1}^T ----
    float eM[R][S * S][V];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int v = 0; v < V; ++v) {
            const int64_t t = tb + r;
            float A[S * S];
#pragma unroll
            for (int a = 0; a < S * S; ++a) {
                if (r + 1 < R) A[a] = jA[r + 1][a][v];
                else if (sub + 1 < NSUB) A[a] = s_firstA[sub + 1][a][cc + v];
                else A[a] = nextA[a][v];
            }
            const bool has_next = (t + 1 < T) && cvalid;
            const bool rvalid = (t < T) && cvalid;
#pragma unroll
            for (int i = 0; i < S; ++i)
#pragma unroll
                for (int m = 0; m < S; ++m) {
                    float val = has_next ? A[m * S + i] : 0.0f;  // transpose
                    if (!rvalid) val = (i == m) ? 1.0f : 0.0f;     // past the end: identity
                    eM[r][i * S + m][v] = val;
                }
        }
#pragma unroll
    for (int v = 0; v < V; ++v) {
        Elem<S> acc;
        elem_identity<S>(acc);
#pragma unroll
        for (int r = R - 1; r >= 0; --r) {
            float M[S * S], g[S];
#pragma unroll
            for (int a = 0; a < S * S; ++a) M[a] = eM[r][a][v];
#pragma unroll
            for (int s = 0; s < S; ++s) g[s] = gr[r][s][v];
            compose_after<S>(M, g, acc);
        }
#pragma unroll
        for (int a = 0; a < S * S; ++a) s_agg[rs][a][cc + v] = acc.A[a];
#pragma unroll
        for (int s = 0; s < S; ++s) s_agg[rs][S * S + s][cc + v] = acc.b[s];
    }
    __syncthreads();

    if (warp == 0) {
        float zero[CPL][S], carry[CPL][S];
#pragma unroll
        for (int j = 0; j < CPL; ++j)
#pragma unroll
            for (int s = 0; s < S; ++s) zero[j][s] = 0.0f;  // lambda_T = 0
        tile_scan_step<S, W, NSUB>(prm.lb, tile, pos, 0, lane, s_agg, s_carry, zero, carry);
    }
    __syncthreads();

    // ---- lambda and the gradient epilogue ----
    float da_acc[G][V];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int v = 0; v < V; ++v) da_acc[g][v] = 0.0f;
    bool bad = false;
#pragma unroll
    for (int v = 0; v < V; ++v) {
        float x[S];
#pragma unroll
        for (int s = 0; s < S; ++s) x[s] = s_carry[rs][s][cc + v];
#pragma unroll
        for (int r = R - 1; r >= 0; --r) {
            float M[S * S], g[S], y[S];
#pragma unroll
            for (int a = 0; a < S * S; ++a) M[a] = eM[r][a][v];
#pragma unroll
            for (int s = 0; s < S; ++s) g[s] = gr[r][s][v];
            apply<S>(M, g, x, y);
#pragma unroll
            for (int s = 0; s < S; ++s) x[s] = y[s];
            float se[NS], dp[G], da[G];
#pragma unroll
            for (int n = 0; n < NS; ++n) se[n] = sens[r][n][v];
            Cell::grads(se, x, dp, da);
            const bool rvalid = (tb + r < T) && cvalid;
            if (rvalid) {
#pragma unroll
                for (int g2 = 0; g2 < G; ++g2) {
                    p[r][g2][v] = dp[g2];  // reuse the pre-activation registers for the output row
                    da_acc[g2][v] += da[g2];
                    bad |= !isfinite(dp[g2]);
                }
            }
            if (r == 0 && tb == 0 && rvalid && prm.dLdh0) {
                // dL/dh0 = A_0^T lambda_0, A_0 at (h0, x_0)
#pragma unroll
                for (int i = 0; i < S; ++i) {
                    float acc = 0.0f;
#pragma unroll
                    for (int m = 0; m < S; ++m) acc = __fmaf_rn(jA[0][m * S + i][v], x[m], acc);
                    prm.dLdh0[(b * S + i) * D + d0 + cc + v] = acc;
                }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int64_t t = tb + r;
        if (t < T && cvalid) {
#pragma unroll
            for (int g = 0; g < G; ++g) store_row<V>(prm.dLdpx + ((b * T + t) * G + g) * D + d0 + cc, p[r][g]);
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(prm.lb.status, kStatusNonFinite);

    // ---- per-tile dL/da partial, summed over sub-chunks in a fixed order ----
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int v = 0; v < V; ++v) s_da[sub][g][cc + v] = da_acc[g][v];
    __syncthreads();
    if (tid < G * W) {
        const int g = tid / W, ch = tid - (tid / W) * W;
        float acc = 0.0f;
#pragma unroll 4
        for (int sb = 0; sb < NSUB; ++sb) acc += s_da[sb][g][ch];
        prm.part[(tile * G + g) * W + ch] = acc;
    }
}

// dL/da[g][d] = sum over batch rows b, then over tiles along time, of the
// per-tile partials: one thread per (g, d), a fixed summation order.
struct ReduceParams {
    const float* part;
    float* dLda;
    int64_t B, D, nCG, nChunks, nGroups;
    int G, W;
};

__global__ void reduce_da_kernel(const ReduceParams prm) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)prm.G * prm.D) return;
    const int g = (int)(i / prm.D);
    const int64_t d = i - (int64_t)g * prm.D;
    const int64_t cg = d / prm.W, ch = d - cg * prm.W;
    float acc = 0.0f;
    for (int64_t b = 0; b < prm.B; ++b) {
        const int64_t gid = b * prm.nCG + cg;
        for (int64_t pos = 0; pos < prm.nChunks; ++pos) {
            const int64_t tile = pos * prm.nGroups + gid;
            acc += prm.part[(tile * prm.G + g) * prm.W + ch];
        }
    }
    prm.dLda[g * prm.D + d] = acc;
}

}  // namespace pararnn
