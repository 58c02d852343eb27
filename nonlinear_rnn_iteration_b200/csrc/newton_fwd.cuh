// newton_fwd.cuh -- the fused Newton forward: every Newton iteration of a
// tile in one thread block, with the tile's pre-activations and iterate kept
// in registers from the first iteration to the last.
//
// Method (pararnn-torch PyPI page, Method section): solve F(H) = 0,
// F_t = h_t - f(h_{t-1}, x_t), by K Newton iterations from the warm start
// h^(0)_t = f(0, x_t), each linear solve an associative scan over time.  The
// scan here is on the direct-form elements
//     h^(k+1)_t = A_t h^(k+1)_{t-1} + beta_t,
//     A_t = df/dh at (h^(k)_{t-1}, x_t),  beta_t = f(h^(k)_{t-1}, x_t) - A_t h^(k)_{t-1}.
//
// Tile = W channels x L time steps of one batch row.  Thread (lc, sub) holds
// V consecutive channels of R consecutive time steps; NSUB sub-chunks tile
// the L steps.  Per Newton iteration:
//   1. every thread evaluates f, A_t, beta_t on its R rows (the previous
//      row's state comes from its neighbour through shared memory) and
//      composes them into one element;
//   2. warp 0 composes the NSUB elements in time order, publishes the tile's
//      element, finds the carry by decoupled look-back over earlier tiles
//      of the same channels, publishes the state after the tile, and hands
//      each sub-chunk its carry-in;
//   3. every thread re-walks its R rows from its carry-in, giving h^(k+1).
// Iteration k+1 needs h^(k)_{t0-1} just before the tile: that is the carry
// found in iteration k, so no extra wait is needed.  Only the
// pre-activations are read from HBM (once) and only h^(K) is written (once).
#pragma once

#include "cells.cuh"
#include "common.cuh"
#include "lookback.cuh"

namespace pararnn {

struct FwdParams {
    const void* px;      // (B,T,G,D) f32 or bf16
    const float* w;      // (G,D) or null
    const float* h0;     // (B,S,D) or null
    float* H;            // (B,T,S,D)
    float* resid;        // K+1 floats or null
    int64_t B, T, D;
    int K;
    int64_t nCG;         // channel groups per batch row
    int64_t nChunks;     // tiles along T
    LookbackCtx lb;      // nGroups = B * nCG, nSlots = K
};

template <class Cell, int V_, int LC_, int NWARPS_, int R_>
struct FwdShape {
    static constexpr int V = V_, LC = LC_, NWARPS = NWARPS_, R = R_;
    static constexpr int G = Cell::G, S = Cell::S, NA = S * S + S;
    static constexpr int TPW = 32 / LC;           // sub-chunks per warp
    static constexpr int NSUB = NWARPS * TPW;     // sub-chunks per tile
    static constexpr int W = LC * V;              // channels per tile
    static constexpr int L = NSUB * R;            // time steps per tile
    static constexpr int NT = NWARPS * 32;
    static_assert(32 % LC == 0 && W % 32 == 0, "tile width must be a multiple of 32 channels");
};

template <class Cell, typename PxT, class Sh>
__global__ void __launch_bounds__(Sh::NT) newton_fwd_kernel(const FwdParams prm) {
    constexpr int G = Sh::G, S = Sh::S, NA = Sh::NA, V = Sh::V, R = Sh::R;
    constexpr int TPW = Sh::TPW, NSUB = Sh::NSUB, W = Sh::W, L = Sh::L, LC = Sh::LC;
    constexpr int CPL = W / 32;

    __shared__ float s_agg[NSUB][NA][W];   // each sub-chunk's composed element
    __shared__ float s_edge[NSUB][S][W];   // each sub-chunk's last state (current iterate)
    __shared__ float s_carry[NSUB][S][W];  // each sub-chunk's carry-in
    __shared__ float s_prev[S][W];         // current iterate just before the tile
    __shared__ unsigned s_ticket;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sub = warp * TPW + lane / LC;
    const int cc = (lane % LC) * V;

    if (tid == 0) s_ticket = atomicAdd(prm.lb.status + 1, 1u);
    __syncthreads();
    const int64_t tile = s_ticket;
    const int64_t chunk = tile / prm.lb.nGroups;
    const int64_t gid = tile - chunk * prm.lb.nGroups;
    const int64_t b = gid / prm.nCG;
    const int64_t d0 = (gid - b * prm.nCG) * W;
    const int64_t t0 = chunk * L;
    const int64_t tb = t0 + (int64_t)sub * R;
    const int64_t T = prm.T, D = prm.D;
    const bool cvalid = d0 + cc < D;  // D is a multiple of V: a vector is wholly in or out
    const bool need_prev = Cell::kNonlinear || prm.resid != nullptr;
    const PxT* px = static_cast<const PxT*>(prm.px);

    float w[V][G];
#pragma unroll
    for (int v = 0; v < V; ++v)
#pragma unroll
        for (int g = 0; g < G; ++g) w[v][g] = (prm.w && cvalid) ? __ldg(prm.w + g * D + d0 + cc + v) : 0.0f;

    // ---- load the tile's pre-activations (the only HBM reads) ----
    float p[R][G][V];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int64_t t = tb + r;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            if (t < T && cvalid) {
                load_row<V>(px + ((b * T + t) * G + g) * D + d0 + cc, p[r][g]);
            } else {
#pragma unroll
                for (int v = 0; v < V; ++v) p[r][g][v] = 0.0f;
            }
        }
    }

    // ---- warm start h^(0)_t = f(0, x_t) ----
    float h[R][S][V];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
        for (int v = 0; v < V; ++v) {
            float pv[G], wv[G], f[S];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                pv[g] = p[r][g][v];
                wv[g] = w[v][g];
            }
            Cell::warm(pv, wv, f);
#pragma unroll
            for (int s = 0; s < S; ++s) h[r][s][v] = f[s];
        }

    // carry into the sequence: h_{-1} = h0 for every iterate
    float first_carry[CPL][S];
    if (warp == 0) {
#pragma unroll
        for (int j = 0; j < CPL; ++j)
#pragma unroll
            for (int s = 0; s < S; ++s) {
                const int64_t d = d0 + lane + 32 * j;
                first_carry[j][s] = (prm.h0 && d < D) ? prm.h0[(b * S + s) * D + d] : 0.0f;
            }
    }
    if (need_prev) {
        // h^(0) just before the tile: h0 for the first tile, else the warm
        // start of the row before
        if (sub == 0) {
#pragma unroll
            for (int v = 0; v < V; ++v) {
                float f[S] = {};
                const int64_t d = d0 + cc + v;
                if (cvalid) {
                    if (t0 == 0) {
#pragma unroll
                        for (int s = 0; s < S; ++s) f[s] = prm.h0 ? prm.h0[(b * S + s) * D + d] : 0.0f;
                    } else {
                        float pv[G], wv[G];
#pragma unroll
                        for (int g = 0; g < G; ++g) {
                            pv[g] = PxTraits<PxT>::cvt(px[((b * T + t0 - 1) * G + g) * D + d]);
                            wv[g] = w[v][g];
                        }
                        Cell::warm(pv, wv, f);
                    }
                }
#pragma unroll
                for (int s = 0; s < S; ++s) s_prev[s][cc + v] = f[s];
            }
        }
#pragma unroll
        for (int s = 0; s < S; ++s)
#pragma unroll
            for (int v = 0; v < V; ++v) s_edge[sub][s][cc + v] = h[R - 1][s][v];
    }

    const int K = prm.K;
    for (int k = 0; k < K; ++k) {
        __syncthreads();
        // ---- 1. elements of this iteration, and the residual of iterate k ----
        float sp[S][V];
        if (need_prev) {
#pragma unroll
            for (int s = 0; s < S; ++s)
#pragma unroll
                for (int v = 0; v < V; ++v) sp[s][v] = sub == 0 ? s_prev[s][cc + v] : s_edge[sub - 1][s][cc + v];
        } else {
#pragma unroll
            for (int s = 0; s < S; ++s)
#pragma unroll
                for (int v = 0; v < V; ++v) sp[s][v] = 0.0f;
        }
        float eA[R][S * S][V], eb[R][S][V];
        float res = 0.0f;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const bool rvalid = (tb + r < T) && cvalid;
#pragma unroll
            for (int v = 0; v < V; ++v) {
                float pv[G], wv[G], spv[S], f[S], A[S * S], be[S];
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    pv[g] = p[r][g][v];
                    wv[g] = w[v][g];
                }
#pragma unroll
                for (int s = 0; s < S; ++s) spv[s] = sp[s][v];
                Cell::elem(pv, wv, spv, f, A, be);
                if (rvalid) {
#pragma unroll
                    for (int s = 0; s < S; ++s) res = nanmax_f(res, fabsf(h[r][s][v] - f[s]));
                } else {
#pragma unroll
                    for (int a = 0; a < S * S; ++a) A[a] = (a % (S + 1) == 0) ? 1.0f : 0.0f;
#pragma unroll
                    for (int s = 0; s < S; ++s) be[s] = 0.0f;
                }
#pragma unroll
                for (int a = 0; a < S * S; ++a) eA[r][a][v] = A[a];
#pragma unroll
                for (int s = 0; s < S; ++s) {
                    eb[r][s][v] = be[s];
                    sp[s][v] = h[r][s][v];
                }
            }
        }
        // compose the R rows in time order
#pragma unroll
        for (int v = 0; v < V; ++v) {
            Elem<S> acc;
            elem_identity<S>(acc);
#pragma unroll
            for (int r = 0; r < R; ++r) {
                float A[S * S], be[S];
#pragma unroll
                for (int a = 0; a < S * S; ++a) A[a] = eA[r][a][v];
#pragma unroll
                for (int s = 0; s < S; ++s) be[s] = eb[r][s][v];
                compose_after<S>(A, be, acc);
            }
#pragma unroll
            for (int a = 0; a < S * S; ++a) s_agg[sub][a][cc + v] = acc.A[a];
#pragma unroll
            for (int s = 0; s < S; ++s) s_agg[sub][S * S + s][cc + v] = acc.b[s];
        }
        if (prm.resid) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) res = nanmax_f(res, __shfl_xor_sync(0xffffffffu, res, o));
            if (lane == 0) atomic_max_nonneg(prm.resid + k, res);
        }
        __syncthreads();

        // ---- 2. tile composition, look-back, carries (warp 0) ----
        if (warp == 0) {
            float carry[CPL][S];
            tile_scan_step<S, W, NSUB>(prm.lb, tile, chunk, k, lane, s_agg, s_carry, first_carry, carry);
#pragma unroll
            for (int j = 0; j < CPL; ++j)
#pragma unroll
                for (int s = 0; s < S; ++s) s_prev[s][lane + 32 * j] = carry[j][s];
        }
        __syncthreads();

        // ---- 3. re-walk the rows from the carry-in: h^(k+1) ----
#pragma unroll
        for (int v = 0; v < V; ++v) {
            float x[S];
#pragma unroll
            for (int s = 0; s < S; ++s) x[s] = s_carry[sub][s][cc + v];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                float A[S * S], be[S], y[S];
#pragma unroll
                for (int a = 0; a < S * S; ++a) A[a] = eA[r][a][v];
#pragma unroll
                for (int s = 0; s < S; ++s) be[s] = eb[r][s][v];
                apply<S>(A, be, x, y);
#pragma unroll
                for (int s = 0; s < S; ++s) {
                    x[s] = y[s];
                    h[r][s][v] = y[s];
                }
            }
        }
        if (need_prev) {
#pragma unroll
            for (int s = 0; s < S; ++s)
#pragma unroll
                for (int v = 0; v < V; ++v) s_edge[sub][s][cc + v] = h[R - 1][s][v];
        }
    }

    // ---- residual of the final iterate ----
    if (prm.resid) {
        __syncthreads();
        float sp[S][V];
#pragma unroll
        for (int s = 0; s < S; ++s)
#pragma unroll
            for (int v = 0; v < V; ++v) sp[s][v] = sub == 0 ? s_prev[s][cc + v] : s_edge[sub - 1][s][cc + v];
        float res = 0.0f;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const bool rvalid = (tb + r < T) && cvalid;
#pragma unroll
            for (int v = 0; v < V; ++v) {
                float pv[G], wv[G], spv[S], f[S], A[S * S], be[S];
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    pv[g] = p[r][g][v];
                    wv[g] = w[v][g];
                }
#pragma unroll
                for (int s = 0; s < S; ++s) spv[s] = sp[s][v];
                Cell::elem(pv, wv, spv, f, A, be);
#pragma unroll
                for (int s = 0; s < S; ++s) {
                    if (rvalid) res = nanmax_f(res, fabsf(h[r][s][v] - f[s]));
                    sp[s][v] = h[r][s][v];
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) res = nanmax_f(res, __shfl_xor_sync(0xffffffffu, res, o));
        if (lane == 0) atomic_max_nonneg(prm.resid + K, res);
    }

    // ---- write h^(K) (the only HBM writes) ----
    bool bad = false;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int64_t t = tb + r;
        if (t < T && cvalid) {
#pragma unroll
            for (int s = 0; s < S; ++s) {
#pragma unroll
                for (int v = 0; v < V; ++v) bad |= !isfinite(h[r][s][v]);
                store_row<V>(prm.H + ((b * T + t) * S + s) * D + d0 + cc, h[r][s]);
            }
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(prm.lb.status, kStatusNonFinite);
}

}  // namespace pararnn
