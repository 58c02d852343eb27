// newton_fwd.cuh -- the fused Newton forward: every Newton iteration of a
// tile in one thread block; the tile's pre-activations are staged once in
// shared memory and the iterate stays in registers from the first iteration
// to the last.
//
// Method (pararnn-torch PyPI page, Method section): solve F(H) = 0,
// F_t = h_t - f(h_{t-1}, x_t), by K Newton iterations from the warm start
// h^(0)_t = f(0, x_t), each linear solve an associative scan over time.  The
// scan is on the direct-form elements
//     h^(k+1)_t = A_t h^(k+1)_{t-1} + beta_t,
//     A_t = df/dh at (h^(k)_{t-1}, x_t),  beta_t = f(h^(k)_{t-1}, x_t) - A_t h^(k)_{t-1}.
//
// Blocks are persistent: each takes tile tickets in increasing order and,
// while it works on one tile, the tensor memory accelerator already streams
// the next tile's pre-activations into the other shared-memory stage.
//
// Tile = W channels x L time steps of one batch row.  Thread (lc, sub) owns
// V consecutive channels of R consecutive steps; NSUB sub-chunks tile the L
// steps.  Per Newton iteration:
//   1. every thread evaluates f, A_t, beta_t on its R rows (the previous
//      row's state comes from its neighbour through shared memory) and
//      composes them into one element;
//   2. warp 0 composes the NSUB elements in time order, publishes the tile's
//      element, finds the carry by decoupled look-back over earlier tiles of
//      the same channels, publishes the state after the tile, and hands each
//      sub-chunk its carry-in;
//   3. every thread re-walks its R rows from its carry-in: h^(k+1).
// Iteration k+1 needs h^(k) just before the tile: that is the carry found in
// iteration k.  HBM traffic is the minimum: pre-activations read once, h^(K)
// written once.
#pragma once

#include "cells.cuh"
#include "common.cuh"
#include "lookback.cuh"
#include "tma.cuh"

namespace pararnn {

struct FwdParams {
    const void* px;      // (B,T,G,D) f32 or bf16
    const float* w;      // (G,D) or null
    const float* h0;     // (B,S,D) or null
    float* H;            // (B,T,S,D)
    float* resid;        // K+1 floats or null
    unsigned* ticket;    // workspace header word 1
    int64_t B, T, D;
    int K;
    int64_t nCG;         // channel groups per batch row
    int64_t nChunks;     // tiles along T
    int64_t nTiles;
    LookbackCtx lb;      // nGroups = B * nCG, nSlots = K
};

// V channels per thread, LC lanes across channels, NW warps, R rows per
// thread, MINB blocks per SM the register budget is sized for, P
// predecessors fetched at once by the look-back.
template <class Cell, typename PxT, int V_, int LC_, int NW_, int R_, int MINB_, bool kTma_>
struct FwdShape {
    static constexpr int V = V_, LC = LC_, NWARPS = NW_, R = R_, MINB = MINB_;
    static constexpr bool kTma = kTma_;
    static constexpr int G = Cell::G, S = Cell::S, NA = S * S + S;
    static constexpr int TPW = 32 / LC;           // sub-chunks per warp
    static constexpr int NSUB = NWARPS * TPW;     // sub-chunks per tile
    static constexpr int W = LC * V;              // channels per tile
    static constexpr int L = NSUB * R;            // time steps per tile
    static constexpr int NT = NWARPS * 32;
    static constexpr int NSTAGE = 2;
    static constexpr int P = S == 1 ? 4 : 2;
    static constexpr uint32_t kStageBytes = L * G * W * sizeof(PxT);
    static_assert(32 % LC == 0 && W % 32 == 0, "tile width must be a multiple of 32 channels");
    static_assert(!kTma || (W * sizeof(PxT)) % 16 == 0, "TMA box rows must be whole 16-byte units");
    static_assert(W <= 256 && L <= 256 && G <= 256, "TMA box dimensions are at most 256");
};

template <class Sh, typename PxT>
struct FwdSmem {
    alignas(128) PxT px[Sh::NSTAGE][Sh::L][Sh::G][Sh::W];  // TMA destination
    float agg[Sh::NSUB][Sh::NA][Sh::W];   // each sub-chunk's composed element
    float edge[Sh::NSUB][Sh::S][Sh::W];   // each sub-chunk's last state (current iterate)
    float carry[Sh::NSUB][Sh::S][Sh::W];  // each sub-chunk's carry-in
    float prev[Sh::S][Sh::W];             // current iterate just before the tile
    float w[Sh::G][Sh::W];                // the tile's recurrent weights
    uint64_t bar[Sh::NSTAGE];
    unsigned ticket[Sh::NSTAGE];
};

template <class Cell, typename PxT, class Sh>
__device__ __forceinline__ void issue_tile_load(const CUtensorMap* map, FwdSmem<Sh, PxT>& sm, const FwdParams& prm,
                                                unsigned tile, int stage) {
    const int64_t chunk = tile / prm.lb.nGroups;
    const int64_t gid = tile - chunk * prm.lb.nGroups;
    const int64_t b = gid / prm.nCG;
    const int64_t d0 = (gid - b * prm.nCG) * Sh::W;
    mbar_arrive_expect_tx(&sm.bar[stage], Sh::kStageBytes);
    tma_load_3d(&sm.px[stage][0][0][0], map, &sm.bar[stage], (int)d0, 0, (int)(b * prm.T + chunk * Sh::L));
}

template <class Cell, typename PxT, class Sh, bool kLean>
__global__ void __launch_bounds__(Sh::NT, Sh::MINB)
    newton_fwd_kernel(const __grid_constant__ CUtensorMap tmap, const FwdParams prm) {
    constexpr int G = Sh::G, S = Sh::S, V = Sh::V, R = Sh::R;
    constexpr int TPW = Sh::TPW, NSUB = Sh::NSUB, W = Sh::W, L = Sh::L, LC = Sh::LC, NT = Sh::NT;
    constexpr int CPL = W / 32;
    using SM = FwdSmem<Sh, PxT>;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    SM& sm = *reinterpret_cast<SM*>(smem_raw);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sub = warp * TPW + lane / LC;
    const int cc = (lane % LC) * V;
    const int64_t T = prm.T, D = prm.D;
    const PxT* pxg = static_cast<const PxT*>(prm.px);
    const bool need_prev = Cell::kNonlinear || prm.resid != nullptr;

    if (tid == 0) {
        if constexpr (Sh::kTma) {
#pragma unroll
            for (int s = 0; s < Sh::NSTAGE; ++s) mbar_init(&sm.bar[s], 1);
            mbar_fence_init();
        }
        const unsigned t = atomicAdd(prm.ticket, 1u);
        sm.ticket[0] = t;
        if constexpr (Sh::kTma)
            if (t < prm.nTiles) issue_tile_load<Cell, PxT, Sh>(&tmap, sm, prm, t, 0);
    }
    __syncthreads();

    for (int it = 0;; ++it) {
        const int st = it % Sh::NSTAGE;
        const unsigned tile_u = sm.ticket[st];
        if (tile_u >= prm.nTiles) break;
        if (tid == 0) {
            // claim the next tile now and start streaming it in
            const unsigned t2 = atomicAdd(prm.ticket, 1u);
            sm.ticket[(it + 1) % Sh::NSTAGE] = t2;
            if constexpr (Sh::kTma)
                if (t2 < prm.nTiles) issue_tile_load<Cell, PxT, Sh>(&tmap, sm, prm, t2, (it + 1) % Sh::NSTAGE);
        }
        const int64_t tile = tile_u;
        const int64_t chunk = tile / prm.lb.nGroups;
        const int64_t gid = tile - chunk * prm.lb.nGroups;
        const int64_t b = gid / prm.nCG;
        const int64_t d0 = (gid - b * prm.nCG) * W;
        const int64_t t0 = chunk * L;
        const int64_t tb = t0 + (int64_t)sub * R;
        const bool cvalid = d0 + cc < D;  // D is a multiple of V: a vector is wholly in or out

        // weights of the tile's channels
        for (int i = tid; i < G * W; i += NT) {
            const int g = i / W, c = i - (i / W) * W;
            sm.w[g][c] = (prm.w && d0 + c < D) ? __ldg(prm.w + g * D + d0 + c) : 0.0f;
        }
        // h^(0) just before the tile: h0 for the first tile, else the warm start of the previous row
        if (need_prev && tid < W) {
            const int64_t d = d0 + tid;
            float f[S] = {};
            if (d < D) {
                if (t0 == 0) {
#pragma unroll
                    for (int s = 0; s < S; ++s) f[s] = prm.h0 ? prm.h0[(b * S + s) * D + d] : 0.0f;
                } else {
                    float pv[G], wv[G];
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        pv[g] = PxTraits<PxT>::cvt(pxg[((b * T + t0 - 1) * G + g) * D + d]);
                        wv[g] = prm.w ? __ldg(prm.w + g * D + d) : 0.0f;
                    }
                    Cell::warm(pv, wv, f);
                }
            }
#pragma unroll
            for (int s = 0; s < S; ++s) sm.prev[s][tid] = f[s];
        }
        // the tile's pre-activations: TMA (already in flight) or a cooperative copy
        if constexpr (Sh::kTma) {
            Deadline dl;
            while (!mbar_try_wait(&sm.bar[st], (it / Sh::NSTAGE) & 1)) {
                if (dl.expired(prm.lb.timeout_ns)) {
                    if (tid == 0) atomicOr(prm.lb.status, kStatusTimeout);
                    break;
                }
            }
        } else {
            for (int i = tid; i < L * G * W; i += NT) {
                const int row = i / (G * W), rem = i - row * (G * W), g = rem / W, c = rem - g * W;
                const int64_t t = t0 + row, d = d0 + c;
                sm.px[st][row][g][c] = (t < T && d < D) ? pxg[((b * T + t) * G + g) * D + d] : PxT(0.0f);
            }
        }
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
        __syncthreads();

        auto load_p = [&](int r, int v, float (&pv)[G], float (&wv)[G]) {
#pragma unroll
            for (int g = 0; g < G; ++g) {
                pv[g] = PxTraits<PxT>::cvt(sm.px[st][sub * R + r][g][cc + v]);
                wv[g] = sm.w[g][cc + v];
            }
        };

        if constexpr (kLean) {
            // ---- the linear cell without a residual: one scan, elements read straight from shared memory ----
#pragma unroll
            for (int v = 0; v < V; ++v) {
                Elem<S> acc;
                elem_identity<S>(acc);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    if (tb + r < T) {
                        float pv[G], wv[G], A[S * S], be[S];
                        load_p(r, v, pv, wv);
                        A[0] = pv[0];
                        be[0] = pv[1];
                        compose_after<S>(A, be, acc);
                    }
                }
                sm.agg[sub][0][cc + v] = acc.A[0];
                sm.agg[sub][1][cc + v] = acc.b[0];
            }
            __syncthreads();
            if (warp == 0) {
                float carry[CPL][S];
                tile_scan_step<S, W, NSUB, Sh::P>(prm.lb, tile, chunk, 0, lane, sm.agg, sm.carry, first_carry, carry);
            }
            __syncthreads();
            float out[R][V];
#pragma unroll
            for (int v = 0; v < V; ++v) {
                float x = sm.carry[sub][0][cc + v];
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    float pv[G], wv[G];
                    load_p(r, v, pv, wv);
                    x = __fmaf_rn(pv[0], x, pv[1]);
                    out[r][v] = x;
                }
            }
            bool bad = false;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int64_t t = tb + r;
                if (t < T && cvalid) {
#pragma unroll
                    for (int v = 0; v < V; ++v) bad |= !isfinite(out[r][v]);
                    store_row<V>(prm.H + (b * T + t) * D + d0 + cc, out[r]);
                }
            }
            if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(prm.lb.status, kStatusNonFinite);
        } else {
            // ---- general path: warm start, K Newton iterations ----
            float h[R][S][V];
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    float pv[G], wv[G], f[S];
                    load_p(r, v, pv, wv);
                    Cell::warm(pv, wv, f);
#pragma unroll
                    for (int s = 0; s < S; ++s) h[r][s][v] = f[s];
                }
            if (need_prev) {
#pragma unroll
                for (int s = 0; s < S; ++s)
#pragma unroll
                    for (int v = 0; v < V; ++v) sm.edge[sub][s][cc + v] = h[R - 1][s][v];
            }
            const int K = prm.K;
            for (int k = 0; k <= K; ++k) {
                __syncthreads();
                // ---- 1. elements of iteration k+1 and the residual of iterate k ----
                float sp[S][V];
#pragma unroll
                for (int s = 0; s < S; ++s)
#pragma unroll
                    for (int v = 0; v < V; ++v)
                        sp[s][v] = !need_prev ? 0.0f : (sub == 0 ? sm.prev[s][cc + v] : sm.edge[sub - 1][s][cc + v]);
                float eA[R][S * S][V], eb[R][S][V];
                float res = 0.0f;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const bool rvalid = (tb + r < T) && cvalid;
#pragma unroll
                    for (int v = 0; v < V; ++v) {
                        float pv[G], wv[G], spv[S], f[S], A[S * S], be[S];
                        load_p(r, v, pv, wv);
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
                if (prm.resid) {
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) res = nanmax_f(res, __shfl_xor_sync(0xffffffffu, res, o));
                    if (lane == 0) atomic_max_nonneg(prm.resid + k, res);
                }
                if (k == K) break;  // the last pass only measured the residual of h^(K)
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
                    for (int a = 0; a < S * S; ++a) sm.agg[sub][a][cc + v] = acc.A[a];
#pragma unroll
                    for (int s = 0; s < S; ++s) sm.agg[sub][S * S + s][cc + v] = acc.b[s];
                }
                __syncthreads();

                // ---- 2. tile composition, look-back, carries (warp 0) ----
                if (warp == 0) {
                    float carry[CPL][S];
                    tile_scan_step<S, W, NSUB, Sh::P>(prm.lb, tile, chunk, k, lane, sm.agg, sm.carry, first_carry,
                                                      carry);
#pragma unroll
                    for (int j = 0; j < CPL; ++j)
#pragma unroll
                        for (int s = 0; s < S; ++s) sm.prev[s][lane + 32 * j] = carry[j][s];
                }
                __syncthreads();

                // ---- 3. re-walk the rows from the carry-in: h^(k+1) ----
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    float x[S];
#pragma unroll
                    for (int s = 0; s < S; ++s) x[s] = sm.carry[sub][s][cc + v];
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
                        for (int v = 0; v < V; ++v) sm.edge[sub][s][cc + v] = h[R - 1][s][v];
                }
                if (k + 1 == K && !prm.resid) break;  // no residual pass wanted
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
        __syncthreads();  // stage st and the ticket slot are free again
    }
}

}  // namespace pararnn
