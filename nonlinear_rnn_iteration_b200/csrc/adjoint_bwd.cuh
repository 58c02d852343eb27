// adjoint_bwd.cuh -- the backward pass: a reverse-time scan for the adjoint
// state and the gradient epilogue, fused in one persistent kernel, plus a
// fixed-order reduction of the per-tile weight-gradient partials.
//
// At the trajectory H (the forward's output), with g_t = dL/dH_t, the adjoint
// of the lower-bidiagonal system F(H) = 0 is
//     lambda_t = g_t + A_{t+1}^T lambda_{t+1},   lambda_{T-1} = g_{T-1},
//     A_t = df/dh at (h_{t-1}, x_t)
// (pararnn-torch PyPI page, Method section: the backward follows the paper's
// adjoint).  The kernel scans the propagated adjoint mu_t = A_t^T lambda_t
// instead of lambda itself:
//     mu_t = A_t^T (g_t + mu_{t+1}),   mu_T = 0,   lambda_t = g_t + mu_{t+1},
// a reverse-time scan of the elements (A_t^T, A_t^T g_t) under the same
// operator as the forward.  Each element needs only its own row's Jacobian
// (no neighbouring row), and dL/dh0 = A_0^T lambda_0 = mu_0 is the scan's
// last state.  Then
//     dL/dp_g[t]  = lambda_t . df/dp_g   at (h_{t-1}, x_t)
//     dL/da_g     = sum_{b,t} lambda_t . df/da_g.
// dL/da is summed within a tile in a fixed order, written per tile, and
// reduced over tiles in a fixed order by a second kernel: no floating-point
// atomics, so the result does not depend on scheduling (Compatibility
// section: the packed VJP is deterministic).
#pragma once

#include "cells.cuh"
#include "common.cuh"
#include "lookback.cuh"
#include "newton_fwd.cuh"
#include "tma.cuh"

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
    unsigned* ticket;
    int64_t B, T, D;
    int64_t nCG, nChunks, nTiles;
    int late_probe;     // probe the predecessor while the tile is evaluated (see the scan warp)
    LookbackCtx lb;     // nSlots = 1
};

// Stage rows: px and dL/dH row i are time t0 + i; H row i is time t0 - 1 + i
// (the state row i is linearised at).  Each array is 128-byte aligned (a
// tensor copy writes to a 128-byte aligned shared address).
template <class Sh, typename PxT>
struct alignas(128) BwdStage {
    alignas(128) PxT px[Sh::L][Sh::G][Sh::W];
    alignas(128) float H[Sh::L][Sh::S][Sh::W];
    alignas(128) float g[Sh::L][Sh::S][Sh::W];
};

template <class Sh, typename PxT>
struct BwdSmem {
    BwdStage<Sh, PxT> stg[Sh::NSTAGE];
    float wagg[Sh::NWARPS][Sh::NA][Sh::W];  // each warp's composed element
    float cin[Sh::S][Sh::W];                // mu just after the tile (the carry)
    float hprev[Sh::S][Sh::W];              // h0 (for the first tile of a row)
    float w[Sh::G][Sh::W];
    float da[2][Sh::NSUB][Sh::G][Sh::W];    // per-sub-chunk dL/da partials, two tiles in turn
    uint64_t bar[Sh::NSTAGE];
    unsigned ticket[Sh::NSTAGE];
};

template <class Sh>
struct BwdMaps {
    CUtensorMap px, H, g;
};

// L2 hints, by cell: the LSTM adjoint (one 11-warp block per SM) ran 6 %
// faster with its tile loads marked evict-first and its dL/dpx stores
// streaming (evict-first alone: 2.5 %, streaming stores alone: 0.6 %); the
// GRU adjoint ran 12 % slower with both, so it keeps the default policy.
template <class Cell>
struct BwdStreamHints {
    static constexpr bool value = false;
};
template <>
struct BwdStreamHints<CellLSTM> {
    static constexpr bool value = true;
};

// tma_load_3d with an L2 evict-first policy (the tile is read once)
__device__ __forceinline__ void tma_load_3d_evict_first(void* dst, const CUtensorMap* map, uint64_t* bar, int c0,
                                                        int c1, int c2) {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4}], [%5], %6;"
        ::"r"(smem_u32(dst)), "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
}

template <bool kStream>
__device__ __forceinline__ void tile_load(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2) {
    if constexpr (kStream)
        tma_load_3d_evict_first(dst, map, bar, c0, c1, c2);
    else
        tma_load_3d(dst, map, bar, c0, c1, c2);
}

// store_row with streaming (evict-first) stores
template <int V, bool kStream>
__device__ __forceinline__ void store_out_row(float* p, const float (&v)[V]) {
    if constexpr (!kStream) {
        store_row<V>(p, v);
    } else if constexpr (V == 4) {
        __stcs(reinterpret_cast<float4*>(p), make_float4(v[0], v[1], v[2], v[3]));
    } else if constexpr (V == 2) {
        __stcs(reinterpret_cast<float2*>(p), make_float2(v[0], v[1]));
    } else {
#pragma unroll
        for (int i = 0; i < V; ++i) __stcs(p + i, v[i]);
    }
}

template <class Cell, typename PxT, class Sh>
__device__ __forceinline__ void issue_bwd_load(const BwdMaps<Sh>* maps, BwdSmem<Sh, PxT>& sm, const BwdParams& prm,
                                               unsigned tile, int stage) {
    const int64_t pos = tile / prm.lb.nGroups;
    const int64_t gid = tile - pos * prm.lb.nGroups;
    const int64_t chunk = prm.nChunks - 1 - pos;
    const int64_t b = gid / prm.nCG;
    const int64_t d0 = (gid - b * prm.nCG) * Sh::W;
    const int row = (int)(b * prm.T + chunk * Sh::L);
    constexpr uint32_t bytes = Sh::L * Sh::W * (Sh::G * sizeof(PxT) + 2 * Sh::S * sizeof(float));
    mbar_arrive_expect_tx(&sm.bar[stage], bytes);
    constexpr bool kStream = BwdStreamHints<Cell>::value;
    tile_load<kStream>(&sm.stg[stage].px[0][0][0], &maps->px, &sm.bar[stage], (int)d0, 0, row);
    // row - 1 may be -1 (first tile of the first batch row): TMA fills zeros there
    tile_load<kStream>(&sm.stg[stage].H[0][0][0], &maps->H, &sm.bar[stage], (int)d0, 0, row - 1);
    tile_load<kStream>(&sm.stg[stage].g[0][0][0], &maps->g, &sm.bar[stage], (int)d0, 0, row);
}

// y = A^T v on a pair of channels
template <int S>
__device__ __forceinline__ void mat_t_vec2(const f2 (&A)[S * S], const f2 (&v)[S], f2 (&y)[S]) {
    if constexpr (S == 1) {
        y[0] = mul2(A[0], v[0]);
    } else {
        y[0] = fma2(A[0], v[0], mul2(A[2], v[1]));
        y[1] = fma2(A[1], v[0], mul2(A[3], v[1]));
    }
}

// y = A^T v
template <int S>
__device__ __forceinline__ void mat_t_vec(const float (&A)[S * S], const float (&v)[S], float (&y)[S]) {
    if constexpr (S == 1) {
        y[0] = A[0] * v[0];
    } else {
        y[0] = __fmaf_rn(A[0], v[0], A[2] * v[1]);
        y[1] = __fmaf_rn(A[1], v[0], A[3] * v[1]);
    }
}

// The dL/da partial of one tile: the sum of its sub-chunks' partials in
// sub-chunk order, written by the scan warp.
template <class Sh, typename PxT>
__device__ __forceinline__ void store_tile_partial(const BwdSmem<Sh, PxT>& sm, int buf, const BwdParams& prm,
                                                   int64_t tile, int lane) {
    constexpr int G = Sh::G, W = Sh::W;
    for (int i = lane; i < G * W; i += 32) {
        const int g = i / W, ch = i - (i / W) * W;
        float acc = 0.0f;
#pragma unroll
        for (int sb = 0; sb < Sh::NSUB; ++sb) acc += sm.da[buf][sb][g][ch];
        prm.part[(tile * G + g) * W + ch] = acc;
    }
}

// kRecompute (packed path only): keep no per-row state in registers across
// the carry barriers -- the epilogue evaluates each row's Jacobian and
// sensitivities again from the tile still staged in shared memory -- so that
// a thread needs far fewer registers and more warps share an SM.
template <class Cell, typename PxT, class Sh, bool kRecompute = false>
__global__ void __launch_bounds__(Sh::NT, Sh::MINB)
    adjoint_bwd_kernel(const __grid_constant__ BwdMaps<Sh> maps, const BwdParams prm) {
    constexpr int G = Sh::G, S = Sh::S, V = Sh::V, R = Sh::R, NS = Cell::NSENS, NW = Sh::NWARPS;
    constexpr int TPW = Sh::TPW, W = Sh::W, L = Sh::L, LC = Sh::LC, NTC = Sh::NTC;
    constexpr int NSTAGE = Sh::NSTAGE;
    constexpr int CPL = W / 32;
    using SM = BwdSmem<Sh, PxT>;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    SM& sm = *reinterpret_cast<SM*>(smem_raw);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool is_scan = warp == NW;
    const int64_t T = prm.T, D = prm.D;
    const PxT* pxg = static_cast<const PxT*>(prm.px);

    if (is_scan && lane == 0) {
        if constexpr (Sh::kTma) {
#pragma unroll
            for (int s = 0; s < NSTAGE; ++s) mbar_init(&sm.bar[s], 1);
            mbar_fence_init();
        }
#pragma unroll
        for (int s = 0; s < NSTAGE - 1; ++s) {
            const unsigned t = atomicAdd(prm.ticket, 1u);
            sm.ticket[s] = t;
            if constexpr (Sh::kTma)
                if (t < prm.nTiles) issue_bwd_load<Cell, PxT, Sh>(&maps, sm, prm, t, s);
        }
    }
    block_sync();

    // Three block barriers per tile: (1) tile set up, (2) warp totals ready,
    // (3) carry ready.  Nothing is shared across the end of a tile without
    // one of them in between: the next tile's stage is refilled only after
    // its barrier (1), the dL/da partials alternate between two buffers and
    // the scan warp reduces a tile's partials between barriers (1) and (2)
    // of the block's next tile.
    int64_t prev_tile = -1;  // scan warp: the tile whose partials sit in da[(it - 1) & 1]
    int it = 0;
    for (;; ++it) {
        const int st = it % NSTAGE;
        const unsigned tile_u = sm.ticket[st];
        if (tile_u >= prm.nTiles) break;
        const int64_t tile = tile_u;
        const int64_t pos = tile / prm.lb.nGroups;
        const int64_t gid = tile - pos * prm.lb.nGroups;
        const int64_t chunk = prm.nChunks - 1 - pos;
        const int64_t b = gid / prm.nCG;
        const int64_t d0 = (gid - b * prm.nCG) * W;
        const int64_t t0 = chunk * L;

        if (is_scan) {
            // ================= scan warp =================
            float zero[CPL][S];
#pragma unroll
            for (int j = 0; j < CPL; ++j)
#pragma unroll
                for (int s = 0; s < S; ++s) zero[j][s] = 0.0f;  // mu_T = 0
            // With at least as many channel groups as resident blocks, a tile's
            // predecessor (one ticket per group earlier) was claimed a whole
            // round of tiles before it and has usually finished: its state is
            // then read once the evaluation has started (after the set-up
            // barrier), and the look-back after the totals barrier is skipped.
            // With fewer groups the predecessor is still running, the probe
            // misses, and its reads cost more than they save (measured: the
            // 8 x 4096 x 2048 GRU adjoint 12 % faster with it, the
            // 1 x 131072 x 4096 GRU 6 % and the 4 x 32768 x 1024 LSTM 3 %
            // slower).  The 2 x 2 cell's adjoint is at its register limit,
            // where even the unused branch costs spills, so it has no late
            // probe.
            Probe<S, W> pr;
            pr.st = 0;
            block_sync();  // (1) tile set up
            if (lane == 0) {
                // claim the tile NSTAGE-1 ahead and start streaming it in
                const int sn = (it + NSTAGE - 1) % NSTAGE;
                const unsigned prev_t = sm.ticket[(it + NSTAGE - 2) % NSTAGE];
                unsigned t2 = prev_t;
                if (prev_t < prm.nTiles) t2 = atomicAdd(prm.ticket, 1u);
                sm.ticket[sn] = t2;
                if constexpr (Sh::kTma)
                    if (t2 < prm.nTiles && prev_t < prm.nTiles) issue_bwd_load<Cell, PxT, Sh>(&maps, sm, prm, t2, sn);
            }
            if constexpr (S == 1) {
                if (prm.late_probe) probe_issue<S, W>(prm.lb, tile, pos, 0, lane, pr);
            }
            if (prev_tile >= 0) store_tile_partial<Sh, PxT>(sm, (it - 1) & 1, prm, prev_tile, lane);
            prev_tile = tile;
            block_sync();  // (2) warp totals ready
            Inclusive<S, W> inc;
            tile_lookback<S, W, NW, true>(prm.lb, tile, pos, 0, lane, sm.wagg, zero, pr, sm.cin, inc);
            block_sync();  // (3) carry ready
            publish_inclusive<S, W>(prm.lb, tile, 0, lane, inc);
        } else {
            // ================= compute warps =================
            const int sub = warp * TPW + lane / LC;
            const int cc = (lane % LC) * V;
            const int64_t tb = t0 + (int64_t)sub * R;
            const bool cvalid = d0 + cc < D;

            for (int i = tid; i < G * W; i += NTC) {
                const int g = i / W, c = i - (i / W) * W;
                sm.w[g][c] = (prm.w && d0 + c < D) ? __ldg(prm.w + g * D + d0 + c) : 0.0f;
            }
            if (t0 == 0 && tid < W) {
                const int64_t d = d0 + tid;
#pragma unroll
                for (int s = 0; s < S; ++s) sm.hprev[s][tid] = (prm.h0 && d < D) ? prm.h0[(b * S + s) * D + d] : 0.0f;
            }
            if constexpr (Sh::kTma) {
                Deadline dl;
                while (!mbar_try_wait(&sm.bar[st], (it / NSTAGE) & 1)) {
                    if (dl.expired(prm.lb.timeout_ns)) {
                        if (tid == 0) atomicOr(prm.lb.status, kStatusTimeout);
                        break;
                    }
                }
            } else {
                for (int i = tid; i < L * G * W; i += NTC) {
                    const int row = i / (G * W), rem = i - row * (G * W), g = rem / W, c = rem - g * W;
                    const int64_t t = t0 + row, d = d0 + c;
                    sm.stg[st].px[row][g][c] = (t < T && d < D) ? pxg[((b * T + t) * G + g) * D + d] : PxT(0.0f);
                }
                for (int i = tid; i < L * S * W; i += NTC) {
                    const int row = i / (S * W), rem = i - row * (S * W), s = rem / W, c = rem - s * W;
                    const int64_t th = t0 - 1 + row, tg = t0 + row, d = d0 + c;
                    sm.stg[st].H[row][s][c] = (th >= 0 && th < T && d < D) ? prm.H[((b * T + th) * S + s) * D + d] : 0.0f;
                    sm.stg[st].g[row][s][c] = (tg < T && d < D) ? prm.dLdH[((b * T + tg) * S + s) * D + d] : 0.0f;
                }
            }
            block_sync();  // (1) tile set up

            float wr[V][G];  // the recurrent weights of this thread's channels
#pragma unroll
            for (int v = 0; v < V; ++v)
#pragma unroll
                for (int g = 0; g < G; ++g) wr[v][g] = sm.w[g][cc + v];

            // two channels per instruction where the thread holds an even
            // number of them (packed f32x2; same rounding as one by one)
            constexpr bool kPack = (V % 2 == 0) && Cell::kNonlinear;
            constexpr int VP = kPack ? V / 2 : 1;
            typename Cell::W2 wp[VP];
            if constexpr (kPack) {
#pragma unroll
                for (int q = 0; q < VP; ++q) wp[q] = Cell::weights2(wr[2 * q], wr[2 * q + 1]);
            }

            // the linearisation of row r at (h_{t-1}, x_t) for channel pair q,
            // from the staged tile: A, the sensitivities and g_t (the identity
            // element and g = 0 past the end of the sequence)
            auto lin2 = [&](int r, int q, f2 (&A)[S * S], f2 (&se)[NS], f2 (&gv)[S]) {
              if constexpr (kPack) {
                const int row = sub * R + r;
                const bool rvalid = (tb + r < T) && cvalid;
                const int c0 = cc + 2 * q;
                f2 pg[G], spv[S];
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    float pv2[2];
                    lds_row<2>(&sm.stg[st].px[row][g][c0], pv2);
                    pg[g] = f2{pv2[0], pv2[1]};
                }
#pragma unroll
                for (int s = 0; s < S; ++s) {
                    float hv2[2], gv2[2];
                    lds_row<2>((t0 == 0 && row == 0) ? &sm.hprev[s][c0] : &sm.stg[st].H[row][s][c0], hv2);
                    lds_row<2>(&sm.stg[st].g[row][s][c0], gv2);
                    spv[s] = f2{hv2[0], hv2[1]};
                    gv[s] = rvalid ? f2{gv2[0], gv2[1]} : splat2(0.0f);
                }
                Cell::bwd2(pg, wp[q], spv, A, se);
                if (!rvalid) {
#pragma unroll
                    for (int a = 0; a < S * S; ++a) A[a] = splat2((a % (S + 1) == 0) ? 1.0f : 0.0f);
                }
              }
            };
            (void)lin2;

            // ---- linearisation at (h_{t-1}, x_t) and the sub-chunk's element,
            //      composed in scan order (latest row first) ----
            float jA[R][S * S][V], sens[R][NS][V], gr[R][S][V];
            ElemV<S, V> mine, excl, pre;
#pragma unroll
            for (int v = 0; v < V; ++v) elem_identity<S>(mine.e[v]);
#pragma unroll
            for (int r = R - 1; r >= 0; --r) {
                const int row = sub * R + r;
                const bool rvalid = (tb + r < T) && cvalid;
                float pv[G][V], hv[S][V];
                if constexpr (!(kPack && kRecompute)) {
#pragma unroll
                    for (int g = 0; g < G; ++g) lds_row<V>(&sm.stg[st].px[row][g][cc], pv[g]);
#pragma unroll
                    for (int s = 0; s < S; ++s)
                        lds_row<V>((t0 == 0 && row == 0) ? &sm.hprev[s][cc] : &sm.stg[st].H[row][s][cc], hv[s]);
#pragma unroll
                    for (int s = 0; s < S; ++s) lds_row<V>(&sm.stg[st].g[row][s][cc], gr[r][s]);
                }
                if constexpr (kPack && kRecompute) {
#pragma unroll
                    for (int q = 0; q < VP; ++q) {
                        const int v0 = 2 * q, v1 = 2 * q + 1;
                        f2 A[S * S], se[NS], gv[S], M[S * S], bv[S], accA[S * S], accb[S];
                        lin2(r, q, A, se, gv);
#pragma unroll
                        for (int i = 0; i < S; ++i)
#pragma unroll
                            for (int m = 0; m < S; ++m) M[i * S + m] = A[m * S + i];  // A^T
                        mat_t_vec2<S>(A, gv, bv);
#pragma unroll
                        for (int a = 0; a < S * S; ++a) accA[a] = f2{mine.e[v0].A[a], mine.e[v1].A[a]};
#pragma unroll
                        for (int s = 0; s < S; ++s) accb[s] = f2{mine.e[v0].b[s], mine.e[v1].b[s]};
                        compose_after2<S>(M, bv, accA, accb);
#pragma unroll
                        for (int a = 0; a < S * S; ++a) {
                            mine.e[v0].A[a] = accA[a].x;
                            mine.e[v1].A[a] = accA[a].y;
                        }
#pragma unroll
                        for (int s = 0; s < S; ++s) {
                            mine.e[v0].b[s] = accb[s].x;
                            mine.e[v1].b[s] = accb[s].y;
                        }
                    }
                } else if constexpr (kPack) {
#pragma unroll
                    for (int q = 0; q < VP; ++q) {
                        const int v0 = 2 * q, v1 = 2 * q + 1;
                        f2 pg[G], spv[S], A[S * S], se[NS], gv[S];
#pragma unroll
                        for (int g = 0; g < G; ++g) pg[g] = f2{pv[g][v0], pv[g][v1]};
#pragma unroll
                        for (int s = 0; s < S; ++s) spv[s] = f2{hv[s][v0], hv[s][v1]};
                        Cell::bwd2(pg, wp[q], spv, A, se);
                        if (!rvalid) {
                            // past the end of the sequence: the identity element
#pragma unroll
                            for (int a = 0; a < S * S; ++a) A[a] = splat2((a % (S + 1) == 0) ? 1.0f : 0.0f);
#pragma unroll
                            for (int s = 0; s < S; ++s) {
                                gr[r][s][v0] = 0.0f;
                                gr[r][s][v1] = 0.0f;
                            }
                        }
#pragma unroll
                        for (int a = 0; a < S * S; ++a) {
                            jA[r][a][v0] = A[a].x;
                            jA[r][a][v1] = A[a].y;
                        }
#pragma unroll
                        for (int n = 0; n < NS; ++n) {
                            sens[r][n][v0] = se[n].x;
                            sens[r][n][v1] = se[n].y;
                        }
                        f2 M[S * S], bv[S], accA[S * S], accb[S];
#pragma unroll
                        for (int i = 0; i < S; ++i)
#pragma unroll
                            for (int m = 0; m < S; ++m) M[i * S + m] = A[m * S + i];  // A^T
#pragma unroll
                        for (int s = 0; s < S; ++s) gv[s] = f2{gr[r][s][v0], gr[r][s][v1]};
                        mat_t_vec2<S>(A, gv, bv);
#pragma unroll
                        for (int a = 0; a < S * S; ++a) accA[a] = f2{mine.e[v0].A[a], mine.e[v1].A[a]};
#pragma unroll
                        for (int s = 0; s < S; ++s) accb[s] = f2{mine.e[v0].b[s], mine.e[v1].b[s]};
                        compose_after2<S>(M, bv, accA, accb);
#pragma unroll
                        for (int a = 0; a < S * S; ++a) {
                            mine.e[v0].A[a] = accA[a].x;
                            mine.e[v1].A[a] = accA[a].y;
                        }
#pragma unroll
                        for (int s = 0; s < S; ++s) {
                            mine.e[v0].b[s] = accb[s].x;
                            mine.e[v1].b[s] = accb[s].y;
                        }
                    }
                } else {
#pragma unroll
                    for (int v = 0; v < V; ++v) {
                        float pg[G], spv[S], A[S * S], se[NS];
#pragma unroll
                        for (int g = 0; g < G; ++g) pg[g] = pv[g][v];
#pragma unroll
                        for (int s = 0; s < S; ++s) spv[s] = hv[s][v];
                        Cell::bwd(pg, wr[v], spv, A, se);
                        if (!rvalid) {
                            // past the end of the sequence: the identity element
#pragma unroll
                            for (int a = 0; a < S * S; ++a) A[a] = (a % (S + 1) == 0) ? 1.0f : 0.0f;
#pragma unroll
                            for (int s = 0; s < S; ++s) gr[r][s][v] = 0.0f;
                        }
#pragma unroll
                        for (int a = 0; a < S * S; ++a) jA[r][a][v] = A[a];
#pragma unroll
                        for (int n = 0; n < NS; ++n) sens[r][n][v] = se[n];
                        float M[S * S], gv[S], bv[S];
#pragma unroll
                        for (int i = 0; i < S; ++i)
#pragma unroll
                            for (int m = 0; m < S; ++m) M[i * S + m] = A[m * S + i];  // A^T
#pragma unroll
                        for (int s = 0; s < S; ++s) gv[s] = gr[r][s][v];
                        mat_t_vec<S>(A, gv, bv);
                        compose_after<S>(M, bv, mine.e[v]);
                    }
                }
            }
            warp_prefix<S, V, LC, W, NW, true>(mine, excl, warp, lane, sm.wagg);
            block_sync();  // (2) warp totals ready
            sub_prefix<S, V, LC, W, NW, true>(excl, warp, lane, sm.wagg, pre);
            block_sync();  // (3) carry ready

            // ---- lambda and the gradient epilogue ----
            float da_acc[G][V];
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int v = 0; v < V; ++v) da_acc[g][v] = 0.0f;
            float outp[R][G][V];
            bool bad = false;
            if constexpr (kPack && kRecompute) {
#pragma unroll
                for (int q = 0; q < VP; ++q) {
                    const int v0 = 2 * q, v1 = 2 * q + 1;
                    f2 x[S], cv[S], PA[S * S], Pb[S], dacc[G];  // x = mu_{t+1}
#pragma unroll
                    for (int s = 0; s < S; ++s) cv[s] = f2{sm.cin[s][cc + v0], sm.cin[s][cc + v1]};
#pragma unroll
                    for (int a = 0; a < S * S; ++a) PA[a] = f2{pre.e[v0].A[a], pre.e[v1].A[a]};
#pragma unroll
                    for (int s = 0; s < S; ++s) Pb[s] = f2{pre.e[v0].b[s], pre.e[v1].b[s]};
                    apply2<S>(PA, Pb, cv, x);
#pragma unroll
                    for (int g = 0; g < G; ++g) dacc[g] = splat2(0.0f);
#pragma unroll
                    for (int r = R - 1; r >= 0; --r) {
                        const int64_t t = tb + r;
                        const bool rvalid = (t < T) && cvalid;
                        f2 lam[S], A[S * S], se[NS], gv[S], dp[G], da[G];
                        lin2(r, q, A, se, gv);
#pragma unroll
                        for (int s = 0; s < S; ++s) lam[s] = add2(gv[s], x[s]);
                        mat_t_vec2<S>(A, lam, x);  // mu_t
                        Cell::grads2(se, lam, dp, da);
                        if (rvalid) {
                            float o0[G], o1[G];
#pragma unroll
                            for (int g2 = 0; g2 < G; ++g2) {
                                dacc[g2] = add2(dacc[g2], da[g2]);
                                bad |= !isfinite(dp[g2].x) || !isfinite(dp[g2].y);
                                o0[g2] = dp[g2].x;
                                o1[g2] = dp[g2].y;
                            }
#pragma unroll
                            for (int g2 = 0; g2 < G; ++g2) {
                                float o2[2] = {o0[g2], o1[g2]};
                                store_out_row<2, BwdStreamHints<Cell>::value>(
                                    prm.dLdpx + ((b * T + t) * G + g2) * D + d0 + cc + v0, o2);
                            }
                        }
                        if (r == 0 && tb == 0 && rvalid && prm.dLdh0) {
                            // dL/dh0 = A_0^T lambda_0 = mu_0
#pragma unroll
                            for (int s = 0; s < S; ++s) {
                                prm.dLdh0[(b * S + s) * D + d0 + cc + v0] = x[s].x;
                                prm.dLdh0[(b * S + s) * D + d0 + cc + v1] = x[s].y;
                            }
                        }
                    }
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        da_acc[g][v0] = dacc[g].x;
                        da_acc[g][v1] = dacc[g].y;
                    }
                }
            } else if constexpr (kPack) {
#pragma unroll
                for (int q = 0; q < VP; ++q) {
                    const int v0 = 2 * q, v1 = 2 * q + 1;
                    f2 x[S], cv[S], PA[S * S], Pb[S], dacc[G];  // x = mu_{t+1}
#pragma unroll
                    for (int s = 0; s < S; ++s) cv[s] = f2{sm.cin[s][cc + v0], sm.cin[s][cc + v1]};
#pragma unroll
                    for (int a = 0; a < S * S; ++a) PA[a] = f2{pre.e[v0].A[a], pre.e[v1].A[a]};
#pragma unroll
                    for (int s = 0; s < S; ++s) Pb[s] = f2{pre.e[v0].b[s], pre.e[v1].b[s]};
                    apply2<S>(PA, Pb, cv, x);
#pragma unroll
                    for (int g = 0; g < G; ++g) dacc[g] = splat2(0.0f);
#pragma unroll
                    for (int r = R - 1; r >= 0; --r) {
                        const bool rvalid = (tb + r < T) && cvalid;
                        f2 lam[S], A[S * S], se[NS], dp[G], da[G];
#pragma unroll
                        for (int s = 0; s < S; ++s) lam[s] = add2(f2{gr[r][s][v0], gr[r][s][v1]}, x[s]);
#pragma unroll
                        for (int a = 0; a < S * S; ++a) A[a] = f2{jA[r][a][v0], jA[r][a][v1]};
                        mat_t_vec2<S>(A, lam, x);  // mu_t
#pragma unroll
                        for (int n = 0; n < NS; ++n) se[n] = f2{sens[r][n][v0], sens[r][n][v1]};
                        Cell::grads2(se, lam, dp, da);
#pragma unroll
                        for (int g2 = 0; g2 < G; ++g2) {
                            outp[r][g2][v0] = dp[g2].x;
                            outp[r][g2][v1] = dp[g2].y;
                        }
                        if (rvalid) {
#pragma unroll
                            for (int g2 = 0; g2 < G; ++g2) {
                                dacc[g2] = add2(dacc[g2], da[g2]);
                                bad |= !isfinite(dp[g2].x) || !isfinite(dp[g2].y);
                            }
                        }
                        if (r == 0 && tb == 0 && rvalid && prm.dLdh0) {
                            // dL/dh0 = A_0^T lambda_0 = mu_0
#pragma unroll
                            for (int s = 0; s < S; ++s) {
                                prm.dLdh0[(b * S + s) * D + d0 + cc + v0] = x[s].x;
                                prm.dLdh0[(b * S + s) * D + d0 + cc + v1] = x[s].y;
                            }
                        }
                    }
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        da_acc[g][v0] = dacc[g].x;
                        da_acc[g][v1] = dacc[g].y;
                    }
                }
            } else {
#pragma unroll
                for (int v = 0; v < V; ++v) {
                    float x[S], cv[S];  // x = mu_{t+1}, the propagated adjoint after row t
#pragma unroll
                    for (int s = 0; s < S; ++s) cv[s] = sm.cin[s][cc + v];
                    apply<S>(pre.e[v].A, pre.e[v].b, cv, x);
#pragma unroll
                    for (int r = R - 1; r >= 0; --r) {
                        const bool rvalid = (tb + r < T) && cvalid;
                        float lam[S], A[S * S];
#pragma unroll
                        for (int s = 0; s < S; ++s) lam[s] = gr[r][s][v] + x[s];
#pragma unroll
                        for (int a = 0; a < S * S; ++a) A[a] = jA[r][a][v];
                        mat_t_vec<S>(A, lam, x);  // mu_t
                        float se[NS], dp[G], da[G];
#pragma unroll
                        for (int n = 0; n < NS; ++n) se[n] = sens[r][n][v];
                        Cell::grads(se, lam, dp, da);
#pragma unroll
                        for (int g2 = 0; g2 < G; ++g2) {
                            outp[r][g2][v] = dp[g2];
                            if (rvalid) {
                                da_acc[g2][v] += da[g2];
                                bad |= !isfinite(dp[g2]);
                            }
                        }
                        if (r == 0 && tb == 0 && rvalid && prm.dLdh0) {
                            // dL/dh0 = A_0^T lambda_0 = mu_0
#pragma unroll
                            for (int s = 0; s < S; ++s) prm.dLdh0[(b * S + s) * D + d0 + cc + v] = x[s];
                        }
                    }
                }
            }
            if constexpr (!(kPack && kRecompute)) {
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const int64_t t = tb + r;
                    if (t < T && cvalid) {
#pragma unroll
                        for (int g = 0; g < G; ++g)
                            store_out_row<V, BwdStreamHints<Cell>::value>(
                                prm.dLdpx + ((b * T + t) * G + g) * D + d0 + cc, outp[r][g]);
                    }
                }
            }
            if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(prm.lb.status, kStatusNonFinite);
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int v = 0; v < V; ++v) sm.da[it & 1][sub][g][cc + v] = da_acc[g][v];
        }
    }
    block_sync();  // the last tile's partials are in place
    if (is_scan && prev_tile >= 0) store_tile_partial<Sh, PxT>(sm, (it - 1) & 1, prm, prev_tile, lane);
}

// dL/da[g][d] = the sum, over batch rows b and tiles along time, of the
// per-tile partials.  One block per (channel group, gate), kReduceSplit warps:
// lane = channel (a warp reads one tile's 32 partials of a gate, 128 bytes,
// coalesced), warp j sums the tiles q = b * nChunks + pos with q = j mod
// kReduceSplit in increasing q, kReduceAhead loads in flight, and the block
// adds the warps' sums in warp order.  The order depends only on (B,
// nChunks), so the result is the same bits on every call and for every slice
// of channels of the same problem.
constexpr int kReduceSplit = 16;
constexpr int kReduceAhead = 8;

struct ReduceParams {
    const float* part;
    float* dLda;
    int64_t B, D, nCG, nChunks, nGroups;
    int G, W;
};

__global__ void __launch_bounds__(32 * kReduceSplit) reduce_da_kernel(const ReduceParams prm) {
    __shared__ float acc_w[kReduceSplit][32];
    const int64_t cg = blockIdx.x;
    const int g = blockIdx.y;
    const int lane = threadIdx.x & 31, j = threadIdx.x >> 5;
    const int64_t Q = prm.B * prm.nChunks;
    auto at = [&](int64_t q, int ch) {
        const int64_t b = q / prm.nChunks, pos = q - b * prm.nChunks;
        const int64_t tile = pos * prm.nGroups + b * prm.nCG + cg;
        return __ldg(prm.part + (tile * prm.G + g) * prm.W + ch);
    };
    // W is a multiple of 32: the block covers W / 32 runs of 32 channels
    for (int c0 = 0; c0 < prm.W; c0 += 32) {
        const int ch = c0 + lane;
        float acc = 0.0f;
        int64_t q = j;
        for (; q + (kReduceAhead - 1) * kReduceSplit < Q; q += kReduceAhead * kReduceSplit) {
            float v[kReduceAhead];
#pragma unroll
            for (int u = 0; u < kReduceAhead; ++u) v[u] = at(q + u * kReduceSplit, ch);
#pragma unroll
            for (int u = 0; u < kReduceAhead; ++u) acc += v[u];
        }
        for (; q < Q; q += kReduceSplit) acc += at(q, ch);
        acc_w[j][lane] = acc;
        __syncthreads();
        if (j == 0) {
            float sum = acc_w[0][lane];
#pragma unroll
            for (int k = 1; k < kReduceSplit; ++k) sum += acc_w[k][lane];
            const int64_t d = cg * prm.W + ch;
            if (d < prm.D) prm.dLda[g * prm.D + d] = sum;
        }
        __syncthreads();
    }
}

}  // namespace pararnn
