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
// Blocks are persistent and warp-specialised:
//   * NW compute warps own the rows.  Thread (warp w, lane l) holds V
//     consecutive channels of R consecutive steps (sub-chunk w*32/LC + l/LC).
//   * one scan warp takes tile tickets, issues the tensor-memory-accelerator
//     loads of the tiles ahead, and does each tile's decoupled look-back.
// Per Newton iteration of a tile:
//   1. compute warps evaluate f, A_t, beta_t on their rows, compose them,
//      and combine the sub-chunks of each warp with a shuffle scan;  [barrier]
//   2. the scan warp composes the warp totals into the tile's element,
//      publishes it, finds the carry by look-back over earlier tiles of the
//      same channels and publishes the state after the tile; meanwhile each
//      compute thread composes the totals of the warps before its own;
//                                                                    [barrier]
//   3. compute warps apply that prefix to the carry and re-walk their rows:
//      h^(k+1).
// The first row of a sub-chunk is linearised at the state just before it.
// For the warm start each thread evaluates f(0, x) on that row itself; after
// iteration k it is h^(k+1) just before the sub-chunk, which is the value the
// re-walk starts from (the prefix applied to the carry), so no state crosses
// between sub-chunks and two block barriers per iteration suffice.  The same
// value is also produced, rounded along a different path, as the last row of
// the sub-chunk before; the two agree to rounding.  HBM traffic is the
// minimum: pre-activations read once, h^(K) written once.
#pragma once

#include "cells.cuh"
#include "cluster.cuh"
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
    int picard;          // Picard sweeps before the Newton iterations (0..kPicardMax)
    int64_t nCG;         // channel groups per batch row
    int64_t nChunks;     // tiles along T
    int64_t nTiles;
    LookbackCtx lb;      // nGroups = B * nCG, nSlots = K
    // the small-problem (cluster) path: status flags tagged with the call
    // number, and the word that names the call the flags belong to
    unsigned long long* tagged_status;  // workspace header bytes 8..15
    unsigned* status_epoch;             // workspace header bytes 16..19
};

// Picard sweeps a forward call may ask for: each sweep reaches one row
// further back, so a thread evaluates up to kPicardMax + 1 rows before its
// own sub-chunk.
constexpr int kPicardMax = 4;

// V channels per thread, LC lanes across channels, NW compute warps, R rows
// per thread, MINB blocks per SM the register budget is sized for, NSTAGE
// shared-memory stages, TMA staging or a cooperative copy.
template <class Cell, typename PxT, int V_, int LC_, int NW_, int R_, int MINB_, int NSTAGE_, bool kTma_>
struct FwdShape {
    static constexpr int V = V_, LC = LC_, NWARPS = NW_, R = R_, MINB = MINB_, NSTAGE = NSTAGE_;
    static constexpr bool kTma = kTma_;
    static constexpr int G = Cell::G, S = Cell::S, NA = S * S + S;
    static constexpr int TPW = 32 / LC;           // sub-chunks per warp
    static constexpr int NSUB = NWARPS * TPW;     // sub-chunks per tile
    static constexpr int W = LC * V;              // channels per tile
    static constexpr int L = NSUB * R;            // time steps per tile
    static constexpr int NTC = NWARPS * 32;       // compute threads
    static constexpr int NT = NTC + 32;           // + the scan warp
    // forward stage rows: a nonlinear cell's tile also carries the row just
    // before it (the warm start there is the first row's previous state)
    static constexpr int ROW0 = Cell::kNonlinear ? 1 : 0;
    static constexpr int LF = L + ROW0;
    static constexpr uint32_t kStageBytes = LF * G * W * sizeof(PxT);
    static_assert(NSTAGE >= 2, "at least one stage in flight while another is used");
    static_assert(32 % LC == 0 && W % 32 == 0, "tile width must be a multiple of 32 channels");
    static_assert(!kTma || (W * sizeof(PxT)) % 16 == 0, "TMA box rows must be whole 16-byte units");
    static_assert(W <= 256 && L + 1 <= 256 && G <= 256, "TMA box dimensions are at most 256");
};

// the largest cluster the small-problem path launches (16 needs the
// non-portable cluster-size attribute), and the most Newton iterations it
// runs (each iteration has its own element buffer and mbarrier)
constexpr int kMaxClusterRanks = 16;
constexpr int kMaxClusterK = 8;

// One TMA destination: a tensor copy writes to a 128-byte aligned shared
// address, so every stage is padded to a multiple of 128 bytes.
template <class Sh, typename PxT>
struct alignas(128) FwdStage {
    PxT v[Sh::LF][Sh::G][Sh::W];  // row i is time t0 - ROW0 + i
};

template <class Sh, typename PxT>
struct FwdSmem {
    static_assert(sizeof(FwdStage<Sh, PxT>) % 128 == 0, "each TMA stage starts 128-byte aligned");
    FwdStage<Sh, PxT> px[Sh::NSTAGE];
    float wagg[Sh::NWARPS][Sh::NA][Sh::W];  // each compute warp's composed element
    float cin[Sh::S][Sh::W];                // the state just before the tile (current iterate)
    float w[Sh::NSTAGE][Sh::G][Sh::W];      // each stage's tile's recurrent weights
    float cagg[kMaxClusterK][Sh::NA][Sh::W];  // cluster path: this tile's element, per iteration
    uint64_t cbar[kMaxClusterK];              // cluster path: the predecessors' elements are ready
    uint64_t bar[Sh::NSTAGE];
    unsigned ticket[Sh::NSTAGE];
};

// The recurrent weights of the channels of tile `tile`, read by the scan
// warp (all 32 lanes, lane l holding channels l + 32 j) when it claims the
// tile, one tile ahead, and written to that tile's stage buffer: their
// global-memory latency is hidden behind the current tile instead of opening
// the next one (the forward of the long-sequence GRU 1.3 % faster; in the
// adjoint, whose evaluation phase is shorter, the scan warp's wait for them
// cost more than it saved).  The tile's channel group is tile mod nGroups.
template <int G, int W>
struct WeightsAhead {
    float v[G][W / 32];
    __device__ __forceinline__ void load(const float* w, int64_t tile, int64_t nGroups, int64_t nCG, int64_t D,
                                         int lane) {
        const int64_t gid = tile % nGroups;
        const int64_t d0 = (gid % nCG) * W;
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int j = 0; j < W / 32; ++j) {
                const int c = lane + 32 * j;
                v[g][j] = (w && d0 + c < D) ? __ldg(w + g * D + d0 + c) : 0.0f;
            }
    }
    __device__ __forceinline__ void store(float (&dst)[G][W], int lane) const {
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int j = 0; j < W / 32; ++j) dst[g][lane + 32 * j] = v[g][j];
    }
};

// The cluster path's carry for one Newton iteration (scan warp, between the
// "warp totals" and "carry" block barriers).  The tiles of one channel group
// along T are the CTAs of one cluster, rank = position along T.  Each
// composes its warp totals into its tile's element (this iteration's own
// buffer), makes it visible at cluster scope and arrives on this
// iteration's mbarrier in every later tile's CTA; it then waits (bounded)
// until the tiles before it have all arrived on its own, reads their
// elements from their shared memory and applies them, in order, to the
// first carry: the same operations, in the same order, as the look-back's
// chain of inclusive states, so the carry has the same bits.  Only scan
// warps take part: the compute warps never wait on another CTA.  Returns
// false if the wait ran out of time (the carry is then not valid).
template <class Sh>
__device__ __forceinline__ bool cluster_carry(const float (&wagg)[Sh::NWARPS][Sh::NA][Sh::W],
                                              float (&cagg)[Sh::NA][Sh::W], uint64_t* cbar,
                                              const float (&first_carry)[Sh::W / 32][Sh::S], uint32_t rank,
                                              uint32_t nranks, int lane, float (&cin)[Sh::S][Sh::W],
                                              uint64_t timeout_ns) {
    constexpr int S = Sh::S, NA = Sh::NA, W = Sh::W, CPL = W / 32;
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
        Elem<S> tot;
        elem_identity<S>(tot);
#pragma unroll
        for (int k = 0; k < Sh::NWARPS; ++k) {
            float A[S * S], b[S];
#pragma unroll
            for (int a = 0; a < S * S; ++a) A[a] = wagg[k][a][lane + 32 * j];
#pragma unroll
            for (int s = 0; s < S; ++s) b[s] = wagg[k][S * S + s][lane + 32 * j];
            compose_after<S>(A, b, tot);
        }
#pragma unroll
        for (int a = 0; a < S * S; ++a) cagg[a][lane + 32 * j] = tot.A[a];
#pragma unroll
        for (int s = 0; s < S; ++s) cagg[S * S + s][lane + 32 * j] = tot.b[s];
    }
    // every lane's element words ordered before any lane's arrive
    fence_acq_rel_cluster();
    __syncwarp();
    for (uint32_t r = rank + 1 + lane; r < nranks; r += 32) mbar_arrive_remote(cbar, r);
    bool ok = true;
    if (rank > 0) {
        Deadline dl;
        while (!mbar_try_wait_cluster(cbar, 0)) {
            if (dl.expired(timeout_ns)) {
                ok = false;
                break;
            }
        }
    }
    // the predecessors' elements are loaded in batches (every remote load of
    // a batch in flight at once: all of them for a scalar state, whose
    // elements are two words), then applied in order
    constexpr int NB = S == 1 ? kMaxClusterRanks : 4;
    static_assert(kMaxClusterRanks % NB == 0, "whole batches of cluster ranks");
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
        float x[S];
#pragma unroll
        for (int s = 0; s < S; ++s) x[s] = first_carry[j][s];
#pragma unroll
        for (uint32_t i0 = 0; i0 < (uint32_t)kMaxClusterRanks; i0 += NB) {
            if (i0 >= rank) break;
            float e[NB][NA];
#pragma unroll
            for (int m = 0; m < NB; ++m)
                if (i0 + m < rank) {
#pragma unroll
                    for (int a = 0; a < NA; ++a) e[m][a] = ld_dsmem(&cagg[a][lane + 32 * j], i0 + m);
                }
#pragma unroll
            for (int m = 0; m < NB; ++m)
                if (i0 + m < rank) {
                    float A[S * S], b[S], y[S];
#pragma unroll
                    for (int a = 0; a < S * S; ++a) A[a] = e[m][a];
#pragma unroll
                    for (int s = 0; s < S; ++s) b[s] = e[m][S * S + s];
                    apply<S>(A, b, x, y);
#pragma unroll
                    for (int s = 0; s < S; ++s) x[s] = y[s];
                }
        }
#pragma unroll
        for (int s = 0; s < S; ++s) cin[s][lane + 32 * j] = x[s];
    }
    return ok;
}

template <class Cell, typename PxT, class Sh>
__device__ __forceinline__ void issue_tile_load(const CUtensorMap* map, FwdSmem<Sh, PxT>& sm, const FwdParams& prm,
                                                unsigned tile, int stage) {
    const int64_t chunk = tile / prm.lb.nGroups;
    const int64_t gid = tile - chunk * prm.lb.nGroups;
    const int64_t b = gid / prm.nCG;
    const int64_t d0 = (gid - b * prm.nCG) * Sh::W;
    mbar_arrive_expect_tx(&sm.bar[stage], Sh::kStageBytes);
    // the row coordinate may be -1 (first tile of the first batch row): TMA fills zeros there
    tma_load_3d(&sm.px[stage].v[0][0][0], map, &sm.bar[stage], (int)d0, 0,
                (int)(b * prm.T + chunk * Sh::L) - Sh::ROW0);
}

// kCluster: the small-problem path.  Every tile is its own CTA, launched in
// clusters of nChunks CTAs (one channel group of one batch row, all along T);
// the carries pass through distributed shared memory (cluster_carry), so
// there is no ticket counter, no look-back and nothing in the workspace but
// the tagged status word.
template <class Cell, typename PxT, class Sh, bool kLean, bool kPicard = false, bool kCluster = false>
__global__ void __launch_bounds__(Sh::NT, Sh::MINB)
    newton_fwd_kernel(const __grid_constant__ CUtensorMap tmap, const FwdParams prm) {
    constexpr int G = Sh::G, S = Sh::S, V = Sh::V, R = Sh::R, NW = Sh::NWARPS, NSTAGE = Sh::NSTAGE;
    constexpr int TPW = Sh::TPW, W = Sh::W, L = Sh::L, LC = Sh::LC, NTC = Sh::NTC;
    constexpr int CPL = W / 32;
    using SM = FwdSmem<Sh, PxT>;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    SM& sm = *reinterpret_cast<SM*>(smem_raw);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if constexpr (kCluster) {
        // Programmatic dependent launch (the cluster path is launched with
        // it): let the stream's next kernel be launched now, so that its
        // launch overlaps this one, and wait until the stream's previous
        // kernel has finished and its writes are visible before reading or
        // writing global memory.  Without the launch attribute both are
        // no-ops.
        asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
        asm volatile("griddepcontrol.wait;" ::: "memory");
    }
    const bool is_scan = warp == NW;
    const int64_t T = prm.T, D = prm.D;
    const PxT* pxg = static_cast<const PxT*>(prm.px);
    const bool need_prev = Cell::kNonlinear || prm.resid != nullptr;
    auto report = [&](unsigned bit) {
        if constexpr (kCluster)
            set_tagged_status(prm.tagged_status, prm.lb.epoch, bit);
        else
            atomicOr(prm.lb.status, bit);
    };

    // prologue (scan warp): claim the first NSTAGE-1 tiles and start streaming them in
    if (is_scan && lane == 0) {
        if constexpr (Sh::kTma) {
#pragma unroll
            for (int s = 0; s < NSTAGE; ++s) mbar_init(&sm.bar[s], 1);
            mbar_fence_init();
        }
        if constexpr (kCluster) {
            // one tile per CTA: blockIdx.x = group * nChunks + position along T
            const int64_t gid = blockIdx.x / prm.nChunks;
            const unsigned t = (unsigned)((int64_t)cluster_ctarank() * prm.lb.nGroups + gid);
            sm.ticket[0] = t;
#pragma unroll
            for (int s = 1; s < NSTAGE; ++s) sm.ticket[s] = (unsigned)prm.nTiles;
            if constexpr (Sh::kTma) issue_tile_load<Cell, PxT, Sh>(&tmap, sm, prm, t, 0);
            if (blockIdx.x == 0) *prm.status_epoch = prm.lb.epoch;  // the flags of this call are the valid ones
            // one mbarrier per Newton iteration, completed by the arrivals of
            // every tile before this one (none for the first)
            const uint32_t rank = cluster_ctarank();
            if (rank > 0) {
                const int nk = kLean ? 1 : prm.K;
                for (int k = 0; k < nk; ++k) mbar_init(&sm.cbar[k], rank);
            }
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        } else {
#pragma unroll
            for (int s = 0; s < NSTAGE - 1; ++s) {
                const unsigned t = atomicAdd(prm.ticket, 1u);
                sm.ticket[s] = t;
                if constexpr (Sh::kTma)
                    if (t < prm.nTiles) issue_tile_load<Cell, PxT, Sh>(&tmap, sm, prm, t, s);
            }
        }
    }
    if (is_scan && !kLean) {
        // the first tiles' weights (read by the compute warps after their
        // set-up barrier; the lean linear scan reads none)
        __syncwarp();
#pragma unroll
        for (int s = 0; s < NSTAGE - 1; ++s) {
            const unsigned t = sm.ticket[s];
            if (t < prm.nTiles) {
                WeightsAhead<G, W> wa;
                wa.load(prm.w, t, prm.lb.nGroups, prm.nCG, D, lane);
                wa.store(sm.w[s], lane);
            }
        }
    }
    block_sync();
    if constexpr (kCluster) {
        // every CTA's mbarriers are initialised before any CTA arrives on them
        cluster_arrive_release();
        cluster_wait_acquire();
    }

    for (int it = 0;; ++it) {
        const int st = it % NSTAGE;
        const unsigned tile_u = sm.ticket[st];
        if (tile_u >= prm.nTiles) break;
        const int64_t tile = tile_u;
        const int64_t chunk = tile / prm.lb.nGroups;
        const int64_t gid = tile - chunk * prm.lb.nGroups;
        const int64_t b = gid / prm.nCG;
        const int64_t d0 = (gid - b * prm.nCG) * W;
        const int64_t t0 = chunk * L;

        if (is_scan) {
            // ================= scan warp =================
            float first_carry[CPL][S];  // h_{-1} = h0 for every iterate
#pragma unroll
            for (int j = 0; j < CPL; ++j)
#pragma unroll
                for (int s = 0; s < S; ++s) {
                    const int64_t d = d0 + lane + 32 * j;
                    first_carry[j][s] = (prm.h0 && d < D) ? prm.h0[(b * S + s) * D + d] : 0.0f;
                }
            // early probe of the predecessor: only where a long evaluation
            // phase hides its round trip (the Newton iterations of a
            // nonlinear cell); elsewhere a probe that misses costs more than
            // it saves
            Probe<S, W> pr;
            pr.st = 0;
            if constexpr (!kLean && !kCluster) probe_issue<S, W>(prm.lb, tile, chunk, 0, lane, pr);
            block_sync();  // tile set up
            if constexpr (kCluster) {
                if (lane == 0) sm.ticket[(it + NSTAGE - 1) % NSTAGE] = (unsigned)prm.nTiles;  // no further tile
            } else if (lane == 0) {
                // claim the tile NSTAGE-1 ahead and start streaming it in; its
                // stage was last read by the previous tile, whose readers have
                // all passed this tile's set-up barrier
                const int sn = (it + NSTAGE - 1) % NSTAGE;
                const unsigned prev_t = sm.ticket[(it + NSTAGE - 2) % NSTAGE];
                unsigned t2 = prev_t;
                if (prev_t < prm.nTiles) t2 = atomicAdd(prm.ticket, 1u);
                sm.ticket[sn] = t2;
                if constexpr (Sh::kTma)
                    if (t2 < prm.nTiles && prev_t < prm.nTiles) issue_tile_load<Cell, PxT, Sh>(&tmap, sm, prm, t2, sn);
            }
            // the claimed tile's weights, into its stage (whose previous
            // readers have passed this tile's set-up barrier); the scan warp
            // waits for them here, while the compute warps evaluate
            if constexpr (!kCluster && !kLean) {
                const int sn = (it + NSTAGE - 1) % NSTAGE;
                const unsigned t2 = __shfl_sync(0xffffffffu, sm.ticket[sn], 0);
                const unsigned prev_t = sm.ticket[(it + NSTAGE - 2) % NSTAGE];
                if (t2 < prm.nTiles && prev_t < prm.nTiles) {
                    WeightsAhead<G, W> wa;
                    wa.load(prm.w, t2, prm.lb.nGroups, prm.nCG, D, lane);
                    wa.store(sm.w[sn], lane);
                }
            }
            Inclusive<S, W> inc;
            if constexpr (kCluster) {
                const int K = kLean ? 1 : prm.K;
                for (int k = 0; k < K; ++k) {
                    block_sync();  // warp totals ready
                    const bool ok = cluster_carry<Sh>(sm.wagg, sm.cagg[k], &sm.cbar[k], first_carry, (uint32_t)chunk,
                                                      (uint32_t)prm.nChunks, lane, sm.cin, prm.lb.timeout_ns);
                    if (!__all_sync(0xffffffffu, ok) && lane == 0) report(kStatusTimeout);
                    block_sync();  // carry ready
                }
            } else if constexpr (kLean) {
                block_sync();  // warp totals ready
                tile_lookback<S, W, NW, false>(prm.lb, tile, chunk, 0, lane, sm.wagg, first_carry, pr, sm.cin, inc);
                block_sync();  // carry ready
                publish_inclusive<S, W>(prm.lb, tile, 0, lane, inc);
            } else {
                const int K = prm.K;
                for (int k = 0; k < K; ++k) {
                    if (k > 0) probe_issue<S, W>(prm.lb, tile, chunk, k, lane, pr);
                    block_sync();  // warp totals ready
                    tile_lookback<S, W, NW, false>(prm.lb, tile, chunk, k, lane, sm.wagg, first_carry, pr, sm.cin, inc);
                    block_sync();  // carry ready
                    publish_inclusive<S, W>(prm.lb, tile, k, lane, inc);
                }
            }
        } else {
            // ================= compute warps =================
            const int sub = warp * TPW + lane / LC;
            const int cc = (lane % LC) * V;
            const int64_t tb = t0 + (int64_t)sub * R;
            const bool cvalid = d0 + cc < D;  // D is a multiple of V: a vector is wholly in or out

            // the tile's pre-activations: TMA (already in flight) or a cooperative copy
            if constexpr (Sh::kTma) {
                Deadline dl;
                while (!mbar_try_wait(&sm.bar[st], (it / NSTAGE) & 1)) {
                    if (dl.expired(prm.lb.timeout_ns)) {
                        if (tid == 0) report(kStatusTimeout);
                        break;
                    }
                }
            } else {
                for (int i = tid; i < Sh::LF * G * W; i += NTC) {
                    const int row = i / (G * W), rem = i - row * (G * W), g = rem / W, c = rem - g * W;
                    const int64_t t = t0 - Sh::ROW0 + row, d = d0 + c;
                    sm.px[st].v[row][g][c] = (t >= 0 && t < T && d < D) ? pxg[((b * T + t) * G + g) * D + d] : PxT(0.0f);
                }
            }
            block_sync();  // tile set up
            // pre-activations of row r of this thread, V channels per gate
            auto load_p = [&](int r, float (&pv)[G][V]) {
#pragma unroll
                for (int g = 0; g < G; ++g) lds_row<V>(&sm.px[st].v[Sh::ROW0 + sub * R + r][g][cc], pv[g]);
            };

            if constexpr (kLean) {
                // ---- the linear cell without a residual: one scan, elements straight from shared memory ----
                ElemV<S, V> mine, excl, pre;
#pragma unroll
                for (int v = 0; v < V; ++v) elem_identity<S>(mine.e[v]);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    if (tb + r < T) {
                        float pv[G][V];
                        load_p(r, pv);
#pragma unroll
                        for (int v = 0; v < V; ++v) {
                            float A[1] = {pv[0][v]}, be[1] = {pv[1][v]};
                            compose_after<S>(A, be, mine.e[v]);
                        }
                    }
                }
                warp_prefix<S, V, LC, W, NW, false>(mine, excl, warp, lane, sm.wagg);
                block_sync();  // warp totals ready
                sub_prefix<S, V, LC, W, NW, false>(excl, warp, lane, sm.wagg, pre);
                block_sync();  // carry ready
                float x[V];
#pragma unroll
                for (int v = 0; v < V; ++v) x[v] = __fmaf_rn(pre.e[v].A[0], sm.cin[0][cc + v], pre.e[v].b[0]);
                bool bad = false;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    float pv[G][V], out[V];
                    load_p(r, pv);
#pragma unroll
                    for (int v = 0; v < V; ++v) {
                        x[v] = __fmaf_rn(pv[0][v], x[v], pv[1][v]);
                        out[v] = x[v];
                    }
                    const int64_t t = tb + r;
                    if (t < T && cvalid) {
#pragma unroll
                        for (int v = 0; v < V; ++v) bad |= !isfinite(out[v]);
                        store_row<V>(prm.H + (b * T + t) * D + d0 + cc, out);
                    }
                }
                if (__any_sync(0xffffffffu, bad) && lane == 0) report(kStatusNonFinite);
            } else {
                // ---- general path: warm start, K Newton iterations ----
                const bool want_resid = prm.resid != nullptr;
                float wr[V][G];  // the recurrent weights of this thread's channels
#pragma unroll
                for (int v = 0; v < V; ++v)
#pragma unroll
                    for (int g = 0; g < G; ++g) wr[v][g] = sm.w[st][g][cc + v];
                // two channels per instruction where the thread holds an even
                // number of them (packed f32x2; same rounding as one by one)
                constexpr bool kPack = (V % 2 == 0) && Cell::kNonlinear;
                constexpr int VP = kPack ? V / 2 : 1;
                // f(0, x) for V channels of one row, pairwise where packed
                auto warm_row = [&](const float (&pv)[G][V], float (&out)[S][V]) {
                    if constexpr (kPack) {
#pragma unroll
                        for (int q = 0; q < VP; ++q) {
                            f2 pg[G], f[S];
#pragma unroll
                            for (int g = 0; g < G; ++g) pg[g] = f2{pv[g][2 * q], pv[g][2 * q + 1]};
                            Cell::warm2(pg, f);
#pragma unroll
                            for (int s = 0; s < S; ++s) {
                                out[s][2 * q] = f[s].x;
                                out[s][2 * q + 1] = f[s].y;
                            }
                        }
                    } else {
#pragma unroll
                        for (int v = 0; v < V; ++v) {
                            float pg[G], f[S];
#pragma unroll
                            for (int g = 0; g < G; ++g) pg[g] = pv[g][v];
                            Cell::warm(pg, wr[v], f);
#pragma unroll
                            for (int s = 0; s < S; ++s) out[s][v] = f[s];
                        }
                    }
                };
                float h[R][S][V];
                if constexpr (!kPicard) {
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        float pv[G][V];
                        load_p(r, pv);
                        warm_row(pv, h[r]);
                    }
                }
                // h^(0) just before the sub-chunk: h0 at the start of a row,
                // else the warm start of the row before (in the stage, except
                // for the linear cell's first sub-chunk)
                float hin[S][V];
#pragma unroll
                for (int s = 0; s < S; ++s)
#pragma unroll
                    for (int v = 0; v < V; ++v) hin[s][v] = 0.0f;
                if constexpr (kPicard) {
                    // Picard sweeps h^(p+1)_t = f(h^(p)_{t-1}, x_t) from the
                    // warm start, on this thread's rows and the P + 1 rows
                    // before them (row j of the window is time tb + j); sweep p
                    // is valid from row -(P+1) + p on, so after P sweeps rows
                    // -1 .. R-1 hold h^(P).  Every thread forms the rows it
                    // shares with its neighbours by the same arithmetic from
                    // the same inputs, so the copies agree bit for bit.
                    constexpr int NWIN = R + kPicardMax + 1;  // window rows j = -(kPicardMax+1) .. R-1
                    constexpr int J0 = kPicardMax + 1;        // window index of row j is j + J0
                    const int P = prm.picard;
                    float win[NWIN][S][V];
                    float h0v[S][V];
#pragma unroll
                    for (int s = 0; s < S; ++s)
#pragma unroll
                        for (int v = 0; v < V; ++v)
                            h0v[s][v] = (prm.h0 && cvalid) ? prm.h0[(b * S + s) * D + d0 + cc + v] : 0.0f;
                    // pre-activations of window row j: the stage holds rows from
                    // t0 - ROW0 on; rows before it come from global memory
                    auto load_pw = [&](int j, float (&pv)[G][V]) {
                        const int srow = Sh::ROW0 + sub * R + j;
                        const int64_t t = tb + j;
                        if (srow >= 0) {
#pragma unroll
                            for (int g = 0; g < G; ++g) lds_row<V>(&sm.px[st].v[srow][g][cc], pv[g]);
                        } else {
#pragma unroll
                            for (int g = 0; g < G; ++g)
#pragma unroll
                                for (int v = 0; v < V; ++v)
                                    pv[g][v] = (t >= 0 && cvalid)
                                                   ? PxTraits<PxT>::cvt(pxg[((b * T + t) * G + g) * D + d0 + cc + v])
                                                   : 0.0f;
                        }
                    };
#pragma unroll
                    for (int jj = 0; jj < NWIN; ++jj) {
                        const int j = jj - J0;
                        if (j < -(P + 1)) continue;
                        float pv[G][V];
                        load_pw(j, pv);
#pragma unroll
                        for (int v = 0; v < V; ++v) {
                            float pg[G], f[S];
#pragma unroll
                            for (int g = 0; g < G; ++g) pg[g] = pv[g][v];
                            Cell::warm(pg, wr[v], f);
#pragma unroll
                            for (int s = 0; s < S; ++s) win[jj][s][v] = (tb + j >= 0) ? f[s] : h0v[s][v];
                        }
                    }
                    for (int p = 1; p <= P; ++p) {
                        // rows from the last back, so row j-1 still holds sweep p-1
#pragma unroll
                        for (int jj = NWIN - 1; jj >= 1; --jj) {
                            const int j = jj - J0;
                            if (j < -(P + 1) + p || tb + j < 0) continue;
                            float pv[G][V];
                            load_pw(j, pv);
#pragma unroll
                            for (int v = 0; v < V; ++v) {
                                float pg[G], spv[S], f[S], A[S * S], be[S];
#pragma unroll
                                for (int g = 0; g < G; ++g) pg[g] = pv[g][v];
#pragma unroll
                                for (int s = 0; s < S; ++s) spv[s] = (tb + j - 1 >= 0) ? win[jj - 1][s][v] : h0v[s][v];
                                Cell::elem(pg, wr[v], spv, f, A, be);
#pragma unroll
                                for (int s = 0; s < S; ++s) win[jj][s][v] = f[s];
                            }
                        }
                    }
#pragma unroll
                    for (int r = 0; r < R; ++r)
#pragma unroll
                        for (int s = 0; s < S; ++s)
#pragma unroll
                            for (int v = 0; v < V; ++v) h[r][s][v] = win[J0 + r][s][v];
#pragma unroll
                    for (int s = 0; s < S; ++s)
#pragma unroll
                        for (int v = 0; v < V; ++v) hin[s][v] = cvalid ? win[J0 - 1][s][v] : 0.0f;
                } else if (need_prev && cvalid) {
                    if (tb == 0) {
                        if (prm.h0)
#pragma unroll
                            for (int s = 0; s < S; ++s)
#pragma unroll
                                for (int v = 0; v < V; ++v) hin[s][v] = prm.h0[(b * S + s) * D + d0 + cc + v];
                    } else {
                        float pv[G][V];
                        if (Sh::ROW0 + sub * R - 1 >= 0) {
#pragma unroll
                            for (int g = 0; g < G; ++g) lds_row<V>(&sm.px[st].v[Sh::ROW0 + sub * R - 1][g][cc], pv[g]);
                        } else {
#pragma unroll
                            for (int g = 0; g < G; ++g)
#pragma unroll
                                for (int v = 0; v < V; ++v)
                                    pv[g][v] = PxTraits<PxT>::cvt(pxg[((b * T + tb - 1) * G + g) * D + d0 + cc + v]);
                        }
                        warm_row(pv, hin);
                    }
                }
                const int K = prm.K;
                typename Cell::W2 wp[VP];
                if constexpr (kPack) {
#pragma unroll
                    for (int q = 0; q < VP; ++q) wp[q] = Cell::weights2(wr[2 * q], wr[2 * q + 1]);
                }
                for (int k = 0; k <= K; ++k) {
                    // ---- 1. elements of iteration k+1 and the residual of iterate k ----
                    float sp[S][V];
#pragma unroll
                    for (int s = 0; s < S; ++s)
#pragma unroll
                        for (int v = 0; v < V; ++v) sp[s][v] = hin[s][v];
                    float eA[R][S * S][V], eb[R][S][V];
                    float res = 0.0f;
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const bool rvalid = (tb + r < T) && cvalid;
                        float pv[G][V];
                        load_p(r, pv);
                        // rows past the end of the sequence (and channels
                        // past D) keep their elements: in time order they
                        // come after every valid row of their channel, so
                        // they reach only scan values nobody reads (the
                        // sequence's last inclusive state and h rows that
                        // are never stored); their pre-activations are
                        // zero-filled, so the values stay finite
                        if constexpr (kPack) {
#pragma unroll
                            for (int q = 0; q < VP; ++q) {
                                const int v0 = 2 * q, v1 = 2 * q + 1;
                                f2 pg[G], spv[S], f[S], A[S * S], be[S];
#pragma unroll
                                for (int g = 0; g < G; ++g) pg[g] = f2{pv[g][v0], pv[g][v1]};
#pragma unroll
                                for (int s = 0; s < S; ++s) spv[s] = f2{sp[s][v0], sp[s][v1]};
                                Cell::elem2(pg, wp[q], spv, f, A, be);
                                if (rvalid && want_resid) {
#pragma unroll
                                    for (int s = 0; s < S; ++s) {
                                        res = nanmax_f(res, fabsf(h[r][s][v0] - f[s].x));
                                        res = nanmax_f(res, fabsf(h[r][s][v1] - f[s].y));
                                    }
                                }
#pragma unroll
                                for (int a = 0; a < S * S; ++a) {
                                    eA[r][a][v0] = A[a].x;
                                    eA[r][a][v1] = A[a].y;
                                }
#pragma unroll
                                for (int s = 0; s < S; ++s) {
                                    eb[r][s][v0] = be[s].x;
                                    eb[r][s][v1] = be[s].y;
                                    sp[s][v0] = h[r][s][v0];
                                    sp[s][v1] = h[r][s][v1];
                                }
                            }
                        } else {
#pragma unroll
                            for (int v = 0; v < V; ++v) {
                                float pg[G], spv[S], f[S], A[S * S], be[S];
#pragma unroll
                                for (int g = 0; g < G; ++g) pg[g] = pv[g][v];
#pragma unroll
                                for (int s = 0; s < S; ++s) spv[s] = sp[s][v];
                                Cell::elem(pg, wr[v], spv, f, A, be);
                                if (rvalid && want_resid) {
#pragma unroll
                                    for (int s = 0; s < S; ++s) res = nanmax_f(res, fabsf(h[r][s][v] - f[s]));
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
                    }
                    if (prm.resid) {
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) res = nanmax_f(res, __shfl_xor_sync(0xffffffffu, res, o));
                        if (lane == 0) atomic_max_nonneg(prm.resid + k, res);
                    }
                    if (k == K) break;  // the last pass only measured the residual of h^(K)
                    ElemV<S, V> mine, excl, pre;
                    if constexpr (kPack) {
#pragma unroll
                        for (int q = 0; q < VP; ++q) {
                            const int v0 = 2 * q, v1 = 2 * q + 1;
                            f2 accA[S * S], accb[S];
#pragma unroll
                            for (int a = 0; a < S * S; ++a) accA[a] = splat2((a % (S + 1) == 0) ? 1.0f : 0.0f);
#pragma unroll
                            for (int s = 0; s < S; ++s) accb[s] = splat2(0.0f);
#pragma unroll
                            for (int r = 0; r < R; ++r) {
                                f2 A[S * S], be[S];
#pragma unroll
                                for (int a = 0; a < S * S; ++a) A[a] = f2{eA[r][a][v0], eA[r][a][v1]};
#pragma unroll
                                for (int s = 0; s < S; ++s) be[s] = f2{eb[r][s][v0], eb[r][s][v1]};
                                compose_after2<S>(A, be, accA, accb);
                            }
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
                            elem_identity<S>(mine.e[v]);
#pragma unroll
                            for (int r = 0; r < R; ++r) {
                                float A[S * S], be[S];
#pragma unroll
                                for (int a = 0; a < S * S; ++a) A[a] = eA[r][a][v];
#pragma unroll
                                for (int s = 0; s < S; ++s) be[s] = eb[r][s][v];
                                compose_after<S>(A, be, mine.e[v]);
                            }
                        }
                    }
                    warp_prefix<S, V, LC, W, NW, false>(mine, excl, warp, lane, sm.wagg);
                    block_sync();  // warp totals ready
                        // ---- 2. prefix of the earlier warps (the scan warp finds the carry meanwhile) ----
                    sub_prefix<S, V, LC, W, NW, false>(excl, warp, lane, sm.wagg, pre);
                        block_sync();  // carry ready
                    // ---- 3. re-walk the rows from the carry-in: h^(k+1) ----
                    if constexpr (kPack) {
#pragma unroll
                        for (int q = 0; q < VP; ++q) {
                            const int v0 = 2 * q, v1 = 2 * q + 1;
                            f2 x[S], cv[S], PA[S * S], Pb[S];
#pragma unroll
                            for (int s = 0; s < S; ++s) cv[s] = f2{sm.cin[s][cc + v0], sm.cin[s][cc + v1]};
#pragma unroll
                            for (int a = 0; a < S * S; ++a) PA[a] = f2{pre.e[v0].A[a], pre.e[v1].A[a]};
#pragma unroll
                            for (int s = 0; s < S; ++s) Pb[s] = f2{pre.e[v0].b[s], pre.e[v1].b[s]};
                            apply2<S>(PA, Pb, cv, x);
#pragma unroll
                            for (int s = 0; s < S; ++s) {
                                hin[s][v0] = x[s].x;  // h^(k+1) just before the sub-chunk
                                hin[s][v1] = x[s].y;
                            }
#pragma unroll
                            for (int r = 0; r < R; ++r) {
                                f2 A[S * S], be[S], y[S];
#pragma unroll
                                for (int a = 0; a < S * S; ++a) A[a] = f2{eA[r][a][v0], eA[r][a][v1]};
#pragma unroll
                                for (int s = 0; s < S; ++s) be[s] = f2{eb[r][s][v0], eb[r][s][v1]};
                                apply2<S>(A, be, x, y);
#pragma unroll
                                for (int s = 0; s < S; ++s) {
                                    x[s] = y[s];
                                    h[r][s][v0] = y[s].x;
                                    h[r][s][v1] = y[s].y;
                                }
                            }
                        }
                    } else {
#pragma unroll
                        for (int v = 0; v < V; ++v) {
                            float x[S], cv[S];
#pragma unroll
                            for (int s = 0; s < S; ++s) cv[s] = sm.cin[s][cc + v];
                            apply<S>(pre.e[v].A, pre.e[v].b, cv, x);
#pragma unroll
                            for (int s = 0; s < S; ++s) hin[s][v] = x[s];  // h^(k+1) just before the sub-chunk
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
                if (__any_sync(0xffffffffu, bad) && lane == 0) report(kStatusNonFinite);
            }
        }
        // No barrier here: the next tile's barrier (tile set up) comes before
        // its scan warp refills a stage or rewrites a ticket slot, and every
        // other shared array is rewritten only after a barrier that all of
        // this tile's readers have passed.
    }
    if constexpr (kCluster) {
        // no CTA leaves while another may still read its shared memory
        cluster_arrive_release();
        cluster_wait_acquire();
    }
}

}  // namespace pararnn
