// lookback.cuh -- decoupled look-back between the tiles of one channel group.
//
// Tiles are numbered by a ticket taken at block start (an atomic counter), in
// scan order: ticket = position_along_the_scan * nGroups + group.  A tile
// therefore waits only on tiles whose tickets were taken earlier, by blocks
// that are already running, so every wait ends (forward progress does not
// depend on the order in which the hardware schedules blocks).
//
// Per (tile, slot) -- slot = Newton iteration in the forward, 0 in the
// backward -- the workspace holds one flag and two payloads, W channels wide:
//   aggregate  the tile's composed scan element (A: S x S, b: S)   [flag 1]
//   inclusive  the state after the tile's last row                  [flag 2]
// The carry into a tile is found by walking back to the nearest predecessor
// with an inclusive value and applying the aggregates in between, in order,
// to it.  Because an inclusive value is itself formed as
// apply(aggregate, carry), the carry comes out bit-identical whichever
// predecessors had already finished: results do not depend on timing.
#pragma once

#include "cells.cuh"
#include "common.cuh"

namespace pararnn {

struct LookbackCtx {
    unsigned* status;
    unsigned* flags;     // [nTiles][nSlots]
    float* agg;          // [nTiles][nSlots][NA][W]
    float* inc;          // [nTiles][nSlots][S][W]
    int64_t nGroups;
    int nSlots;
    uint64_t timeout_ns;
};

// Bounded wait for a flag to reach `want` (or more).  Returns false if the
// time limit passed first; the caller records the time-out and carries on, so
// that the kernel always finishes.
__device__ __forceinline__ bool wait_flag(const unsigned* flag, unsigned want, uint64_t timeout_ns, unsigned& seen) {
    seen = ld_acquire_gpu(flag);
    if (seen >= want) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        __nanosleep(64);
        seen = ld_acquire_gpu(flag);
        if (seen >= want) return true;
        if (globaltimer_ns() - t0 > timeout_ns) return false;
    }
}

// Publish one payload row set and then the flag.  Called by all 32 lanes of
// one warp; lane l owns channels l, l+32, ... of the tile.
template <int N, int W>
__device__ __forceinline__ void publish(float* dst, const float (&vals)[W / 32][N], unsigned* flag, unsigned flag_value,
                                        int lane) {
#pragma unroll
    for (int j = 0; j < W / 32; ++j)
#pragma unroll
        for (int n = 0; n < N; ++n) dst[n * W + lane + 32 * j] = vals[j][n];
    __threadfence();
    __syncwarp();
    if (lane == 0) st_release_gpu(flag, flag_value);
}

// Carry into `tile` for scan slot `slot`: the state just before the tile's
// first row.  `dist_max` = number of predecessors (the tile's position along
// the scan).  Called by all 32 lanes of one warp.
template <int S, int W>
__device__ void lookback_carry(const LookbackCtx& cx, int64_t tile, int64_t dist_max, int slot, int lane,
                               float (&carry)[W / 32][S]) {
    constexpr int NA = S * S + S;
    constexpr int CPL = W / 32;
    // 1. find the nearest predecessor with an inclusive value; lanes read the
    //    flags of 32 predecessors at once
    int64_t base = 1, found = -1;
    uint64_t t_start = 0;
    bool timed_out = false;
    while (true) {
        const int64_t j = base + lane;
        unsigned f = kFlagAggregate;
        if (j <= dist_max) f = ld_acquire_gpu(cx.flags + (tile - j * cx.nGroups) * cx.nSlots + slot);
        const unsigned inc_mask = __ballot_sync(0xffffffffu, j <= dist_max && f == kFlagInclusive);
        const unsigned empty_mask = __ballot_sync(0xffffffffu, j <= dist_max && f == kFlagEmpty);
        if (inc_mask) {
            const int first = __ffs(inc_mask) - 1;
            const unsigned before = first ? (empty_mask & ((1u << first) - 1u)) : 0u;
            if (!before) {
                found = base + first;
                break;
            }
        } else if (!empty_mask) {
            base += 32;  // 32 aggregates in a row: look further back
            if (base <= dist_max) continue;
            // the first tile of the scan publishes only an inclusive value, so
            // this is unreachable unless the workspace was overwritten
            timed_out = true;
            break;
        }
        if (t_start == 0) {
            t_start = globaltimer_ns() | 1;
        } else if (globaltimer_ns() - t_start > cx.timeout_ns) {
            timed_out = true;
            break;
        }
        __nanosleep(64);
    }
    __syncwarp();
    if (timed_out) {
        if (lane == 0) atomicOr(cx.status, kStatusTimeout);
#pragma unroll
        for (int j = 0; j < CPL; ++j)
#pragma unroll
            for (int s = 0; s < S; ++s) carry[j][s] = 0.0f;
        return;
    }
    // 2. x = inclusive(found), then apply the aggregates of predecessors
    //    found-1, ..., 1 in that order; loads are issued in batches so that
    //    several L2 round trips overlap
    constexpr int BATCH = 4;
    float x[CPL][S];
    {
        const float* ip = cx.inc + ((tile - found * cx.nGroups) * cx.nSlots + slot) * S * W;
#pragma unroll
        for (int j = 0; j < CPL; ++j)
#pragma unroll
            for (int s = 0; s < S; ++s) x[j][s] = ld_relaxed_gpu(ip + s * W + lane + 32 * j);
    }
    for (int64_t i = found - 1; i >= 1; i -= BATCH) {
        float e[BATCH][CPL][NA];
#pragma unroll
        for (int m = 0; m < BATCH; ++m) {
            if (i - m >= 1) {
                const float* ap = cx.agg + ((tile - (i - m) * cx.nGroups) * cx.nSlots + slot) * NA * W;
#pragma unroll
                for (int j = 0; j < CPL; ++j)
#pragma unroll
                    for (int a = 0; a < NA; ++a) e[m][j][a] = ld_relaxed_gpu(ap + a * W + lane + 32 * j);
            }
        }
#pragma unroll
        for (int m = 0; m < BATCH; ++m) {
            if (i - m >= 1) {
#pragma unroll
                for (int j = 0; j < CPL; ++j) {
                    float A[S * S], b[S], y[S];
#pragma unroll
                    for (int a = 0; a < S * S; ++a) A[a] = e[m][j][a];
#pragma unroll
                    for (int s = 0; s < S; ++s) b[s] = e[m][j][S * S + s];
                    apply<S>(A, b, x[j], y);
#pragma unroll
                    for (int s = 0; s < S; ++s) x[j][s] = y[s];
                }
            }
        }
    }
#pragma unroll
    for (int j = 0; j < CPL; ++j)
#pragma unroll
        for (int s = 0; s < S; ++s) carry[j][s] = x[j][s];
}

// The work warp 0 does between the two block barriers of one scan step:
// compose the NSUB sub-chunk elements (s_agg, in scan order) into the tile's
// element, publish it, find the carry, publish the inclusive state, and
// write each sub-chunk's carry-in to s_carry.  Returns (in carry_out) the
// carry into the tile.
template <int S, int W, int NSUB>
__device__ __forceinline__ void tile_scan_step(const LookbackCtx& cx, int64_t tile, int64_t pos, int slot, int lane,
                                               const float (&s_agg)[NSUB][S * S + S][W], float (&s_carry)[NSUB][S][W],
                                               const float (&first_carry)[W / 32][S], float (&carry_out)[W / 32][S]) {
    constexpr int NA = S * S + S;
    constexpr int CPL = W / 32;
    Elem<S> tot[CPL];
#pragma unroll
    for (int j = 0; j < CPL; ++j) elem_identity<S>(tot[j]);
#pragma unroll 4
    for (int sb = 0; sb < NSUB; ++sb) {
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
            float A[S * S], b[S];
#pragma unroll
            for (int a = 0; a < S * S; ++a) A[a] = s_agg[sb][a][lane + 32 * j];
#pragma unroll
            for (int s = 0; s < S; ++s) b[s] = s_agg[sb][S * S + s][lane + 32 * j];
            compose_after<S>(A, b, tot[j]);
        }
    }
    unsigned* flag = cx.flags + tile * cx.nSlots + slot;
    float carry[CPL][S];
    if (pos == 0) {
#pragma unroll
        for (int j = 0; j < CPL; ++j)
#pragma unroll
            for (int s = 0; s < S; ++s) carry[j][s] = first_carry[j][s];
    } else {
        float vals[CPL][NA];
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
#pragma unroll
            for (int a = 0; a < S * S; ++a) vals[j][a] = tot[j].A[a];
#pragma unroll
            for (int s = 0; s < S; ++s) vals[j][S * S + s] = tot[j].b[s];
        }
        publish<NA, W>(cx.agg + (tile * cx.nSlots + slot) * NA * W, vals, flag, kFlagAggregate, lane);
        lookback_carry<S, W>(cx, tile, pos, slot, lane, carry);
    }
    {
        float vals[CPL][S];
#pragma unroll
        for (int j = 0; j < CPL; ++j) apply<S>(tot[j].A, tot[j].b, carry[j], vals[j]);
        publish<S, W>(cx.inc + (tile * cx.nSlots + slot) * S * W, vals, flag, kFlagInclusive, lane);
    }
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
        float x[S];
#pragma unroll
        for (int s = 0; s < S; ++s) x[s] = carry[j][s];
#pragma unroll 4
        for (int sb = 0; sb < NSUB; ++sb) {
            float A[S * S], b[S], y[S];
#pragma unroll
            for (int s = 0; s < S; ++s) s_carry[sb][s][lane + 32 * j] = x[s];
#pragma unroll
            for (int a = 0; a < S * S; ++a) A[a] = s_agg[sb][a][lane + 32 * j];
#pragma unroll
            for (int s = 0; s < S; ++s) b[s] = s_agg[sb][S * S + s][lane + 32 * j];
            apply<S>(A, b, x, y);
#pragma unroll
            for (int s = 0; s < S; ++s) x[s] = y[s];
        }
#pragma unroll
        for (int s = 0; s < S; ++s) carry_out[j][s] = carry[j][s];
    }
}

}  // namespace pararnn
