// lookback.cuh -- decoupled look-back between the tiles of one channel group.
//
// Tiles are numbered by a ticket taken from an atomic counter, in scan
// order: ticket = position_along_the_scan * nGroups + group.  A block
// processes its tickets in increasing order, so the smallest unfinished
// ticket always belongs to a running block and every wait ends (forward
// progress does not depend on how the hardware schedules blocks).
//
// Per (tile, slot) -- slot = Newton iteration in the forward, 0 in the
// backward -- the workspace holds 64-bit words
//     { high 32 bits: the call's epoch tag, low 32 bits: a value }
//   status     one word: 1 = aggregate published, 2 = inclusive published
//   aggregate  per channel, the tile's composed scan element (A, b)  NA words
//   inclusive  per channel, the state after the tile's last row      S words
// A word is valid when its tag equals this call's epoch, so a value and its
// "ready" flag travel in one single-copy-atomic store: no fence is needed.
// The host clears every look-back word on the stream before the kernel runs,
// and a cleared word never matches (epochs start at 1).  The status word
// lets one warp read 32 predecessors' states in one round trip; payload
// words are checked again when they are read, so a status seen before its
// payload costs a retry, never a wrong value.
//
// The carry into a tile is found by walking back to the nearest predecessor
// with an inclusive value and applying the aggregates in between, in order,
// to it.  An inclusive value is itself formed as apply(aggregate, carry), so
// the carry is bit-identical whichever predecessors had finished: results do
// not depend on timing.
#pragma once

#include "cells.cuh"
#include "common.cuh"

namespace pararnn {

typedef unsigned long long word_t;

struct LookbackCtx {
    unsigned* status;  // workspace header word 0
    word_t* tstat;     // [nTiles][nSlots] tile status words
    word_t* agg;       // [nTiles][nSlots][NA][W]
    word_t* inc;       // [nTiles][nSlots][S][W]
    int64_t nGroups;
    int nSlots;
    uint32_t epoch;
    uint64_t timeout_ns;
    int stall_first;   // test hook: the tile with ticket 0 never publishes its state
};

__device__ __forceinline__ void st_word(word_t* p, float v, uint32_t epoch) {
    const word_t w = (static_cast<word_t>(epoch) << 32) | __float_as_uint(v);
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}

__device__ __forceinline__ word_t ld_word(const word_t* p) {
    word_t w;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(w) : "l"(p) : "memory");
    return w;
}

__device__ __forceinline__ bool word_ok(word_t w, uint32_t epoch) { return static_cast<uint32_t>(w >> 32) == epoch; }
__device__ __forceinline__ float word_val(word_t w) { return __uint_as_float(static_cast<uint32_t>(w)); }

// Bounded wait for an mbarrier phase or a flag: returns false once
// `timeout_ns` has passed, so that the caller can record the time-out and
// finish instead of spinning for ever.
struct Deadline {
    uint64_t start = 0;
    __device__ __forceinline__ bool expired(uint64_t timeout_ns) {
        const uint64_t now = globaltimer_ns();
        if (start == 0) {
            start = now | 1;
            return false;
        }
        return now - start > timeout_ns;
    }
};

template <int N, int W>
__device__ __forceinline__ void publish_words(word_t* dst, const float (&vals)[W / 32][N], uint32_t epoch, int lane) {
#pragma unroll
    for (int j = 0; j < W / 32; ++j)
#pragma unroll
        for (int n = 0; n < N; ++n) st_word(dst + n * W + lane + 32 * j, vals[j][n], epoch);
}

constexpr uint32_t kTileAggregate = 1u, kTileInclusive = 2u;

__device__ __forceinline__ void st_status(word_t* p, uint32_t state, uint32_t epoch) {
    const word_t w = (static_cast<word_t>(epoch) << 32) | state;
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}

// Carry into `tile` for scan slot `slot`: the state just before the tile's
// first row, for the W/32 channels this lane owns.  `dist_max` = the tile's
// position along the scan (its number of predecessors).  All 32 lanes of one
// warp call this.
//   1. lane j reads the status of predecessor base+j; the nearest one with an
//      inclusive value, with only aggregates between it and this tile, ends
//      the walk (32 predecessors per round trip);
//   2. the payload words of that inclusive value and of the aggregates in
//      between are read in batches of NB predecessors, and the aggregates are
//      applied to the inclusive value in order, nearest last.
// The inclusive words of the first predecessor are fetched with step 1, so
// the common case costs one round trip.
template <int S, int W>
__device__ void lookback_carry(const LookbackCtx& cx, int64_t tile, int64_t dist_max, int slot, int lane,
                               float (&carry)[W / 32][S]) {
    constexpr int NA = S * S + S;
    constexpr int CPL = W / 32;
    constexpr int NB = S == 1 ? 4 : 2;  // aggregates read per batch
    Deadline dl;
    int64_t base = 1, found = -1;
    bool ok = true;
    // ---- 1. walk the status words ----
    while (true) {
        const int64_t j = base + lane;
        uint32_t state = 0;
        if (j <= dist_max) {
            const word_t w = ld_word(cx.tstat + (tile - j * cx.nGroups) * cx.nSlots + slot);
            if (word_ok(w, cx.epoch)) state = static_cast<uint32_t>(w);
        }
        float spec[CPL][S];  // inclusive words of the nearest predecessor, fetched speculatively
        bool spec_ok = true;
        if (base == 1) {
            const float* dummy = nullptr;
            (void)dummy;
#pragma unroll
            for (int jj = 0; jj < CPL; ++jj)
#pragma unroll
                for (int s = 0; s < S; ++s) {
                    const word_t w = ld_word(cx.inc + (((tile - cx.nGroups) * cx.nSlots + slot) * S + s) * W + lane + 32 * jj);
                    spec_ok &= word_ok(w, cx.epoch);
                    spec[jj][s] = word_val(w);
                }
        }
        const unsigned inc_mask = __ballot_sync(0xffffffffu, j <= dist_max && state == kTileInclusive);
        const unsigned not_ready = __ballot_sync(0xffffffffu, j <= dist_max && state == 0);
        if (inc_mask) {
            const int first = __ffs(inc_mask) - 1;
            const unsigned before = first ? (not_ready & ((1u << first) - 1u)) : 0u;
            if (!before) {
                found = base + first;
                if (found == 1 && __all_sync(0xffffffffu, spec_ok)) {
#pragma unroll
                    for (int jj = 0; jj < CPL; ++jj)
#pragma unroll
                        for (int s = 0; s < S; ++s) carry[jj][s] = spec[jj][s];
                    return;
                }
                break;
            }
        } else if (!not_ready) {
            // 32 aggregates in a row: look further back
            base += 32;
            if (base <= dist_max) continue;
            ok = false;  // the first tile of the scan never publishes an aggregate only
            break;
        }
        if (dl.expired(cx.timeout_ns)) {
            ok = false;
            break;
        }
        __nanosleep(20);
    }
    // ---- 2. payloads: inclusive(found), then aggregates found-1 .. 1 ----
    if (ok) {
        float x[CPL][S];
        Deadline dl2;
        while (true) {
            bool good = true;
#pragma unroll
            for (int jj = 0; jj < CPL; ++jj)
#pragma unroll
                for (int s = 0; s < S; ++s) {
                    const word_t w = ld_word(cx.inc + (((tile - found * cx.nGroups) * cx.nSlots + slot) * S + s) * W + lane + 32 * jj);
                    good &= word_ok(w, cx.epoch);
                    x[jj][s] = word_val(w);
                }
            for (int64_t i = found - 1; i >= 1 && good; i -= NB) {
                word_t e[NB][CPL][NA];
#pragma unroll
                for (int m = 0; m < NB; ++m)
                    if (i - m >= 1) {
                        const word_t* ap = cx.agg + ((tile - (i - m) * cx.nGroups) * cx.nSlots + slot) * NA * W;
#pragma unroll
                        for (int jj = 0; jj < CPL; ++jj)
#pragma unroll
                            for (int a = 0; a < NA; ++a) e[m][jj][a] = ld_word(ap + a * W + lane + 32 * jj);
                    }
#pragma unroll
                for (int m = 0; m < NB; ++m)
                    if (i - m >= 1) {
#pragma unroll
                        for (int jj = 0; jj < CPL; ++jj) {
                            float A[S * S], b[S], y[S];
#pragma unroll
                            for (int a = 0; a < S * S; ++a) {
                                good &= word_ok(e[m][jj][a], cx.epoch);
                                A[a] = word_val(e[m][jj][a]);
                            }
#pragma unroll
                            for (int s = 0; s < S; ++s) {
                                good &= word_ok(e[m][jj][S * S + s], cx.epoch);
                                b[s] = word_val(e[m][jj][S * S + s]);
                            }
                            apply<S>(A, b, x[jj], y);
#pragma unroll
                            for (int s = 0; s < S; ++s) x[jj][s] = y[s];
                        }
                    }
            }
            if (__all_sync(0xffffffffu, good)) {
#pragma unroll
                for (int jj = 0; jj < CPL; ++jj)
#pragma unroll
                    for (int s = 0; s < S; ++s) carry[jj][s] = x[jj][s];
                return;
            }
            // a status word became visible before its payload: read again
            if (dl2.expired(cx.timeout_ns)) break;
            __nanosleep(20);
        }
    }
    if (lane == 0) atomicOr(cx.status, kStatusTimeout);
#pragma unroll
    for (int jj = 0; jj < CPL; ++jj)
#pragma unroll
        for (int s = 0; s < S; ++s) carry[jj][s] = 0.0f;
}

// The predecessor's status and inclusive words, loaded early (while the
// compute warps evaluate) and used after they have composed the tile: when
// the predecessor had already finished, the carry costs no waiting at all.
template <int S, int W>
struct Probe {
    word_t st;
    word_t inc[W / 32][S];
};

template <int S, int W>
__device__ __forceinline__ void probe_issue(const LookbackCtx& cx, int64_t tile, int64_t pos, int slot, int lane,
                                            Probe<S, W>& pr) {
    pr.st = 0;
    if (pos == 0) return;
    const int64_t tp = tile - cx.nGroups;
    pr.st = ld_word(cx.tstat + tp * cx.nSlots + slot);
#pragma unroll
    for (int j = 0; j < W / 32; ++j)
#pragma unroll
        for (int s = 0; s < S; ++s) pr.inc[j][s] = ld_word(cx.inc + ((tp * cx.nSlots + slot) * S + s) * W + lane + 32 * j);
}

// ---- the block-level part of one scan step --------------------------------
// Thread (warp w, lane l) owns sub-chunk sub = w * TPW + l / LC of the tile
// and the V channels cc .. cc+V-1, cc = (l % LC) * V.  Scan order is time
// order (forward) or reverse time order (backward).

// A scan element of V channels held by one thread.
template <int S, int V>
struct ElemV {
    Elem<S> e[V];
};

template <int S>
__device__ __forceinline__ Elem<S> shfl_elem(const Elem<S>& x, int src_lane_delta, bool up) {
    Elem<S> y;
#pragma unroll
    for (int a = 0; a < S * S; ++a)
        y.A[a] = up ? __shfl_up_sync(0xffffffffu, x.A[a], src_lane_delta) : __shfl_down_sync(0xffffffffu, x.A[a], src_lane_delta);
#pragma unroll
    for (int s = 0; s < S; ++s)
        y.b[s] = up ? __shfl_up_sync(0xffffffffu, x.b[s], src_lane_delta) : __shfl_down_sync(0xffffffffu, x.b[s], src_lane_delta);
    return y;
}

// acc <- x o acc
template <int S>
__device__ __forceinline__ void compose_elem(const Elem<S>& x, Elem<S>& acc) {
    compose_after<S>(x.A, x.b, acc);
}

// Step 1 (all threads, between the local composition and the first barrier):
// scan the TPW sub-chunks of each warp with shuffles.  Returns in `excl` the
// composition of the sub-chunks before this one inside its warp (identity for
// the first), and writes each warp's total to wagg[w] (by the lanes of the
// warp's last sub-chunk in scan order).
template <int S, int V, int LC, int W, int NW, bool kReverse>
__device__ __forceinline__ void warp_prefix(const ElemV<S, V>& mine, ElemV<S, V>& excl, int warp, int lane,
                                            float (&wagg)[NW][S * S + S][W]) {
    constexpr int TPW = 32 / LC;
    const int q = lane / LC;                          // sub-chunk index inside the warp, time order
    const int qs = kReverse ? (TPW - 1 - q) : q;      // ... in scan order
    const int cc = (lane % LC) * V;
#pragma unroll
    for (int v = 0; v < V; ++v) {
        Elem<S> incl = mine.e[v];
#pragma unroll
        for (int d = 1; d < TPW; d *= 2) {
            // the sub-chunk d places earlier in scan order sits d*LC lanes below
            // (forward) or above (reverse)
            const Elem<S> other = shfl_elem<S>(incl, d * LC, !kReverse);
            if (qs >= d) {
                Elem<S> t = other;   // incl <- incl o other (other first)
                compose_elem<S>(incl, t);
                incl = t;
            }
        }
        Elem<S> ex = shfl_elem<S>(incl, LC, !kReverse);
        if (qs == 0) elem_identity<S>(ex);
        excl.e[v] = ex;
        if (qs == TPW - 1) {
#pragma unroll
            for (int a = 0; a < S * S; ++a) wagg[warp][a][cc + v] = incl.A[a];
#pragma unroll
            for (int s = 0; s < S; ++s) wagg[warp][S * S + s][cc + v] = incl.b[s];
        }
    }
}

// Step 2a (all threads, after the first barrier): the composition of every
// earlier warp (scan order) followed by the earlier sub-chunks of this warp:
// the element that maps the tile's carry-in to this sub-chunk's carry-in.
template <int S, int V, int LC, int W, int NW, bool kReverse>
__device__ __forceinline__ void sub_prefix(const ElemV<S, V>& excl, int warp, int lane,
                                           const float (&wagg)[NW][S * S + S][W], ElemV<S, V>& pre) {
    const int cc = (lane % LC) * V;
    const int ws = kReverse ? (NW - 1 - warp) : warp;  // this warp's position in scan order
#pragma unroll
    for (int v = 0; v < V; ++v) {
        Elem<S> acc;
        elem_identity<S>(acc);
        // the same compositions in the same order either way.  A scalar state
        // unrolls over the block's warps with the position test inside, so
        // that the shared-memory loads can all be issued before the chain of
        // compositions (measured 2-5 % faster); a 2 x 2 state keeps the loop,
        // whose six words per warp would otherwise cost registers (measured
        // 3-4 % slower unrolled)
        if constexpr (S == 1) {
#pragma unroll
            for (int k = 0; k < NW; ++k) {
                if (k < ws) {
                    const int wk = kReverse ? (NW - 1 - k) : k;
                    float A[S * S], b[S];
#pragma unroll
                    for (int a = 0; a < S * S; ++a) A[a] = wagg[wk][a][cc + v];
#pragma unroll
                    for (int s = 0; s < S; ++s) b[s] = wagg[wk][S * S + s][cc + v];
                    compose_after<S>(A, b, acc);
                }
            }
        } else {
            for (int k = 0; k < ws; ++k) {
                const int wk = kReverse ? (NW - 1 - k) : k;
                float A[S * S], b[S];
#pragma unroll
                for (int a = 0; a < S * S; ++a) A[a] = wagg[wk][a][cc + v];
#pragma unroll
                for (int s = 0; s < S; ++s) b[s] = wagg[wk][S * S + s][cc + v];
                compose_after<S>(A, b, acc);
            }
        }
        compose_elem<S>(excl.e[v], acc);
        pre.e[v] = acc;
    }
}

// The state after a tile, for the W/32 channels of one scan-warp lane,
// computed before the carry barrier and published after it.
template <int S, int W>
struct Inclusive {
    float v[W / 32][S];
};

// Step 2b (the scan warp, after the first barrier): compose the warp totals
// into the tile's element, find the carry and write it to cin; return the
// state after the tile in `out`, to be published by publish_inclusive once
// the compute warps have been released.  When the early probe found the
// predecessor's state, nobody waits on this tile's aggregate -- its own
// state follows within a barrier's time -- so the aggregate is published
// only before a real look-back, where successors may need it meanwhile.
template <int S, int W, int NW, bool kReverse>
__device__ __forceinline__ void tile_lookback(const LookbackCtx& cx, int64_t tile, int64_t pos, int slot, int lane,
                                              const float (&wagg)[NW][S * S + S][W],
                                              const float (&first_carry)[W / 32][S], const Probe<S, W>& pr,
                                              float (&cin)[S][W], Inclusive<S, W>& out) {
    constexpr int NA = S * S + S;
    constexpr int CPL = W / 32;
    Elem<S> tot[CPL];
#pragma unroll
    for (int j = 0; j < CPL; ++j) elem_identity<S>(tot[j]);
#pragma unroll
    for (int k = 0; k < NW; ++k) {
        const int wk = kReverse ? (NW - 1 - k) : k;
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
            float A[S * S], b[S];
#pragma unroll
            for (int a = 0; a < S * S; ++a) A[a] = wagg[wk][a][lane + 32 * j];
#pragma unroll
            for (int s = 0; s < S; ++s) b[s] = wagg[wk][S * S + s][lane + 32 * j];
            compose_after<S>(A, b, tot[j]);
        }
    }
    float carry[CPL][S];
    if (pos == 0) {
#pragma unroll
        for (int j = 0; j < CPL; ++j)
#pragma unroll
            for (int s = 0; s < S; ++s) carry[j][s] = first_carry[j][s];
    } else {
        // the predecessor's inclusive state, if the early probe found it published
        bool ok = word_ok(pr.st, cx.epoch) && static_cast<uint32_t>(pr.st) == kTileInclusive;
#pragma unroll
        for (int j = 0; j < CPL; ++j)
#pragma unroll
            for (int s = 0; s < S; ++s) {
                ok &= word_ok(pr.inc[j][s], cx.epoch);
                carry[j][s] = word_val(pr.inc[j][s]);
            }
        if (!__all_sync(0xffffffffu, ok)) {
            // publish the aggregate first, so that successors never wait on
            // this tile's look-back
            float vals[CPL][NA];
#pragma unroll
            for (int j = 0; j < CPL; ++j) {
#pragma unroll
                for (int a = 0; a < S * S; ++a) vals[j][a] = tot[j].A[a];
#pragma unroll
                for (int s = 0; s < S; ++s) vals[j][S * S + s] = tot[j].b[s];
            }
            publish_words<NA, W>(cx.agg + (tile * cx.nSlots + slot) * NA * W, vals, cx.epoch, lane);
            __syncwarp();
            if (lane == 0) st_status(cx.tstat + tile * cx.nSlots + slot, kTileAggregate, cx.epoch);
            lookback_carry<S, W>(cx, tile, pos, slot, lane, carry);
        }
    }
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
        apply<S>(tot[j].A, tot[j].b, carry[j], out.v[j]);
#pragma unroll
        for (int s = 0; s < S; ++s) cin[s][lane + 32 * j] = carry[j][s];
    }
}

// Step 3 (the scan warp, after the carry barrier): publish the state after
// the tile (inclusive words, then the status word).
template <int S, int W>
__device__ __forceinline__ void publish_inclusive(const LookbackCtx& cx, int64_t tile, int slot, int lane,
                                                  const Inclusive<S, W>& out) {
    // the stall hook: the first tile of the scan withholds its state, so its
    // successor's bounded look-back runs out (the time-out path under test)
    if (cx.stall_first && tile == 0) return;
    publish_words<S, W>(cx.inc + (tile * cx.nSlots + slot) * S * W, out.v, cx.epoch, lane);
    __syncwarp();
    if (lane == 0) st_status(cx.tstat + tile * cx.nSlots + slot, kTileInclusive, cx.epoch);
}

}  // namespace pararnn
