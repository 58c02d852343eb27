// pararnn_abi.cu -- the C ABI declared in include/pararnn_b200.h: argument
// checks, workspace layout, choice of tile shape and kernel launches.
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "pararnn_b200.h"

#include "adjoint_bwd.cuh"
#include "newton_fwd.cuh"

using namespace pararnn;

namespace {

thread_local char g_last_error[512] = "";

pararnn_status fail(pararnn_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return st;
}

pararnn_status cuda_fail(cudaError_t e, const char* what) {
    return fail(PARARNN_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ---- tile shapes (V channels per thread, LC lanes across channels, warps, rows per thread) ----
// vector path (D a multiple of 4, 16-byte aligned rows): 2 or 4 channels per thread, 64 channels per tile
using FwdLinV = FwdShape<CellLinear, 4, 16, 8, 4>;
using FwdGruV = FwdShape<CellGRU, 2, 32, 8, 4>;
using FwdLstmV = FwdShape<CellLSTM, 2, 32, 8, 2>;
using BwdLinV = FwdShape<CellLinear, 2, 32, 8, 4>;
using BwdGruV = FwdShape<CellGRU, 2, 32, 8, 2>;
using BwdLstmV = FwdShape<CellLSTM, 2, 32, 8, 1>;
// scalar path (D not a multiple of 4, or unaligned pointers): 32 channels per tile
using FwdLinS = FwdShape<CellLinear, 1, 32, 8, 8>;
using FwdGruS = FwdShape<CellGRU, 1, 32, 8, 4>;
using FwdLstmS = FwdShape<CellLSTM, 1, 32, 8, 2>;
using BwdLinS = FwdShape<CellLinear, 1, 32, 8, 4>;
using BwdGruS = FwdShape<CellGRU, 1, 32, 8, 2>;
using BwdLstmS = FwdShape<CellLSTM, 1, 32, 8, 1>;

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s: far beyond any legitimate wait
constexpr int kMaxK = 64;

struct Geometry {
    int W = 0, L = 0, S = 0, G = 0, NA = 0, nSlots = 0;
};

Geometry geometry(pararnn_cell cell, bool fwd, bool vec, int K) {
    Geometry g;
    auto set = [&](auto sh) {
        using Sh = decltype(sh);
        g.W = Sh::W;
        g.L = Sh::L;
        g.S = Sh::S;
        g.G = Sh::G;
        g.NA = Sh::NA;
    };
    if (cell == PARARNN_CELL_LINEAR) {
        if (fwd) vec ? set(FwdLinV{}) : set(FwdLinS{});
        else vec ? set(BwdLinV{}) : set(BwdLinS{});
    } else if (cell == PARARNN_CELL_DIAG_GRU) {
        if (fwd) vec ? set(FwdGruV{}) : set(FwdGruS{});
        else vec ? set(BwdGruV{}) : set(BwdGruS{});
    } else {
        if (fwd) vec ? set(FwdLstmV{}) : set(FwdLstmS{});
        else vec ? set(BwdLstmV{}) : set(BwdLstmS{});
    }
    g.nSlots = fwd ? (cell == PARARNN_CELL_LINEAR ? 1 : K) : 1;
    return g;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct Plan {
    int64_t nCG = 0, nChunks = 0, nGroups = 0, nTiles = 0;
    size_t off_flags = 0, off_agg = 0, off_inc = 0, off_part = 0, total = 0;
    Geometry g;
};

Plan make_plan(pararnn_cell cell, int64_t B, int64_t T, int64_t D, int K, bool fwd, bool vec) {
    Plan p;
    p.g = geometry(cell, fwd, vec, K);
    p.nCG = (D + p.g.W - 1) / p.g.W;
    p.nChunks = (T + p.g.L - 1) / p.g.L;
    p.nGroups = B * p.nCG;
    p.nTiles = p.nGroups * p.nChunks;
    const size_t nt = (size_t)p.nTiles, ns = (size_t)p.g.nSlots, W = (size_t)p.g.W;
    p.off_flags = kHeaderBytes;
    p.off_agg = align256(p.off_flags + nt * ns * sizeof(unsigned));
    p.off_inc = align256(p.off_agg + nt * ns * p.g.NA * W * sizeof(float));
    p.off_part = align256(p.off_inc + nt * ns * p.g.S * W * sizeof(float));
    p.total = fwd ? p.off_part : align256(p.off_part + nt * p.g.G * W * sizeof(float));
    return p;
}

bool cell_ok(pararnn_cell c) {
    return c == PARARNN_CELL_LINEAR || c == PARARNN_CELL_DIAG_GRU || c == PARARNN_CELL_DIAG_LSTM;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// A pointer the GPU can dereference: device, managed, or registered host memory.
bool device_reachable(const void* p) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged ||
           (at.type == cudaMemoryTypeHost && at.devicePointer != nullptr);
}

pararnn_status check_sizes(pararnn_cell cell, int64_t B, int64_t T, int64_t D) {
    if (!cell_ok(cell)) return fail(PARARNN_EINVAL, "unknown cell %d", (int)cell);
    if (B < 0 || T < 0 || D < 0) return fail(PARARNN_EINVAL, "negative size B=%lld T=%lld D=%lld", (long long)B,
                                             (long long)T, (long long)D);
    const int64_t lim = int64_t(1) << 40;
    if (B > lim || T > lim || D > lim || (B && T && D && (double)B * T * D * 4 > 9.0e18 / 16))
        return fail(PARARNN_EINVAL, "problem too large");
    return PARARNN_OK;
}

template <class Cell, typename PxT, class Sh>
pararnn_status launch_fwd(const Plan& pl, FwdParams prm, cudaStream_t st) {
    prm.nCG = pl.nCG;
    prm.nChunks = pl.nChunks;
    newton_fwd_kernel<Cell, PxT, Sh><<<(unsigned)pl.nTiles, Sh::NT, 0, st>>>(prm);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? PARARNN_OK : cuda_fail(e, "forward kernel launch");
}

template <class Cell, typename PxT, class Sh>
pararnn_status launch_bwd(const Plan& pl, BwdParams prm, float* dLda, cudaStream_t st) {
    prm.nCG = pl.nCG;
    prm.nChunks = pl.nChunks;
    adjoint_bwd_kernel<Cell, PxT, Sh><<<(unsigned)pl.nTiles, Sh::NT, 0, st>>>(prm);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "backward kernel launch");
    if (dLda) {
        ReduceParams rp;
        rp.part = prm.part;
        rp.dLda = dLda;
        rp.B = prm.B;
        rp.D = prm.D;
        rp.nCG = pl.nCG;
        rp.nChunks = pl.nChunks;
        rp.nGroups = pl.nGroups;
        rp.G = Sh::G;
        rp.W = Sh::W;
        const int64_t n = (int64_t)Sh::G * prm.D;
        reduce_da_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(rp);
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "dL/da reduction launch");
    }
    return PARARNN_OK;
}

__global__ void probe_wait_kernel(unsigned* status, const unsigned* flag, uint64_t timeout_ns) {
    unsigned seen;
    if (threadIdx.x == 0 && !wait_flag(flag, kFlagInclusive, timeout_ns, seen)) atomicOr(status, kStatusTimeout);
}

}  // namespace

extern "C" {

int pararnn_num_gates(pararnn_cell cell) {
    return cell == PARARNN_CELL_LINEAR ? 2 : cell == PARARNN_CELL_DIAG_GRU ? 3 : cell == PARARNN_CELL_DIAG_LSTM ? 4 : -1;
}

int pararnn_state_width(pararnn_cell cell) {
    return cell == PARARNN_CELL_LINEAR ? 1 : cell == PARARNN_CELL_DIAG_GRU ? 1 : cell == PARARNN_CELL_DIAG_LSTM ? 2 : -1;
}

size_t pararnn_workspace_bytes(pararnn_cell cell, int64_t B, int64_t T, int64_t D, int K) {
    if (check_sizes(cell, B, T, D) != PARARNN_OK) return 0;
    if (K < 1) K = 1;
    if (K > kMaxK) K = kMaxK;
    size_t m = kHeaderBytes + 256;
    for (int fwd = 0; fwd < 2; ++fwd)
        for (int vec = 0; vec < 2; ++vec) {
            const Plan p = make_plan(cell, B, T, D, K, fwd != 0, vec != 0);
            if (p.total > m) m = p.total;
        }
    return m;
}

pararnn_status pararnn_newton_forward(pararnn_cell cell, int64_t B, int64_t T, int64_t D, pararnn_dtype px_dtype,
                                      const void* preacts, const float* diag_w, const float* h0, int K,
                                      float* H_out, void* workspace, size_t ws_bytes, float* resid_hist,
                                      void* stream) {
    g_last_error[0] = 0;
    pararnn_status st = check_sizes(cell, B, T, D);
    if (st != PARARNN_OK) return st;
    if (px_dtype != PARARNN_F32 && px_dtype != PARARNN_BF16)
        return fail(PARARNN_EINVAL, "unknown pre-activation dtype %d", (int)px_dtype);
    if (K < 1 || K > kMaxK) return fail(PARARNN_EINVAL, "K=%d outside 1..%d", K, kMaxK);
    if (!workspace) return fail(PARARNN_EINVAL, "workspace is NULL");
    if (!aligned(workspace, 16)) return fail(PARARNN_EINVAL, "workspace not 16-byte aligned");
    const size_t need = pararnn_workspace_bytes(cell, B, T, D, K);
    if (ws_bytes < need) return fail(PARARNN_EINVAL, "workspace %zu bytes < %zu required", ws_bytes, need);
    const size_t esz = px_dtype == PARARNN_F32 ? 4 : 2;
    const bool empty = (B == 0 || T == 0 || D == 0);
    if (!empty) {
        if (!preacts || !H_out) return fail(PARARNN_EINVAL, "preacts and H_out must not be NULL");
        if (!aligned(preacts, esz) || !aligned(H_out, 4) || (diag_w && !aligned(diag_w, 4)) || (h0 && !aligned(h0, 4)))
            return fail(PARARNN_EINVAL, "pointer not aligned to its element size");
        if (!device_reachable(preacts) || !device_reachable(H_out) || !device_reachable(workspace) ||
            (diag_w && !device_reachable(diag_w)) || (h0 && !device_reachable(h0)))
            return fail(PARARNN_EINVAL, "a pointer is not device-accessible memory");
    }
    if (resid_hist && (!aligned(resid_hist, 4) || !device_reachable(resid_hist)))
        return fail(PARARNN_EINVAL, "resid_hist is not device-accessible float memory");

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool vec = (D % 4 == 0) && aligned(preacts, 16) && aligned(H_out, 16);
    const int Keff = cell == PARARNN_CELL_LINEAR ? 1 : K;
    const Plan pl = make_plan(cell, B, T, D, Keff, true, vec);
    if (pl.nTiles >= (int64_t(1) << 31)) return fail(PARARNN_EINVAL, "too many tiles");

    char* ws = static_cast<char*>(workspace);
    cudaError_t e = cudaMemsetAsync(ws, 0, empty ? kHeaderBytes : pl.off_agg, s);
    if (e != cudaSuccess) return cuda_fail(e, "workspace reset");
    if (resid_hist) {
        e = cudaMemsetAsync(resid_hist, 0, sizeof(float) * (K + 1), s);
        if (e != cudaSuccess) return cuda_fail(e, "resid_hist reset");
    }
    if (empty) return PARARNN_OK;

    FwdParams prm;
    memset(&prm, 0, sizeof prm);
    prm.px = preacts;
    prm.w = diag_w;
    prm.h0 = h0;
    prm.H = H_out;
    prm.resid = resid_hist;
    prm.B = B;
    prm.T = T;
    prm.D = D;
    prm.K = Keff;
    prm.lb.status = reinterpret_cast<unsigned*>(ws);
    prm.lb.flags = reinterpret_cast<unsigned*>(ws + pl.off_flags);
    prm.lb.agg = reinterpret_cast<float*>(ws + pl.off_agg);
    prm.lb.inc = reinterpret_cast<float*>(ws + pl.off_inc);
    prm.lb.nGroups = pl.nGroups;
    prm.lb.nSlots = pl.g.nSlots;
    prm.lb.timeout_ns = kWaitLimitNs;

    const bool bf = px_dtype == PARARNN_BF16;
    if (cell == PARARNN_CELL_LINEAR) {
        if (vec) st = bf ? launch_fwd<CellLinear, __nv_bfloat16, FwdLinV>(pl, prm, s) : launch_fwd<CellLinear, float, FwdLinV>(pl, prm, s);
        else st = bf ? launch_fwd<CellLinear, __nv_bfloat16, FwdLinS>(pl, prm, s) : launch_fwd<CellLinear, float, FwdLinS>(pl, prm, s);
    } else if (cell == PARARNN_CELL_DIAG_GRU) {
        if (vec) st = bf ? launch_fwd<CellGRU, __nv_bfloat16, FwdGruV>(pl, prm, s) : launch_fwd<CellGRU, float, FwdGruV>(pl, prm, s);
        else st = bf ? launch_fwd<CellGRU, __nv_bfloat16, FwdGruS>(pl, prm, s) : launch_fwd<CellGRU, float, FwdGruS>(pl, prm, s);
    } else {
        if (vec) st = bf ? launch_fwd<CellLSTM, __nv_bfloat16, FwdLstmV>(pl, prm, s) : launch_fwd<CellLSTM, float, FwdLstmV>(pl, prm, s);
        else st = bf ? launch_fwd<CellLSTM, __nv_bfloat16, FwdLstmS>(pl, prm, s) : launch_fwd<CellLSTM, float, FwdLstmS>(pl, prm, s);
    }
    if (st != PARARNN_OK) return st;
    if (resid_hist && Keff < K) {
        // the linear cell is exact after its one scan: later iterates equal it
        for (int k = Keff + 1; k <= K; ++k) {
            e = cudaMemcpyAsync(resid_hist + k, resid_hist + Keff, sizeof(float), cudaMemcpyDeviceToDevice, s);
            if (e != cudaSuccess) return cuda_fail(e, "resid_hist copy");
        }
    }
    return PARARNN_OK;
}

pararnn_status pararnn_newton_backward(pararnn_cell cell, int64_t B, int64_t T, int64_t D, pararnn_dtype px_dtype,
                                       const void* preacts, const float* diag_w, const float* h0, const float* H,
                                       const float* dL_dH, float* dL_dpx, float* dL_da, float* dL_dh0,
                                       void* workspace, size_t ws_bytes, void* stream) {
    g_last_error[0] = 0;
    pararnn_status st = check_sizes(cell, B, T, D);
    if (st != PARARNN_OK) return st;
    if (px_dtype != PARARNN_F32 && px_dtype != PARARNN_BF16)
        return fail(PARARNN_EINVAL, "unknown pre-activation dtype %d", (int)px_dtype);
    if (!workspace) return fail(PARARNN_EINVAL, "workspace is NULL");
    if (!aligned(workspace, 16)) return fail(PARARNN_EINVAL, "workspace not 16-byte aligned");
    const size_t need = pararnn_workspace_bytes(cell, B, T, D, 1);
    if (ws_bytes < need) return fail(PARARNN_EINVAL, "workspace %zu bytes < %zu required", ws_bytes, need);
    if (cell == PARARNN_CELL_LINEAR) dL_da = nullptr;  // no recurrent weights
    const size_t esz = px_dtype == PARARNN_F32 ? 4 : 2;
    const bool empty = (B == 0 || T == 0 || D == 0);
    if (!empty) {
        if (!preacts || !H || !dL_dH || !dL_dpx)
            return fail(PARARNN_EINVAL, "preacts, H, dL_dH and dL_dpx must not be NULL");
        if (!aligned(preacts, esz) || !aligned(H, 4) || !aligned(dL_dH, 4) || !aligned(dL_dpx, 4) ||
            (diag_w && !aligned(diag_w, 4)) || (h0 && !aligned(h0, 4)) || (dL_dh0 && !aligned(dL_dh0, 4)))
            return fail(PARARNN_EINVAL, "pointer not aligned to its element size");
        if (!device_reachable(preacts) || !device_reachable(H) || !device_reachable(dL_dH) ||
            !device_reachable(dL_dpx) || !device_reachable(workspace) || (diag_w && !device_reachable(diag_w)) ||
            (h0 && !device_reachable(h0)) || (dL_dh0 && !device_reachable(dL_dh0)))
            return fail(PARARNN_EINVAL, "a pointer is not device-accessible memory");
    }
    if (dL_da && (!aligned(dL_da, 4) || !device_reachable(dL_da)))
        return fail(PARARNN_EINVAL, "dL_da is not device-accessible float memory");

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool vec = (D % 4 == 0) && aligned(preacts, 16) && aligned(H, 16) && aligned(dL_dH, 16) &&
                     aligned(dL_dpx, 16);
    const Plan pl = make_plan(cell, B, T, D, 1, false, vec);
    if (pl.nTiles >= (int64_t(1) << 31)) return fail(PARARNN_EINVAL, "too many tiles");

    char* ws = static_cast<char*>(workspace);
    cudaError_t e = cudaMemsetAsync(ws, 0, empty ? kHeaderBytes : pl.off_agg, s);
    if (e != cudaSuccess) return cuda_fail(e, "workspace reset");
    if (empty) {
        const int G = pararnn_num_gates(cell);
        if (dL_da && D > 0) {
            e = cudaMemsetAsync(dL_da, 0, sizeof(float) * G * D, s);
            if (e != cudaSuccess) return cuda_fail(e, "dL_da reset");
        }
        if (dL_dh0 && B > 0 && D > 0) {
            e = cudaMemsetAsync(dL_dh0, 0, sizeof(float) * B * pararnn_state_width(cell) * D, s);
            if (e != cudaSuccess) return cuda_fail(e, "dL_dh0 reset");
        }
        return PARARNN_OK;
    }

    BwdParams prm;
    memset(&prm, 0, sizeof prm);
    prm.px = preacts;
    prm.w = diag_w;
    prm.h0 = h0;
    prm.H = H;
    prm.dLdH = dL_dH;
    prm.dLdpx = dL_dpx;
    prm.dLdh0 = dL_dh0;
    prm.part = reinterpret_cast<float*>(ws + pl.off_part);
    prm.B = B;
    prm.T = T;
    prm.D = D;
    prm.lb.status = reinterpret_cast<unsigned*>(ws);
    prm.lb.flags = reinterpret_cast<unsigned*>(ws + pl.off_flags);
    prm.lb.agg = reinterpret_cast<float*>(ws + pl.off_agg);
    prm.lb.inc = reinterpret_cast<float*>(ws + pl.off_inc);
    prm.lb.nGroups = pl.nGroups;
    prm.lb.nSlots = 1;
    prm.lb.timeout_ns = kWaitLimitNs;

    const bool bf = px_dtype == PARARNN_BF16;
    if (cell == PARARNN_CELL_LINEAR) {
        if (vec) st = bf ? launch_bwd<CellLinear, __nv_bfloat16, BwdLinV>(pl, prm, dL_da, s) : launch_bwd<CellLinear, float, BwdLinV>(pl, prm, dL_da, s);
        else st = bf ? launch_bwd<CellLinear, __nv_bfloat16, BwdLinS>(pl, prm, dL_da, s) : launch_bwd<CellLinear, float, BwdLinS>(pl, prm, dL_da, s);
    } else if (cell == PARARNN_CELL_DIAG_GRU) {
        if (vec) st = bf ? launch_bwd<CellGRU, __nv_bfloat16, BwdGruV>(pl, prm, dL_da, s) : launch_bwd<CellGRU, float, BwdGruV>(pl, prm, dL_da, s);
        else st = bf ? launch_bwd<CellGRU, __nv_bfloat16, BwdGruS>(pl, prm, dL_da, s) : launch_bwd<CellGRU, float, BwdGruS>(pl, prm, dL_da, s);
    } else {
        if (vec) st = bf ? launch_bwd<CellLSTM, __nv_bfloat16, BwdLstmV>(pl, prm, dL_da, s) : launch_bwd<CellLSTM, float, BwdLstmV>(pl, prm, dL_da, s);
        else st = bf ? launch_bwd<CellLSTM, __nv_bfloat16, BwdLstmS>(pl, prm, dL_da, s) : launch_bwd<CellLSTM, float, BwdLstmS>(pl, prm, dL_da, s);
    }
    return st;
}

pararnn_status pararnn_status_sync(const void* workspace, void* stream) {
    if (!workspace) return fail(PARARNN_EINVAL, "workspace is NULL");
    unsigned word = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof word, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return cuda_fail(e, "status copy");
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    if (word & kStatusTimeout) return PARARNN_ETIMEOUT;
    if (word & kStatusNonFinite) return PARARNN_ENONFINITE;
    return PARARNN_OK;
}

const char* pararnn_status_string(pararnn_status status) {
    switch (status) {
        case PARARNN_OK: return "PARARNN_OK";
        case PARARNN_EINVAL: return "PARARNN_EINVAL";
        case PARARNN_ENONFINITE: return "PARARNN_ENONFINITE";
        case PARARNN_ETIMEOUT: return "PARARNN_ETIMEOUT";
        case PARARNN_ECUDA: return "PARARNN_ECUDA";
    }
    return "PARARNN_UNKNOWN";
}

const char* pararnn_last_error(void) { return g_last_error; }

pararnn_status pararnn_probe_wait_timeout(void* workspace, size_t ws_bytes, uint64_t timeout_ns, void* stream) {
    g_last_error[0] = 0;
    if (!workspace || !aligned(workspace, 16)) return fail(PARARNN_EINVAL, "workspace NULL or misaligned");
    if (ws_bytes < kHeaderBytes + 256) return fail(PARARNN_EINVAL, "workspace too small");
    if (timeout_ns == 0 || timeout_ns > 10000000000ull) return fail(PARARNN_EINVAL, "timeout outside (0, 10 s]");
    if (!device_reachable(workspace)) return fail(PARARNN_EINVAL, "workspace is not device-accessible memory");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    cudaError_t e = cudaMemsetAsync(ws, 0, kHeaderBytes + 256, s);
    if (e != cudaSuccess) return cuda_fail(e, "workspace reset");
    probe_wait_kernel<<<1, 32, 0, s>>>(reinterpret_cast<unsigned*>(ws),
                                         reinterpret_cast<const unsigned*>(ws + kHeaderBytes), timeout_ns);
    e = cudaGetLastError();
    return e == cudaSuccess ? PARARNN_OK : cuda_fail(e, "probe launch");
}

}  // extern "C"
